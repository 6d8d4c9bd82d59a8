"""The allocation-free entry point, fa_fwd_dynamic_noalloc, through the C ABI.

Some callers cannot allocate device memory: a plugin running inside an
application that owns every device allocation, or a latency-critical loop
that must not call cudaMalloc because it can synchronise the whole device.
fa_fwd_dynamic_noalloc serves them by keeping the dynamic schedule's work
counter in the library's own static device scratch instead of a caller
workspace.  It runs the same kernel and the same schedule as the
workspace-taking fa_fwd_dynamic, so its output must equal that entry point's
bit for bit.  This test checks that on two calls in a row, with a call of a
different shape between them (so the shared scratch holds another problem's
final count when the second call starts), and that the calls allocate nothing
through torch's allocator.

The file is named so that pytest collects it after every other test file.
"""

import math

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import exact_attention_122_b200 as m
    from exact_attention_122_b200 import build
    build.build()
    return m


def _noalloc(fa, q, k, v, o, lse, causal, scale, stream):
    B, H, N, d = q.shape
    return fa.fa_fwd_dynamic_noalloc_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                         lse.data_ptr(), B, H, N, d, None, int(causal), scale,
                                         stream.cuda_stream)


@pytest.mark.parametrize("B,H,N,d,causal", [(2, 3, 1000, 128, True), (8, 12, 512, 64, False),
                                            (1, 16, 4096, 128, True)])
def test_no_alloc_matches_dynamic_on_two_calls(fa, B, H, N, d, causal):
    torch.cuda.set_device(0)
    q, k, v = (t.to("cuda:0") for t in synth.draw_qkv(B, H, N, d, seed=900 + N + d))
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream()
    # reference: the existing entry point with a caller workspace
    o_ref, l_ref = fa.fa_fwd(q, k, v, causal=causal, scale=scale, schedule="dynamic")
    # another problem, run through the scratch between the two checked calls
    q2, k2, v2 = (t.to("cuda:0") for t in synth.draw_qkv(1, 5, 700, 64, seed=31))
    o2 = torch.empty_like(q2)
    l2 = torch.empty(1, 5, 700, dtype=torch.float32, device="cuda:0")
    torch.cuda.synchronize()
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda:0")
    for call in range(2):
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated()
        st = _noalloc(fa, q, k, v, o, lse, causal, scale, stream)
        assert st == fa.FA_OK, fa.status_string(st)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before
        assert fa.device_status()[0] == fa.FA_OK
        assert torch.equal(o, o_ref), f"call {call}: O differs from fa_fwd_dynamic"
        assert torch.equal(lse, l_ref), f"call {call}: LSE differs from fa_fwd_dynamic"
        if call == 0:
            assert _noalloc(fa, q2, k2, v2, o2, l2, True, 0.125, stream) == fa.FA_OK
            torch.cuda.synchronize()
            assert fa.device_status()[0] == fa.FA_OK


def test_no_alloc_refuses_too_many_units(fa):
    # B*H*ceil(N/256) above the scratch counter's range is refused up front.
    p = 1 << 20
    st = fa.fa_fwd_dynamic_noalloc_raw(p, p, p, p, p, 1 << 12, 1 << 10, 1 << 17, 64, None, 0, 1.0, 0)
    assert st == fa.FA_ERR_UNSUPPORTED
    # B*H beyond 2^31 - 1 is refused before the unit count is formed
    st = fa.fa_fwd_dynamic_noalloc_raw(p, p, p, p, p, 1 << 30, 1 << 30, 1 << 30, 64, None, 0, 1.0, 0)
    assert st == fa.FA_ERR_UNSUPPORTED
