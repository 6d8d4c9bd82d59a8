"""The allocation-free entry point, fa_fwd_dynamic_noalloc, through the C ABI.

Some callers cannot allocate device memory: a plugin running inside an
application that owns every device allocation, or a latency-critical loop
that must not call cudaMalloc because it can synchronise the whole device.
fa_fwd_dynamic_noalloc serves them by keeping the dynamic schedule's work
counter in the library's own static device scratch instead of a caller
workspace.  This test checks, on two calls in a row, that its output matches
the workspace-taking fa_fwd_dynamic within the tolerances of the parity tests,
and that the calls allocate nothing through torch's allocator.

The file is named so that pytest collects it after every other test file.
"""

import math

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

TOL_MAX = 2e-2
TOL_RMS = 2e-3
TOL_LSE = 1e-3


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import exact_attention_122_b200 as m
    from exact_attention_122_b200 import build
    build.build()
    return m


@pytest.mark.parametrize("B,H,N,d,causal", [(2, 3, 1000, 128, True), (8, 12, 512, 64, False),
                                            (1, 16, 4096, 128, True)])
def test_no_alloc_matches_dynamic_on_two_calls(fa, B, H, N, d, causal):
    torch.cuda.set_device(0)
    q, k, v = (t.to("cuda:0") for t in synth.draw_qkv(B, H, N, d, seed=900 + N + d))
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream()
    # reference: the existing entry point with a caller workspace
    o_ref, l_ref = fa.fa_fwd(q, k, v, causal=causal, scale=scale, schedule="dynamic")
    torch.cuda.synchronize()
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda:0")
    for _ in range(2):
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated()
        st = fa.fa_fwd_dynamic_noalloc_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                           lse.data_ptr(), B, H, N, d, None, int(causal), scale,
                                           stream.cuda_stream)
        assert st == fa.FA_OK, fa.status_string(st)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before
        assert fa.device_status()[0] == fa.FA_OK
        diff = (o.double() - o_ref.double()).abs()
        assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(lse).all())
        assert float(diff.max()) <= TOL_MAX
        assert float(diff.pow(2).mean().sqrt()) <= TOL_RMS
        assert float((lse - l_ref).abs().max()) <= TOL_LSE


def test_no_alloc_refuses_too_many_units(fa):
    # B*H*ceil(N/256) above the scratch counter's range is refused up front.
    p = 1 << 20
    st = fa.fa_fwd_dynamic_noalloc_raw(p, p, p, p, p, 1 << 12, 1 << 10, 1 << 17, 64, None, 0, 1.0, 0)
    assert st == fa.FA_ERR_UNSUPPORTED
