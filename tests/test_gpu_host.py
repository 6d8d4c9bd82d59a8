"""GPU tests of fa_fwd_host: the forward on host-resident tensors, with the
transfers of chunks of heads overlapped with the attention.

The chunks run the same tiled kernel as fa_fwd, and a row's arithmetic does not
depend on which CTA or launch computes it, so O and LSE must equal fa_fwd's bit
for bit; small cases are also compared with the fp64 oracle under the forward
tolerances (max |dO| <= 2e-2, RMS <= 2e-3, max |dLSE| <= 1e-3).
"""

import math

import numpy as np
import pytest
import torch

import oracle
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


def _device_result(fa, q, k, v, causal, scale):
    o, lse = fa.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _check_oracle(o, lse, q, k, v, causal, scale):
    O, L = oracle.attention_fp64(q, k, v, causal=causal, scale=scale)
    e = np.abs(o.float().numpy().astype(np.float64) - O)
    assert e.max() <= 2e-2 and math.sqrt(float(np.mean(e * e))) <= 2e-3, e.max()
    assert np.abs(lse.numpy().astype(np.float64) - L).max() <= 1e-3


# (B, H, N, d, causal): one head per chunk; 34 heads in chunks of 3 with a
# one-head last chunk; a ragged length; a single head (one chunk, no overlap).
CASES = [(1, 3, 300, 128, True), (2, 17, 200, 64, False), (3, 5, 129, 128, True),
         (1, 1, 1, 64, False), (1, 1, 700, 128, False)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dN%dd%d%s" % (*c[:4], "c" if c[4] else ""))
@pytest.mark.parametrize("pinned", [True, False], ids=["pinned", "pageable"])
def test_host_matches_oracle_and_device_path(fa, case, pinned):
    B, H, N, d, causal = case
    q, k, v = synth.draw_qkv(B, H, N, d, seed=3100 + N + H)
    scale = 1.0 / math.sqrt(d)
    hq, hk, hv = (t.pin_memory() if pinned else t.clone() for t in (q, k, v))
    out = lse = None
    if not pinned:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16)
        lse = torch.empty((B, H, N), dtype=torch.float32)
    o, l = fa.fa_fwd_host(hq, hk, hv, causal=causal, scale=scale, out=out, lse=lse)
    torch.cuda.synchronize()
    st, word = fa.device_status()
    assert st == fa.FA_OK, (fa.status_string(st), hex(word))
    od, ld = _device_result(fa, q, k, v, causal, scale)
    assert torch.equal(o, od) and torch.equal(l, ld)
    _check_oracle(o, l, q, k, v, causal, scale)


def test_calls_sharing_a_workspace_on_one_stream(fa):
    """Two calls on one stream and one workspace, synchronised once: the
    second may only overwrite the slots after the first's copies back."""
    B, H, N, d = 2, 9, 257, 128
    a = synth.draw_qkv(B, H, N, d, seed=3201)
    b = synth.draw_qkv(B, H, N, d, seed=3202)
    ws = torch.empty(fa.host_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda:0")
    s = torch.cuda.Stream()
    ha = [t.pin_memory() for t in a]
    hb = [t.pin_memory() for t in b]
    oa, la = fa.fa_fwd_host(*ha, causal=True, workspace=ws, stream=s)
    ob, lb = fa.fa_fwd_host(*hb, causal=False, workspace=ws, stream=s)
    s.synchronize()
    for (o, l), x, causal in (((oa, la), a, True), ((ob, lb), b, False)):
        od, ld = _device_result(fa, *x, causal, 1 / math.sqrt(d))
        assert torch.equal(o, od) and torch.equal(l, ld)


def test_host_full_size_long_context_causal(fa):
    """B=2, H=32, N=8192, d=128, causal (16 chunks of 4 heads): bit-identical
    to the device-resident forward, plus sampled rows against the oracle."""
    w = synth.workload("long_context_causal")
    q, k, v = synth.workload_qkv(w)
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    o, l = fa.fa_fwd_host(hq, hk, hv, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    od, ld = _device_result(fa, q, k, v, w.causal, w.scale)
    assert torch.equal(o, od) and torch.equal(l, ld)
    rows = np.array([0, 1, 4095, 8191])
    for b, h in ((0, 0), (1, 31)):
        qb, kb, vb = (oracle.exact_attention._as_f64(t[b, h]) for t in (q, k, v))
        O, L = oracle.attention_rows_fp64(qb, kb, vb, rows, causal=w.causal, scale=w.scale)
        assert np.abs(o[b, h, rows].float().numpy() - O).max() <= 2e-2
        assert np.abs(l[b, h, rows].numpy() - L).max() <= 1e-3


def test_python_wrapper_rejects_device_tensors(fa):
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16, device="cuda:0")
    with pytest.raises(ValueError):
        fa.fa_fwd_host(q, q, q)
