"""GPU parity of the backward pass: fa_fwd then fa_bwd through the C ABI,
against the fp64 oracle's analytic gradients on the same bf16 inputs.

Tolerance (the pages fix none for gradients; derived from the arithmetic):
each of dQ, dK, dV is compared as a whole tensor,
    max |G - G_ref| <= 2e-2 * max |G_ref|   and   rms(G - G_ref) <= 1e-2 * rms(G_ref).
The kernel rounds P and dS to bf16 (relative 2^-9 each) before the tensor-core
products, takes D_i from the bf16 forward output O (relative 2^-9), uses the
forward's LSE (absolute error <= 1e-3, a relative error <= 1e-3 on every P of
the row) and rounds the gradients to bf16 (2^-9).  Summed, these give a few
tenths of a percent of relative RMS error; the bound leaves a factor of about
two to three above that.  A dropped term, wrong sign or transposed operand
gives an error of the order of the gradient itself.  Where the exact gradient
is identically zero the bound is taken against a floor of 1e-3 instead.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

REL_MAX = 2e-2
REL_RMS = 1e-2
ZERO_FLOOR = 1e-3


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import exact_attention_122_b200 as m
    from exact_attention_122_b200 import build
    build.build()
    return m


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def gpu_grads(fa, q, k, v, do, causal, scale):
    qd, kd, vd, dod = (t.to("cuda:0") for t in (q, k, v, do))
    o, lse = fa.fa_fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = fa.fa_bwd(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, word = fa.device_status()
    assert st == fa.FA_OK, f"device status {fa.status_string(st)} {word:#x}"
    return dq, dk, dv


def check_grad(g, ref, what):
    G = f64(g)
    assert np.all(np.isfinite(G)), what
    d = np.abs(G - ref)
    # A gradient that is exactly zero (N = 1: the only key has weight 1, so
    # dS = 0) leaves fp32 rounding of D - dP; the floor makes the bound
    # absolute there (2e-5 on the maximum).
    ref_max = max(float(np.abs(ref).max()), ZERO_FLOOR)
    ref_rms = max(float(np.sqrt(np.mean(ref * ref))), ZERO_FLOOR)
    err_max = float(d.max())
    err_rms = float(np.sqrt(np.mean(d * d)))
    assert err_max <= REL_MAX * ref_max, f"{what}: max err {err_max} vs max|ref| {ref_max}"
    assert err_rms <= REL_RMS * ref_rms, f"{what}: rms err {err_rms} vs rms ref {ref_rms}"
    return err_max / ref_max, err_rms / ref_rms


def compare_all(fa, B, H, N, d, causal, seed, qk_std=1.0, scale=None):
    q, k, v = synth.draw_qkv(B, H, N, d, seed=seed, qk_std=qk_std)
    do = synth.draw_dout(B, H, N, d, seed=seed)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    dq, dk, dv = gpu_grads(fa, q, k, v, do, causal, scale)
    dQ, dK, dV, _ = oracle.attention_bwd_fp64(q, k, v, do, causal=causal, scale=scale)
    tag = f"B={B} H={H} N={N} d={d} causal={causal}"
    return (check_grad(dq, dQ, "dQ " + tag), check_grad(dk, dK, "dK " + tag),
            check_grad(dv, dV, "dV " + tag))


@pytest.mark.parametrize("index", [1, 2, 3])
def test_bwd_workloads_full(fa, index):
    w = synth.workload(index)
    compare_all(fa, w.B, w.H, w.N, w.d, w.causal, w.seed, w.qk_std)


RAGGED = [1, 17, 64, 127, 128, 129, 200, 255, 257, 333, 640, 1000]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", RAGGED)
def test_bwd_ragged(fa, N, d, causal):
    compare_all(fa, 1, 2, N, d, causal, seed=300 + N + d)


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_many_key_blocks(fa, d):
    compare_all(fa, 1, 3, 2048, d, True, seed=41)


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_peaked_scores(fa, d):
    # q, k with std 3: scaled scores with std 9, nearly one-hot rows.
    compare_all(fa, 1, 2, 768, d, True, seed=43, qk_std=3.0)


def test_bwd_nonstandard_scale(fa):
    compare_all(fa, 2, 2, 300, 64, False, seed=45, scale=0.37)


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_equal_scores_closed_forms(fa, d):
    """Q = 0: every score is 0 and P is uniform over the allowed keys, so
    dK = scale dS^T Q is exactly zero, and dV_j is the sum of dO_i / (number
    of keys row i sees) over the rows i that see key j -- closed forms,
    independent of the oracle.  dQ is compared with the oracle."""
    B, H, N = 1, 2, 640
    _, k, v = synth.draw_qkv(B, H, N, d, seed=91)
    q = torch.zeros_like(k)
    do = synth.draw_dout(B, H, N, d, seed=91)
    scale = 1 / math.sqrt(d)
    DO = do.double().numpy()
    for causal in (True, False):
        dq, dk, dv = gpu_grads(fa, q, k, v, do, causal, scale)
        assert float(dk.abs().max()) == 0.0, f"dK of Q = 0 must vanish (causal={causal})"
        if causal:
            w = DO / np.arange(1, N + 1, dtype=np.float64)[None, None, :, None]
            dv_ref = np.flip(np.cumsum(np.flip(w, axis=2), axis=2), axis=2)
        else:
            dv_ref = np.broadcast_to(DO.sum(axis=2, keepdims=True) / N, DO.shape)
        check_grad(dv, dv_ref, f"dV equal scores d={d} causal={causal}")
        dq_ref, _, _, _ = oracle.attention_bwd_fp64(q, k, v, do, causal=causal, scale=scale)
        check_grad(dq, dq_ref, f"dQ equal scores d={d} causal={causal}")


def test_bwd_causal_row0_and_sums(fa):
    """Properties of the exact gradients: causal query 0 has dQ = 0 (its only
    key has weight 1); the keys' dV sum to the queries' dO sum (every P row
    sums to 1)."""
    B, H, N, d = 1, 4, 1024, 128
    q, k, v = synth.draw_qkv(B, H, N, d, seed=47)
    do = synth.draw_dout(B, H, N, d, seed=47)
    dq, dk, dv = gpu_grads(fa, q, k, v, do, True, 1 / math.sqrt(d))
    # D_0 (a fp32 dot product) and dP_00 (a tensor-core sum) round differently,
    # so dS_00 is zero only up to fp32 rounding.
    assert float(dq[:, :, 0].abs().max()) <= 1e-3 * float(dq.abs().max())
    s_dv = dv.double().sum(dim=2).cpu()
    s_do = do.double().sum(dim=2)
    assert float((s_dv - s_do).abs().max()) <= 2e-2 * float(s_do.abs().max())


def test_bwd_dk_dv_deterministic(fa):
    B, H, N, d = 2, 4, 1536, 128
    q, k, v = synth.draw_qkv(B, H, N, d, seed=49)
    do = synth.draw_dout(B, H, N, d, seed=49)
    a = gpu_grads(fa, q, k, v, do, True, 1 / math.sqrt(d))
    b = gpu_grads(fa, q, k, v, do, True, 1 / math.sqrt(d))
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    # dQ sums partials with atomic adds: equal up to fp32 reassociation.
    assert float((a[0].float() - b[0].float()).abs().max()) <= 1e-2 * float(a[0].float().abs().max())


def test_bwd_writes_stay_in_bounds(fa):
    """Gradients pre-filled with NaN and followed by canaries."""
    B, H, N, d = 1, 3, 300, 128
    q, k, v = synth.draw_qkv(B, H, N, d, seed=51)
    do = synth.draw_dout(B, H, N, d, seed=51)
    qd, kd, vd, dod = (t.to("cuda:0") for t in (q, k, v, do))
    o, lse = fa.fa_fwd(qd, kd, vd, causal=True)
    n, pad = B * H * N * d, 4096
    bufs = []
    for _ in range(3):
        buf = torch.full((n + pad,), float("nan"), dtype=torch.bfloat16, device="cuda:0")
        buf[n:] = 7.0
        bufs.append(buf)
    dq, dk, dv = (b_[:n].view(B, H, N, d) for b_ in bufs)
    fa.fa_bwd(qd, kd, vd, o, lse, dod, causal=True, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    for g in (dq, dk, dv):
        assert bool(torch.isfinite(g).all())
    for b_ in bufs:
        assert bool((b_[n:] == 7.0).all())


def test_bwd_full_size_sampled_heads(fa):
    """The long causal workload (B=2, H=32, N=8192, d=128) in one launch; the
    oracle recomputes two whole heads (every row and key of them)."""
    w = synth.workload(4)
    q, k, v = synth.workload_qkv(w)
    do = synth.draw_dout(w.B, w.H, w.N, w.d, seed=w.seed)
    dq, dk, dv = gpu_grads(fa, q, k, v, do, w.causal, w.scale)
    for b, h in [(0, 0), (1, 31)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        dQ, dK, dV, _ = oracle.attention_bwd_fp64(q[sl], k[sl], v[sl], do[sl], causal=True,
                                                  scale=w.scale)
        check_grad(dq[sl], dQ, f"dQ head {b},{h}")
        check_grad(dk[sl], dK, f"dK head {b},{h}")
        check_grad(dv[sl], dV, f"dV head {b},{h}")


def test_bwd_argument_errors_on_device(fa):
    t = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16, device="cuda:0")
    lse = torch.zeros(1, 1, 64, dtype=torch.float32, device="cuda:0")
    ws = torch.empty(fa.bwd_workspace_bytes(1, 1, 64, 128), dtype=torch.uint8, device="cuda:0")
    p = t.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    args = [p, p, p, p, p, lse.data_ptr(), p, p, p, 1, 1, 64, 128, 0, 0.1, ws.data_ptr()]
    assert fa.fa_bwd_raw(*args, ws.numel() - 1, s) == fa.FA_ERR_INVALID_ARG
    bad = list(args); bad[4] = p + 2
    assert fa.fa_bwd_raw(*bad, ws.numel(), s) == fa.FA_ERR_MISALIGNED
    torch.cuda.synchronize()
    assert fa.device_status()[0] == fa.FA_OK


def test_bwd_watchdog_reports_timeout_and_context_survives(fa):
    """Host-chosen fault injection: CTA 0's producer never issues its first
    Q / dO block.  The waits on it end by the watchdog (200 ms), the status
    word reads FA_ERR_TIMEOUT, and the next call is correct."""
    B, H, N, d = 1, 2, 512, 128
    q, k, v = synth.draw_qkv(B, H, N, d, seed=71)
    do = synth.draw_dout(B, H, N, d, seed=71)
    qd, kd, vd, dod = (t.to("cuda:0") for t in (q, k, v, do))
    o, lse = fa.fa_fwd(qd, kd, vd, causal=True)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws = torch.empty(fa.bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda:0")
    s = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    assert fa.device_status()[0] == fa.FA_OK
    st = fa.fa_bwd_debug_raw(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(),
                             dod.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                             dv.data_ptr(), B, H, N, d, 1, 1 / math.sqrt(d), ws.data_ptr(),
                             ws.numel(), s, 200, 1)
    assert st == fa.FA_OK
    st, word = fa.device_status(s)
    assert st == fa.FA_ERR_TIMEOUT, (fa.status_string(st), hex(word))
    assert fa.device_status(s)[0] == fa.FA_OK                      # read-and-clear
    compare_all(fa, B, H, N, d, True, seed=71)                     # the context still works


@pytest.mark.parametrize("causal", [False, True])
def test_autograd_attention_matches_oracle(fa, causal):
    """exact_attention_122_b200.attention under torch.autograd: loss = sum(O * dO)
    gives dL/dq, dL/dk, dL/dv = the oracle's gradients for upstream dO."""
    B, H, N, d = 2, 2, 333, 64
    q, k, v = synth.draw_qkv(B, H, N, d, seed=73)
    do = synth.draw_dout(B, H, N, d, seed=73)
    qd, kd, vd = (t.to("cuda:0").requires_grad_(True) for t in (q, k, v))
    o = fa.attention(qd, kd, vd, causal=causal)
    (o.float() * do.to("cuda:0").float()).sum().backward()
    dQ, dK, dV, _ = oracle.attention_bwd_fp64(q, k, v, do, causal=causal, scale=1 / math.sqrt(d))
    check_grad(qd.grad, dQ, "autograd dQ")
    check_grad(kd.grad, dK, "autograd dK")
    check_grad(vd.grad, dV, "autograd dV")
    O_ref, _ = oracle.attention_fp64(q, k, v, causal=causal, scale=1 / math.sqrt(d))
    assert float(np.abs(o.detach().float().cpu().numpy() - O_ref).max()) <= 2e-2


def _bnhd(t):
    """A (B, H, N, d) view of a [B][N][H][d] tensor holding the same values."""
    return t.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)


@pytest.mark.parametrize("d,N,causal", [(64, 300, True), (128, 513, False), (128, 1024, True)])
def test_bwd_strided_views_match_contiguous(fa, d, N, causal):
    """BNHD views of every operand (inputs and outputs) give the same dK and
    dV bits as the contiguous call and dQ equal up to the order of its atomic
    fp32 additions; both match the oracle."""
    B, H = 2, 3
    q, k, v = synth.draw_qkv(B, H, N, d, seed=77 + N)
    do = synth.draw_dout(B, H, N, d, seed=77 + N)
    qd, kd, vd, dod = (t.to("cuda:0") for t in (q, k, v, do))
    o, lse = fa.fa_fwd(qd, kd, vd, causal=causal)
    dq0, dk0, dv0 = fa.fa_bwd(qd, kd, vd, o, lse, dod, causal=causal)
    qs, ks, vs, os_, dos = (_bnhd(t) for t in (qd, kd, vd, o, dod))
    outs = [_bnhd(torch.empty_like(qd)) for _ in range(3)]
    assert not qs.is_contiguous() and not outs[0].is_contiguous()
    dq1, dk1, dv1 = fa.fa_bwd(qs, ks, vs, os_, lse, dos, causal=causal, dq=outs[0], dk=outs[1],
                              dv=outs[2])
    torch.cuda.synchronize()
    assert torch.equal(dk1, dk0) and torch.equal(dv1, dv0)
    assert float((dq1.float() - dq0.float()).abs().max()) <= 1e-2 * float(dq0.float().abs().max())
    dQ, dK, dV, _ = oracle.attention_bwd_fp64(q, k, v, do, causal=causal, scale=1 / math.sqrt(d))
    check_grad(dq1, dQ, "strided dQ")
    check_grad(dk1, dK, "strided dK")
    check_grad(dv1, dV, "strided dV")
