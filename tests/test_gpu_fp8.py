"""GPU parity of the FP8 forward (fa_fwd_fp8) against the fp64 oracle.

The oracle is exact attention of the dequantized inputs (code * per-tensor
scale), so the only approximation the kernel adds is rounding P to E4M3
before the P V product (S is formed exactly from the codes; the row sum l
uses the unrounded fp32 P; O is divided by l + lc, lc the rounding error of
each 128-key tile's largest P).  The pages fix no FP8 tolerance; the bounds
below follow from that rounding.

Max error, per output element, derived for every P value (normal and
subnormal E4M3):
* The kernel's P is k * P_j, P_j = exp(S_j - max S) and k = 2^(max - m) in
  [1, 2^8] (the lazy reference m is at most 8 log2 units below the row max,
  so P never reaches E4M3's 448 and never saturates).
* Rounding to nearest E4M3 moves a value p >= 2^-6 by at most 2^-4 p (3
  mantissa bits), a subnormal p < 2^-6 by at most 2^-10 (half the 2^-9
  subnormal spacing), and never by more than p itself (values up to 2^-10
  round to 0 or to 2^-9): |e(p)| <= r(p) = min(p, max(2^-4 p, 2^-10)), and
  r(k P) / k <= min(P, max(2^-4 P, 2^-10)) =: r_j for every k >= 1.  As the
  row max has P = 1 and r <= 2^-4 there, sum_j P_j - sum_j r_j > 0.
* With b_j = p_j + e_j, E = sum_j e_j v_j, O = sum_j p_j v_j / l:
  O_gpu - O = (E - lc O) / (l + lc)
            = (sum_j e_j (v_j - O) + O sum_{j not a tile top} e_j) / (l + lc),
  so |O_gpu - O|_c <= (sum_j r_j |v_jc - O_c| + |O_c| sum_{j not top} r_j)
                      / (sum_j P_j - sum_j r_j),
  plus bf16 rounding of the output (at most 2^-8 relative: 8 significant
  bits) and fp32 accumulation (1e-5 of max |V|).  A dominant key contributes almost nothing (v_j ~ O),
  which is what the tile-top correction buys.
The RMS bound, rms(O - O_ref) <= 0.08 rms(O_ref), is the statistical check:
the RMS relative rounding error of E4M3 is a few percent and averages over a
row.  max |LSE - LSE_ref| <= 1e-3 as for the bf16 path (LSE never sees the
rounded P).  A dropped scale, a transposed operand or a wrong byte order
gives errors of the order of O itself and fails the RMS bound.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

TOL_LSE = 1e-3
REL_RMS = 0.08


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import exact_attention_122_b200 as m
    from exact_attention_122_b200 import build
    build.build()
    return m


def deq(x8, s):
    return oracle.e4m3_bits_to_f64(x8.numpy()) * s


def run(fa, q8, k8, v8, scales, causal, scale):
    o, lse = fa.fa_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), *scales, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, word = fa.device_status()
    assert st == fa.FA_OK, f"device status {fa.status_string(st)} {word:#x}"
    return o, lse


def max_err_bound(Q, K, V, O_ref, rows, causal, scale):
    """Per-element bound on |O_gpu - O_ref| for the given rows of one head
    (module docstring): Q, K, V float64 (N, d) dequantized; O_ref the
    oracle's rows.  The row weights come from the oracle's softmax of the
    scaled scores."""
    N = K.shape[0]
    S = scale * (Q[rows] @ K.T)
    if causal:
        S = np.where(np.arange(N)[None, :] <= np.asarray(rows)[:, None], S, -np.inf)
    Pn, _, Z = oracle.softmax_rows_fp64(S)
    P = Pn * Z[:, None]                                   # relative to the row max (max = 1)
    allowed = np.isfinite(S)
    r = np.where(allowed, np.minimum(P, np.maximum(2.0 ** -4 * P, 2.0 ** -10)), 0.0)
    # each 128-key tile's largest P (the kernel's normaliser correction)
    top = np.zeros_like(allowed)
    for t0 in range(0, N, 128):
        blk = np.where(allowed[:, t0:t0 + 128], P[:, t0:t0 + 128], -1.0)
        idx = np.argmax(blk, axis=1)
        ok = blk[np.arange(len(rows)), idx] >= 0
        top[np.arange(len(rows))[ok], t0 + idx[ok]] = True
    denom = P.sum(axis=1) - r.sum(axis=1)
    assert np.all(denom > 0)
    # sum_j r_j |v_jc - O_c|, a few rows at a time (bounded host memory)
    term1 = np.empty_like(O_ref)
    step = max(1, (1 << 22) // (N * V.shape[1]))
    for i0 in range(0, len(rows), step):
        i1 = min(len(rows), i0 + step)
        num = np.abs(V[None, :, :] - O_ref[i0:i1, None, :])
        term1[i0:i1] = np.einsum("ij,ijc->ic", r[i0:i1], num)
    term2 = np.abs(O_ref) * np.where(top, 0.0, r).sum(axis=1)[:, None]
    bound = (term1 + term2) / denom[:, None]
    vmax = float(np.abs(V).max())
    return bound + 2.0 ** -8 * (np.abs(O_ref) + bound) + 1e-5 * vmax


def check(o, lse, O_ref, L_ref, bound, what):
    O = o.float().cpu().numpy().astype(np.float64)
    L = lse.cpu().numpy().astype(np.float64)
    assert np.isfinite(O).all() and np.isfinite(L).all(), what
    d = np.abs(O - O_ref)
    err_rms = float(np.sqrt(np.mean(d * d)))
    ref_rms = float(np.sqrt(np.mean(O_ref * O_ref)))
    worst = float((d / bound).max())
    assert worst <= 1.0, f"{what}: max err / bound = {worst}"
    assert err_rms <= REL_RMS * ref_rms, f"{what}: rms err {err_rms} vs rms O {ref_rms}"
    assert float(np.abs(L - L_ref).max()) <= TOL_LSE, what


def compare(fa, B, H, N, causal, seed, qk_std=1.0, d=128):
    (q8, k8, v8), sc = synth.draw_qkv_fp8(B, H, N, d, seed=seed, qk_std=qk_std)
    scale = 1 / math.sqrt(d)
    o, lse = run(fa, q8, k8, v8, sc, causal, scale)
    Q, K, V = deq(q8, sc[0]), deq(k8, sc[1]), deq(v8, sc[2])
    O, L = oracle.attention_fp64(Q, K, V, causal=causal, scale=scale)
    bound = np.empty_like(O)
    rows = np.arange(N)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, 256):
                rr = rows[r0:r0 + 256]
                bound[b, h, rr] = max_err_bound(Q[b, h], K[b, h], V[b, h], O[b, h, rr], rr,
                                                causal, scale)
    check(o, lse, O, L, bound, f"B={B} H={H} N={N} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 17, 128, 129, 255, 256, 333, 1000, 2048])
def test_fp8_ragged(fa, N, causal):
    compare(fa, 1, 2, N, causal, seed=500 + N)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 256, 257, 1000, 2048])
def test_fp8_ragged_d64(fa, N, causal):
    compare(fa, 1, 2, N, causal, seed=600 + N, d=64)


def test_fp8_d64_workload_shapes(fa):
    # the BERT- and GPT-2-shaped workloads in FP8
    compare(fa, 8, 12, 512, False, seed=1222, d=64)
    compare(fa, 8, 12, 1024, True, seed=1223, d=64)


def test_fp8_batch_heads(fa):
    compare(fa, 2, 3, 1000, True, seed=61)


def test_fp8_peaked_scores(fa):
    compare(fa, 1, 2, 1024, True, seed=63, qk_std=3.0)


def test_fp8_full_size_sampled(fa):
    """The long causal shape (B=2, H=32, N=8192, d=128) in FP8, one launch; the
    oracle recomputes sampled rows of every fifth head."""
    w = synth.workload(4)
    (q8, k8, v8), sc = synth.draw_qkv_fp8(w.B, w.H, w.N, w.d, seed=w.seed)
    o, lse = run(fa, q8, k8, v8, sc, True, w.scale)
    Q, K, V = deq(q8, sc[0]), deq(k8, sc[1]), deq(v8, sc[2])
    rng = np.random.default_rng(7)
    Og = o.float().cpu().numpy().astype(np.float64)
    Lg = lse.cpu().numpy().astype(np.float64)
    errs, refs = [], []
    for b in range(w.B):
        for h in range(0, w.H, 5):
            rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, w.N - 1],
                                             rng.integers(0, w.N, 24)]))
            O, L = oracle.attention_rows_fp64(Q[b, h], K[b, h], V[b, h], rows, True, w.scale)
            d = np.abs(Og[b, h, rows] - O)
            bound = max_err_bound(Q[b, h], K[b, h], V[b, h], O, rows, True, w.scale)
            assert float((d / bound).max()) <= 1.0
            assert float(np.abs(Lg[b, h, rows] - L).max()) <= TOL_LSE
            errs.append(d.ravel())
            refs.append(O.ravel())
    e, r = np.concatenate(errs), np.concatenate(refs)
    assert float(np.sqrt(np.mean(e * e))) <= REL_RMS * float(np.sqrt(np.mean(r * r)))


@pytest.mark.parametrize("d", [64, 128])
def test_fp8_equal_scores_give_prefix_means(fa, d):
    """Q = 0 (E4M3 zero bytes): every score is 0 and every P is exactly 1 in
    E4M3, so O is the prefix mean (causal) or the mean of the decoded V, up to
    fp32 accumulation and the bf16 output (2^-8 relative), and LSE = ln(#keys)."""
    N = 900
    (_, k8, v8), sc = synth.draw_qkv_fp8(1, 2, N, d, seed=96)
    q8 = torch.zeros_like(k8)
    V = deq(v8, sc[2])
    vmax = float(np.abs(V).max())
    for causal in (True, False):
        o, lse = run(fa, q8, k8, v8, sc, causal, 1 / math.sqrt(d))
        O = o.float().cpu().numpy().astype(np.float64)
        L = lse.cpu().numpy().astype(np.float64)
        if causal:
            counts = np.arange(1, N + 1, dtype=np.float64)
            O_ref = np.cumsum(V, axis=2) / counts[None, None, :, None]
        else:
            counts = np.full(N, float(N))
            O_ref = np.broadcast_to(V.mean(axis=2, keepdims=True), V.shape)
        bound = 2.0 ** -8 * np.abs(O_ref) + 1e-5 * vmax
        assert float((np.abs(O - O_ref) / bound).max()) <= 1.0, f"d={d} causal={causal}"
        assert float(np.abs(L - np.log(counts)[None, None, :]).max()) <= TOL_LSE


def test_fp8_deterministic(fa):
    (q8, k8, v8), sc = synth.draw_qkv_fp8(1, 4, 1536, 128, seed=65)
    a = run(fa, q8, k8, v8, sc, True, 0.0883883)
    b = run(fa, q8, k8, v8, sc, True, 0.0883883)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_fp8_descales_fold_exactly(fa):
    """Doubling descale_v doubles O exactly (a power-of-two scale of bf16
    values), and moving a factor 2 from descale_q to descale_k changes no
    bit: the descales enter as exact power-of-two factors of products."""
    (q8, k8, v8), (sq, sk, sv) = synth.draw_qkv_fp8(1, 2, 512, 128, seed=67)
    o1, l1 = run(fa, q8, k8, v8, (sq, sk, sv), False, 0.0883883)
    o2, l2 = run(fa, q8, k8, v8, (sq, sk, 2 * sv), False, 0.0883883)
    o3, l3 = run(fa, q8, k8, v8, (2 * sq, sk / 2, sv), False, 0.0883883)
    assert torch.equal(o2.float(), 2 * o1.float()) and torch.equal(l1, l2)
    assert torch.equal(o3, o1) and torch.equal(l3, l1)


def test_fp8_argument_errors_on_device(fa):
    t = torch.zeros(1, 1, 64, 128, dtype=torch.uint8, device="cuda:0")
    o = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16, device="cuda:0")
    lse = torch.zeros(1, 1, 64, dtype=torch.float32, device="cuda:0")
    ws = torch.empty(fa.fp8_workspace_bytes(1, 1, 64, 128), dtype=torch.uint8, device="cuda:0")
    p = t.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    args = [p, p, p, o.data_ptr(), lse.data_ptr(), 1, 1, 64, 128, 0, 0.1, 1.0, 1.0, 1.0,
            ws.data_ptr()]
    assert fa.fa_fwd_fp8_raw(*args, ws.numel() - 1, s) == fa.FA_ERR_INVALID_ARG
    bad = list(args); bad[1] = p + 8
    assert fa.fa_fwd_fp8_raw(*bad, ws.numel(), s) == fa.FA_ERR_MISALIGNED
    bad = list(args); bad[8] = 96
    assert fa.fa_fwd_fp8_raw(*bad, ws.numel(), s) == fa.FA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert fa.device_status()[0] == fa.FA_OK
