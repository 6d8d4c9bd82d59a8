"""GPU parity of the FP8 forward (fa_fwd_fp8) against the fp64 oracle.

The oracle is exact attention of the dequantized inputs (code * per-tensor
scale), so the only approximation the kernel adds is rounding P to E4M3
before the P V product (S is formed exactly from the codes; the row sum uses
the unrounded fp32 P).  Tolerances (the pages fix none for FP8; derived from
that rounding):

* max |O - O_ref| <= 2^-4 * max |V|: E4M3 keeps 3 mantissa bits, so a P value
  in the normal range moves by at most 2^-4 of itself, and
  |sum_j dP_j v_j| / l <= 2^-4 * max |V| * sum_j P_j / l = 2^-4 * max |V|.
* rms(O - O_ref) <= 0.08 * rms(O_ref): the RMS relative rounding error of
  E4M3 is about 2^-3 / sqrt(12) ~ 0.036 of a value's binade step (~0.028
  relative on average); with random V the error of a row relative to its
  output is of that order, and the bound leaves a factor of about three.
* max |LSE - LSE_ref| <= 1e-3, as for the bf16 path (LSE never sees the
  rounded P).
A dropped scale, a transposed operand or a wrong byte order gives errors of
the order of O itself and fails the RMS bound.
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


def check(o, lse, O_ref, L_ref, vmax, what):
    O = o.float().cpu().numpy().astype(np.float64)
    L = lse.cpu().numpy().astype(np.float64)
    assert np.isfinite(O).all() and np.isfinite(L).all(), what
    d = np.abs(O - O_ref)
    err_max, err_rms = float(d.max()), float(np.sqrt(np.mean(d * d)))
    ref_rms = float(np.sqrt(np.mean(O_ref * O_ref)))
    assert err_max <= 2.0 ** -4 * vmax, f"{what}: max err {err_max} > 2^-4 * {vmax}"
    assert err_rms <= REL_RMS * ref_rms, f"{what}: rms err {err_rms} vs rms O {ref_rms}"
    assert float(np.abs(L - L_ref).max()) <= TOL_LSE, what


def compare(fa, B, H, N, causal, seed, qk_std=1.0, d=128):
    (q8, k8, v8), sc = synth.draw_qkv_fp8(B, H, N, d, seed=seed, qk_std=qk_std)
    scale = 1 / math.sqrt(d)
    o, lse = run(fa, q8, k8, v8, sc, causal, scale)
    V = deq(v8, sc[2])
    O, L = oracle.attention_fp64(deq(q8, sc[0]), deq(k8, sc[1]), V, causal=causal, scale=scale)
    check(o, lse, O, L, float(np.abs(V).max()), f"B={B} H={H} N={N} causal={causal}")


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
    vmax = float(np.abs(V).max())
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
            assert float(d.max()) <= 2.0 ** -4 * vmax
            assert float(np.abs(Lg[b, h, rows] - L).max()) <= TOL_LSE
            errs.append(d.ravel())
            refs.append(O.ravel())
    e, r = np.concatenate(errs), np.concatenate(refs)
    assert float(np.sqrt(np.mean(e * e))) <= REL_RMS * float(np.sqrt(np.mean(r * r)))


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
