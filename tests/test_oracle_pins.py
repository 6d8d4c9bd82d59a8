"""Pins for the fp64 oracle: checks against what the pages and mathematics fix.

Each pin compares the oracle with something other than itself: values the page
"Flash attention optimization" prints for its worked example and exercise
(fixtures under tests/golden/), closed forms, invariants, brute force of the
tiled recurrence on tiny inputs, and an independent library routine (torch's
float64 CPU scaled-dot-product attention and scipy's logsumexp).  The mutation
tests at the end plant plausible mistakes in the oracle and check that at
least one pin fails for each.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import oracle.exact_attention as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _row_problem(scores, values):
    """Embed a one-row problem as (1,1,n,1) attention with scale = 1.

    q = [1], k_j = [s_j], v_j = [v_j] gives the score row s exactly
    (scores on the page are already scaled)."""
    s = np.asarray(scores, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    n = s.shape[0]
    q = np.zeros((1, 1, n, 1))
    q[0, 0, :, 0] = 1.0
    k = s.reshape(1, 1, n, 1).copy()
    vv = v.reshape(1, 1, n, 1).copy()
    return q, k, vv


# ---------------------------------------------------------------------------
# Pins (each raises AssertionError when the oracle disagrees)
# ---------------------------------------------------------------------------

def pin_worked_example_direct():
    g = _load("online_softmax_worked_example.json")
    q, k, v = _row_problem(g["scores"], g["values"])
    O, LSE = oracle.attention_fp64(q, k, v, causal=False, scale=1.0)
    # Row n-1 (query = 1) sees every key with score s_j.
    o = O[0, 0, -1, 0]
    tol = 0.5 * 10.0 ** (-g["printed_decimals"])
    assert abs(o - g["direct"]["O"]) <= tol, o
    # The page's NumPy listing prints 36.880565891447...
    assert abs(o - float(g["listing_output_prefix"])) < 1e-12, repr(o)
    S = np.asarray(g["scores"])[None, :]
    P, M, Z = oracle.softmax_rows_fp64(S)
    assert np.allclose(P[0], g["direct"]["weights"], atol=0.5e-5)
    # The page's sum is the sum of its four 5-decimal rounded terms, so it
    # carries up to 4 x 0.5e-5 of rounding (exact value 1.2034380).
    assert abs(Z[0] - g["direct"]["sum"]) <= 4 * 0.5e-5
    assert np.allclose(np.exp(S[0] - M[0]), g["direct"]["exp_shifted"], atol=0.5e-5)
    # LSE = max + ln(sum): 5 + ln(1.20345), within the page sum's rounding.
    assert abs(LSE[0, 0, -1] - (5.0 + math.log(g["direct"]["sum"]))) <= 4 * 0.5e-5 / 1.2


def pin_worked_example_tiled():
    g = _load("online_softmax_worked_example.json")
    O, m, l, trace = oracle.online_softmax_row_blockmax(g["scores"], g["values"], g["block_size"])
    b1 = g["tiled"]["block1"]
    m1, l1, acc1 = trace[0]
    assert m1 == b1["m"]
    assert abs(l1 - b1["l"]) <= 0.5e-5 and abs(float(acc1) - b1["acc"]) <= 0.5e-4
    mg = g["tiled"]["merged"]
    # The page merges rounded intermediates (acc1 to 4 decimals, scale_old to
    # 5, acc2 to 4), so its merged figures carry their propagated rounding:
    # |d acc| <= acc1 * 0.5e-5 + scale_old * 0.5e-4 + 0.5e-4 + 0.5e-4.
    sc_old = g["tiled"]["block2"]["scale_old"]
    tol_acc = b1["acc"] * 0.5e-5 + sc_old * 0.5e-4 + 2 * 0.5e-4
    assert abs(l - mg["l"]) <= 4 * 0.5e-5 and abs(float(trace[1][2]) - mg["acc"]) <= tol_acc
    assert abs(float(O) - mg["O"]) <= 0.5e-4
    O2, m2, l2 = oracle.online_softmax_row_runningmax(g["scores"], g["values"], g["block_size"])
    assert abs(float(O2) - mg["O"]) <= 0.5e-4 and m2 == g["tiled"]["block2"]["m_new"]


def pin_exercise1():
    g = _load("online_softmax_exercise1.json")
    O, m, l, trace = oracle.online_softmax_row_blockmax(g["scores"], g["values"], g["block_size"])
    assert trace[0][0] == g["block1"]["m"]
    assert abs(trace[0][1] - g["block1"]["l"]) <= 0.5e-4
    assert abs(float(trace[0][2]) - g["block1"]["acc"]) <= 0.5e-4
    # Second block: the running max does not grow, so the old total is not rescaled.
    assert trace[1][0] == g["block2"]["m_new"]
    assert math.exp(trace[0][0] - trace[1][0]) == g["block2"]["scale_old"]
    # The answer merges 4-decimal intermediates (l1, l_block, scale_new), so
    # its merged l carries their propagated rounding plus its own:
    # 0.5e-4 + 0.5e-4 * scale_new + l_block * 0.5e-4 + 0.5e-4.
    sn, lb = g["block2"]["scale_new"], g["block2"]["l_block"]
    tol_l = 0.5e-4 + 0.5e-4 * sn + lb * 0.5e-4 + 0.5e-4
    assert abs(l - g["merged"]["l"]) <= tol_l
    tol_acc = 0.5e-4 + 0.5e-4 * sn + g["block2"]["acc_block"] * 0.5e-4 + 0.5e-4
    assert abs(float(trace[1][2]) - g["merged"]["acc"]) <= tol_acc
    assert abs(float(O) - g["merged"]["O"]) <= 0.5e-3
    q, k, v = _row_problem(g["scores"], g["values"])
    Od, _ = oracle.attention_fp64(q, k, v, causal=False, scale=1.0)
    assert abs(Od[0, 0, -1, 0] - g["merged"]["O"]) <= 0.5e-3


def pin_brute_force_tiling(seed=7):
    """Blocked recurrences (both forms) equal the direct result to 1e-12."""
    rng = np.random.default_rng(seed)
    for n in (1, 2, 3, 5, 8, 13, 31, 64):
        d = int(rng.integers(1, 9))
        q = rng.standard_normal((1, 1, n, d))
        k = rng.standard_normal((1, 1, n, d))
        v = rng.standard_normal((1, 1, n, d))
        scale = 1.0 / math.sqrt(d)
        for causal in (False, True):
            O, LSE = oracle.attention_fp64(q, k, v, causal=causal, scale=scale)
            for blk in range(1, n + 1):
                Ot, Lt = oracle.tiled_attention_fp64(q[0, 0], k[0, 0], v[0, 0], causal, scale,
                                                     block_q=max(1, blk // 2 + 1), block_k=blk)
                assert np.max(np.abs(Ot - O[0, 0])) <= 1e-12
                assert np.max(np.abs(Lt - LSE[0, 0])) <= 1e-12
            i = n - 1                      # last row sees every key in both modes
            s = scale * (q[0, 0, i] @ k[0, 0].T)
            for blk in range(1, n + 1):
                Ob, mb, lb, _ = oracle.online_softmax_row_blockmax(s, v[0, 0], blk)
                Or, mr, lr = oracle.online_softmax_row_runningmax(s, v[0, 0], blk)
                assert np.max(np.abs(Ob - O[0, 0, i])) <= 1e-12
                assert np.max(np.abs(Or - O[0, 0, i])) <= 1e-12
                assert abs(mb + math.log(lb) - LSE[0, 0, i]) <= 1e-12


def pin_invariants(seed=11):
    """P rows sum to 1, P >= 0, masked weights exactly 0; O rows are convex
    combinations of the allowed V rows; causal row 0 returns v_0."""
    rng = np.random.default_rng(seed)
    B, H, N, d = 2, 3, 37, 16
    q = rng.standard_normal((B, H, N, d)) * 2
    k = rng.standard_normal((B, H, N, d)) * 2
    v = rng.standard_normal((B, H, N, d))
    scale = 1 / math.sqrt(d)
    for causal in (False, True):
        O, LSE = oracle.attention_fp64(q, k, v, causal=causal, scale=scale, row_chunk=8)
        for b in range(B):
            for h in range(H):
                S = scale * (q[b, h] @ k[b, h].T)
                if causal:
                    S = np.where(np.tril(np.ones((N, N), bool)), S, -np.inf)
                P, M, Z = oracle.softmax_rows_fp64(S)
                assert np.all(P >= 0)
                assert np.max(np.abs(P.sum(axis=1) - 1)) <= 1e-12
                if causal:
                    assert np.all(P[np.triu(np.ones((N, N), bool), 1)] == 0.0)
                for i in range(N):
                    allowed = v[b, h, : i + 1] if causal else v[b, h]
                    assert np.all(O[b, h, i] >= allowed.min(axis=0) - 1e-12)
                    assert np.all(O[b, h, i] <= allowed.max(axis=0) + 1e-12)
                    # LSE is at least the row max and at most max + ln(#allowed)
                    srow = S[i][np.isfinite(S[i])]
                    assert srow.max() - 1e-12 <= LSE[b, h, i] <= srow.max() + math.log(len(srow)) + 1e-12
                if causal:
                    assert np.array_equal(O[b, h, 0], v[b, h, 0])
                    assert abs(LSE[b, h, 0] - scale * float(q[b, h, 0] @ k[b, h, 0])) <= 1e-12


def pin_closed_forms(seed=13):
    """Equal scores -> mean of the allowed V rows, LSE = ln(#allowed) + s;
    one dominant key -> O = v of that key (weight of the rest below e^-200)."""
    rng = np.random.default_rng(seed)
    N, d = 24, 8
    v = rng.standard_normal((1, 1, N, d))
    q = np.zeros((1, 1, N, d))
    k = rng.standard_normal((1, 1, N, d))
    for causal in (False, True):
        O, LSE = oracle.attention_fp64(q, k, v, causal=causal, scale=0.3)
        for i in range(N):
            cnt = i + 1 if causal else N
            assert np.max(np.abs(O[0, 0, i] - v[0, 0, :cnt].mean(axis=0))) <= 1e-12
            assert abs(LSE[0, 0, i] - math.log(cnt)) <= 1e-12
    # dominant key: k_5 aligned with every q, others orthogonal
    q = np.zeros((1, 1, N, d)); q[..., 0] = 1.0
    k = np.zeros((1, 1, N, d)); k[0, 0, 5, 0] = 400.0
    O, LSE = oracle.attention_fp64(q, k, v, causal=False, scale=1.0)
    assert np.max(np.abs(O[0, 0] - v[0, 0, 5])) <= 1e-12
    assert np.max(np.abs(LSE[0, 0] - 400.0)) <= 1e-12


def pin_scale_handling(seed=17):
    """scale = 1/sqrt(d) on q*sqrt(d) equals scale = 1 on q (the worked
    example's "already sqrt(d)-scaled" scores); default scale is 1/sqrt(d)."""
    rng = np.random.default_rng(seed)
    d = 16
    q = rng.standard_normal((1, 2, 20, d))
    k = rng.standard_normal((1, 2, 20, d))
    v = rng.standard_normal((1, 2, 20, d))
    O1, L1 = oracle.attention_fp64(q, k, v, causal=True, scale=1.0)
    O2, L2 = oracle.attention_fp64(q * 4.0, k, v, causal=True, scale=0.25)
    O3, L3 = oracle.attention_fp64(q * 4.0, k, v, causal=True)
    assert np.max(np.abs(O1 - O2)) <= 1e-12 and np.max(np.abs(L1 - L2)) <= 1e-12
    assert np.max(np.abs(O1 - O3)) <= 1e-12 and np.max(np.abs(L1 - L3)) <= 1e-12


def pin_library_routine(seed=19):
    """Independent implementation: torch's CPU float64 SDPA (math path) for O
    and scipy's logsumexp over the scaled, masked scores for LSE."""
    rng = np.random.default_rng(seed)
    for (B, H, N, d) in ((1, 1, 7, 4), (2, 3, 45, 16), (1, 2, 130, 64)):
        q = rng.standard_normal((B, H, N, d)) * 3
        k = rng.standard_normal((B, H, N, d)) * 3
        v = rng.standard_normal((B, H, N, d))
        scale = 1 / math.sqrt(d)
        for causal in (False, True):
            O, LSE = oracle.attention_fp64(q, k, v, causal=causal, scale=scale, row_chunk=16)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
                is_causal=causal, scale=scale).numpy()
            assert np.max(np.abs(O - ref)) <= 1e-12
            S = scale * np.einsum("bhid,bhjd->bhij", q, k)
            if causal:
                S = np.where(np.tril(np.ones((N, N), bool)), S, -np.inf)
            assert np.max(np.abs(LSE - scipy.special.logsumexp(S, axis=-1))) <= 1e-12


def pin_decode_library(seed=23):
    """N_q < N_k (queries = the last N_q positions): torch float64 SDPA with an
    explicit lower-right boolean mask, and scipy logsumexp for LSE."""
    rng = np.random.default_rng(seed)
    for (Nq, Nk, d) in ((1, 37, 8), (5, 64, 16), (16, 300, 32)):
        q = rng.standard_normal((2, 3, Nq, d)) * 2
        k = rng.standard_normal((2, 3, Nk, d)) * 2
        v = rng.standard_normal((2, 3, Nk, d))
        scale = 1 / math.sqrt(d)
        mask = np.tril(np.ones((Nq, Nk), bool), k=Nk - Nq)
        for causal in (False, True):
            O, LSE = oracle.attention_fp64(q, k, v, causal=causal, scale=scale)
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
                attn_mask=torch.from_numpy(mask) if causal else None, scale=scale).numpy()
            assert np.max(np.abs(O - ref)) <= 1e-12
            S = scale * np.einsum("bhid,bhjd->bhij", q, k)
            if causal:
                S = np.where(mask, S, -np.inf)
            assert np.max(np.abs(LSE - scipy.special.logsumexp(S, axis=-1))) <= 1e-12


def pin_decode_closed_form(seed=29):
    """Equal scores with N_q < N_k: query i sees keys 0..i+N_k-N_q, so O_i is
    their mean and LSE_i = ln(i + N_k - N_q + 1)."""
    rng = np.random.default_rng(seed)
    Nq, Nk, d = 4, 19, 8
    q = np.zeros((1, 1, Nq, d))
    k = rng.standard_normal((1, 1, Nk, d))
    v = rng.standard_normal((1, 1, Nk, d))
    O, LSE = oracle.attention_fp64(q, k, v, causal=True, scale=0.5)
    for i in range(Nq):
        cnt = i + Nk - Nq + 1
        assert np.max(np.abs(O[0, 0, i] - v[0, 0, :cnt].mean(axis=0))) <= 1e-12
        assert abs(LSE[0, 0, i] - math.log(cnt)) <= 1e-12


def pin_decode_brute_force(seed=31):
    """Tiny N_q < N_k case written out with scalar loops."""
    rng = np.random.default_rng(seed)
    Nq, Nk, d = 3, 7, 2
    q = rng.standard_normal((1, 1, Nq, d))
    k = rng.standard_normal((1, 1, Nk, d))
    v = rng.standard_normal((1, 1, Nk, d))
    scale = 0.7
    O, LSE = oracle.attention_fp64(q, k, v, causal=True, scale=scale)
    for i in range(Nq):
        keys = [j for j in range(Nk) if j <= i + (Nk - Nq)]
        sc = [scale * sum(q[0, 0, i, t] * k[0, 0, j, t] for t in range(d)) for j in keys]
        mx = max(sc)
        w = [math.exp(x - mx) for x in sc]
        z = sum(w)
        for t in range(d):
            o = sum(wj * v[0, 0, j, t] for wj, j in zip(w, keys)) / z
            assert abs(O[0, 0, i, t] - o) <= 1e-12
        assert abs(LSE[0, 0, i] - (mx + math.log(z))) <= 1e-12


PINS = [pin_worked_example_direct, pin_worked_example_tiled, pin_exercise1,
        pin_brute_force_tiling, pin_invariants, pin_closed_forms, pin_scale_handling,
        pin_library_routine, pin_decode_library, pin_decode_closed_form, pin_decode_brute_force]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


def test_bf16_conversion_exact():
    """bf16 bit patterns -> float64 agrees with torch's own widening cast."""
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 1 << 16, size=200_000, dtype=np.uint32).astype(np.uint16)
    exp_field = (bits >> 7) & 0xFF
    bits = bits[exp_field != 0xFF]                       # skip NaN/Inf patterns
    ours = oracle.bf16_bits_to_f64(bits)
    t = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, t)


def test_rows_match_full():
    """attention_rows_fp64 on scattered rows equals the chunked full result."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 1, 300, 32)); k = rng.standard_normal((1, 1, 300, 32))
    v = rng.standard_normal((1, 1, 300, 32))
    O, L = oracle.attention_fp64(q, k, v, causal=True, scale=0.2, row_chunk=64)
    rows = np.array([0, 1, 63, 64, 127, 128, 299])
    Or, Lr = oracle.attention_rows_fp64(q[0, 0], k[0, 0], v[0, 0], rows, True, 0.2)
    assert np.max(np.abs(Or - O[0, 0, rows])) == 0.0 and np.max(np.abs(Lr - L[0, 0, rows])) == 0.0


# ---------------------------------------------------------------------------
# Mutation tests: a plausible mistake planted in the oracle must fail a pin.
# ---------------------------------------------------------------------------

def _mut_causal_strict(q_bh, k_bh, v_bh, rows, causal, scale, key_offset=0):
    rows = np.asarray(rows); N = k_bh.shape[0]
    S = scale * (q_bh[rows] @ k_bh.T)
    if causal:
        S = np.where(np.arange(N)[None, :] < rows[:, None] + key_offset, S, -np.inf)   # j < i, not j <= i
    P, M, Z = oa.softmax_rows_fp64(S)
    return P @ v_bh, M + np.log(Z)


def _mut_no_scale(q_bh, k_bh, v_bh, rows, causal, scale, key_offset=0):
    return _ORIG_ROWS(q_bh, k_bh, v_bh, rows, causal, 1.0, key_offset)    # scale dropped


def _mut_lse_without_max(q_bh, k_bh, v_bh, rows, causal, scale, key_offset=0):
    rows = np.asarray(rows); N = k_bh.shape[0]
    S = scale * (q_bh[rows] @ k_bh.T)
    if causal:
        S = np.where(np.arange(N)[None, :] <= rows[:, None] + key_offset, S, -np.inf)
    P, M, Z = oa.softmax_rows_fp64(S)
    return P @ v_bh, np.log(Z)                                            # M term dropped


def _mut_transposed_keys(q_bh, k_bh, v_bh, rows, causal, scale, key_offset=0):
    rows = np.asarray(rows); N = k_bh.shape[0]
    S = scale * (q_bh[rows] @ k_bh[::-1].T)                               # key order reversed
    if causal:
        S = np.where(np.arange(N)[None, :] <= rows[:, None] + key_offset, S, -np.inf)
    P, M, Z = oa.softmax_rows_fp64(S)
    return P @ v_bh, M + np.log(Z)


def _mut_softmax_sign(S):
    M = np.max(S, axis=1, keepdims=True)
    E = np.exp(M - S)                                                     # sign flipped
    E = np.where(np.isfinite(S), E, 0.0)
    Z = np.sum(E, axis=1, keepdims=True)
    return E / Z, M[:, 0], Z[:, 0]


def _mut_blockmax_no_rescale(scores, values, block):
    s = np.asarray(scores, dtype=np.float64); vals = np.asarray(values, dtype=np.float64)
    m, l, acc, trace = -np.inf, 0.0, np.zeros(vals.shape[1:]), []
    for start in range(0, len(s), block):
        sb, vb = s[start:start + block], vals[start:start + block]
        m_block = np.max(sb); p = np.exp(sb - m_block)
        m_new = max(m, m_block)
        l = l + np.sum(p) * np.exp(m_block - m_new)                       # old total never rescaled
        acc = acc + np.tensordot(p, vb, axes=(0, 0)) * np.exp(m_block - m_new)
        m = m_new
        trace.append((m, l, np.array(acc, copy=True)))
    return acc / l, m, l, trace


def _mut_offset_ignored(q_bh, k_bh, v_bh, rows, causal, scale, key_offset=0):
    return _ORIG_ROWS(q_bh, k_bh, v_bh, rows, causal, scale, 0)            # N_k - N_q dropped


_ORIG_ROWS = oa.attention_rows_fp64

MUTANTS = {
    "causal_strict": ("attention_rows_fp64", _mut_causal_strict),
    "no_scale": ("attention_rows_fp64", _mut_no_scale),
    "lse_without_max": ("attention_rows_fp64", _mut_lse_without_max),
    "transposed_keys": ("attention_rows_fp64", _mut_transposed_keys),
    "offset_ignored": ("attention_rows_fp64", _mut_offset_ignored),
    "softmax_sign": ("softmax_rows_fp64", _mut_softmax_sign),
    "blockmax_no_rescale": ("online_softmax_row_blockmax", _mut_blockmax_no_rescale),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(oa, attr, fn)
    monkeypatch.setattr(oracle, attr, fn)
    failed = []
    with np.errstate(all="ignore"):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError, FloatingPointError):
                failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
