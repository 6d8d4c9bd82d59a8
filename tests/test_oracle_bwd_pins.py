"""Pins for the oracle's backward pass (gradients of the exact forward).

The pages print no gradient formula (the page "Flash attention optimization",
section "Sizing a tile, and why the backward pass recomputes instead of
storing", only says P is rebuilt from Q, K, V and the per-row statistics), so
each pin checks the oracle's dQ, dK, dV against something that does not use
its formulas:

* the worked example's printed weights and output (tests/golden/), from which
  dV, dK and dQ of the example's query row follow by hand;
* central finite differences of the forward oracle (already pinned on its own);
* torch.autograd through a plain float64 softmax attention (a library routine);
* invariants of the softmax Jacobian and a closed form for uniform attention.

The mutation tests plant plausible mistakes in the backward rows function and
check that some pin fails for each.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import oracle.exact_attention as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bwd(*args, **kw):
    return oracle.attention_bwd_fp64(*args, **kw)


def _fwd_loss(q, k, v, do, causal, scale):
    O, _ = oracle.attention_fp64(q, k, v, causal=causal, scale=scale)
    return float(np.sum(O * do))


# ---------------------------------------------------------------------------
# Pins
# ---------------------------------------------------------------------------

def pin_bwd_worked_example():
    """One query row with scores s = [1, 3, 2, 5] and values [10, 20, 30, 40]
    (scale 1, d = 1) and upstream gradient dO = 1 on that row only.

    By hand from the definition: dV_j = w_j, dK_j = w_j (v_j - O) q and
    dQ = sum_j w_j (v_j - O) k_j, with w the page's printed weights and O its
    printed output (5 and 4 decimals)."""
    with open(os.path.join(GOLDEN, "online_softmax_worked_example.json")) as f:
        g = json.load(f)
    s = np.array(g["scores"]); vals = np.array(g["values"])
    w = np.array(g["direct"]["weights"]); O = g["direct"]["O"]
    n = len(s)
    q = np.zeros((1, 1, 1, 1)); q[0, 0, 0, 0] = 1.0
    k = s.reshape(1, 1, n, 1); v = vals.reshape(1, 1, n, 1)
    do = np.ones((1, 1, 1, 1))
    dQ, dK, dV, D = _bwd(q, k, v, do, causal=False, scale=1.0)
    ew, eo = 0.5e-5, 0.5e-4                     # half a unit in the printed last digit
    assert np.all(np.abs(dV[0, 0, :, 0] - w) <= ew), dV[0, 0, :, 0]
    exp_dk = w * (vals - O)
    tol_dk = ew * np.abs(vals - O) + w * eo + ew * eo
    assert np.all(np.abs(dK[0, 0, :, 0] - exp_dk) <= tol_dk), (dK[0, 0, :, 0], exp_dk)
    exp_dq = float(np.sum(w * (vals - O) * s))
    tol_dq = float(np.sum(np.abs(s) * tol_dk))
    assert abs(dQ[0, 0, 0, 0] - exp_dq) <= tol_dq, (dQ[0, 0, 0, 0], exp_dq)
    assert abs(D[0, 0, 0] - O) <= eo


def pin_bwd_finite_differences():
    """Central differences of L = sum(O * dO), with O from the forward oracle."""
    rng = np.random.default_rng(11)
    for causal, Nq, Nk in [(False, 5, 5), (True, 5, 5), (True, 3, 6), (False, 4, 7)]:
        d, scale, h = 3, 0.7, 1e-6
        q = rng.standard_normal((1, 2, Nq, d)); do = rng.standard_normal((1, 2, Nq, d))
        k = rng.standard_normal((1, 2, Nk, d)); v = rng.standard_normal((1, 2, Nk, d))
        dQ, dK, dV, _ = _bwd(q, k, v, do, causal=causal, scale=scale)
        for name, x, g in (("q", q, dQ), ("k", k, dK), ("v", v, dV)):
            num = np.empty_like(x)
            for idx in np.ndindex(x.shape):
                xp = x.copy(); xp[idx] += h
                xm = x.copy(); xm[idx] -= h
                args = {"q": q, "k": k, "v": v}
                args[name] = xp
                lp = _fwd_loss(args["q"], args["k"], args["v"], do, causal, scale)
                args[name] = xm
                lm = _fwd_loss(args["q"], args["k"], args["v"], do, causal, scale)
                num[idx] = (lp - lm) / (2 * h)
            err = np.max(np.abs(num - g))
            assert err <= 1e-7 * max(1.0, np.max(np.abs(g))), (name, causal, Nq, Nk, err)


def pin_bwd_library_routine():
    """torch.autograd through softmax(scale * q k^T + mask) v in float64."""
    rng = np.random.default_rng(12)
    for causal, Nq, Nk, d in [(False, 37, 37, 8), (True, 45, 45, 8), (True, 20, 33, 4)]:
        scale = 0.3
        q = rng.standard_normal((2, 1, Nq, d)); do = rng.standard_normal((2, 1, Nq, d))
        k = rng.standard_normal((2, 1, Nk, d)); v = rng.standard_normal((2, 1, Nk, d))
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        s = scale * tq @ tk.transpose(-1, -2)
        if causal:
            allowed = torch.arange(Nk)[None, :] <= torch.arange(Nq)[:, None] + (Nk - Nq)
            s = s.masked_fill(~allowed, float("-inf"))
        o = torch.softmax(s, dim=-1) @ tv
        o.backward(torch.tensor(do))
        dQ, dK, dV, _ = _bwd(q, k, v, do, causal=causal, scale=scale)
        for ours, ref in ((dQ, tq.grad), (dK, tk.grad), (dV, tv.grad)):
            assert np.max(np.abs(ours - ref.numpy())) <= 1e-12, (causal, Nq, Nk)


def pin_bwd_invariants():
    """Softmax-Jacobian invariants on a random causal and non-causal head.

    Every row of dS sums to 0, so the keys' dK sum to 0; every row of P sums to
    1, so the keys' dV sum to the queries' dO sum; causal row 0 sees one key
    with weight 1, so its dQ is 0; the last key is seen by the last query only,
    so its dV is P[N-1, N-1] dO[N-1]."""
    rng = np.random.default_rng(13)
    N, d, scale = 40, 6, 0.45
    q = rng.standard_normal((1, 1, N, d)); k = rng.standard_normal((1, 1, N, d))
    v = rng.standard_normal((1, 1, N, d)); do = rng.standard_normal((1, 1, N, d))
    for causal in (False, True):
        dQ, dK, dV, D = _bwd(q, k, v, do, causal=causal, scale=scale, row_chunk=7)
        assert np.max(np.abs(dK[0, 0].sum(axis=0))) <= 1e-12
        assert np.max(np.abs(dV[0, 0].sum(axis=0) - do[0, 0].sum(axis=0))) <= 1e-12
        O, _ = oracle.attention_fp64(q, k, v, causal=causal, scale=scale)
        assert np.max(np.abs(D[0, 0] - np.sum(O[0, 0] * do[0, 0], axis=1))) <= 1e-12
        if causal:
            assert np.max(np.abs(dQ[0, 0, 0])) <= 1e-15
            s_last = scale * q[0, 0, -1] @ k[0, 0].T
            p_last = math.exp(s_last[-1] - s_last.max()) / np.sum(np.exp(s_last - s_last.max()))
            assert np.max(np.abs(dV[0, 0, -1] - p_last * do[0, 0, -1])) <= 1e-12


def pin_bwd_closed_form_uniform():
    """q = 0 (non-causal): every weight is 1/N, so dV_j = mean_i dO_i for every
    key, dK = 0 (dK is a combination of the zero queries) and
    dQ_i = scale/N * sum_j (dO_i . (v_j - mean v)) k_j."""
    rng = np.random.default_rng(14)
    N, d, scale = 24, 5, 0.8
    q = np.zeros((1, 1, N, d)); k = rng.standard_normal((1, 1, N, d))
    v = rng.standard_normal((1, 1, N, d)); do = rng.standard_normal((1, 1, N, d))
    dQ, dK, dV, _ = _bwd(q, k, v, do, causal=False, scale=scale)
    vbar = v[0, 0].mean(axis=0)
    for j in range(N):
        assert np.max(np.abs(dV[0, 0, j] - do[0, 0].mean(axis=0))) <= 1e-13
    assert np.max(np.abs(dK)) == 0.0
    for i in range(N):
        acc = np.zeros(d)
        for j in range(N):
            acc += float(np.dot(do[0, 0, i], v[0, 0, j] - vbar)) * k[0, 0, j]
        assert np.max(np.abs(dQ[0, 0, i] - scale / N * acc)) <= 1e-12


BWD_PINS = [pin_bwd_worked_example, pin_bwd_finite_differences, pin_bwd_library_routine,
            pin_bwd_invariants, pin_bwd_closed_form_uniform]


@pytest.mark.parametrize("pin", BWD_PINS, ids=[p.__name__ for p in BWD_PINS])
def test_bwd_pin(pin):
    pin()


def test_bwd_row_chunking_changes_nothing():
    rng = np.random.default_rng(15)
    q, k, v, do = (rng.standard_normal((1, 2, 50, 4)) for _ in range(4))
    a = _bwd(q, k, v, do, causal=True, scale=0.5, row_chunk=1)
    b = _bwd(q, k, v, do, causal=True, scale=0.5, row_chunk=512)
    for x, y in zip(a, b):
        assert np.max(np.abs(x - y)) <= 1e-12


# ---------------------------------------------------------------------------
# Mutation tests
# ---------------------------------------------------------------------------

def _make_mutant(kind):
    def rows_fn(q_bh, k_bh, v_bh, do_bh, rows, causal, scale, key_offset=0):
        rows = np.asarray(rows, dtype=np.int64)
        N = k_bh.shape[0]
        S = scale * (q_bh[rows] @ k_bh.T)
        if causal and kind != "mask_ignored":
            allowed = np.arange(N)[None, :] <= rows[:, None] + key_offset
            S = np.where(allowed, S, -np.inf)
        P, _, _ = oa.softmax_rows_fp64(S)
        dO = do_bh[rows]
        O = P @ v_bh
        dV = P.T @ dO
        dP = dO @ v_bh.T
        D = np.sum(dO * O, axis=1)
        if kind == "d_unweighted":
            D = np.sum(dP, axis=1)                      # P weight dropped from D
        dS = P * (dP - D[:, None])
        if kind == "no_d":
            dS = P * dP                                 # D term dropped
        dQ = scale * (dS @ k_bh)
        dK = scale * (dS.T @ q_bh[rows])
        if kind == "dq_no_scale":
            dQ = dS @ k_bh
        if kind == "dk_no_scale":
            dK = dS.T @ q_bh[rows]
        if kind == "dq_uses_v":
            dQ = scale * (dS @ v_bh)
        if kind == "dk_uses_do":
            dK = scale * (dS.T @ dO)
        if kind == "dv_uses_ds":
            dV = dS.T @ dO
        return dQ, dK, dV, D
    return rows_fn


BWD_MUTANTS = ["no_d", "d_unweighted", "dq_no_scale", "dk_no_scale", "dq_uses_v", "dk_uses_do",
               "dv_uses_ds", "mask_ignored"]


@pytest.mark.parametrize("kind", BWD_MUTANTS)
def test_bwd_mutant_is_caught(kind, monkeypatch):
    fn = _make_mutant(kind)
    monkeypatch.setattr(oa, "attention_bwd_rows_fp64", fn)
    monkeypatch.setattr(oracle, "attention_bwd_rows_fp64", fn)
    failed = []
    with np.errstate(all="ignore"):
        for pin in BWD_PINS:
            try:
                pin()
            except (AssertionError, ValueError, FloatingPointError):
                failed.append(pin.__name__)
    assert failed, f"mutant {kind} passed every pin"
