"""fp64 CPU oracle for the exact attention forward pass (test infrastructure).

Test infrastructure only: imported by the tests, ``__graft_entry__.smoke()``
and the CPU-baseline / reference arm of ``bench.py``; never by the product path.
It shares no code, header, table or constant with the CUDA library.

What it computes (the plain definition, materialising S and P):

* Page "Flash attention optimization" (aicomputerinstitute.com), section
  "Attention is not slow because of arithmetic": for Q, K, V in R^{N x d},
  S = Q K^T / sqrt(d), P = softmax(S) row-wise, O = P V.  The 1/sqrt(d) factor
  is the caller's ``scale`` (default 1/sqrt(d)).
* Same page, section "Worked example: online softmax by hand": the direct
  softmax subtracts the row's global maximum before exponentiating, then
  normalises by the sum of exponentials.
* Causal mask (the ``is_causal=True`` flag of the page "FlashAttention: The GPU
  Memory Hack That Changed Everything", section "Integration: It's
  Everywhere"): key j is allowed for query i iff j <= i.  Masked scores are
  -inf, so their weight exp(-inf - M) is exactly 0.
* The saved per-row statistic (section "Sizing a tile, and why the backward
  pass recomputes instead of storing" keeps the row max m and sum l):
  exported as LSE_i = M_i + ln(sum_j exp(S_ij - M_i)), natural-log units,
  scale included.

The two online-softmax row functions restate, in fp64, the recurrence of the
"The fix: tile the computation, never materialize the full matrix" section
(block-local max, then scale_old / scale_new) and the running-max form of the
first page's "The Tiling Strategy" pseudocode.  They exist only so the
self-tests can check that tiling reaches the direct result; the oracle proper
is the direct (materialising) definition.

The backward functions differentiate that definition (formulas in the
backward section below); the page's backward paragraph (same section as the
saved statistic) only says P is recomputed from Q, K, V and the statistics.

Parity is pinned by the CPU tests (worked example, exercise 1, closed forms,
invariants, brute force and an independent library routine); nothing here is
"parity unpinned".
"""

from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------------------
# Input conversion
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact conversion of raw bfloat16 bit patterns (uint16) to float64.

    A bfloat16 is the upper 16 bits of an IEEE binary32; shifting the pattern
    left by 16 gives that binary32 exactly, and binary32 -> binary64 is exact.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_bits_to_f64(bits) -> np.ndarray:
    """Exact value of FP8 E4M3 codes (uint8) as float64.

    E4M3 (the "fn" variant: no infinities): 1 sign bit, 4 exponent bits with
    bias 7, 3 mantissa bits.  Exponent field 0 is subnormal,
    (-1)^s * 2^-6 * m/8; otherwise (-1)^s * 2^(e-7) * (1 + m/8).  The codes
    0x7F and 0xFF (exponent and mantissa all ones) are NaN; 0x7E = 448 is the
    largest finite value.
    """
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    val = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64)))
    val = sign * val
    return np.where((b & 0x7F) == 0x7F, np.nan, val)


def _as_f64(x) -> np.ndarray:
    """Accept a numpy array or a CPU torch tensor (any real dtype) -> float64."""
    if hasattr(x, "detach"):  # torch tensor: go through float32, exact for bf16/fp16/fp32
        import torch

        x = x.detach().to("cpu")
        if x.dtype != torch.float64:
            x = x.to(torch.float32)
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Direct (materialising) definition
# ---------------------------------------------------------------------------

def softmax_rows_fp64(S: np.ndarray):
    """Row softmax of a score block with global-max subtraction.

    Returns (P, M, Z): P = exp(S - M) / Z row-wise, M the row max and
    Z = sum exp(S - M).  A row's masked entries are -inf and get weight 0.
    """
    M = np.max(S, axis=1, keepdims=True)
    E = np.exp(S - M)
    Z = np.sum(E, axis=1, keepdims=True)
    return E / Z, M[:, 0], Z[:, 0]


def attention_rows_fp64(q_bh, k_bh, v_bh, rows, causal: bool, scale: float,
                        key_offset: int = 0):
    """O and LSE for selected query rows of one (batch, head).

    q_bh: (N_q, d), k_bh, v_bh: (N_k, d) float64.  rows: 1-D int array of
    query indices.  Materialises the full score rows S[rows, :] and P[rows, :]
    (all N_k keys), then O = P V.  With causal masking query i may see key j
    iff j <= i + key_offset (0 for square problems; N_k - N_q when the N_q
    queries are the last N_q positions of the key sequence).  A row with no
    allowed key gets O = 0 and LSE = -inf (the empty sum).
    Returns (O (len(rows), d), LSE (len(rows),)).
    """
    rows = np.asarray(rows, dtype=np.int64)
    N = k_bh.shape[0]
    S = scale * (q_bh[rows] @ k_bh.T)                       # S = Q K^T * scale
    if causal:
        keys = np.arange(N, dtype=np.int64)
        allowed = keys[None, :] <= rows[:, None] + key_offset
        S = np.where(allowed, S, -np.inf)                   # allowed iff j <= i (+ offset)
        empty = ~allowed.any(axis=1)
        if empty.any():
            O = np.zeros((len(rows), v_bh.shape[1]))
            LSE = np.full(len(rows), -np.inf)
            keep = ~empty
            if keep.any():
                O[keep], LSE[keep] = attention_rows_fp64(q_bh, k_bh, v_bh, rows[keep], causal,
                                                         scale, key_offset)
            return O, LSE
    P, M, Z = softmax_rows_fp64(S)                          # P = softmax(S)
    O = P @ v_bh                                            # O = P V
    LSE = M + np.log(Z)
    return O, LSE


def attention_fp64(q, k, v, causal: bool = False, scale: float | None = None,
                   row_chunk: int = 512):
    """Exact attention forward in float64: q (B, H, N_q, d), k and v
    (B, H, N_k, d) (N_q = N_k for the square problems).

    Materialises S and P one chunk of ``row_chunk`` query rows at a time (rows
    are independent, so chunking changes no result; it bounds host memory for
    N = 32768).  Causal masking when N_q < N_k treats the queries as the last
    N_q positions: query i may see key j iff j <= i + N_k - N_q.
    Returns (O (B,H,N_q,d) float64, LSE (B,H,N_q) float64).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    if q.ndim != 4 or k.ndim != 4 or v.shape != k.shape or q.shape[:2] != k.shape[:2] \
            or q.shape[3] != k.shape[3]:
        raise ValueError("q must be (B, H, N_q, d) and k, v (B, H, N_k, d)")
    B, H, N, d = q.shape
    Nk = k.shape[2]
    # N_q queries are the last N_q positions of the N_k keys (causal offset).
    key_offset = Nk - N
    if causal and key_offset < 0:
        raise ValueError("causal attention needs N_q <= N_k")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = np.empty((B, H, N, d), dtype=np.float64)
    LSE = np.empty((B, H, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, row_chunk):
                r1 = min(N, r0 + row_chunk)
                rows = np.arange(r0, r1)
                O[b, h, r0:r1], LSE[b, h, r0:r1] = attention_rows_fp64(
                    q[b, h], k[b, h], v[b, h], rows, causal, scale, key_offset)
    return O, LSE


# ---------------------------------------------------------------------------
# Backward pass (gradients of the direct definition)
# ---------------------------------------------------------------------------
#
# The page "Flash attention optimization", section "Sizing a tile, and why the
# backward pass recomputes instead of storing", says the backward pass needs P
# again and rebuilds it from the saved Q, K, V and per-row statistics instead
# of storing it; it prints no gradient formula.  The oracle therefore
# differentiates the forward definition above.  For a scalar loss with upstream
# gradient dO = dL/dO, and with S = scale * Q K^T (masked), P = softmax(S)
# row-wise, O = P V:
#
#   dV = P^T dO                       (O is linear in V)
#   dP = dO V^T
#   D_i = sum_t dO_it O_it            (= sum_j P_ij dP_ij)
#   dS = P * (dP - D[:, None])        (Jacobian of the row softmax)
#   dQ = scale * dS K,   dK = scale * dS^T Q
#
# P is recomputed exactly as in the forward (global-max subtraction), so masked
# entries are exactly 0 and contribute nothing.

def attention_bwd_rows_fp64(q_bh, k_bh, v_bh, do_bh, rows, causal: bool, scale: float,
                            key_offset: int = 0):
    """Gradient contributions of selected query rows of one (batch, head).

    q_bh, do_bh: (N_q, d); k_bh, v_bh: (N_k, d) float64.  Materialises
    S[rows, :] and P[rows, :] over all keys, then applies the formulas above.
    Returns (dQ_rows (len(rows), d), dK_part (N_k, d), dV_part (N_k, d),
    D_rows (len(rows),)): dQ of these rows is complete; dK and dV are the sums
    over these rows only (the caller adds the parts of all row chunks).  Rows
    with no allowed key (causal, N_q > N_k) contribute nothing.
    """
    rows = np.asarray(rows, dtype=np.int64)
    N = k_bh.shape[0]
    S = scale * (q_bh[rows] @ k_bh.T)                       # S = Q K^T * scale
    if causal:
        allowed = np.arange(N, dtype=np.int64)[None, :] <= rows[:, None] + key_offset
        S = np.where(allowed, S, -np.inf)
        keep = allowed.any(axis=1)
        if not keep.all():
            dQ = np.zeros((len(rows), q_bh.shape[1]))
            D = np.zeros(len(rows))
            dK = np.zeros_like(k_bh)
            dV = np.zeros_like(v_bh)
            if keep.any():
                dQ[keep], dK, dV, D[keep] = attention_bwd_rows_fp64(
                    q_bh, k_bh, v_bh, do_bh, rows[keep], causal, scale, key_offset)
            return dQ, dK, dV, D
    P, _, _ = softmax_rows_fp64(S)                          # P recomputed
    dO = do_bh[rows]
    O = P @ v_bh                                            # O = P V
    dV = P.T @ dO                                           # dV = P^T dO
    dP = dO @ v_bh.T                                        # dP = dO V^T
    D = np.sum(dO * O, axis=1)                              # D_i = dO_i . O_i
    dS = P * (dP - D[:, None])                              # softmax Jacobian
    dQ = scale * (dS @ k_bh)                                # dQ = scale dS K
    dK = scale * (dS.T @ q_bh[rows])                        # dK = scale dS^T Q
    return dQ, dK, dV, D


def attention_bwd_fp64(q, k, v, do, causal: bool = False, scale: float | None = None,
                       row_chunk: int = 512):
    """Exact attention backward in float64: q, do (B, H, N_q, d); k, v (B, H, N_k, d).

    Returns (dQ, dK, dV, D) as float64 arrays of the inputs' shapes (D has
    shape (B, H, N_q)).  Rows are processed ``row_chunk`` at a time; dK and dV
    are the sums of the chunks' parts.  Causal masking follows the forward:
    query i may see key j iff j <= i + N_k - N_q.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    if q.ndim != 4 or k.ndim != 4 or v.shape != k.shape or q.shape[:2] != k.shape[:2] \
            or q.shape[3] != k.shape[3] or do.shape != q.shape:
        raise ValueError("q and do must be (B, H, N_q, d) and k, v (B, H, N_k, d)")
    B, H, N, d = q.shape
    key_offset = k.shape[2] - N
    if causal and key_offset < 0:
        raise ValueError("causal attention needs N_q <= N_k")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dQ = np.empty_like(q)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    D = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, row_chunk):
                rows = np.arange(r0, min(N, r0 + row_chunk))
                dq, dk, dv, dd = attention_bwd_rows_fp64(q[b, h], k[b, h], v[b, h], do[b, h],
                                                         rows, causal, scale, key_offset)
                dQ[b, h, rows] = dq
                dK[b, h] += dk
                dV[b, h] += dv
                D[b, h, rows] = dd
    return dQ, dK, dV, D


# ---------------------------------------------------------------------------
# Tiled forms (self-test companions, never the oracle)
# ---------------------------------------------------------------------------

def online_softmax_row_blockmax(scores, values, block: int):
    """One query row, tiled, with each block's exponentials taken relative to
    that block's own max and merged with scale_old = exp(m_old - m_new) and
    scale_new = exp(m_block - m_new) (page "Flash attention optimization",
    section "The fix: tile the computation, never materialize the full
    matrix").  ``values`` is (n,) or (n, d).  Returns (O, m, l, trace) where
    trace lists the running (m, l, acc) after each block.
    """
    s = np.asarray(scores, dtype=np.float64)
    vals = np.asarray(values, dtype=np.float64)
    n = s.shape[0]
    m = -np.inf
    l = 0.0
    acc = np.zeros(vals.shape[1:], dtype=np.float64)
    trace = []
    for start in range(0, n, block):
        sb = s[start:start + block]
        vb = vals[start:start + block]
        m_block = np.max(sb)
        p = np.exp(sb - m_block)
        l_block = np.sum(p)
        acc_block = np.tensordot(p, vb, axes=(0, 0))
        m_new = max(m, m_block)
        # With m = -inf on the first block this factor is exp(-inf) = 0:
        # the empty running state is discarded without a special case.
        scale_old = np.exp(m - m_new)
        scale_new = np.exp(m_block - m_new)
        l = l * scale_old + l_block * scale_new
        acc = acc * scale_old + acc_block * scale_new
        m = m_new
        trace.append((m, l, np.array(acc, copy=True)))
    return acc / l, m, l, trace


def online_softmax_row_runningmax(scores, values, block: int):
    """One query row, tiled, with exponentials taken relative to the updated
    running max (page "FlashAttention: The GPU Memory Hack That Changed
    Everything", section "The Tiling Strategy": l = l*exp(m - m_new) +
    sum exp(S - m_new); O = O*exp(m - m_new) + exp(S - m_new) V; final O/l).
    Returns (O, m, l).
    """
    s = np.asarray(scores, dtype=np.float64)
    vals = np.asarray(values, dtype=np.float64)
    n = s.shape[0]
    m = -np.inf
    l = 0.0
    acc = np.zeros(vals.shape[1:], dtype=np.float64)
    for start in range(0, n, block):
        sb = s[start:start + block]
        vb = vals[start:start + block]
        m_new = max(m, np.max(sb))
        alpha = np.exp(m - m_new)
        p = np.exp(sb - m_new)
        l = l * alpha + np.sum(p)
        acc = acc * alpha + np.tensordot(p, vb, axes=(0, 0))
        m = m_new
    return acc / l, m, l


def tiled_attention_fp64(q, k, v, causal: bool, scale: float, block_q: int,
                         block_k: int):
    """Whole-matrix tiled forward for one (N, d) head: Q blocks outer, K/V
    blocks inner, running (m, l, acc) per row (page "FlashAttention: The GPU
    Memory Hack That Changed Everything", section "The Tiling Strategy").
    Causal K/V blocks that lie entirely above the diagonal are skipped, and
    partially masked entries are -inf.  Self-test companion only.
    Returns (O (N, d), LSE (N,)).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    N, d = q.shape
    O = np.empty((N, d))
    LSE = np.empty(N)
    for i0 in range(0, N, block_q):
        i1 = min(N, i0 + block_q)
        qi = q[i0:i1]
        m = np.full(i1 - i0, -np.inf)
        l = np.zeros(i1 - i0)
        acc = np.zeros((i1 - i0, d))
        for j0 in range(0, N, block_k):
            if causal and j0 > i1 - 1:
                break                                   # block fully above the diagonal
            j1 = min(N, j0 + block_k)
            Sij = scale * (qi @ k[j0:j1].T)
            if causal:
                ii = np.arange(i0, i1)[:, None]
                jj = np.arange(j0, j1)[None, :]
                Sij = np.where(jj <= ii, Sij, -np.inf)
            m_new = np.maximum(m, Sij.max(axis=1))
            alpha = np.exp(m - m_new)
            p = np.exp(Sij - m_new[:, None])
            l = l * alpha + p.sum(axis=1)
            acc = acc * alpha[:, None] + p @ v[j0:j1]
            m = m_new
        O[i0:i1] = acc / l[:, None]
        LSE[i0:i1] = m + np.log(l)
    return O, LSE
