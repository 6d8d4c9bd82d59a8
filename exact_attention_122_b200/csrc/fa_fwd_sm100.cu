// fa_fwd_sm100.cu -- exact attention forward for B200 (sm_100a).
//
// Computes, per (batch, head), O = softmax(scale * Q K^T [+ causal mask]) V
// and the per-row log-sum-exp, tile by tile with the online-softmax
// recurrence, so the N x N score matrix never leaves the SM:
//   * page "Flash attention optimization", section "Attention is not slow
//     because of arithmetic" (the definition) and "The fix: tile the
//     computation, never materialize the full matrix" (running max m,
//     running sum l, rescaled accumulator, final acc / l);
//   * page "FlashAttention: The GPU Memory Hack That Changed Everything",
//     section "The Tiling Strategy" (Q blocks outer, K/V blocks inner, the
//     exponent taken relative to the updated running max) and
//     "FlashAttention-2: Even Faster" (work split over the sequence as well
//     as batch x heads; fewer non-matmul operations);
//   * same page, "FlashAttention-3: Hopper Architecture" (asynchronous
//     copies, warp specialisation), re-done for sm_100a with TMA, mbarriers,
//     tcgen05 MMAs and tensor memory (TMEM).
//
// Kernel organisation (one persistent CTA per SM, 384 threads):
//   warps 0-3  softmax warpgroup 0: rows 0..127 of the current 256-row unit
//   warps 4-7  softmax warpgroup 1: rows 128..255
//   warp  8    MMA issuer (one thread): S_t = Q_t K_j^T and O_t += P_t V_j
//   warp  9    TMA producer (one thread): Q_0, Q_1 per unit, then K_j, V_j
//              through an NS-stage shared-memory ring
//   warps 10-11 idle (they complete the third warpgroup)
// The third warpgroup gives registers to the softmax warpgroups with
// setmaxnreg (Regs<D, F8>::SOFTMAX / OTHER below).
// Each softmax thread owns one query row (TMEM lane == row), so the row max
// and row sum are in-thread.  S_t (fp32, 128 columns) and O_t (fp32, d
// columns) live in TMEM; P_t is written back as bf16 over the first 64
// columns of S_t (bf16 d = 64: into 64 columns of its own) and read from
// TMEM by the PV MMA.  The two warpgroups alternate with the single MMA
// issuer, so the tensor core works on one sub-tile while the other
// sub-tile's exponentials run; with P in its own columns the next tile's
// S_t is issued as soon as the softmax has read the current one.
//
// Every mbarrier wait is bounded by a %globaltimer watchdog.  A wait that
// runs out records FA_ERR_TIMEOUT in g_fa_status, raises a CTA-wide abort
// flag so every role leaves its loop, drains its own TMA copies and MMAs
// (again bounded), frees TMEM and returns.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <vector>

#include "fa.h"
#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {

using namespace sm100;

// ---------------------------------------------------------------------------
// Tile geometry
// ---------------------------------------------------------------------------
constexpr int BM = 128;            // query rows per sub-tile (= TMEM lanes)
constexpr int BN = 128;            // keys per K/V tile
constexpr int UNIT_ROWS = 2 * BM;  // query rows per work unit (two sub-tiles)
constexpr int NUM_THREADS = 384;
constexpr int MMA_WARP = 8;
constexpr int TMA_WARP = 9;
// Register split.  The launch gives every thread REGS_LAUNCH registers
// (65536 / 384, rounded down to 8 and to the sub-partition share: 168).
// Warpgroup 2 drops to Regs::OTHER once at the start and never rises again;
// warpgroups 0 and 1 rise to Regs::SOFTMAX.  The sum must not exceed the
// launch total or setmaxnreg.inc never returns.
constexpr int REGS_LAUNCH = 168;
// The bf16 d = 128 kernel spilled registers (ptxas -v) with 80 for the third
// warpgroup; with 96 there and 200 for the softmax warpgroups it does not.
template <int D, bool F8>
struct Regs {
    static constexpr int SOFTMAX = (D == 128 && !F8) ? 200 : 208;
    static constexpr int OTHER = (D == 128 && !F8) ? 96 : 80;
    static_assert(2 * 128 * SOFTMAX + 128 * OTHER <= NUM_THREADS * REGS_LAUNCH,
                  "register split exceeds the launch allocation");
};
constexpr int SW_COLS = 64;        // bf16 elements per 128-byte swizzled row
// Lazy rescale: the running max that l and O refer to is only moved when a
// row's new maximum exceeds it by more than rescale_log2<F8> (log2 units), so
// P stays below 2^rescale_log2 and O is rescaled rarely.  l and O share the
// stale reference, so O = acc / l and LSE = (m + log2 l) ln 2 stay exact.
// bf16 P takes 2^12 (rescales on peaked rows are fewer: +1.5 % on the 32K
// peaked workload over 2^8); E4M3 P saturates at 448, so FP8 keeps 2^8.
template <bool F8>
__host__ __device__ constexpr float rescale_log2() { return F8 ? 8.0f : 12.0f; }
enum : uint32_t {
    ROLE_SOFTMAX = 1u, ROLE_MMA = 2u, ROLE_PRODUCER = 3u, ROLE_DRAIN = 4u
};

// F8: Q, K, V are FP8 E4M3 (one byte per element) and V arrives transposed
// (d rows x keys), so every operand is K-major; a 128-byte swizzled row then
// holds 128 elements instead of 64.
template <int D, int NS, bool F8 = false>
struct Layout {
    static constexpr int EB = F8 ? 1 : 2;            // bytes per element
    static constexpr int Q_BYTES = BM * D * EB;      // one sub-tile of Q
    static constexpr int KV_BYTES = BN * D * EB;     // one K or V tile
    static constexpr int HALF_BYTES = BM * 128;      // one 128-byte-wide slab (16 KiB)
    // FP8 at d = 64: a Q / K row is 64 bytes, held in 64-byte-swizzled tiles
    // (one slab); every other case uses 128-byte rows.
    static constexpr bool SW64 = F8 && D == 64;
    static constexpr int SLABS = SW64 ? 1 : D * EB / 128;   // slabs per Q / K tile
    static constexpr int SLAB_ELEMS = 128 / EB;      // elements per slab row
    static constexpr int QK_STEPS = D * EB / 32;     // 32-byte K steps of S = Q K^T
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = 2 * Q_BYTES;
    static constexpr int OFF_BAR = OFF_KV + NS * KV_BYTES;
    // barrier slots
    static constexpr int B_KV_FULL = 0;
    static constexpr int B_KV_EMPTY = NS;
    static constexpr int B_Q_FULL = 2 * NS;
    static constexpr int B_Q_EMPTY = 2 * NS + 1;
    static constexpr int B_S_FULL = 2 * NS + 2;      // [2]
    static constexpr int B_P_FULL = 2 * NS + 4;      // [2]
    static constexpr int B_O_FULL = B_P_FULL + 2;    // [2]
    static constexpr int B_O_EMPTY = B_O_FULL + 2;   // [2]
    static constexpr int B_DRAIN = B_O_EMPTY + 2;
    static constexpr int B_UFULL = B_DRAIN + 1;      // [2] unit queue (dynamic schedule)
    static constexpr int B_UEMPTY = B_UFULL + 2;     // [2]
    static constexpr int B_S_FREE = B_UEMPTY + 2;    // [2] S_t read into registers (SEP_P)
    static constexpr int B_PV_DONE = B_S_FREE + 2;   // [2] P_t V complete (SEP_P)
    static constexpr int NUM_BARS = B_PV_DONE + 2;
    // tmem base, abort flag, zero flag, spare, unit queue slots [2]
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int OFF_UNIT = OFF_MISC + 16;
    static constexpr int BYTES = OFF_MISC + 32;
    static constexpr int ALLOC = BYTES + 1024;       // slack to align the base to 1 KiB
    // TMEM columns.  SEP_P (bf16, d = 64): P_t gets its own 64 columns
    // instead of overwriting S_t, so S_t of the next K/V tile can be computed
    // while the softmax of the current one runs (S 2 x 128 + P 2 x 64 + O
    // 2 x 64 = 512 columns).  Otherwise P_t aliases the first columns of S_t.
    static constexpr bool SEP_P = D == 64 && !F8;
    static constexpr uint32_t TM_S0 = 0, TM_S1 = 128;
    static constexpr uint32_t TM_P0 = SEP_P ? 256 : TM_S0, TM_P1 = SEP_P ? 320 : TM_S1;
    static constexpr uint32_t TM_O0 = SEP_P ? 384 : 256, TM_O1 = TM_O0 + D;
    static constexpr uint32_t TM_COLS = 512;
    static_assert(TM_O1 + D <= TM_COLS, "TMEM columns");
    static_assert(ALLOC <= 227 * 1024, "shared memory budget");
    static_assert(BYTES > 116 * 1024, "one CTA per SM keeps TMEM allocation uncontended");
};

__device__ unsigned int g_fa_status;  // 0 = fine; else (FA_ERR_TIMEOUT << 24) | role << 20 | unit

struct Watchdog {
    volatile int* abort_flag;
    uint64_t limit_ns;
};

// Waits for the phase of `bar` with the given parity to complete.  Returns
// false if the CTA is aborting or this wait ran past the watchdog limit (in
// which case it records the timeout and raises the abort flag).
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, Watchdog wd,
                                        uint32_t role, uint32_t unit) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*wd.abort_flag) return false;
        if (global_timer_ns() - t0 > wd.limit_ns) {
            atomicCAS(&g_fa_status, 0u,
                      (uint32_t(FA_ERR_TIMEOUT) << 24) | (role << 20) | (unit & 0xFFFFFu));
            *wd.abort_flag = 1;
            __threadfence_block();
            return false;
        }
    }
}

// Barrier 0 over all NUM_THREADS threads, usable from different branches.
__device__ __forceinline__ void cta_sync() {
    asm volatile("bar.sync 0, %0;" ::"n"(NUM_THREADS) : "memory");
}

// ---------------------------------------------------------------------------
// Work decomposition: units of 256 query rows of one (batch, head), named by
// the id c = bh * nq2 + qb2 (qb2: the unit's 256-row block).
//
// Both schedules walk heads in groups of `hg` (sized on the host so a
// group's K and V stay resident in L2 while the CTAs working on it stream
// them).
//  * Sequence order (the dynamic schedule's claim order, and the static
//    "snake" assignment): inside a group, by row block, the longest causal
//    rows first; static CTA b takes sequence indices in boustrophedon order
//    (b, 2S-1-b, 2S+b, ...) so long and short units pair up across CTAs.
//  * Paired static assignment (causal): the row blocks q and nq2-1-q of one
//    head form a pair whose K/V tile count hardly depends on q, so dealing
//    pairs round-robin (CTA b takes pairs b, b+S, b+2S, ..., the long unit of
//    each pair first) balances the CTAs to within one pair whatever the group
//    size.  With an odd nq2 the middle row block is a pair of one unit.
// ---------------------------------------------------------------------------
struct Unit {
    int bh, r0, nb0, nb1;  // first row, K/V tile counts of sub-tiles 0 and 1
};

constexpr int UNIT_END = -1;   // no more units for this CTA
constexpr int UNIT_SKIP = -2;  // static paired schedule: empty second half of a pair

__device__ __forceinline__ int unit_index(int k, int cta, int ctas) {
    return k * ctas + ((k & 1) ? (ctas - 1 - cta) : cta);
}

// Sequence index i (grouped, longest first) -> unit id.
__device__ __forceinline__ int seq_to_unit(int i, int BH, int nq2, int causal, int hg) {
    const int per_group = hg * nq2;
    const int g = i / per_group;
    const int r = i - g * per_group;
    const int gh = min(hg, BH - g * hg);       // heads in this group
    const int level = r / gh;
    const int bh = g * hg + (r - level * gh);
    return bh * nq2 + (causal ? (nq2 - 1 - level) : level);
}

// The kq-th unit of CTA `cta` under the static schedule: a unit id,
// UNIT_END, or UNIT_SKIP (move on to kq + 1).
__device__ __forceinline__ int static_unit(int kq, int cta, int ctas, int BH, int nq2, int causal,
                                           int hg, int paired) {
    if (!paired) {
        const int i = unit_index(kq, cta, ctas);
        return i < BH * nq2 ? seq_to_unit(i, BH, nq2, causal, hg) : UNIT_END;
    }
    const int npl = (nq2 + 1) / 2;             // pairs per head
    const int p = (kq >> 1) * ctas + cta;
    if (p >= BH * npl) return UNIT_END;
    const int per_group = hg * npl;
    const int g = p / per_group;
    const int r = p - g * per_group;
    const int gh = min(hg, BH - g * hg);
    const int pl = r / gh;
    const int bh = g * hg + (r - pl * gh);
    const int q_long = nq2 - 1 - pl;
    if (kq & 1) return pl == q_long ? UNIT_SKIP : bh * nq2 + pl;
    return bh * nq2 + q_long;
}

// N_q query rows and N_k keys per (batch, head); with causal masking query i
// may see key j iff j <= i + N_k - N_q (the queries are the last N_q
// positions), so a sub-tile's last row r sees keys up to r + N_k - N_q.
__device__ __forceinline__ Unit decode_unit(int c, int Nq, int Nk, int causal) {
    const int nq2 = (Nq + UNIT_ROWS - 1) / UNIT_ROWS;
    const int nkb = (Nk + BN - 1) / BN;
    const int off = Nk - Nq;
    Unit w;
    w.bh = c / nq2;
    w.r0 = (c - w.bh * nq2) * UNIT_ROWS;
    if (causal) {
        w.nb0 = min((w.r0 + BM - 1 + off) / BN + 1, nkb);
        w.nb1 = min((w.r0 + 2 * BM - 1 + off) / BN + 1, nkb);
    } else {
        w.nb0 = nkb;
        w.nb1 = nkb;
    }
    return w;
}

// S = Q K^T for one sub-tile: M=128 query rows, N=128 keys, K=d in steps
// of 16.  Both operands K-major with 128-byte swizzle: a step is 32 bytes
// inside a swizzled row, and 64-column slabs are HALF_BYTES apart.
// A step is 16 bf16 or 32 FP8 elements: 32 bytes either way.
template <int STEPS, int HALF_BYTES, bool F8>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc,
                                         uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < STEPS; ++kk) {
        const uint32_t off = uint32_t(((kk / 4) * HALF_BYTES + (kk % 4) * 32) >> 4);
        if constexpr (F8)
            mma_ss_f8(d_tmem, desc_add(q_desc, off), desc_add(k_desc, off), idesc, kk > 0 ? 1u : 0u);
        else
            mma_ss(d_tmem, desc_add(q_desc, off), desc_add(k_desc, off), idesc, kk > 0 ? 1u : 0u);
    }
}

// O += P V for one sub-tile: A = P from TMEM (8 columns per step: 16 keys
// as bf16 pairs, or 32 keys as FP8 quads).  bf16: B = V MN-major, 16 key
// rows of 128 bytes per step.  FP8: B = V^T K-major (d rows of 128 keys), a
// step is 32 bytes inside the swizzled rows.  `first`: the unit's first tile
// overwrites O instead of accumulating.
template <bool F8>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint64_t v_desc,
                                         uint32_t idesc, bool first) {
    if constexpr (F8) {
#pragma unroll
        for (int kk = 0; kk < BN / 32; ++kk)
            mma_ts_f8(o_tmem, p_tmem + kk * 8, desc_add(v_desc, uint32_t((kk * 32) >> 4)), idesc,
                      (first && kk == 0) ? 0u : 1u);
    } else {
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
            const uint32_t off = uint32_t((kk * 16 * 128) >> 4);
            mma_ts(o_tmem, p_tmem + kk * 8, desc_add(v_desc, off), idesc,
                   (first && kk == 0) ? 0u : 1u);
        }
    }
}

// p rounded the way exp_row_to_p rounds P for the P V product: bf16 (nearest
// even) or, with F8, FP8 E4M3 (nearest even, saturating).
template <bool F8>
__device__ __forceinline__ float round_as_p(float p) {
    if constexpr (F8) {
        uint16_t q8;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(q8) : "f"(0.0f), "f"(p));
        uint32_t h2;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(q8));
        return __half2float(__ushort_as_half(uint16_t(h2 & 0xFFFFu)));
    } else {
        return __bfloat162float(__float2bfloat16_rn(p));
    }
}

// P = 2^(s * scale_log2 - m) for one score row held in registers, written
// to TMEM over the row's first columns: bf16 pairs (64 columns) or, with F8,
// FP8 E4M3 quads (32 columns).  The row sum (of the unrounded fp32 P) goes to
// four packed partial accumulators.  The caller waits for the TMEM stores
// and publishes P.
template <bool F8>
__device__ __forceinline__ void exp_row_to_p(const float (&s)[BN], float scale_log2, float neg_m,
                                             uint64_t (&acc)[4], uint32_t tS) {
    const uint64_t c2 = f2_pack(scale_log2, scale_log2);
    const uint64_t m2 = f2_pack(neg_m, neg_m);
    uint64_t pf_prev = 0;                        // F8: the previous pair of P values
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(s[c * 32 + 2 * i], s[c * 32 + 2 * i + 1]), c2, m2), x0, x1);
            const float p0 = ex2(x0);
            const float p1 = ex2(x1);
            acc[i & 3] = f2_add(acc[i & 3], f2_pack(p0, p1));
            if constexpr (F8) {
                // keys 2i-2 .. 2i+1 go into word i/2 once both pairs exist
                if (i & 1) {
                    float q0, q1;
                    f2_unpack(pf_prev, q0, q1);
                    pk[i / 2] = pack_e4m3x4(q0, q1, p0, p1);
                } else {
                    pf_prev = f2_pack(p0, p1);
                }
            } else {
                pk[i] = pack_bf16x2(p0, p1);
            }
        }
        if constexpr (F8)
            tmem_st8(tS + c * 8, pk);            // P (FP8) over S columns [0, 32)
        else
            tmem_st16(tS + c * 16, pk);          // P (bf16) over S columns [0, 64)
    }
}

// One K/V tile of the online softmax for the row held in s[] (the thread's
// TMEM lane): mask (keys past N_k on the last tile; causal keys past the row's
// limit on tiles that cross the sub-tile's first limit), row max, lazy rescale
// of the reference m and of O in TMEM, P into TMEM over S, publication of P on
// p_bar, then the row sums.  a: the sub-tile's first row; row: this thread's
// row.
template <int D, bool F8, typename PreP>
__device__ __forceinline__ bool softmax_tile(float (&s)[BN], int j, int nkb, int Nk, int causal,
                                             int a, int row, int koff, float scale_log2, float& m,
                                             float& l, float& lc, uint32_t tP, uint32_t tO,
                                             uint32_t p_bar, PreP&& pre_p) {
    // Mask: keys beyond N_k on the last tile; causal: keys past
    // the row's limit on the tiles that cross the sub-tile's
    // first limit (the diagonal).
    const bool tail = (j == nkb - 1) && (Nk % BN != 0);
    const bool diag = causal && (j * BN + BN - 1 > a + koff);
    if (tail || diag) {
        const int lim_tail = Nk - j * BN;          // key c allowed iff c < lim_tail
        const int lim_diag = row + koff - j * BN;  // key c allowed iff c <= lim_diag
#pragma unroll
        for (int c = 0; c < BN; ++c) {
            const bool bad = (c >= lim_tail) || (causal && c > lim_diag);
            s[c] = bad ? -INFINITY : s[c];
        }
    }
    // Row max: eight chains of three-input max (chain i takes
    // columns i, i+8, ..., i+120; one instruction folds two
    // columns), then a tree.
    float mx8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mx8[i] = fmax3(s[i], s[8 + i], s[16 + i]);
#pragma unroll
    for (int c = 24; c < BN - 8; c += 16) {
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = fmax3(mx8[i], s[c + i], s[c + 8 + i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) mx8[i] = fmaxf(mx8[i], s[BN - 8 + i]);
    const float s_top = fmaxf(fmax3(fmax3(mx8[0], mx8[1], mx8[2]),
                                    fmax3(mx8[3], mx8[4], mx8[5]), mx8[6]),
                              mx8[7]);
    const float m_blk = s_top * scale_log2;
    // With P in its own columns, the previous tile's P V may still be running:
    // pre_p waits for it before O is rescaled or P overwritten.
    if (!pre_p()) return false;
    // Lazy rescale: the reference m (that l and O refer to) moves
    // to the row's new maximum only when some row of the warp
    // exceeds it by more than rescale_log2 (first tile: m = -inf,
    // so every lane moves).  O is then rescaled in TMEM: the P V
    // of tile j-1 is complete (P over S: its commit preceded the
    // S_t commit waited on by the caller; P apart: pre_p waited).
    if (__any_sync(0xffffffffu, m_blk > m + rescale_log2<F8>())) {
        const float m_new = fmaxf(m, m_blk);
        const float alpha = ex2(m - m_new);      // 0 on the first tile
        if (j > 0) {
            // 16 columns at a time: with the score row live, wider chunks
            // push the softmax warps past their register budget (spills).
#pragma unroll
            for (int c = 0; c < D / 16; ++c) {
                uint32_t r[16];
                tmem_ld16(tO + c * 16, r);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                tmem_st16(tO + c * 16, r);
            }
        }
        l *= alpha;
        lc *= alpha;
        m = m_new;
    }
    uint64_t acc[4] = {0, 0, 0, 0};              // four packed (0.f, 0.f)
    exp_row_to_p<F8>(s, scale_log2, -m, acc, tP);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(p_bar);
    // The P V product takes P rounded to its operand type, while
    // l sums the unrounded P.  O is normalised by l + lc, lc
    // holding the rounding error of each tile's largest P: with a
    // stale reference m that P is not a power of two, and when it
    // dominates the row (peaked attention) its rounding then
    // cancels between O's numerator and normaliser.  The LSE
    // keeps the unrounded l.
    {
        const float p_top = ex2(fmaf(s_top, scale_log2, -m));
        lc += round_as_p<F8>(p_top) - p_top;
    }
    {
        float a0, a1, a2, a3, a4, a5, a6, a7;
        f2_unpack(acc[0], a0, a1);
        f2_unpack(acc[1], a2, a3);
        f2_unpack(acc[2], a4, a5);
        f2_unpack(acc[3], a6, a7);
        l += ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
    }
    return true;
}

// Epilogue of one row: O / (l + lc) -> bf16 -> the row of o_head (element
// stride o_sn between rows), LSE = (m + log2 l) ln 2 -> lse_head[row]; rows
// at or past N_q are not stored.  o_scale multiplies O (FP8: V's scale).
template <int D, bool F8>
__device__ __forceinline__ void store_o_row(uint32_t tO, __nv_bfloat16* o_head, float* lse_head,
                                            int row, int Nq, long long o_sn, float m, float l,
                                            float lc, float o_scale) {
    float inv_l = 1.f / (l + lc);
    if constexpr (F8) inv_l *= o_scale;
    const bool store = row < Nq;
    __nv_bfloat16* orow = o_head + (long long)(store ? row : 0) * o_sn;
    uint32_t ro[D];
    if constexpr (D == 128) {
        tmem_ld128(tO, ro);
    } else {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) ro[c * 32 + i] = r[i];
        }
    }
    if (store) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
        for (int v4 = 0; v4 < D / 8; ++v4) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                pk[i] = pack_bf16x2(__uint_as_float(ro[8 * v4 + 2 * i]) * inv_l,
                                    __uint_as_float(ro[8 * v4 + 2 * i + 1]) * inv_l);
            dst[v4] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        lse_head[row] = (m + log2f(l)) * 0.69314718055994530942f;
    }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
// F8: Q, K and V^T are E4M3 (tmV then maps V^T, d rows x keys); scale_log2
// includes the Q and K dequantisation scales and o_scale (V's scale)
// multiplies O in the epilogue.  Unused (1) in the bf16 kernel.
template <int D, int NS, bool F8 = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, __nv_bfloat16* __restrict__ Og,
                  float* __restrict__ LSEg, int BH, int H, int Nq, int Nk, int causal,
                  float scale_log2,
                  int hg, int paired, long long o_sb, long long o_sh, long long o_sn,
                  int* __restrict__ sched,
                  unsigned long long watchdog_ns, int inject, float o_scale) {
    using L = Layout<D, NS, F8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t sQ = sbase + L::OFF_Q;
    const uint32_t sKV = sbase + L::OFF_KV;
    const uint32_t sBar = sbase + L::OFF_BAR;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    // Always 0: the abort flag of the drain waits, which must not be cut
    // short by the CTA's own abort.
    volatile int* zero_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8);
    volatile int* unit_slot = reinterpret_cast<volatile int*>(smem + L::OFF_UNIT);
    auto bar = [&](int i) { return sBar + 8u * uint32_t(i); };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nq2 = (Nq + UNIT_ROWS - 1) / UNIT_ROWS;
    const int num_units = nq2 * BH;
    const int nkb = (Nk + BN - 1) / BN;
    const int koff = Nk - Nq;                  // causal: key j allowed for row i iff j <= i + koff
    const Watchdog wd_in{abort_flag, watchdog_ns};
    // Unit queue.  Static schedule (sched == nullptr): every role walks the
    // same assignment (static_unit), skipping the same empty entries.
    // Dynamic schedule: the producer claims sequence indices from the global
    // counter *sched and publishes their unit ids in two shared-memory slots
    // (full: producer; empty: MMA thread and every softmax thread); -1 ends
    // the CTA's work.
    auto next_static = [&](int& kq) -> int {
        int u;
        while ((u = static_unit(kq, blockIdx.x, gridDim.x, BH, nq2, causal, hg, paired)) ==
               UNIT_SKIP)
            ++kq;
        return u;
    };
    auto next_unit_consumer = [&](int& kq, bool& ok_out, uint32_t role) -> int {
        if (!sched) return next_static(kq);
        const int slot = kq & 1;
        bool got = wait_phase(bar(L::B_UFULL + slot), uint32_t(kq >> 1) & 1u, wd_in, role, 0);
        if (role == ROLE_SOFTMAX) got = __all_sync(0xffffffffu, got);
        if (!got) {
            ok_out = false;
            return -1;
        }
        const int u = unit_slot[slot];
        mbar_arrive(bar(L::B_UEMPTY + slot));
        return u;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(L::B_KV_FULL + s), 1);
            mbar_init(bar(L::B_KV_EMPTY + s), 1);
        }
        mbar_init(bar(L::B_Q_FULL), 1);
        mbar_init(bar(L::B_Q_EMPTY), 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(L::B_S_FULL + t), 1);
            mbar_init(bar(L::B_P_FULL + t), BM);
            mbar_init(bar(L::B_O_FULL + t), 1);
            mbar_init(bar(L::B_O_EMPTY + t), BM);
            mbar_init(bar(L::B_S_FREE + t), BM);
            mbar_init(bar(L::B_PV_DONE + t), 1);
        }
        mbar_init(bar(L::B_DRAIN), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(L::B_UFULL + i), 1);
            mbar_init(bar(L::B_UEMPTY + i), 1 + 2 * BM);   // MMA thread + softmax threads
        }
        *abort_flag = 0;
        *zero_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == MMA_WARP) {
        tmem_alloc(smem_addr(tmem_slot), L::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Watchdog wd{abort_flag, watchdog_ns};

    // Each role's code sits inside the branch that set its register budget,
    // so ptxas allocates it against that budget.
    if (warp >= 8) {
    regs_dec<Regs<D, F8>::OTHER>();
    if (warp >= 10) {
        // idle warps of the third warpgroup
    } else if (warp == TMA_WARP) {
        // ------------------------------------------------------------------
        // Producer: Q_0/Q_1 per unit, then K_0, V_0, K_1, V_1, ... through
        // the ring.  fills counts ring loads over the CTA's lifetime.
        // ------------------------------------------------------------------
        if (lane == 0) {
            uint32_t fills = 0, units = 0, q_issued = 0;
            bool ok = true;
            bool skipped = false;           // fault injection: fill 0 was never issued
            for (int kq = 0; ok; ++kq, ++units) {
                int u;
                if (sched) {
                    // claim the next unit and publish it to the other roles
                    const int slot = kq & 1;
                    if (!wait_phase(bar(L::B_UEMPTY + slot), (uint32_t(kq >> 1) & 1u) ^ 1u, wd,
                                    ROLE_PRODUCER, 0)) {
                        ok = false;
                        break;
                    }
                    u = atomicAdd(sched, 1);
                    u = u < num_units ? seq_to_unit(u, BH, nq2, causal, hg) : UNIT_END;
                    unit_slot[slot] = u;
                    mbar_arrive(bar(L::B_UFULL + slot));
                } else {
                    u = next_static(kq);
                }
                if (u < 0) break;
                const Unit w = decode_unit(u, Nq, Nk, causal);
                const int wb = w.bh / H, wh = w.bh - (w.bh / H) * H;   // batch, head
                if (!wait_phase(bar(L::B_Q_EMPTY), (units & 1u) ^ 1u, wd, ROLE_PRODUCER, u)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(bar(L::B_Q_FULL), 2 * L::Q_BYTES);
                for (int t = 0; t < 2; ++t)
                    for (int h = 0; h < L::SLABS; ++h)
                        tma_load_4d(sQ + t * L::Q_BYTES + h * L::HALF_BYTES, &tmQ,
                                    h * L::SLAB_ELEMS, w.r0 + t * BM, wh, wb, bar(L::B_Q_FULL));
                ++q_issued;
                for (int j = 0; j < w.nb1 && ok; ++j) {
                    for (int kind = 0; kind < 2; ++kind) {
                        const uint32_t s = fills % NS;
                        const uint32_t ph = (fills / NS) & 1u;
                        if (!wait_phase(bar(L::B_KV_EMPTY + s), ph ^ 1u, wd, ROLE_PRODUCER, u)) {
                            ok = false;
                            break;
                        }
                        const bool skip = inject == 1 && !skipped && blockIdx.x == 0;
                        if (skip) {
                            skipped = true;  // fault injection: this copy is never issued
                        } else {
                            mbar_arrive_expect_tx(bar(L::B_KV_FULL + s), L::KV_BYTES);
                            if (F8 && kind == 1) {
                                // V^T tile: all d rows, keys j*BN .. j*BN+127
                                tma_load_4d(sKV + s * L::KV_BYTES, &tmV, j * BN, 0, wh, wb,
                                            bar(L::B_KV_FULL + s));
                            } else {
                                const CUtensorMap* map = kind == 0 ? &tmK : &tmV;
                                for (int h = 0; h < L::SLABS; ++h)
                                    tma_load_4d(sKV + s * L::KV_BYTES + h * L::HALF_BYTES, map,
                                                h * L::SLAB_ELEMS, j * BN, wh, wb,
                                                bar(L::B_KV_FULL + s));
                            }
                        }
                        ++fills;
                    }
                }
            }
            if (!ok) {
                // Drain: wait (bounded) for every copy this thread issued:
                // the last fill of each stage, f = fills-1-((fills-1-s) mod NS).
                const Watchdog dwd{zero_flag, wd.limit_ns};
                for (uint32_t s = 0; s < NS; ++s) {
                    if (fills <= s) continue;
                    const uint32_t f = fills - 1 - ((fills - 1 - s) % NS);
                    if (skipped && f == 0) continue;
                    wait_phase(bar(L::B_KV_FULL + s), (f / NS) & 1u, dwd, ROLE_DRAIN, 0);
                }
                if (q_issued > 0)
                    wait_phase(bar(L::B_Q_FULL), (q_issued - 1) & 1u, dwd, ROLE_DRAIN, 0);
            }
        }
        __syncwarp();
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------------
        // MMA issuer.  Per unit: S_0 = Q_0 K_0^T, S_1 = Q_1 K_0^T; then per
        // K/V tile j: O_0 += P_0 V_j, S_0 = Q_0 K_{j+1}^T, O_1 += P_1 V_j,
        // S_1 = Q_1 K_{j+1}^T.  tcgen05 MMAs from one thread execute in
        // issue order, so P_t (aliasing S_t) is consumed before the next S_t
        // overwrites it, and a commit after S_t also covers the PV before it.
        // ------------------------------------------------------------------
        if (lane == 0) {
            constexpr uint32_t ID_S = F8 ? idesc_e4m3(BM, BN) : idesc_bf16(BM, BN, false);
            constexpr uint32_t ID_PV = F8 ? idesc_e4m3(BM, D) : idesc_bf16(BM, D, true);
            uint32_t cons = 0, units = 0, pcnt0 = 0, pcnt1 = 0;
            bool ok = true;
            bool issued = false;
            // Descriptors, built once: Q sub-tiles and ring stages (K-major
            // view for K, MN-major view for V: leading byte offset = the
            // 16 KiB between d slabs, stride byte offset = 8 rows x 128 B).
            const uint64_t dq0 = L::SW64 ? sdesc_sw64(sQ) : sdesc_sw128(sQ, 16, 1024);
            const uint64_t dq1 = L::SW64 ? sdesc_sw64(sQ + L::Q_BYTES)
                                         : sdesc_sw128(sQ + L::Q_BYTES, 16, 1024);
            const uint64_t dk0 = L::SW64 ? sdesc_sw64(sKV) : sdesc_sw128(sKV, 16, 1024);
            const uint64_t dv0 = F8 ? sdesc_sw128(sKV, 16, 1024)     // V^T: K-major
                                    : sdesc_sw128(sKV, L::HALF_BYTES, 1024);
            const uint32_t stage_step = uint32_t(L::KV_BYTES >> 4);
            const uint32_t tS0 = tmem + L::TM_S0, tS1 = tmem + L::TM_S1;
            const uint32_t tO0 = tmem + L::TM_O0, tO1 = tmem + L::TM_O1;
            // O_t += P_t V for one tile once the softmax warpgroup has
            // published P_t.
            auto pv = [&](int t, uint32_t pcnt, uint32_t tO, uint32_t tS, uint64_t v_desc,
                          bool first, int u) -> bool {
                if (!wait_phase(bar(L::B_P_FULL + t), pcnt & 1u, wd, ROLE_MMA, u)) return false;
                tc_fence_after();
                issue_pv<F8>(tO, tS, v_desc, ID_PV, first);
                return true;
            };
            if constexpr (L::SEP_P) {
            // P apart from S: per K/V tile j, S_0(j+1) and S_1(j+1) go out as
            // soon as each softmax warpgroup has read S_t(j) (S_FREE), ahead
            // of O_0 += P_0 V_j and O_1 += P_1 V_j; each P V is committed to
            // PV_DONE_t, which the softmax waits for before it writes the
            // next P_t or rescales O_t.  K_{j+1} is used before V_j: both
            // stages are found from the fill count (K_j, V_j, K_{j+1}, ...).
            const uint32_t tP0 = tmem + L::TM_P0, tP1 = tmem + L::TM_P1;
            uint32_t sc0 = 0, sc1 = 0;              // S_t issued over the CTA's lifetime
            auto issue_s = [&](int t, uint32_t& sc, uint32_t sK, int u) -> bool {
                if (sc > 0 &&
                    !wait_phase(bar(L::B_S_FREE + t), (sc - 1) & 1u, wd, ROLE_MMA, u))
                    return false;
                tc_fence_after();
                issue_qk<L::QK_STEPS, L::HALF_BYTES, F8>(t ? tS1 : tS0, t ? dq1 : dq0,
                                                         desc_add(dk0, sK * stage_step), ID_S);
                tc_commit(bar(L::B_S_FULL + t));
                ++sc;
                return true;
            };
            for (int kq = 0; ok; ++kq, ++units) {
                const int u = next_unit_consumer(kq, ok, ROLE_MMA);
                if (u < 0) break;
                const Unit w = decode_unit(u, Nq, Nk, causal);
                if (!wait_phase(bar(L::B_Q_FULL), units & 1u, wd, ROLE_MMA, u)) { ok = false; break; }
                const uint32_t sK0 = cons % NS;
                if (!wait_phase(bar(L::B_KV_FULL + sK0), (cons / NS) & 1u, wd, ROLE_MMA, u)) {
                    ok = false;
                    break;
                }
                ++cons;
                if (!issue_s(0, sc0, sK0, u) || !issue_s(1, sc1, sK0, u)) { ok = false; break; }
                tc_commit(bar(L::B_KV_EMPTY + sK0));
                issued = true;
                if (w.nb1 == 1) tc_commit(bar(L::B_Q_EMPTY));
                for (int j = 0; j < w.nb1; ++j) {
                    const bool next = j + 1 < w.nb1;
                    const uint32_t cV = cons, cK = cons + 1;
                    cons += next ? 2u : 1u;
                    if (next) {
                        const uint32_t sK = cK % NS;
                        if (!wait_phase(bar(L::B_KV_FULL + sK), (cK / NS) & 1u, wd, ROLE_MMA, u)) {
                            ok = false;
                            break;
                        }
                        if (j + 1 < w.nb0 && !issue_s(0, sc0, sK, u)) { ok = false; break; }
                        if (!issue_s(1, sc1, sK, u)) { ok = false; break; }
                        tc_commit(bar(L::B_KV_EMPTY + sK));
                        if (j + 1 == w.nb1 - 1) tc_commit(bar(L::B_Q_EMPTY));
                    }
                    const uint32_t sV = cV % NS;
                    if (!wait_phase(bar(L::B_KV_FULL + sV), (cV / NS) & 1u, wd, ROLE_MMA, u)) {
                        ok = false;
                        break;
                    }
                    if (j < w.nb0) {
                        if (j == 0 && !wait_phase(bar(L::B_O_EMPTY + 0), (units & 1u) ^ 1u, wd,
                                                  ROLE_MMA, u)) {
                            ok = false;
                            break;
                        }
                        if (!pv(0, pcnt0, tO0, tP0, desc_add(dv0, sV * stage_step), j == 0, u)) {
                            ok = false;
                            break;
                        }
                        ++pcnt0;
                        tc_commit(bar(L::B_PV_DONE + 0));
                        if (j == w.nb0 - 1) tc_commit(bar(L::B_O_FULL + 0));
                    }
                    if (j == 0 && !wait_phase(bar(L::B_O_EMPTY + 1), (units & 1u) ^ 1u, wd,
                                              ROLE_MMA, u)) {
                        ok = false;
                        break;
                    }
                    if (!pv(1, pcnt1, tO1, tP1, desc_add(dv0, sV * stage_step), j == 0, u)) {
                        ok = false;
                        break;
                    }
                    ++pcnt1;
                    tc_commit(bar(L::B_PV_DONE + 1));
                    tc_commit(bar(L::B_KV_EMPTY + sV));
                    if (j == w.nb1 - 1) tc_commit(bar(L::B_O_FULL + 1));
                }
            }
            } else {
            for (int kq = 0; ok; ++kq, ++units) {
                const int u = next_unit_consumer(kq, ok, ROLE_MMA);
                if (u < 0) break;
                const Unit w = decode_unit(u, Nq, Nk, causal);
                if (!wait_phase(bar(L::B_Q_FULL), units & 1u, wd, ROLE_MMA, u)) { ok = false; break; }
                uint32_t sK = cons % NS;
                if (!wait_phase(bar(L::B_KV_FULL + sK), (cons / NS) & 1u, wd, ROLE_MMA, u)) {
                    ok = false;
                    break;
                }
                ++cons;
                issue_qk<L::QK_STEPS, L::HALF_BYTES, F8>(tS0, dq0, desc_add(dk0, sK * stage_step), ID_S);
                tc_commit(bar(L::B_S_FULL + 0));
                issue_qk<L::QK_STEPS, L::HALF_BYTES, F8>(tS1, dq1, desc_add(dk0, sK * stage_step), ID_S);
                tc_commit(bar(L::B_S_FULL + 1));
                tc_commit(bar(L::B_KV_EMPTY + sK));
                issued = true;
                if (w.nb1 == 1) tc_commit(bar(L::B_Q_EMPTY));
                for (int j = 0; j < w.nb1; ++j) {
                    const uint32_t sV = cons % NS;
                    if (!wait_phase(bar(L::B_KV_FULL + sV), (cons / NS) & 1u, wd, ROLE_MMA, u)) {
                        ok = false;
                        break;
                    }
                    ++cons;
                    const bool next = j + 1 < w.nb1;
                    // K_{j+1} is waited for only when the first S of tile
                    // j+1 is issued, after P V of tile j.
                    bool have_k = false;
                    auto wait_next_k = [&]() -> bool {
                        if (have_k) return true;
                        sK = cons % NS;
                        if (!wait_phase(bar(L::B_KV_FULL + sK), (cons / NS) & 1u, wd, ROLE_MMA, u))
                            return false;
                        ++cons;
                        have_k = true;
                        return true;
                    };
                    if (j < w.nb0) {
                        if (j == 0 && !wait_phase(bar(L::B_O_EMPTY + 0), (units & 1u) ^ 1u, wd,
                                                  ROLE_MMA, u)) {
                            ok = false;
                            break;
                        }
                        if (!pv(0, pcnt0, tO0, tS0, desc_add(dv0, sV * stage_step), j == 0, u)) {
                            ok = false;
                            break;
                        }
                        ++pcnt0;
                        if (j + 1 < w.nb0) {
                            if (!wait_next_k()) {
                                ok = false;
                                break;
                            }
                            issue_qk<L::QK_STEPS, L::HALF_BYTES, F8>(tS0, dq0, desc_add(dk0, sK * stage_step), ID_S);
                            tc_commit(bar(L::B_S_FULL + 0));
                        }
                        if (j == w.nb0 - 1) tc_commit(bar(L::B_O_FULL + 0));
                    }
                    if (j == 0 && !wait_phase(bar(L::B_O_EMPTY + 1), (units & 1u) ^ 1u, wd, ROLE_MMA, u)) {
                        ok = false;
                        break;
                    }
                    if (!pv(1, pcnt1, tO1, tS1, desc_add(dv0, sV * stage_step), j == 0, u)) {
                        ok = false;
                        break;
                    }
                    ++pcnt1;
                    // V_j is free once both P V products have read it: its
                    // stage is released before S_1(j+1) is queued, so the
                    // producer refills it one QK^T group earlier.
                    tc_commit(bar(L::B_KV_EMPTY + sV));
                    if (next) {
                        if (!wait_next_k()) {
                            ok = false;
                            break;
                        }
                        issue_qk<L::QK_STEPS, L::HALF_BYTES, F8>(tS1, dq1, desc_add(dk0, sK * stage_step), ID_S);
                        tc_commit(bar(L::B_S_FULL + 1));
                    }
                    if (next) tc_commit(bar(L::B_KV_EMPTY + sK));
                    if (next && j + 1 == w.nb1 - 1) tc_commit(bar(L::B_Q_EMPTY));
                    if (j == w.nb1 - 1) tc_commit(bar(L::B_O_FULL + 1));
                }
            }
            }
            if (issued) {
                // Every MMA this thread issued must finish before TMEM is
                // freed; on the normal path the softmax warps have already
                // waited for the last O commit, so this returns at once.
                const Watchdog dwd{zero_flag, wd.limit_ns};
                tc_commit(bar(L::B_DRAIN));
                wait_phase(bar(L::B_DRAIN), 0, dwd, ROLE_DRAIN, 0);
            }
        }
        __syncwarp();
    }
    // Teardown of warpgroup 2: after every thread of the CTA is done with
    // TMEM, the allocating warp frees it.
    tc_fence_before();
    cta_sync();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TM_COLS);
    }
    } else {
        // ------------------------------------------------------------------
        // Softmax warpgroups.  Thread = query row; TMEM lane = row.
        // ------------------------------------------------------------------
        regs_inc<Regs<D, F8>::SOFTMAX>();
        const int t = warp >> 2;                     // sub-tile 0 or 1
        const int wr = (warp & 3) * 32 + lane;       // row within the sub-tile
        const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + (t == 0 ? L::TM_S0 : L::TM_S1);
        const uint32_t tP = tmem + lane_base + (t == 0 ? L::TM_P0 : L::TM_P1);
        const uint32_t tO = tmem + lane_base + (t == 0 ? L::TM_O0 : L::TM_O1);
        uint32_t scnt = 0, ocnt = 0;
        bool ok = true;
        for (int kq = 0; ok; ++kq) {
            const int u = next_unit_consumer(kq, ok, ROLE_SOFTMAX);
            if (u < 0) break;
            const Unit w = decode_unit(u, Nq, Nk, causal);
            const int a = w.r0 + t * BM;             // first row of this sub-tile
            const int row = a + wr;
            const int nb = t == 0 ? w.nb0 : w.nb1;
            float m = -INFINITY;                     // running max, log2 units
            float l = 0.f;                           // running sum of exponentials
            float lc = 0.f;                          // rounding correction of l for O
            for (int j = 0; j < nb; ++j) {
                const uint32_t k = scnt;             // this sub-tile's tile count so far
                bool got = wait_phase(bar(L::B_S_FULL + t), scnt & 1u, wd, ROLE_SOFTMAX, u);
                ++scnt;
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                tc_fence_after();
                float s[BN];
                {
                    uint32_t r[BN];
                    tmem_ld128(tS, r);
#pragma unroll
                    for (int c = 0; c < BN; ++c) s[c] = __uint_as_float(r[c]);
                }
                if constexpr (L::SEP_P) {
                    // S_t is in registers: the MMA thread may overwrite it
                    tc_fence_before();
                    mbar_arrive(bar(L::B_S_FREE + t));
                }
                auto pre_p = [&]() -> bool {
                    if constexpr (L::SEP_P) {
                        if (k == 0) return true;
                        const bool done = wait_phase(bar(L::B_PV_DONE + t), (k - 1) & 1u, wd,
                                                     ROLE_SOFTMAX, u);
                        if (!__all_sync(0xffffffffu, done)) return false;
                        tc_fence_after();
                    }
                    return true;
                };
                if (!softmax_tile<D, F8>(s, j, nkb, Nk, causal, a, row, koff, scale_log2, m, l, lc,
                                         tP, tO, bar(L::B_P_FULL + t), pre_p)) {
                    ok = false;
                    break;
                }
            }
            if (!ok) break;
            // Epilogue: O / l -> bf16 -> global; LSE.
            bool got = wait_phase(bar(L::B_O_FULL + t), ocnt & 1u, wd, ROLE_SOFTMAX, u);
            ++ocnt;
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            const int wb = w.bh / H, wh = w.bh - (w.bh / H) * H;     // batch, head
            store_o_row<D, F8>(tO, Og + wb * o_sb + wh * o_sh, LSEg + size_t(w.bh) * Nq, row, Nq,
                               o_sn, m, l, lc, o_scale);
            tc_fence_before();
            mbar_arrive(bar(L::B_O_EMPTY + t));
        }
        tc_fence_before();
        cta_sync();
    }
    // The two branches meet only at kernel exit: no code runs after them,
    // so neither warpgroup has to give its register budget back.
}

}  // namespace fa

// ===========================================================================
// Host side: validation, tensor maps, launch.
// ===========================================================================
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

thread_local int t_last_cuda_error = 0;

}  // namespace

void fa_internal::set_last_cuda_error(int e) { t_last_cuda_error = e; }

namespace {

constexpr int MAX_DEVICES = 64;
struct DeviceInfo {
    std::once_flag once;
    int ok = 0;
    int sm_count = 0;
    int cc_major = 0, cc_minor = 0;
};
DeviceInfo g_dev[MAX_DEVICES];
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

template <int D, int NS, bool F8>
struct Instance {
    static std::once_flag once[MAX_DEVICES];
    static cudaError_t attr_err[MAX_DEVICES];
    static int regs[MAX_DEVICES];
};
template <int D, int NS, bool F8>
std::once_flag Instance<D, NS, F8>::once[MAX_DEVICES];
template <int D, int NS, bool F8>
cudaError_t Instance<D, NS, F8>::attr_err[MAX_DEVICES];
template <int D, int NS, bool F8>
int Instance<D, NS, F8>::regs[MAX_DEVICES];

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Element strides (batch, head, sequence) of one bf16 [B][H][N][d] operand;
// the head dimension is always contiguous.
struct Strides3 {
    long long b, h, n;
};

// 4-D tensor map (d, N, H, B) with a (64, 128, 1, 1) box and 128-byte swizzle.
fa_status encode_map(CUtensorMap* map, const void* base, int d, int N, int H, int B,
                     const Strides3& st, int box_rows = fa::BM) {
    const cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(H), cuuint64_t(B)};
    const cuuint64_t strides[3] = {cuuint64_t(st.n) * 2, cuuint64_t(st.h) * 2, cuuint64_t(st.b) * 2};
    const cuuint32_t box[4] = {cuuint32_t(fa::SW_COLS), cuuint32_t(box_rows), 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_UNSUPPORTED;
}

}  // namespace

int fa_internal::current_device(int* dev_out, int* sm_count) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
        t_last_cuda_error = int(e);
        return FA_ERR_NO_DEVICE;
    }
    DeviceInfo& di = g_dev[dev];
    std::call_once(di.once, [&] {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return;
        di.sm_count = prop.multiProcessorCount;
        di.cc_major = prop.major;
        di.cc_minor = prop.minor;
        di.ok = 1;
    });
    if (!di.ok) return FA_ERR_NO_DEVICE;
    if (di.cc_major != 10 || di.cc_minor != 0) return FA_ERR_UNSUPPORTED;
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    if (!g_encode) return FA_ERR_NO_DEVICE;
    *dev_out = dev;
    *sm_count = di.sm_count;
    return FA_OK;
}

int fa_internal::encode_bhnd_map(CUtensorMap* map, const void* base, int d, int N, int H, int B,
                                 long long sb, long long sh, long long sn, int box_rows) {
    return encode_map(map, base, d, N, H, B, Strides3{sb, sh, sn}, box_rows);
}

namespace {

// Static schedule choice: the assignment (snake or paired, see static_unit)
// and the heads per group.  Small groups keep the K/V that concurrently
// running CTAs stream resident in L2; with the snake, large groups balance
// the CTAs better, while the paired assignment balances long causal
// problems at any group size once every CTA holds several pairs.  This
// replays the kernel's assignment on the host for both assignments and
// hg = 1, 2, 4, ..., BH (K/V tiles per unit plus a fixed per-unit overhead
// as the cost) and takes the lowest (max CTA load / mean CTA load) x
// (1 + L2 penalty), the penalty growing with the group's K/V bytes: 0 up to
// 16 MiB, then 3 %, 6 %, 9 % and 12 % past 16, 32, 64 and 128 MiB
// (calibrated on the 8K and 32K causal workloads, where 2-head snake groups
// measured 4-7 % faster than 8- or all-head groups).  Decisions are cached
// per shape.
struct HgKey {
    long long BH;
    int Nq, Nk, D, causal, grid, unit_rows;
    bool operator==(const HgKey& o) const {
        return BH == o.BH && Nq == o.Nq && Nk == o.Nk && D == o.D && causal == o.causal &&
               grid == o.grid && unit_rows == o.unit_rows;
    }
};
struct StaticPlan {
    long long hg;
    int paired;
};
std::mutex g_hg_mutex;
HgKey g_hg_keys[64];
StaticPlan g_hg_vals[64];
int g_hg_count = 0;

// Max CTA load over mean CTA load of the static assignment, replayed.
double static_imbalance(long long BH, int Nq, int Nk, int causal, long long hg, int paired,
                        int grid, int unit_rows) {
    const long long nq2 = (Nq + unit_rows - 1) / unit_rows;
    const long long nkb = (Nk + fa::BN - 1) / fa::BN;
    const long long off = Nk - Nq;
    std::vector<long long> load(size_t(grid), 0);
    // K/V tiles of both sub-tiles (the tiles of each half unit's last row)
    // plus a fixed per-unit overhead.
    auto cost = [&](long long qb2) {
        const long long r0 = qb2 * unit_rows;
        const long long half = unit_rows / 2;
        const long long nb0 = causal ? std::min((r0 + half - 1 + off) / fa::BN + 1, nkb) : nkb;
        const long long nb1 = causal ? std::min((r0 + unit_rows - 1 + off) / fa::BN + 1, nkb) : nkb;
        return nb0 + nb1 + 2;
    };
    if (!paired) {
        const long long units = nq2 * BH;
        const long long per_group = hg * nq2;
        for (long long i = 0; i < units; ++i) {
            const long long g = i / per_group;
            const long long r = i - g * per_group;
            const long long gh = std::min(hg, BH - g * hg);
            const long long level = r / gh;
            const long long k = i / grid, c = i - k * grid;
            load[size_t((k & 1) ? (grid - 1 - c) : c)] += cost(causal ? nq2 - 1 - level : level);
        }
    } else {
        // CTA c takes pairs c, c + grid, ... (both units of each pair).
        const long long npl = (nq2 + 1) / 2;
        const long long per_group = hg * npl;
        for (long long p = 0; p < BH * npl; ++p) {
            const long long g = p / per_group;
            const long long r = p - g * per_group;
            const long long gh = std::min(hg, BH - g * hg);
            const long long pl = r / gh;
            const long long q_long = nq2 - 1 - pl;
            load[size_t(p % grid)] += cost(q_long) + (pl == q_long ? 0 : cost(pl));
        }
    }
    long long mx = 0, sum = 0;
    for (long long x : load) {
        mx = std::max(mx, x);
        sum += x;
    }
    return double(mx) * grid / double(sum);
}

StaticPlan choose_static_plan(long long BH, int Nq, int Nk, int D, int causal, int grid,
                              int unit_rows) {
    const HgKey key{BH, Nq, Nk, D, causal, grid, unit_rows};
    {
        std::lock_guard<std::mutex> lk(g_hg_mutex);
        for (int i = 0; i < g_hg_count; ++i)
            if (g_hg_keys[i] == key) return g_hg_vals[i];
    }
    const long long kv_head_bytes = 2LL * Nk * D * 2;
    StaticPlan best{BH, 0};
    double best_cost = 1e30;
    // Bound the replay work for very large problems: beyond ~4M units the
    // assignment statistics no longer depend on hg, so all heads form one group.
    const long long units = ((Nq + unit_rows - 1) / unit_rows) * BH;
    if (units <= (4LL << 20)) {
        for (int paired = 0; paired <= (causal ? 1 : 0); ++paired) {
            for (long long hg = 1;; hg = std::min(hg * 2, BH)) {
                const double ws = double(hg * kv_head_bytes);
                const double pen = ws <= 16.0 * (1 << 20) ? 0.0
                                 : ws <= 32.0 * (1 << 20) ? 0.03
                                 : ws <= 64.0 * (1 << 20) ? 0.06
                                 : ws <= 128.0 * (1 << 20) ? 0.09 : 0.12;
                const double cost =
                    static_imbalance(BH, Nq, Nk, causal, hg, paired, grid, unit_rows) * (1.0 + pen);
                if (cost < best_cost - 1e-9) {
                    best_cost = cost;
                    best = StaticPlan{hg, paired};
                }
                if (hg == BH) break;
            }
        }
    }
    std::lock_guard<std::mutex> lk(g_hg_mutex);
    const int slot = g_hg_count < 64 ? g_hg_count++ : int(BH % 64);
    g_hg_keys[slot] = key;
    g_hg_vals[slot] = best;
    return best;
}

// Launches fa_fwd_kernel<D, NS, F8> on prepared tensor maps: per-device
// attribute setup, head-group choice, dynamic-schedule counter reset.
template <int D, int NS, bool F8>
fa_status launch_kernel(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        void* o, float* lse, int B, int H, int Nq, int Nk, const Strides3& ost,
                        int causal, float scale_log2, float o_scale, int* sched,
                        cudaStream_t stream, int dev, unsigned long long watchdog_ns, int inject) {
    using L = fa::Layout<D, NS, F8>;
    using I = Instance<D, NS, F8>;
    auto kern = fa::fa_fwd_kernel<D, NS, F8>;
    std::call_once(I::once[dev], [&] {
        I::attr_err[dev] =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
        cudaFuncAttributes fa_attr;
        if (I::attr_err[dev] == cudaSuccess && cudaFuncGetAttributes(&fa_attr, kern) == cudaSuccess)
            I::regs[dev] = fa_attr.numRegs;
    });
    if (I::attr_err[dev] != cudaSuccess) {
        t_last_cuda_error = int(I::attr_err[dev]);
        return FA_ERR_LAUNCH;
    }
    // The setmaxnreg split was sized for REGS_LAUNCH registers per thread;
    // with any other launch allocation setmaxnreg.inc could wait forever,
    // so such a build is refused rather than launched.
    if (I::regs[dev] != fa::REGS_LAUNCH) return FA_ERR_UNSUPPORTED;
    const long long BH = (long long)B * H;
    const long long nq2 = (Nq + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS;
    const long long units = nq2 * BH;
    const int grid = int(units < g_dev[dev].sm_count ? units : g_dev[dev].sm_count);
    // Static schedule: group size from the replayed assignment.  Dynamic
    // schedule: CTAs claim units greedily, so balance no longer depends on the
    // group size; groups then hold about 16 MiB of K/V (all heads when the
    // whole K/V fits in 32 MiB).
    const long long kv_head_bytes = 2LL * Nk * D * L::EB;
    StaticPlan plan{BH, 0};
    if (sched)
        plan.hg = (BH * kv_head_bytes <= (32LL << 20)) ? BH : (16LL << 20) / kv_head_bytes;
    else
        plan = choose_static_plan(BH, Nq, Nk, D, causal, grid, fa::UNIT_ROWS);
#ifdef FA_HEAD_GROUP
    plan.hg = FA_HEAD_GROUP;
#endif
#ifdef FA_STATIC_PAIRED
    plan.paired = causal ? FA_STATIC_PAIRED : 0;
#endif
    const long long hg = plan.hg < 1 ? 1 : (plan.hg > BH ? BH : plan.hg);
    if (sched) {
        const cudaError_t me = cudaMemsetAsync(sched, 0, sizeof(int), stream);
        if (me != cudaSuccess) {
            t_last_cuda_error = int(me);
            return FA_ERR_LAUNCH;
        }
    }
    kern<<<grid, fa::NUM_THREADS, L::ALLOC, stream>>>(mq, mk, mv, static_cast<__nv_bfloat16*>(o),
                                                     lse, int(BH), H, Nq, Nk, causal, scale_log2,
                                                     int(hg), plan.paired, ost.b, ost.h, ost.n,
                                                     sched,
                                                     watchdog_ns, inject, o_scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        t_last_cuda_error = int(e);
        return FA_ERR_LAUNCH;
    }
    return FA_OK;
}

template <int D, int NS>
fa_status launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int Nq, int Nk, const Strides3 (&st)[4], int causal, float scale, int* sched,
                 cudaStream_t stream, int dev, unsigned long long watchdog_ns, int inject) {
    CUtensorMap mq, mk, mv;
    if (encode_map(&mq, q, D, Nq, H, B, st[0]) != FA_OK ||
        encode_map(&mk, k, D, Nk, H, B, st[1]) != FA_OK ||
        encode_map(&mv, v, D, Nk, H, B, st[2]) != FA_OK)
        return FA_ERR_UNSUPPORTED;
    const float scale_log2 = scale * 1.4426950408889634f;
    return launch_kernel<D, NS, false>(mq, mk, mv, o, lse, B, H, Nq, Nk, st[3], causal, scale_log2,
                                       1.f, sched, stream, dev, watchdog_ns, inject);
}

// ---------------------------------------------------------------------------
// FP8 forward: V^T pre-pass, E4M3 tensor maps, kernel launch.
// ---------------------------------------------------------------------------
// Ring stages: 16 KiB K or V^T tiles at d = 128 (8 stages), 8 KiB at d = 64 (16).
constexpr int FP8_NS_128 = 8;
constexpr int FP8_NS_64 = 16;

long long fp8_npad(int N) { return ((long long)N + fa::BN - 1) / fa::BN * fa::BN; }

// V [BH][N][D] -> V^T [BH][D][Npad] (keys n >= N zero), one 64-key block of
// one (batch, head) per CTA, through a shared-memory tile.
template <int D>
__global__ void __launch_bounds__(256) transpose_v_e4m3(const uint8_t* __restrict__ v,
                                                        uint8_t* __restrict__ vt, int N,
                                                        long long Npad) {
    __shared__ __align__(16) uint8_t tile[64][D + 16];
    const long long bh = blockIdx.y;
    const int k0 = blockIdx.x * 64;
    const uint8_t* src = v + bh * (long long)N * D;
    for (int i = threadIdx.x; i < 64 * D / 16; i += 256) {
        const int r = i / (D / 16), c = i % (D / 16);
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (k0 + r < N) x = *reinterpret_cast<const uint4*>(src + (long long)(k0 + r) * D + c * 16);
        *reinterpret_cast<uint4*>(&tile[r][c * 16]) = x;
    }
    __syncthreads();
    uint8_t* dst = vt + bh * D * Npad;
    for (int i = threadIdx.x; i < D * 4; i += 256) {
        const int dr = i / 4, kc = i % 4;            // d row, 16-key chunk
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int k = kc * 16 + 4 * q;
            w[q] = uint32_t(tile[k][dr]) | (uint32_t(tile[k + 1][dr]) << 8) |
                   (uint32_t(tile[k + 2][dr]) << 16) | (uint32_t(tile[k + 3][dr]) << 24);
        }
        *reinterpret_cast<uint4*>(dst + (long long)dr * Npad + k0 + kc * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// 4-D E4M3 tensor map (inner, rows, H, B), contiguous, byte strides; box
// (box_inner, box_rows, 1, 1) in 128-byte swizzle, or 64-byte swizzle for a
// 64-byte inner box.
fa_status encode_map_e4m3(CUtensorMap* map, const void* base, long long inner, long long rows,
                          int H, int B, int box_inner, int box_rows) {
    const cuuint64_t dims[4] = {cuuint64_t(inner), cuuint64_t(rows), cuuint64_t(H), cuuint64_t(B)};
    const cuuint64_t strides[3] = {cuuint64_t(inner), cuuint64_t(inner * rows),
                                   cuuint64_t(inner * rows * H)};
    const cuuint32_t box[4] = {cuuint32_t(box_inner), cuuint32_t(box_rows), 1u, 1u};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          box_inner == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_UNSUPPORTED;
}

size_t fp8_workspace_bytes(long long BH, int N, int d) {
    return size_t(FA_DYNAMIC_WORKSPACE_BYTES) + size_t(BH * d * fp8_npad(N));
}

fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int Nq, int Nk, int d, const long long* strides12, int causal, float scale,
                   int* sched, void* stream, unsigned watchdog_ms, int inject) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (causal && Nq > Nk) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (inject != 0 && inject != 1) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if ((long long)B * H > 0x7fffffffLL || Nq > (1 << 30) || Nk > (1 << 30))
        return FA_ERR_UNSUPPORTED;
    // The kernel numbers 256-row units with 32-bit ints (and the dynamic
    // schedule claims up to units + grid indices).
    if (((long long)Nq + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS * B * H > (1LL << 30))
        return FA_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return FA_ERR_MISALIGNED;
    // Strides: q, k, v, o in that order, each (batch, head, sequence) in
    // elements; NULL means contiguous [B][H][N][d] (N = N_q for q and o, N_k
    // for k and v).
    Strides3 st[4];
    for (int i = 0; i < 4; ++i) {
        const int n = (i == 1 || i == 2) ? Nk : Nq;
        if (strides12) {
            st[i] = Strides3{strides12[3 * i], strides12[3 * i + 1], strides12[3 * i + 2]};
        } else {
            st[i] = Strides3{(long long)H * n * d, (long long)n * d, (long long)d};
        }
        // The stride of a dimension of size 1 is never used; frameworks may
        // report any value there, so it is replaced by a valid one.
        if (B == 1) st[i].b = d;
        if (H == 1) st[i].h = d;
        if (n == 1) st[i].n = d;
        const long long v3[3] = {st[i].b, st[i].h, st[i].n};
        for (long long x : v3) {
            if (x < d) return FA_ERR_INVALID_ARG;               // rows may not overlap within a head dim
            if ((x * 2) % 16 != 0) return FA_ERR_MISALIGNED;   // TMA strides are multiples of 16 bytes
            if (x * 2 >= (1LL << 40)) return FA_ERR_UNSUPPORTED;
        }
    }

    int dev = -1, sm_count = 0;
    const fa_status ds = static_cast<fa_status>(fa_internal::current_device(&dev, &sm_count));
    if (ds != FA_OK) return ds;

    const unsigned long long wd_ns = (watchdog_ms ? watchdog_ms : 4000u) * 1000000ull;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d == 64)
        return launch<64, 8>(q, k, v, o, lse, B, H, Nq, Nk, st, causal, scale, sched, s, dev, wd_ns,
                             inject);
    return launch<128, 4>(q, k, v, o, lse, B, H, Nq, Nk, st, causal, scale, sched, s, dev, wd_ns,
                          inject);
}

}  // namespace

int fa_internal::forward_qk(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int H, int Nq, int Nk, int d, int causal, float scale,
                            int* counter, void* stream) {
    return fwd_impl(q, k, v, o, lse, B, H, Nq, Nk, d, nullptr, causal, scale, counter, stream, 0,
                    0);
}

// ===========================================================================
// Allocation-free variant of fa_fwd_dynamic (fa_fwd_dynamic_noalloc).
//
// Some callers cannot allocate device memory at all: a plugin loaded into an
// application that owns every device allocation, or a latency-critical loop
// that must not call cudaMalloc (it can synchronise the whole device).  For
// them the dynamic schedule's work counter lives in this file-scope array
// instead of a caller-provided workspace.  Every device that loads the
// library holds these bytes from module load until the process exits.
// ===========================================================================
namespace fa {
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];
static_assert(FA_DYNAMIC_WORKSPACE_BYTES <= FA_NOALLOC_SCRATCH_BYTES,
              "the dynamic schedule's workspace must fit the static scratch");
}  // namespace fa

namespace {

// Device address of g_noalloc_scratch, resolved once per device.  In host
// code the array's name only stands for the device symbol: it is not a
// device address and must never be handed to a kernel directly.
struct NoallocScratch {
    std::once_flag once;
    cudaError_t err = cudaSuccess;
    void* ptr = nullptr;
};
NoallocScratch g_noalloc[MAX_DEVICES];

}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, int causal, float scale, void* stream) {
    return fwd_impl(q, k, v, o, lse, B, H, N, N, d, nullptr, causal, scale, nullptr, stream, 0, 0);
}

fa_status fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int N, int d, const long long* strides, int causal, float scale,
                         void* stream) {
    if (!strides) return FA_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, o, lse, B, H, N, N, d, strides, causal, scale, nullptr, stream, 0, 0);
}

fa_status fa_fwd_dynamic(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int N, int d, const long long* strides, int causal, float scale,
                         void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace) return FA_ERR_INVALID_ARG;
    if (workspace_bytes < FA_DYNAMIC_WORKSPACE_BYTES) return FA_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return FA_ERR_MISALIGNED;
    return fwd_impl(q, k, v, o, lse, B, H, N, N, d, strides, causal, scale,
                    static_cast<int*>(workspace), stream, 0, 0);
}

fa_status fa_fwd_dynamic_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int B, int H, int N, int d, const long long* strides, int causal,
                                 float scale, void* stream) {
    // The scratch holds one 32-bit counter of claimed units: problems with
    // more units than it may count are refused before anything else.  B*H is
    // bounded first so the unit count cannot overflow.
    if (B >= 1 && H >= 1 && N >= 1) {
        const long long bh = (long long)B * H;
        if (bh > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
        if (((long long)N + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS > FA_NOALLOC_MAX_UNITS / bh)
            return FA_ERR_UNSUPPORTED;
    }
    if (FA_DYNAMIC_WORKSPACE_BYTES > sizeof(fa::g_noalloc_scratch)) return FA_ERR_UNSUPPORTED;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
        t_last_cuda_error = int(e);
        return FA_ERR_NO_DEVICE;
    }
    // Set-up on the first call on this device (the device is current here).
    NoallocScratch& ns = g_noalloc[dev];
    std::call_once(ns.once, [&] { ns.err = cudaGetSymbolAddress(&ns.ptr, fa::g_noalloc_scratch); });
    if (ns.err != cudaSuccess || ns.ptr == nullptr) {
        t_last_cuda_error = int(ns.err);
        return FA_ERR_LAUNCH;
    }
    // Same launch path as fa_fwd_dynamic: the counter is cleared on `stream`
    // before the kernel runs.
    return fwd_impl(q, k, v, o, lse, B, H, N, N, d, strides, causal, scale,
                    static_cast<int*>(ns.ptr), stream, 0, 0);
}

size_t fa_fwd_fp8_workspace_bytes(int B, int H, int N, int d) {
    if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
    if ((long long)B * H > 0x7fffffffLL || N > (1 << 30)) return 0;
    return fp8_workspace_bytes((long long)B * H, N, d);
}

fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, void* o, float* lse, int B,
                     int H, int N, int d, int causal, float scale, float descale_q,
                     float descale_k, float descale_v, void* workspace, size_t workspace_bytes,
                     void* stream) {
    if (!q8 || !k8 || !v8 || !o || !lse || !workspace) return FA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    for (float x : {scale, descale_q, descale_k, descale_v})
        if (!std::isfinite(x) || !(x > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    const long long BH = (long long)B * H;
    if (BH > 0xffffLL || N > (1 << 30)) return FA_ERR_UNSUPPORTED;   // grid.y of the V^T pass
    if (((long long)N + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS * BH > (1LL << 30))
        return FA_ERR_UNSUPPORTED;
    if (workspace_bytes < fp8_workspace_bytes(BH, N, d)) return FA_ERR_INVALID_ARG;
    if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v8, 16) || !aligned(o, 16) ||
        !aligned(lse, 4) || !aligned(workspace, 256))
        return FA_ERR_MISALIGNED;
    int dev = -1, sm_count = 0;
    const fa_status ds = static_cast<fa_status>(fa_internal::current_device(&dev, &sm_count));
    if (ds != FA_OK) return ds;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* sched = static_cast<int*>(workspace);
    uint8_t* vt = static_cast<uint8_t*>(workspace) + FA_DYNAMIC_WORKSPACE_BYTES;
    const long long npad = fp8_npad(N);
    CUtensorMap mq, mk, mv;
    if (encode_map_e4m3(&mq, q8, d, N, H, B, d, fa::BM) != FA_OK ||
        encode_map_e4m3(&mk, k8, d, N, H, B, d, fa::BN) != FA_OK ||
        encode_map_e4m3(&mv, vt, npad, d, H, B, 128, d) != FA_OK)
        return FA_ERR_UNSUPPORTED;
    if (d == 64)
        transpose_v_e4m3<64><<<dim3(unsigned(npad / 64), unsigned(BH)), 256, 0, s>>>(
            static_cast<const uint8_t*>(v8), vt, N, npad);
    else
        transpose_v_e4m3<128><<<dim3(unsigned(npad / 64), unsigned(BH)), 256, 0, s>>>(
            static_cast<const uint8_t*>(v8), vt, N, npad);
    const float scale_log2 = scale * descale_q * descale_k * 1.4426950408889634f;
    const Strides3 ost{(long long)H * N * d, (long long)N * d, (long long)d};
    if (d == 64)
        return launch_kernel<64, FP8_NS_64, true>(mq, mk, mv, o, lse, B, H, N, N, ost, causal,
                                                  scale_log2, descale_v, sched, s, dev,
                                                  4000ull * 1000000ull, 0);
    return launch_kernel<128, FP8_NS_128, true>(mq, mk, mv, o, lse, B, H, N, N, ost, causal,
                                                scale_log2,
                                              descale_v, sched, s, dev, 4000ull * 1000000ull, 0);
}

fa_status fa_fwd_debug(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int N, int d, int causal, float scale, void* stream,
                       unsigned watchdog_ms, int inject) {
    return fwd_impl(q, k, v, o, lse, B, H, N, N, d, nullptr, causal, scale, nullptr, stream,
                    watchdog_ms, inject);
}

fa_status fa_get_device_status(void* stream, unsigned* detail) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned word = 0;
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&word, fa::g_fa_status, sizeof(word));
    const unsigned zero = 0;
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(fa::g_fa_status, &zero, sizeof(zero));
    unsigned bwd_word = 0;
    if (e == cudaSuccess) e = static_cast<cudaError_t>(fa_internal::take_bwd_status(&bwd_word));
    if (word == 0) word = bwd_word;
    if (e != cudaSuccess) {
        t_last_cuda_error = int(e);
        return e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver ? FA_ERR_NO_DEVICE
                                                                           : FA_ERR_LAUNCH;
    }
    if (detail) *detail = word;
    if (word == 0) return FA_OK;
    // The top byte holds the status the kernel recorded.
    const unsigned code = word >> 24;
    return code == unsigned(FA_ERR_LAUNCH) ? FA_ERR_LAUNCH : FA_ERR_TIMEOUT;
}

const char* fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "FA_OK";
        case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
        case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED";
        case FA_ERR_LAUNCH: return "FA_ERR_LAUNCH";
        case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
        case FA_ERR_NO_DEVICE: return "FA_ERR_NO_DEVICE";
        default: return "FA_ERR_UNKNOWN";
    }
}

int fa_last_cuda_error(void) { return t_last_cuda_error; }

int fa_version(void) { return 100; }

}  // extern "C"
