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
// setmaxnreg (REGS_SOFTMAX / REGS_OTHER below).
// Each softmax thread owns one query row (TMEM lane == row), so the row max
// and row sum are in-thread.  S_t (fp32, 128 columns) and O_t (fp32, d
// columns) live in TMEM; P_t is written back as bf16 over the first 64
// columns of S_t and read from TMEM by the PV MMA.  The two warpgroups
// alternate with the single MMA issuer, so the tensor core works on one
// sub-tile while the other sub-tile's exponentials run.
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
// Warpgroup 2 drops to REGS_OTHER once at the start and never rises again;
// warpgroups 0 and 1 rise to REGS_SOFTMAX.  The sum must not exceed the
// launch total or setmaxnreg.inc never returns.
constexpr int REGS_LAUNCH = 168;
constexpr int REGS_SOFTMAX = 208;
constexpr int REGS_OTHER = 80;
static_assert(2 * 128 * REGS_SOFTMAX + 128 * REGS_OTHER <= NUM_THREADS * REGS_LAUNCH,
              "register split exceeds the launch allocation");
constexpr int SW_COLS = 64;        // bf16 elements per 128-byte swizzled row
// Lazy rescale: the running max that l and O refer to is only moved when a
// row's new maximum exceeds it by more than RESCALE_LOG2 (log2 units), so P
// stays below 2^RESCALE_LOG2 and O is rescaled rarely.  l and O share the
// stale reference, so O = acc / l and LSE = (m + log2 l) ln 2 stay exact.
constexpr float RESCALE_LOG2 = 8.0f;
// Columns of every 32-column chunk of an unmasked score row whose
// exponential is computed by exp2_poly instead of MUFU ex2.
// Measured on B200: every nonzero setting was slower on the long causal
// workloads (the softmax is not MUFU-bound once the rescale is lazy), so the
// default is 0; the polynomial path stays for tuning other shapes.
#ifndef FA_POLY_COLS
#define FA_POLY_COLS 0
#endif
constexpr int POLY_COLS = FA_POLY_COLS;
static_assert(POLY_COLS >= 0 && POLY_COLS <= 32 && POLY_COLS % 2 == 0, "poly columns");

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
    static constexpr int B_O_FULL = 2 * NS + 6;      // [2]
    static constexpr int B_O_EMPTY = 2 * NS + 8;     // [2]
    static constexpr int B_DRAIN = 2 * NS + 10;
    static constexpr int B_UFULL = 2 * NS + 11;      // [2] unit queue (dynamic schedule)
    static constexpr int B_UEMPTY = 2 * NS + 13;     // [2]
    static constexpr int NUM_BARS = 2 * NS + 15;
    // tmem base, abort flag, zero flag, spare, unit queue slots [2]
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int OFF_UNIT = OFF_MISC + 16;
    static constexpr int BYTES = OFF_MISC + 32;
    static constexpr int ALLOC = BYTES + 1024;       // slack to align the base to 1 KiB
    // TMEM columns
    static constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O0 = 256, TM_O1 = 256 + D;
    static constexpr uint32_t TM_COLS = 512;
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

// Software 2^x on the FMA pipe, used for part of each score row so the
// MUFU unit (ex2) is not the only source of exponentials.  Method:
// Cody-Waite range reduction x = n + f with n = rint(x) (the 1.5 * 2^23
// rounding constant), f in [-1/2, 1/2]; 2^f by a degree-3 polynomial whose
// coefficients minimise the maximum relative error on [-1/2, 1/2] (Remez
// exchange; csrc/gen_exp2_poly.py reproduces them, max relative error
// 7.5e-5, below the 2^-9 rounding of the bf16 P it feeds); 2^n is added to
// the exponent field.  Valid for x in [-126, 64]; inputs below -126 are
// clamped (results below 2^-125 are meaningless there, so the kernel only
// uses it on tiles without masked scores).
constexpr float EXP2_C0 = 9.999280572e-01f;
constexpr float EXP2_C1 = 6.932609677e-01f;
constexpr float EXP2_C2 = 2.426111251e-01f;
constexpr float EXP2_C3 = 5.517166853e-02f;

__device__ __forceinline__ float exp2_poly(float x) {
    x = fmaxf(x, -126.0f);
    const float t = x + 12582912.0f;            // 1.5 * 2^23: t's low bits hold rint(x)
    const float n = t - 12582912.0f;
    const float f = x - n;
    const float p = fmaf(fmaf(fmaf(EXP2_C3, f, EXP2_C2), f, EXP2_C1), f, EXP2_C0);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// ---------------------------------------------------------------------------
// Work decomposition: units of 256 query rows of one (batch, head).
// Units are ordered in groups of `hg` heads (sized on the host so a group's
// K and V stay resident in L2 while the CTAs working on it stream them);
// inside a group the order is by row block, the longest causal rows first.
// CTA b takes sequence indices in boustrophedon order (b, 2S-1-b, 2S+b, ...)
// so long and short units pair up across CTAs.
// ---------------------------------------------------------------------------
struct Unit {
    int bh, r0, nb0, nb1;  // first row, K/V tile counts of sub-tiles 0 and 1
};

__device__ __forceinline__ int unit_index(int k, int cta, int ctas) {
    return k * ctas + ((k & 1) ? (ctas - 1 - cta) : cta);
}

// N_q query rows and N_k keys per (batch, head); with causal masking query i
// may see key j iff j <= i + N_k - N_q (the queries are the last N_q
// positions), so a sub-tile's last row r sees keys up to r + N_k - N_q.
__device__ __forceinline__ Unit decode_unit(int i, int BH, int Nq, int Nk, int causal, int hg) {
    const int nq2 = (Nq + UNIT_ROWS - 1) / UNIT_ROWS;
    const int nkb = (Nk + BN - 1) / BN;
    const int off = Nk - Nq;
    const int per_group = hg * nq2;
    const int g = i / per_group;
    const int r = i - g * per_group;
    const int gh = min(hg, BH - g * hg);       // heads in this group
    const int level = r / gh;
    Unit w;
    w.bh = g * hg + (r - level * gh);
    const int qb2 = causal ? (nq2 - 1 - level) : level;
    w.r0 = qb2 * UNIT_ROWS;
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
// step is 32 bytes inside the swizzled rows.
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

// P = 2^(s * scale_log2 - m) for one score row held in registers, written
// to TMEM over the row's first columns: bf16 pairs (64 columns) or, with F8,
// FP8 E4M3 quads (32 columns).  The row sum (of the unrounded fp32 P) goes to
// four packed partial accumulators.  The first NPOLY columns of every
// 32-column chunk use exp2_poly, the rest MUFU ex2.
template <int NPOLY, bool F8 = false>
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
            float p0, p1;
            if (2 * i < NPOLY) {
                p0 = exp2_poly(x0);
                p1 = exp2_poly(x1);
            } else {
                p0 = ex2(x0);
                p1 = ex2(x1);
            }
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
                  int hg, long long o_sb, long long o_sh, long long o_sn, int* __restrict__ sched,
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
    // same boustrophedon sequence.  Dynamic schedule: the producer claims
    // sequence indices from the global counter *sched and publishes them in
    // two shared-memory slots (full: producer; empty: MMA thread and every
    // softmax thread); -1 ends the CTA's work.
    auto next_unit_consumer = [&](int kq, bool& ok_out, uint32_t role) -> int {
        if (!sched) {
            const int u = unit_index(kq, blockIdx.x, gridDim.x);
            return u < num_units ? u : -1;
        }
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
    regs_dec<REGS_OTHER>();
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
                    if (u >= num_units) u = -1;
                    unit_slot[slot] = u;
                    mbar_arrive(bar(L::B_UFULL + slot));
                } else {
                    u = unit_index(kq, blockIdx.x, gridDim.x);
                    if (u >= num_units) u = -1;
                }
                if (u < 0) break;
                const Unit w = decode_unit(u, BH, Nq, Nk, causal, hg);
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
            for (int kq = 0; ok; ++kq, ++units) {
                const int u = next_unit_consumer(kq, ok, ROLE_MMA);
                if (u < 0) break;
                const Unit w = decode_unit(u, BH, Nq, Nk, causal, hg);
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
                    if (next) {
                        sK = cons % NS;
                        if (!wait_phase(bar(L::B_KV_FULL + sK), (cons / NS) & 1u, wd, ROLE_MMA, u)) {
                            ok = false;
                            break;
                        }
                        ++cons;
                    }
                    if (j < w.nb0) {
                        if (j == 0 && !wait_phase(bar(L::B_O_EMPTY + 0), (units & 1u) ^ 1u, wd,
                                                  ROLE_MMA, u)) {
                            ok = false;
                            break;
                        }
                        if (!wait_phase(bar(L::B_P_FULL + 0), pcnt0 & 1u, wd, ROLE_MMA, u)) {
                            ok = false;
                            break;
                        }
                        ++pcnt0;
                        tc_fence_after();
                        issue_pv<F8>(tO0, tS0, desc_add(dv0, sV * stage_step), ID_PV, j == 0);
                        if (j + 1 < w.nb0) {
                            issue_qk<L::QK_STEPS, L::HALF_BYTES, F8>(tS0, dq0, desc_add(dk0, sK * stage_step), ID_S);
                            tc_commit(bar(L::B_S_FULL + 0));
                        }
                        if (j == w.nb0 - 1) tc_commit(bar(L::B_O_FULL + 0));
                    }
                    if (j == 0 && !wait_phase(bar(L::B_O_EMPTY + 1), (units & 1u) ^ 1u, wd, ROLE_MMA, u)) {
                        ok = false;
                        break;
                    }
                    if (!wait_phase(bar(L::B_P_FULL + 1), pcnt1 & 1u, wd, ROLE_MMA, u)) {
                        ok = false;
                        break;
                    }
                    ++pcnt1;
                    tc_fence_after();
                    issue_pv<F8>(tO1, tS1, desc_add(dv0, sV * stage_step), ID_PV, j == 0);
                    if (next) {
                        issue_qk<L::QK_STEPS, L::HALF_BYTES, F8>(tS1, dq1, desc_add(dk0, sK * stage_step), ID_S);
                        tc_commit(bar(L::B_S_FULL + 1));
                    }
                    tc_commit(bar(L::B_KV_EMPTY + sV));
                    if (next) tc_commit(bar(L::B_KV_EMPTY + sK));
                    if (next && j + 1 == w.nb1 - 1) tc_commit(bar(L::B_Q_EMPTY));
                    if (j == w.nb1 - 1) tc_commit(bar(L::B_O_FULL + 1));
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
        regs_inc<REGS_SOFTMAX>();
        const int t = warp >> 2;                     // sub-tile 0 or 1
        const int wr = (warp & 3) * 32 + lane;       // row within the sub-tile
        const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + (t == 0 ? L::TM_S0 : L::TM_S1);
        const uint32_t tO = tmem + lane_base + (t == 0 ? L::TM_O0 : L::TM_O1);
        uint32_t scnt = 0, ocnt = 0;
        bool ok = true;
        for (int kq = 0; ok; ++kq) {
            const int u = next_unit_consumer(kq, ok, ROLE_SOFTMAX);
            if (u < 0) break;
            const Unit w = decode_unit(u, BH, Nq, Nk, causal, hg);
            const int a = w.r0 + t * BM;             // first row of this sub-tile
            const int row = a + wr;
            const int nb = t == 0 ? w.nb0 : w.nb1;
            float m = -INFINITY;                     // running max, log2 units
            float l = 0.f;                           // running sum of exponentials
            for (int j = 0; j < nb; ++j) {
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
                // Row max: eight independent chains, then a tree.  (The
                // three-input max.f32 form measured inexact here: it broke the
                // bit-exact causal row 0 of the parity tests.)
                float mx8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mx8[i] = s[i];
#pragma unroll
                for (int c = 8; c < BN; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
                const float m_blk =
                    fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                          fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * scale_log2;
                // Lazy rescale (first tile: m = -inf, so every lane moves).
                if (__any_sync(0xffffffffu, m_blk > m + RESCALE_LOG2)) {
                    const float m_new = fmaxf(m, m_blk);
                    const float alpha = ex2(m - m_new);      // 0 on the first tile
                    if (j > 0) {
                        // The PV of tile j-1 is complete: its commit
                        // preceded the S_t commit waited on above.
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t r[32];
                            tmem_ld32(tO + c * 32, r);
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                            tmem_st32(tO + c * 32, r);
                        }
                    }
                    l *= alpha;
                    m = m_new;
                }
                const float neg_m = -m;
                uint64_t acc[4] = {0, 0, 0, 0};              // four packed (0.f, 0.f)
                // Tiles without masked scores may use the FMA-pipe 2^x for
                // part of the row; the choice is warp-uniform, made once.
                if (POLY_COLS > 0 && !(tail || diag))
                    exp_row_to_p<POLY_COLS, F8>(s, scale_log2, neg_m, acc, tS);
                else
                    exp_row_to_p<0, F8>(s, scale_log2, neg_m, acc, tS);
                {
                    float a0, a1, a2, a3, a4, a5, a6, a7;
                    f2_unpack(acc[0], a0, a1);
                    f2_unpack(acc[1], a2, a3);
                    f2_unpack(acc[2], a4, a5);
                    f2_unpack(acc[3], a6, a7);
                    l += ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(L::B_P_FULL + t));
            }
            if (!ok) break;
            // Epilogue: O / l -> bf16 -> global; LSE.
            bool got = wait_phase(bar(L::B_O_FULL + t), ocnt & 1u, wd, ROLE_SOFTMAX, u);
            ++ocnt;
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            float inv_l = 1.f / l;
            if constexpr (F8) inv_l *= o_scale;
            const bool store = row < Nq;
            const int wb = w.bh / H, wh = w.bh - (w.bh / H) * H;     // batch, head
            __nv_bfloat16* orow = Og + wb * o_sb + wh * o_sh + (long long)(store ? row : 0) * o_sn;
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
            }
            if (store) LSEg[size_t(w.bh) * Nq + row] = (m + log2f(l)) * 0.69314718055994530942f;
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

// Heads per scheduling group.  The kernel orders units in groups of `hg`
// heads (longest causal row blocks first inside a group) and deals them to
// CTAs in boustrophedon order (decode_unit / unit_index).  Small groups keep
// the K/V that concurrently running CTAs stream resident in L2; large groups
// balance the CTAs better.  This replays the kernel's assignment on the host
// for hg = 1, 2, 4, ..., BH (K/V tiles per unit as the cost) and takes the
// lowest  (max CTA load / mean CTA load) x (1 + L2 penalty), the penalty
// growing with the group's K/V bytes: 0 up to 16 MiB, then 3 %, 6 %, 9 % and
// 12 % past 16, 32, 64 and 128 MiB (calibrated on the 8K and 32K causal
// workloads, where 2-head groups measured 4-7 % faster than 8- or all-head
// groups).  Decisions are cached per shape.
struct HgKey {
    long long BH;
    int Nq, Nk, D, causal, grid;
    bool operator==(const HgKey& o) const {
        return BH == o.BH && Nq == o.Nq && Nk == o.Nk && D == o.D && causal == o.causal &&
               grid == o.grid;
    }
};
std::mutex g_hg_mutex;
HgKey g_hg_keys[64];
long long g_hg_vals[64];
int g_hg_count = 0;

double snake_imbalance(long long BH, int Nq, int Nk, int causal, long long hg, int grid) {
    const long long nq2 = (Nq + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS;
    const long long nkb = (Nk + fa::BN - 1) / fa::BN;
    const long long off = Nk - Nq;
    const long long units = nq2 * BH;
    std::vector<long long> load(size_t(grid), 0);
    const long long per_group = hg * nq2;
    for (long long i = 0; i < units; ++i) {
        const long long g = i / per_group;
        const long long r = i - g * per_group;
        const long long gh = std::min(hg, BH - g * hg);
        const long long level = r / gh;
        const long long r0 = (causal ? (nq2 - 1 - level) : level) * fa::UNIT_ROWS;
        const long long nb0 = causal ? std::min((r0 + fa::BM - 1 + off) / fa::BN + 1, nkb) : nkb;
        const long long nb1 =
            causal ? std::min((r0 + 2 * fa::BM - 1 + off) / fa::BN + 1, nkb) : nkb;
        const long long k = i / grid, c = i - k * grid;
        load[size_t((k & 1) ? (grid - 1 - c) : c)] += nb0 + nb1 + 2;   // +2: per-unit overhead
    }
    long long mx = 0, sum = 0;
    for (long long x : load) {
        mx = std::max(mx, x);
        sum += x;
    }
    return double(mx) * grid / double(sum);
}

long long choose_head_group(long long BH, int Nq, int Nk, int D, int causal, int grid) {
    const HgKey key{BH, Nq, Nk, D, causal, grid};
    {
        std::lock_guard<std::mutex> lk(g_hg_mutex);
        for (int i = 0; i < g_hg_count; ++i)
            if (g_hg_keys[i] == key) return g_hg_vals[i];
    }
    const long long kv_head_bytes = 2LL * Nk * D * 2;
    long long best = BH;
    double best_cost = 1e30;
    // Bound the replay work for very large problems: beyond ~4M units the
    // assignment statistics no longer depend on hg, so all heads form one group.
    const long long units = ((Nq + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS) * BH;
    if (units <= (4LL << 20)) {
        for (long long hg = 1;; hg = std::min(hg * 2, BH)) {
            const double ws = double(hg * kv_head_bytes);
            const double pen = ws <= 16.0 * (1 << 20) ? 0.0
                             : ws <= 32.0 * (1 << 20) ? 0.03
                             : ws <= 64.0 * (1 << 20) ? 0.06
                             : ws <= 128.0 * (1 << 20) ? 0.09 : 0.12;
            const double cost = snake_imbalance(BH, Nq, Nk, causal, hg, grid) * (1.0 + pen);
            if (cost < best_cost - 1e-9) {
                best_cost = cost;
                best = hg;
            }
            if (hg == BH) break;
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
    long long hg = sched ? ((BH * kv_head_bytes <= (32LL << 20)) ? BH : (16LL << 20) / kv_head_bytes)
                         : choose_head_group(BH, Nq, Nk, D, causal, grid);
#ifdef FA_HEAD_GROUP
    hg = FA_HEAD_GROUP;
#endif
    hg = hg < 1 ? 1 : (hg > BH ? BH : hg);
    if (sched) {
        const cudaError_t me = cudaMemsetAsync(sched, 0, sizeof(int), stream);
        if (me != cudaSuccess) {
            t_last_cuda_error = int(me);
            return FA_ERR_LAUNCH;
        }
    }
    kern<<<grid, fa::NUM_THREADS, L::ALLOC, stream>>>(mq, mk, mv, static_cast<__nv_bfloat16*>(o),
                                                     lse, int(BH), H, Nq, Nk, causal, scale_log2,
                                                     int(hg), ost.b, ost.h, ost.n, sched,
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
    // more units than it may count are refused before anything else.
    if (B >= 1 && H >= 1 && N >= 1 &&
        ((long long)N + fa::UNIT_ROWS - 1) / fa::UNIT_ROWS * B * H > FA_NOALLOC_MAX_UNITS)
        return FA_ERR_UNSUPPORTED;
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
    return word == 0 ? FA_OK : FA_ERR_TIMEOUT;
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
