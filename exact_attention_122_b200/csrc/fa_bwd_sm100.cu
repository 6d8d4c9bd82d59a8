// fa_bwd_sm100.cu -- exact attention backward for B200 (sm_100a).
//
// Given Q, K, V, the forward's output O and per-row log-sum-exp LSE, and the
// upstream gradient dO, computes dQ, dK, dV of O = softmax(scale Q K^T
// [+ causal mask]) V without storing P: every P block is rebuilt from Q, K
// and LSE on chip (page "Flash attention optimization", section "Sizing a
// tile, and why the backward pass recomputes instead of storing": only the
// per-row statistics are kept and the needed P blocks are recomputed from the
// saved Q, K, V tiles).  The gradient formulas are those of the softmax:
//   P = exp(scale S - LSE),  dV = P^T dO,  dP = dO V^T,
//   D_i = sum_t dO_it O_it,  dS = P * (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels, all on the caller's stream:
//   bwd_prep     D_i and LSE_i * log2(e) per row into the workspace (padded
//                rows get D = 0, LSE = +inf, so their P is 0), and zeroes
//                the fp32 dQ accumulator.
//   bwd_kernel_x (d = 128, below) or
//   bwd_kernel   (d = 64) one CTA per 128-key block of one (batch, head),
//                448 threads:
//                  warps 0-7   compute: P, dS for the key block's 128 rows
//                              (warp w: TMEM lane quarter w % 4, half of the
//                              query columns w / 4)
//                  warps 8-11  dQ drain: read this step's dQ partial from
//                              TMEM and add it to the fp32 accumulator in
//                              global memory with coalesced reductions
//                  warp  12    MMA issuer (one thread)
//                  warp  13    TMA producer (one thread): K, V once, then
//                              Q, dO, LSE, D of each query block through an
//                              NS-stage ring
//                K_j, V_j stay in shared memory and dK_j, dV_j accumulate in
//                TMEM over all query blocks; per query block of BQ rows the
//                tensor core computes S^T = K Q^T and dP^T = V dO^T (keys on
//                the TMEM lanes), then dV += P^T dO (P from TMEM), dK += dS^T Q
//                and the dQ partial (dS from shared memory).  The MMAs of
//                block i-1's gradients are issued after block i's S^T and
//                dP^T, so the compute warps' exponentials for block i overlap
//                the tensor core's work on block i-1.
//                bwd_kernel_x keeps the same division of work with 128
//                query rows per step and its own TMEM plan (see there).
//   bwd_dq_out   dQ = bf16(scale * accumulator).
//
// Every mbarrier wait is bounded by a %globaltimer watchdog, as in the
// forward kernel: a wait that runs out records FA_ERR_TIMEOUT in
// g_bwd_status, raises a CTA-wide abort flag, and every role leaves its
// loop, drains its own copies and MMAs (bounded), frees TMEM and returns.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"
#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace bwd {

using namespace sm100;

constexpr int BK = 128;             // keys per CTA (TMEM lanes of S^T, dP^T, dK, dV)
constexpr int NUM_THREADS = 448;
constexpr int COMPUTE_WARPS = 8;
constexpr int DQ_WARP0 = 8;
constexpr int MMA_WARP = 12;
constexpr int TMA_WARP = 13;
// Q / dO ring stages.  A stage is held from its load until block i's
// gradient MMAs have run, about two steps; with two stages the next load's
// latency was exposed on every step (measured on B200: three stages 24 %
// faster on the 8K causal workload).
constexpr int NS = 3;
constexpr float LOG2E = 1.4426950408889634f;

enum : uint32_t { ROLE_COMPUTE = 1u, ROLE_MMA = 2u, ROLE_PRODUCER = 3u, ROLE_DQ = 4u,
                  ROLE_DRAIN = 5u };

// bwd_kernel's layout (d = 64; d = 128 runs bwd_kernel_x): 128 query rows per
// step and dQ with the queries on the TMEM lanes; every MMA at M = 128, within
// the 512 TMEM columns.
template <int D>
struct Cfg {
    static_assert(D == 64, "bwd_kernel runs d = 64 only");
    static constexpr int BQ = 128;
    static constexpr int KV_BYTES = BK * D * 2;
    static constexpr int KV_SLAB = BK * 128;             // 64 columns of a K/V tile
    static constexpr int QD_BYTES = BQ * D * 2;
    static constexpr int QD_SLAB = BQ * 128;             // 64 columns of a Q/dO tile
    static constexpr int DS_BYTES = BK * BQ * 2;
    static constexpr int DS_SLAB = BK * 128;             // 64 queries of dS, all keys
    static constexpr int VEC_BYTES = 2 * BQ * 4;         // LSE2 and D of one query block
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KV_BYTES;
    static constexpr int OFF_Q = OFF_V + KV_BYTES;
    static constexpr int OFF_DO = OFF_Q + NS * QD_BYTES;
    static constexpr int OFF_DS = OFF_DO + NS * QD_BYTES;
    static constexpr int OFF_VEC = OFF_DS + 2 * DS_BYTES;
    // dQ staging: per dQ warp 16 rows of d fp32, rows 16 bytes apart beyond
    // their length so the row-per-lane stores hit distinct banks.
    static constexpr int STG_ROW = D * 4 + 16;
    static constexpr int STG_WARP = 16 * STG_ROW;
    static constexpr int OFF_STG = OFF_VEC + NS * VEC_BYTES;
    static constexpr int OFF_BAR = OFF_STG + 4 * STG_WARP;
    static constexpr int B_KV_FULL = 0;
    static constexpr int B_QD_FULL = 1;                  // [NS]
    static constexpr int B_QD_EMPTY = 1 + NS;            // [NS]
    static constexpr int B_SDP_FULL = 1 + 2 * NS;
    static constexpr int B_SDP_FREE = 2 + 2 * NS;
    static constexpr int B_DS_READY = 3 + 2 * NS;        // [2]
    static constexpr int B_K_TMEM = 5 + 2 * NS;          // K copied into TMEM
    static constexpr int B_DS_FREE = 7 + 2 * NS;         // [2]
    static constexpr int B_DQ_FULL = 9 + 2 * NS;
    static constexpr int B_DQ_EMPTY = 10 + 2 * NS;
    static constexpr int B_ACC_FULL = 11 + 2 * NS;
    static constexpr int B_DRAIN = 12 + 2 * NS;
    static constexpr int NUM_BARS = 13 + 2 * NS;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;   // tmem base, abort flag
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
    // TMEM columns.  P of block n (bf16, BQ/2 columns) lives in the first
    // columns of the dQ region: it is written after the dQ warps have read
    // dQ of block n-1, and the dQ MMA of block n overwrites it only after the
    // dV MMA that reads it (MMAs from one thread run in issue order).  K is
    // held in TMEM as the A operand of S^T = K Q^T (bf16, D/2 columns).
    static constexpr uint32_t TM_S = 0;
    static constexpr uint32_t TM_DP = BQ;
    static constexpr uint32_t TM_DQ = 2 * BQ;                  // dQ^T: BQ cols; dQ: D cols
    static constexpr uint32_t TM_P = TM_DQ;
    static constexpr uint32_t DQ_COLS = D;
    static constexpr uint32_t TM_K = TM_DQ + DQ_COLS;
    static constexpr uint32_t TM_DV = TM_K + D / 2;
    static constexpr uint32_t TM_DK = TM_DV + D;
    static constexpr uint32_t TM_COLS = 512;
    static_assert(TM_DK + D <= TM_COLS, "TMEM budget");
    static_assert(BQ / 2 <= DQ_COLS, "P fits in the dQ columns");
    static_assert(ALLOC <= 227 * 1024, "shared memory budget");
    static_assert(BYTES > 116 * 1024, "one CTA per SM keeps TMEM allocation uncontended");
    static_assert((BQ / 2) % 32 == 0, "compute warps take 32-column chunks");
};

// Element strides (batch, head, sequence) of one bf16 [B][H][N][d] operand;
// the head dimension d is contiguous.
struct St3 {
    long long b, h, n;
    __host__ __device__ long long row(long long bh, int H, long long r) const {
        return (bh / H) * b + (bh % H) * h + r * n;
    }
};

__device__ unsigned int g_bwd_status;   // 0 = fine; else (FA_ERR_TIMEOUT << 24) | role << 20 | block

struct Watchdog {
    volatile int* abort_flag;
    uint64_t limit_ns;
};

__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, Watchdog wd,
                                           uint32_t role, uint32_t blk) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*wd.abort_flag) return false;
        if (global_timer_ns() - t0 > wd.limit_ns) {
            atomicCAS(&g_bwd_status, 0u,
                      (uint32_t(FA_ERR_TIMEOUT) << 24) | (role << 20) | (blk & 0xFFFFFu));
            *wd.abort_flag = 1;
            __threadfence_block();
            return false;
        }
    }
}

// wait_phase taken by a whole warp: the warp goes on only if every lane's
// wait succeeded, so the warp-collective tcgen05 loads and stores that follow
// are never reached by part of a warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, Watchdog wd,
                                          uint32_t role, uint32_t blk) {
    const bool ok = wait_phase(bar, parity, wd, role, blk);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag: used only to drain this thread's
// own copies and MMAs before the CTA exits.
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) {
            atomicCAS(&g_bwd_status, 0u, (uint32_t(FA_ERR_TIMEOUT) << 24) | (ROLE_DRAIN << 20));
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void cta_sync() {
    asm volatile("bar.sync 0, %0;" ::"n"(NUM_THREADS) : "memory");
}

// 1-D bulk copy global -> shared completing on an mbarrier (16-byte aligned
// addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ void red_add_f32(float* p, float v) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

__device__ __forceinline__ void red_add_v4_f32(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

// ---------------------------------------------------------------------------
// Pre-pass: -D_i = -(dO_i . O_i) (fp32), -LSE2_i = -LSE_i log2(e), zero
// dQ_acc.  Rows r in [N, Npad) get -D = 0 and -LSE2 = -inf (so P = 0).
// Both are stored negated so the compute warps add them with packed f32x2
// fused multiply-adds.  D / 8 threads per row, each
// on 8 consecutive elements.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_prep(const __nv_bfloat16* __restrict__ o,
                                                const __nv_bfloat16* __restrict__ dout,
                                                const float* __restrict__ lse,
                                                float* __restrict__ nlse2,
                                                float* __restrict__ ndvec,
                                                float* __restrict__ dq_acc, long long BH, int H,
                                                int N, int Npad, St3 so, St3 sdo) {
    constexpr int TPR = D / 8;                          // threads per row
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long row = t / TPR;                      // over BH * Npad
    const int part = int(t % TPR);
    const bool live = row < BH * Npad;                  // every lane joins the shuffles below
    const long long bh = row / Npad;
    const int r = int(row - bh * Npad);
    float acc = 0.f;
    if (live && r < N) {
        const uint4 a = *reinterpret_cast<const uint4*>(o + so.row(bh, H, r) + part * 8);
        const uint4 b = *reinterpret_cast<const uint4*>(dout + sdo.row(bh, H, r) + part * 8);
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 x = __bfloat1622float2(a2[i]);
            const float2 y = __bfloat1622float2(b2[i]);
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
        }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (!live) return;
    float4* z = reinterpret_cast<float4*>(dq_acc + row * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (part == 0) {
        ndvec[row] = r < N ? -acc : 0.f;
        nlse2[row] = r < N ? -lse[bh * N + r] * LOG2E : -INFINITY;
    }
}

// dQ = bf16(scale * dQ_acc) for rows < N; 8 elements per thread.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_out(const float* __restrict__ dq_acc,
                                                  __nv_bfloat16* __restrict__ dq, long long BH,
                                                  int H, int N, int Npad, float scale, St3 sdq) {
    constexpr int TPR = D / 8;
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long row = t / TPR;                      // over BH * N
    const int part = int(t % TPR);
    if (row >= BH * N) return;
    const long long bh = row / N;
    const long long r = row - bh * N;
    const float4* a = reinterpret_cast<const float4*>(dq_acc + (bh * Npad + r) * D + part * 8);
    const float4 x = a[0], y = a[1];
    uint4 out;
    out.x = pack_bf16x2(scale * x.x, scale * x.y);
    out.y = pack_bf16x2(scale * x.z, scale * x.w);
    out.z = pack_bf16x2(scale * y.x, scale * y.y);
    out.w = pack_bf16x2(scale * y.z, scale * y.w);
    *reinterpret_cast<uint4*>(dq + sdq.row(bh, H, r) + part * 8) = out;
}

// P and dS for 32 query columns of one key row (this thread's TMEM lane):
//   p = 2^(s * scale log2(e) - LSE2),  ds = p * (dP - D),
// both rounded to bf16 pairs.  nl / nd point at -LSE2 and -D of the 32
// columns (shared memory).  MASK: zero p where the query precedes the key
// (causal), or the query or key is past N.  Pairs of columns go through the
// packed f32x2 pipe.
template <bool MASK>
__device__ __forceinline__ void p_ds_chunk(const uint32_t (&sv)[32], const uint32_t (&dpv)[32],
                                           const float* nl, const float* nd, float cs, int qi0,
                                           int key, int N, int causal, uint32_t (&pu)[16],
                                           uint32_t (&du)[16]) {
    const uint64_t cs2 = f2_pack(cs, cs);
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(nl + j);
        const float4 d4 = *reinterpret_cast<const float4*>(nd + j);
        const uint64_t l01 = f2_pack(l4.x, l4.y), l23 = f2_pack(l4.z, l4.w);
        const uint64_t d01 = f2_pack(d4.x, d4.y), d23 = f2_pack(d4.z, d4.w);
        const uint64_t x01 = f2_fma(f2_pack(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])),
                                    cs2, l01);
        const uint64_t x23 = f2_fma(
            f2_pack(__uint_as_float(sv[j + 2]), __uint_as_float(sv[j + 3])), cs2, l23);
        float x[4], p[4];
        f2_unpack(x01, x[0], x[1]);
        f2_unpack(x23, x[2], x[3]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            p[u] = ex2(x[u]);
            if (MASK) {
                const int qi = qi0 + j + u;
                if ((causal && qi < key) || qi >= N || key >= N) p[u] = 0.f;
            }
        }
        const uint64_t t01 = f2_add(
            f2_pack(__uint_as_float(dpv[j]), __uint_as_float(dpv[j + 1])), d01);
        const uint64_t t23 = f2_add(
            f2_pack(__uint_as_float(dpv[j + 2]), __uint_as_float(dpv[j + 3])), d23);
        float ds[4];
        f2_unpack(f2_mul(f2_pack(p[0], p[1]), t01), ds[0], ds[1]);
        f2_unpack(f2_mul(f2_pack(p[2], p[3]), t23), ds[2], ds[3]);
        pu[j / 2] = pack_bf16x2(p[0], p[1]);
        pu[j / 2 + 1] = pack_bf16x2(p[2], p[3]);
        du[j / 2] = pack_bf16x2(ds[0], ds[1]);
        du[j / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
    }
}

// ---------------------------------------------------------------------------
// Main kernel
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
           const float* __restrict__ nlse2, const float* __restrict__ ndvec,
           float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dk,
           __nv_bfloat16* __restrict__ dv, int BH, int H, int N, int Npad, int causal,
           float scale, int hg, unsigned long long watchdog_ns, int inject, St3 sdk, St3 sdv) {
    using C = Cfg<D>;
    constexpr int BQ = C::BQ;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    // Work order: groups of hg heads (sized on the host so a group's Q, dO,
    // K, V and dQ accumulator stay in L2 while its CTAs run); inside a group
    // key-block-major, so the longest causal blocks (the first key blocks)
    // of the group's heads start first.
    const int nkb = (N + BK - 1) / BK;
    const int per_group = hg * nkb;
    const int g = int(blockIdx.x) / per_group;
    const int r_in = int(blockIdx.x) - g * per_group;
    const int gh = min(hg, BH - g * hg);              // heads in this group
    const int kb = r_in / gh;
    const int bh = g * hg + (r_in - kb * gh);
    const int b = bh / H, h = bh - (bh / H) * H;
    const int k0 = kb * BK;
    const int nqb = (N + BQ - 1) / BQ;
    const int qb_first = causal ? k0 / BQ : 0;
    const int nsteps = nqb - qb_first;

    if (threadIdx.x == 0) {
        mbar_init(bar(C::B_KV_FULL), 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(C::B_QD_FULL + s), 1);
            mbar_init(bar(C::B_QD_EMPTY + s), 1 + COMPUTE_WARPS);
        }
        mbar_init(bar(C::B_SDP_FULL), 1);
        mbar_init(bar(C::B_SDP_FREE), COMPUTE_WARPS);
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(C::B_DS_READY + i), COMPUTE_WARPS);
            mbar_init(bar(C::B_DS_FREE + i), 1);
        }
        mbar_init(bar(C::B_DQ_FULL), 1);
        mbar_init(bar(C::B_DQ_EMPTY), 4);
        mbar_init(bar(C::B_K_TMEM), COMPUTE_WARPS);
        mbar_init(bar(C::B_ACC_FULL), 1);
        mbar_init(bar(C::B_DRAIN), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == MMA_WARP) {
        tmem_alloc(smem_addr(tmem_slot), C::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    cta_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Watchdog wd{abort_flag, watchdog_ns};
    const uint32_t blk_id = blockIdx.x;

    if (warp == TMA_WARP) {
        // ------------------------------------------------------------------
        // Producer
        // ------------------------------------------------------------------
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(C::B_KV_FULL), 2 * C::KV_BYTES);
#pragma unroll
            for (int sl = 0; sl < D / 64; ++sl) {
                tma_load_4d(sbase + C::OFF_K + sl * C::KV_SLAB, &tmK, sl * 64, k0, h, b,
                            bar(C::B_KV_FULL));
                tma_load_4d(sbase + C::OFF_V + sl * C::KV_SLAB, &tmV, sl * 64, k0, h, b,
                            bar(C::B_KV_FULL));
            }
            int issued = 0;
            // Host-chosen fault injection (inject = 1): CTA 0 never issues its
            // first Q / dO block, so the waits on it can only end by the watchdog.
            const bool skip0 = inject == 1 && blockIdx.x == 0;
            for (int n = 0; n < nsteps; ++n) {
                const int s = n % NS;
                if (n >= NS && !wait_phase(bar(C::B_QD_EMPTY + s), ((n / NS) - 1) & 1, wd,
                                           ROLE_PRODUCER, blk_id))
                    break;
                ++issued;
                if (skip0 && n == 0) continue;
                const int q0 = (qb_first + n) * BQ;
                const uint32_t full = bar(C::B_QD_FULL + s);
                mbar_arrive_expect_tx(full, 2 * C::QD_BYTES + C::VEC_BYTES);
#pragma unroll
                for (int sl = 0; sl < D / 64; ++sl) {
                    tma_load_4d(sbase + C::OFF_Q + s * C::QD_BYTES + sl * C::QD_SLAB, &tmQ,
                                sl * 64, q0, h, b, full);
                    tma_load_4d(sbase + C::OFF_DO + s * C::QD_BYTES + sl * C::QD_SLAB, &tmDO,
                                sl * 64, q0, h, b, full);
                }
                const long long vrow = (long long)bh * Npad + q0;
                bulk_load(sbase + C::OFF_VEC + s * C::VEC_BYTES, nlse2 + vrow, BQ * 4, full);
                bulk_load(sbase + C::OFF_VEC + s * C::VEC_BYTES + BQ * 4, ndvec + vrow, BQ * 4,
                          full);
            }
            // Drain: every copy this thread issued has landed before exit.
            wait_drain(bar(C::B_KV_FULL), 0, watchdog_ns);
            for (int n = (issued > NS ? issued - NS : 0); n < issued; ++n)
                if (!(skip0 && n == 0))
                    wait_drain(bar(C::B_QD_FULL + n % NS), (n / NS) & 1, watchdog_ns);
        }
    } else if (warp == MMA_WARP) {
        // ------------------------------------------------------------------
        // MMA issuer
        // ------------------------------------------------------------------
        if (lane == 0) {
            constexpr uint32_t ID_S = idesc_bf16(128, BQ, false);          // S^T, dP^T
            constexpr uint32_t ID_G = idesc_bf16(128, D, true);            // dV, dK
            constexpr uint32_t ID_Q = idesc_bf16(128, D, true, true);      // dQ = dS K
            const uint64_t dV_kmaj = sdesc_sw128(sbase + C::OFF_V, 16, 1024);
            const uint64_t dK_mn = sdesc_sw128(sbase + C::OFF_K, C::KV_SLAB, 1024);
            bool ok = wait_phase(bar(C::B_KV_FULL), 0, wd, ROLE_MMA, blk_id) &&
                      wait_phase(bar(C::B_K_TMEM), 0, wd, ROLE_MMA, blk_id);
            tc_fence_after();

            auto grads = [&](int m) -> bool {
                const int s = m % NS, db = m % 2;
                if (!wait_phase(bar(C::B_DS_READY + db), (m / 2) & 1, wd, ROLE_MMA, blk_id))
                    return false;
                tc_fence_after();
                const uint32_t sq = sbase + C::OFF_Q + s * C::QD_BYTES;
                const uint32_t sdo = sbase + C::OFF_DO + s * C::QD_BYTES;
                const uint32_t sds = sbase + C::OFF_DS + db * C::DS_BYTES;
                // dV += P^T dO: A = P (TMEM, 16 queries = 8 columns per step),
                // B = dO MN-major (16 query rows of 128 bytes per step).
                const uint64_t do_mn = sdesc_sw128(sdo, C::QD_SLAB, 1024);
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk)
                    mma_ts(tmem + C::TM_DV, tmem + C::TM_P + kk * 8,
                           desc_add(do_mn, uint32_t((kk * 2048) >> 4)), ID_G,
                           (m > 0 || kk > 0) ? 1u : 0u);
                // dK += dS^T Q: A = dS K-major (keys x queries), B = Q MN-major.
                const uint64_t ds_kmaj = sdesc_sw128(sds, 16, 1024);
                const uint64_t q_mn = sdesc_sw128(sq, C::QD_SLAB, 1024);
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk)
                    mma_ss(tmem + C::TM_DK,
                           desc_add(ds_kmaj, uint32_t(((kk / 4) * C::DS_SLAB + (kk % 4) * 32) >> 4)),
                           desc_add(q_mn, uint32_t((kk * 2048) >> 4)), ID_G,
                           (m > 0 || kk > 0) ? 1u : 0u);
                // dQ partial of this query block: K = 128 keys in steps of 16.
                if (m >= 1 && !wait_phase(bar(C::B_DQ_EMPTY), (m - 1) & 1, wd, ROLE_MMA, blk_id))
                    return false;
                tc_fence_after();
                const uint64_t ds_mn = sdesc_sw128(sds, C::DS_SLAB, 1024);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint32_t off = uint32_t((kk * 2048) >> 4);
                    // dQ = dS K: A = dS MN-major (queries x keys), B = K MN-major
                    mma_ss(tmem + C::TM_DQ, desc_add(ds_mn, off), desc_add(dK_mn, off), ID_Q,
                           kk > 0 ? 1u : 0u);
                }
                // One commit for the block's gradients: the dQ warps, which
                // wait on it every step, pass the release of the dS buffer and
                // of the Q / dO stage on with plain arrivals (each commit costs
                // tensor-pipe time).
                tc_commit(bar(C::B_DQ_FULL));
                return true;
            };

            for (int n = 0; ok && n < nsteps; ++n) {
                const int s = n % NS;
                if (!wait_phase(bar(C::B_QD_FULL + s), (n / NS) & 1, wd, ROLE_MMA, blk_id)) {
                    ok = false;
                    break;
                }
                if (n >= 1 && !wait_phase(bar(C::B_SDP_FREE), (n - 1) & 1, wd, ROLE_MMA, blk_id)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sq = sbase + C::OFF_Q + s * C::QD_BYTES;
                const uint32_t sdo = sbase + C::OFF_DO + s * C::QD_BYTES;
                const uint64_t q_kmaj = sdesc_sw128(sq, 16, 1024);
                const uint64_t do_kmaj = sdesc_sw128(sdo, 16, 1024);
                // S^T = K Q^T (A = K from TMEM, 8 columns per 16 d) and
                // dP^T = V dO^T (A = V from SMEM): M = 128 keys, N = BQ queries, K = d.
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t ob = uint32_t(((kk / 4) * C::QD_SLAB + (kk % 4) * 32) >> 4);
                    mma_ts(tmem + C::TM_S, tmem + C::TM_K + kk * 8, desc_add(q_kmaj, ob), ID_S,
                           kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t oa = uint32_t(((kk / 4) * C::KV_SLAB + (kk % 4) * 32) >> 4);
                    const uint32_t ob = uint32_t(((kk / 4) * C::QD_SLAB + (kk % 4) * 32) >> 4);
                    mma_ss(tmem + C::TM_DP, desc_add(dV_kmaj, oa), desc_add(do_kmaj, ob), ID_S,
                           kk > 0 ? 1u : 0u);
                }
                tc_commit(bar(C::B_SDP_FULL));
                if (n >= 1 && !grads(n - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok) ok = grads(nsteps - 1);
            if (ok) tc_commit(bar(C::B_ACC_FULL));
            // Drain: every MMA this thread issued has completed before TMEM is freed.
            tc_commit(bar(C::B_DRAIN));
            wait_drain(bar(C::B_DRAIN), 0, watchdog_ns);
        }
    } else if (warp >= DQ_WARP0) {
        // ------------------------------------------------------------------
        // dQ drain: TMEM -> fp32 reductions into dq_acc
        // ------------------------------------------------------------------
        const int qw = warp - DQ_WARP0;                       // lane quarter
        const uint32_t lane_base = uint32_t(32 * qw) << 16;
        for (int n = 0; n < nsteps; ++n) {
            if (!warp_wait(bar(C::B_DQ_FULL), n & 1, wd, ROLE_DQ, blk_id)) break;
            tc_fence_after();
            if (qw == 0 && lane == 0) {
                // block n's dV, dK and dQ products are complete: its dS
                // buffer and its Q / dO stage are free
                mbar_arrive(bar(C::B_DS_FREE + (n % 2)));
                mbar_arrive(bar(C::B_QD_EMPTY + (n % NS)));
            }
            const int q0 = (qb_first + n) * BQ;
            {
                // lane = query row; columns = d.  The rows go through shared
                // memory, 16 at a time, so the reductions are issued with lane
                // = column: each instruction covers 128 contiguous bytes of one
                // row (a lane per row would touch 32 rows in 16-byte pieces).
                uint32_t r0[32], r1[32];
                tmem_ld32(tmem + lane_base + C::TM_DQ, r0);
                tmem_ld32(tmem + lane_base + C::TM_DQ + 32, r1);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_DQ_EMPTY));
                const uint32_t stg = sbase + C::OFF_STG + qw * C::STG_WARP;
                const int rows = min(32, N - (q0 + 32 * qw));      // valid rows of this warp
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    if ((lane >> 4) == hr) {
                        const uint32_t dst = stg + (lane & 15) * C::STG_ROW;
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            st_shared_v4(dst + j * 4, r0[j], r0[j + 1], r0[j + 2], r0[j + 3]);
                            st_shared_v4(dst + 128 + j * 4, r1[j], r1[j + 1], r1[j + 2], r1[j + 3]);
                        }
                    }
                    __syncwarp();
#pragma unroll 4
                    for (int i = 0; i < 16; ++i) {
                        const int lr = 16 * hr + i;               // row within the warp's 32
                        if (lr < rows) {
                            float a, c;
                            asm volatile("ld.shared.f32 %0, [%1];"
                                         : "=f"(a) : "r"(stg + i * C::STG_ROW + lane * 4));
                            asm volatile("ld.shared.f32 %0, [%1];"
                                         : "=f"(c) : "r"(stg + i * C::STG_ROW + 128 + lane * 4));
                            float* base =
                                dq_acc + ((long long)bh * Npad + q0 + 32 * qw + lr) * D + lane;
                            red_add_f32(base, a);
                            red_add_f32(base + 32, c);
                        }
                    }
                    __syncwarp();
                }
            }
        }
    } else {
        // ------------------------------------------------------------------
        // Compute warps: P and dS for key rows r (TMEM lane), half of the
        // query columns each.
        // ------------------------------------------------------------------
        const int qw = warp % 4, half = warp / 4;
        const int r = 32 * qw + lane;                         // key row in the block
        const int key = k0 + r;
        const uint32_t lane_base = uint32_t(32 * qw) << 16;
        const float cs = scale * LOG2E;
        bool ok = warp_wait(bar(C::B_KV_FULL), 0, wd, ROLE_COMPUTE, blk_id);
        if (ok) {
            // K row r, d columns half*64 .. half*64+63 (one 128-byte swizzled
            // slab row) -> TMEM columns TM_K + half*32 .. +31 as bf16 pairs.
            uint32_t kr[32];
            const uint32_t krow = sbase + C::OFF_K + half * C::KV_SLAB + (r / 8) * 1024 +
                                  (r % 8) * 128;
            if (half < D / 64) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t a = krow + uint32_t((c ^ (r % 8)) * 16);
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(kr[4 * c]), "=r"(kr[4 * c + 1]), "=r"(kr[4 * c + 2]),
                                   "=r"(kr[4 * c + 3])
                                 : "r"(a));
                }
                tmem_st32(tmem + lane_base + C::TM_K + half * 32, kr);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_K_TMEM));
        }
        for (int n = 0; ok && n < nsteps; ++n) {
            const int s = n % NS, db = n % 2;
            const int q0 = (qb_first + n) * BQ;
            // QD_FULL: the LSE2 / D vectors of this block (bulk copies) have
            // landed; SDP_FULL: S^T and dP^T are in TMEM.
            if (!warp_wait(bar(C::B_QD_FULL + s), (n / NS) & 1, wd, ROLE_COMPUTE, blk_id) ||
                !warp_wait(bar(C::B_SDP_FULL), n & 1, wd, ROLE_COMPUTE, blk_id)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const bool need_mask = (causal && q0 < k0 + BK) || (q0 + BQ > N) || (k0 + BK > N);
            const float* vl = reinterpret_cast<const float*>(smem + C::OFF_VEC + s * C::VEC_BYTES);
            const float* vd = vl + BQ;
            const uint32_t sds = sbase + C::OFF_DS + db * C::DS_BYTES;
            constexpr int CHUNKS = (BQ / 2) / 32;
#pragma unroll 1
            for (int c = 0; c < CHUNKS; ++c) {
                const int col0 = half * (BQ / 2) + c * 32;
                uint32_t sv[32], dpv[32];
                tmem_ld32(tmem + lane_base + C::TM_S + col0, sv);
                tmem_ld32(tmem + lane_base + C::TM_DP + col0, dpv);
                if (c == CHUNKS - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(C::B_SDP_FREE));
                }
                uint32_t pu[16], du[16];
                if (need_mask)
                    p_ds_chunk<true>(sv, dpv, vl + col0, vd + col0, cs, q0 + col0, key, N, causal,
                                     pu, du);
                else
                    p_ds_chunk<false>(sv, dpv, vl + col0, vd + col0, cs, q0 + col0, key, N, causal,
                                      pu, du);
                if (c == 0) {
                    // The P columns (dQ region) are free once the dQ warps have
                    // read dQ of step n - 1; dS buffer db once dK and dQ of
                    // step n - 2 have run.
                    if (n >= 1 && !warp_wait(bar(C::B_DQ_EMPTY), (n - 1) & 1, wd, ROLE_COMPUTE,
                                             blk_id)) {
                        ok = false;
                        break;
                    }
                    if (n >= 2 && !warp_wait(bar(C::B_DS_FREE + db), ((n / 2) - 1) & 1, wd,
                                             ROLE_COMPUTE, blk_id)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                }
                tmem_st16(tmem + lane_base + C::TM_P + col0 / 2, pu);
                // dS row r, queries col0..col0+31, in the 128-byte-swizzled
                // layout (16-byte chunk index XOR row % 8 inside 1 KiB atoms).
                const uint32_t row_base = sds + (col0 / 64) * C::DS_SLAB + (r / 8) * 1024 +
                                          (r % 8) * 128;
                const int ch0 = (col0 % 64) / 8;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const uint32_t phys = uint32_t((ch0 + k4) ^ (r % 8));
                    st_shared_v4(row_base + phys * 16, du[4 * k4], du[4 * k4 + 1], du[4 * k4 + 2],
                                 du[4 * k4 + 3]);
                }
            }
            if (!ok) break;
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(C::B_DS_READY + db));
                mbar_arrive(bar(C::B_QD_EMPTY + s));
            }
        }
        // Epilogue: dV and scale * dK of this warp's rows and column half.
        if (ok && warp_wait(bar(C::B_ACC_FULL), 0, wd, ROLE_COMPUTE, blk_id)) {
            tc_fence_after();
            constexpr int HC = D / 2;                         // columns per half
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const uint32_t tcol = (which == 0 ? C::TM_DV : C::TM_DK) + half * HC;
                const float mul = which == 0 ? 1.f : scale;
                __nv_bfloat16* dst = (which == 0 ? dv + sdv.row(bh, H, key) : dk + sdk.row(bh, H, key)) +
                                     half * HC;
#pragma unroll
                for (int c = 0; c < HC / 32; ++c) {
                    uint32_t x[32];
                    tmem_ld32(tmem + lane_base + tcol + c * 32, x);
                    if (key < N) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            uint4 w;
                            w.x = pack_bf16x2(mul * __uint_as_float(x[8 * k4 + 0]),
                                              mul * __uint_as_float(x[8 * k4 + 1]));
                            w.y = pack_bf16x2(mul * __uint_as_float(x[8 * k4 + 2]),
                                              mul * __uint_as_float(x[8 * k4 + 3]));
                            w.z = pack_bf16x2(mul * __uint_as_float(x[8 * k4 + 4]),
                                              mul * __uint_as_float(x[8 * k4 + 5]));
                            w.w = pack_bf16x2(mul * __uint_as_float(x[8 * k4 + 6]),
                                              mul * __uint_as_float(x[8 * k4 + 7]));
                            d4[k4] = w;
                        }
                    }
                }
            }
        }
    }

    __syncwarp();          // single-lane roles rejoin their warps before the aligned barrier
    tc_fence_before();
    cta_sync();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TM_COLS);
    }
}

// ---------------------------------------------------------------------------
// d = 128 kernel: 128 query rows per step, every MMA at M = N = 128.
//
// TMEM holds dV and dK (128 columns each) and two 128-column regions:
//   X  S^T of the step, then dP^T of the step once the compute warps have
//      read S^T;
//   Y  P of the step as bf16 pairs (columns 0-63, written by the compute
//      warps once the dQ warps have read those columns of the previous
//      dQ^T), then dQ^T of the step (the dQ MMA is issued after the dV MMA
//      that reads P, and after the dQ warps have read all of the previous
//      dQ^T).
// K stays in shared memory, so S^T = K Q^T and dP^T = V dO^T are SS
// products.  Per step n the MMA thread issues
//   (S^T(n) read) dP^T(n) | (P(n) in Y) dV(n) | (dP^T(n) read) S^T(n+1) |
//   (dS(n) written) dK(n), dQ(n)
// so the compute warps' exponentials of step n+1 run while the tensor core
// works on the gradients of step n, dV(n) runs while dS(n) is computed, and
// the Q / dO stage of step n is released right after dK(n).
// 512 threads: warps 0-7 compute, 8-11 dQ drain, 12 MMA, 13 TMA, 14-15 idle;
// the compute warpgroups take 176 registers, the dQ warpgroup 72 and the
// last warpgroup 80 (setmaxnreg, from 128 at launch).
// ---------------------------------------------------------------------------
struct CfgX {
    static constexpr int D = 128;
    static constexpr int BQ = 128;
    static constexpr int NSX = 2;                        // Q / dO stages
    static constexpr int THREADS = 512;
    static constexpr int REGS_LAUNCH = 128;
    static constexpr int REGS_COMPUTE = 176;
    static constexpr int REGS_DQ = 72;
    static constexpr int REGS_OTHER = 80;
    static_assert(256 * REGS_COMPUTE + 128 * REGS_DQ + 128 * REGS_OTHER <=
                      THREADS * REGS_LAUNCH,
                  "setmaxnreg split within the launch's registers");
    static constexpr int KV_BYTES = BK * D * 2;          // 32 KiB
    static constexpr int KV_SLAB = BK * 128;             // 64 columns of a K / V tile
    static constexpr int QD_BYTES = BQ * D * 2;          // 32 KiB
    static constexpr int QD_SLAB = BQ * 128;             // 64 columns of a Q / dO tile
    static constexpr int DS_BYTES = BK * BQ * 2;         // 32 KiB
    static constexpr int DS_SLAB = BK * 128;             // 64 queries of dS, all keys
    static constexpr int VEC_BYTES = 2 * BQ * 4;         // -LSE2 and -D of one query block
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KV_BYTES;
    static constexpr int OFF_Q = OFF_V + KV_BYTES;
    static constexpr int OFF_DO = OFF_Q + NSX * QD_BYTES;
    static constexpr int OFF_DS = OFF_DO + NSX * QD_BYTES;
    static constexpr int OFF_VEC = OFF_DS + DS_BYTES;
    static constexpr int OFF_BAR = OFF_VEC + NSX * VEC_BYTES;
    static constexpr int B_KV_FULL = 0;
    static constexpr int B_QD_FULL = 1;                  // [NSX]
    static constexpr int B_QD_EMPTY = 1 + NSX;           // [NSX]
    static constexpr int B_S_FULL = 1 + 2 * NSX;
    static constexpr int B_S_FREE = 2 + 2 * NSX;
    static constexpr int B_DP_FULL = 3 + 2 * NSX;
    static constexpr int B_DS_READY = 4 + 2 * NSX;
    static constexpr int B_DQ_FULL = 5 + 2 * NSX;
    static constexpr int B_DQ_EMPTY = 6 + 2 * NSX;
    static constexpr int B_ACC_FULL = 7 + 2 * NSX;
    static constexpr int B_DRAIN = 8 + 2 * NSX;
    static constexpr int B_DP_FREE = 9 + 2 * NSX;
    static constexpr int B_DQ_LO_EMPTY = 10 + 2 * NSX;   // Y's P columns read
    static constexpr int B_P_READY = 11 + 2 * NSX;       // P of the step in Y
    static constexpr int NUM_BARS = 12 + 2 * NSX;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;   // tmem base, abort flag
    static constexpr int BYTES = OFF_MISC + 16;
    // The whole 227 KiB: what is left over after BYTES absorbs the rounding
    // of the dynamic shared-memory base up to 1 KiB (checked in the kernel).
    static constexpr int ALLOC = 227 * 1024;
    static_assert(BYTES <= ALLOC, "shared memory budget");
    static constexpr uint32_t TM_X = 0;                  // S^T, then dP^T
    static constexpr uint32_t TM_DQ = 128;               // Y: P, then dQ^T (d on the lanes)
    static constexpr uint32_t TM_DV = 256;
    static constexpr uint32_t TM_DK = 384;
    static constexpr uint32_t TM_COLS = 512;
};

// p = 2^(s * scale log2(e) - LSE2) for 32 query columns of one key row, with
// the same masking as p_ds_chunk; kept in fp32 for dS.
template <bool MASK>
__device__ __forceinline__ void p_chunk(const uint32_t* sv, const float* nl, float cs, int qi0,
                                        int key, int N, int causal, float* p) {
    const uint64_t cs2 = f2_pack(cs, cs);
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(nl + j);
        const uint64_t x01 = f2_fma(f2_pack(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])),
                                    cs2, f2_pack(l4.x, l4.y));
        const uint64_t x23 = f2_fma(
            f2_pack(__uint_as_float(sv[j + 2]), __uint_as_float(sv[j + 3])), cs2,
            f2_pack(l4.z, l4.w));
        float x[4];
        f2_unpack(x01, x[0], x[1]);
        f2_unpack(x23, x[2], x[3]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            p[j + u] = ex2(x[u]);
            if (MASK) {
                const int qi = qi0 + j + u;
                if ((causal && qi < key) || qi >= N || key >= N) p[j + u] = 0.f;
            }
        }
    }
}

// ds = p * (dP - D) for 32 query columns, rounded to bf16 pairs.
__device__ __forceinline__ void ds_chunk(const float* p, const uint32_t* dpv,
                                         const float* nd, uint32_t (&du)[16]) {
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        const float4 d4 = *reinterpret_cast<const float4*>(nd + j);
        const uint64_t t01 = f2_add(
            f2_pack(__uint_as_float(dpv[j]), __uint_as_float(dpv[j + 1])), f2_pack(d4.x, d4.y));
        const uint64_t t23 = f2_add(
            f2_pack(__uint_as_float(dpv[j + 2]), __uint_as_float(dpv[j + 3])),
            f2_pack(d4.z, d4.w));
        float ds[4];
        f2_unpack(f2_mul(f2_pack(p[j], p[j + 1]), t01), ds[0], ds[1]);
        f2_unpack(f2_mul(f2_pack(p[j + 2], p[j + 3]), t23), ds[2], ds[3]);
        du[j / 2] = pack_bf16x2(ds[0], ds[1]);
        du[j / 2 + 1] = pack_bf16x2(ds[2], ds[3]);
    }
}

__device__ __forceinline__ void cta_sync_x() {
    asm volatile("bar.sync 0, %0;" ::"n"(CfgX::THREADS) : "memory");
}

__global__ void __launch_bounds__(CfgX::THREADS, 1)
bwd_kernel_x(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
             const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
             const float* __restrict__ nlse2, const float* __restrict__ ndvec,
             float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dk,
             __nv_bfloat16* __restrict__ dv, int BH, int H, int N, int Npad, int causal,
             float scale, int hg, unsigned long long watchdog_ns, int inject, St3 sdk, St3 sdv) {
    using X = CfgX;
    constexpr int D = X::D;
    constexpr int BQ = X::BQ;
    constexpr int NSX = X::NSX;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // The layout needs BYTES from a 1 KiB boundary; the allocation leaves
    // ALLOC - BYTES for the rounding.  If the base is placed worse than that,
    // every thread leaves before touching shared memory or TMEM.
    if (smem + X::BYTES > smem_raw + X::ALLOC) {
        if (threadIdx.x == 0)
            atomicCAS(&g_bwd_status, 0u, (uint32_t(FA_ERR_LAUNCH) << 24) | (ROLE_DRAIN << 20));
        return;
    }
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bar0 = sbase + X::OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + X::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + X::OFF_MISC + 4);

    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    // Work order as in bwd_kernel: head groups of hg, key-block-major inside.
    const int nkb = (N + BK - 1) / BK;
    const int per_group = hg * nkb;
    const int g = int(blockIdx.x) / per_group;
    const int r_in = int(blockIdx.x) - g * per_group;
    const int gh = min(hg, BH - g * hg);
    const int kb = r_in / gh;
    const int bh = g * hg + (r_in - kb * gh);
    const int b = bh / H, h = bh - (bh / H) * H;
    const int k0 = kb * BK;
    const int nqb = (N + BQ - 1) / BQ;
    const int qb_first = causal ? k0 / BQ : 0;
    const int nsteps = nqb - qb_first;

    if (threadIdx.x == 0) {
        mbar_init(bar(X::B_KV_FULL), 1);
        for (int s = 0; s < NSX; ++s) {
            mbar_init(bar(X::B_QD_FULL + s), 1);
            mbar_init(bar(X::B_QD_EMPTY + s), 1);
        }
        mbar_init(bar(X::B_S_FULL), 1);
        mbar_init(bar(X::B_S_FREE), COMPUTE_WARPS);
        mbar_init(bar(X::B_DP_FULL), 1);
        mbar_init(bar(X::B_DP_FREE), COMPUTE_WARPS);
        mbar_init(bar(X::B_DS_READY), COMPUTE_WARPS);
        mbar_init(bar(X::B_DQ_FULL), 1);
        mbar_init(bar(X::B_DQ_EMPTY), 4);
        mbar_init(bar(X::B_DQ_LO_EMPTY), 4);
        mbar_init(bar(X::B_P_READY), COMPUTE_WARPS);
        mbar_init(bar(X::B_ACC_FULL), 1);
        mbar_init(bar(X::B_DRAIN), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == MMA_WARP) {
        tmem_alloc(smem_addr(tmem_slot), X::TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    cta_sync_x();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const Watchdog wd{abort_flag, watchdog_ns};
    const uint32_t blk_id = blockIdx.x;

    if (warp >= MMA_WARP) {
        regs_dec<X::REGS_OTHER>();
        if (warp == TMA_WARP && lane == 0) {
            // ------------------------------------------------------------------
            // Producer: K, V once; then Q, dO, -LSE2, -D of each query block.
            // ------------------------------------------------------------------
            mbar_arrive_expect_tx(bar(X::B_KV_FULL), 2 * X::KV_BYTES);
#pragma unroll
            for (int sl = 0; sl < D / 64; ++sl) {
                tma_load_4d(sbase + X::OFF_K + sl * X::KV_SLAB, &tmK, sl * 64, k0, h, b,
                            bar(X::B_KV_FULL));
                tma_load_4d(sbase + X::OFF_V + sl * X::KV_SLAB, &tmV, sl * 64, k0, h, b,
                            bar(X::B_KV_FULL));
            }
            int issued = 0;
            // Host-chosen fault injection (inject = 1): CTA 0 never issues its
            // first Q / dO block, so the waits on it can only end by the watchdog.
            const bool skip0 = inject == 1 && blockIdx.x == 0;
            for (int n = 0; n < nsteps; ++n) {
                const int s = n % NSX;
                if (n >= NSX && !wait_phase(bar(X::B_QD_EMPTY + s), ((n / NSX) - 1) & 1, wd,
                                            ROLE_PRODUCER, blk_id))
                    break;
                ++issued;
                if (skip0 && n == 0) continue;
                const int q0 = (qb_first + n) * BQ;
                const uint32_t full = bar(X::B_QD_FULL + s);
                mbar_arrive_expect_tx(full, 2 * X::QD_BYTES + X::VEC_BYTES);
#pragma unroll
                for (int sl = 0; sl < D / 64; ++sl) {
                    tma_load_4d(sbase + X::OFF_Q + s * X::QD_BYTES + sl * X::QD_SLAB, &tmQ,
                                sl * 64, q0, h, b, full);
                    tma_load_4d(sbase + X::OFF_DO + s * X::QD_BYTES + sl * X::QD_SLAB, &tmDO,
                                sl * 64, q0, h, b, full);
                }
                const long long vrow = (long long)bh * Npad + q0;
                bulk_load(sbase + X::OFF_VEC + s * X::VEC_BYTES, nlse2 + vrow, BQ * 4, full);
                bulk_load(sbase + X::OFF_VEC + s * X::VEC_BYTES + BQ * 4, ndvec + vrow, BQ * 4,
                          full);
            }
            // Drain: every copy this thread issued has landed before exit.
            wait_drain(bar(X::B_KV_FULL), 0, watchdog_ns);
            for (int n = (issued > NSX ? issued - NSX : 0); n < issued; ++n)
                if (!(skip0 && n == 0))
                    wait_drain(bar(X::B_QD_FULL + n % NSX), (n / NSX) & 1, watchdog_ns);
        } else if (warp == MMA_WARP && lane == 0) {
            // ------------------------------------------------------------------
            // MMA issuer
            // ------------------------------------------------------------------
            constexpr uint32_t ID_S = idesc_bf16(128, BQ, false);          // S^T, dP^T
            constexpr uint32_t ID_G = idesc_bf16(128, D, true);            // dV, dK
            constexpr uint32_t ID_Q = idesc_bf16(128, BQ, true, true);     // dQ^T = K^T dS^T
            const uint64_t k_kmaj = sdesc_sw128(sbase + X::OFF_K, 16, 1024);
            const uint64_t v_kmaj = sdesc_sw128(sbase + X::OFF_V, 16, 1024);
            const uint64_t k_mn = sdesc_sw128(sbase + X::OFF_K, X::KV_SLAB, 1024);
            const uint64_t ds_kmaj = sdesc_sw128(sbase + X::OFF_DS, 16, 1024);
            const uint64_t ds_mn = sdesc_sw128(sbase + X::OFF_DS, X::DS_SLAB, 1024);
            bool ok = wait_phase(bar(X::B_KV_FULL), 0, wd, ROLE_MMA, blk_id);
            tc_fence_after();

            // S^T = K Q^T for step m into X: A = K K-major, B = Q K-major.
            auto s_of = [&](int m) -> bool {
                const int sm = m % NSX;
                if (!wait_phase(bar(X::B_QD_FULL + sm), (m / NSX) & 1, wd, ROLE_MMA, blk_id))
                    return false;
                tc_fence_after();
                const uint64_t q_kmaj = sdesc_sw128(sbase + X::OFF_Q + sm * X::QD_BYTES, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t oa = uint32_t(((kk / 4) * X::KV_SLAB + (kk % 4) * 32) >> 4);
                    const uint32_t ob = uint32_t(((kk / 4) * X::QD_SLAB + (kk % 4) * 32) >> 4);
                    mma_ss(tmem + X::TM_X, desc_add(k_kmaj, oa), desc_add(q_kmaj, ob), ID_S,
                           kk > 0 ? 1u : 0u);
                }
                tc_commit(bar(X::B_S_FULL));
                return true;
            };
            if (ok) ok = s_of(0);
            for (int n = 0; ok && n < nsteps; ++n) {
                const int s = n % NSX;
                const uint32_t sq = sbase + X::OFF_Q + s * X::QD_BYTES;
                const uint32_t sdo = sbase + X::OFF_DO + s * X::QD_BYTES;
                // dP^T = V dO^T into X once every compute warp has read S^T(n).
                if (!wait_phase(bar(X::B_S_FREE), n & 1, wd, ROLE_MMA, blk_id)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t do_kmaj = sdesc_sw128(sdo, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t oa = uint32_t(((kk / 4) * X::KV_SLAB + (kk % 4) * 32) >> 4);
                    const uint32_t ob = uint32_t(((kk / 4) * X::QD_SLAB + (kk % 4) * 32) >> 4);
                    mma_ss(tmem + X::TM_X, desc_add(v_kmaj, oa), desc_add(do_kmaj, ob), ID_S,
                           kk > 0 ? 1u : 0u);
                }
                tc_commit(bar(X::B_DP_FULL));
                // dV += P^T dO once P(n) is in Y: A = P from TMEM (16 queries =
                // 8 columns per step), B = dO MN-major (16 query rows of 128
                // bytes).
                if (!wait_phase(bar(X::B_P_READY), n & 1, wd, ROLE_MMA, blk_id)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t do_mn = sdesc_sw128(sdo, X::QD_SLAB, 1024);
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk)
                    mma_ts(tmem + X::TM_DV, tmem + X::TM_DQ + uint32_t(kk * 8),
                           desc_add(do_mn, uint32_t((kk * 2048) >> 4)), ID_G,
                           (n > 0 || kk > 0) ? 1u : 0u);
                // S^T(n+1) into X once every compute warp has read dP^T(n).
                if (!wait_phase(bar(X::B_DP_FREE), n & 1, wd, ROLE_MMA, blk_id)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (n + 1 < nsteps && !s_of(n + 1)) {
                    ok = false;
                    break;
                }
                // Once dS(n) is in shared memory: dK += dS^T Q: A = dS K-major
                // (keys x queries), B = Q MN-major.
                if (!wait_phase(bar(X::B_DS_READY), n & 1, wd, ROLE_MMA, blk_id)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t q_mn = sdesc_sw128(sq, X::QD_SLAB, 1024);
#pragma unroll
                for (int kk = 0; kk < BQ / 16; ++kk)
                    mma_ss(tmem + X::TM_DK,
                           desc_add(ds_kmaj, uint32_t(((kk / 4) * X::DS_SLAB + (kk % 4) * 32) >> 4)),
                           desc_add(q_mn, uint32_t((kk * 2048) >> 4)), ID_G,
                           (n > 0 || kk > 0) ? 1u : 0u);
                // Q, dO (and -LSE2, -D, read before DS_READY) of step n are
                // no longer needed: the producer may refill the stage.
                tc_commit(bar(X::B_QD_EMPTY + s));
                // dQ^T = K^T dS^T into Y (after the dV MMA that read P, and
                // once the dQ warps have read all of dQ^T(n-1)): A = K MN-major
                // (d x keys), B = dS^T MN-major (queries x keys), 16 keys per
                // step.  With d on the TMEM lanes the dQ warps' reductions
                // cover whole 128-byte lines.
                if (n >= 1 && !wait_phase(bar(X::B_DQ_EMPTY), (n - 1) & 1, wd, ROLE_MMA, blk_id)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint32_t off = uint32_t((kk * 2048) >> 4);
                    mma_ss(tmem + X::TM_DQ, desc_add(k_mn, off), desc_add(ds_mn, off), ID_Q,
                           kk > 0 ? 1u : 0u);
                }
                tc_commit(bar(X::B_DQ_FULL));
            }
            if (ok) tc_commit(bar(X::B_ACC_FULL));
            // Drain: every MMA this thread issued has completed before TMEM is freed.
            tc_commit(bar(X::B_DRAIN));
            wait_drain(bar(X::B_DRAIN), 0, watchdog_ns);
        }
    } else if (warp >= DQ_WARP0) {
        regs_dec<X::REGS_DQ>();
        // ------------------------------------------------------------------
        // dQ drain: TMEM (lane = d index, columns = the step's queries) ->
        // fp32 reductions, a warp covering 32 consecutive d of one row.
        // ------------------------------------------------------------------
        const int qw = warp - DQ_WARP0;                       // lane quarter
        const uint32_t lane_base = uint32_t(32 * qw) << 16;
        const int t = 32 * qw + lane;
        for (int n = 0; n < nsteps; ++n) {
            if (!warp_wait(bar(X::B_DQ_FULL), n & 1, wd, ROLE_DQ, blk_id)) break;
            tc_fence_after();
            const int q0 = (qb_first + n) * BQ;
            const int rows = min(BQ, N - q0);
            float* base = dq_acc + ((long long)bh * Npad + q0) * D + t;
            // Two halves of 64 queries: the first half's columns are where the
            // compute warps put P of the next step, so they are released
            // (DQ_LO_EMPTY) before any reduction is issued; the whole region
            // (DQ_EMPTY) before the next dQ MMA.
#pragma unroll
            for (int hq = 0; hq < 2; ++hq) {
                uint32_t r[64];
                tmem_ld32(tmem + lane_base + X::TM_DQ + hq * 64, *reinterpret_cast<uint32_t(*)[32]>(r));
                tmem_ld32(tmem + lane_base + X::TM_DQ + hq * 64 + 32,
                          *reinterpret_cast<uint32_t(*)[32]>(r + 32));
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(hq == 0 ? X::B_DQ_LO_EMPTY : X::B_DQ_EMPTY));
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (hq * 64 + j < rows)
                        red_add_f32(base + (long long)(hq * 64 + j) * D, __uint_as_float(r[j]));
            }
        }
    } else {
        regs_inc<X::REGS_COMPUTE>();
        // ------------------------------------------------------------------
        // Compute warps: key row r (TMEM lane), query columns half*64 ..
        // half*64+63.
        // ------------------------------------------------------------------
        const int qw = warp % 4, half = warp / 4;
        const int r = 32 * qw + lane;                         // key row in the block
        const int key = k0 + r;
        const uint32_t lane_base = uint32_t(32 * qw) << 16;
        const uint32_t xcol = X::TM_X + uint32_t(half * 64);  // this warp's X columns
        const float cs = scale * LOG2E;
        bool ok = true;
        for (int n = 0; ok && n < nsteps; ++n) {
            const int s = n % NSX;
            const int q0 = (qb_first + n) * BQ;
            // QD_FULL: -LSE2 / -D of this block have landed; S_FULL: S^T in X.
            if (!warp_wait(bar(X::B_QD_FULL + s), (n / NSX) & 1, wd, ROLE_COMPUTE, blk_id) ||
                !warp_wait(bar(X::B_S_FULL), n & 1, wd, ROLE_COMPUTE, blk_id)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const bool need_mask = (causal && q0 < k0 + BK) || (q0 + BQ > N) || (k0 + BK > N);
            const float* vl = reinterpret_cast<const float*>(smem + X::OFF_VEC + s * X::VEC_BYTES) +
                              half * 64;
            const float* vd = vl + BQ;
            const int qi0 = q0 + half * 64;
            float p[64];
            {
                uint32_t sv[64];
                tmem_ld32(tmem + lane_base + xcol, *reinterpret_cast<uint32_t(*)[32]>(sv));
                tmem_ld32(tmem + lane_base + xcol + 32,
                          *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(X::B_S_FREE));
                if (need_mask) {
                    p_chunk<true>(sv, vl, cs, qi0, key, N, causal, p);
                    p_chunk<true>(sv + 32, vl + 32, cs, qi0 + 32, key, N, causal, p + 32);
                } else {
                    p_chunk<false>(sv, vl, cs, qi0, key, N, causal, p);
                    p_chunk<false>(sv + 32, vl + 32, cs, qi0 + 32, key, N, causal, p + 32);
                }
            }
            // P(n) into Y (queries half*64 .. +63 at columns half*32 .. +31)
            // once the dQ warps have read those columns of dQ^T(n-1); the dV
            // MMA can then start before dP^T(n) is read.
            {
                uint32_t pu[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) pu[i] = pack_bf16x2(p[2 * i], p[2 * i + 1]);
                if (n >= 1 &&
                    !warp_wait(bar(X::B_DQ_LO_EMPTY), (n - 1) & 1, wd, ROLE_COMPUTE, blk_id)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                tmem_st16(tmem + lane_base + X::TM_DQ + uint32_t(half * 32), pu);
                tmem_st16(tmem + lane_base + X::TM_DQ + uint32_t(half * 32 + 16), pu + 16);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(X::B_P_READY));
            }
            // DP_FULL: dP^T in X; it also follows dK and dQ of step n-1, so
            // the dS buffer is free.
            if (!warp_wait(bar(X::B_DP_FULL), n & 1, wd, ROLE_COMPUTE, blk_id)) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                uint32_t dpv[64];
                tmem_ld32(tmem + lane_base + xcol, *reinterpret_cast<uint32_t(*)[32]>(dpv));
                tmem_ld32(tmem + lane_base + xcol + 32,
                          *reinterpret_cast<uint32_t(*)[32]>(dpv + 32));
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(X::B_DP_FREE));
                const uint32_t sds = sbase + X::OFF_DS;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t du[16];
                    ds_chunk(p + c * 32, dpv + c * 32, vd + c * 32, du);
                    // dS row r, queries half*64 + 32c .. +31, 128-byte swizzled
                    // (16-byte chunk index XOR row % 8 inside 1 KiB atoms).
                    const uint32_t row_base =
                        sds + half * X::DS_SLAB + (r / 8) * 1024 + (r % 8) * 128;
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const uint32_t phys = uint32_t((c * 4 + k4) ^ (r % 8));
                        st_shared_v4(row_base + phys * 16, du[4 * k4], du[4 * k4 + 1],
                                     du[4 * k4 + 2], du[4 * k4 + 3]);
                    }
                }
            }
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(X::B_DS_READY));
        }
        // Epilogue: dV and scale * dK of this warp's rows and column half.
        if (ok && warp_wait(bar(X::B_ACC_FULL), 0, wd, ROLE_COMPUTE, blk_id)) {
            tc_fence_after();
            constexpr int HC = D / 2;                         // columns per half
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const uint32_t tcol = (which == 0 ? X::TM_DV : X::TM_DK) + half * HC;
                const float mul = which == 0 ? 1.f : scale;
                __nv_bfloat16* dst =
                    (which == 0 ? dv + sdv.row(bh, H, key) : dk + sdk.row(bh, H, key)) + half * HC;
#pragma unroll
                for (int c = 0; c < HC / 32; ++c) {
                    uint32_t x[32];
                    tmem_ld32(tmem + lane_base + tcol + c * 32, x);
                    if (key < N) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            uint4 w;
                            w.x = pack_bf16x2(mul * __uint_as_float(x[8 * k4 + 0]),
                                              mul * __uint_as_float(x[8 * k4 + 1]));
                            w.y = pack_bf16x2(mul * __uint_as_float(x[8 * k4 + 2]),
                                              mul * __uint_as_float(x[8 * k4 + 3]));
                            w.z = pack_bf16x2(mul * __uint_as_float(x[8 * k4 + 4]),
                                              mul * __uint_as_float(x[8 * k4 + 5]));
                            w.w = pack_bf16x2(mul * __uint_as_float(x[8 * k4 + 6]),
                                              mul * __uint_as_float(x[8 * k4 + 7]));
                            d4[k4] = w;
                        }
                    }
                }
            }
        }
    }
    // Teardown: after every thread is done with TMEM, the allocating warp frees it.
    tc_fence_before();
    cta_sync_x();
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, X::TM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;             // current_device() accepts indices below this

long long npad_of(int N) { return ((long long)N + BK - 1) / BK * BK; }

struct WsLayout {
    size_t dq_acc, nlse2, ndvec, total;
};

WsLayout ws_layout(long long BH, int N, int d) {
    const long long np = npad_of(N);
    WsLayout w;
    w.dq_acc = 0;
    w.nlse2 = size_t(BH * np * d * 4);
    w.ndvec = w.nlse2 + size_t(BH * np * 4);
    w.total = w.ndvec + size_t(BH * np * 4);
    return w;
}

template <int D>
fa_status launch(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, int B, int H, int N,
                 const St3 (&st)[8], int causal, float scale, unsigned char* ws,
                 cudaStream_t stream, int dev, unsigned long long wd_ns, int inject) {
    using C = Cfg<64>;                 // bwd_kernel's layout (the d = 64 path)
    const long long BH = (long long)B * H;
    const long long np = npad_of(N);
    const WsLayout wl = ws_layout(BH, N, D);
    float* dq_acc = reinterpret_cast<float*>(ws + wl.dq_acc);
    float* nlse2 = reinterpret_cast<float*>(ws + wl.nlse2);
    float* ndvec = reinterpret_cast<float*>(ws + wl.ndvec);

    // Operand order of st: q, k, v, o, dout, dq, dk, dv.
    CUtensorMap mq, mk, mv, mdo;
    auto enc = [&](CUtensorMap* m, const void* p, const St3& x, int rows) {
        return fa_internal::encode_bhnd_map(m, p, D, N, H, B, x.b, x.h, x.n, rows);
    };
    // d = 128 runs bwd_kernel_x (128 query rows per step), d = 64 bwd_kernel.
    constexpr bool WIDE = D == 128;
    constexpr int BQ = WIDE ? CfgX::BQ : C::BQ;
    constexpr int ALLOC = WIDE ? CfgX::ALLOC : C::ALLOC;
    if (enc(&mq, q, st[0], BQ) != FA_OK || enc(&mk, k, st[1], BK) != FA_OK ||
        enc(&mv, v, st[2], BK) != FA_OK || enc(&mdo, dout, st[4], BQ) != FA_OK)
        return FA_ERR_UNSUPPORTED;

    // The dynamic shared-memory limit is a per-device function attribute: set
    // once per (instantiation, device).  bwd_kernel_x's setmaxnreg split needs
    // the launch to give every thread CfgX::REGS_LAUNCH registers: its
    // compiled count is checked once per device as well.
    static std::once_flag once[kMaxDevices];
    static cudaError_t attr_err[kMaxDevices];
    static int regs[kMaxDevices];
    std::call_once(once[dev], [&] {
        const void* fn;
        if constexpr (WIDE)
            fn = reinterpret_cast<const void*>(bwd_kernel_x);
        else
            fn = reinterpret_cast<const void*>(bwd_kernel<64>);
        attr_err[dev] = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             ALLOC);
        cudaFuncAttributes fa_attr{};
        if (attr_err[dev] == cudaSuccess) attr_err[dev] = cudaFuncGetAttributes(&fa_attr, fn);
        regs[dev] = fa_attr.numRegs;
    });
    cudaError_t e = attr_err[dev];
    if (e != cudaSuccess) {
        fa_internal::set_last_cuda_error(int(e));
        return FA_ERR_LAUNCH;
    }
    if (WIDE && regs[dev] != CfgX::REGS_LAUNCH) return FA_ERR_UNSUPPORTED;

    const long long prep_threads = BH * np * (D / 8);
    bwd_prep<D><<<unsigned((prep_threads + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, nlse2,
        ndvec, dq_acc, BH, H, N, int(np), st[3], st[4]);
    const long long nkb = (N + BK - 1) / BK;
    // Heads per group: about 48 MiB of per-head data (Q, dO, K, V in bf16 and
    // the fp32 dQ accumulator, 12 bytes per element of one tensor) so the
    // groups in flight stay inside the 126 MB L2.  A host simulation of the
    // block scheduler puts the tail cost of grouping at <= 1 % for the
    // long causal workloads (one-head groups: 3.4 %).
    const long long head_bytes = 12LL * np * D;
    long long hg = (48LL << 20) / head_bytes;
    hg = hg < 1 ? 1 : (hg > BH ? BH : hg);
    if constexpr (WIDE)
        bwd_kernel_x<<<unsigned(nkb * BH), CfgX::THREADS, CfgX::ALLOC, stream>>>(
            mq, mk, mv, mdo, nlse2, ndvec, dq_acc, static_cast<__nv_bfloat16*>(dk),
            static_cast<__nv_bfloat16*>(dv), int(BH), H, N, int(np), causal, scale, int(hg),
            wd_ns, inject, st[6], st[7]);
    else
        bwd_kernel<64><<<unsigned(nkb * BH), NUM_THREADS, C::ALLOC, stream>>>(
            mq, mk, mv, mdo, nlse2, ndvec, dq_acc, static_cast<__nv_bfloat16*>(dk),
            static_cast<__nv_bfloat16*>(dv), int(BH), H, N, int(np), causal, scale, int(hg),
            wd_ns, inject, st[6], st[7]);
    const long long out_threads = BH * N * (D / 8);
    bwd_dq_out<D><<<unsigned((out_threads + 255) / 256), 256, 0, stream>>>(
        dq_acc, static_cast<__nv_bfloat16*>(dq), BH, H, N, int(np), scale, st[5]);
    e = cudaGetLastError();
    if (e != cudaSuccess) {
        fa_internal::set_last_cuda_error(int(e));
        return FA_ERR_LAUNCH;
    }
    return FA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace bwd

int fa_internal::take_bwd_status(unsigned* word) {
    unsigned w = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&w, bwd::g_bwd_status, sizeof(w));
    const unsigned zero = 0;
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(bwd::g_bwd_status, &zero, sizeof(zero));
    *word = w;
    return int(e);
}

extern "C" {

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
    if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
    if ((long long)B * H > 0x7fffffffLL || N > (1 << 30)) return 0;
    return bwd::ws_layout((long long)B * H, N, d).total;
}

static fa_status bwd_impl(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                          int H, int N, int d, const long long* strides24, int causal, float scale,
                          void* workspace, size_t workspace_bytes, void* stream,
                          unsigned watchdog_ms, int inject) {
    using bwd::aligned;
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace)
        return FA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (inject != 0 && inject != 1) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    const long long BH = (long long)B * H;
    if (BH > 0x7fffffffLL || N > (1 << 30)) return FA_ERR_UNSUPPORTED;
    // One CTA per (key block, batch x head): the grid is a 1-D unsigned count.
    if ((((long long)N + bwd::BK - 1) / bwd::BK) * BH > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    if (workspace_bytes < bwd::ws_layout(BH, N, d).total) return FA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(lse, 4) || !aligned(workspace, 256))
        return FA_ERR_MISALIGNED;
    // Strides of q, k, v, o, dout, dq, dk, dv, each (batch, head, sequence) in
    // elements; NULL means contiguous [B][H][N][d].  Same rules as the
    // forward's: >= d, a multiple of 8 elements (16 bytes), below 2^39; the
    // stride of a dimension of size 1 is never used.
    bwd::St3 st[8];
    for (int i = 0; i < 8; ++i) {
        if (strides24)
            st[i] = bwd::St3{strides24[3 * i], strides24[3 * i + 1], strides24[3 * i + 2]};
        else
            st[i] = bwd::St3{(long long)H * N * d, (long long)N * d, (long long)d};
        if (B == 1) st[i].b = d;
        if (H == 1) st[i].h = d;
        if (N == 1) st[i].n = d;
        for (long long x : {st[i].b, st[i].h, st[i].n}) {
            if (x < d) return FA_ERR_INVALID_ARG;
            if ((x * 2) % 16 != 0) return FA_ERR_MISALIGNED;
            if (x * 2 >= (1LL << 40)) return FA_ERR_UNSUPPORTED;
        }
    }

    int dev = -1, sm_count = 0;
    const int ds = fa_internal::current_device(&dev, &sm_count);
    if (ds != FA_OK) return static_cast<fa_status>(ds);
    const unsigned long long wd_ns = (watchdog_ms ? watchdog_ms : 4000u) * 1000000ull;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    if (d == 64)
        return bwd::launch<64>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, st, causal, scale, ws,
                               s, dev, wd_ns, inject);
    return bwd::launch<128>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, st, causal, scale, ws, s,
                            dev, wd_ns, inject);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                 int causal, float scale, void* workspace, size_t workspace_bytes, void* stream) {
    return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, nullptr, causal, scale,
                    workspace, workspace_bytes, stream, 0, 0);
}

fa_status fa_bwd_strided(const void* q, const void* k, const void* v, const void* o,
                         const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, const long long* strides, int causal, float scale,
                         void* workspace, size_t workspace_bytes, void* stream) {
    if (!strides) return FA_ERR_INVALID_ARG;
    return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, strides, causal, scale,
                    workspace, workspace_bytes, stream, 0, 0);
}

fa_status fa_bwd_debug(const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                       int H, int N, int d, int causal, float scale, void* workspace,
                       size_t workspace_bytes, void* stream, unsigned watchdog_ms, int inject) {
    return bwd_impl(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, nullptr, causal, scale,
                    workspace, workspace_bytes, stream, watchdog_ms, inject);
}

}  // extern "C"
