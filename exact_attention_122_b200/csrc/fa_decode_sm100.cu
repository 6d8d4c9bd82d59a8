// fa_decode_sm100.cu -- decode-shaped exact attention forward (few queries,
// long key sequence) for B200 (sm_100a).
//
// With N_q <= 16 query rows per (batch, head) the score and PV products are
// matrix-vector shaped: about one FLOP per byte of K and V, far below the
// B200 ridge, so this path runs on the CUDA cores and is bound by streaming K
// and V from HBM once.  The keys are split into `splits` contiguous ranges
// processed by separate CTAs; each split keeps the online-softmax running
// state (max m, sum l, rescaled accumulator) of the page "Flash attention
// optimization", section "The fix: tile the computation, never materialize
// the full matrix", and writes its normalised partial output with its
// log-sum-exp.  A second kernel merges the splits with the same rule the page
// uses to merge blocks (scale_old = exp(m_old - m_new), scale_new =
// exp(m_block - m_new)), expressed through the partial log-sum-exps.
//
// Causal masking with N_q < N_k treats the queries as the last N_q positions
// of the key sequence: query i may see key j iff j <= i + N_k - N_q.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "fa.h"
#include "fa_internal.h"

namespace fa_decode {

constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;
constexpr int TILE = 32;      // keys per warp step (one per lane in the score phase)

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// bf16 pair (low, high) of a 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// One split of one (batch, head): keys [k0, k1).  Writes the normalised
// partial output (fp32) and its natural-log LSE (-inf when the split holds no
// allowed key for the row).
template <int NQ, int D>
__global__ void __launch_bounds__(THREADS)
    decode_split_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                        const __nv_bfloat16* __restrict__ V, float* __restrict__ Opart,
                        float* __restrict__ Lpart, int BH, int Nq, int Nk, int causal,
                        float scale_log2, int chunk) {
    constexpr int DL = D / 32;                       // d elements per lane in the PV phase
    __shared__ __align__(16) float sq[NQ][D];        // q * scale * log2(e)
    __shared__ float sm_m[WARPS][NQ], sm_l[WARPS][NQ];
    __shared__ float sm_o[WARPS][NQ][D];

    const int split = blockIdx.x, bh = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k0 = split * chunk;
    const int k1 = min(Nk, k0 + chunk);
    const int off = Nk - Nq;                         // causal: key j allowed iff j <= i + off

    const __nv_bfloat16* Qb = Q + size_t(bh) * Nq * D;
    const __nv_bfloat16* Kb = K + size_t(bh) * Nk * D;
    const __nv_bfloat16* Vb = V + size_t(bh) * Nk * D;
    for (int e = threadIdx.x; e < NQ * D; e += THREADS) {
        const int i = e / D, t = e - (e / D) * D;
        sq[i][t] = i < Nq ? __bfloat162float(Qb[size_t(i) * D + t]) * scale_log2 : 0.f;
    }
    __syncthreads();

    float m[NQ], l[NQ], o[NQ][DL];
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        m[i] = -INFINITY;
        l[i] = 0.f;
#pragma unroll
        for (int e = 0; e < DL; ++e) o[i][e] = 0.f;
    }

    for (int kb = k0 + warp * TILE; kb < k1; kb += WARPS * TILE) {
        // ---- scores: lane = key
        const int j = kb + lane;
        float s[NQ];
#pragma unroll
        for (int i = 0; i < NQ; ++i) s[i] = 0.f;
        if (j < k1) {
            const uint4* krow = reinterpret_cast<const uint4*>(Kb + size_t(j) * D);
#pragma unroll 4
            for (int c = 0; c < D / 8; ++c) {
                const uint4 w = __ldg(krow + c);
                const float kv[8] = {bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y),
                                     bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w)};
#pragma unroll
                for (int i = 0; i < NQ; ++i) {
                    // two 16-byte shared loads feed eight FMAs
                    const float4 qa = *reinterpret_cast<const float4*>(&sq[i][c * 8]);
                    const float4 qb = *reinterpret_cast<const float4*>(&sq[i][c * 8 + 4]);
                    s[i] = fmaf(qa.x, kv[0], s[i]);
                    s[i] = fmaf(qa.y, kv[1], s[i]);
                    s[i] = fmaf(qa.z, kv[2], s[i]);
                    s[i] = fmaf(qa.w, kv[3], s[i]);
                    s[i] = fmaf(qb.x, kv[4], s[i]);
                    s[i] = fmaf(qb.y, kv[5], s[i]);
                    s[i] = fmaf(qb.z, kv[6], s[i]);
                    s[i] = fmaf(qb.w, kv[7], s[i]);
                }
            }
        }
        float p[NQ];
#pragma unroll
        for (int i = 0; i < NQ; ++i) {
            const bool ok = j < k1 && i < Nq && (!causal || j <= i + off);
            const float si = ok ? s[i] : -INFINITY;
            const float m_new = fmaxf(m[i], warp_max(si));
            // m_new = -inf: no allowed key yet for this row; keep the empty state.
            const float alpha = m_new == -INFINITY ? 1.f : ex2(m[i] - m_new);
            p[i] = m_new == -INFINITY ? 0.f : ex2(si - m_new);
            l[i] = l[i] * alpha + p[i];               // per-lane partial sum, shared reference m
#pragma unroll
            for (int e = 0; e < DL; ++e) o[i][e] *= alpha;
            m[i] = m_new;
        }
        // ---- O += P V: lanes split d, p of key jj broadcast from lane jj
        const int nkeys = min(TILE, k1 - kb);
        for (int jj = 0; jj < nkeys; ++jj) {
            const __nv_bfloat16* vrow = Vb + size_t(kb + jj) * D + lane * DL;
            float vv[DL];
            if constexpr (DL == 4) {
                const uint2 w = __ldg(reinterpret_cast<const uint2*>(vrow));
                vv[0] = bf_lo(w.x); vv[1] = bf_hi(w.x); vv[2] = bf_lo(w.y); vv[3] = bf_hi(w.y);
            } else {
                const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(vrow));
                vv[0] = bf_lo(w); vv[1] = bf_hi(w);
            }
#pragma unroll
            for (int i = 0; i < NQ; ++i) {
                const float pj = __shfl_sync(0xffffffffu, p[i], jj);
#pragma unroll
                for (int e = 0; e < DL; ++e) o[i][e] = fmaf(pj, vv[e], o[i][e]);
            }
        }
    }

    // ---- merge the warps of this CTA (same rule, in shared memory)
#pragma unroll
    for (int i = 0; i < NQ; ++i) {
        const float lw = warp_sum(l[i]);
        if (lane == 0) {
            sm_m[warp][i] = m[i];
            sm_l[warp][i] = lw;
        }
#pragma unroll
        for (int e = 0; e < DL; ++e) sm_o[warp][i][lane * DL + e] = o[i][e];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < NQ * D; e += THREADS) {
        const int i = e / D, t = e - (e / D) * D;
        if (i >= Nq) continue;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) M = fmaxf(M, sm_m[w][i]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < WARPS; ++w) {
                const float f = sm_m[w][i] == -INFINITY ? 0.f : ex2(sm_m[w][i] - M);
                L += sm_l[w][i] * f;
                acc += sm_o[w][i][t] * f;
            }
        }
        const size_t row = (size_t(split) * BH + bh) * Nq + i;
        Opart[row * D + t] = L > 0.f ? acc / L : 0.f;
        if (t == 0) Lpart[row] = L > 0.f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
    }
}

// Merge of the splits of one (batch*head, query row): block of D threads,
// thread t = output element t.
template <int D>
__global__ void __launch_bounds__(D)
    decode_merge_kernel(const float* __restrict__ Opart, const float* __restrict__ Lpart,
                        __nv_bfloat16* __restrict__ O, float* __restrict__ LSE, int rows,
                        int splits) {
    const int r = blockIdx.x;                        // (bh, i) flattened
    const int t = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, Lpart[size_t(s) * rows + r]);
    float W = 0.f, acc = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float ls = Lpart[size_t(s) * rows + r];
            if (ls == -INFINITY) continue;
            const float w = __expf(ls - M);
            W += w;
            acc += w * Opart[(size_t(s) * rows + r) * D + t];
        }
    }
    O[size_t(r) * D + t] = __float2bfloat16_rn(W > 0.f ? acc / W : 0.f);
    if (t == 0) LSE[r] = W > 0.f ? M + logf(W) : -INFINITY;
}

int auto_splits(long long BH, int Nk) {
    // At least 8 splits (measured on B200 with B*H = 512, Nk = 32K: 1 split
    // reaches 47 % of the copy bandwidth, 8 or more splits 83 %), enough to
    // cover the SMs twice for small B*H, at least 512 keys per split, at
    // most 64 splits.
    long long s = (2 * 148 + BH - 1) / BH;
    if (s < 8) s = 8;
    const long long by_keys = (Nk + 511) / 512;
    if (s > by_keys) s = by_keys;
    if (s > 64) s = 64;
    return int(s < 1 ? 1 : s);
}

size_t workspace_bytes(long long BH, int Nq, int d, int splits) {
    const size_t rows = size_t(BH) * Nq;
    const size_t o_bytes = size_t(splits) * rows * d * sizeof(float);
    const size_t l_bytes = size_t(splits) * rows * sizeof(float);
    return ((o_bytes + 255) & ~size_t(255)) + l_bytes;
}

template <int NQ, int D>
cudaError_t launch_split(dim3 grid, cudaStream_t s, const void* q, const void* k, const void* v,
                         float* op, float* lp, int BH, int Nq, int Nk, int causal, float sl2,
                         int chunk) {
    decode_split_kernel<NQ, D><<<grid, THREADS, 0, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), op, lp, BH, Nq, Nk, causal, sl2, chunk);
    return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_split(int nq_t, dim3 grid, cudaStream_t s, const void* q, const void* k,
                           const void* v, float* op, float* lp, int BH, int Nq, int Nk, int causal,
                           float sl2, int chunk) {
    switch (nq_t) {
        case 1: return launch_split<1, D>(grid, s, q, k, v, op, lp, BH, Nq, Nk, causal, sl2, chunk);
        case 2: return launch_split<2, D>(grid, s, q, k, v, op, lp, BH, Nq, Nk, causal, sl2, chunk);
        case 4: return launch_split<4, D>(grid, s, q, k, v, op, lp, BH, Nq, Nk, causal, sl2, chunk);
        case 8: return launch_split<8, D>(grid, s, q, k, v, op, lp, BH, Nq, Nk, causal, sl2, chunk);
        default: return launch_split<16, D>(grid, s, q, k, v, op, lp, BH, Nq, Nk, causal, sl2, chunk);
    }
}

}  // namespace fa_decode

extern "C" {

size_t fa_fwd_decode_workspace_bytes(int B, int H, int Nq, int Nk, int d, int num_splits) {
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || (d != 64 && d != 128) || num_splits < 0 ||
        num_splits > FA_DECODE_MAX_SPLITS)
        return 0;
    const long long BH = (long long)B * H;
    const int splits = num_splits ? num_splits : fa_decode::auto_splits(BH, Nk);
    return fa_decode::workspace_bytes(BH, Nq, d, splits);
}

fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int Nq, int Nk, int d, int causal, float scale, int num_splits,
                        void* workspace, size_t ws_bytes, void* stream) {
    if (!q || !k || !v || !o || !lse || !workspace) return FA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
    if (causal && Nq > Nk) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (num_splits < 0 || num_splits > FA_DECODE_MAX_SPLITS) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (Nq > FA_DECODE_MAX_QUERIES) return FA_ERR_UNSUPPORTED;
    if ((long long)B * H > 65535 || Nk > (1 << 30)) return FA_ERR_UNSUPPORTED;
    auto al = [](const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; };
    if (!al(q, 16) || !al(k, 16) || !al(v, 16) || !al(o, 16) || !al(lse, 4) || !al(workspace, 256))
        return FA_ERR_MISALIGNED;
    const long long BH = (long long)B * H;
    const int splits = num_splits ? num_splits : fa_decode::auto_splits(BH, Nk);
    if (ws_bytes < fa_decode::workspace_bytes(BH, Nq, d, splits)) return FA_ERR_INVALID_ARG;

    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        fa_internal::set_last_cuda_error(int(e));
        return FA_ERR_NO_DEVICE;
    }
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return FA_ERR_UNSUPPORTED;

    // Keys per split, a multiple of the 32-key warp step.
    int chunk = int(((long long)Nk + splits - 1) / splits);
    chunk = (chunk + fa_decode::TILE - 1) / fa_decode::TILE * fa_decode::TILE;
    const int used = (Nk + chunk - 1) / chunk;       // splits that hold keys
    float* opart = static_cast<float*>(workspace);
    const size_t o_bytes = size_t(used) * BH * Nq * d * sizeof(float);
    float* lpart = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                            ((o_bytes + 255) & ~size_t(255)));
    const int nq_t = Nq <= 1 ? 1 : Nq <= 2 ? 2 : Nq <= 4 ? 4 : Nq <= 8 ? 8 : 16;
    const float sl2 = scale * 1.4426950408889634f;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const dim3 grid{unsigned(used), unsigned(BH), 1u};
    e = d == 64 ? fa_decode::dispatch_split<64>(nq_t, grid, s, q, k, v, opart, lpart, int(BH), Nq,
                                                 Nk, causal, sl2, chunk)
                : fa_decode::dispatch_split<128>(nq_t, grid, s, q, k, v, opart, lpart, int(BH), Nq,
                                                  Nk, causal, sl2, chunk);
    if (e == cudaSuccess) {
        const int rows = int(BH) * Nq;
        if (d == 64)
            fa_decode::decode_merge_kernel<64><<<rows, 64, 0, s>>>(
                opart, lpart, static_cast<__nv_bfloat16*>(o), lse, rows, used);
        else
            fa_decode::decode_merge_kernel<128><<<rows, 128, 0, s>>>(
                opart, lpart, static_cast<__nv_bfloat16*>(o), lse, rows, used);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) {
        fa_internal::set_last_cuda_error(int(e));
        return FA_ERR_LAUNCH;
    }
    return FA_OK;
}

}  // extern "C"
