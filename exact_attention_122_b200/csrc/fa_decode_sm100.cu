// fa_decode_sm100.cu -- decode-shaped exact attention forward (few queries,
// long key sequence) for B200 (sm_100a).
//
// With N_q query rows per (batch, head) the score and PV products do about
// N_q FLOPs per byte of K and V, far below the B200 ridge, so the path is
// bound by streaming K and V from HBM once.  From N_q = 5 on, the FP32 pipes
// could not keep up with that stream (16 queries need about 100 TFLOP/s at
// the copy bandwidth), so decode_mma_kernel takes the queries in blocks of 16 rows and
// forms both products with the warp-level m16n8k16 bf16 tensor-core MMA.  The
// same kernel serves N_q <= 4: its coalesced, double-buffered cp.async
// staging streams K and V faster than the earlier lane-per-key CUDA-core
// kernel did (measured on B200 at N_q = 1: 6.9 against 5.5 TB/s).  The keys are split into `splits` contiguous ranges
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

#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace fa_decode {

constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------------------
// Split kernel: a CTA takes one key split of one (batch, head) and one block
// of MQ = 16 query rows (m16n8k16; the last block padded with zero rows).  Each warp streams 16-key tiles of its split
// through two shared-memory stages (cp.async), forms S = Q K^T with K
// fragments from ldmatrix, runs the online softmax on the accumulator
// fragments (rows lane/4 and lane/4 + 8, a quad per row), repacks P as the A
// operand and adds P V with V fragments from ldmatrix.trans.  The warps of a
// CTA are merged in shared memory and the splits by decode_merge_kernel,
// with the rescale-and-merge rule of the page section above.
// ---------------------------------------------------------------------------
constexpr int MQ = 16;        // query rows of the tensor-core path
constexpr int KT = 16;        // keys per warp tile

template <int D>
struct MmaSmem {
    static constexpr int ROW = (D + 8) * 2;              // padded bf16 row (conflict-free ldmatrix)
    static constexpr int TILE_BYTES = KT * ROW;          // one K or V tile
    static constexpr int WARP_BYTES = 2 * 2 * TILE_BYTES;  // two stages of (K, V)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_W = MQ * ROW;
    static constexpr int STREAM_BYTES = OFF_W + WARPS * WARP_BYTES;
    // after the key loop the warp area holds the merge buffers
    static constexpr int MERGE_BYTES = WARPS * MQ * (D + 2) * 4;
    static constexpr int ALLOC =
        STREAM_BYTES > OFF_W + MERGE_BYTES ? STREAM_BYTES : OFF_W + MERGE_BYTES;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// 16-byte asynchronous copy; src_bytes = 0 zero-fills without reading.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <int D>
__global__ void __launch_bounds__(THREADS)
    decode_mma_kernel(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                      const __nv_bfloat16* __restrict__ V, float* __restrict__ Opart,
                      float* __restrict__ Lpart, int BH, int Nq, int Nk, int causal,
                      float scale_log2, int chunk) {
    using S = MmaSmem<D>;
    extern __shared__ __align__(16) unsigned char dsm[];
    const uint32_t sb = smem_u32(dsm);
    // Query blocks vary fastest in the launch order, so the CTAs that read
    // the same keys run together and all but one take K and V from L2.
    const int split = blockIdx.y, bh = blockIdx.z;
    const int q0 = blockIdx.x * MQ;                   // first query row of this CTA
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k0 = split * chunk;
    const int k1 = min(Nk, k0 + chunk);
    const int off = Nk - Nq;                          // causal: key j allowed iff j <= i + off
    const __nv_bfloat16* Qb = Q + size_t(bh) * Nq * D;
    const __nv_bfloat16* Kb = K + size_t(bh) * Nk * D;
    const __nv_bfloat16* Vb = V + size_t(bh) * Nk * D;

    // Q rows (zero past N_q) -> shared memory -> A fragments.
    for (int e = threadIdx.x; e < MQ * D / 8; e += THREADS) {
        const int row = e / (D / 8), c = e - (e / (D / 8)) * (D / 8);
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (q0 + row < Nq) x = *reinterpret_cast<const uint4*>(Qb + size_t(q0 + row) * D + c * 8);
        *reinterpret_cast<uint4*>(dsm + S::OFF_Q + row * S::ROW + c * 16) = x;
    }
    __syncthreads();
    const int mi = lane >> 3, mr = lane & 7;          // ldmatrix: matrix index, row in it
    uint32_t qa[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
        ldsm_x4(sb + S::OFF_Q + (mr + (mi & 1) * 8) * S::ROW + (kk * 16 + (mi >> 1) * 8) * 2,
                qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);

    const uint32_t wbase = sb + S::OFF_W + warp * S::WARP_BYTES;
    auto load_tile = [&](int kt, int stage) {
        const uint32_t sk = wbase + stage * 2 * S::TILE_BYTES, sv = sk + S::TILE_BYTES;
#pragma unroll
        for (int i = 0; i < KT * D / 8 / 32; ++i) {
            const int e = lane + 32 * i;
            const int row = e / (D / 8), c = e - (e / (D / 8)) * (D / 8);
            const int key = kt + row;
            const bool in = key < k1;
            const size_t src = size_t(in ? key : k0) * D + c * 8;
            cp_async16(sk + row * S::ROW + c * 16, Kb + src, in ? 16u : 0u);
            cp_async16(sv + row * S::ROW + c * 16, Vb + src, in ? 16u : 0u);
        }
        cp_async_commit();
    };

    const int r0 = lane >> 2, cq = (lane & 3) * 2;    // fragment row and column pair
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float o[D / 8][4];
#pragma unroll
    for (int nb = 0; nb < D / 8; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;

    int kt = k0 + warp * KT;
    if (kt < k1) load_tile(kt, 0);
    for (int t = 0; kt < k1; kt += WARPS * KT, ++t) {
        const int stage = t & 1;
        if (kt + WARPS * KT < k1) {
            load_tile(kt + WARPS * KT, stage ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncwarp();
        const uint32_t sk = wbase + stage * 2 * S::TILE_BYTES, sv = sk + S::TILE_BYTES;
        // S = Q K^T: 16 queries x 16 keys (two n8 blocks).
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            uint32_t b00, b01, b10, b11;
            ldsm_x4(sk + (mr + (mi >> 1) * 8) * S::ROW + (kk * 16 + (mi & 1) * 8) * 2, b00, b01,
                    b10, b11);
            mma_bf16_16816(sc[0], qa[kk], b00, b01);
            mma_bf16_16816(sc[1], qa[kk], b10, b11);
        }
        // Scale to log2 units and mask (keys past the split, causal).
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int key = kt + nb * 8 + cq + (c & 1);
                const int row = q0 + r0 + (c >> 1) * 8;
                const bool ok = key < k1 && (!causal || key <= row + off);
                sc[nb][c] = ok ? sc[nb][c] * scale_log2 : -INFINITY;
            }
        float alpha[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float mt = fmaxf(fmaxf(sc[0][2 * h], sc[0][2 * h + 1]),
                             fmaxf(sc[1][2 * h], sc[1][2 * h + 1]));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
            const float m_new = fmaxf(m[h], mt);
            // m_new = -inf: no allowed key yet for this row; keep the empty state.
            alpha[h] = m_new == -INFINITY ? 1.f : ex2(m[h] - m_new);
            m[h] = m_new;
            l[h] *= alpha[h];
        }
        float p[2][4];
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int h = c >> 1;
                p[nb][c] = m[h] == -INFINITY ? 0.f : ex2(sc[nb][c] - m[h]);
                l[h] += p[nb][c];
            }
#pragma unroll
        for (int nb = 0; nb < D / 8; ++nb) {
            o[nb][0] *= alpha[0];
            o[nb][1] *= alpha[0];
            o[nb][2] *= alpha[1];
            o[nb][3] *= alpha[1];
        }
        const uint32_t pa[4] = {pack_bf16(p[0][0], p[0][1]), pack_bf16(p[0][2], p[0][3]),
                                pack_bf16(p[1][0], p[1][1]), pack_bf16(p[1][2], p[1][3])};
        // O += P V: V fragments (keys x d) through ldmatrix.trans.
#pragma unroll
        for (int db = 0; db < D / 16; ++db) {
            uint32_t v00, v01, v10, v11;
            ldsm_x4_t(sv + (mr + (mi & 1) * 8) * S::ROW + (db * 16 + (mi >> 1) * 8) * 2, v00, v01,
                      v10, v11);
            mma_bf16_16816(o[2 * db], pa, v00, v01);
            mma_bf16_16816(o[2 * db + 1], pa, v10, v11);
        }
        __syncwarp();                                 // this stage is refilled next-but-one tile
    }
    cp_async_wait<0>();

    // Per-row sums over the quad; then merge the warps (shared memory reused).
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
    }
    __syncthreads();
    float* sm_m = reinterpret_cast<float*>(dsm + S::OFF_W);           // [WARPS][MQ]
    float* sm_l = sm_m + WARPS * MQ;                                   // [WARPS][MQ]
    float* sm_o = sm_l + WARPS * MQ;                                   // [WARPS][MQ][D]
    if ((lane & 3) == 0) {
        sm_m[warp * MQ + r0] = m[0];
        sm_m[warp * MQ + r0 + 8] = m[1];
        sm_l[warp * MQ + r0] = l[0];
        sm_l[warp * MQ + r0 + 8] = l[1];
    }
#pragma unroll
    for (int nb = 0; nb < D / 8; ++nb)
#pragma unroll
        for (int c = 0; c < 4; ++c)
            sm_o[(warp * MQ + r0 + (c >> 1) * 8) * D + nb * 8 + cq + (c & 1)] = o[nb][c];
    __syncthreads();
    for (int e = threadIdx.x; e < MQ * D; e += THREADS) {
        const int il = e / D, t = e - (e / D) * D;    // local row, column
        const int i = q0 + il;
        if (i >= Nq) continue;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) M = fmaxf(M, sm_m[w * MQ + il]);
        float L = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < WARPS; ++w) {
                const float mw = sm_m[w * MQ + il];
                const float f = mw == -INFINITY ? 0.f : ex2(mw - M);
                L += sm_l[w * MQ + il] * f;
                acc += sm_o[(w * MQ + il) * D + t] * f;
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

int auto_splits(long long BH, int Nq, int Nk) {
    // Enough CTAs (splits x B*H x query blocks) to cover the SMs twice; with
    // a single query block at least 8 splits (measured on B200 with
    // B*H = 512, Nk = 32K: 1 split reaches 47 % of the copy bandwidth, 8 or
    // more splits 83 %); at least 512 keys per split, at most 64 splits.
    const long long qblocks = (Nq + MQ - 1) / MQ;
    long long s = (2 * 148 + BH * qblocks - 1) / (BH * qblocks);
    if (qblocks == 1 && s < 8) s = 8;
    const long long by_keys = (Nk + 511) / 512;
    if (s > by_keys) s = by_keys;
    if (s > 64) s = 64;
    return int(s < 1 ? 1 : s);
}

// Above this many queries the persistent tiled kernel (128-row tcgen05 tiles)
// does the work; it needs only its 256-byte work counter as workspace.
constexpr int TILED_MIN_NQ = 33;

size_t workspace_bytes(long long BH, int Nq, int d, int splits) {
    if (Nq >= TILED_MIN_NQ) return FA_DYNAMIC_WORKSPACE_BYTES;
    const size_t rows = size_t(BH) * Nq;
    const size_t o_bytes = size_t(splits) * rows * d * sizeof(float);
    const size_t l_bytes = size_t(splits) * rows * sizeof(float);
    return ((o_bytes + 255) & ~size_t(255)) + l_bytes;
}

template <int D>
cudaError_t launch_mma(dim3 grid, cudaStream_t s, const void* q, const void* k, const void* v,
                       float* op, float* lp, int BH, int Nq, int Nk, int causal, float sl2,
                       int chunk) {
    using S = MmaSmem<D>;
    constexpr int kMaxDevices = 64;
    static std::once_flag once[kMaxDevices];
    static cudaError_t attr[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&] {
        attr[dev] = cudaFuncSetAttribute(decode_mma_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, S::ALLOC);
    });
    if (attr[dev] != cudaSuccess) return attr[dev];
    decode_mma_kernel<D><<<grid, THREADS, S::ALLOC, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), op, lp, BH, Nq, Nk, causal, sl2, chunk);
    return cudaGetLastError();
}

}  // namespace fa_decode

extern "C" {

size_t fa_fwd_decode_workspace_bytes(int B, int H, int Nq, int Nk, int d, int num_splits) {
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || (d != 64 && d != 128) || num_splits < 0 ||
        num_splits > FA_DECODE_MAX_SPLITS)
        return 0;
    const long long BH = (long long)B * H;
    const int splits = num_splits ? num_splits : fa_decode::auto_splits(BH, Nq, Nk);
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
    const int splits = num_splits ? num_splits : fa_decode::auto_splits(BH, Nq, Nk);
    if (ws_bytes < fa_decode::workspace_bytes(BH, Nq, d, splits)) return FA_ERR_INVALID_ARG;
    if (Nq >= fa_decode::TILED_MIN_NQ)
        return static_cast<fa_status>(fa_internal::forward_qk(q, k, v, o, lse, B, H, Nq, Nk, d,
                                                               causal, scale,
                                                               static_cast<int*>(workspace),
                                                               stream));

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

    // Keys per split, a multiple of the 16-key warp tile.
    int chunk = int(((long long)Nk + splits - 1) / splits);
    chunk = (chunk + fa_decode::KT - 1) / fa_decode::KT * fa_decode::KT;
    const int used = (Nk + chunk - 1) / chunk;       // splits that hold keys
    float* opart = static_cast<float*>(workspace);
    const size_t o_bytes = size_t(used) * BH * Nq * d * sizeof(float);
    float* lpart = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                            ((o_bytes + 255) & ~size_t(255)));
    const float sl2 = scale * 1.4426950408889634f;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const dim3 grid{unsigned((Nq + fa_decode::MQ - 1) / fa_decode::MQ), unsigned(used), unsigned(BH)};
    e = d == 64 ? fa_decode::launch_mma<64>(grid, s, q, k, v, opart, lpart, int(BH), Nq, Nk,
                                            causal, sl2, chunk)
                : fa_decode::launch_mma<128>(grid, s, q, k, v, opart, lpart, int(BH), Nq, Nk,
                                             causal, sl2, chunk);
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
