// fa_internal.h -- helpers shared by the library's translation units (not
// part of the C ABI).
#ifndef FA_B200_INTERNAL_H
#define FA_B200_INTERNAL_H

#include <cuda.h>

namespace fa_internal {
// Records the cudaError_t behind an FA_ERR_LAUNCH / FA_ERR_NO_DEVICE of the
// calling thread (read back by fa_last_cuda_error).
void set_last_cuda_error(int e);

// Current device, checked once per device: FA_OK and its index and SM count
// when it is an sm_100 device and the tensor-map encoder is available;
// FA_ERR_NO_DEVICE or FA_ERR_UNSUPPORTED otherwise.  Device indices of 64
// and above are refused (FA_ERR_NO_DEVICE), so per-device tables of 64
// entries are safe to index with the returned index.
int current_device(int* dev, int* sm_count);

// 4-D bf16 tensor map over (d, N, H, B) with element strides (batch, head,
// sequence) and a (64, box_rows, 1, 1) box in 128-byte swizzle.  FA_OK or
// FA_ERR_UNSUPPORTED.
int encode_bhnd_map(CUtensorMap* map, const void* base, int d, int N, int H, int B, long long sb,
                    long long sh, long long sn, int box_rows);

// The persistent tiled forward for N_q query rows against N_k keys (causal:
// the queries are the last N_q positions), dynamic schedule with its 4-byte
// work counter at `counter` (device memory).  Returns an fa_status.
int forward_qk(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int Nq, int Nk, int d, int causal, float scale, int* counter, void* stream);

// Reads and clears the backward kernels' watchdog word (after the caller has
// synchronised): 0 when no wait ran out.  Returns a cudaError_t.
int take_bwd_status(unsigned* word);
}  // namespace fa_internal

#endif
