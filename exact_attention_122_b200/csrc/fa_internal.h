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
// FA_ERR_NO_DEVICE or FA_ERR_UNSUPPORTED otherwise.
int current_device(int* dev, int* sm_count);

// 4-D bf16 tensor map over (d, N, H, B) with element strides (batch, head,
// sequence) and a (64, box_rows, 1, 1) box in 128-byte swizzle.  FA_OK or
// FA_ERR_UNSUPPORTED.
int encode_bhnd_map(CUtensorMap* map, const void* base, int d, int N, int H, int B, long long sb,
                    long long sh, long long sn, int box_rows);

// Reads and clears the backward kernels' watchdog word (after the caller has
// synchronised): 0 when no wait ran out.  Returns a cudaError_t.
int take_bwd_status(unsigned* word);
}  // namespace fa_internal

#endif
