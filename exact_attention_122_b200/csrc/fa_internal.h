// fa_internal.h -- helpers shared by the library's translation units (not
// part of the C ABI).
#ifndef FA_B200_INTERNAL_H
#define FA_B200_INTERNAL_H

namespace fa_internal {
// Records the cudaError_t behind an FA_ERR_LAUNCH / FA_ERR_NO_DEVICE of the
// calling thread (read back by fa_last_cuda_error).
void set_last_cuda_error(int e);
}  // namespace fa_internal

#endif
