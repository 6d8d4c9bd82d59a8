"""exact_attention_122_b200 -- exact attention forward and backward on B200 (sm_100a).

The computation lives in the CUDA library libfa_b200.so behind the C ABI of
include/fa.h; this module only marshals arguments to it (torch supplies
device memory and streams).  There is no CPU fallback: if the library is
missing, importing the binding raises.
"""

from ._binding import (  # noqa: F401
    FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_MISALIGNED, FA_ERR_LAUNCH,
    FA_ERR_TIMEOUT, FA_ERR_NO_DEVICE, EXPORTED_SYMBOLS, DYNAMIC_WORKSPACE_BYTES,
    DECODE_MAX_QUERIES, DECODE_MAX_SPLITS, decode_workspace_bytes, fa_fwd_decode, fa_fwd_decode_raw,
    FaError, library, library_path, status_string, version,
    fa_fwd, fa_fwd_raw, fa_fwd_strided_raw, fa_fwd_dynamic_raw, fa_fwd_dynamic_noalloc_raw,
    fa_fwd_debug_raw, device_status, bwd_workspace_bytes, fa_bwd, fa_bwd_raw, fa_bwd_strided_raw, fa_bwd_debug_raw,
    fp8_workspace_bytes, fa_fwd_fp8, fa_fwd_fp8_raw, host_workspace_bytes, fa_fwd_host,
    fa_fwd_host_raw, resolve_schedule,
)
from .autograd import attention  # noqa: F401,E402
