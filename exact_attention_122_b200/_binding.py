"""ctypes binding of libfa_b200.so (include/fa.h).  Argument marshalling only."""

from __future__ import annotations

import ctypes
import math
import os

FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_MISALIGNED = 3
FA_ERR_LAUNCH = 4
FA_ERR_TIMEOUT = 5
FA_ERR_NO_DEVICE = 6

EXPORTED_SYMBOLS = ("fa_fwd", "fa_fwd_strided", "fa_fwd_dynamic", "fa_fwd_dynamic_noalloc",
                    "fa_fwd_decode_workspace_bytes", "fa_fwd_decode", "fa_bwd_workspace_bytes",
                    "fa_bwd", "fa_bwd_strided", "fa_bwd_debug", "fa_fwd_fp8_workspace_bytes",
                    "fa_fwd_fp8", "fa_fwd_host_workspace_bytes", "fa_fwd_host",
                    "fa_fwd_debug",
                    "fa_get_device_status", "fa_status_string", "fa_last_cuda_error", "fa_version")
DECODE_MAX_QUERIES = 1 << 30           # FA_DECODE_MAX_QUERIES
DECODE_MAX_SPLITS = 256                # FA_DECODE_MAX_SPLITS
DYNAMIC_WORKSPACE_BYTES = 256          # FA_DYNAMIC_WORKSPACE_BYTES in include/fa.h

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


def library_path() -> str:
    return os.path.join(_HERE, "libfa_b200.so")


def library() -> ctypes.CDLL:
    """Load libfa_b200.so once; raise if it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m exact_attention_122_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    vp, i, f, u = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint
    fwd_args = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
    lib.fa_fwd.argtypes = fwd_args
    lib.fa_fwd.restype = i
    lib.fa_fwd_strided.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, ctypes.POINTER(ctypes.c_longlong),
                                   i, f, vp]
    lib.fa_fwd_strided.restype = i
    lib.fa_fwd_dynamic.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, ctypes.POINTER(ctypes.c_longlong),
                                   i, f, vp, ctypes.c_size_t, vp]
    lib.fa_fwd_dynamic.restype = i
    lib.fa_fwd_dynamic_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i,
                                           ctypes.POINTER(ctypes.c_longlong), i, f, vp]
    lib.fa_fwd_dynamic_noalloc.restype = i
    lib.fa_fwd_decode_workspace_bytes.argtypes = [i, i, i, i, i, i]
    lib.fa_fwd_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_fwd_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, ctypes.c_size_t, vp]
    lib.fa_fwd_decode.restype = i
    lib.fa_bwd_workspace_bytes.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp,
                           ctypes.c_size_t, vp]
    lib.fa_bwd.restype = i
    lib.fa_bwd_strided.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i,
                                   ctypes.POINTER(ctypes.c_longlong), i, f, vp, ctypes.c_size_t, vp]
    lib.fa_bwd_strided.restype = i
    lib.fa_bwd_debug.argtypes = lib.fa_bwd.argtypes + [u, i]
    lib.fa_bwd_debug.restype = i
    lib.fa_fwd_fp8_workspace_bytes.argtypes = [i, i, i, i]
    lib.fa_fwd_fp8_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, f, f, vp, ctypes.c_size_t,
                               vp]
    lib.fa_fwd_fp8.restype = i
    lib.fa_fwd_host_workspace_bytes.argtypes = [i, i, i, i]
    lib.fa_fwd_host_workspace_bytes.restype = ctypes.c_size_t
    lib.fa_fwd_host.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, ctypes.c_size_t, vp]
    lib.fa_fwd_host.restype = i
    lib.fa_fwd_debug.argtypes = fwd_args + [u, i]
    lib.fa_fwd_debug.restype = i
    lib.fa_get_device_status.argtypes = [vp, ctypes.POINTER(u)]
    lib.fa_get_device_status.restype = i
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_last_cuda_error.argtypes = []
    lib.fa_last_cuda_error.restype = i
    lib.fa_version.argtypes = []
    lib.fa_version.restype = i
    _LIB = lib
    return lib


class FaError(RuntimeError):
    def __init__(self, status: int, what: str = "fa_fwd"):
        self.status = status
        name = status_string(status)
        extra = ""
        if status in (FA_ERR_LAUNCH, FA_ERR_NO_DEVICE):
            extra = f" (cudaError {library().fa_last_cuda_error()})"
        super().__init__(f"{what} failed: {name}{extra}")


def status_string(status: int) -> str:
    return library().fa_status_string(int(status)).decode()


def version() -> int:
    return library().fa_version()


def fa_fwd_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, H: int,
               N: int, d: int, causal: int, scale: float, stream_ptr: int) -> int:
    """Direct call of the C entry point; returns the fa_status code."""
    return library().fa_fwd(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, causal, scale,
                            stream_ptr)


def fa_fwd_strided_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int,
                       H: int, N: int, d: int, strides, causal: int, scale: float,
                       stream_ptr: int) -> int:
    """Direct call of fa_fwd_strided; ``strides`` = 12 element strides
    (batch, head, seq) of q, k, v, o.  Returns the fa_status code."""
    arr = (ctypes.c_longlong * 12)(*[int(x) for x in strides])
    return library().fa_fwd_strided(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, arr, causal,
                                    scale, stream_ptr)


def fa_fwd_dynamic_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int,
                       H: int, N: int, d: int, strides, causal: int, scale: float, ws_ptr: int,
                       ws_bytes: int, stream_ptr: int) -> int:
    """Direct call of fa_fwd_dynamic; ``strides`` = None or 12 element strides."""
    arr = None if strides is None else (ctypes.c_longlong * 12)(*[int(x) for x in strides])
    return library().fa_fwd_dynamic(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, arr, causal,
                                    scale, ws_ptr, ws_bytes, stream_ptr)


def fa_fwd_dynamic_noalloc_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int,
                               B: int, H: int, N: int, d: int, strides, causal: int, scale: float,
                               stream_ptr: int) -> int:
    """Direct call of fa_fwd_dynamic_noalloc (no workspace: the library's
    static device scratch holds the work counter).  ``strides`` = None or 12
    element strides.  Returns the fa_status code."""
    arr = None if strides is None else (ctypes.c_longlong * 12)(*[int(x) for x in strides])
    return library().fa_fwd_dynamic_noalloc(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, arr,
                                            causal, scale, stream_ptr)


def decode_workspace_bytes(B: int, H: int, Nq: int, Nk: int, d: int, num_splits: int = 0) -> int:
    return int(library().fa_fwd_decode_workspace_bytes(B, H, Nq, Nk, d, num_splits))


def fa_fwd_decode_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, H: int,
                      Nq: int, Nk: int, d: int, causal: int, scale: float, num_splits: int,
                      ws_ptr: int, ws_bytes: int, stream_ptr: int) -> int:
    """Direct call of fa_fwd_decode; returns the fa_status code."""
    return library().fa_fwd_decode(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, Nq, Nk, d, causal,
                                   scale, num_splits, ws_ptr, ws_bytes, stream_ptr)


def fa_fwd_decode(q, k, v, causal: bool = False, scale: float | None = None, num_splits: int = 0,
                  out=None, lse=None, workspace=None, stream=None):
    """O, LSE for few queries q (B, H, Nq, d) against k, v (B, H, Nk, d), bf16
    contiguous CUDA tensors (Nq <= DECODE_MAX_QUERIES).  ``workspace`` (a
    device tensor of at least decode_workspace_bytes(...) bytes) is allocated
    with torch when not given."""
    import torch

    for name, t in (("q", q), ("k", k), ("v", v)):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if k.shape != (B, H, Nk, d) or v.shape != k.shape:
        raise ValueError("k and v must be (B, H, Nk, d) with q's B, H, d")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    need = decode_workspace_bytes(B, H, Nq, Nk, d, num_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        st = fa_fwd_decode_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse.data_ptr(), B, H, Nq, Nk, d, 1 if causal else 0, float(scale),
                               int(num_splits), workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), s.cuda_stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_decode")
    return out, lse


def bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(library().fa_bwd_workspace_bytes(B, H, N, d))


def fa_bwd_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, do_ptr: int, lse_ptr: int,
               dq_ptr: int, dk_ptr: int, dv_ptr: int, B: int, H: int, N: int, d: int, causal: int,
               scale: float, ws_ptr: int, ws_bytes: int, stream_ptr: int) -> int:
    """Direct call of fa_bwd; returns the fa_status code."""
    return library().fa_bwd(q_ptr, k_ptr, v_ptr, o_ptr, do_ptr, lse_ptr, dq_ptr, dk_ptr, dv_ptr,
                            B, H, N, d, causal, scale, ws_ptr, ws_bytes, stream_ptr)


def fa_bwd_strided_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, do_ptr: int, lse_ptr: int,
                       dq_ptr: int, dk_ptr: int, dv_ptr: int, B: int, H: int, N: int, d: int,
                       strides, causal: int, scale: float, ws_ptr: int, ws_bytes: int,
                       stream_ptr: int) -> int:
    """Direct call of fa_bwd_strided (strides: 24 ints or None); returns the fa_status code."""
    arr = None if strides is None else (ctypes.c_longlong * 24)(*strides)
    return library().fa_bwd_strided(q_ptr, k_ptr, v_ptr, o_ptr, do_ptr, lse_ptr, dq_ptr, dk_ptr,
                                    dv_ptr, B, H, N, d, arr, causal, scale, ws_ptr, ws_bytes,
                                    stream_ptr)


def fa_bwd_debug_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, do_ptr: int, lse_ptr: int,
                     dq_ptr: int, dk_ptr: int, dv_ptr: int, B: int, H: int, N: int, d: int,
                     causal: int, scale: float, ws_ptr: int, ws_bytes: int, stream_ptr: int,
                     watchdog_ms: int, inject: int) -> int:
    """Direct call of fa_bwd_debug; returns the fa_status code."""
    return library().fa_bwd_debug(q_ptr, k_ptr, v_ptr, o_ptr, do_ptr, lse_ptr, dq_ptr, dk_ptr,
                                  dv_ptr, B, H, N, d, causal, scale, ws_ptr, ws_bytes, stream_ptr,
                                  watchdog_ms, inject)


def fa_bwd(q, k, v, out, lse, dout, causal: bool = False, scale: float | None = None,
           dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of attention for bf16 CUDA tensors q, k, v, out, dout
    (B, H, N, d) and the forward's fp32 lse (B, H, N, contiguous).  The bf16
    tensors may be strided views with a contiguous last dimension (strided
    calls go through fa_bwd_strided); dq, dk, dv are allocated contiguous when
    not given.  ``workspace`` (at least bwd_workspace_bytes(B, H, N, d) bytes
    of device memory) is allocated with torch when not given."""
    import torch

    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.stride(-1) == 1):
            raise ValueError(f"{name} must be a bf16 CUDA tensor (B, H, N, d) with a contiguous "
                             "last dimension")
    B, H, N, d = q.shape
    for t in (k, v, out, dout):
        if t.shape != q.shape:
            raise ValueError("q, k, v, out and dout must have one shape (B, H, N, d)")
    if not (lse.is_cuda and lse.dtype == torch.float32 and lse.shape == (B, H, N)
            and lse.is_contiguous()):
        raise ValueError("lse must be a contiguous fp32 CUDA tensor (B, H, N)")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q, memory_format=torch.contiguous_format) if dq is None else dq
    dk = torch.empty_like(k, memory_format=torch.contiguous_format) if dk is None else dk
    dv = torch.empty_like(v, memory_format=torch.contiguous_format) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.shape == q.shape and t.stride(-1) == 1):
            raise ValueError(f"{name} must be a bf16 CUDA tensor shaped like q with a contiguous "
                             "last dimension")
    need = bwd_workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    tensors = (q, k, v, out, dout, dq, dk, dv)
    with torch.cuda.device(q.device):
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        args = [t.data_ptr() for t in tensors[:5]] + [lse.data_ptr()] + \
               [t.data_ptr() for t in tensors[5:]]
        ws = (workspace.data_ptr(), workspace.numel() * workspace.element_size())
        if all(t.is_contiguous() for t in tensors):
            st = fa_bwd_raw(*args, B, H, N, d, 1 if causal else 0, float(scale), *ws,
                            s.cuda_stream)
        else:
            strides = [x for t in tensors for x in t.stride()[:3]]
            st = fa_bwd_strided_raw(*args, B, H, N, d, strides, 1 if causal else 0, float(scale),
                                    *ws, s.cuda_stream)
    if st != FA_OK:
        raise FaError(st, "fa_bwd")
    return dq, dk, dv


def fp8_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(library().fa_fwd_fp8_workspace_bytes(B, H, N, d))


def fa_fwd_fp8_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, H: int,
                   N: int, d: int, causal: int, scale: float, descale_q: float, descale_k: float,
                   descale_v: float, ws_ptr: int, ws_bytes: int, stream_ptr: int) -> int:
    """Direct call of fa_fwd_fp8; returns the fa_status code."""
    return library().fa_fwd_fp8(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, causal, scale,
                                descale_q, descale_k, descale_v, ws_ptr, ws_bytes, stream_ptr)


def fa_fwd_fp8(q8, k8, v8, descale_q: float, descale_k: float, descale_v: float,
               causal: bool = False, scale: float | None = None, out=None, lse=None,
               workspace=None, stream=None):
    """O (bf16), LSE of attention over FP8 E4M3 inputs: q8, k8, v8 contiguous
    CUDA tensors (B, H, N, d), d in {64, 128}, of dtype uint8 or torch.float8_e4m3fn holding
    the codes; the values are code * descale_x.  ``workspace`` (at least
    fp8_workspace_bytes(B, H, N, d) bytes) is allocated with torch when not
    given."""
    import torch

    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        if not (t.is_cuda and t.element_size() == 1 and t.dim() == 4 and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous one-byte CUDA tensor")
    B, H, N, d = q8.shape
    if k8.shape != q8.shape or v8.shape != q8.shape:
        raise ValueError("q8, k8 and v8 must have one shape (B, H, N, d)")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device)
    need = fp8_workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q8.device)
    with torch.cuda.device(q8.device):
        s = stream if stream is not None else torch.cuda.current_stream(q8.device)
        st = fa_fwd_fp8_raw(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), out.data_ptr(),
                            lse.data_ptr(), B, H, N, d, 1 if causal else 0, float(scale),
                            float(descale_q), float(descale_k), float(descale_v),
                            workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                            s.cuda_stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_fp8")
    return out, lse


def host_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(library().fa_fwd_host_workspace_bytes(B, H, N, d))


def fa_fwd_host_raw(q_ptr: int, k_ptr: int, v_ptr: int, o_ptr: int, lse_ptr: int, B: int, H: int,
                    N: int, d: int, causal: int, scale: float, ws_ptr: int, ws_bytes: int,
                    stream_ptr: int) -> int:
    """Direct call of fa_fwd_host (host q/k/v/o/lse); returns the fa_status code."""
    return library().fa_fwd_host(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, causal, scale,
                                 ws_ptr, ws_bytes, stream_ptr)


def fa_fwd_host(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
                workspace=None, stream=None, device=None):
    """O, LSE of exact attention for bf16 (B, H, N, d) tensors in HOST memory
    (page-locked for overlap: ``tensor.pin_memory()``), through fa_fwd_host:
    chunks of heads are copied to ``device``, computed and copied back with
    the transfers overlapped.  ``out`` / ``lse`` (host, allocated pinned when
    not given) hold the results once ``stream`` (default: the current torch
    stream of ``device``) has been synchronised.  ``workspace`` is a device
    tensor of at least host_workspace_bytes(B, H, N, d) bytes, allocated when
    not given."""
    import torch

    for name, t in (("q", q), ("k", k), ("v", v)):
        if not (t.device.type == "cpu" and t.dtype == torch.bfloat16 and t.dim() == 4
                and t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous bf16 host tensor (B, H, N, d)")
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share one shape (B, H, N, d)")
    B, H, N, d = q.shape
    device = torch.device(device) if device is not None else torch.device(
        "cuda", torch.cuda.current_device())
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, pin_memory=True)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, pin_memory=True)
    if not (out.device.type == "cpu" and out.dtype == torch.bfloat16 and out.shape == q.shape
            and out.is_contiguous()):
        raise ValueError("out must be a contiguous bf16 host tensor shaped like q")
    if not (lse.device.type == "cpu" and lse.dtype == torch.float32
            and tuple(lse.shape) == (B, H, N) and lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 host tensor of shape (B, H, N)")
    need = host_workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    with torch.cuda.device(device):
        s = stream if stream is not None else torch.cuda.current_stream(device)
        st = fa_fwd_host_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr(), B, H, N, d, 1 if causal else 0, float(scale),
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             s.cuda_stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_host")
    return out, lse


_WORKSPACES = {}


def _workspace(device, stream):
    """A DYNAMIC_WORKSPACE_BYTES device buffer per (device, stream): calls on one
    stream are ordered, so they can share it."""
    import torch

    key = (str(device), int(stream.cuda_stream))
    ws = _WORKSPACES.get(key)
    if ws is None:
        ws = torch.empty(DYNAMIC_WORKSPACE_BYTES, dtype=torch.uint8, device=device)
        _WORKSPACES[key] = ws
    return ws


def fa_fwd_debug_raw(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, causal, scale, stream_ptr,
                     watchdog_ms: int, inject: int) -> int:
    return library().fa_fwd_debug(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, causal, scale,
                                  stream_ptr, watchdog_ms, inject)


def device_status(stream_ptr: int = 0):
    """(status, raw word) of the kernel watchdog; synchronises the stream."""
    word = ctypes.c_uint(0)
    st = library().fa_get_device_status(stream_ptr, ctypes.byref(word))
    return st, word.value


UNIT_ROWS = 256                        # query rows per work unit of the forward kernel
AUTO_DYNAMIC_UNITS_PER_SM = (4, 12)    # "auto": the dynamic schedule in this units-per-SM band


def resolve_schedule(schedule: str, B: int, H: int, N: int, sm_count: int) -> str:
    """The schedule fa_fwd uses: "static" or "dynamic" as given; "auto" picks
    the dynamic schedule when the problem has between 4 and 12 units of work
    per SM (B*H*ceil(N/256) units), the static one otherwise.  Both give
    identical results.  Measured on B200: below 4 units per SM the dynamic
    schedule's counter reset and claims cost a few microseconds per launch;
    from 12 units per SM the static schedule's paired causal assignment
    balances the CTAs to within one pair and is as fast or faster; in between
    (e.g. one batch of 32 heads at N = 8192) the greedy claims balance
    better."""
    if schedule not in ("auto", "static", "dynamic"):
        raise ValueError("schedule must be 'auto', 'static' or 'dynamic'")
    if schedule != "auto":
        return schedule
    units = B * H * ((N + UNIT_ROWS - 1) // UNIT_ROWS)
    lo, hi = AUTO_DYNAMIC_UNITS_PER_SM
    return "dynamic" if lo * sm_count <= units < hi * sm_count else "static"


def fa_fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
           stream=None, schedule: str = "auto", workspace=None):
    """O, LSE = exact attention forward of bf16 (B, H, N, d) CUDA tensors.

    q, k, v and ``out`` may be strided views (for example a (B, N, H, d)
    tensor transposed to (B, H, N, d)) as long as the head dimension is
    contiguous; ``out`` (bf16) is allocated contiguous when not given and
    ``lse`` (float32, contiguous (B, H, N)) likewise.  Runs asynchronously on
    ``stream`` (default: the current torch stream of q's device).
    ``schedule="static"`` calls fa_fwd / fa_fwd_strided; ``"dynamic"`` calls
    fa_fwd_dynamic with ``workspace`` (a device tensor of at least
    DYNAMIC_WORKSPACE_BYTES bytes; one cached per stream when not given);
    ``"auto"`` (default) picks one by problem size (resolve_schedule).
    """
    import torch

    for name, t in (("q", q), ("k", k), ("v", v)):
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.stride(-1) == 1):
            raise ValueError(f"{name} must be a bf16 CUDA tensor of shape (B, H, N, d) with a "
                             "contiguous last dimension")
    if k.shape != q.shape or v.shape != q.shape or k.device != q.device or v.device != q.device:
        raise ValueError("q, k, v must share shape and device")
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if not (out.is_cuda and out.dtype == torch.bfloat16 and out.shape == q.shape and out.stride(-1) == 1):
        raise ValueError("out must be a bf16 CUDA tensor shaped like q with a contiguous last dimension")
    if not (lse.is_cuda and lse.dtype == torch.float32 and tuple(lse.shape) == (B, H, N) and lse.is_contiguous()):
        raise ValueError("lse must be a contiguous float32 CUDA tensor of shape (B, H, N)")
    schedule = resolve_schedule(schedule, B, H, N,
                                torch.cuda.get_device_properties(q.device).multi_processor_count)
    with torch.cuda.device(q.device):
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        contiguous = all(t.is_contiguous() for t in (q, k, v, out))
        if schedule == "dynamic":
            ws = workspace if workspace is not None else _workspace(q.device, s)
            strides = None if contiguous else [x for t in (q, k, v, out) for x in t.stride()[:3]]
            st = fa_fwd_dynamic_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    lse.data_ptr(), B, H, N, d, strides, 1 if causal else 0,
                                    float(scale), ws.data_ptr(), ws.numel() * ws.element_size(),
                                    s.cuda_stream)
        elif contiguous:
            st = fa_fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                            B, H, N, d, 1 if causal else 0, float(scale), s.cuda_stream)
        else:
            strides = [x for t in (q, k, v, out) for x in t.stride()[:3]]
            st = fa_fwd_strided_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    lse.data_ptr(), B, H, N, d, strides, 1 if causal else 0,
                                    float(scale), s.cuda_stream)
    if st != FA_OK:
        raise FaError(st)
    return out, lse
