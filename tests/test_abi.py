"""C-ABI checks that need no GPU: the library loads, exports every symbol that
include/fa.h declares, and rejects bad arguments before touching a device."""

import ctypes
import os
import re

import pytest

import exact_attention_122_b200 as fa
from exact_attention_122_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    fa_build.build()
    return fa.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_exports():
    assert declared_functions() == sorted(fa.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fa.library_path())
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version():
    for code, name in [(0, "FA_OK"), (1, "FA_ERR_INVALID_ARG"), (2, "FA_ERR_UNSUPPORTED"),
                       (3, "FA_ERR_MISALIGNED"), (4, "FA_ERR_LAUNCH"), (5, "FA_ERR_TIMEOUT"),
                       (6, "FA_ERR_NO_DEVICE")]:
        assert fa.status_string(code) == name
    assert fa.status_string(99) == "FA_ERR_UNKNOWN"
    assert fa.version() >= 100


# Fake, never-dereferenced addresses: validation happens before any device
# work, so these calls are safe without a GPU.
P = 1 << 20


@pytest.mark.parametrize("args,expect", [
    ((0, P, P, P, P, 1, 1, 8, 64, 0, 1.0), fa.FA_ERR_INVALID_ARG),        # NULL q
    ((P, P, P, P, 0, 1, 1, 8, 64, 0, 1.0), fa.FA_ERR_INVALID_ARG),        # NULL lse
    ((P, P, P, P, P, 0, 1, 8, 64, 0, 1.0), fa.FA_ERR_INVALID_ARG),        # B = 0
    ((P, P, P, P, P, 1, -2, 8, 64, 0, 1.0), fa.FA_ERR_INVALID_ARG),       # H < 0
    ((P, P, P, P, P, 1, 1, 0, 64, 0, 1.0), fa.FA_ERR_INVALID_ARG),        # N = 0
    ((P, P, P, P, P, 1, 1, 8, 64, 2, 1.0), fa.FA_ERR_INVALID_ARG),        # causal flag
    ((P, P, P, P, P, 1, 1, 8, 64, 0, 0.0), fa.FA_ERR_INVALID_ARG),        # scale 0
    ((P, P, P, P, P, 1, 1, 8, 64, 0, -1.0), fa.FA_ERR_INVALID_ARG),       # scale < 0
    ((P, P, P, P, P, 1, 1, 8, 64, 0, float("nan")), fa.FA_ERR_INVALID_ARG),
    ((P, P, P, P, P, 1, 1, 8, 64, 0, float("inf")), fa.FA_ERR_INVALID_ARG),
    ((P, P, P, P, P, 1, 1, 8, 96, 0, 1.0), fa.FA_ERR_UNSUPPORTED),        # d = 96
    ((P, P, P, P, P, 1, 1, 8, 256, 0, 1.0), fa.FA_ERR_UNSUPPORTED),       # d = 256
    ((P, P, P, P, P, 1, 1, (1 << 30) + 1, 64, 0, 1.0), fa.FA_ERR_UNSUPPORTED),
    ((P, P, P, P, P, 1 << 16, 1 << 16, 8, 64, 0, 1.0), fa.FA_ERR_UNSUPPORTED),  # B*H > 2^31-1
    ((P + 8, P, P, P, P, 1, 1, 8, 64, 0, 1.0), fa.FA_ERR_MISALIGNED),     # q not 16-B aligned
    ((P, P, P + 2, P, P, 1, 1, 8, 128, 1, 1.0), fa.FA_ERR_MISALIGNED),    # v
    ((P, P, P, P + 4, P, 1, 1, 8, 64, 0, 1.0), fa.FA_ERR_MISALIGNED),     # o
    ((P, P, P, P, P + 2, 1, 1, 8, 64, 0, 1.0), fa.FA_ERR_MISALIGNED),     # lse not 4-B aligned
])
def test_argument_validation(args, expect):
    assert fa.fa_fwd_raw(*args, 0) == expect


def test_debug_entry_validates_inject():
    assert fa.fa_fwd_debug_raw(P, P, P, P, P, 1, 1, 8, 64, 0, 1.0, 0, 100, 7) == fa.FA_ERR_INVALID_ARG


def test_python_wrapper_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.fa_fwd(q, q, q)


def _contig(B, H, N, d):
    return [H * N * d, N * d, d] * 4


@pytest.mark.parametrize("mutate,expect", [
    (lambda s: None, None),                                              # placeholder: NULL strides
    (lambda s: s.__setitem__(2, 32), fa.FA_ERR_INVALID_ARG),            # q seq stride < d
    (lambda s: s.__setitem__(5, 130), fa.FA_ERR_MISALIGNED),            # k seq stride not 8-aligned
    (lambda s: s.__setitem__(9, 1 << 40), fa.FA_ERR_UNSUPPORTED),       # o batch stride too large
    (lambda s: s.__setitem__(4, -128), fa.FA_ERR_INVALID_ARG),          # negative head stride
])
def test_strided_argument_validation(mutate, expect):
    B, H, N, d = 2, 3, 8, 64
    if expect is None:
        lib = fa.library()
        assert lib.fa_fwd_strided(P, P, P, P, P, B, H, N, d, None, 0, 1.0, 0) == fa.FA_ERR_INVALID_ARG
        return
    s = _contig(B, H, N, d)
    mutate(s)
    assert fa.fa_fwd_strided_raw(P, P, P, P, P, B, H, N, d, s, 0, 1.0, 0) == expect


def test_strided_size_one_dims_ignore_their_strides():
    # B = 1 and H = 1: any batch/head strides are accepted (they are never used);
    # without a GPU the call then stops at the device query.
    s = [1, 3, 64] * 4
    assert fa.fa_fwd_strided_raw(P, P, P, P, P, 1, 1, 8, 64, s, 0, 1.0, 0) == fa.FA_ERR_NO_DEVICE


def test_dynamic_argument_validation():
    ws = 1 << 22
    args = (P, P, P, P, P, 2, 3, 8, 64, None, 0, 1.0)
    assert fa.fa_fwd_dynamic_raw(*args, 0, 256, 0) == fa.FA_ERR_INVALID_ARG          # NULL workspace
    assert fa.fa_fwd_dynamic_raw(*args, ws, 255, 0) == fa.FA_ERR_INVALID_ARG         # too small
    assert fa.fa_fwd_dynamic_raw(*args, ws + 4, 256, 0) == fa.FA_ERR_MISALIGNED      # misaligned
    assert fa.DYNAMIC_WORKSPACE_BYTES == 256
    text = open(HEADER).read()
    assert "#define FA_DYNAMIC_WORKSPACE_BYTES 256" in text


def test_unit_count_limit():
    # B*H*ceil(N/256) beyond 2^30 is refused before any device work.
    assert fa.fa_fwd_raw(P, P, P, P, P, 1 << 12, 1 << 10, 1 << 17, 64, 0, 1.0, 0) == fa.FA_ERR_UNSUPPORTED


def test_decode_argument_validation_and_workspace_size():
    W = 1 << 22
    ok = (P, P, P, P, P, 2, 3, 1, 1000, 128, 0, 0.1, 0, W, 1 << 30, 0)
    a = list(ok); a[13] = 0
    assert fa.fa_fwd_decode_raw(*a) == fa.FA_ERR_INVALID_ARG                 # NULL workspace
    a = list(ok); a[7] = (1 << 30) + 1
    assert fa.fa_fwd_decode_raw(*a) == fa.FA_ERR_UNSUPPORTED                 # Nq > 2^30
    a = list(ok); a[7] = 8; a[8] = 4; a[10] = 1
    assert fa.fa_fwd_decode_raw(*a) == fa.FA_ERR_INVALID_ARG                 # causal with Nq > Nk
    a = list(ok); a[12] = 257
    assert fa.fa_fwd_decode_raw(*a) == fa.FA_ERR_INVALID_ARG                 # too many splits
    a = list(ok); a[14] = 64
    assert fa.fa_fwd_decode_raw(*a) == fa.FA_ERR_INVALID_ARG                 # workspace too small
    a = list(ok); a[13] = W + 16
    assert fa.fa_fwd_decode_raw(*a) == fa.FA_ERR_MISALIGNED                  # workspace alignment
    a = list(ok); a[9] = 96
    assert fa.fa_fwd_decode_raw(*a) == fa.FA_ERR_UNSUPPORTED                 # d = 96
    # workspace: splits x B*H x Nq x d fp32 partial outputs (256-byte padded) + partial LSEs
    assert fa.decode_workspace_bytes(2, 3, 4, 1000, 128, 5) == 5 * 6 * 4 * 128 * 4 + 5 * 6 * 4 * 4
    assert fa.decode_workspace_bytes(2, 3, 4, 1000, 128, 300) == 0
    assert fa.decode_workspace_bytes(2, 3, 4, 1000, 128, 0) > 0
    # Nq > 32 runs the tiled kernel: only its 256-byte work counter
    assert fa.decode_workspace_bytes(2, 3, 33, 1000, 128, 0) == 256
    assert fa.decode_workspace_bytes(2, 3, 32, 1000, 128, 1) == 32 * 6 * 128 * 4 + 32 * 6 * 4
    assert fa.fa_fwd_decode_raw(*ok) == fa.FA_ERR_NO_DEVICE                  # valid: stops at the device query


def test_bwd_argument_validation_and_workspace_size():
    W = 1 << 22
    ok = [P, P, P, P, P, P, P, P, P, 2, 3, 1000, 128, 1, 0.1, W, 1 << 30, 0]
    assert fa.fa_bwd_raw(*ok) == fa.FA_ERR_NO_DEVICE                         # valid: stops at the device query
    for i in range(9):                                                        # any NULL tensor
        a = list(ok); a[i] = 0
        assert fa.fa_bwd_raw(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok); a[15] = 0
    assert fa.fa_bwd_raw(*a) == fa.FA_ERR_INVALID_ARG                        # NULL workspace
    a = list(ok); a[16] = fa.bwd_workspace_bytes(2, 3, 1000, 128) - 1
    assert fa.fa_bwd_raw(*a) == fa.FA_ERR_INVALID_ARG                        # workspace too small
    a = list(ok); a[13] = 2
    assert fa.fa_bwd_raw(*a) == fa.FA_ERR_INVALID_ARG                        # causal flag
    a = list(ok); a[14] = -1.0
    assert fa.fa_bwd_raw(*a) == fa.FA_ERR_INVALID_ARG                        # scale
    a = list(ok); a[12] = 96
    assert fa.fa_bwd_raw(*a) == fa.FA_ERR_UNSUPPORTED                        # d = 96
    a = list(ok); a[4] = P + 2
    assert fa.fa_bwd_raw(*a) == fa.FA_ERR_MISALIGNED                         # dout alignment
    a = list(ok); a[5] = P + 2
    assert fa.fa_bwd_raw(*a) == fa.FA_ERR_MISALIGNED                         # lse alignment
    a = list(ok); a[15] = W + 128
    assert fa.fa_bwd_raw(*a) == fa.FA_ERR_MISALIGNED                         # workspace alignment
    # workspace: fp32 dQ accumulator and two fp32 row vectors over N rounded up to 128
    assert fa.bwd_workspace_bytes(2, 3, 1000, 128) == 6 * 1024 * 128 * 4 + 2 * 6 * 1024 * 4
    assert fa.bwd_workspace_bytes(2, 3, 1000, 96) == 0
    assert fa.bwd_workspace_bytes(0, 3, 1000, 64) == 0


def test_fp8_argument_validation_and_workspace_size():
    W = 1 << 22
    ok = [P, P, P, P, P, 2, 3, 1000, 128, 1, 0.1, 0.01, 0.02, 0.03, W, 1 << 30, 0]
    assert fa.fa_fwd_fp8_raw(*ok) == fa.FA_ERR_NO_DEVICE                     # valid: stops at the device query
    for i in (0, 1, 2, 3, 4, 14):                                             # NULL pointer or workspace
        a = list(ok); a[i] = 0
        assert fa.fa_fwd_fp8_raw(*a) == fa.FA_ERR_INVALID_ARG
    for i in (10, 11, 12, 13):                                                # scale / descales
        for bad in (0.0, -1.0, float("nan"), float("inf")):
            a = list(ok); a[i] = bad
            assert fa.fa_fwd_fp8_raw(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok); a[8] = 96
    assert fa.fa_fwd_fp8_raw(*a) == fa.FA_ERR_UNSUPPORTED                    # d = 96
    a = list(ok); a[5] = 300; a[6] = 300
    assert fa.fa_fwd_fp8_raw(*a) == fa.FA_ERR_UNSUPPORTED                    # B*H > 65535
    a = list(ok); a[15] = fa.fp8_workspace_bytes(2, 3, 1000, 128) - 1
    assert fa.fa_fwd_fp8_raw(*a) == fa.FA_ERR_INVALID_ARG                    # workspace too small
    a = list(ok); a[1] = P + 8
    assert fa.fa_fwd_fp8_raw(*a) == fa.FA_ERR_MISALIGNED
    a = list(ok); a[14] = W + 16
    assert fa.fa_fwd_fp8_raw(*a) == fa.FA_ERR_MISALIGNED
    # workspace: 256-byte work counter + V^T (B*H*d*Npad bytes, Npad = N rounded up to 128)
    assert fa.fp8_workspace_bytes(2, 3, 1000, 128) == 256 + 6 * 128 * 1024
    assert fa.fp8_workspace_bytes(2, 3, 1000, 64) == 256 + 6 * 64 * 1024
    assert fa.fp8_workspace_bytes(2, 3, 1000, 96) == 0


def test_bwd_debug_validates_inject():
    W = 1 << 22
    args = [P, P, P, P, P, P, P, P, P, 2, 3, 1000, 128, 1, 0.1, W, 1 << 30, 0]
    assert fa.fa_bwd_debug_raw(*args, 100, 7) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_bwd_debug_raw(*args, 100, 1) == fa.FA_ERR_NO_DEVICE       # valid: stops at the device query


def test_bwd_strided_argument_validation():
    W = 1 << 22
    B, H, N, d = 2, 3, 8, 64
    st = [H * N * d, N * d, d] * 8
    base = [P, P, P, P, P, P, P, P, P, B, H, N, d]
    tail = [1, 0.1, W, 1 << 30, 0]
    assert fa.fa_bwd_strided_raw(*base, st, *tail) == fa.FA_ERR_NO_DEVICE   # valid
    assert fa.fa_bwd_strided_raw(*base, None, *tail) == fa.FA_ERR_INVALID_ARG
    bad = list(st); bad[17] = 32                                         # dq seq stride < d
    assert fa.fa_bwd_strided_raw(*base, bad, *tail) == fa.FA_ERR_INVALID_ARG
    bad = list(st); bad[22] = 130                                        # dv head stride not 8-aligned
    assert fa.fa_bwd_strided_raw(*base, bad, *tail) == fa.FA_ERR_MISALIGNED
    bad = list(st); bad[12] = 1 << 40                                    # dout batch stride too large
    assert fa.fa_bwd_strided_raw(*base, bad, *tail) == fa.FA_ERR_UNSUPPORTED


def _host_ws(B, H, N, d):
    """fa_fwd_host's workspace: two slots of one chunk (ceil(B*H/16) heads) each,
    Q, K, V, O (bf16) and LSE (fp32) padded to 256 bytes, plus a 256-byte counter."""
    up = lambda x: (x + 255) // 256 * 256
    hc = -(-(B * H) // 16)
    return 2 * (4 * up(hc * N * d * 2) + up(hc * N * 4) + 256)


def test_host_argument_validation_and_workspace_size():
    W = 1 << 22
    need = fa.host_workspace_bytes(2, 3, 1000, 128)
    assert need == _host_ws(2, 3, 1000, 128) == 2056704
    assert fa.host_workspace_bytes(2, 32, 8192, 128) == _host_ws(2, 32, 8192, 128)
    assert fa.host_workspace_bytes(1, 1, 33, 64) == _host_ws(1, 1, 33, 64)
    assert fa.host_workspace_bytes(2, 3, 1000, 96) == 0
    assert fa.host_workspace_bytes(0, 3, 1000, 64) == 0
    ok = [P + 1, P + 3, P + 5, P + 7, P + 2, 2, 3, 1000, 128, 1, 0.1, W, need, 0]
    assert fa.fa_fwd_host_raw(*ok) == fa.FA_ERR_NO_DEVICE   # host buffers need no alignment
    for i in (0, 1, 2, 3, 4, 11):                            # NULL pointer or workspace
        a = list(ok); a[i] = 0
        assert fa.fa_fwd_host_raw(*a) == fa.FA_ERR_INVALID_ARG
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        a = list(ok); a[10] = bad
        assert fa.fa_fwd_host_raw(*a) == fa.FA_ERR_INVALID_ARG
    a = list(ok); a[9] = 2
    assert fa.fa_fwd_host_raw(*a) == fa.FA_ERR_INVALID_ARG  # causal flag
    a = list(ok); a[7] = 0
    assert fa.fa_fwd_host_raw(*a) == fa.FA_ERR_INVALID_ARG  # N < 1
    a = list(ok); a[8] = 96
    assert fa.fa_fwd_host_raw(*a) == fa.FA_ERR_UNSUPPORTED  # d = 96
    a = list(ok); a[5] = 1 << 16; a[6] = 1 << 16
    assert fa.fa_fwd_host_raw(*a) == fa.FA_ERR_UNSUPPORTED  # B*H = 2^32
    a = list(ok); a[5] = 1 << 15; a[6] = 1 << 15
    assert fa.fa_fwd_host_raw(*a) == fa.FA_ERR_UNSUPPORTED  # 2^30 heads * 4 units > 2^30
    a = list(ok); a[12] = need - 1
    assert fa.fa_fwd_host_raw(*a) == fa.FA_ERR_INVALID_ARG  # workspace too small
    a = list(ok); a[11] = W + 16
    assert fa.fa_fwd_host_raw(*a) == fa.FA_ERR_MISALIGNED   # workspace not 256-byte aligned
