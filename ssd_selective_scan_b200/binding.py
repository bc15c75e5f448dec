"""ctypes binding of libssd.so -- the C ABI declared in include/ssd.h.

Argument marshalling only: every function here passes integers (device
pointers, sizes, a cudaStream_t handle) straight to the C entry point of the
same name and returns its status code.  There is no computation and no
fallback: if libssd.so is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libssd.so")

# ssd_status_t
SSD_OK = 0
SSD_ERR_INVALID_ARG = 1
SSD_ERR_UNSUPPORTED = 2
SSD_ERR_CUDA = 3
SSD_ERR_TIMEOUT = 4
# ssd_dtype_t
SSD_F32 = 0
SSD_BF16 = 1

# Every exported entry point and its ctypes signature (restype, argtypes).
_vp, _i, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
SIGNATURES = {
    "ssd_status_string": (ctypes.c_char_p, [_i]),
    "ssd_abi_version": (_i, []),
    "ssd_conv1d_silu": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "ssd_chunk_scan_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "ssd_chunk_scan_fwd": (_i, [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp, _vp]),
    "ssd_state_update": (_i, [_vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp,
                              _i, _i, _i, _i, _i, _i, _vp]),
    "ssd_chunk_scan_fwd_static": (_i, [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp]),
    "ssd_selftest_bounded_wait": (_i, [_vp, ctypes.c_uint64, _vp]),
    "ssd_chunk_scan_varlen_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "ssd_chunk_scan_fwd_varlen": (_i, [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                       _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp, _vp]),
    "ssd_conv_scan_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "ssd_decode_step": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                             _i, _i, _i, _i, _i, _i, _i, _vp]),
    "ssd_decode_step_workspace_bytes": (_sz, [_i, _i]),
    "ssd_decode_step_ws": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "ssd_chunk_scan_bwd_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "ssd_chunk_scan_bwd": (_i, [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "ssd_conv_scan_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                               _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp, _vp]),
    "ssd_linear_bf16": (_i, [_vp, _i64, _vp, _i64, _vp, _i64, _i, _i, _i, _vp, _vp]),
    "ssd_mixer_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "ssd_mixer_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                           _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, ctypes.c_float, _i, _vp, _sz, _vp, _vp]),
}

_lock = threading.Lock()
_lib = None


class SsdError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


def load() -> ctypes.CDLL:
    """Load libssd.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libssd.so not found at {LIB_PATH}: build it with "
                    "`python -m ssd_selective_scan_b200.build` (there is no fallback path)")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().ssd_status_string(int(status)).decode()


def ssd_abi_version() -> int:
    return load().ssd_abi_version()


def ssd_conv1d_silu(xBC, out, w, bias, conv_state, b, L, conv_dim, k, dtype, stream) -> int:
    return load().ssd_conv1d_silu(xBC, out, w, bias, conv_state, b, L, conv_dim, k, dtype, stream)


def ssd_chunk_scan_workspace_bytes(b, L, H, P, N, G, Q, dtype) -> int:
    return load().ssd_chunk_scan_workspace_bytes(b, L, H, P, N, G, Q, dtype)


def ssd_chunk_scan_fwd(x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, y, final_state,
                       b, L, H, P, N, G, Q, dtype, workspace, workspace_bytes, status, stream) -> int:
    return load().ssd_chunk_scan_fwd(x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, y,
                                     final_state, b, L, H, P, N, G, Q, dtype, workspace,
                                     workspace_bytes, status, stream)


def ssd_chunk_scan_fwd_static(x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, y,
                              final_state, b, L, H, P, N, G, Q, dtype, status, stream) -> int:
    return load().ssd_chunk_scan_fwd_static(x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state,
                                            y, final_state, b, L, H, P, N, G, Q, dtype, status,
                                            stream)


def ssd_state_update(state, x, B, C, row_stride, dt_raw, dt_bias, A, D, y, b, H, P, N, G, dtype,
                     stream) -> int:
    return load().ssd_state_update(state, x, B, C, row_stride, dt_raw, dt_bias, A, D, y, b, H, P,
                                   N, G, dtype, stream)


def ssd_chunk_scan_varlen_workspace_bytes(nseq, T, H, P, N, G, Q, dtype) -> int:
    return load().ssd_chunk_scan_varlen_workspace_bytes(nseq, T, H, P, N, G, Q, dtype)


def ssd_chunk_scan_fwd_varlen(x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, y, final_state,
                              cu_seqlens, nseq, T, H, P, N, G, Q, dtype, workspace, workspace_bytes,
                              status, stream) -> int:
    return load().ssd_chunk_scan_fwd_varlen(x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, y,
                                            final_state, cu_seqlens, nseq, T, H, P, N, G, Q, dtype,
                                            workspace, workspace_bytes, status, stream)


def ssd_conv_scan_workspace_bytes(b, L, H, P, N, G, Q, k, dtype) -> int:
    return load().ssd_conv_scan_workspace_bytes(b, L, H, P, N, G, Q, k, dtype)


def ssd_conv_scan_fwd(xBC, w, bias, conv_state, dt_raw, dt_bias, A, D, init_state, y, final_state,
                      b, L, H, P, N, G, Q, k, dtype, workspace, workspace_bytes, status, stream) -> int:
    return load().ssd_conv_scan_fwd(xBC, w, bias, conv_state, dt_raw, dt_bias, A, D, init_state, y,
                                    final_state, b, L, H, P, N, G, Q, k, dtype, workspace,
                                    workspace_bytes, status, stream)


def ssd_decode_step(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P, N, G, k,
                    dtype, stream) -> int:
    return load().ssd_decode_step(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P,
                                  N, G, k, dtype, stream)


def ssd_decode_step_workspace_bytes(b, G) -> int:
    return load().ssd_decode_step_workspace_bytes(b, G)


def ssd_decode_step_ws(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P, N, G, k,
                       dtype, workspace, workspace_bytes, stream) -> int:
    return load().ssd_decode_step_ws(state, conv_state, xBC, w, bias, dt_raw, dt_bias, A, D, y, b, H, P,
                                     N, G, k, dtype, workspace, workspace_bytes, stream)


def ssd_chunk_scan_bwd_workspace_bytes(b, L, H, P, N, G, dtype) -> int:
    return load().ssd_chunk_scan_bwd_workspace_bytes(b, L, H, P, N, G, dtype)


def ssd_chunk_scan_bwd(x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, dy, dfinal, dx, dB, dC,
                       ddt_raw, dA, dD, ddt_bias, dinit, b, L, H, P, N, G, dtype, workspace,
                       workspace_bytes, stream) -> int:
    return load().ssd_chunk_scan_bwd(x, B, C, row_stride, dt_raw, dt_bias, A, D, init_state, dy, dfinal,
                                     dx, dB, dC, ddt_raw, dA, dD, ddt_bias, dinit, b, L, H, P, N, G,
                                     dtype, workspace, workspace_bytes, stream)


def ssd_selftest_bounded_wait(status, limit_ns, stream) -> int:
    return load().ssd_selftest_bounded_wait(status, limit_ns, stream)


def check(fn: str, status: int) -> None:
    if status != SSD_OK:
        raise SsdError(fn, status)


def ssd_linear_bf16(x, ldx, w, ldw, y, ldy, M, N, K, status, stream) -> int:
    return load().ssd_linear_bf16(x, ldx, w, ldw, y, ldy, M, N, K, status, stream)


def ssd_mixer_workspace_bytes(b, L, d_model, H, P, N, G, Q, k, dtype) -> int:
    return load().ssd_mixer_workspace_bytes(b, L, d_model, H, P, N, G, Q, k, dtype)


def ssd_mixer_fwd(hidden, W_in, conv_w, conv_bias, conv_state, dt_bias, A, D, norm_w, W_out, init_state, out,
                  final_state, b, L, d_model, H, P, N, G, Q, k, norm_groups, eps, dtype, workspace,
                  workspace_bytes, status, stream) -> int:
    return load().ssd_mixer_fwd(hidden, W_in, conv_w, conv_bias, conv_state, dt_bias, A, D, norm_w, W_out,
                                init_state, out, final_state, b, L, d_model, H, P, N, G, Q, k, norm_groups, eps,
                                dtype, workspace, workspace_bytes, status, stream)
