"""ctypes declarations of libhstu's C ABI (include/hstu.h). No fallback: if the
library cannot be loaded, every call raises."""

from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libhstu.so")

c_i32, c_i64, c_f32, c_sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
c_p = ctypes.c_void_p

# name -> (restype, argtypes), mirroring include/hstu.h
SIGNATURES = {
    "hstu_abi_version": (c_i32, []),
    "hstu_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "hstu_device_status": (ctypes.c_int, [c_p]),
    "hstu_attn_workspace_bytes": (c_sz, [c_i32, c_i64, c_i32, c_i32, c_i32]),
    "hstu_attn_plan": (ctypes.c_int, [c_p, c_i32, c_i64, c_i32, c_p, c_sz, c_p]),
    "hstu_attn_run": (ctypes.c_int, [ctypes.c_int, c_p, c_i64, c_p, c_i64, c_p, c_i64, c_p, c_i32,
                                     c_i64, c_i32, c_i32, c_i32, c_p, c_p, c_i32, c_p, c_i32,
                                     c_i32, c_p, c_i64, c_p, c_sz, c_p]),
    "hstu_attn_fwd": (ctypes.c_int, [ctypes.c_int, c_p, c_i64, c_p, c_i64, c_p, c_i64, c_p, c_i32,
                                     c_i64, c_i32, c_i32, c_i32, c_p, c_p, c_i32, c_p, c_i32,
                                     c_i32, c_p, c_i64, c_p, c_sz, c_p]),
    "hstu_attn_fwd_noalloc": (ctypes.c_int, [ctypes.c_int, c_p, c_i64, c_p, c_i64, c_p, c_i64,
                                             c_p, c_i32, c_i64, c_i32, c_i32, c_i32, c_p, c_p,
                                             c_i32, c_p, c_i32, c_i32, c_p, c_i64, c_p]),
    "hstu_debug_bias_indices": (ctypes.c_int, [c_p, c_i32, c_i64, c_p, c_i32, c_i32, c_p, c_p,
                                               c_p]),
    "hstu_debug_wait_timeout": (ctypes.c_int, [c_i32, c_p]),
    "hstu_linear_fwd": (ctypes.c_int, [c_p, c_i64, c_i64, c_i32, c_p, c_i64, c_i32, c_p,
                                       ctypes.c_int, c_p, c_i64, c_p, c_i64, c_p]),
    "hstu_attn_bwd_f32": (ctypes.c_int, [c_p, c_p, c_p, c_p, c_p, c_i32, c_i64, c_i32, c_i32,
                                         c_i32, c_p, c_p, c_i32, c_p, c_i32, c_i32, c_p, c_p, c_p,
                                         c_p, c_p, c_p]),
    "hstu_attn_bwd_workspace_bytes": (c_sz, [c_i32, c_i64, c_i32]),
    "hstu_attn_bwd": (ctypes.c_int, [ctypes.c_int, c_p, c_i64, c_p, c_i64, c_p, c_i64, c_p, c_i64,
                                     c_p, c_i32, c_i64, c_i32, c_i32, c_p, c_p, c_i32, c_p, c_i32,
                                     c_i32, c_p, c_p, c_p, c_p, c_p, c_p, c_sz, c_p]),
    "hstu_quant_rows_e4m3": (ctypes.c_int, [c_p, c_i64, c_i64, c_i32, c_p, c_i64, c_p, c_p]),
    "hstu_linear_fp8_fwd": (ctypes.c_int, [c_p, c_i64, c_p, c_i64, c_i32, c_p, c_i64, c_p, c_i32,
                                           c_p, ctypes.c_int, c_p, c_i64, c_p, c_i64, c_p]),
    "hstu_layernorm_gate_fwd": (ctypes.c_int, [c_p, c_i64, c_p, c_i64, c_i64, c_i32, c_p, c_p,
                                               c_f32, c_p, c_i64, c_p]),
    "hstu_layernorm_fwd": (ctypes.c_int, [c_p, c_i64, c_i64, c_i32, c_p, c_p, c_f32, c_p, c_i64,
                                          c_p]),
    "hstu_layernorm_fp8_fwd": (ctypes.c_int, [c_p, c_i64, c_i64, c_i32, c_p, c_p, c_f32, c_p,
                                              c_i64, c_p, c_p]),
    "hstu_layer_workspace_bytes": (c_sz, [c_i64, c_i32, c_i32, c_i32, c_i32, c_i32]),
    "hstu_layer_fwd": (ctypes.c_int, [c_p, c_i64, c_i32, c_p, c_p, c_p, c_p, c_p, c_p, c_f32,
                                      c_i32, c_p, c_p, c_p, c_i32, c_i32, c_i32, c_p, c_p, c_i32,
                                      c_p, c_i32, c_i32, c_p, c_p, c_sz, c_p]),
    "hstu_layernorm_gate_fp8_fwd": (ctypes.c_int, [c_p, c_i64, c_p, c_i64, c_i64, c_i32, c_p, c_p,
                                                   c_f32, c_p, c_i64, c_p, c_p]),
    "hstu_layer_fp8_workspace_bytes": (c_sz, [c_i64, c_i32, c_i32, c_i32, c_i32, c_i32]),
    "hstu_layer_fp8_fwd": (ctypes.c_int, [c_p, c_i64, c_i32, c_p, c_p, c_p, c_p, c_p, c_p, c_p,
                                          c_p, c_f32, c_i32, c_p, c_p, c_p, c_i32, c_i32, c_i32,
                                          c_p, c_p, c_i32, c_p, c_i32, c_i32, c_p, c_p, c_sz, c_p]),
}

HSTU_OK, HSTU_ERR_INVALID_ARG, HSTU_ERR_UNSUPPORTED, HSTU_ERR_CUDA, HSTU_ERR_TIMEOUT, \
    HSTU_ERR_BAD_INPUT = range(6)
HSTU_DTYPE_F32, HSTU_DTYPE_BF16 = 0, 1
HSTU_EPI_NONE, HSTU_EPI_SILU, HSTU_EPI_RESIDUAL = 0, 1, 2

_lib = None


class HstuError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__("%s failed: %s (status %d)" % (fn, msg, status))
        self.status = status


def load(path: str = LIB_PATH):
    """Load libhstu.so; raises if it has not been built."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError("libhstu.so is not built (%s); run "
                          "`python -m jagged_pointwise_attention_b200.build`" % path)
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def check(fn_name: str, status: int) -> None:
    if status != HSTU_OK:
        msg = load().hstu_status_string(status).decode()
        raise HstuError(fn_name, status, msg)
