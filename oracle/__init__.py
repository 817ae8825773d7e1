"""fp64 CPU oracle for HSTU jagged attention and the HSTU layer (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. The product path never does; it shares no code
with the CUDA implementation. The arithmetic lives in ``hstu_oracle.c`` (plain
C, double precision, one output row at a time); this module only compiles it,
loads it with ctypes and converts numpy arrays.

Parity pins (tests/test_oracle_pins.py) tie each function below to something
other than itself: brute-force dense evaluation, closed forms, invariants and
library routines.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_hstu.so")
_lib = None

_i32, _i64, _f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
_p = ctypes.c_void_p


def build(src: str = _SRC, out: str = _LIB, force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def _bind(lib):
    lib.hstu_oracle_floor_log2.restype = _i32
    lib.hstu_oracle_floor_log2.argtypes = [_i64]
    lib.hstu_oracle_time_bucket.restype = _i32
    lib.hstu_oracle_time_bucket.argtypes = [_i64, _i32]
    lib.hstu_oracle_pos_index.restype = _i32
    lib.hstu_oracle_pos_index.argtypes = [_i64, _i64, _i32]
    lib.hstu_oracle_silu.restype = _f64
    lib.hstu_oracle_silu.argtypes = [_f64]
    lib.hstu_oracle_bias_indices.restype = None
    lib.hstu_oracle_bias_indices.argtypes = [_p, _i32, _p, _i32, _i32, _p, _p]
    lib.hstu_oracle_attn.restype = ctypes.c_int
    lib.hstu_oracle_attn.argtypes = [_p, _i32, _i32, _i32, _i32, _p, _i64, _p, _i64, _p, _i64,
                                     _p, _p, _i32, _p, _i32, _i32, _p, _i64, _p]
    lib.hstu_oracle_linear.restype = None
    lib.hstu_oracle_linear.argtypes = [_i64, _i32, _i32, _p, _p, _p, _i32, _p, _p]
    lib.hstu_oracle_layernorm_gate.restype = None
    lib.hstu_oracle_layernorm_gate.argtypes = [_i64, _i32, _p, _i64, _p, _i64, _p, _p, _f64, _p]
    lib.hstu_oracle_layer.restype = ctypes.c_int
    lib.hstu_oracle_layer.argtypes = [_i64, _i32, _p, _p, _p, _p, _p, _p, _p, _f64, _p, _p,
                                      _i32, _p, _i32, _i32, _i32, _p, _p, _i32, _p, _i32, _i32,
                                      _p, _i64, _p]
    lib.hstu_oracle_layernorm.restype = None
    lib.hstu_oracle_layernorm.argtypes = [_i64, _i32, _p, _i64, _p, _p, _f64, _p]
    lib.hstu_oracle_e4m3_to_float.restype = ctypes.c_float
    lib.hstu_oracle_e4m3_to_float.argtypes = [ctypes.c_uint8]
    lib.hstu_oracle_e4m3_from_float.restype = ctypes.c_uint8
    lib.hstu_oracle_e4m3_from_float.argtypes = [ctypes.c_float]
    lib.hstu_oracle_quant_rows_e4m3.restype = None
    lib.hstu_oracle_quant_rows_e4m3.argtypes = [_i64, _i32, _p, _p, _p]
    lib.hstu_oracle_linear_fp8.restype = None
    lib.hstu_oracle_linear_fp8.argtypes = [_i64, _i32, _i32, _p, _p, _p, _p, _p, _i32, _p, _p]
    lib.hstu_oracle_silu_grad.restype = _f64
    lib.hstu_oracle_silu_grad.argtypes = [_f64]
    lib.hstu_oracle_attn_bwd.restype = None
    lib.hstu_oracle_attn_bwd.argtypes = [_p, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _p, _i32,
                                         _p, _i32, _i32, _p, _p, _p, _p, _p, _p]
    lib.hstu_oracle_num_threads.restype = ctypes.c_int
    lib.hstu_oracle_num_threads.argtypes = []
    return lib


def load(path: Optional[str] = None):
    """Load (building first if needed) the oracle library; ``path`` overrides it."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64a(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _i64a(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.int64)


def num_threads(lib=None) -> int:
    return int((lib or load()).hstu_oracle_num_threads())


def floor_log2(x: int, lib=None) -> int:
    return int((lib or load()).hstu_oracle_floor_log2(int(x)))


def time_bucket(dt: int, num_buckets: int, lib=None) -> int:
    return int((lib or load()).hstu_oracle_time_bucket(int(dt), int(num_buckets)))


def pos_index(i: int, j: int, num_pos: int, lib=None) -> int:
    return int((lib or load()).hstu_oracle_pos_index(int(i), int(j), int(num_pos)))


def silu(x: float, lib=None) -> float:
    return float((lib or load()).hstu_oracle_silu(float(x)))


def bias_indices(seq_offsets, timestamps, num_pos: int, num_buckets: int, lib=None):
    """Relative-position index and time bucket of every causal pair (i, j<=i),
    sequence by sequence, row-major. Returns two int32 arrays."""
    lib = lib or load()
    off = _i64a(seq_offsets)
    ts = _i64a(timestamps)
    n = np.diff(off)
    E = int((n * (n + 1) // 2).sum())
    pos = np.zeros(max(E, 1), dtype=np.int32)
    bkt = np.zeros(max(E, 1), dtype=np.int32)
    lib.hstu_oracle_bias_indices(_ptr(off), len(off) - 1, _ptr(ts), int(num_pos),
                                 int(num_buckets), _ptr(pos), _ptr(bkt))
    return pos[:E], bkt[:E]


def attn(seq_offsets, q, k, v, timestamps, pos_bias, time_bias, max_seqlen: int,
         rows: Optional[Sequence[int]] = None, lib=None) -> np.ndarray:
    """Attention forward in fp64. q,k: [T,H,dqk]; v: [T,H,dv].
    pos_bias [H,P], time_bias [H,NB] and timestamps may be None (term dropped).
    Returns [T,H,dv], or [len(rows),H,dv] when ``rows`` is given."""
    lib = lib or load()
    off = _i64a(seq_offsets)
    q, k, v = _f64a(q), _f64a(k), _f64a(v)
    T, H, dqk = q.shape
    dv = v.shape[2]
    pos, tb, ts = _f64a(pos_bias), _f64a(time_bias), _i64a(timestamps)
    P = 0 if pos is None else pos.shape[1]
    NB = 0 if tb is None else tb.shape[1]
    r = None if rows is None else _i64a(rows)
    n = T if r is None else r.shape[0]
    out = np.zeros((max(n, 1), H, dv), dtype=np.float64)
    rc = lib.hstu_oracle_attn(_ptr(off), len(off) - 1, H, dqk, dv, _ptr(q), H * dqk, _ptr(k),
                              H * dqk, _ptr(v), H * dv, _ptr(ts), _ptr(pos), P, _ptr(tb), NB,
                              int(max_seqlen), _ptr(r), 0 if r is None else n, _ptr(out))
    if rc != 0:
        raise ValueError("oracle: requested row outside every sequence")
    return out[:n]


def linear(x, W, bias=None, act_silu: bool = False, residual=None, lib=None) -> np.ndarray:
    """act(x W^T + bias) + residual, fp64. x [M,K], W [N,K]."""
    lib = lib or load()
    x, W, bias, residual = _f64a(x), _f64a(W), _f64a(bias), _f64a(residual)
    M, K = x.shape
    N = W.shape[0]
    y = np.zeros((max(M, 1), N), dtype=np.float64)
    lib.hstu_oracle_linear(M, K, N, _ptr(x), _ptr(W), _ptr(bias), int(bool(act_silu)),
                           _ptr(residual), _ptr(y))
    return y[:M]


def attn_bwd(seq_offsets, q, k, v, timestamps, pos_bias, time_bias, max_seqlen: int, dout,
             lib=None):
    """Gradients of attn() for the upstream gradient dout, fp64:
    (dq, dk, dv, dpos, dtime); dpos / dtime are None when the term is absent."""
    lib = lib or load()
    off = _i64a(seq_offsets)
    q, k, v, dout = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, k, v, dout))
    T, H, dqk = q.shape
    dv = v.shape[2]
    pos, tb, ts = _f64a(pos_bias), _f64a(time_bias), _i64a(timestamps)
    P = 0 if pos is None else pos.shape[1]
    NB = 0 if tb is None else tb.shape[1]
    dq = np.zeros((max(T, 1), H, dqk))
    dk = np.zeros((max(T, 1), H, dqk))
    dvv = np.zeros((max(T, 1), H, dv))
    dpos = None if pos is None else np.zeros((H, P))
    dtime = None if (tb is None or ts is None) else np.zeros((H, NB))
    lib.hstu_oracle_attn_bwd(_ptr(off), len(off) - 1, H, dqk, dv, _ptr(q), _ptr(k), _ptr(v),
                             _ptr(ts), _ptr(pos), P, _ptr(tb), NB, int(max_seqlen), _ptr(dout),
                             _ptr(dq), _ptr(dk), _ptr(dvv), _ptr(dpos), _ptr(dtime))
    return dq[:T], dk[:T], dvv[:T], dpos, dtime


def e4m3_to_float(codes, lib=None) -> np.ndarray:
    """Values of E4M3 codes (uint8 array) as float32."""
    lib = lib or load()
    table = np.array([lib.hstu_oracle_e4m3_to_float(c) for c in range(256)], dtype=np.float32)
    return table[np.asarray(codes, dtype=np.uint8)]


def e4m3_from_float(x, lib=None) -> np.ndarray:
    """E4M3 codes of float32 values: nearest, ties to even, saturating at +-448."""
    lib = lib or load()
    x = np.asarray(x, dtype=np.float32)
    return np.array([lib.hstu_oracle_e4m3_from_float(float(v)) for v in x.ravel()],
                    dtype=np.uint8).reshape(x.shape)


def quant_rows_e4m3(x, lib=None):
    """Row-wise E4M3 quantization of x [M, K] (float32 values): (codes uint8
    [M, K], scales float32 [M]) with x ~ value(codes) * scales[:, None]."""
    lib = lib or load()
    x = np.ascontiguousarray(x, dtype=np.float32)
    M, K = x.shape
    codes = np.zeros((max(M, 1), K), dtype=np.uint8)
    scales = np.zeros(max(M, 1), dtype=np.float32)
    lib.hstu_oracle_quant_rows_e4m3(M, K, _ptr(x), _ptr(codes), _ptr(scales))
    return codes[:M], scales[:M]


def linear_fp8(xq, sx, wq, sw, bias=None, act_silu: bool = False, residual=None,
               lib=None) -> np.ndarray:
    """act(value(xq) value(wq)^T * sx[:, None] * sw[None, :] + bias) + residual,
    fp64 from the E4M3 codes. xq [M, K], wq [N, K] uint8."""
    lib = lib or load()
    xq = np.ascontiguousarray(xq, dtype=np.uint8)
    wq = np.ascontiguousarray(wq, dtype=np.uint8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    bias, residual = _f64a(bias), _f64a(residual)
    M, K = xq.shape
    N = wq.shape[0]
    y = np.zeros((max(M, 1), N), dtype=np.float64)
    lib.hstu_oracle_linear_fp8(M, K, N, _ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), _ptr(bias),
                               int(bool(act_silu)), _ptr(residual), _ptr(y))
    return y[:M]


def layernorm_gate(a, u, gamma=None, beta=None, eps: float = 1e-5, lib=None) -> np.ndarray:
    """LayerNorm(a) * u over the last axis, fp64. a, u: [M, F]."""
    lib = lib or load()
    a, u, gamma, beta = _f64a(a), _f64a(u), _f64a(gamma), _f64a(beta)
    M, F = a.shape
    y = np.zeros((max(M, 1), F), dtype=np.float64)
    lib.hstu_oracle_layernorm_gate(M, F, _ptr(a), F, _ptr(u), F, _ptr(gamma), _ptr(beta),
                                   float(eps), _ptr(y))
    return y[:M]


def layernorm(a, gamma=None, beta=None, eps: float = 1e-5, lib=None) -> np.ndarray:
    """LayerNorm over the last axis in fp64 (biased variance, eps inside the
    square root, affine gamma / beta or identity). a: [M, F]."""
    lib = lib or load()
    a, gamma, beta = _f64a(a), _f64a(gamma), _f64a(beta)
    M, F = a.shape
    y = np.zeros((max(M, 1), F), dtype=np.float64)
    lib.hstu_oracle_layernorm(M, F, _ptr(a), F, _ptr(gamma), _ptr(beta), float(eps), _ptr(y))
    return y[:M]


def layer(seq_offsets, x, W1, W2, H: int, d: int, timestamps, pos_bias, time_bias,
          max_seqlen: int, b1=None, b2=None, ln_gamma=None, ln_beta=None,
          ln_eps: float = 1e-5, rows: Optional[Sequence[int]] = None, lib=None,
          input_norm: bool = False, in_gamma=None, in_beta=None) -> np.ndarray:
    """HSTU layer forward in fp64: x + (LayerNorm(attn(Q,K,V)) * U) W2^T + b2 with
    U|V|Q|K = silu(x' W1^T + b1), x' = x or, with input_norm, LayerNorm(x)
    (affine in_gamma / in_beta, the same eps). Returns [T,D] or [len(rows),D]."""
    lib = lib or load()
    off = _i64a(seq_offsets)
    x, W1, W2 = _f64a(x), _f64a(W1), _f64a(W2)
    b1, b2, g, bt = _f64a(b1), _f64a(b2), _f64a(ln_gamma), _f64a(ln_beta)
    pos, tb, ts = _f64a(pos_bias), _f64a(time_bias), _i64a(timestamps)
    T, D = x.shape
    P = 0 if pos is None else pos.shape[1]
    NB = 0 if tb is None else tb.shape[1]
    r = None if rows is None else _i64a(rows)
    n = T if r is None else r.shape[0]
    out = np.zeros((max(n, 1), D), dtype=np.float64)
    ig, ib = _f64a(in_gamma), _f64a(in_beta)
    rc = lib.hstu_oracle_layer(T, D, _ptr(x), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(g),
                               _ptr(bt), float(ln_eps), _ptr(ig), _ptr(ib), 1 if input_norm else 0,
                               _ptr(off), len(off) - 1, H, d, _ptr(ts),
                               _ptr(pos), P, _ptr(tb), NB, int(max_seqlen), _ptr(r),
                               0 if r is None else n, _ptr(out))
    if rc != 0:
        raise ValueError("oracle layer failed (%d)" % rc)
    return out[:n]

