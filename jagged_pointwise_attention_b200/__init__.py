"""HSTU jagged causal pointwise attention and the HSTU layer forward on B200.

Thin Python binding over libhstu (include/hstu.h). Each function takes torch
tensors that already live on the current CUDA device, checks dtypes and
shapes, and passes raw pointers, strides and the current stream to the C ABI;
every step of the computation runs in the library's sm_100a kernels. There is
no CPU or PyTorch fallback: a missing library or a failed call raises.

The operation (HSTU, arXiv 2402.17152; generative-recommenders README,
"HSTU Ultra attention benchmark" for the layer order): for j <= i in one
sequence, s_ij = q_i.k_j + pos[h][min(i-j, P-1)] + time[h][bucket(t_i - t_j)],
out_i = (1/max_seqlen) sum_j silu(s_ij) v_j.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import _native
from ._native import HstuError  # noqa: F401

__all__ = [
    "hstu_attn_fwd", "hstu_attn_plan", "hstu_attn_run", "hstu_attn_workspace_bytes",
    "hstu_layer_fwd", "hstu_layer_workspace_bytes", "hstu_linear_fwd",
    "hstu_layernorm_gate_fwd", "hstu_debug_bias_indices", "hstu_debug_wait_timeout",
    "hstu_attn_bwd", "hstu_attn_bwd_workspace_bytes", "hstu_attn_bwd_f32", "hstu_quant_rows_e4m3", "hstu_linear_fp8_fwd",
    "hstu_layernorm_gate_fp8_fwd", "hstu_layernorm_fwd", "hstu_layernorm_fp8_fwd",
    "hstu_layer_fp8_workspace_bytes", "hstu_layer_fp8_fwd",
    "hstu_device_status", "HstuError", "library_path",
]


def library_path() -> str:
    return _native.LIB_PATH


def _lib():
    return _native.load()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _native.HSTU_DTYPE_BF16
    if t.dtype == torch.float32:
        return _native.HSTU_DTYPE_F32
    raise TypeError("q/k/v must be bfloat16 or float32, got %s" % t.dtype)


def _tok_stride(t: torch.Tensor, H: int, d: int) -> int:
    """Token stride of a [T, H, d] view whose heads are contiguous inside a token."""
    if t.dim() != 3 or t.shape[1] != H or t.shape[2] != d:
        raise ValueError("expected [T, %d, %d], got %s" % (H, d, tuple(t.shape)))
    if t.shape[0] == 0:
        return H * d          # empty batch: strides of a size-0 tensor are arbitrary
    if t.stride(2) != 1 or (H > 1 and t.stride(1) != d):
        raise ValueError("heads and features must be contiguous inside a token")
    return t.stride(0)


def _on_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be on a CUDA device")


def hstu_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return _lib().hstu_device_status(_stream(stream))


def hstu_attn_workspace_bytes(B: int, total_tokens: int, max_seqlen: int, H: int,
                              num_pos: int = 1) -> int:
    """Workspace of hstu_attn_plan + hstu_attn_run (bf16): the plan's work list,
    then the run's bias tables (num_pos: the position table's length, or 1
    without a position term)."""
    return int(_lib().hstu_attn_workspace_bytes(B, total_tokens, max_seqlen, H, max(num_pos, 1)))


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def hstu_attn_plan(seq_offsets: torch.Tensor, max_seqlen: int, total_tokens: int,
                   workspace: torch.Tensor, stream=None) -> None:
    _on_cuda(seq_offsets, workspace)
    B = seq_offsets.numel() - 1
    _native.check("hstu_attn_plan", _lib().hstu_attn_plan(
        _ptr(seq_offsets), B, total_tokens, max_seqlen, _ptr(workspace), workspace.numel(),
        _stream(stream)))


def _attn_args(q, k, v, seq_offsets, timestamps, pos_bias, time_bias, max_seqlen, out):
    _on_cuda(q, k, v, seq_offsets, timestamps, pos_bias, time_bias, out)
    if seq_offsets.dtype != torch.int64:
        raise TypeError("seq_offsets must be int64")
    if timestamps is not None and timestamps.dtype != torch.int64:
        raise TypeError("timestamps must be int64")
    for tbl in (pos_bias, time_bias):
        if tbl is not None and (tbl.dtype != torch.float32 or not tbl.is_contiguous()):
            raise TypeError("bias tables must be contiguous float32 [H, n]")
    T, H, dqk = q.shape
    dv = v.shape[2]
    for t in (k, v, out):
        if t.dtype != q.dtype or t.shape[0] != T:
            raise ValueError("q, k, v and out must share dtype and token count")
    B = seq_offsets.numel() - 1
    return dict(dtype=_dtype_code(q), q=_ptr(q), qs=_tok_stride(q, H, dqk), k=_ptr(k),
                ks=_tok_stride(k, H, dqk), v=_ptr(v), vs=_tok_stride(v, H, dv),
                off=_ptr(seq_offsets), B=B, T=T, H=H, dqk=dqk, dv=dv, ts=_ptr(timestamps),
                pos=_ptr(pos_bias), P=0 if pos_bias is None else pos_bias.shape[1],
                tb=_ptr(time_bias), NB=0 if time_bias is None else time_bias.shape[1],
                N=int(max_seqlen), out=_ptr(out), os=_tok_stride(out, H, dv))


def hstu_attn_run(q, k, v, seq_offsets, timestamps, pos_bias, time_bias, max_seqlen: int,
                  out: torch.Tensor, workspace: Optional[torch.Tensor], stream=None):
    """Attention on a batch planned by hstu_attn_plan (bf16) or directly (fp32)."""
    a = _attn_args(q, k, v, seq_offsets, timestamps, pos_bias, time_bias, max_seqlen, out)
    _native.check("hstu_attn_run", _lib().hstu_attn_run(
        a["dtype"], a["q"], a["qs"], a["k"], a["ks"], a["v"], a["vs"], a["off"], a["B"], a["T"],
        a["H"], a["dqk"], a["dv"], a["ts"], a["pos"], a["P"], a["tb"], a["NB"], a["N"], a["out"],
        a["os"], _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream(stream)))
    return out


def hstu_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, seq_offsets: torch.Tensor,
                  timestamps: Optional[torch.Tensor], pos_bias: Optional[torch.Tensor],
                  time_bias: Optional[torch.Tensor], max_seqlen: int,
                  out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """HSTU jagged causal attention forward.

    q, k: [T, H, d_qk]; v: [T, H, d_v] (bf16 or fp32, heads contiguous per token,
    any token stride); seq_offsets: int64 [B+1]; timestamps: int64 [T] or None;
    pos_bias: fp32 [H, P] or None; time_bias: fp32 [H, NB] or None.
    Returns out [T, H, d_v] = (1/max_seqlen) sum_{j<=i} silu(s_ij) v_j.
    """
    T, H, _ = q.shape
    if out is None:
        out = torch.empty((T, H, v.shape[2]), dtype=q.dtype, device=q.device)
    a = _attn_args(q, k, v, seq_offsets, timestamps, pos_bias, time_bias, max_seqlen, out)
    if workspace is None and a["dtype"] == _native.HSTU_DTYPE_BF16:
        workspace = _workspace(hstu_attn_workspace_bytes(a["B"], T, max_seqlen, a["H"], a["P"]),
                               q.device)
    _native.check("hstu_attn_fwd", _lib().hstu_attn_fwd(
        a["dtype"], a["q"], a["qs"], a["k"], a["ks"], a["v"], a["vs"], a["off"], a["B"], a["T"],
        a["H"], a["dqk"], a["dv"], a["ts"], a["pos"], a["P"], a["tb"], a["NB"], a["N"], a["out"],
        a["os"], _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream(stream)))
    return out


def hstu_debug_bias_indices(seq_offsets: torch.Tensor, timestamps: torch.Tensor, num_pos: int,
                            num_buckets: int, stream=None):
    """Position index and time bucket of every causal pair, as the kernel computes them."""
    _on_cuda(seq_offsets, timestamps)
    n = torch.diff(seq_offsets.cpu())
    E = int((n * (n + 1) // 2).sum())
    pos = torch.zeros(max(E, 1), dtype=torch.int32, device=seq_offsets.device)
    bkt = torch.zeros(max(E, 1), dtype=torch.int32, device=seq_offsets.device)
    _native.check("hstu_debug_bias_indices", _lib().hstu_debug_bias_indices(
        _ptr(seq_offsets), seq_offsets.numel() - 1, timestamps.numel(), _ptr(timestamps),
        num_pos, num_buckets, _ptr(pos), _ptr(bkt), _stream(stream)))
    return pos[:E], bkt[:E]


def hstu_debug_wait_timeout(wait_us: int, stream=None) -> None:
    _native.check("hstu_debug_wait_timeout",
                  _lib().hstu_debug_wait_timeout(int(wait_us), _stream(stream)))


def hstu_linear_fwd(x: torch.Tensor, W: torch.Tensor, bias: Optional[torch.Tensor] = None,
                    epilogue: str = "none", residual: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """epilogue(x W^T + bias): "none", "silu" or "residual" (adds `residual`). bf16."""
    _on_cuda(x, W, bias, residual, out)
    M, K = x.shape
    N = W.shape[0]
    epi = {"none": _native.HSTU_EPI_NONE, "silu": _native.HSTU_EPI_SILU,
           "residual": _native.HSTU_EPI_RESIDUAL}[epilogue]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    for t in (x, W, out) + ((residual,) if residual is not None else ()):
        if t.dtype != torch.bfloat16 or t.stride(1) != 1:
            raise ValueError("x, W, residual, out must be bf16 with unit column stride")
    _native.check("hstu_linear_fwd", _lib().hstu_linear_fwd(
        _ptr(x), x.stride(0), M, K, _ptr(W), W.stride(0), N, _ptr(bias), epi, _ptr(residual),
        0 if residual is None else residual.stride(0), _ptr(out), out.stride(0), _stream(stream)))
    return out


def hstu_quant_rows_e4m3(x: torch.Tensor, stream=None):
    """Row-wise E4M3 quantization of a bf16 [M, K] matrix: (codes uint8 [M, K],
    scales fp32 [M]) with x ~ value(codes) * scales[:, None]."""
    _on_cuda(x)
    if x.dtype != torch.bfloat16 or x.stride(1) != 1:
        raise ValueError("x must be bf16 with unit column stride")
    M, K = x.shape
    codes = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    scales = torch.empty(M, dtype=torch.float32, device=x.device)
    _native.check("hstu_quant_rows_e4m3", _lib().hstu_quant_rows_e4m3(
        _ptr(x), x.stride(0), M, K, _ptr(codes), codes.stride(0), _ptr(scales), _stream(stream)))
    return codes, scales


def hstu_linear_fp8_fwd(xq: torch.Tensor, x_scales: torch.Tensor, wq: torch.Tensor,
                        w_scales: torch.Tensor, bias: Optional[torch.Tensor] = None,
                        epilogue: str = "none", residual: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """epilogue(value(xq) value(wq)^T * x_scales[:, None] * w_scales + bias) with
    E4M3 codes from hstu_quant_rows_e4m3; bf16 out (and residual)."""
    _on_cuda(xq, x_scales, wq, w_scales, bias, residual, out)
    M, K = xq.shape
    N = wq.shape[0]
    epi = {"none": _native.HSTU_EPI_NONE, "silu": _native.HSTU_EPI_SILU,
           "residual": _native.HSTU_EPI_RESIDUAL}[epilogue]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    if xq.dtype != torch.uint8 or wq.dtype != torch.uint8 or xq.stride(1) != 1 or wq.stride(1) != 1:
        raise ValueError("xq, wq must be uint8 E4M3 codes with unit column stride")
    if x_scales.dtype != torch.float32 or w_scales.dtype != torch.float32:
        raise ValueError("scales must be fp32")
    _native.check("hstu_linear_fp8_fwd", _lib().hstu_linear_fp8_fwd(
        _ptr(xq), xq.stride(0), _ptr(x_scales), M, K, _ptr(wq), wq.stride(0), _ptr(w_scales), N,
        _ptr(bias), epi, _ptr(residual), 0 if residual is None else residual.stride(0),
        _ptr(out), out.stride(0), _stream(stream)))
    return out


def hstu_layernorm_gate_fwd(a: torch.Tensor, u: torch.Tensor, gamma=None, beta=None,
                            eps: float = 1e-5, out: Optional[torch.Tensor] = None,
                            stream=None) -> torch.Tensor:
    """LayerNorm(a) * u over the last axis (bf16 rows, any row stride)."""
    _on_cuda(a, u, gamma, beta, out)
    M, F = a.shape
    if out is None:
        out = torch.empty((M, F), dtype=torch.bfloat16, device=a.device)
    _native.check("hstu_layernorm_gate_fwd", _lib().hstu_layernorm_gate_fwd(
        _ptr(a), a.stride(0), _ptr(u), u.stride(0), M, F, _ptr(gamma), _ptr(beta), float(eps),
        _ptr(out), out.stride(0), _stream(stream)))
    return out


def hstu_layernorm_fwd(a: torch.Tensor, gamma=None, beta=None, eps: float = 1e-5,
                       out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """LayerNorm(a) over the last axis (bf16 rows, any row stride): the layer's
    input normalization."""
    _on_cuda(a, gamma, beta, out)
    M, F = a.shape
    if out is None:
        out = torch.empty((M, F), dtype=torch.bfloat16, device=a.device)
    _native.check("hstu_layernorm_fwd", _lib().hstu_layernorm_fwd(
        _ptr(a), a.stride(0), M, F, _ptr(gamma), _ptr(beta), float(eps), _ptr(out),
        out.stride(0), _stream(stream)))
    return out


def hstu_layernorm_fp8_fwd(a: torch.Tensor, gamma=None, beta=None, eps: float = 1e-5,
                           stream=None):
    """LayerNorm(a) with the bf16 result rows quantized to E4M3 in the same
    kernel: (codes uint8 [M, F], scales fp32 [M])."""
    _on_cuda(a, gamma, beta)
    M, F = a.shape
    codes = torch.empty((M, F), dtype=torch.uint8, device=a.device)
    scales = torch.empty(M, dtype=torch.float32, device=a.device)
    _native.check("hstu_layernorm_fp8_fwd", _lib().hstu_layernorm_fp8_fwd(
        _ptr(a), a.stride(0), M, F, _ptr(gamma), _ptr(beta), float(eps), _ptr(codes),
        codes.stride(0), _ptr(scales), _stream(stream)))
    return codes, scales


def hstu_layer_workspace_bytes(total_tokens: int, B: int, D: int, H: int, d: int,
                               max_seqlen: int) -> int:
    return int(_lib().hstu_layer_workspace_bytes(total_tokens, B, D, H, d, max_seqlen))


def hstu_layer_fwd(x: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor, seq_offsets: torch.Tensor,
                   timestamps: Optional[torch.Tensor], pos_bias: Optional[torch.Tensor],
                   time_bias: Optional[torch.Tensor], H: int, d: int, max_seqlen: int,
                   b1=None, b2=None, ln_gamma=None, ln_beta=None, ln_eps: float = 1e-5,
                   out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   stream=None, input_norm: bool = False, in_gamma=None,
                   in_beta=None) -> torch.Tensor:
    """One HSTU layer forward: x + (LayerNorm(attn(Q, K, V)) * U) W2^T + b2 with
    U|V|Q|K = silu(x' W1^T + b1), x' = x or, with input_norm, LayerNorm(x)
    (affine in_gamma, in_beta). x [T, D] bf16, W1 [4Hd, D], W2 [D, Hd]."""
    _on_cuda(x, W1, W2, seq_offsets, timestamps, pos_bias, time_bias, b1, b2, ln_gamma, ln_beta,
             in_gamma, in_beta)
    T, D = x.shape
    B = seq_offsets.numel() - 1
    for t in (x, W1, W2):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("x, W1, W2 must be contiguous bf16")
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = _workspace(hstu_layer_workspace_bytes(T, B, D, H, d, max_seqlen), x.device)
    _native.check("hstu_layer_fwd", _lib().hstu_layer_fwd(
        _ptr(x), T, D, _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(ln_gamma), _ptr(ln_beta),
        float(ln_eps), 1 if input_norm else 0, _ptr(in_gamma), _ptr(in_beta),
        _ptr(seq_offsets), B, H, d, _ptr(timestamps), _ptr(pos_bias),
        0 if pos_bias is None else pos_bias.shape[1], _ptr(time_bias),
        0 if time_bias is None else time_bias.shape[1], int(max_seqlen), _ptr(out),
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def hstu_layernorm_gate_fp8_fwd(a: torch.Tensor, u: torch.Tensor, gamma=None, beta=None,
                                eps: float = 1e-5, stream=None):
    """LayerNorm(a) * u with the bf16 result rows quantized to E4M3 in the same
    kernel: (codes uint8 [M, F], scales fp32 [M])."""
    _on_cuda(a, u, gamma, beta)
    M, F = a.shape
    codes = torch.empty((M, F), dtype=torch.uint8, device=a.device)
    scales = torch.empty(M, dtype=torch.float32, device=a.device)
    _native.check("hstu_layernorm_gate_fp8_fwd", _lib().hstu_layernorm_gate_fp8_fwd(
        _ptr(a), a.stride(0), _ptr(u), u.stride(0), M, F, _ptr(gamma), _ptr(beta), float(eps),
        _ptr(codes), codes.stride(0), _ptr(scales), _stream(stream)))
    return codes, scales


def hstu_layer_fp8_workspace_bytes(total_tokens: int, B: int, D: int, H: int, d: int,
                                   max_seqlen: int) -> int:
    return int(_lib().hstu_layer_fp8_workspace_bytes(total_tokens, B, D, H, d, max_seqlen))


def hstu_layer_fp8_fwd(x: torch.Tensor, W1q: torch.Tensor, w1_scales: torch.Tensor,
                       W2q: torch.Tensor, w2_scales: torch.Tensor, seq_offsets: torch.Tensor,
                       timestamps: Optional[torch.Tensor], pos_bias: Optional[torch.Tensor],
                       time_bias: Optional[torch.Tensor], H: int, d: int, max_seqlen: int,
                       b1=None, b2=None, ln_gamma=None, ln_beta=None, ln_eps: float = 1e-5,
                       out: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None,
                       input_norm: bool = False, in_gamma=None, in_beta=None) -> torch.Tensor:
    """hstu_layer_fwd with both projections in FP8 (E4M3 weights from
    hstu_quant_rows_e4m3, quantized once; activations quantized in the call,
    with input_norm the input LayerNorm in the same pass)."""
    _on_cuda(x, W1q, w1_scales, W2q, w2_scales, seq_offsets, timestamps, pos_bias, time_bias, b1,
             b2, ln_gamma, ln_beta, in_gamma, in_beta)
    T, D = x.shape
    B = seq_offsets.numel() - 1
    if x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError("x must be contiguous bf16")
    for t in (W1q, W2q):
        if t.dtype != torch.uint8 or not t.is_contiguous():
            raise ValueError("W1q, W2q must be contiguous uint8 E4M3 codes")
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = _workspace(hstu_layer_fp8_workspace_bytes(T, B, D, H, d, max_seqlen), x.device)
    _native.check("hstu_layer_fp8_fwd", _lib().hstu_layer_fp8_fwd(
        _ptr(x), T, D, _ptr(W1q), _ptr(w1_scales), _ptr(b1), _ptr(W2q), _ptr(w2_scales), _ptr(b2),
        _ptr(ln_gamma), _ptr(ln_beta), float(ln_eps), 1 if input_norm else 0, _ptr(in_gamma),
        _ptr(in_beta), _ptr(seq_offsets), B, H, d,
        _ptr(timestamps), _ptr(pos_bias), 0 if pos_bias is None else pos_bias.shape[1],
        _ptr(time_bias), 0 if time_bias is None else time_bias.shape[1], int(max_seqlen),
        _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def hstu_attn_bwd_workspace_bytes(B: int, total_tokens: int, max_seqlen: int) -> int:
    return int(_lib().hstu_attn_bwd_workspace_bytes(B, total_tokens, max_seqlen))


def hstu_attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dout: torch.Tensor,
                  seq_offsets: torch.Tensor, timestamps: Optional[torch.Tensor],
                  pos_bias: Optional[torch.Tensor], time_bias: Optional[torch.Tensor],
                  max_seqlen: int, workspace: Optional[torch.Tensor] = None, out=None,
                  stream=None):
    """Gradients of the attention on tensor cores for the upstream gradient
    dout: q, k, v, dout bf16 [T, H, d] (d = 64 or 128, heads contiguous per
    token, any token stride); returns fp32 (dq, dk, dv, dpos, dtime), dpos /
    dtime None when the term is absent. `out` may pass preallocated (dq, dk,
    dv, dpos, dtime)."""
    _on_cuda(q, k, v, dout, seq_offsets, timestamps, pos_bias, time_bias)
    for t in (q, k, v, dout):
        if t.dtype != torch.bfloat16 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError("q, k, v, dout must be bf16 with heads contiguous in a token")
    T, H, d = q.shape
    B = seq_offsets.numel() - 1
    use_time = timestamps is not None and time_bias is not None
    if out is None:
        f32 = dict(dtype=torch.float32, device=q.device)
        out = (torch.empty((T, H, d), **f32), torch.empty((T, H, d), **f32),
               torch.empty((T, H, d), **f32),
               None if pos_bias is None else torch.empty_like(pos_bias),
               torch.empty_like(time_bias) if use_time else None)
    dq, dk, dv, dpos, dtime = out
    if workspace is None:
        workspace = _workspace(hstu_attn_bwd_workspace_bytes(B, T, max_seqlen), q.device)
    _native.check("hstu_attn_bwd", _lib().hstu_attn_bwd(
        _native.HSTU_DTYPE_BF16, _ptr(q), q.stride(0), _ptr(k), k.stride(0), _ptr(v), v.stride(0),
        _ptr(dout), dout.stride(0), _ptr(seq_offsets), B, T, H, d, _ptr(timestamps),
        _ptr(pos_bias), 0 if pos_bias is None else pos_bias.shape[1], _ptr(time_bias),
        0 if time_bias is None else time_bias.shape[1], int(max_seqlen), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(dpos), _ptr(dtime), _ptr(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv, dpos, dtime


def hstu_attn_bwd_f32(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dout: torch.Tensor,
                      seq_offsets: torch.Tensor, timestamps: Optional[torch.Tensor],
                      pos_bias: Optional[torch.Tensor], time_bias: Optional[torch.Tensor],
                      max_seqlen: int, stream=None):
    """Gradients of the attention for the upstream gradient dout (fp32):
    (dq, dk, dv, dpos, dtime); dpos / dtime are None when the term is absent."""
    _on_cuda(q, k, v, dout, seq_offsets, timestamps, pos_bias, time_bias)
    for t in (q, k, v, dout):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError("q, k, v, dout must be contiguous fp32")
    T, H, dqk = q.shape
    dvd = v.shape[2]
    B = seq_offsets.numel() - 1
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dpos = None if pos_bias is None else torch.empty_like(pos_bias)
    use_time = timestamps is not None and time_bias is not None
    dtime = torch.empty_like(time_bias) if use_time else None
    _native.check("hstu_attn_bwd_f32", _lib().hstu_attn_bwd_f32(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(seq_offsets), B, T, H, dqk, dvd,
        _ptr(timestamps), _ptr(pos_bias), 0 if pos_bias is None else pos_bias.shape[1],
        _ptr(time_bias), 0 if time_bias is None else time_bias.shape[1], int(max_seqlen),
        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dpos), _ptr(dtime), _stream(stream)))
    return dq, dk, dv, dpos, dtime
