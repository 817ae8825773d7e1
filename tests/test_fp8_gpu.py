"""Row-wise E4M3 quantization and the FP8 projections on the GPU (through the
C ABI) against the fp64 oracle: codes and scales bit-exact, products within
the bf16 output tolerance."""

import numpy as np
import pytest
import torch

import jagged_pointwise_attention_b200 as hstu
import oracle
from gen import round_to_bf16
from gpu_util import assert_bf16_close, dev, errors

pytestmark = pytest.mark.gpu


def bf(a):
    return dev(a, torch.bfloat16)


def _quant_both(x):
    """GPU codes/scales of x (already bf16-representable) and the oracle's."""
    codes, scales = hstu.hstu_quant_rows_e4m3(bf(x))
    assert hstu.hstu_device_status() == 0
    want_c, want_s = oracle.quant_rows_e4m3(x.astype(np.float32))
    return codes.cpu().numpy(), scales.cpu().numpy(), want_c, want_s


@pytest.mark.parametrize("M,K", [(1, 16), (37, 512), (300, 2048), (5, 272)])
def test_quant_codes_bit_exact(M, K):
    rng = np.random.default_rng(M + K)
    x = round_to_bf16((rng.standard_normal((M, K)) *
                       np.exp(rng.uniform(-8, 8, (M, 1)))).astype(np.float32))
    got_c, got_s, want_c, want_s = _quant_both(x)
    assert np.array_equal(got_s, want_s), "scales"
    bad = np.argwhere(got_c != want_c)
    assert bad.size == 0, "codes differ at %s" % bad[:5].tolist()


def test_quant_edge_rows():
    """All-zero rows (signed zeros kept), a row whose amax is a power of two,
    one tiny value among large ones (underflow to a subnormal or zero code),
    a row of equal magnitudes, and a row too small for a finite 448 / amax
    (quantized like a zero row, never to NaN codes)."""
    K = 64
    x = np.zeros((7, K), dtype=np.float32)
    x[1, ::2] = -0.0
    x[2] = np.linspace(-4, 4, K)
    x[3, 0], x[3, 1:] = 3e-6, 1000.0
    x[4] = -7.5
    x[5] = round_to_bf16(np.random.default_rng(0).standard_normal(K).astype(np.float32)) * 1e-30
    x[6] = np.random.default_rng(1).standard_normal(K).astype(np.float32) * 1e-37
    x = round_to_bf16(x)
    got_c, got_s, want_c, want_s = _quant_both(x)
    assert np.array_equal(got_s, want_s)
    assert np.array_equal(got_c, want_c)
    assert not np.any((got_c & 0x7F) == 0x7F), "NaN codes"


@pytest.mark.parametrize("M,K,N,epi", [(300, 512, 384, "silu"), (1000, 512, 2048, "silu"),
                                       (257, 512, 512, "residual"), (130, 256, 128, "none")])
def test_linear_fp8_matches_oracle(M, K, N, epi):
    """FP8 projection from GPU-quantized operands (several N tiles, ragged M)
    against the oracle's fp64 product of the same codes."""
    rng = np.random.default_rng(M * 7 + N)
    x = round_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    W = round_to_bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    b = (0.1 * rng.standard_normal(N)).astype(np.float32)
    r = round_to_bf16(rng.standard_normal((M, N)).astype(np.float32)) if epi == "residual" else None
    xq, sx = hstu.hstu_quant_rows_e4m3(bf(x))
    wq, sw = hstu.hstu_quant_rows_e4m3(bf(W))
    got = hstu.hstu_linear_fp8_fwd(xq, sx, wq, sw, dev(b), epi,
                                   residual=None if r is None else bf(r))
    assert hstu.hstu_device_status() == 0
    oxq, osx = oracle.quant_rows_e4m3(x)
    owq, osw = oracle.quant_rows_e4m3(W)
    assert np.array_equal(xq.cpu().numpy(), oxq) and np.array_equal(wq.cpu().numpy(), owq)
    want = oracle.linear_fp8(oxq, osx, owq, osw, b, act_silu=epi == "silu", residual=r)
    assert_bf16_close(got.float().cpu().numpy(), want, "fp8 %s" % epi)


def test_linear_fp8_persistent_tiles():
    """More output tiles than two per SM (both TMEM accumulators reused),
    sampled rows."""
    rng = np.random.default_rng(11)
    M, K, N = 9000, 512, 2048
    x = round_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    W = round_to_bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    xq, sx = hstu.hstu_quant_rows_e4m3(bf(x))
    wq, sw = hstu.hstu_quant_rows_e4m3(bf(W))
    got = hstu.hstu_linear_fp8_fwd(xq, sx, wq, sw, None, "silu")
    assert hstu.hstu_device_status() == 0
    rows = np.concatenate([np.arange(0, M, 61), np.arange(M - 70, M)])
    oxq, osx = oracle.quant_rows_e4m3(x[rows])
    owq, osw = oracle.quant_rows_e4m3(W)
    want = oracle.linear_fp8(oxq, osx, owq, osw, act_silu=True)
    assert_bf16_close(got.float().cpu().numpy()[rows], want, "fp8 persistent")


def test_fp8_close_to_bf16_projection():
    """The FP8 projection stays near the bf16 one (quantization error of a
    3-bit mantissa on both operands), a sanity bound, not the parity bar."""
    rng = np.random.default_rng(5)
    M, K, N = 512, 512, 512
    x = round_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    W = round_to_bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    xq, sx = hstu.hstu_quant_rows_e4m3(bf(x))
    wq, sw = hstu.hstu_quant_rows_e4m3(bf(W))
    f8 = hstu.hstu_linear_fp8_fwd(xq, sx, wq, sw).float().cpu().numpy()
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    assert np.linalg.norm(f8 - ref) / np.linalg.norm(ref) < 0.06


def test_fp8_argument_checks():
    x = torch.zeros((4, 100), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hstu.HstuError):
        hstu.hstu_quant_rows_e4m3(x)              # K % 16
    q = torch.zeros((4, 192), dtype=torch.uint8, device="cuda")
    s = torch.ones(4, dtype=torch.float32, device="cuda")
    with pytest.raises(hstu.HstuError):
        hstu.hstu_linear_fp8_fwd(q, s, torch.zeros((128, 192), dtype=torch.uint8, device="cuda"),
                                 torch.ones(128, dtype=torch.float32, device="cuda"))   # K % 128


# --------------------------------------------------------------------------- FP8 layer

from gen import make_layer_inputs  # noqa: E402


def test_ln_gate_fp8_is_quant_of_bf16_ln_gate():
    """The fused LayerNorm-gate-to-E4M3 kernel gives exactly the codes and
    scales of quantizing the bf16 LayerNorm gate output (both parts are
    checked against the oracle on their own)."""
    rng = np.random.default_rng(21)
    M, F = 777, 512
    a = round_to_bf16((rng.standard_normal((M, F)) * 0.01 + 0.003).astype(np.float32))
    u = round_to_bf16(rng.standard_normal((M, 4 * F)).astype(np.float32))
    ad, ud = bf(a), bf(u)
    g = dev((1 + 0.1 * rng.standard_normal(F)).astype(np.float32))
    bt = dev((0.1 * rng.standard_normal(F)).astype(np.float32))
    codes, scales = hstu.hstu_layernorm_gate_fp8_fwd(ad, ud[:, :F], g, bt, 1e-5)
    y = hstu.hstu_layernorm_gate_fwd(ad, ud[:, :F], g, bt, 1e-5)
    want_c, want_s = hstu.hstu_quant_rows_e4m3(y)
    assert hstu.hstu_device_status() == 0
    assert torch.equal(scales, want_s)
    assert torch.equal(codes, want_c)


def _layer_fp8_oracle(li, W1q, s1, W2q, s2):
    """The FP8 layer composed from the oracle's pieces in fp64: x quantized
    row-wise (the same fp32 decision as the kernel: x is bf16-exact), f1 from
    the codes, attention, LayerNorm gate, Y quantized row-wise, f2 from the
    codes plus the residual. The kernel quantizes the bf16 value of Y, so the
    oracle takes that integer decision in the same precision: on Y rounded to
    bf16."""
    H, d = li.H, li.d
    F = H * d
    xq, sx = oracle.quant_rows_e4m3(li.x)
    uvqk = oracle.linear_fp8(xq, sx, W1q, s1, act_silu=True)
    T = li.x.shape[0]
    u, v, q, k = (uvqk[:, i * F:(i + 1) * F] for i in range(4))
    a = oracle.attn(li.seq_offsets, q.reshape(T, H, d), k.reshape(T, H, d), v.reshape(T, H, d),
                    li.timestamps, li.pos_bias, li.time_bias, li.max_seqlen).reshape(T, F)
    y = oracle.layernorm_gate(a, u, eps=li.ln_eps)
    yq, sy = oracle.quant_rows_e4m3(round_to_bf16(y.astype(np.float32)))
    return oracle.linear_fp8(yq, sy, W2q, s2, residual=li.x)


def test_layer_fp8_matches_oracle():
    li = make_layer_inputs(5, lengths_override=[130, 0, 1, 257, 40])
    W1q, s1 = hstu.hstu_quant_rows_e4m3(bf(li.W1))
    W2q, s2 = hstu.hstu_quant_rows_e4m3(bf(li.W2))
    got = hstu.hstu_layer_fp8_fwd(bf(li.x), W1q, s1, W2q, s2, dev(li.seq_offsets),
                                  dev(li.timestamps), dev(li.pos_bias), dev(li.time_bias), li.H,
                                  li.d, li.max_seqlen, ln_eps=li.ln_eps)
    assert hstu.hstu_device_status() == 0
    want = _layer_fp8_oracle(li, W1q.cpu().numpy(), s1.cpu().numpy(), W2q.cpu().numpy(),
                             s2.cpu().numpy())
    # The FP8 layer's bar is twice the bf16 bar (rel-Frobenius 2e-2, max-abs
    # unchanged): besides the bf16 layer's roundings (U, V, Q, K, A and Y in
    # bf16), Y's E4M3 codes are decided on the kernel's bf16 Y and on the
    # oracle's bf16(fp64 Y); where the two bf16 values straddle an E4M3
    # rounding boundary the code differs by one step (2^-3 relative), and f2
    # sums those differences.
    rel, mx = errors(got.float().cpu().numpy(), want)
    assert rel <= 2e-2 and mx <= 3e-2 * max(1.0, float(np.abs(want).max())), (rel, mx)


def test_layer_fp8_close_to_bf16_layer():
    """FP8 and bf16 layers on the same inputs differ by the quantization of the
    projections only (a sanity bound, not the parity bar)."""
    li = make_layer_inputs(5, lengths_override=[300, 700, 5])
    W1q, s1 = hstu.hstu_quant_rows_e4m3(bf(li.W1))
    W2q, s2 = hstu.hstu_quant_rows_e4m3(bf(li.W2))
    args = (dev(li.seq_offsets), dev(li.timestamps), dev(li.pos_bias), dev(li.time_bias), li.H,
            li.d, li.max_seqlen)
    f8 = hstu.hstu_layer_fp8_fwd(bf(li.x), W1q, s1, W2q, s2, *args, ln_eps=li.ln_eps)
    b16 = hstu.hstu_layer_fwd(bf(li.x), bf(li.W1), bf(li.W2), *args, ln_eps=li.ln_eps)
    assert hstu.hstu_device_status() == 0
    f8, b16, x = f8.float(), b16.float(), bf(li.x).float()
    # compare the layer's contribution (out - x), where the quantization shows
    rel = ((f8 - x) - (b16 - x)).norm() / (b16 - x).norm()
    assert rel.item() < 0.08
