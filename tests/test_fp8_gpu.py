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


# --------------------------------------------------------------------------- input LayerNorm -> E4M3

import dataclasses  # noqa: E402


def test_layernorm_fp8_is_quant_of_bf16_layernorm():
    """The fused input-LayerNorm-to-E4M3 kernel gives exactly the codes and
    scales of quantizing the bf16 LayerNorm output (both checked against the
    oracle on their own), with and without the affine terms, on a strided view."""
    rng = np.random.default_rng(23)
    M, F = 517, 1024
    a = round_to_bf16((rng.standard_normal((M, F)) * 3.0 - 1.0).astype(np.float32))
    a[:3] *= 1e-4
    g = dev((1 + 0.1 * rng.standard_normal(F)).astype(np.float32))
    bt = dev((0.1 * rng.standard_normal(F)).astype(np.float32))
    wide = torch.zeros((M, F + 512), dtype=torch.bfloat16, device="cuda")
    wide[:, 256:256 + F] = bf(a)
    for src in (bf(a), wide[:, 256:256 + F]):
        for gamma, beta in ((g, bt), (None, None)):
            codes, scales = hstu.hstu_layernorm_fp8_fwd(src, gamma, beta, 1e-5)
            want_c, want_s = hstu.hstu_quant_rows_e4m3(hstu.hstu_layernorm_fwd(src, gamma, beta,
                                                                               1e-5))
            assert hstu.hstu_device_status() == 0
            assert torch.equal(scales, want_s)
            assert torch.equal(codes, want_c)


def _fp8_weights(li):
    W1q, s1 = hstu.hstu_quant_rows_e4m3(bf(li.W1))
    W2q, s2 = hstu.hstu_quant_rows_e4m3(bf(li.W2))
    return W1q, s1, W2q, s2


def _shifted(li):
    rng = np.random.default_rng(li.seed + 1)
    T = li.x.shape[0]
    x = li.x * rng.uniform(0.3, 2.5, (T, 1)) + rng.uniform(-1.5, 1.5, (T, 1))
    return dataclasses.replace(li, x=round_to_bf16(x.astype(np.float32)))


def _layer_fp8_input_norm_oracle(li, ig, ib, W1q, s1, W2q, s2):
    """The FP8 layer with the input LayerNorm, from the oracle's pieces in fp64.
    The kernel quantizes the bf16 value of LayerNorm(x) and of Y, so the oracle
    takes those integer decisions on the same precision: on its fp64 values
    rounded to bf16."""
    H, d, T = li.H, li.d, li.x.shape[0]
    F = H * d
    xn = round_to_bf16(oracle.layernorm(li.x, ig, ib, li.ln_eps).astype(np.float32))
    xq, sx = oracle.quant_rows_e4m3(xn)
    uvqk = oracle.linear_fp8(xq, sx, W1q, s1, act_silu=True)
    u, v, q, k = (uvqk[:, i * F:(i + 1) * F] for i in range(4))
    a = oracle.attn(li.seq_offsets, q.reshape(T, H, d), k.reshape(T, H, d), v.reshape(T, H, d),
                    li.timestamps, li.pos_bias, li.time_bias, li.max_seqlen).reshape(T, F)
    y = oracle.layernorm_gate(a, u, eps=li.ln_eps)
    yq, sy = oracle.quant_rows_e4m3(round_to_bf16(y.astype(np.float32)))
    return oracle.linear_fp8(yq, sy, W2q, s2, residual=li.x), xq, yq


def test_layer_fp8_input_norm_matches_oracle():
    li = _shifted(make_layer_inputs(5, lengths_override=[130, 0, 1, 257, 40]))
    rng = np.random.default_rng(31)
    D = li.x.shape[1]
    ig = (1 + 0.2 * rng.standard_normal(D)).astype(np.float32)
    ib = (0.2 * rng.standard_normal(D)).astype(np.float32)
    W1q, s1, W2q, s2 = _fp8_weights(li)
    got = hstu.hstu_layer_fp8_fwd(bf(li.x), W1q, s1, W2q, s2, dev(li.seq_offsets),
                                  dev(li.timestamps), dev(li.pos_bias), dev(li.time_bias), li.H,
                                  li.d, li.max_seqlen, ln_eps=li.ln_eps, input_norm=True,
                                  in_gamma=dev(ig), in_beta=dev(ib))
    assert hstu.hstu_device_status() == 0
    want, _, _ = _layer_fp8_input_norm_oracle(li, ig, ib, W1q.cpu().numpy(), s1.cpu().numpy(),
                                              W2q.cpu().numpy(), s2.cpu().numpy())
    # the FP8 layer bar (twice the bf16 bar, see test_layer_fp8_matches_oracle),
    # on the layer's contribution out - x
    g = got.float().cpu().numpy()
    rel, mx = errors(g - li.x, want - li.x)
    assert rel <= 2e-2 and mx <= 3e-2 * max(1.0, float(np.abs(want - li.x).max())), (rel, mx)


def test_layer_fp8_is_its_pieces_and_each_piece_meets_the_bf16_bar():
    """The tight form of the FP8 layer's parity. The layer equals, bit for bit,
    its public pieces run one after another (input LayerNorm to E4M3, f1, the
    attention, the LayerNorm gate to E4M3, f2); each piece, fed the kernel's
    own inputs to it (the E4M3 codes and scales included), meets the bf16 bar
    against the oracle; and the E4M3 codes that the kernels decide differ from
    the oracle's end-to-end fp64 decisions in a small, reported fraction."""
    li = _shifted(make_layer_inputs(5, lengths_override=[300, 0, 700, 1, 129]))
    rng = np.random.default_rng(37)
    D = li.x.shape[1]
    H, d, T = li.H, li.d, li.x.shape[0]
    F = H * d
    ig = dev((1 + 0.2 * rng.standard_normal(D)).astype(np.float32))
    ib = dev((0.2 * rng.standard_normal(D)).astype(np.float32))
    W1q, s1, W2q, s2 = _fp8_weights(li)
    x, off, ts, pb, tb = (bf(li.x), dev(li.seq_offsets), dev(li.timestamps), dev(li.pos_bias),
                          dev(li.time_bias))
    layer = hstu.hstu_layer_fp8_fwd(x, W1q, s1, W2q, s2, off, ts, pb, tb, H, d, li.max_seqlen,
                                    ln_eps=li.ln_eps, input_norm=True, in_gamma=ig, in_beta=ib)
    xq, sx = hstu.hstu_layernorm_fp8_fwd(x, ig, ib, li.ln_eps)
    uvqk = hstu.hstu_linear_fp8_fwd(xq, sx, W1q, s1, epilogue="silu")
    u, v, q, k = (uvqk[:, i * F:(i + 1) * F] for i in range(4))
    a = hstu.hstu_attn_fwd(q.view(T, H, d), k.view(T, H, d), v.view(T, H, d), off, ts, pb, tb,
                           li.max_seqlen).view(T, F)
    yq, sy = hstu.hstu_layernorm_gate_fp8_fwd(a, u, eps=li.ln_eps)
    out = hstu.hstu_linear_fp8_fwd(yq, sy, W2q, s2, epilogue="residual", residual=x)
    assert hstu.hstu_device_status() == 0
    assert torch.equal(layer, out), "the layer is not the composition of its pieces"
    n = lambda t: t.cpu().numpy()  # noqa: E731
    W1n, s1n, W2n, s2n = n(W1q), n(s1), n(W2q), n(s2)
    # f1 and f2 from the kernel's own codes: the bf16 bar
    assert_bf16_close(n(uvqk.float()), oracle.linear_fp8(n(xq), n(sx), W1n, s1n, act_silu=True),
                      "f1 from the kernel's x codes")
    f2 = oracle.linear_fp8(n(yq), n(sy), W2n, s2n, residual=li.x)
    assert_bf16_close(n(layer.float()) - li.x, f2 - li.x, "f2 from the kernel's Y codes")
    # the attention and the LayerNorm gate from the kernel's own U, V, Q, K and A
    uv = n(uvqk.float())
    U, V, Q, K = (uv[:, i * F:(i + 1) * F] for i in range(4))
    a_o = oracle.attn(li.seq_offsets, Q.reshape(T, H, d), K.reshape(T, H, d), V.reshape(T, H, d),
                      li.timestamps, li.pos_bias, li.time_bias, li.max_seqlen).reshape(T, F)
    assert_bf16_close(n(a.float()), a_o, "attention from the kernel's Q, K, V")
    y_o = oracle.layernorm_gate(n(a.float()), U, eps=li.ln_eps)
    yq_p, sy_p = oracle.quant_rows_e4m3(round_to_bf16(y_o.astype(np.float32)))
    flips_piece = float(np.mean(n(yq) != yq_p))
    # E4M3 codes against the oracle's decisions. The input LayerNorm's codes
    # differ only where the kernel's bf16 LayerNorm and the oracle's
    # bf16(fp64 LayerNorm) differ by an ulp across an E4M3 rounding boundary:
    # rarely. Y's codes, decided from the kernel's own A and U, likewise. Y's
    # codes against the oracle's end-to-end fp64 chain differ far more often:
    # the kernel rounds U, V, Q, K, P and A to bf16 (2^-9 relative), and a
    # code flips wherever that moves Y across an E4M3 rounding boundary
    # (spaced 2^-4 to 2^-3 relative), so about a tenth of the codes; f2 sums
    # those one-step differences, which is why the end-to-end bar is twice
    # the bf16 bar.
    _, xq_o, yq_o = _layer_fp8_input_norm_oracle(li, n(ig), n(ib), W1n, s1n, W2n, s2n)
    flips_x = float(np.mean(n(xq) != xq_o))
    flips_y = float(np.mean(n(yq) != yq_o))
    print("E4M3 code flips against the oracle: x' %.4f%%, Y from the kernel's A and U %.4f%%, "
          "Y end to end %.4f%%" % (100 * flips_x, 100 * flips_piece, 100 * flips_y))
    assert flips_x <= 1e-3 and flips_piece <= 1e-2 and flips_y <= 0.2, (flips_x, flips_piece,
                                                                         flips_y)
