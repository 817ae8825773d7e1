"""Row-wise E4M3 quantization and the FP8 projections on the GPU (through the
C ABI) against the fp64 oracle: codes and scales bit-exact, products within
the bf16 output tolerance."""

import numpy as np
import pytest
import torch

import jagged_pointwise_attention_b200 as hstu
import oracle
from gen import round_to_bf16
from gpu_util import assert_bf16_close, dev

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
    a row of equal magnitudes."""
    K = 64
    x = np.zeros((6, K), dtype=np.float32)
    x[1, ::2] = -0.0
    x[2] = np.linspace(-4, 4, K)
    x[3, 0], x[3, 1:] = 3e-6, 1000.0
    x[4] = -7.5
    x[5] = round_to_bf16(np.random.default_rng(0).standard_normal(K).astype(np.float32)) * 1e-30
    x = round_to_bf16(x)
    got_c, got_s, want_c, want_s = _quant_both(x)
    assert np.array_equal(got_s, want_s)
    assert np.array_equal(got_c, want_c)


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
