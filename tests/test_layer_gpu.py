"""HSTU layer pieces and the full layer on the GPU (through the C ABI) against
the fp64 oracle."""

import numpy as np
import pytest
import torch

import jagged_pointwise_attention_b200 as hstu
import oracle
from gen import make_layer_inputs, round_to_bf16
from gpu_util import assert_bf16_close, dev, errors

pytestmark = pytest.mark.gpu


def bf(a):
    return dev(a, torch.bfloat16)


def test_linear_silu_and_residual():
    rng = np.random.default_rng(0)
    M, K, N = 300, 512, 384          # ragged M tail, several N tiles
    x = round_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    W = round_to_bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    b = (0.1 * rng.standard_normal(N)).astype(np.float32)
    r = round_to_bf16(rng.standard_normal((M, N)).astype(np.float32))
    got = hstu.hstu_linear_fwd(bf(x), bf(W), dev(b), "silu")
    assert hstu.hstu_device_status() == 0
    assert_bf16_close(got.float().cpu().numpy(), oracle.linear(x, W, b, act_silu=True), "silu")
    got = hstu.hstu_linear_fwd(bf(x), bf(W), None, "residual", residual=bf(r))
    assert_bf16_close(got.float().cpu().numpy(), oracle.linear(x, W, None, False, r), "residual")
    got = hstu.hstu_linear_fwd(bf(x), bf(W), dev(b), "none")
    assert_bf16_close(got.float().cpu().numpy(), oracle.linear(x, W, b), "plain")


def test_linear_projection_shapes():
    """The layer's shapes: [T, 512] x [2048, 512]^T and [T, 512] x [512, 512]^T."""
    rng = np.random.default_rng(1)
    M = 1000
    x = round_to_bf16(rng.standard_normal((M, 512)).astype(np.float32))
    W1 = round_to_bf16((rng.standard_normal((2048, 512)) / np.sqrt(512)).astype(np.float32))
    got = hstu.hstu_linear_fwd(bf(x), bf(W1), None, "silu")
    assert hstu.hstu_device_status() == 0
    rows = np.arange(0, M, 7)
    assert_bf16_close(got.float().cpu().numpy()[rows], oracle.linear(x[rows], W1, act_silu=True),
                      "f1 shape")


@pytest.mark.parametrize("N,epi", [(2048, "silu"), (512, "residual"), (384, "none")])
def test_linear_persistent_tiles(N, epi):
    """More output tiles than two per SM, so every CTA reuses both TMEM
    accumulators and several k-block rings; ragged last row block."""
    rng = np.random.default_rng(3)
    M, K = 41000 if N != 2048 else 5300, 512
    x = round_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    W = round_to_bf16((rng.standard_normal((N, K)) / np.sqrt(K)).astype(np.float32))
    b = (0.1 * rng.standard_normal(N)).astype(np.float32)
    r = round_to_bf16(rng.standard_normal((M, N)).astype(np.float32)) if epi == "residual" else None
    got = hstu.hstu_linear_fwd(bf(x), bf(W), dev(b), epi,
                               residual=None if r is None else bf(r))
    assert hstu.hstu_device_status() == 0
    rows = np.concatenate([np.arange(0, M, 97), np.arange(M - 130, M)])
    want = oracle.linear(x[rows], W, b, act_silu=epi == "silu",
                         residual=None if r is None else r[rows])
    assert_bf16_close(got.float().cpu().numpy()[rows], want, f"{epi} N={N}")


def test_layernorm_gate():
    rng = np.random.default_rng(2)
    M, F = 517, 512
    a = round_to_bf16((rng.standard_normal((M, F)) * 0.01 + 0.003).astype(np.float32))
    a[:5] *= 1e-3                                   # rows where eps dominates the variance
    u = round_to_bf16(rng.standard_normal((M, 4 * F)).astype(np.float32))
    g = (1 + 0.1 * rng.standard_normal(F)).astype(np.float32)
    bt = (0.1 * rng.standard_normal(F)).astype(np.float32)
    ud = bf(u)
    got = hstu.hstu_layernorm_gate_fwd(bf(a), ud[:, :F], dev(g), dev(bt), 1e-5)
    assert hstu.hstu_device_status() == 0
    want = oracle.layernorm_gate(a, u[:, :F], g, bt, 1e-5)
    assert_bf16_close(got.float().cpu().numpy(), want, "ln gate")
    got = hstu.hstu_layernorm_gate_fwd(bf(a), ud[:, :F])
    assert_bf16_close(got.float().cpu().numpy(), oracle.layernorm_gate(a, u[:, :F]), "ln identity")


def _layer_gpu(li, **kw):
    out = hstu.hstu_layer_fwd(bf(li.x), bf(li.W1), bf(li.W2), dev(li.seq_offsets),
                              dev(li.timestamps), dev(li.pos_bias), dev(li.time_bias), li.H, li.d,
                              li.max_seqlen, ln_eps=li.ln_eps, **kw)
    assert hstu.hstu_device_status() == 0
    return out.float().cpu().numpy()


def _layer_oracle(li, rows=None):
    return oracle.layer(li.seq_offsets, li.x, li.W1, li.W2, li.H, li.d, li.timestamps,
                        li.pos_bias, li.time_bias, li.max_seqlen, ln_eps=li.ln_eps, rows=rows)


def test_layer_small_full():
    li = make_layer_inputs(5, lengths_override=[130, 0, 1, 257, 40])
    assert_bf16_close(_layer_gpu(li), _layer_oracle(li), "layer small")


def test_layer_workload_sampled_rows():
    li = make_layer_inputs(5)
    got = _layer_gpu(li)
    assert np.all(np.isfinite(got))
    # rows from a few sequences keep the oracle's projection prefixes short
    off = li.seq_offsets
    lens = np.diff(off)
    seqs = [int(np.argmin(lens)), 3, 17]
    rows = []
    for s in seqs:
        o, n = int(off[s]), int(lens[s])
        rows += [o, o + 1, o + 127, o + 128, o + n // 2, o + n - 1]
    rows = np.array(sorted(set(r for r in rows if r < li.T)), dtype=np.int64)
    assert_bf16_close(got[rows], _layer_oracle(li, rows), "layer workload", strict_abs=True)


# --------------------------------------------------------------------------- input LayerNorm

import dataclasses  # noqa: E402


def test_layernorm():
    """The layer's input normalization, affine and identity, on rows where
    eps dominates the variance, on a row-strided view, and M = 0."""
    rng = np.random.default_rng(3)
    M, F = 333, 768
    a = round_to_bf16((rng.standard_normal((M, F)) * 2.0 + 0.5).astype(np.float32))
    a[:4] *= 1e-4
    g = (1 + 0.1 * rng.standard_normal(F)).astype(np.float32)
    bt = (0.1 * rng.standard_normal(F)).astype(np.float32)
    got = hstu.hstu_layernorm_fwd(bf(a), dev(g), dev(bt), 1e-5)
    assert hstu.hstu_device_status() == 0
    assert_bf16_close(got.float().cpu().numpy(), oracle.layernorm(a, g, bt, 1e-5), "layernorm")
    got = hstu.hstu_layernorm_fwd(bf(a))
    assert_bf16_close(got.float().cpu().numpy(), oracle.layernorm(a), "layernorm identity")
    wide = torch.zeros((M, F + 256), dtype=torch.bfloat16, device="cuda")
    wide[:, 128:128 + F] = bf(a)
    got = hstu.hstu_layernorm_fwd(wide[:, 128:128 + F], dev(g), None, 1e-3)
    assert_bf16_close(got.float().cpu().numpy(), oracle.layernorm(a, g, None, 1e-3), "strided")
    assert hstu.hstu_layernorm_fwd(bf(a[:0])).shape == (0, F)


def _shifted(li):
    """Layer inputs whose rows have a mean and a spread far from 0 and 1, so the
    input normalization changes x (the workload's x is N(0, 1) per element)."""
    rng = np.random.default_rng(li.seed + 1)
    T, D = li.x.shape
    x = li.x * rng.uniform(0.3, 2.5, (T, 1)) + rng.uniform(-1.5, 1.5, (T, 1))
    return dataclasses.replace(li, x=round_to_bf16(x.astype(np.float32)))


def _in_affine(D, seed=9):
    rng = np.random.default_rng(seed)
    return ((1 + 0.2 * rng.standard_normal(D)).astype(np.float32),
            (0.2 * rng.standard_normal(D)).astype(np.float32))


def test_layer_input_norm_small_full():
    li = _shifted(make_layer_inputs(5, lengths_override=[130, 0, 1, 257, 40]))
    ig, ib = _in_affine(li.x.shape[1])
    got = _layer_gpu(li, input_norm=True, in_gamma=dev(ig), in_beta=dev(ib))
    want = oracle.layer(li.seq_offsets, li.x, li.W1, li.W2, li.H, li.d, li.timestamps,
                        li.pos_bias, li.time_bias, li.max_seqlen, ln_eps=li.ln_eps,
                        input_norm=True, in_gamma=ig, in_beta=ib)
    assert_bf16_close(got - li.x, want - li.x, "layer input norm (out - x)")
    # without the affine terms, and the normalization is really applied
    got = _layer_gpu(li, input_norm=True)
    want = oracle.layer(li.seq_offsets, li.x, li.W1, li.W2, li.H, li.d, li.timestamps,
                        li.pos_bias, li.time_bias, li.max_seqlen, ln_eps=li.ln_eps,
                        input_norm=True)
    assert_bf16_close(got - li.x, want - li.x, "layer input norm identity (out - x)")
    plain = _layer_gpu(li)
    rel, _ = errors(plain - li.x, want - li.x)
    assert rel > 0.1, rel


def test_layer_input_norm_workload_sampled_rows():
    li = _shifted(make_layer_inputs(5))
    ig, ib = _in_affine(li.x.shape[1])
    got = _layer_gpu(li, input_norm=True, in_gamma=dev(ig), in_beta=dev(ib))
    assert np.all(np.isfinite(got))
    off, lens = li.seq_offsets, np.diff(li.seq_offsets)
    rows = []
    for s in (int(np.argmin(lens)), 5, 29):
        o, n = int(off[s]), int(lens[s])
        rows += [o, o + 64, o + n // 3, o + n - 1]
    rows = np.array(sorted(set(r for r in rows if r < li.T)), dtype=np.int64)
    want = oracle.layer(li.seq_offsets, li.x, li.W1, li.W2, li.H, li.d, li.timestamps,
                        li.pos_bias, li.time_bias, li.max_seqlen, ln_eps=li.ln_eps, rows=rows,
                        input_norm=True, in_gamma=ig, in_beta=ib)
    assert_bf16_close(got[rows] - li.x[rows], want - li.x[rows], "layer input norm workload")
