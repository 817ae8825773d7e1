"""Attention backward on the GPU (fp32, through the C ABI) against the fp64
oracle's gradients."""

import numpy as np
import pytest
import torch

import jagged_pointwise_attention_b200 as hstu
import oracle
from gen import custom_attn_inputs, round_to_bf16
from gpu_util import dev, errors

pytestmark = pytest.mark.gpu

F32_REL = 1e-4


def _check(inp, dout, what, pos=True, time=True):
    ts = inp.timestamps if time else None
    tb = inp.time_bias if time else None
    pb = inp.pos_bias if pos else None
    got = hstu.hstu_attn_bwd_f32(dev(inp.q), dev(inp.k), dev(inp.v), dev(dout),
                                 dev(inp.seq_offsets), None if ts is None else dev(ts),
                                 None if pb is None else dev(pb), None if tb is None else dev(tb),
                                 inp.max_seqlen)
    assert hstu.hstu_device_status() == 0
    want = oracle.attn_bwd(inp.seq_offsets, inp.q, inp.k, inp.v, ts, pb, tb, inp.max_seqlen, dout)
    for name, g, w in zip(("dq", "dk", "dv", "dpos", "dtime"), got, want):
        if w is None:
            assert g is None, name
            continue
        rel, mx = errors(g.cpu().numpy(), w)
        assert rel <= F32_REL, "%s %s: rel-Frobenius %.3e" % (what, name, rel)


@pytest.mark.parametrize("d", [32, 64, 128])
def test_bwd_ragged_batch(d):
    """Ragged lengths over several 128-token blocks, an empty and a length-one
    sequence; position clip and bucket clamp both bind (small tables)."""
    inp = custom_attn_inputs([1, 200, 0, 37, 300, 130], H=2, d=d, num_pos=96, num_buckets=24,
                             dtype="f32", seed=d)
    dout = np.random.default_rng(d).standard_normal(inp.v.shape).astype(np.float32)
    _check(inp, dout, "d=%d" % d)


def test_bwd_terms_dropped():
    inp = custom_attn_inputs([50, 3, 90], H=1, d=32, num_pos=64, num_buckets=32, dtype="f32",
                             seed=2)
    dout = np.random.default_rng(2).standard_normal(inp.v.shape).astype(np.float32)
    _check(inp, dout, "no time", time=False)
    _check(inp, dout, "no pos", pos=False)
    _check(inp, dout, "no bias", pos=False, time=False)


def test_bwd_linear_in_dout():
    """dv is linear in dout: doubling dout doubles every gradient (a property
    that holds whatever the size)."""
    inp = custom_attn_inputs([400, 260], H=2, d=64, num_pos=512, num_buckets=128, dtype="f32",
                             seed=9)
    dout = np.random.default_rng(9).standard_normal(inp.v.shape).astype(np.float32)
    a = hstu.hstu_attn_bwd_f32(dev(inp.q), dev(inp.k), dev(inp.v), dev(dout),
                               dev(inp.seq_offsets), dev(inp.timestamps), dev(inp.pos_bias),
                               dev(inp.time_bias), inp.max_seqlen)
    b = hstu.hstu_attn_bwd_f32(dev(inp.q), dev(inp.k), dev(inp.v), dev(2 * dout),
                               dev(inp.seq_offsets), dev(inp.timestamps), dev(inp.pos_bias),
                               dev(inp.time_bias), inp.max_seqlen)
    assert hstu.hstu_device_status() == 0
    for x, y in zip(a, b):
        assert torch.allclose(2 * x, y, rtol=1e-5, atol=1e-6)


# --------------------------------------------------------------------------- tensor-core backward

BF16_GRAD_REL = 1e-2   # the bf16 bar: p and ds are rounded to bf16 (2^-9) before the products


def _bf16_inputs(lengths, H, d, num_pos, num_buckets, seed):
    inp = custom_attn_inputs(lengths, H=H, d=d, num_pos=num_pos, num_buckets=num_buckets,
                             dtype="bf16", seed=seed)
    dout = round_to_bf16(np.random.default_rng(seed + 1).standard_normal(inp.v.shape)
                         .astype(np.float32))
    return inp, dout


def _tc_bwd(inp, dout, pos=True, time=True):
    bf = torch.bfloat16
    ts = dev(inp.timestamps) if time else None
    tb = dev(inp.time_bias) if time else None
    pb = dev(inp.pos_bias) if pos else None
    got = hstu.hstu_attn_bwd(dev(inp.q, bf), dev(inp.k, bf), dev(inp.v, bf), dev(dout, bf),
                             dev(inp.seq_offsets), ts, pb, tb, inp.max_seqlen)
    assert hstu.hstu_device_status() == 0
    return got


def _check_tc(inp, dout, what, pos=True, time=True):
    got = _tc_bwd(inp, dout, pos, time)
    want = oracle.attn_bwd(inp.seq_offsets, inp.q, inp.k, inp.v, inp.timestamps if time else None,
                           inp.pos_bias if pos else None, inp.time_bias if time else None,
                           inp.max_seqlen, dout)
    for name, g, w in zip(("dq", "dk", "dv", "dpos", "dtime"), got, want):
        if w is None:
            assert g is None, name
            continue
        g = g.cpu().numpy()
        assert np.all(np.isfinite(g)), "%s %s: non-finite" % (what, name)
        rel, _ = errors(g, w)
        assert rel <= BF16_GRAD_REL, "%s %s: rel-Frobenius %.3e" % (what, name, rel)


@pytest.mark.parametrize("d", [64, 128])
def test_tc_bwd_ragged_batch(d):
    """Lengths over several 128-token tiles with ragged tails, an empty and a
    length-one sequence, short ones packed into shared tiles; position clip
    and bucket clamp both bind (small tables)."""
    inp, dout = _bf16_inputs([1, 200, 0, 37, 300, 130, 5, 64], H=2, d=d, num_pos=96,
                             num_buckets=24, seed=40 + d)
    _check_tc(inp, dout, "d=%d" % d)


def test_tc_bwd_long_sequences_many_steps():
    """Key tiles that walk many query tiles (the dK/dV accumulation across
    steps, the two-stage Q/dO ring and item boundaries)."""
    inp, dout = _bf16_inputs([700, 129, 256, 0, 513], H=2, d=128, num_pos=1024,
                             num_buckets=64, seed=7)
    _check_tc(inp, dout, "long")


def test_tc_bwd_sequence_over_2k_tokens():
    """A ragged batch with a 2100-token sequence (17 key tiles walking up to
    17 query tiles each) against the oracle, d = 128, bias tables that clip
    and clamp."""
    inp, dout = _bf16_inputs([2100, 300, 1], H=1, d=128, num_pos=1500, num_buckets=40, seed=14)
    _check_tc(inp, dout, "2100 tokens")


def test_tc_bwd_packed_short_sequences():
    """Batches of short sequences share tiles: pairs across a sequence
    boundary inside a tile must contribute nothing."""
    lengths = [3, 90, 1, 20, 0, 5, 128, 64, 17, 17, 40, 2]
    inp, dout = _bf16_inputs(lengths, H=3, d=64, num_pos=200, num_buckets=128, seed=11)
    _check_tc(inp, dout, "packed")


def test_tc_bwd_terms_dropped():
    inp, dout = _bf16_inputs([50, 3, 190], H=1, d=64, num_pos=64, num_buckets=32, seed=12)
    _check_tc(inp, dout, "no time", time=False)
    _check_tc(inp, dout, "no pos", pos=False)
    _check_tc(inp, dout, "no bias", pos=False, time=False)


def test_tc_bwd_linear_in_dout():
    """Doubling dout doubles every gradient (exactly up to the order of the
    atomic sums), at any size."""
    inp, dout = _bf16_inputs([400, 260, 1000], H=2, d=128, num_pos=512, num_buckets=128, seed=13)
    a = _tc_bwd(inp, dout)
    b = _tc_bwd(inp, 2 * dout)
    # dv is a sum in TMEM of exactly doubled terms: exactly doubled; dk too
    # (ds doubles exactly, so does its bf16 rounding); dq and the tables are
    # sums of atomics in run-dependent order, with cancellation in the tables
    for name, x, y in zip(("dq", "dk", "dv", "dpos", "dtime"), a, b):
        if name in ("dk", "dv"):
            assert torch.equal(2 * x, y), name
        else:
            rel = ((2 * x - y).double().norm() / y.double().norm()).item()
            assert rel <= 1e-5, (name, rel)


@pytest.mark.parametrize("cfg", [2, 4])
def test_tc_bwd_workload_against_fp32_backward(cfg):
    """At the workloads' full sizes the fp64 oracle is out of reach; the fp32
    backward (pinned to the oracle at 1e-4 above) on the same bf16 values
    stands in for it, at the bf16 bar."""
    from gen import make_attn_inputs
    inp = make_attn_inputs(cfg)
    dout = round_to_bf16(np.random.default_rng(cfg).standard_normal(inp.v.shape)
                         .astype(np.float32))
    got = _tc_bwd(inp, dout)
    f32 = hstu.hstu_attn_bwd_f32(dev(inp.q), dev(inp.k), dev(inp.v), dev(dout),
                                 dev(inp.seq_offsets), dev(inp.timestamps), dev(inp.pos_bias),
                                 dev(inp.time_bias), inp.max_seqlen)
    assert hstu.hstu_device_status() == 0
    for name, g, w in zip(("dq", "dk", "dv", "dpos", "dtime"), got, f32):
        g, w = g.double(), w.double()
        rel = ((g - w).norm() / w.norm()).item()
        assert torch.isfinite(g).all(), name
        assert rel <= BF16_GRAD_REL, "cfg %d %s: rel-Frobenius %.3e" % (cfg, name, rel)
