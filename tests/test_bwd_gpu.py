"""Attention backward on the GPU (fp32, through the C ABI) against the fp64
oracle's gradients."""

import numpy as np
import pytest
import torch

import jagged_pointwise_attention_b200 as hstu
import oracle
from gen import custom_attn_inputs
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
