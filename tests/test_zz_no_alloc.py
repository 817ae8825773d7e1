"""hstu_attn_fwd_noalloc: the attention entry point for callers that cannot
allocate device memory when they run it (for instance an inference-engine
plugin whose enqueue step must not call cudaMalloc). It keeps its work list in
a fixed device array inside the library instead of a caller workspace.

Called through the C ABI and compared with hstu_attn_fwd (which takes a
workspace) bit for bit, and with the oracle, on several batches in a row, so
the later calls also show that the shared array left over from an earlier,
larger call does no harm. The file name makes pytest collect it after every
other test."""

import numpy as np
import pytest
import torch

import jagged_pointwise_attention_b200 as hstu
from jagged_pointwise_attention_b200 import _native
import oracle
from gen import custom_attn_inputs, make_attn_inputs
from gpu_util import assert_bf16_close, attn_tensors

pytestmark = pytest.mark.gpu


def _noalloc(lib, t, inp, out, ts=True, pos=True, tb=True):
    T, H, d = t["q"].shape
    p = lambda x, on: x.data_ptr() if on else None  # noqa: E731
    st = lib.hstu_attn_fwd_noalloc(
        _native.HSTU_DTYPE_BF16, t["q"].data_ptr(), H * d, t["k"].data_ptr(), H * d,
        t["v"].data_ptr(), H * d, t["seq_offsets"].data_ptr(), inp.B, T, H, d, d,
        p(t["timestamps"], ts), p(t["pos_bias"], pos), t["pos_bias"].shape[1] if pos else 0,
        p(t["time_bias"], tb), t["time_bias"].shape[1] if tb else 0, inp.max_seqlen,
        out.data_ptr(), H * d, torch.cuda.current_stream().cuda_stream)
    return st


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    """Bit-identical to hstu_attn_fwd (the same kernels on the same inputs),
    within the bf16 bar of the oracle, on four calls in a row: a short-history
    batch, a smaller batch with long sequences and empty ones, and then, after
    the larger batch has left its work list in the shared array, a small batch
    without the time term and then without any bias term. Every output row is
    pre-filled with NaN, so an unwritten row fails."""
    lib = _native.load()
    small = custom_attn_inputs([3, 90, 1, 200], H=2, d=64, num_pos=256, num_buckets=64,
                               dtype="bf16", seed=78, bias_std=0.5)
    calls = [(make_attn_inputs(2), {}),
             (custom_attn_inputs([700, 1, 0, 129, 256], H=3, d=128, num_pos=1024,
                                 num_buckets=128, dtype="bf16", seed=77), {}),
             (small, dict(ts=False, tb=False)),
             (small, dict(ts=False, pos=False, tb=False))]
    for n, (inp, drop) in enumerate(calls):
        t = attn_tensors(inp)
        ts = t["timestamps"] if drop.get("ts", True) else None
        pos = t["pos_bias"] if drop.get("pos", True) else None
        tb = t["time_bias"] if drop.get("tb", True) else None
        want = hstu.hstu_attn_fwd(t["q"], t["k"], t["v"], t["seq_offsets"], ts, pos, tb,
                                  inp.max_seqlen)
        got = torch.full_like(want, float("nan"))
        assert _noalloc(lib, t, inp, got, **drop) == _native.HSTU_OK
        assert hstu.hstu_device_status() == 0
        g, w = got.float().cpu().numpy(), want.float().cpu().numpy()
        assert np.all(np.isfinite(g)), "call %d left rows unwritten" % n
        assert np.array_equal(g, w), "call %d differs from hstu_attn_fwd" % n
        if n > 0:   # the short-history batch is checked against the oracle elsewhere
            ref = oracle.attn(inp.seq_offsets, inp.q, inp.k, inp.v,
                              inp.timestamps if drop.get("ts", True) else None,
                              inp.pos_bias if drop.get("pos", True) else None,
                              inp.time_bias if drop.get("tb", True) else None, inp.max_seqlen)
            assert_bf16_close(g, ref, "no-alloc call %d against the oracle" % n)


def test_noalloc_rejects_batches_beyond_its_scratch():
    lib = _native.load()
    # 70000 sequences (70000 work units: 2.2 MB of work list, 40 MB of key
    # summaries) need more than the 16 MiB scratch array: refused on the host
    # before anything is launched
    B, T = 70000, 70000 * 4
    st = lib.hstu_attn_fwd_noalloc(_native.HSTU_DTYPE_BF16, 16, 512, 16, 512, 16, 512, 16, B, T,
                                   4, 128, 128, None, None, 0, None, 0, 4, 16, 512, None)
    assert st == _native.HSTU_ERR_UNSUPPORTED
