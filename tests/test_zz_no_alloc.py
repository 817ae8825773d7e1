"""hstu_attn_fwd_noalloc: the attention entry point for callers that cannot
allocate device memory when they run it (for instance an inference-engine
plugin whose enqueue step must not call cudaMalloc). It keeps its work list in
a fixed device array inside the library instead of a caller workspace.

Called through the C ABI and compared with hstu_attn_fwd (which takes a
workspace) on two different batches in a row, so the second call also shows
that the shared array left over from the first call does no harm. The file
name makes pytest collect it after every other test."""

import numpy as np
import pytest
import torch

import jagged_pointwise_attention_b200 as hstu
from jagged_pointwise_attention_b200 import _native
from gen import custom_attn_inputs, make_attn_inputs
from gpu_util import assert_bf16_close, attn_tensors

pytestmark = pytest.mark.gpu


def _noalloc(lib, t, inp, out):
    T, H, d = t["q"].shape
    st = lib.hstu_attn_fwd_noalloc(
        _native.HSTU_DTYPE_BF16, t["q"].data_ptr(), H * d, t["k"].data_ptr(), H * d,
        t["v"].data_ptr(), H * d, t["seq_offsets"].data_ptr(), inp.B, T, H, d, d,
        t["timestamps"].data_ptr(), t["pos_bias"].data_ptr(), t["pos_bias"].shape[1],
        t["time_bias"].data_ptr(), t["time_bias"].shape[1], inp.max_seqlen, out.data_ptr(), H * d,
        torch.cuda.current_stream().cuda_stream)
    return st


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    lib = _native.load()
    batches = [make_attn_inputs(2),
               custom_attn_inputs([700, 1, 0, 129, 256], H=3, d=128, num_pos=1024,
                                  num_buckets=128, dtype="bf16", seed=77)]
    for n, inp in enumerate(batches):
        t = attn_tensors(inp)
        want = hstu.hstu_attn_fwd(t["q"], t["k"], t["v"], t["seq_offsets"], t["timestamps"],
                                  t["pos_bias"], t["time_bias"], inp.max_seqlen)
        got = torch.full_like(want, float("nan"))
        assert _noalloc(lib, t, inp, got) == _native.HSTU_OK
        assert hstu.hstu_device_status() == 0
        g, w = got.float().cpu().numpy(), want.float().cpu().numpy()
        assert np.all(np.isfinite(g)), "call %d left rows unwritten" % n
        assert_bf16_close(g, w, "no-alloc call %d" % n)


def test_noalloc_rejects_batches_beyond_its_scratch():
    lib = _native.load()
    # 70000 sequences (70000 work units: 2.2 MB of work list, 40 MB of key
    # summaries) need more than the 16 MiB scratch array: refused on the host
    # before anything is launched
    B, T = 70000, 70000 * 4
    st = lib.hstu_attn_fwd_noalloc(_native.HSTU_DTYPE_BF16, 16, 512, 16, 512, 16, 512, 16, B, T,
                                   4, 128, 128, None, None, 0, None, 0, 4, 16, 512, None)
    assert st == _native.HSTU_ERR_UNSUPPORTED
