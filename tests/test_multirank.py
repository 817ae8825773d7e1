"""Multi-rank host logic with world size 2 over gloo on CPU: sequence sharding
covers the batch exactly once with balanced cost, sharded results reassemble
to the unsharded ones, and the benchmark's timing reductions (max time, summed
work) agree across ranks."""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from jagged_pointwise_attention_b200.shard import partition_sequences, sequence_costs, shard_offsets


def test_partition_covers_once_and_balances():
    rng = np.random.default_rng(0)
    for world in (1, 2, 3, 8):
        lens = rng.integers(0, 8193, size=37)
        parts = partition_sequences(lens, world)
        allx = np.sort(np.concatenate(parts))
        assert np.array_equal(allx, np.arange(len(lens)))
        loads = [int(sequence_costs(lens[p]).sum()) for p in parts]
        # LPT bound: max load <= mean + largest single cost
        assert max(loads) <= np.mean(loads) + sequence_costs(lens).max()
    assert [len(p) for p in partition_sequences([5, 5], 4)] == [1, 1, 0, 0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import torch.distributed as dist
    import oracle
    from bench import reduce_timing
    from gen import custom_attn_inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = custom_attn_inputs([7, 30, 0, 12, 25, 3], H=2, d=8, num_pos=32, num_buckets=16,
                                 dtype="f32", seed=42)
        mine = partition_sequences(inp.lengths, world)[rank]
        tok, loc = shard_offsets(inp.seq_offsets, mine)
        # each rank computes its shard alone (the fp64 oracle stands in for the kernel here)
        part = oracle.attn(loc, inp.q[tok], inp.k[tok], inp.v[tok], inp.timestamps[tok],
                           inp.pos_bias, inp.time_bias, inp.max_seqlen)
        ms, units = reduce_timing(10.0 + rank, float(len(tok)), world)
        gathered = [None] * world
        dist.all_gather_object(gathered, (tok, part))
        results[rank] = (ms, units, gathered)
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_shards_reassemble():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        results = dict(results)
    import oracle
    from gen import custom_attn_inputs
    inp = custom_attn_inputs([7, 30, 0, 12, 25, 3], H=2, d=8, num_pos=32, num_buckets=16,
                             dtype="f32", seed=42)
    full = oracle.attn(inp.seq_offsets, inp.q, inp.k, inp.v, inp.timestamps, inp.pos_bias,
                       inp.time_bias, inp.max_seqlen)
    for rank in range(world):
        ms, units, gathered = results[rank]
        assert ms == 11.0                      # max over ranks
        assert units == float(inp.T)           # every token counted once
        out = np.full_like(full, np.nan)
        for tok, part in gathered:
            out[tok] = part
        assert np.array_equal(out, full)


if __name__ == "__main__":
    pytest.main([__file__, "-q"])
