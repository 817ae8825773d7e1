"""The seeded input generator: determinism, shapes, value structure. CPU only."""

import numpy as np
import torch

from gen import CONFIGS, make_attn_inputs, make_layer_inputs, round_to_bf16


def test_round_to_bf16_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        # exact ties between two bf16 values, both parities
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8)],
                                 dtype=np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(round_to_bf16(x), want)


def test_attn_configs_shapes_and_structure():
    for cid in (1, 2, 3, 4):
        cfg = CONFIGS[cid]
        inp = make_attn_inputs(cid)
        lens = inp.lengths
        assert inp.B == cfg["B"]
        assert inp.q.shape == (inp.T, cfg["H"], cfg["d"])
        assert inp.pos_bias.shape == (cfg["H"], cfg["num_pos"])
        assert inp.time_bias.shape == (cfg["H"], cfg["num_buckets"])
        assert inp.max_seqlen == lens.max()
        if "len_lo" in cfg:
            assert lens.min() >= cfg["len_lo"] and lens.max() <= cfg["len_hi"]
        else:
            assert lens.min() >= 1 and lens.max() <= cfg["len_beta_max"]
        for b in range(inp.B):
            t = inp.timestamps[inp.seq_offsets[b]:inp.seq_offsets[b + 1]]
            assert np.all(np.diff(t) >= 1)
        if cfg["dtype"] == "bf16":
            assert np.array_equal(round_to_bf16(inp.q), inp.q)
        assert abs(float(inp.pos_bias.std()) - 0.02) < 0.005


def test_determinism_and_seed():
    a = make_attn_inputs(2)
    b = make_attn_inputs(2)
    c = make_attn_inputs(2, seed=7)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.timestamps, b.timestamps)
    assert not np.array_equal(a.seq_offsets, c.seq_offsets)


def test_long_config_length_distribution():
    inp = make_attn_inputs(4, seed=12345)
    # Beta(2,1) has mean 2/3: 16 draws average well above 4096
    assert inp.lengths.mean() > 3000


def test_layer_inputs():
    li = make_layer_inputs(5, lengths_override=[3, 0, 5])
    assert li.x.shape == (8, 512) and li.W1.shape == (2048, 512) and li.W2.shape == (512, 512)
    assert abs(float(li.W1.std()) * np.sqrt(512) - 1.0) < 0.02
