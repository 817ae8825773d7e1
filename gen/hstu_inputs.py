"""Seeded synthetic jagged batches shaped like the HSTU workloads.

The five workloads mirror the shapes the Generative Recommenders pages talk
about: a tiny fp32 case, an ML-1M-like short-history batch (sequences up to
200 actions, cf. the ``exps/ml-1m-l200`` log folder in the README's
"Verify results" step), a very short and wide memory-bound batch, the
8192-length regime of the paper's efficiency claim (abstract: "5.3x to 15.2x
faster than FlashAttention2-based Transformers on 8192 length sequences"),
and a full HSTU layer (README, "HSTU Ultra attention benchmark": UVQK
projection, attention, output normalization and projection, residual).
No public dataset is used; every value is drawn here from a seeded numpy
generator in a fixed order:

    1. sequence lengths
    2. timestamps (per-sequence start, then exponential gaps)
    3. q, k, v  (or x, W1, W2 for the layer)
    4. relative-position bias table
    5. time-bucket bias table

bf16 workloads are rounded to bf16 (round-to-nearest-even) on the host, so
the oracle and the GPU see exactly the same input values.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

T0_BASE = 1_700_000_000      # seconds; start of the first action of a sequence
T0_SPREAD = 31_500_000.0     # per-sequence start drawn uniformly in [0, ~1 year)
GAP_MEAN_S = 3600.0          # exponential inter-action gap, mean one hour
BIAS_STD = 0.02              # N(0, 0.02^2) bias tables


# name -> description; sizes follow the five workloads of the target statement.
CONFIGS = {
    1: dict(name="tiny_fp32", kind="attn", dtype="f32", B=4, len_lo=1, len_hi=64,
            H=2, d=32, num_pos=64, num_buckets=128),
    2: dict(name="short_history_b128_l20-200_h2_d64", kind="attn", dtype="bf16", B=128,
            len_lo=20, len_hi=200, H=2, d=64, num_pos=200, num_buckets=128),
    3: dict(name="very_short_wide_b2048_l5-50_h4_d64", kind="attn", dtype="bf16", B=2048,
            len_lo=5, len_hi=50, H=4, d=64, num_pos=200, num_buckets=128),
    4: dict(name="long_b16_beta21_max8192_h4_d128", kind="attn", dtype="bf16", B=16,
            len_beta_max=8192, H=4, d=128, num_pos=8192, num_buckets=128),
    5: dict(name="layer_b32_l256-4096_D512_h4_d128", kind="layer", dtype="bf16", B=32,
            len_lo=256, len_hi=4096, D=512, H=4, d=128, num_pos=8192, num_buckets=128),
}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    # NaN/Inf cannot occur for these generators; keep them untouched anyway.
    special = (bits & 0x7F800000) == 0x7F800000
    rounded = np.where(special, bits, rounded)
    return rounded.astype(np.uint32).view(np.float32).reshape(a.shape)


@dataclasses.dataclass
class AttnInputs:
    name: str
    dtype: str                  # "f32" or "bf16": the arithmetic type of the path
    seq_offsets: np.ndarray     # int64 [B+1]
    timestamps: np.ndarray      # int64 [T]
    q: np.ndarray               # float32 [T, H, d] (bf16-exact values when dtype == "bf16")
    k: np.ndarray
    v: np.ndarray
    pos_bias: np.ndarray        # float32 [H, num_pos]
    time_bias: np.ndarray       # float32 [H, num_buckets]
    max_seqlen: int
    seed: int

    @property
    def B(self) -> int:
        return int(self.seq_offsets.shape[0] - 1)

    @property
    def T(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def H(self) -> int:
        return int(self.q.shape[1])

    @property
    def d(self) -> int:
        return int(self.q.shape[2])

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.seq_offsets)


@dataclasses.dataclass
class LayerInputs:
    name: str
    seq_offsets: np.ndarray     # int64 [B+1]
    timestamps: np.ndarray      # int64 [T]
    x: np.ndarray               # float32 [T, D], bf16-exact
    W1: np.ndarray              # float32 [4*H*d, D], bf16-exact; rows ordered U|V|Q|K
    W2: np.ndarray              # float32 [D, H*d], bf16-exact
    b1: Optional[np.ndarray]    # None (the workload specifies weights only)
    b2: Optional[np.ndarray]
    ln_gamma: Optional[np.ndarray]   # None = identity affine
    ln_beta: Optional[np.ndarray]
    ln_eps: float
    pos_bias: np.ndarray        # float32 [H, num_pos]
    time_bias: np.ndarray       # float32 [H, num_buckets]
    H: int
    d: int
    max_seqlen: int
    seed: int

    @property
    def B(self) -> int:
        return int(self.seq_offsets.shape[0] - 1)

    @property
    def T(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def D(self) -> int:
        return int(self.x.shape[1])


def _lengths(rng: np.random.Generator, cfg: dict) -> np.ndarray:
    B = cfg["B"]
    if "len_beta_max" in cfg:
        m = cfg["len_beta_max"]
        lens = np.floor(m * rng.beta(2.0, 1.0, size=B)).astype(np.int64)
        return np.maximum(lens, 1)
    return rng.integers(cfg["len_lo"], cfg["len_hi"] + 1, size=B).astype(np.int64)


def _timestamps(rng: np.random.Generator, lengths: np.ndarray) -> np.ndarray:
    """Strictly increasing int64 seconds inside each sequence."""
    B = lengths.shape[0]
    T = int(lengths.sum())
    t0 = T0_BASE + np.floor(rng.uniform(0.0, T0_SPREAD, size=B)).astype(np.int64)
    gaps = np.maximum(1, np.rint(rng.exponential(GAP_MEAN_S, size=T))).astype(np.int64)
    ts = np.empty(T, dtype=np.int64)
    off = 0
    for b in range(B):
        n = int(lengths[b])
        if n:
            g = gaps[off:off + n].copy()
            g[0] = 0
            ts[off:off + n] = t0[b] + np.cumsum(g)
        off += n
    return ts


def _offsets(lengths: np.ndarray) -> np.ndarray:
    off = np.zeros(lengths.shape[0] + 1, dtype=np.int64)
    np.cumsum(lengths, out=off[1:])
    return off


def _maybe_bf16(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    return round_to_bf16(a) if dtype == "bf16" else a


def make_attn_inputs(cfg_id: int, seed: Optional[int] = None,
                     max_batch: Optional[int] = None) -> AttnInputs:
    """Draw one attention workload. ``max_batch`` keeps only the first sequences."""
    cfg = CONFIGS[cfg_id]
    assert cfg["kind"] == "attn"
    seed = 1000 + cfg_id if seed is None else seed
    rng = np.random.default_rng(seed)
    lengths = _lengths(rng, cfg)
    ts = _timestamps(rng, lengths)
    T, H, d = int(lengths.sum()), cfg["H"], cfg["d"]
    q = rng.standard_normal((T, H, d), dtype=np.float32)
    k = rng.standard_normal((T, H, d), dtype=np.float32)
    v = rng.standard_normal((T, H, d), dtype=np.float32)
    pos = (BIAS_STD * rng.standard_normal((H, cfg["num_pos"]))).astype(np.float32)
    tb = (BIAS_STD * rng.standard_normal((H, cfg["num_buckets"]))).astype(np.float32)
    inp = AttnInputs(cfg["name"], cfg["dtype"], _offsets(lengths), ts,
                     _maybe_bf16(q, cfg["dtype"]), _maybe_bf16(k, cfg["dtype"]),
                     _maybe_bf16(v, cfg["dtype"]), pos, tb,
                     int(max(1, lengths.max())), seed)
    if max_batch is not None and max_batch < inp.B:
        inp = take_sequences(inp, list(range(max_batch)))
    return inp


def take_sequences(inp: AttnInputs, seqs) -> AttnInputs:
    """A new batch made of the listed sequences of ``inp`` (same tables, same N)."""
    lens = inp.lengths
    parts = [np.arange(inp.seq_offsets[s], inp.seq_offsets[s + 1]) for s in seqs]
    idx = np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)
    new_off = _offsets(np.array([lens[s] for s in seqs], dtype=np.int64))
    return dataclasses.replace(
        inp, seq_offsets=new_off, timestamps=inp.timestamps[idx].copy(),
        q=inp.q[idx].copy(), k=inp.k[idx].copy(), v=inp.v[idx].copy())


def custom_attn_inputs(lengths, H: int, d: int, num_pos: int, num_buckets: int,
                       dtype: str = "bf16", seed: int = 0, max_seqlen: Optional[int] = None,
                       qkv_scale: float = 1.0, bias_std: float = BIAS_STD) -> AttnInputs:
    """Same generators as the workloads, with caller-chosen lengths (zeros allowed)."""
    rng = np.random.default_rng(seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    ts = _timestamps(rng, lengths)
    T = int(lengths.sum())
    q = qkv_scale * rng.standard_normal((T, H, d), dtype=np.float32)
    k = qkv_scale * rng.standard_normal((T, H, d), dtype=np.float32)
    v = rng.standard_normal((T, H, d), dtype=np.float32)
    pos = (bias_std * rng.standard_normal((H, num_pos))).astype(np.float32)
    tb = (bias_std * rng.standard_normal((H, num_buckets))).astype(np.float32)
    n = int(max(1, lengths.max() if lengths.size else 1)) if max_seqlen is None else max_seqlen
    return AttnInputs("custom", dtype, _offsets(lengths), ts, _maybe_bf16(q, dtype),
                      _maybe_bf16(k, dtype), _maybe_bf16(v, dtype), pos, tb, n, seed)


def make_layer_inputs(cfg_id: int = 5, seed: Optional[int] = None,
                      lengths_override=None) -> LayerInputs:
    cfg = CONFIGS[cfg_id]
    assert cfg["kind"] == "layer"
    seed = 1000 + cfg_id if seed is None else seed
    rng = np.random.default_rng(seed)
    lengths = _lengths(rng, cfg)
    if lengths_override is not None:
        lengths = np.asarray(lengths_override, dtype=np.int64)
    ts = _timestamps(rng, lengths)
    T, D, H, d = int(lengths.sum()), cfg["D"], cfg["H"], cfg["d"]
    x = rng.standard_normal((T, D), dtype=np.float32)
    # weights ~ N(0, std = 1/sqrt(fan_in))
    W1 = rng.standard_normal((4 * H * d, D), dtype=np.float32) / np.sqrt(D)
    W2 = rng.standard_normal((D, H * d), dtype=np.float32) / np.sqrt(H * d)
    pos = (BIAS_STD * rng.standard_normal((H, cfg["num_pos"]))).astype(np.float32)
    tb = (BIAS_STD * rng.standard_normal((H, cfg["num_buckets"]))).astype(np.float32)
    return LayerInputs(cfg["name"], _offsets(lengths), ts, round_to_bf16(x),
                       round_to_bf16(W1), round_to_bf16(W2), None, None, None, None, 1e-5,
                       pos, tb, H, d, int(max(1, lengths.max())), seed)


def make_inputs(cfg_id: int, seed: Optional[int] = None):
    if CONFIGS[cfg_id]["kind"] == "layer":
        return make_layer_inputs(cfg_id, seed)
    return make_attn_inputs(cfg_id, seed)
