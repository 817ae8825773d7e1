"""Helpers for GPU parity tests: move generator inputs to the device, compare
with the oracle, pick sampled rows for full-size checks."""

from __future__ import annotations

import numpy as np
import torch

# Tolerances of the target statement: bf16 path vs the fp64 oracle, fp32 path.
BF16_REL_FROB = 1e-2
BF16_MAX_ABS = 3e-2
F32_REL_FROB = 1e-4


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def attn_tensors(inp):
    """Device tensors of an AttnInputs (q/k/v in the workload's dtype)."""
    dt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    return dict(q=dev(inp.q, dt), k=dev(inp.k, dt), v=dev(inp.v, dt),
                seq_offsets=dev(inp.seq_offsets), timestamps=dev(inp.timestamps),
                pos_bias=dev(inp.pos_bias), time_bias=dev(inp.time_bias),
                max_seqlen=inp.max_seqlen)


def errors(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    if got.size == 0:
        return 0.0, 0.0
    diff = got - want
    denom = np.linalg.norm(want)
    rel = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    return rel, float(np.abs(diff).max())


def assert_bf16_close(got, want, what="", strict_abs=False):
    """bf16 bar: relative Frobenius error <= 1e-2 and max abs error <= 3e-2.
    The absolute bar presumes outputs of magnitude <= 1, which the workloads
    have (the 1/N scale); bf16 rounds P and the output to 2^-9 relative, so for
    edge cases at other scales (strict_abs=False) it is applied relative to the
    largest |output|."""
    rel, mx = errors(got, want)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), what + ": non-finite output"
    want_a = np.asarray(want, dtype=np.float64)
    scale = 1.0 if strict_abs or want_a.size == 0 else max(1.0, float(np.abs(want_a).max()))
    bound = BF16_MAX_ABS * scale
    assert rel <= BF16_REL_FROB and mx <= bound, \
        "%s: rel-Frobenius %.3e (<= %.0e), max-abs %.3e (<= %.3e)" % (
            what, rel, BF16_REL_FROB, mx, bound)
    return rel, mx


def assert_f32_close(got, want, what=""):
    rel, mx = errors(got, want)
    assert rel <= F32_REL_FROB, "%s: rel-Frobenius %.3e (<= %.0e)" % (what, rel, F32_REL_FROB)
    return rel, mx


def sampled_rows(seq_offsets, n_random=192, seed=0):
    """Rows for full-size checks: first/last rows of sequences, rows around every
    128-row tile boundary of the longest sequences, and random rows."""
    off = np.asarray(seq_offsets, dtype=np.int64)
    T = int(off[-1])
    rng = np.random.default_rng(seed)
    rows = set(rng.integers(0, T, size=n_random).tolist())
    lens = np.diff(off)
    for b in np.argsort(-lens)[:3]:
        o, n = int(off[b]), int(lens[b])
        for t in range(0, n, 128 * max(1, n // (128 * 8))):
            for dlt in (-1, 0, 1, 127):
                if 0 <= t + dlt < n:
                    rows.add(o + t + dlt)
        rows.update([o, o + n - 1])
    for b in range(0, len(lens), max(1, len(lens) // 16)):
        if lens[b] > 0:
            rows.update([int(off[b]), int(off[b + 1]) - 1])
    return np.array(sorted(r for r in rows if 0 <= r < T), dtype=np.int64)
