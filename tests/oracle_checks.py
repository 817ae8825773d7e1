"""Checks that pin the fp64 oracle to things other than itself.

Each ``check_*`` takes a loaded oracle library and raises AssertionError when
the oracle disagrees with an independent statement of the same mathematics:
a library routine (numpy matmul, torch silu / layer_norm, frexp, int
bit_length), a closed form, an invariant (causality, batch independence), or a
brute-force dense evaluation written with different primitives. The same
checks run against mutated copies of the oracle (test_oracle_mutations.py)
to show that a dropped term, a wrong sign or index, or a transposed operand
is caught.

Definition being pinned (HSTU attention; operands from the benchmark spec
of the Generative Recommenders HSTU layer): for j <= i in one sequence,
s_ij = q_i.k_j + pos[h][min(i-j, P-1)] + time[h][clamp(floor(log2(max(1, t_i-t_j))), 0, NB-1)],
A_i = (1/N) sum_j silu(s_ij) v_j.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from gen import custom_attn_inputs

RTOL = 1e-12


def _close(a, b, tol=RTOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    scale = max(1.0, float(np.abs(b).max()) if b.size else 1.0)
    err = float(np.abs(a - b).max()) if a.size else 0.0
    assert err <= tol * scale, "%s: max abs err %.3e (scale %.3e)" % (what, err, scale)


def _small_gap_timestamps(rng, lengths, max_gap=40):
    """Increasing timestamps with small gaps so that buckets 0..~10 all occur."""
    ts = []
    for n in lengths:
        t = int(rng.integers(0, 1000))
        for _ in range(int(n)):
            ts.append(t)
            t += int(rng.integers(0, max_gap))
    return np.array(ts, dtype=np.int64)


def tiny_case(seed=0, lengths=(0, 1, 7, 13, 2, 20), H=2, d=5, P=8, NB=12, small_gaps=True):
    inp = custom_attn_inputs(lengths, H=H, d=d, num_pos=P, num_buckets=NB, dtype="f32",
                             seed=seed, qkv_scale=0.7, bias_std=0.5)
    if small_gaps:
        inp.timestamps = _small_gap_timestamps(np.random.default_rng(seed + 99), lengths)
    return inp


def _silu_t(x):
    return torch.nn.functional.silu(torch.from_numpy(np.asarray(x, dtype=np.float64))).numpy()


def _floor_log2_frexp(x):
    """floor(log2(x)) for integer-valued x >= 1 below 2^53, via frexp (x = m 2^e, m in [0.5,1))."""
    _, e = np.frexp(np.asarray(x, dtype=np.float64))
    return e - 1


def dense_reference(off, q, k, v, ts, pos, tb, N):
    """Per-sequence dense evaluation: full n x n score matrix with numpy matmul,
    bias matrices by fancy indexing, lower-triangular mask, torch silu, matmul."""
    T, H, _ = q.shape
    dv = v.shape[2]
    out = np.zeros((T, H, dv))
    for b in range(len(off) - 1):
        o, n = int(off[b]), int(off[b + 1] - off[b])
        if n == 0:
            continue
        I, J = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        mask = np.tril(np.ones((n, n)))
        for h in range(H):
            S = q[o:o + n, h, :].astype(np.float64) @ k[o:o + n, h, :].astype(np.float64).T
            if pos is not None:
                P = pos.shape[1]
                S = S + pos[h][np.clip(I - J, 0, P - 1)]
            if tb is not None:
                NB = tb.shape[1]
                dt = ts[o + I] - ts[o + J]
                bkt = np.clip(_floor_log2_frexp(np.maximum(dt, 1)), 0, NB - 1)
                S = S + tb[h][bkt]
            Pm = _silu_t(S) * mask
            out[o:o + n, h, :] = Pm @ v[o:o + n, h, :].astype(np.float64) / N
    return out


def padded_reference(off, q, k, v, ts, pos, tb, N):
    """Batched evaluation on a zero-padded [B, L, H, d] layout with torch einsum
    and a (causal and length) mask; results unpadded back to the jagged layout."""
    lens = np.diff(off)
    B, L = len(lens), int(max(1, lens.max()))
    T, H, dqk = q.shape
    dv = v.shape[2]
    Qp = torch.zeros(B, L, H, dqk, dtype=torch.float64)
    Kp = torch.zeros(B, L, H, dqk, dtype=torch.float64)
    Vp = torch.zeros(B, L, H, dv, dtype=torch.float64)
    Tp = torch.zeros(B, L, dtype=torch.int64)
    for b in range(B):
        o, n = int(off[b]), int(lens[b])
        Qp[b, :n] = torch.from_numpy(q[o:o + n].astype(np.float64))
        Kp[b, :n] = torch.from_numpy(k[o:o + n].astype(np.float64))
        Vp[b, :n] = torch.from_numpy(v[o:o + n].astype(np.float64))
        Tp[b, :n] = torch.from_numpy(ts[o:o + n])
    S = torch.einsum("bihd,bjhd->bhij", Qp, Kp)
    ar = torch.arange(L)
    rel = ar[:, None] - ar[None, :]
    if pos is not None:
        pt = torch.from_numpy(pos.astype(np.float64))
        S = S + pt[:, rel.clamp(0, pt.shape[1] - 1)][None]
    if tb is not None:
        tt = torch.from_numpy(tb.astype(np.float64))
        dt = (Tp[:, :, None] - Tp[:, None, :]).clamp(min=1)
        bkt = torch.from_numpy(_floor_log2_frexp(dt.numpy())).clamp(0, tt.shape[1] - 1)
        S = S + tt[:, bkt].permute(1, 0, 2, 3)
    valid = torch.from_numpy(np.arange(L)[None, :] < lens[:, None])
    mask = (rel >= 0)[None, None] & valid[:, None, :, None] & valid[:, None, None, :]
    Pm = torch.nn.functional.silu(S) * mask
    A = torch.einsum("bhij,bjhd->bihd", Pm, Vp) / N
    out = np.zeros((T, H, dv))
    for b in range(B):
        o, n = int(off[b]), int(lens[b])
        out[o:o + n] = A[b, :n].numpy()
    return out


def _run(lib, inp, **kw):
    args = dict(seq_offsets=inp.seq_offsets, q=inp.q, k=inp.k, v=inp.v,
                timestamps=inp.timestamps, pos_bias=inp.pos_bias, time_bias=inp.time_bias,
                max_seqlen=inp.max_seqlen)
    args.update(kw)
    return oracle.attn(lib=lib, **args)


# --------------------------------------------------------------------------- indices

def check_floor_log2(lib):
    xs = list(range(1, 2049)) + [2 ** e + dlt for e in range(1, 63) for dlt in (-1, 0, 1)]
    xs += [2 ** 63 - 1]
    for x in xs:
        assert oracle.floor_log2(x, lib) == x.bit_length() - 1, x


def check_time_bucket(lib):
    dts = [-(2 ** 62), -5, -1, 0, 1, 2, 3, 4, 5, 7, 8, 9, 1023, 1024, 1025, 3600, 86400,
           2 ** 31 - 1, 2 ** 31, 2 ** 32 + 7, 2 ** 53 + 1, 2 ** 62, 2 ** 63 - 1]
    for nb in (1, 2, 8, 12, 31, 32, 64, 128):
        for dt in dts:
            want = min(max(0, max(1, dt).bit_length() - 1), nb - 1)
            assert oracle.time_bucket(dt, nb, lib) == want, (dt, nb)


def check_pos_index(lib):
    for P in (1, 2, 8, 64, 200):
        for i in range(0, 70):
            for j in range(0, i + 1):
                assert oracle.pos_index(i, j, P, lib) == min(i - j, P - 1)


def check_bias_indices_array(lib):
    inp = tiny_case(seed=3)
    P, NB = inp.pos_bias.shape[1], inp.time_bias.shape[1]
    pos, bkt = oracle.bias_indices(inp.seq_offsets, inp.timestamps, P, NB, lib)
    want_p, want_b = [], []
    for b in range(inp.B):
        o, n = int(inp.seq_offsets[b]), int(inp.lengths[b])
        for i in range(n):
            for j in range(i + 1):
                want_p.append(min(i - j, P - 1))
                dt = int(inp.timestamps[o + i] - inp.timestamps[o + j])
                want_b.append(min(max(1, dt).bit_length() - 1, NB - 1))
    assert np.array_equal(pos, np.array(want_p, dtype=np.int32))
    assert np.array_equal(bkt, np.array(want_b, dtype=np.int32))


def check_silu(lib):
    xs = np.concatenate([np.linspace(-40, 40, 801), [0.0, 1e-8, -1e-8, 700.0, -700.0]])
    got = np.array([oracle.silu(x, lib) for x in xs])
    _close(got, _silu_t(xs), 1e-15, "silu")


# --------------------------------------------------------------------------- attention

def check_dense_bruteforce(lib):
    for seed in range(4):
        inp = tiny_case(seed=seed)
        got = _run(lib, inp)
        want = dense_reference(inp.seq_offsets, inp.q, inp.k, inp.v, inp.timestamps,
                               inp.pos_bias, inp.time_bias, inp.max_seqlen)
        _close(got, want, what="dense seed %d" % seed)
    # real-scale timestamps (hour gaps): buckets 10..20, no clamp
    inp = custom_attn_inputs([9, 17, 1], H=3, d=6, num_pos=64, num_buckets=128, dtype="f32",
                             seed=11, bias_std=0.5)
    _close(_run(lib, inp), dense_reference(inp.seq_offsets, inp.q, inp.k, inp.v, inp.timestamps,
                                           inp.pos_bias, inp.time_bias, inp.max_seqlen),
           what="dense hour gaps")


def check_padded_equals_jagged(lib):
    inp = tiny_case(seed=5, lengths=(4, 0, 11, 1, 19))
    got = _run(lib, inp)
    want = padded_reference(inp.seq_offsets, inp.q, inp.k, inp.v, inp.timestamps,
                            inp.pos_bias, inp.time_bias, inp.max_seqlen)
    _close(got, want, what="padded")


def check_causality(lib):
    inp = tiny_case(seed=7, lengths=(3, 16, 5))
    base = _run(lib, inp)
    o = int(inp.seq_offsets[1])
    for cut in (0, 5, 15):
        pert = tiny_case(seed=7, lengths=(3, 16, 5))
        sl = slice(o + cut + 1, o + 16)
        rng = np.random.default_rng(cut)
        pert.q[sl] += rng.standard_normal(pert.q[sl].shape).astype(np.float32)
        pert.k[sl] += rng.standard_normal(pert.k[sl].shape).astype(np.float32)
        pert.v[sl] += rng.standard_normal(pert.v[sl].shape).astype(np.float32)
        pert.timestamps[sl] += 12345
        got = _run(lib, pert)
        keep = np.r_[0:o + cut + 1, o + 16:inp.T]
        assert np.array_equal(got[keep], base[keep]), "rows <= %d changed" % cut
        if cut < 15:
            assert not np.array_equal(got[o + 15], base[o + 15]), "later rows must see the change"


def check_batch_independence(lib):
    inp = tiny_case(seed=9, lengths=(6, 0, 14, 2))
    full = _run(lib, inp)
    for b in range(inp.B):
        o, n = int(inp.seq_offsets[b]), int(inp.lengths[b])
        sl = slice(o, o + n)
        alone = oracle.attn(np.array([0, n]), inp.q[sl], inp.k[sl], inp.v[sl],
                            inp.timestamps[sl], inp.pos_bias, inp.time_bias, inp.max_seqlen,
                            lib=lib)
        assert np.array_equal(alone, full[sl]), b


def check_rows_subset(lib):
    inp = tiny_case(seed=13)
    full = _run(lib, inp)
    rows = [inp.T - 1, 0, 5, 17, 3]
    got = _run(lib, inp, rows=rows)
    assert np.array_equal(got, full[rows])


def check_empty_and_length_one(lib):
    inp = tiny_case(seed=2, lengths=(0, 1, 0, 3, 1, 0))
    got = _run(lib, inp)
    assert got.shape[0] == 5
    N = inp.max_seqlen
    for t in (0, 4):     # the two length-1 sequences
        for h in range(inp.H):
            s = float(np.dot(inp.q[t, h].astype(np.float64), inp.k[t, h].astype(np.float64)))
            s += float(inp.pos_bias[h, 0]) + float(inp.time_bias[h, 0])
            want = s / (1.0 + np.exp(-s)) * inp.v[t, h].astype(np.float64) / N
            _close(got[t, h], want, what="len1")
    # a batch of only empty sequences has no rows and must not fail
    emp = tiny_case(seed=2, lengths=(0, 0))
    assert _run(lib, emp).shape[0] == 0


def check_closed_form_prefix_sum(lib):
    """q = k = 0, constant position bias c, no time bias: A_i = silu(c)/N * cumsum(v)_i."""
    inp = tiny_case(seed=4, lengths=(9, 4))
    inp.q[:] = 0
    inp.k[:] = 0
    for c in (0.0, 0.75, -1.3):
        inp.pos_bias[:] = c
        got = _run(lib, inp, timestamps=None, time_bias=None)
        c = float(inp.pos_bias[0, 0])          # the float32 value actually stored
        sil = c / (1.0 + np.exp(-c))
        for b in range(inp.B):
            o, n = int(inp.seq_offsets[b]), int(inp.lengths[b])
            want = sil / inp.max_seqlen * np.cumsum(inp.v[o:o + n].astype(np.float64), axis=0)
            _close(got[o:o + n], want, what="prefix c=%g" % c)


def check_time_only_closed_form(lib):
    """Timestamps 2^m - 1: for j < i, t_i - t_j = 2^i - 2^j lies in [2^(i-1), 2^i), so its
    bucket is i-1; the diagonal has dt = 0 and bucket 0. With q = k = 0 and no position
    bias, A_i = (silu(tb[0]) v_i + silu(tb[i-1]) sum_{j<i} v_j) / N."""
    n, H, d, NB = 12, 2, 3, 128
    inp = custom_attn_inputs([n], H=H, d=d, num_pos=4, num_buckets=NB, dtype="f32", seed=21)
    inp.timestamps = np.array([2 ** m - 1 for m in range(n)], dtype=np.int64)
    inp.q[:] = 0
    inp.k[:] = 0
    inp.time_bias[:] = np.linspace(-2.0, 2.0, NB)[None, :] * np.array([[1.0], [-0.5]])
    got = _run(lib, inp, pos_bias=None)
    v = inp.v.astype(np.float64)
    sil = lambda x: x / (1.0 + np.exp(-x))  # noqa: E731
    for h in range(H):
        tb = inp.time_bias[h].astype(np.float64)
        for i in range(n):
            want = sil(tb[0]) * v[i, h]
            if i > 0:
                want = want + sil(tb[i - 1]) * v[:i, h].sum(axis=0)
            _close(got[i, h], want / n, what="time-only i=%d" % i)


def check_pos_only_toeplitz(lib):
    """No time bias, q = k = 0, P = 3 < n: the score matrix is the Toeplitz matrix of
    pos[h][min(r, P-1)], so A = (silu(toeplitz) * tril) v / N."""
    from scipy.linalg import toeplitz
    n, H, d, P = 7, 2, 4, 3
    inp = custom_attn_inputs([n], H=H, d=d, num_pos=P, num_buckets=4, dtype="f32", seed=8,
                             bias_std=1.0)
    inp.q[:] = 0
    inp.k[:] = 0
    got = _run(lib, inp, time_bias=None)
    for h in range(H):
        col = np.array([inp.pos_bias[h, min(r, P - 1)] for r in range(n)], dtype=np.float64)
        S = toeplitz(col, np.full(n, 123.0))      # upper triangle is masked anyway
        want = (_silu_t(S) * np.tril(np.ones((n, n)))) @ inp.v[:, h].astype(np.float64) / n
        _close(got[:, h], want, what="toeplitz h=%d" % h)


def check_scale_is_max_seqlen(lib):
    inp = tiny_case(seed=6)
    a = _run(lib, inp)
    b = _run(lib, inp, max_seqlen=2 * inp.max_seqlen)
    _close(b * 2.0, a, 1e-15, "1/N scaling")


def check_qk_asymmetry(lib):
    """A single pair with q_1.k_0 != q_0.k_1: row 1 must use q_1.k_0."""
    inp = custom_attn_inputs([2], H=1, d=2, num_pos=4, num_buckets=4, dtype="f32", seed=1)
    inp.q[:] = np.array([[[0.0, 0.0]], [[1.0, 2.0]]])
    inp.k[:] = np.array([[[3.0, -1.0]], [[0.5, 0.5]]])
    inp.v[:] = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])
    got = _run(lib, inp, timestamps=None, time_bias=None, pos_bias=None)
    sil = lambda x: x / (1.0 + np.exp(-x))  # noqa: E731
    s10, s11 = 1 * 3 + 2 * -1, 1 * 0.5 + 2 * 0.5
    want1 = np.array([sil(s10), sil(s11)]) / 2
    want0 = np.array([sil(0.0), 0.0]) / 2
    _close(got[1, 0], want1, what="row1")
    _close(got[0, 0], want0, what="row0")


# --------------------------------------------------------------------------- layer pieces

def check_linear(lib):
    rng = np.random.default_rng(0)
    x = rng.standard_normal((9, 7))
    W = rng.standard_normal((5, 7))
    b = rng.standard_normal(5)
    r = rng.standard_normal((9, 5))
    _close(oracle.linear(x, W, lib=lib), x @ W.T, what="linear")
    _close(oracle.linear(x, W, b, act_silu=True, lib=lib), _silu_t(x @ W.T + b), what="silu lin")
    _close(oracle.linear(x, W, None, False, r, lib=lib), x @ W.T + r, what="residual")


def check_layernorm_gate(lib):
    rng = np.random.default_rng(1)
    a = rng.standard_normal((6, 16)) * 3 + 1
    u = rng.standard_normal((6, 16))
    g = rng.standard_normal(16)
    bt = rng.standard_normal(16)
    ln = torch.nn.functional.layer_norm(torch.from_numpy(a), (16,), torch.from_numpy(g),
                                        torch.from_numpy(bt), eps=1e-5).numpy()
    _close(oracle.layernorm_gate(a, u, g, bt, 1e-5, lib=lib), ln * u, what="ln gate")
    # identity affine, u = 1: normalised rows have mean 0 and (biased) variance v/(v+eps)
    y = oracle.layernorm_gate(a, np.ones_like(a), eps=1e-5, lib=lib)
    var = a.var(axis=1)
    _close(y.mean(axis=1), np.zeros(6), what="ln mean")
    _close(y.var(axis=1), var / (var + 1e-5), what="ln var")
    # tiny rows: eps dominates (variance << eps), output ~ (a - mean)/sqrt(eps)
    small = a * 1e-4
    want = (small - small.mean(1, keepdims=True)) / np.sqrt(small.var(1, keepdims=True) + 1e-5)
    _close(oracle.layernorm_gate(small, np.ones_like(a), eps=1e-5, lib=lib), want, what="ln eps")


def _tiny_layer(seed=0, lengths=(5, 0, 9, 1), D=12, H=2, d=4):
    rng = np.random.default_rng(seed)
    T = int(sum(lengths))
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    x = rng.standard_normal((T, D))
    W1 = rng.standard_normal((4 * H * d, D)) / np.sqrt(D)
    W2 = rng.standard_normal((D, H * d)) / np.sqrt(H * d)
    ts = _small_gap_timestamps(rng, lengths)
    pos = rng.standard_normal((H, 6)) * 0.3
    tb = rng.standard_normal((H, 10)) * 0.3
    return off, x, W1, W2, H, d, ts, pos, tb, int(max(lengths))


def check_layer_composition(lib):
    off, x, W1, W2, H, d, ts, pos, tb, N = _tiny_layer()
    T = x.shape[0]
    F = H * d
    rng = np.random.default_rng(5)
    b1, b2 = rng.standard_normal(4 * F) * 0.1, rng.standard_normal(x.shape[1]) * 0.1
    g, bt = 1 + rng.standard_normal(F) * 0.1, rng.standard_normal(F) * 0.1
    got = oracle.layer(off, x, W1, W2, H, d, ts, pos, tb, N, b1=b1, b2=b2, ln_gamma=g,
                       ln_beta=bt, ln_eps=1e-5, lib=lib)
    uvqk = _silu_t(x @ W1.T + b1)
    U, V, Q, K = (uvqk[:, i * F:(i + 1) * F].reshape(T, H, d) for i in range(4))
    A = dense_reference(off, Q, K, V, ts, pos, tb, N).reshape(T, F)
    Y = torch.nn.functional.layer_norm(torch.from_numpy(A), (F,), torch.from_numpy(g),
                                       torch.from_numpy(bt), eps=1e-5).numpy() * U.reshape(T, F)
    _close(got, x + Y @ W2.T + b2, what="layer")
    rows = [T - 1, 2, 7]
    _close(oracle.layer(off, x, W1, W2, H, d, ts, pos, tb, N, b1=b1, b2=b2, ln_gamma=g,
                        ln_beta=bt, rows=rows, lib=lib), got[rows], 0, "layer rows")


def check_layernorm(lib):
    """The input LayerNorm against torch.layer_norm (a library routine), with
    and without the affine parameters."""
    rng = np.random.default_rng(11)
    a = rng.standard_normal((7, 24)) * 2.5 - 0.7
    g = 1 + rng.standard_normal(24) * 0.2
    bt = rng.standard_normal(24) * 0.2
    t = torch.from_numpy(a)
    _close(oracle.layernorm(a, g, bt, 1e-5, lib=lib),
           torch.nn.functional.layer_norm(t, (24,), torch.from_numpy(g), torch.from_numpy(bt),
                                          eps=1e-5).numpy(), what="layernorm affine")
    _close(oracle.layernorm(a, eps=1e-3, lib=lib),
           torch.nn.functional.layer_norm(t, (24,), eps=1e-3).numpy(), what="layernorm")


def check_layer_input_norm(lib):
    """The layer with an input LayerNorm: the projection reads LayerNorm(x),
    the residual adds x itself (torch composition with the dense reference)."""
    off, x, W1, W2, H, d, ts, pos, tb, N = _tiny_layer(seed=4)
    T, D = x.shape
    F = H * d
    rng = np.random.default_rng(6)
    ig, ib = 1 + rng.standard_normal(D) * 0.2, rng.standard_normal(D) * 0.2
    got = oracle.layer(off, x, W1, W2, H, d, ts, pos, tb, N, ln_eps=1e-5, lib=lib,
                       input_norm=True, in_gamma=ig, in_beta=ib)
    xn = torch.nn.functional.layer_norm(torch.from_numpy(x), (D,), torch.from_numpy(ig),
                                        torch.from_numpy(ib), eps=1e-5).numpy()
    uvqk = _silu_t(xn @ W1.T)
    U, V, Q, K = (uvqk[:, i * F:(i + 1) * F].reshape(T, H, d) for i in range(4))
    A = dense_reference(off, Q, K, V, ts, pos, tb, N).reshape(T, F)
    Y = torch.nn.functional.layer_norm(torch.from_numpy(A), (F,), eps=1e-5).numpy() * U.reshape(T, F)
    _close(got, x + Y @ W2.T, what="layer with input norm")
    rows = [T - 1, 0, 6]
    _close(oracle.layer(off, x, W1, W2, H, d, ts, pos, tb, N, ln_eps=1e-5, rows=rows, lib=lib,
                        input_norm=True, in_gamma=ig, in_beta=ib), got[rows], 0,
           "layer with input norm, rows")


def check_layer_identities(lib):
    off, x, W1, W2, H, d, ts, pos, tb, N = _tiny_layer(seed=3)
    F = H * d
    out = oracle.layer(off, x, W1, np.zeros_like(W2), H, d, ts, pos, tb, N, lib=lib)
    assert np.array_equal(out, x), "W2 = 0 must give out = x"
    W1u0 = W1.copy()
    W1u0[:F] = 0                      # U = silu(0) = 0
    out = oracle.layer(off, x, W1u0, W2, H, d, ts, pos, tb, N, lib=lib)
    _close(out, x, 0.0, "U = 0 must give out = x")


# --------------------------------------------------------------------------- backward

def check_silu_grad(lib):
    """silu'(s) against torch autograd of torch's SiLU (a library routine)."""
    xs = np.array([-30.0, -5.0, -1.3, -1e-3, 0.0, 2e-4, 0.7, 3.0, 12.0, 40.0])
    t = torch.from_numpy(xs).requires_grad_(True)
    torch.nn.functional.silu(t).sum().backward()
    got = np.array([lib.hstu_oracle_silu_grad(float(x)) for x in xs])
    _close(got, t.grad.numpy(), what="silu'")


def _loss(lib, inp, dout, **kw):
    return float(np.sum(_run(lib, inp, **kw) * dout))


def check_attn_bwd_finite_differences(lib):
    """Every gradient against central differences of <dout, attn(...)> in fp64
    on a tiny ragged batch: sampled entries of q, k, v, every entry of the
    position and time tables."""
    inp = tiny_case(seed=3, lengths=(0, 1, 6, 11, 3), H=2, d=4, P=6, NB=9)
    rng = np.random.default_rng(5)
    dout = rng.standard_normal(inp.v.shape)
    dq, dk, dv, dpos, dtime = oracle.attn_bwd(inp.seq_offsets, inp.q, inp.k, inp.v,
                                              inp.timestamps, inp.pos_bias, inp.time_bias,
                                              inp.max_seqlen, dout, lib=lib)
    eps = 1e-6
    base = dict(q=inp.q.astype(np.float64), k=inp.k.astype(np.float64),
                v=inp.v.astype(np.float64), pos_bias=inp.pos_bias.astype(np.float64),
                time_bias=inp.time_bias.astype(np.float64))
    grads = dict(q=dq, k=dk, v=dv, pos_bias=dpos, time_bias=dtime)
    for name, arr in base.items():
        idx = [tuple(int(rng.integers(0, n)) for n in arr.shape) for _ in range(12)]
        if name in ("pos_bias", "time_bias"):
            idx = list(np.ndindex(*arr.shape))
        for ix in idx:
            plus, minus = arr.copy(), arr.copy()
            plus[ix] += eps
            minus[ix] -= eps
            fd = (_loss(lib, inp, dout, **{name: plus}) - _loss(lib, inp, dout, **{name: minus})) \
                / (2 * eps)
            g = grads[name][ix]
            assert abs(fd - g) <= 1e-6 * max(1.0, abs(fd)), "%s%s: fd %.9g grad %.9g" % (
                name, ix, fd, g)


def check_attn_bwd_against_torch_autograd(lib):
    """The oracle's gradients against torch autograd of a dense, per-sequence
    torch formulation of the forward (matmul scores, gathered bias matrices,
    lower-triangular mask, torch SiLU), written independently of the oracle."""
    inp = tiny_case(seed=6, lengths=(4, 0, 9, 1, 12), H=2, d=3, P=5, NB=7)
    rng = np.random.default_rng(13)
    dout = rng.standard_normal(inp.v.shape)
    tq = torch.tensor(inp.q, dtype=torch.float64, requires_grad=True)
    tk = torch.tensor(inp.k, dtype=torch.float64, requires_grad=True)
    tv = torch.tensor(inp.v, dtype=torch.float64, requires_grad=True)
    tpos = torch.tensor(inp.pos_bias, dtype=torch.float64, requires_grad=True)
    ttb = torch.tensor(inp.time_bias, dtype=torch.float64, requires_grad=True)
    off, ts, N = inp.seq_offsets, inp.timestamps, inp.max_seqlen
    P, NB = inp.pos_bias.shape[1], inp.time_bias.shape[1]
    loss = torch.zeros((), dtype=torch.float64)
    for b in range(len(off) - 1):
        o, n = int(off[b]), int(off[b + 1] - off[b])
        if n == 0:
            continue
        I, J = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
        pidx = torch.from_numpy(np.clip(I - J, 0, P - 1))
        dt = ts[o + I] - ts[o + J]
        bidx = torch.from_numpy(np.clip(_floor_log2_frexp(np.maximum(dt, 1)), 0, NB - 1))
        mask = torch.tril(torch.ones((n, n), dtype=torch.float64))
        for h in range(inp.H):
            S = tq[o:o + n, h] @ tk[o:o + n, h].T + tpos[h][pidx] + ttb[h][bidx]
            out = (torch.nn.functional.silu(S) * mask) @ tv[o:o + n, h] / N
            loss = loss + (out * torch.from_numpy(dout[o:o + n, h])).sum()
    loss.backward()
    got = oracle.attn_bwd(off, inp.q, inp.k, inp.v, ts, inp.pos_bias, inp.time_bias, N, dout,
                          lib=lib)
    for name, g, t in zip(("dq", "dk", "dv", "dpos", "dtime"), got,
                          (tq, tk, tv, tpos, ttb)):
        _close(g, t.grad.numpy(), what="autograd " + name)


def check_attn_bwd_closed_form(lib):
    """q = k = 0 and constant biases c: every score is c, so dv[j] = silu(c)/N
    times the suffix sum of dout over the rows i >= j of j's sequence, and the
    position- and time-table gradients each sum to sum_{i>=j} (dout_i . v_j)
    silu'(c) / N."""
    inp = tiny_case(seed=4, lengths=(5, 0, 8, 1), H=1, d=3, P=4, NB=6)
    c = 0.4
    q0 = np.zeros_like(inp.q, dtype=np.float64)
    pos = np.full_like(inp.pos_bias, c / 2, dtype=np.float64)
    tb = np.full_like(inp.time_bias, c / 2, dtype=np.float64)
    rng = np.random.default_rng(8)
    dout = rng.standard_normal(inp.v.shape)
    v = inp.v.astype(np.float64)
    N = inp.max_seqlen
    _, _, dv, dpos, dtime = oracle.attn_bwd(inp.seq_offsets, q0, q0, v, inp.timestamps, pos, tb,
                                            N, dout, lib=lib)
    sil = c / (1 + np.exp(-c))
    sg = 1 / (1 + np.exp(-c))
    dsil = sg * (1 + c * (1 - sg))
    want_dv = np.zeros_like(v)
    total = 0.0
    off = inp.seq_offsets
    for b in range(len(off) - 1):
        for j in range(off[b], off[b + 1]):
            want_dv[j] = sil / N * dout[j:off[b + 1]].sum(axis=0)
            for i in range(j, off[b + 1]):
                total += float(np.sum(dout[i] * v[j])) * dsil / N
    _close(dv, want_dv, what="dv suffix sums")
    _close(dpos.sum(), total, what="sum dpos")
    _close(dtime.sum(), total, what="sum dtime")


# --------------------------------------------------------------------------- FP8 (E4M3)

def _e4m3_grid():
    """Every finite non-negative E4M3 value from the format's definition:
    subnormals m/8 * 2^-6, normals (1 + m/8) * 2^(e - 7), e = 1..15, without
    the NaN pattern e = 15, m = 7."""
    vals = [m / 8.0 * 2.0 ** -6 for m in range(8)]
    vals += [(1 + m / 8.0) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8)
             if not (e == 15 and m == 7)]
    return np.array(vals)


def check_e4m3_table(lib):
    """Decoding every code gives the format's value grid (by construction here),
    NaN for the two all-ones patterns, and encoding a decoded value gives the
    code back."""
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_to_float(codes, lib=lib).astype(np.float64)
    assert np.isnan(vals[0x7F]) and np.isnan(vals[0xFF])
    pos = np.delete(vals[:128], 0x7F)
    assert np.array_equal(pos, _e4m3_grid()), "positive codes 0..126"
    assert np.array_equal(np.delete(vals[128:], 0x7F), -_e4m3_grid()), "negative codes"
    assert vals[0x7E] == 448.0 and vals[1] == 2.0 ** -9
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    back = oracle.e4m3_from_float(oracle.e4m3_to_float(finite, lib=lib), lib=lib)
    assert np.array_equal(back, finite), "round trip"


def check_e4m3_rounding_against_torch(lib):
    """Encoding agrees with torch's float8_e4m3fn cast (round to nearest, ties
    to even) on every grid value, every midpoint between neighbours, points
    just off the midpoints, and random values, of both signs, below the
    saturation threshold."""
    import torch
    g = _e4m3_grid()
    mids = (g[:-1] + g[1:]) / 2
    off = np.concatenate([mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20)])
    rng = np.random.default_rng(7)
    rnd = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(440.0), 4000))
    x = np.concatenate([g, mids, off, rnd, [2.0 ** -11, 3 * 2.0 ** -11, 1e-30]]).astype(np.float32)
    x = np.concatenate([x, -x])
    got = oracle.e4m3_from_float(x, lib=lib)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, "codes differ from torch at %s" % x[bad[:5]]


def check_e4m3_saturation(lib):
    """Finite overflow and infinity saturate to +-448 (code 0x7E / 0xFE); NaN
    stays NaN."""
    x = np.array([448.0, 449.0, 464.0, 480.0, 1e6, np.inf, -500.0, -np.inf], dtype=np.float32)
    got = oracle.e4m3_from_float(x, lib=lib)
    assert list(got) == [0x7E] * 6 + [0xFE] * 2
    assert oracle.e4m3_from_float(np.array([np.nan], np.float32), lib=lib)[0] == 0x7F


def check_quant_rows(lib):
    """Row-wise quantization: the row's largest magnitude maps to 448 exactly;
    scaling a row by a power of two leaves its codes alone and scales its
    scale; an all-zero row gives zero codes and scale 1; the dequantized
    values are within half a step of the E4M3 grid (relative 2^-4 in the
    normal range, 2^-10 * scale below it)."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((6, 40)) * np.array([1, 10, 1e-3, 300, 2.0 ** 20, 1])[:, None]).astype(np.float32)
    x[5] = 0.0
    codes, scales = oracle.quant_rows_e4m3(x, lib=lib)
    amax = np.abs(x).max(axis=1)
    for r in range(5):
        i = int(np.argmax(np.abs(x[r])))
        assert codes[r, i] & 0x7F == 0x7E, "row %d amax code" % r
        assert scales[r] == np.float32(amax[r] / np.float32(448.0))
    assert np.all(codes[5] & 0x7F == 0) and scales[5] == 1.0
    c2, s2 = oracle.quant_rows_e4m3(x * np.float32(8.0), lib=lib)
    assert np.array_equal(c2, codes) and np.array_equal(s2[:5], scales[:5] * 8)
    deq = oracle.e4m3_to_float(codes, lib=lib).astype(np.float64) * scales[:, None]
    err = np.abs(deq - x)
    normal = np.abs(x) >= (2.0 ** -6) * scales[:, None] * 1.0001
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(x[normal]) * (1 + 1e-6)), "normal range"
    assert np.all(err[~normal] <= 2.0 ** -10 * np.broadcast_to(scales[:, None], x.shape)[~normal]
                  * (1 + 1e-6)), "subnormal range"
    # rows too small for a finite 448 / amax in fp32 (amax < 448 / FLT_MAX):
    # never NaN codes, and the dequantized row is within that bound of x
    fmax = float(np.finfo(np.float32).max)
    tiny = np.array([[1e-37, -3e-38, 0.0, 2e-37], [1.2e-38, 0.0, -1.2e-38, 5e-37]], np.float32)
    tc, ts_ = oracle.quant_rows_e4m3(tiny, lib=lib)
    assert not np.any((tc & 0x7F) == 0x7F), "NaN codes for a tiny row"
    tdeq = oracle.e4m3_to_float(tc, lib=lib).astype(np.float64) * ts_[:, None]
    assert np.all(np.isfinite(tdeq)) and np.all(np.abs(tdeq - tiny) <= 448.0 / fmax), "tiny rows"


def check_linear_fp8(lib):
    """FP8 addmm equals the fp64 product of the dequantized operands (numpy),
    with bias, SiLU and residual as in the plain linear."""
    rng = np.random.default_rng(4)
    x = rng.standard_normal((9, 32)).astype(np.float32)
    W = rng.standard_normal((5, 32)).astype(np.float32)
    xq, sx = oracle.quant_rows_e4m3(x, lib=lib)
    wq, sw = oracle.quant_rows_e4m3(W, lib=lib)
    xd = oracle.e4m3_to_float(xq, lib=lib).astype(np.float64) * sx[:, None]
    wd = oracle.e4m3_to_float(wq, lib=lib).astype(np.float64) * sw[:, None]
    b = rng.standard_normal(5)
    r = rng.standard_normal((9, 5))
    _close(oracle.linear_fp8(xq, sx, wq, sw, lib=lib), xd @ wd.T, what="fp8 linear")
    _close(oracle.linear_fp8(xq, sx, wq, sw, b, True, lib=lib), _silu_t(xd @ wd.T + b),
           what="fp8 silu")
    _close(oracle.linear_fp8(xq, sx, wq, sw, None, False, r, lib=lib), xd @ wd.T + r,
           what="fp8 residual")
    # and it approximates the unquantized product
    assert np.linalg.norm(xd @ wd.T - x.astype(np.float64) @ W.T.astype(np.float64)) < \
        0.1 * np.linalg.norm(x.astype(np.float64) @ W.T.astype(np.float64))


ALL_CHECKS = [
    check_floor_log2, check_time_bucket, check_pos_index, check_bias_indices_array, check_silu,
    check_dense_bruteforce, check_padded_equals_jagged, check_causality,
    check_batch_independence, check_rows_subset, check_empty_and_length_one,
    check_closed_form_prefix_sum, check_time_only_closed_form, check_pos_only_toeplitz,
    check_scale_is_max_seqlen, check_qk_asymmetry, check_linear, check_layernorm_gate,
    check_layer_composition, check_layer_identities, check_layernorm, check_layer_input_norm,
    check_e4m3_table,
    check_e4m3_rounding_against_torch, check_e4m3_saturation, check_quant_rows, check_linear_fp8,
    check_silu_grad, check_attn_bwd_finite_differences, check_attn_bwd_closed_form,
    check_attn_bwd_against_torch_autograd,
]
