#!/usr/bin/env python
"""Benchmark of the HSTU jagged causal attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4] [--impl ours|reference]

One step is one full pass of the hot path over one seeded synthetic batch:
the work-list plan kernel plus the attention kernel (for --config 5, the
whole HSTU layer: UVQK projection, plan, attention, LayerNorm gate, output
projection). Inputs are resident in HBM before the timed region; the timed
region is bracketed by a barrier and a device synchronisation on both sides
and measured with CUDA events on the launching stream (max over ranks).

Default workload: the 8192-length regime (16 sequences, lengths 8192*Beta(2,1),
4 heads, d = 128), whose inputs (~0.3 GB) exceed the 126 MB L2, so no flush is
needed between steps. Short workloads (--config 2/3) rotate over enough input
copies to exceed 2x L2.

For N > 1 (torchrun), every rank runs its own independently seeded batch of the
same shape (weak scaling); there is no collective in the data path, only the
timing reductions. Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only reference this project
has) on the host cores, on a bounded sample of the same workload per step.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "HSTU jagged attn fwd TFLOP/s (causal) & % of B200 BF16 peak; tokens/s"
L2_BYTES = 126 * 2 ** 20
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_DIR = os.path.join(ROOT, "profiles")
ATTN_SRC = os.path.join(ROOT, "jagged_pointwise_attention_b200", "csrc", "attn_tc.cuh")


# ----------------------------------------------------------------------------- accounting

def causal_flops(lengths, H, dqk, dv) -> int:
    """sum_b H (dqk + dv) n_b (n_b + 1): QK^T and PV over the causal lower
    triangle including the diagonal, 2 flops per multiply-add."""
    n = np.asarray(lengths, dtype=np.int64)
    return int((H * (dqk + dv) * n * (n + 1)).sum())


def row_causal_flops(pos_in_seq, H, dqk, dv) -> int:
    """Causal flops of individual query rows (0-based position i: i+1 keys)."""
    i = np.asarray(pos_in_seq, dtype=np.int64)
    return int((2 * H * (dqk + dv) * (i + 1)).sum())


def attn_bytes(T, B, H, dqk, dv, P, NB, elem=2) -> int:
    """Algorithmic bytes of one attention pass: q, k, v read once, out written
    once, timestamps, offsets and both bias tables read once."""
    return T * H * (2 * dqk + dv) * elem + T * H * dv * elem + 8 * T + 8 * (B + 1) + 4 * H * (P + NB)


def layer_flops(T, D, H, d) -> int:
    return 2 * T * D * 4 * H * d + 2 * T * H * d * D


# ----------------------------------------------------------------------------- env

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_timing(local_ms: float, local_units: float, world: int, device=None):
    """(max elapsed ms over ranks, sum of work units over ranks)."""
    if world == 1:
        return local_ms, local_units
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    u = torch.tensor([local_units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = [(0x1, "gpu_idle"), (0x2, "applications_clocks_setting"), (0x4, "sw_power_cap"),
               (0x8, "hw_slowdown"), (0x10, "sync_boost"), (0x20, "sw_thermal_slowdown"),
               (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"),
               (0x100, "display_clock_setting")]

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.handle = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:   # clocks are reported as unavailable, never faked
            self.error = str(e)

    def _handle(self, device_index):
        import torch
        pynvml = self.nv
        try:
            p = torch.cuda.get_device_properties(device_index)
            bus = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(device_index)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
                self.reasons |= int(r)
            except Exception:
                pass
            self._stop.wait(self.period)

    def start(self):
        if self.handle is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()

    def stop(self):
        if self._thr is not None:
            self._stop.set()
            self._thr.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        names = [n for bit, n in self.REASONS if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def source_digest(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def profiled_traffic(kernel_tag: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, if it was taken on the current kernel source; else None."""
    path = os.path.join(PROFILE_DIR, kernel_tag + ".md")
    try:
        txt = open(path).read()
    except OSError:
        return None
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    m_h = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", txt)
    if not m_b or not m_h or m_h.group(1) != source_digest(ATTN_SRC):
        return None
    return float(m_b.group(1))


# ----------------------------------------------------------------------------- oracle leg

def oracle_sample_rate(inp, budget_s: float, seed: int = 0):
    """Time the fp64 oracle on a random sample of query rows of ``inp`` sized to
    about ``budget_s`` seconds. Returns (TFLOP/s, rows, seconds, threads)."""
    import oracle
    rng = np.random.default_rng(seed)
    off = inp.seq_offsets
    T = inp.T
    seq_of = np.repeat(np.arange(inp.B), np.diff(off))
    pos = np.arange(T) - off[seq_of]
    H, dqk, dv = inp.H, inp.q.shape[2], inp.v.shape[2]

    def run(rows):
        t0 = time.perf_counter()
        oracle.attn(off, inp.q, inp.k, inp.v, inp.timestamps, inp.pos_bias, inp.time_bias,
                    inp.max_seqlen, rows=rows)
        return time.perf_counter() - t0

    order = rng.permutation(T)
    n = 16
    while True:                     # grow the probe until its rate is stable
        probe = np.sort(order[:n])
        dt = max(run(probe), 1e-6)
        if dt >= min(1.0, budget_s / 8) or n >= T:
            break
        n = min(T, n * 4)
    rate = row_causal_flops(pos[probe], H, dqk, dv) / dt          # flops / s
    target = rate * budget_s
    cum = np.cumsum(2 * H * (dqk + dv) * (pos[order] + 1))
    nrows = int(np.clip(np.searchsorted(cum, target) + 1, 16, T))
    rows = np.sort(order[:nrows])
    dt = run(rows)
    fl = row_causal_flops(pos[rows], H, dqk, dv)
    return fl / dt / 1e12, nrows, dt, oracle.num_threads()


# ----------------------------------------------------------------------------- GPU arm

def l2_note(in_bytes, ncopies):
    """How the timing keeps HBM honest: inputs larger than L2, or rotating
    input copies whose total is more than twice L2."""
    if ncopies == 1:
        return "inputs %.0f MB > L2" % (in_bytes / 2 ** 20)
    return "rotating %d input copies (%.0f MB) > 2x L2" % (ncopies, ncopies * in_bytes / 2 ** 20)


def attn_copies(in_bytes):
    return max(1, int(np.ceil(2 * L2_BYTES / max(in_bytes, 1))))


def workload_config(cfg_id, B, T, max_seqlen, seed, world, extra):
    """The ``config`` dict of a line; both arms print the same one."""
    from gen import CONFIGS
    cfg = CONFIGS[cfg_id]
    c = {"workload": cfg["name"], "B": B, "total_tokens": T, "max_seqlen": max_seqlen,
         "num_pos": cfg["num_pos"], "num_time_buckets": cfg["num_buckets"], "seed": seed,
         "parallelism": "dp%d" % world}
    c.update(extra)
    return c


def launch_floor_ms(dev, steps):
    """Per-launch time of a graph of ``steps`` launches of a one-element torch
    kernel: the floor a graph-replayed step of one launch cannot go below."""
    import torch
    x = torch.zeros(1, device=dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(steps):
            x.add_(1.0)
    g.replay()
    torch.cuda.synchronize(dev)
    best = None
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize(dev)
        t = a.elapsed_time(b) / steps
        best = t if best is None else min(best, t)
    del g
    return best


def bench_attention(args, rank, world, local, peaks, peak_kind, cfg_id=None, cpu_budget_s=None):
    import torch
    import jagged_pointwise_attention_b200 as hstu
    from gen import CONFIGS, make_attn_inputs

    cfg_id = args.config if cfg_id is None else cfg_id
    cfg = CONFIGS[cfg_id]
    seed = 1000 + cfg_id + 7919 * rank
    inp = make_attn_inputs(cfg_id, seed=seed)
    if args.sample_seqs:
        # a smaller case of the same kernel (the workload's first sequences):
        # for profiler captures, not for bench lines
        from gen import take_sequences
        inp = take_sequences(inp, list(range(min(args.sample_seqs, inp.B))))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    bf = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
    H, d = inp.H, inp.d
    lengths = inp.lengths
    flops = causal_flops(lengths, H, d, d)
    nbytes = attn_bytes(inp.T, inp.B, H, d, d, inp.pos_bias.shape[1], inp.time_bias.shape[1],
                        2 if inp.dtype == "bf16" else 4)
    in_bytes = inp.T * H * 3 * d * (2 if bf == torch.bfloat16 else 4)
    ncopies = attn_copies(in_bytes)

    def to_dev(a, dt=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.to(dt) if dt is not None else t).to(dev)

    copies = []
    for _ in range(ncopies):
        copies.append(dict(q=to_dev(inp.q, bf), k=to_dev(inp.k, bf), v=to_dev(inp.v, bf),
                           out=torch.empty((inp.T, H, d), dtype=bf, device=dev)))
    off = to_dev(inp.seq_offsets)
    ts = to_dev(inp.timestamps)
    pos = to_dev(inp.pos_bias)
    tb = to_dev(inp.time_bias)
    ws = torch.empty(max(16, hstu.hstu_attn_workspace_bytes(inp.B, inp.T, inp.max_seqlen, inp.H,
                                                                inp.pos_bias.shape[1])),
                     dtype=torch.uint8, device=dev)

    def step(i, ev=None):
        c = copies[i % ncopies]
        if bf == torch.bfloat16:
            hstu.hstu_attn_plan(off, inp.max_seqlen, inp.T, ws)
        if ev is not None:
            ev[0].record(stream)
        hstu.hstu_attn_run(c["q"], c["k"], c["v"], off, ts, pos, tb, inp.max_seqlen, c["out"], ws)
        if ev is not None:
            ev[1].record(stream)

    launches_per_step = 3 if bf == torch.bfloat16 else 1   # plan, bias tables, attention
    for i in range(args.warmup):
        step(i)
    st = hstu.hstu_device_status()
    if st != 0:
        raise RuntimeError("device status %d after warm-up" % st)

    # Kernel-only time of the attention launch (roofline): eager steps with
    # events around the run call, outside the timed region. A short device-side
    # spin ahead of each step keeps the GPU busy while the host queues the
    # step, so that host launch latency does not fall between the events.
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    spin = getattr(torch.cuda, "_sleep", None)
    for i in range(args.steps):
        if spin is not None:
            spin(100000)
        step(i, kev[i])
    torch.cuda.synchronize(dev)
    kernel_ms = [a.elapsed_time(b) for a, b in kev]

    # The timed steps are replayed from one CUDA graph holding all K steps
    # (each a plan + run over its step's input copy), so neither the host's
    # launch cost nor gaps between graph launches are part of the step time.
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(args.steps):
                step(i)
        graph.replay()
        torch.cuda.synchronize(dev)
        stream = torch.cuda.current_stream(dev)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    _barrier(world)
    torch.cuda.synchronize(dev)
    sampler.start()
    e0.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for i in range(args.steps):
            step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.stop()
    _barrier(world)
    local_ms = e0.elapsed_time(e1)
    del graph
    st = hstu.hstu_device_status()
    if st != 0:
        raise RuntimeError("device status %d after timed steps" % st)
    max_ms, total_flops = reduce_timing(local_ms, float(flops) * args.steps, world, dev)
    _, total_tokens = reduce_timing(0.0, float(inp.T) * args.steps, world, dev)
    ms_per_step = max_ms / args.steps
    value = total_flops / (max_ms * 1e-3) / 1e12

    # roofline of the attention kernel: tensor-bound for long sequences (the
    # 8192 regime), HBM-bound for the short-history batches
    k_avg_ms = float(np.mean(kernel_ms))
    tflops = flops / (k_avg_ms * 1e-3) / 1e12
    gbs = nbytes / (k_avg_ms * 1e-3) / 1e9
    tag = "attn_fwd_bf16_" + cfg["name"]
    traffic = profiled_traffic(tag)
    if cfg_id == 4:
        roofline = {"bound": "tensor", "achieved": round(tflops, 2),
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": round(tflops / peaks["bf16_tflops"], 4),
                    "peak_kind": "burst bf16 dense, %s" % peak_kind,
                    "frac_of_nominal_2250": round(tflops / NOMINAL_BF16_TFLOPS, 4)}
    else:
        roofline = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                    "peak_kind": "copy bandwidth, %s" % peak_kind,
                    "frac_of_nominal_8000": round(gbs / 8000.0, 4)}
    roofline.update({"traffic": traffic, "algorithmic_bytes": nbytes,
                     "kernel": "attn_fwd_bf16_kernel<%d>" % d, "kernel_ms": round(k_avg_ms, 4),
                     "tflops_causal": round(tflops, 2), "hbm_gbs_achieved": round(gbs, 1)})

    # end to end: pinned host inputs -> device, public API call, result -> pinned host
    e2e = e2e_attention(args, inp, dev, stream, flops, world)

    if cfg_id != 4:
        # the short batches are latency-bound: report the launch floor of a
        # graph-replayed step and the HBM-bar time next to the step
        floor = launch_floor_ms(dev, max(args.steps, 10))
        roofline.update({"launch_floor_ms": round(floor, 4),
                         "hbm_bar_ms": round(nbytes / (0.6 * peaks["hbm_gbs"] * 1e9) * 1e3, 4),
                         "step_over_kernel": round(ms_per_step / k_avg_ms, 3)})

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        v, nrows, secs, thr = oracle_sample_rate(
            inp, args.cpu_budget_s if cpu_budget_s is None else cpu_budget_s)
        cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
               "sample": "%d random query rows (all heads) of the same batch, fp64, %.3f s"
                         % (nrows, secs)}

    clocks = sampler.summary()
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": inp.dtype,
        "data": "synthetic (seeded generator; no dataset)",
        "config": workload_config(cfg_id, inp.B, inp.T, inp.max_seqlen, seed, world,
                                  {"H": H, "d": d, "l2": l2_note(in_bytes, ncopies),
                                   **({"first_sequences_only": inp.B} if args.sample_seqs else {})}),
        "launch": "eager" if args.no_graph else "one CUDA graph of the K steps (plan + run each)",
        "pct_of_bf16_peak": {"measured_burst": round(100 * value / peaks["bf16_tflops"], 2),
                             "nominal_2250": round(100 * value / NOMINAL_BF16_TFLOPS, 2)},
        "tokens_per_s": round(total_tokens / (max_ms * 1e-3), 1),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps, "clocks": clocks,
    }
    return line


def e2e_attention(args, inp, dev, stream, flops, world):
    """End to end through the public call: every step copies its inputs from
    pinned host memory, runs ``hstu_attn_fwd`` and copies the output back.
    Steps are pipelined the way a serving loop would run them: step i's
    host-to-device copies (copy stream) overlap step i-1's attention (the
    compute stream) and step i-2's device-to-host copy (a third stream), with
    two device buffer sets."""
    import torch
    import jagged_pointwise_attention_b200 as hstu
    bf = torch.bfloat16 if inp.dtype == "bf16" else torch.float32

    def pinned(a, dt=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.to(dt) if dt is not None else t).pin_memory()

    host = dict(q=pinned(inp.q, bf), k=pinned(inp.k, bf), v=pinned(inp.v, bf),
                off=pinned(inp.seq_offsets), ts=pinned(inp.timestamps), pos=pinned(inp.pos_bias),
                tb=pinned(inp.time_bias))
    shape = (inp.T, inp.H, inp.d)
    devb = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(2)]
    out_dev = [torch.empty(shape, dtype=bf, device=dev) for _ in range(2)]
    out_host = [torch.empty(shape, dtype=bf).pin_memory() for _ in range(2)]
    ws = torch.empty(max(16, hstu.hstu_attn_workspace_bytes(inp.B, inp.T, inp.max_seqlen, inp.H,
                                                                inp.pos_bias.shape[1])),
                     dtype=torch.uint8, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "run", "out")}
    used = [False, False]

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev["run"][b])        # step i-2 is done with buffer set b
            for k in host:
                devb[b][k].copy_(host[k], non_blocking=True)
            ev["in"][b].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev["in"][b])
            if used[b]:
                stream.wait_event(ev["out"][b])      # step i-2's output has been read
            d = devb[b]
            hstu.hstu_attn_fwd(d["q"], d["k"], d["v"], d["off"], d["ts"], d["pos"], d["tb"],
                               inp.max_seqlen, out=out_dev[b], workspace=ws, stream=stream)
            ev["run"][b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["run"][b])
            out_host[b].copy_(out_dev[b], non_blocking=True)
            ev["out"][b].record(s_out)
        used[b] = True

    for i in range(max(2, min(args.warmup, 3))):
        step(i)
    n = max(1, min(args.steps, args.e2e_steps))
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize(dev)
    a.record(stream)
    s_in.wait_stream(stream)        # the first copy starts after the start event
    for i in range(n):
        step(i)
    for b in range(2):
        stream.wait_event(ev["out"][b])
        stream.wait_event(ev["in"][b])
    e.record(stream)
    torch.cuda.synchronize(dev)
    _barrier(world)
    ms, tot = reduce_timing(a.elapsed_time(e), float(flops) * n, world, dev)
    return {"value": round(tot / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n,
            "ms_per_step": round(ms / n, 4),
            "pipeline": "step i's host-to-device copies overlap step i-1's attention and "
                        "step i-2's device-to-host copy (three streams, two buffer sets)"}


def oracle_layer_rate(li, budget_s: float, seed: int = 0):
    """Time the fp64 oracle's whole layer on a random subset of whole
    sequences of ``li`` sized to about ``budget_s`` seconds. Returns
    (TFLOP/s, sequences, tokens, seconds, threads)."""
    import oracle
    rng = np.random.default_rng(seed)
    off = li.seq_offsets
    order = rng.permutation(li.B)

    def run(seqs):
        seqs = np.sort(seqs)
        idx = np.concatenate([np.arange(off[b], off[b + 1]) for b in seqs])
        lens = np.diff(off)[seqs]
        o = np.zeros(len(seqs) + 1, np.int64)
        np.cumsum(lens, out=o[1:])
        t0 = time.perf_counter()
        oracle.layer(o, li.x[idx], li.W1, li.W2, li.H, li.d, li.timestamps[idx], li.pos_bias,
                     li.time_bias, li.max_seqlen, ln_eps=li.ln_eps)
        dt = time.perf_counter() - t0
        fl = causal_flops(lens, li.H, li.d, li.d) + layer_flops(int(lens.sum()), li.D, li.H, li.d)
        return fl, dt, int(lens.sum())

    k = 1
    while True:
        fl, dt, ntok = run(order[:k])
        if dt >= budget_s / 4 or k >= li.B:
            break
        k = min(li.B, max(k + 1, int(k * budget_s / 4 / max(dt, 1e-3))))
    rate = fl / dt
    return rate / 1e12, k, ntok, dt, oracle.num_threads()


def bench_layer(args, rank, world, local, peaks, peak_kind, cfg_id=None, cpu_budget_s=None,
                fp8=None, input_norm=None):
    import torch
    import jagged_pointwise_attention_b200 as hstu
    from gen import CONFIGS, make_layer_inputs

    cfg_id = args.config if cfg_id is None else cfg_id
    fp8 = args.fp8 if fp8 is None else fp8
    input_norm = args.input_norm if input_norm is None else input_norm
    cfg = CONFIGS[cfg_id]
    seed = 1000 + cfg_id + 7919 * rank
    li = make_layer_inputs(cfg_id, seed=seed)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    bf = torch.bfloat16
    to = lambda a, dt=None: (torch.from_numpy(np.ascontiguousarray(a)).to(dt)  # noqa: E731
                             if dt else torch.from_numpy(np.ascontiguousarray(a))).to(dev)
    x, W1, W2 = to(li.x, bf), to(li.W1, bf), to(li.W2, bf)
    off, ts, pos, tb = to(li.seq_offsets), to(li.timestamps), to(li.pos_bias), to(li.time_bias)
    out = torch.empty_like(x)
    ws = torch.empty(hstu.hstu_layer_workspace_bytes(li.T, li.B, li.D, li.H, li.d, li.max_seqlen),
                     dtype=torch.uint8, device=dev)
    lengths = np.diff(li.seq_offsets)
    fl = causal_flops(lengths, li.H, li.d, li.d) + layer_flops(li.T, li.D, li.H, li.d)

    # the input LayerNorm's affine terms (the model's parameters)
    rng = np.random.default_rng(seed + 1)
    in_g = to((1 + 0.1 * rng.standard_normal(li.D)).astype(np.float32)) if input_norm else None
    in_b = to((0.1 * rng.standard_normal(li.D)).astype(np.float32)) if input_norm else None
    if fp8:
        W1q, s1 = hstu.hstu_quant_rows_e4m3(W1)
        W2q, s2 = hstu.hstu_quant_rows_e4m3(W2)
        ws = torch.empty(hstu.hstu_layer_fp8_workspace_bytes(li.T, li.B, li.D, li.H, li.d,
                                                              li.max_seqlen),
                         dtype=torch.uint8, device=dev)

    def layer_call(xx, oo, o, sq, strm=None):   # x, out, seq_offsets, timestamps
        if fp8:
            hstu.hstu_layer_fp8_fwd(xx, W1q, s1, W2q, s2, o, sq, pos, tb, li.H, li.d,
                                    li.max_seqlen, ln_eps=li.ln_eps, out=oo, workspace=ws,
                                    stream=strm, input_norm=input_norm, in_gamma=in_g,
                                    in_beta=in_b)
        else:
            hstu.hstu_layer_fwd(xx, W1, W2, o, sq, pos, tb, li.H, li.d, li.max_seqlen,
                                ln_eps=li.ln_eps, out=oo, workspace=ws, stream=strm,
                                input_norm=input_norm, in_gamma=in_g, in_beta=in_b)

    def step():
        layer_call(x, out, off, ts)

    for _ in range(args.warmup):
        step()
    assert hstu.hstu_device_status() == 0
    sampler = ClockSampler(local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize(dev)
    sampler.start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.stop()
    _barrier(world)
    assert hstu.hstu_device_status() == 0
    max_ms, tot = reduce_timing(e0.elapsed_time(e1), float(fl) * args.steps, world, dev)
    _, toks = reduce_timing(0.0, float(li.T) * args.steps, world, dev)
    value = tot / (max_ms * 1e-3) / 1e12
    # the step's six launches are timed together: the roofline is the step's
    # FLOPs against the dense bf16 peak (the layer is tensor-bound throughout)
    step_tf = fl / (max_ms / args.steps * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": round(step_tf, 2), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(step_tf / peaks["bf16_tflops"], 4),
                "peak_kind": "burst bf16 dense, %s" % peak_kind, "traffic": None,
                "kernel": "whole layer step (%sf1, plan, bias tables, attention, LayerNorm "
                          "gate, f2)" % ("input LayerNorm, " if input_norm else "")}
    e2e = e2e_layer(args, li, dev, stream, fl, world, layer_call)
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline and cpu_budget_s != 0:
        v, nseq, ntok, secs, thr = oracle_layer_rate(
            li, args.cpu_budget_s if cpu_budget_s is None else cpu_budget_s)
        cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
               "sample": "%d random whole sequences (%d tokens) of the same batch, the whole "
                         "layer in fp64, %.3f s" % (nseq, ntok, secs)}
    return {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 projections, bf16 attention" if fp8 else "bf16",
        "data": "synthetic (seeded generator; no dataset)",
        "config": workload_config(cfg_id, li.B, li.T, li.max_seqlen, seed, world,
                                  {"D": li.D, "H": li.H, "d": li.d,
                                   "projections": "e4m3" if fp8 else "bf16",
                                   "input_layernorm": bool(input_norm),
                                   "l2": "layer working set %.0f MB > L2" % (
                                       (ws.numel() + 2 * x.numel() * 2) / 2 ** 20)}),
        "launch": "eager, one call per step",
        "tokens_per_s": round(toks / (max_ms * 1e-3), 1),
        "pct_of_bf16_peak": {"measured_burst": round(100 * value / peaks["bf16_tflops"], 2)},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": (7 if fp8 or input_norm else 6) * args.steps,
        "clocks": sampler.summary(),
    }


def e2e_layer(args, li, dev, stream, flops, world, layer_call):
    """End to end through the layer entry point that `layer_call` makes
    (hstu_layer_fwd or hstu_layer_fp8_fwd): every step copies its activations x,
    offsets and timestamps from pinned host memory and the output back; the
    weights and bias tables are the model's parameters and stay on the device.
    Pipelined like the attention's: step i's copies in overlap step i-1's
    layer and step i-2's copy out."""
    import torch
    bf = torch.bfloat16

    def pinned(a, dt=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.to(dt) if dt is not None else t).pin_memory()

    host = dict(x=pinned(li.x, bf), off=pinned(li.seq_offsets), ts=pinned(li.timestamps))
    devb = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(2)]
    out_dev = [torch.empty((li.T, li.D), dtype=bf, device=dev) for _ in range(2)]
    out_host = [torch.empty((li.T, li.D), dtype=bf).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "run", "out")}
    used = [False, False]

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev["run"][b])
            for k in host:
                devb[b][k].copy_(host[k], non_blocking=True)
            ev["in"][b].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(ev["in"][b])
            if used[b]:
                stream.wait_event(ev["out"][b])
            d = devb[b]
            layer_call(d["x"], out_dev[b], d["off"], d["ts"], stream)
            ev["run"][b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["run"][b])
            out_host[b].copy_(out_dev[b], non_blocking=True)
            ev["out"][b].record(s_out)
        used[b] = True

    for i in range(max(2, min(args.warmup, 3))):
        step(i)
    n = max(1, min(args.steps, args.e2e_steps))
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize(dev)
    a.record(stream)
    s_in.wait_stream(stream)
    for i in range(n):
        step(i)
    for b in range(2):
        stream.wait_event(ev["out"][b])
        stream.wait_event(ev["in"][b])
    e.record(stream)
    torch.cuda.synchronize(dev)
    _barrier(world)
    ms, tot = reduce_timing(a.elapsed_time(e), float(flops) * n, world, dev)
    return {"value": round(tot / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n,
            "ms_per_step": round(ms / n, 4),
            "pipeline": "step i's host-to-device copies overlap step i-1's layer and step "
                        "i-2's device-to-host copy (three streams, two buffer sets)"}


def bench_backward(args, rank, world, local, peaks, peak_kind, cfg_id=None):
    """The attention backward on tensor cores (hstu_attn_bwd: bf16 inputs,
    fp32 gradients) on an attention workload (its lengths, heads, head
    dimension and bias tables). One step: the clears of dq and the table
    gradients, the plan, the backward kernel. Algorithmic FLOPs: the four
    contractions dV = P^T dO, dP = dO V^T, dQ = dS K, dK = dS^T Q over the
    causal pairs, twice the forward's (the kernel also recomputes S = Q K^T,
    which is not counted). Roofline: those FLOPs against the dense bf16 peak."""
    import torch
    import jagged_pointwise_attention_b200 as hstu
    from gen import CONFIGS, make_attn_inputs
    cfg_id = args.config if cfg_id is None else cfg_id
    cfg = CONFIGS[cfg_id]
    if cfg["kind"] == "layer":
        raise SystemExit("--backward takes an attention workload (--config 2, 3 or 4)")
    seed = 1000 + cfg_id + 7919 * rank
    inp = make_attn_inputs(cfg_id, seed=seed)
    if args.sample_seqs:
        # a smaller case of the same kernel (the workload's first sequences):
        # for profiler captures, not for bench lines
        from gen import take_sequences
        inp = take_sequences(inp, list(range(min(args.sample_seqs, inp.B))))
    dev = torch.device("cuda", local)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev).to(torch.bfloat16)  # noqa: E731
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)  # noqa: E731
    i64 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
    q, k, v = bf(inp.q), bf(inp.k), bf(inp.v)
    dout = torch.randn(v.shape, generator=torch.Generator().manual_seed(7),
                       dtype=torch.float32).to(dev).to(torch.bfloat16)
    off, ts, pos, tb = i64(inp.seq_offsets), i64(inp.timestamps), f32(inp.pos_bias), f32(inp.time_bias)
    lengths = np.diff(inp.seq_offsets)
    d = int(inp.q.shape[2])
    flops = 2 * causal_flops(lengths, inp.H, d, int(inp.v.shape[2]))
    T, H = inp.T, inp.H
    outs = (torch.empty((T, H, d), dtype=torch.float32, device=dev),
            torch.empty((T, H, d), dtype=torch.float32, device=dev),
            torch.empty((T, H, d), dtype=torch.float32, device=dev),
            torch.empty_like(pos), torch.empty_like(tb))
    ws = torch.empty(hstu.hstu_attn_bwd_workspace_bytes(inp.B, T, inp.max_seqlen),
                     dtype=torch.uint8, device=dev)

    def step():
        hstu.hstu_attn_bwd(q, k, v, dout, off, ts, pos, tb, inp.max_seqlen, workspace=ws,
                           out=outs)

    for _ in range(args.warmup):
        step()
    assert hstu.hstu_device_status() == 0
    sampler = ClockSampler(local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize(dev)
    sampler.start()
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize(dev)
    sampler.stop()
    _barrier(world)
    assert hstu.hstu_device_status() == 0
    max_ms, tot = reduce_timing(e0.elapsed_time(e1), float(flops) * args.steps, world, dev)
    value = tot / (max_ms * 1e-3) / 1e12
    step_tf = flops / (max_ms / args.steps * 1e-3) / 1e12
    in_mb = 4 * T * H * d * 2 / 2 ** 20
    return {"metric": "HSTU jagged attn bwd TFLOP/s (causal, bf16 tensor cores)",
            "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16 inputs, fp32 gradients",
            "data": "synthetic (seeded generator; no dataset)",
            "config": {"workload": cfg["name"] + "_backward" + (
                           "_first%d" % inp.B if args.sample_seqs else ""), "B": inp.B, "H": H, "d": d,
                       "total_tokens": T, "seed": seed, "parallelism": "dp%d" % world,
                       "l2": "q, k, v, dout %.0f MB, dq/dk/dv %.0f MB: %s" % (
                           in_mb, 3 * T * H * d * 4 / 2 ** 20,
                           "inputs larger than L2" if in_mb > 126 else
                           "short workload: inputs fit in L2 (timed back to back)")},
            "roofline": {"bound": "tensor", "achieved": round(step_tf, 2),
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(step_tf / peaks["bf16_tflops"], 4),
                         "peak_kind": "burst bf16 dense, %s" % peak_kind, "traffic": None,
                         "kernel": "whole backward step (clears, plan, attn_bwd_bf16_kernel)"},
            "gpu_launches": 2 * args.steps, "clocks": sampler.summary()}


def bench_fp8_linear(args, rank, world, local, peaks, peak_kind):
    """Row-wise E4M3 projections against bf16 ones on the layer's f1 shape
    (79,913 x 512 -> 2048, SiLU) and the FP8 benchmark shape of the
    generative-recommenders README (4096 x 512 -> 512). A step = quantize the
    activations + FP8 GEMM (weights quantized once, as a model would cache
    them); the GEMM alone is timed too. FP8 peak = measured bf16 burst x 2
    (the nominal dense ratio)."""
    import torch
    import jagged_pointwise_attention_b200 as hstu
    dev = torch.device("cuda", local)
    g = torch.Generator(device="cpu").manual_seed(1234 + rank)
    fp8_peak = 2 * peaks["bf16_tflops"]
    shapes = [("f1_layer_T79913_K512_N2048_silu", 79913, 512, 2048, "silu"),
              ("addmm_bench_m4096_k512_n512", 4096, 512, 512, "none")]
    if args.sample_rows:
        # a smaller case of the same kernels (for profiler captures)
        shapes = [("f1_rows%d_K512_N2048_silu" % args.sample_rows, args.sample_rows, 512, 2048,
                   "silu")]
    out = []

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / args.steps

    for name, M, K, N, epi in shapes:
        x = torch.randn((M, K), generator=g).to(torch.bfloat16).to(dev)
        W = (torch.randn((N, K), generator=g) / K ** 0.5).to(torch.bfloat16).to(dev)
        wq, sw = hstu.hstu_quant_rows_e4m3(W)
        xq, sx = hstu.hstu_quant_rows_e4m3(x)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        flops = 2.0 * M * N * K

        def fp8_step():
            q, s_ = hstu.hstu_quant_rows_e4m3(x)
            hstu.hstu_linear_fp8_fwd(q, s_, wq, sw, None, epi, out=y)

        ms_step = timed(fp8_step)
        ms_gemm = timed(lambda: hstu.hstu_linear_fp8_fwd(xq, sx, wq, sw, None, epi, out=y))
        ms_bf16 = timed(lambda: hstu.hstu_linear_fwd(x, W, None, epi, out=y))
        assert hstu.hstu_device_status() == 0
        out.append({"shape": name, "M": M, "K": K, "N": N, "epilogue": epi,
                    "fp8_step_ms": round(ms_step, 4), "fp8_gemm_ms": round(ms_gemm, 4),
                    "bf16_gemm_ms": round(ms_bf16, 4),
                    "fp8_gemm_tflops": round(flops / (ms_gemm * 1e-3) / 1e12, 1),
                    "fp8_step_tflops": round(flops / (ms_step * 1e-3) / 1e12, 1),
                    "bf16_gemm_tflops": round(flops / (ms_bf16 * 1e-3) / 1e12, 1),
                    "fp8_gemm_frac_of_peak": round(flops / (ms_gemm * 1e-3) / 1e12 / fp8_peak, 4)})
    main_ = out[0]
    return {"metric": "row-wise E4M3 projection TFLOP/s (quantize + FP8 GEMM)",
            "value": main_["fp8_step_tflops"], "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "dtype": "e4m3 x e4m3 -> f32 -> bf16", "data": "synthetic (seeded generator)",
            "config": {"workload": main_["shape"], "parallelism": "dp%d" % world},
            "roofline": {"bound": "tensor", "achieved": main_["fp8_gemm_tflops"],
                         "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": main_["fp8_gemm_frac_of_peak"],
                         "peak_kind": "fp8 dense = 2 x measured bf16 burst (nominal ratio), %s"
                                      % peak_kind, "traffic": None,
                         "kernel": "gemm_bf16_kernel<EPI, BN, FP8=true>"},
            "shapes": out}


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- reference arm

def bench_reference(args, rank, world):
    """The fp64 CPU oracle on the host cores: each step a bounded sample of the
    same workload (random query rows of the attention batch, or random whole
    sequences of the layer batch), sized so the whole run ends within a few
    minutes. ``ms_per_step`` is the measured wall time of one sampled step;
    the time the oracle would take for the whole batch is extrapolated from
    the rate and labelled as such."""
    if rank != 0:
        return None
    from gen import CONFIGS, make_attn_inputs, make_layer_inputs
    import oracle
    cfg_id = 4 if args.config is None else args.config
    cfg = CONFIGS[cfg_id]
    seed = 1000 + cfg_id
    n_steps = args.steps + args.warmup
    per_step = max(0.5, min(20.0, args.reference_budget_s / max(n_steps, 1)))
    rates, walls, secs, units = [], [], 0.0, 0
    if cfg["kind"] == "layer":
        li = make_layer_inputs(cfg_id, seed=seed)
        fl_batch = causal_flops(np.diff(li.seq_offsets), li.H, li.d, li.d) + \
            layer_flops(li.T, li.D, li.H, li.d)
        ws_bytes = 2 * li.T * (4 + 1 + 1) * li.H * li.d
        conf = workload_config(cfg_id, li.B, li.T, li.max_seqlen, seed, world,
                               {"D": li.D, "H": li.H, "d": li.d, "projections": "bf16",
                                "l2": "layer working set %.0f MB > L2" % (
                                    (ws_bytes + 2 * li.T * li.D * 2) / 2 ** 20)})
        what = "random whole sequences"
    else:
        inp = make_attn_inputs(cfg_id, seed=seed)
        fl_batch = causal_flops(inp.lengths, inp.H, inp.d, inp.d)
        in_bytes = inp.T * inp.H * 3 * inp.d * (2 if inp.dtype == "bf16" else 4)
        conf = workload_config(cfg_id, inp.B, inp.T, inp.max_seqlen, seed, world,
                               {"H": inp.H, "d": inp.d,
                                "l2": l2_note(in_bytes, attn_copies(in_bytes))})
        what = "random query rows (all heads)"
    for s in range(n_steps):
        t0 = time.perf_counter()
        if cfg["kind"] == "layer":
            v, nu, _, dt, thr = oracle_layer_rate(li, per_step, seed=s)
        else:
            v, nu, dt, thr = oracle_sample_rate(inp, per_step, seed=s)
        wall = time.perf_counter() - t0
        if s >= args.warmup:
            rates.append(v)
            walls.append(wall)
            secs += dt
            units += nu
    value = float(np.mean(rates))
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * float(np.mean(walls)), 3),
        "ms_per_full_batch_extrapolated": round(fl_batch / (value * 1e12) * 1e3, 3)
        if value > 0 else None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded generator; no dataset)",
        "config": conf, "launch": "host cores (OpenMP), no GPU",
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": "%d %s over %d steps (%.1f s of fp64 CPU work); each step a "
                                   "bounded sample of the batch" % (units, what, args.steps, secs)},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ----------------------------------------------------------------------------- main

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=None, choices=[2, 3, 4, 5],
                    help="time one workload only (default: the 8192-length workload as the "
                         "headline line, with the other workloads' lines under 'configs')")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    ap.add_argument("--reference-budget-s", type=float, default=120.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fp8", action="store_true",
                    help="with --config 5: the layer with both projections in FP8 "
                         "(hstu_layer_fp8_fwd, weights quantized once)")
    ap.add_argument("--input-norm", action="store_true",
                    help="with --config 5: LayerNorm on the layer's input before f1 (fused with "
                         "the E4M3 quantization under --fp8)")
    ap.add_argument("--backward", action="store_true",
                    help="time the tensor-core attention backward (hstu_attn_bwd) on the "
                         "--config workload instead of the forward")
    ap.add_argument("--sample-seqs", type=int, default=0,
                    help="only the workload's first N sequences (a smaller case of the same "
                         "kernels, for profiler captures)")
    ap.add_argument("--sample-rows", type=int, default=0,
                    help="with --fp8-linear: only the f1 shape, with this many rows (a smaller "
                         "case of the same kernels, for profiler captures)")
    ap.add_argument("--fp8-linear", action="store_true",
                    help="time the row-wise E4M3 projections (quantize + FP8 GEMM) against the "
                         "bf16 ones on the projection shapes instead of the attention")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps one call at a time instead of replaying "
                         "CUDA graphs")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    return a


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        line = bench_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    peaks, kind = load_peaks()
    from gen import CONFIGS
    if args.backward or args.fp8_linear:
        if args.config is None:
            args.config = 4
        fn = bench_backward if args.backward else bench_fp8_linear
        line = fn(args, rank, world, local, peaks, kind)
    elif args.config is not None:
        fn = bench_layer if CONFIGS[args.config]["kind"] == "layer" else bench_attention
        line = fn(args, rank, world, local, peaks, kind)
    else:
        # headline: the 8192-length workload; the other workloads' lines,
        # each timed the same way, under "configs"
        line = bench_attention(args, rank, world, local, peaks, kind, cfg_id=4)
        subs = {}
        for c in (2, 3, 5):
            fn = bench_layer if CONFIGS[c]["kind"] == "layer" else bench_attention
            sub = fn(args, rank, world, local, peaks, kind, cfg_id=c,
                     cpu_budget_s=min(args.cpu_budget_s, 8.0))
            subs[sub["config"]["workload"]] = sub
        # the layer's variants: E4M3 projections, and the input LayerNorm (for
        # the FP8 layer fused with x's quantization); the oracle's rate is the
        # bf16 line's
        for fp8, norm in ((True, False), (False, True), (True, True)):
            sub = bench_layer(args, rank, world, local, peaks, kind, cfg_id=5, cpu_budget_s=0,
                              fp8=fp8, input_norm=norm)
            name = sub["config"]["workload"] + ("_fp8" if fp8 else "") + ("_input_ln" if norm
                                                                          else "")
            subs[name] = sub
        # the attention backward on the long and the short-history workloads
        for c in (4, 2):
            sub = bench_backward(args, rank, world, local, peaks, kind, cfg_id=c)
            subs[sub["config"]["workload"]] = sub
        line["configs"] = subs
        line["gpu_launches_all_lines"] = line["gpu_launches"] + sum(
            v["gpu_launches"] for v in subs.values())
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
