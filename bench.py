#!/usr/bin/env python
"""Benchmark of the jagged candidate-isolated attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the hot path over one batch of the 256-user workload (256 users,
lognormal histories with median 280 clipped to [0, 4096], 4 prefix tokens and 64 candidates per
user, H = 8, d_head = 128, bf16, seed 0): offsets from lengths, then the plan (segment IDs, bounds,
cost-sorted work queue) and the attention kernel, all through the C ABI of libjca.so. Inputs are
resident in HBM when the timed region starts; Q/K/V (837 MB) exceed the 126 MB L2, so no flush is
needed between steps. The metric is effective attention TFLOP/s: 4 * d_head * H FLOPs per
(query, key) pair the candidate-isolation mask allows (padding and masked pairs not counted).

With torchrun (N > 1) every rank runs its own batch (weak scaling, no data-path collective); the
time is the max over ranks and the value counts the work of all ranks. ``--impl reference`` times
the CPU oracle (the reference arm of this build) on a bounded sample of the same workload.
Rank 0 prints one JSON line.
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
sys.path.insert(0, ROOT)

METRIC = "effective attention TFLOP/s (unpadded) and tokens/s, % of B200 bf16 peak"
WORKLOAD = ("users256: 256 users, history lengths floor(lognormal(ln 280, 1)) clipped to [0, 4096] "
            "(users 0, 64, 128, 192 empty, user 1 = 4096), 4 prefix + 64 candidates per user, "
            "H=8, d_head=128, bf16 N(0,1), seed 0")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def kernel_source_sha() -> str:
    """Hash of the attention kernel's source with comments and blank space removed, so that only a
    change of the code (not of its comments) invalidates a recorded capture."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "candidate_isolated_jagged_b200", "csrc")
    for name in ("attention.cu", "jca_device.cuh"):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(name: str):
    """DRAM bytes per launch recorded in profiles/<name>.md by an ncu capture, or None when the
    summary is missing or the kernel source changed since it was taken."""
    path = os.path.join(ROOT, "profiles", name + ".md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_sha = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_b or m_sha.group(1) != kernel_source_sha():
        return None
    return float(m_b.group(1))


class ClockSampler:
    """Samples SM clocks and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.times, self.reasons, self.ok = [], [], set(), False
        self.t_mark = None
        self.max_mhz = None
        self._stop = threading.Event()
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 - NVML missing: report no clocks
            self.ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.times.append(time.perf_counter())
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()

    def mark(self):
        """Start of the timed region (the samples before it cover the warm-up's identical load)."""
        self.t_mark = time.perf_counter()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "note": "NVML unavailable" if not self.ok else "no samples"}
        timed = [c for c, t in zip(self.samples, self.times)
                 if self.t_mark is not None and t >= self.t_mark]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "samples_timed_region": len(timed),
                "sm_mhz_timed_region": float(statistics.median(timed)) if timed else None,
                "window_ms": 1e3 * (self.times[-1] - self.times[0]),
                "covers": "back-to-back warm-up steps (at least 100 ms) and the timed region"}


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise max of per-rank timings (every rank calls this; a no-op on one process)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def weak_scaling_value(units_per_rank: float, world: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return world * units_per_rank * steps / (elapsed_ms / 1e3)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


# ------------------------------------------------------------------------------------------------
# CPU oracle arm
# ------------------------------------------------------------------------------------------------

def oracle_sample_users(batch, stride: int, phase: int):
    return [u for u in range(batch.B) if u % stride == phase]


def time_oracle(batch, users, repeats: int = 1):
    """Effective TFLOP/s of the fp64 oracle on the given users of the batch (host cores)."""
    import oracle
    from candidate_isolated_jagged_b200 import metrics
    off = oracle.offsets_from_lengths(batch.row_lengths)
    seg = oracle.segment_ids(off, batch.cand_start, batch.valid)
    n1 = (batch.prefix + batch.hist_real)[users]
    pairs = metrics.allowed_pairs_from_counts(n1, batch.n_cand[users])
    flops = metrics.effective_flops(pairs, batch.H, batch.d)
    tokens = int(np.sum(batch.row_lengths[users]))
    times = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        oracle.jagged_cand_attn(batch.q, batch.k, batch.v, off, seg, batch.scale, users=users)
        times.append(time.perf_counter() - t0)
    return flops, tokens, times


def run_reference(args, rank: int):
    if rank != 0:
        return 0
    import synth
    batch = synth.users256()
    # Each step: the oracle over 8 representative users (index = 5 mod 32) of the same batch.
    users = oracle_sample_users(batch, 32, 5)
    flops, tokens, _ = time_oracle(batch, users, repeats=max(1, args.warmup))
    _, _, times = time_oracle(batch, users, repeats=args.steps)
    total = float(np.sum(times))
    value = flops * args.steps / total / 1e12
    cores = blas_threads()
    sample = (f"users with index = 5 mod 32 ({len(users)} of 256, {tokens} rows, "
              f"{flops / 1e9:.2f} effective GFLOP) per step, fp64 numpy")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": sample},
        "tokens_per_s": tokens * args.steps / total,
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------

def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import synth
    from candidate_isolated_jagged_b200 import jca, metrics

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist  # noqa: F811

    peaks = load_peaks()
    shard_info = None
    if args.shard == "users":
        # One global batch split over the ranks by users (LPT over tile cost); each rank draws and
        # computes only its own users, and its outputs stay on its GPU.
        G = args.global_users or 256 * world
        hist = synth.lognormal_history_lengths(G, 0)
        shard, load = jca.shard_users(hist + 68, hist + 4, world)
        mine = np.nonzero(shard == rank)[0]
        batch = synth.users_batch(hist, mine, 4, 64, 8, 128, seed=0, name=f"users{G}_shard{rank}")
        g_pairs = metrics.allowed_pairs_from_counts(hist + 4, np.full(G, 64))
        job_flops = metrics.effective_flops(g_pairs, 8, 128)
        job_tokens = int((hist + 68).sum())
        shard_info = {"global_users": int(G), "users_this_rank": int(mine.size),
                      "tile_cost_per_rank": [int(x) for x in load],
                      "imbalance": float(load.max() / max(load.mean(), 1e-30))}
        scaling = "weak" if args.global_users is None else "strong"
    else:
        batch = synth.users256()
        scaling = "weak"
    B, T, H, d = batch.B, batch.T, batch.H, batch.d
    n1 = batch.prefix + batch.hist_real
    pairs = metrics.allowed_pairs_from_counts(n1, batch.n_cand)
    flops = metrics.effective_flops(pairs, H, d)
    valid_tokens = int(batch.row_lengths.sum()) if batch.valid is None else int(batch.valid.sum())
    if shard_info is None:   # replicas: every rank runs its own copy of the batch
        job_flops, job_tokens = world * flops, world * valid_tokens

    stream = torch.cuda.current_stream(dev)
    q, k, v = (t.to(dev) for t in (batch.q, batch.k, batch.v))
    lengths = torch.tensor(batch.row_lengths, dtype=torch.int64, device=dev)
    cand_start = torch.tensor(batch.cand_start, dtype=torch.int64, device=dev)
    offsets = torch.empty(B + 1, dtype=torch.int64, device=dev)
    out = torch.empty(T, H, d, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(jca.jca_workspace_bytes(B, T, H, d), dtype=torch.uint8, device=dev)
    status = jca.new_status(dev)
    launches_per_step = 4  # offsets, segment IDs + bounds (one pass), work queue, attention

    def step(ev=None, s=stream):
        jca.jca_offsets_from_lengths(lengths, offsets, status, s)
        jca.jagged_cand_attn_plan(offsets, cand_start, None, T, H, d, ws, status, s)
        if ev is not None:
            ev[0].record(s)
        jca.jagged_cand_attn_run(q, k, v, out, None, B, ws, status, stream=s)
        if ev is not None:
            ev[1].record(s)

    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    with sampler:
        # Warm-up under the clock sampler: at least W steps and at least 100 ms of back-to-back
        # steps, so that the clock record covers the same load even when the timed region is short.
        t_w, n_w = time.perf_counter(), 0
        while n_w < args.warmup or time.perf_counter() - t_w < 0.1:
            step()
            n_w += 1
            if n_w % 32 == 0:
                torch.cuda.synchronize(dev)
        torch.cuda.synchronize(dev)
        jca.check_status(status, "warm-up")
        assert bool(torch.isfinite(out.float()).all()), "non-finite attention output"
        # The step's four launches (offsets, segment IDs + bounds, work queue, attention) as one
        # CUDA graph, replayed once per timed step: the same kernels and work, without the host
        # launch gaps between them. Every call is capturable (no host synchronisation, no
        # allocation).
        graph = None
        if not args.no_graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step(s=torch.cuda.current_stream(dev))
            graph.replay()
            torch.cuda.synchronize(dev)
            jca.check_status(status, "graph warm-up")
        if dist:
            dist.barrier()
        torch.cuda.synchronize(dev)
        sampler.mark()
        t_start.record(stream)
        for i in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                step(kev[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        if graph is not None:
            # The attention kernel's own time, with CUDA events around its launch on the stream,
            # over the same number of steps right after (for the roofline).
            for i in range(args.steps):
                step(kev[i])
            torch.cuda.synchronize(dev)
        if dist:
            dist.barrier()
    jca.check_status(status, "timed region")
    elapsed_ms = t_start.elapsed_time(t_end)
    kernel_ms = float(np.mean([a.elapsed_time(b) for a, b in kev]))
    elapsed_ms, kernel_ms = max_over_ranks([elapsed_ms, kernel_ms], dist, dev)
    ms_per_step = elapsed_ms / args.steps
    value = job_flops * args.steps / (elapsed_ms / 1e3) / 1e12

    # ---- end to end through the public API: host inputs in, host output back ----
    # Every step copies its inputs from pinned host memory and reads its output back. The copies
    # run on their own streams and the device tensors are double-buffered, so that step i + 1's
    # inputs cross PCIe while step i computes and step i - 1's output comes back (the link is
    # full duplex); the timed region spans the first input copy to the last output copy.
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    pin = lambda t: t.pin_memory()  # noqa: E731
    q_h, k_h, v_h = pin(batch.q), pin(batch.k), pin(batch.v)
    len_h = pin(torch.tensor(batch.row_lengths, dtype=torch.int64))
    cs_h = pin(torch.tensor(batch.cand_start, dtype=torch.int64))
    out_hs = [torch.empty(T, H, d, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h, len_h, cs_h))
    d2h = out_hs[0].numel() * out_hs[0].element_size()
    bufs = [dict(q=q, k=k, v=v, lengths=lengths, cs=cand_start, off=offsets, out=out, ws=ws)]
    bufs.append(dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
                     lengths=torch.empty_like(lengths), cs=torch.empty_like(cand_start),
                     off=torch.empty_like(offsets), out=torch.empty_like(out),
                     ws=torch.empty_like(ws)))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n_steps):
        ev_in = [torch.cuda.Event() for _ in range(n_steps)]
        ev_c = [torch.cuda.Event() for _ in range(n_steps)]
        ev_out = [torch.cuda.Event() for _ in range(n_steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(n_steps):
            b = bufs[i & 1]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_c[i - 2])       # step i - 2 has finished reading b
                for dst, src in ((b["q"], q_h), (b["k"], k_h), (b["v"], v_h),
                                 (b["lengths"], len_h), (b["cs"], cs_h)):
                    dst.copy_(src, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])       # b's previous output has been read back
            jca.jca_offsets_from_lengths(b["lengths"], b["off"], status, stream)
            jca.jagged_cand_attn_plan(b["off"], b["cs"], None, T, H, d, b["ws"], status, stream)
            jca.jagged_cand_attn_run(b["q"], b["k"], b["v"], b["out"], None, B, b["ws"], status,
                                     stream=stream)
            ev_c[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[i])
                out_hs[i & 1].copy_(b["out"], non_blocking=True)
                ev_out[i].record(s_out)
        s_in.wait_stream(s_out)
        s_in.wait_stream(stream)
        t1.record(s_in)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1)

    e2e_run(2)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks([e2e_run(e2e_steps)], dist, dev)[0]
    jca.check_status(status, "end-to-end")
    assert torch.equal(out_hs[(e2e_steps - 1) & 1], out.cpu()), "end-to-end output differs"
    e2e_value = job_flops * e2e_steps / (e2e_ms / 1e3) / 1e12

    # Per GPU: this rank's work over its own kernel time (replicas), or the job's average work per
    # rank over the slowest rank's kernel time (users split over the ranks).
    achieved = (flops if shard_info is None else job_flops / world) / (kernel_ms / 1e3) / 1e12
    roofline = {
        "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
        "frac": achieved / peaks["bf16_tflops"],
        "traffic": profiled_traffic("attn_users256_d128") if shard_info is None else None,
        "kernel": "jagged_attn_kernel<128>", "kernel_ms": kernel_ms,
        "peak_source": f"{peaks['source']} bf16_tflops (burst)",
        "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
        "algorithmic_flops_per_launch": flops,
        "algorithmic_bytes_per_launch": metrics.full_attention_bytes(T, H, d),
    }

    if shard_info is None:
        workload = WORKLOAD
        parallelism = f"dp{world}: one batch per rank (replicas), no collective"
    else:
        workload = (f"users{shard_info['global_users']}: {shard_info['global_users']} users drawn "
                    "like users256 (lognormal histories, median 280, clipped to [0, 4096], 4 prefix"
                    " + 64 candidates, H=8, d_head=128, per-user seeded bf16 N(0,1))")
        parallelism = (f"dp{world}: the batch's users split over the ranks (LPT over tile cost), "
                       "outputs stay sharded, no collective")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": scaling, "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload, "rows": T, "valid_tokens": valid_tokens,
                   "allowed_pairs": pairs, "effective_flops_per_step": flops,
                   "job_effective_flops_per_step": job_flops,
                   "l2": "inputs (Q/K/V 837 MB) larger than L2 (126 MB); no flush",
                   "step": ("one CUDA graph of the four launches per step, replayed"
                            if not args.no_graph else "four launches per step"),
                   "parallelism": parallelism},
        "tokens_per_s": job_tokens * args.steps / (elapsed_ms / 1e3),
        "pct_of_bf16_peak": 100.0 * value / (world * peaks["bf16_tflops"]),
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "ms_per_step": e2e_ms / e2e_steps},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": sampler.summary(),
    }
    if shard_info is not None:
        line["config"]["shard"] = shard_info
    del q_h, k_h, v_h, out_hs, bufs

    if rank == 0 and world == 1 and not args.no_extras:
        line["cand_only"] = run_cand_only_extras(args, dev, stream, peaks)
        line["rope"] = run_rope_extras(args, dev, stream, peaks)
        line["stack"] = run_stack_extras(args, dev, stream, peaks)
        line["backward"] = run_backward_extras(args, dev, stream, peaks)
        line["seqpack"] = run_seqpack_extras(args, dev, stream, peaks)
        line["causal"] = run_causal_extras(args, dev, stream, peaks)
        line["ug_sep"] = run_ug_extras(args, dev, stream, peaks)
        line["configs"] = run_config_block(args, dev, stream, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        users = oracle_sample_users(batch, args.cpu_sample_stride, 3)
        fl, tok, times = time_oracle(batch, users, repeats=1)
        line["cpu_baseline"] = {
            "value": fl / times[0] / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle", "seconds": times[0],
            "sample": (f"users with index = 3 mod {args.cpu_sample_stride} ({len(users)} of 256,"
                       f" {tok} rows, {fl / 1e9:.1f} effective GFLOP), fp64 numpy, one pass")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def time_calls(fn, stream, dev, n: int, flush=None, warmup: int = 10):
    """Per-call device times (ms) of `fn` on `stream`, each bracketed by its own CUDA events; with
    `flush`, the L2 is overwritten before every call (outside the events)."""
    import torch
    for _ in range(warmup):
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    torch.cuda.synchronize(dev)
    for a, b in ev:
        if flush is not None:
            flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize(dev)
    return [a.elapsed_time(b) for a, b in ev]


def run_config_block(args, dev, stream, peaks):
    """Every workload of the benchmark's configuration list, each through its public entry point
    (plan + attention kernel per call, as a caller runs it): the median device time of 50 calls
    with the L2 flushed before each call (a 512 MB write) and of 50 back-to-back calls (warm L2),
    the effective TFLOP/s, the roofline fraction of the bound that applies, and the CPU oracle
    timed on the host cores on a stated sample of the same workload."""
    import torch
    import oracle
    import synth
    from candidate_isolated_jagged_b200 import jca, metrics
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.fill_(1)

    n_calls = 50
    out = {}
    cores = blas_threads()

    def gpu_entry(fl, byts, bound, fn):
        cold = time_calls(fn, stream, dev, n_calls, flush)
        warm = time_calls(fn, stream, dev, n_calls)
        mc, mw = statistics.median(cold), statistics.median(warm)
        tf = fl / mc / 1e9
        gbs = byts / mc / 1e6
        frac = tf / peaks["bf16_tflops"] if bound == "tensor" else gbs / peaks["hbm_gbs"]
        return {"ms_cold_l2_median": mc, "ms_warm_l2_median": mw, "calls": n_calls,
                "effective_tflops_cold": tf, "effective_tflops_warm": fl / mw / 1e9,
                "algorithmic_gb_s_cold": gbs, "bound": bound, "roofline_frac_cold": frac,
                "effective_flops": fl, "algorithmic_bytes": byts}

    # ---- full op: tiny, three_users, users256 ----
    for name, make, bound, sample_users in (
            ("tiny", synth.tiny, "latency", None),
            ("three_users", synth.three_users, "latency", None),
            ("users256", synth.users256, "tensor", "every 16th user (index = 3 mod 16)")):
        b = make()
        B, T, H, d = b.B, b.T, b.H, b.d
        off_np = oracle.offsets_from_lengths(b.row_lengths)
        seg_np = oracle.segment_ids(off_np, b.cand_start, b.valid)
        q, k, v = (t.to(dev) for t in (b.q, b.k, b.v))
        off = torch.tensor(off_np, device=dev)
        cs = torch.tensor(b.cand_start, device=dev)
        seg = torch.tensor(seg_np, device=dev) if b.valid is not None else None
        o = torch.empty(T, H, d, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(jca.jca_workspace_bytes(B, T, H, d), dtype=torch.uint8, device=dev)
        st = jca.new_status(dev)
        fl = metrics.effective_flops(metrics.allowed_pairs_from_counts(b.prefix + b.hist_real,
                                                                       b.n_cand), H, d)
        byts = metrics.full_attention_bytes(T, H, d)
        entry = gpu_entry(fl, byts, bound, lambda: jca.jagged_cand_attn_fwd(
            q, k, v, o, off, None if seg is not None else cs, seg, workspace=ws, status=st,
            stream=stream))
        jca.check_status(st, name)
        users = list(range(B)) if sample_users is None else [u for u in range(B) if u % 16 == 3]
        ofl = metrics.effective_flops(metrics.allowed_pairs_from_counts(
            (b.prefix + b.hist_real)[users], b.n_cand[users]), H, d)
        t0 = time.perf_counter()
        oracle.jagged_cand_attn(b.q, b.k, b.v, off_np, seg_np, b.scale, users=users)
        osec = time.perf_counter() - t0
        entry["oracle"] = {"seconds": osec, "effective_tflops": ofl / osec / 1e12, "cores": cores,
                           "sample": "whole workload" if sample_users is None else
                           f"{sample_users}: {len(users)} of {B} users, {ofl / 1e9:.1f} GFLOP"}
        out[name] = entry
        del q, k, v, o, ws

    # ---- candidate-only: cand_only256, retrieval ----
    for name, make, per_user in (("cand_only256", synth.cand_only256, 64),
                                 ("retrieval", synth.retrieval, 500)):
        cb = make()
        coff_np = oracle.offsets_from_lengths(cb.cand_counts)
        hoff_np = oracle.offsets_from_lengths(cb.hist_lengths)
        coff, hoff = torch.tensor(coff_np, device=dev), torch.tensor(hoff_np, device=dev)
        cq, ck, cv, hk, hv = (t.to(dev) for t in (cb.cq, cb.ck, cb.cv, cb.hk, cb.hv))
        o = torch.empty(cq.shape, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(jca.jca_workspace_bytes(cb.B, cb.Nc, cb.H, cb.d), dtype=torch.uint8,
                         device=dev)
        st = jca.new_status(dev)
        pairs = int(np.sum(cb.cand_counts * (cb.hist_lengths + 1)))
        fl = metrics.effective_flops(pairs, cb.H, cb.d)
        byts = metrics.cand_only_bytes(cb.Nc, cb.Th, cb.H, cb.d)
        entry = gpu_entry(fl, byts, "hbm", lambda: jca.cand_only_attn_fwd(
            cq, ck, cv, coff, hk, hv, hoff, o, None, workspace=ws, status=st, stream=stream))
        jca.check_status(st, name)
        # oracle: the first `per_user` candidates of every 8th user (request)
        users = list(range(0, cb.B, 8)) if cb.B > 2 else list(range(cb.B))
        rows = np.concatenate([np.arange(coff_np[u], coff_np[u] + min(per_user, cb.cand_counts[u]))
                               for u in users])
        ucount = np.array([min(per_user, cb.cand_counts[u]) for u in users])
        ofl = metrics.effective_flops(int(np.sum(ucount * (cb.hist_lengths[users] + 1))), cb.H,
                                      cb.d)
        t0 = time.perf_counter()
        oracle.cand_only_attn(cb.cq, cb.ck, cb.cv, coff_np, cb.hk, cb.hv, hoff_np, None, cb.scale,
                              cand_rows=rows)
        osec = time.perf_counter() - t0
        entry["oracle"] = {"seconds": osec, "effective_tflops": ofl / osec / 1e12, "cores": cores,
                           "candidates_per_s": rows.size / osec,
                           "sample": f"the first {per_user} candidates of every 8th user or "
                                     f"request ({len(users)} of {cb.B}, {rows.size} candidates)"}
        out[name] = entry
        del cq, ck, cv, hk, hv, o, ws
    del flush_buf
    torch.cuda.empty_cache()
    return out


def run_rope_extras(args, dev, stream, peaks):
    """Right-anchored RoPE on the 256-user workload's queries and keys: positions, then the
    rotation of each tensor in place. The rotation reads and writes the tensor once (HBM-bound);
    reported: kernel time per tensor and algorithmic GB/s against the measured copy bandwidth."""
    import torch
    import oracle
    import synth
    from candidate_isolated_jagged_b200 import jca
    b = synth.users256()
    off_np = oracle.offsets_from_lengths(b.row_lengths)
    seg = torch.tensor(oracle.segment_ids(off_np, b.cand_start), device=dev)
    off = torch.tensor(off_np, device=dev)
    q, k = b.q.to(dev), b.k.to(dev)
    pos = torch.empty(b.T, dtype=torch.int32, device=dev)
    st = jca.new_status(dev)
    for _ in range(3):
        jca.jca_rope_positions(seg, off, pos, 4096, st, stream=stream)
        jca.jca_apply_rope(q, q, pos, stream=stream)
    n = max(10, min(args.steps, 50))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    torch.cuda.synchronize(dev)
    ev[0].record(stream)
    for _ in range(n):
        jca.jca_rope_positions(seg, off, pos, 4096, st, stream=stream)
    ev[1].record(stream)
    for _ in range(n):
        jca.jca_apply_rope(q, q, pos, stream=stream)
        jca.jca_apply_rope(k, k, pos, stream=stream)
    ev[2].record(stream)
    torch.cuda.synchronize(dev)
    jca.check_status(st, "rope")
    pos_ms = ev[0].elapsed_time(ev[1]) / n
    rot_ms = ev[1].elapsed_time(ev[2]) / (2 * n)
    byts = 2 * q.numel() * 2   # one bf16 read and one bf16 write per element
    # Attention with RoPE: in-kernel rotation (one call) against the pre-pass path (positions, two
    # rotations, attention) and against attention without RoPE, each per call with its plan.
    q0, k0 = b.q.to(dev), b.k.to(dev)
    v0 = b.v.to(dev)
    cs = torch.tensor(b.cand_start, device=dev)
    out = torch.empty_like(q0)
    wsr = torch.empty(jca.jca_rope_attn_workspace_bytes(b.B, b.T, b.H, b.d), dtype=torch.uint8,
                      device=dev)
    wsa = torch.empty(jca.jca_workspace_bytes(b.B, b.T, b.H, b.d), dtype=torch.uint8, device=dev)
    qr, kr = torch.empty_like(q0), torch.empty_like(k0)

    def fused():
        jca.jagged_cand_attn_rope_fwd(q0, k0, v0, out, off, cs, None, history_end=4096,
                                      workspace=wsr, status=st, stream=stream)

    def prepass():
        jca.jca_rope_positions(seg, off, pos, 4096, st, stream=stream)
        jca.jca_apply_rope(q0, qr, pos, stream=stream)
        jca.jca_apply_rope(k0, kr, pos, stream=stream)
        jca.jagged_cand_attn_fwd(qr, kr, v0, out, off, cs, None, workspace=wsa, status=st,
                                 stream=stream)

    def plain():
        jca.jagged_cand_attn_fwd(q0, k0, v0, out, off, cs, None, workspace=wsa, status=st,
                                 stream=stream)

    times = {}
    for name, fn in (("plain", plain), ("fused", fused), ("prepass", prepass)):
        times[name] = statistics.median(time_calls(fn, stream, dev, 30))
    jca.check_status(st, "rope attention")
    res = {
        "workload": "users256 queries and keys (T=%d, H=%d, d=%d), history_end 4096" % (b.T, b.H, b.d),
        "positions_ms": pos_ms,
        "rotate_ms_per_tensor": rot_ms,
        "roofline": {"bound": "hbm", "achieved": byts / rot_ms / 1e6, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": byts / rot_ms / 1e6 / peaks["hbm_gbs"],
                     "algorithmic_bytes_per_launch": byts},
        "launches_timed": 3 * n,
        "attention_with_rope": {
            "workload": "users256, history_end 4096; median of 30 calls each, plan included",
            "fused_ms": times["fused"], "prepass_path_ms": times["prepass"],
            "no_rope_ms": times["plain"],
            "fused_over_no_rope": times["fused"] / times["plain"],
            "prepass_over_no_rope": times["prepass"] / times["plain"]},
    }
    del q, k, q0, k0, v0, out, wsr, wsa, qr, kr
    torch.cuda.empty_cache()
    return res


def run_causal_extras(args, dev, stream, peaks):
    """The per-user causal variant on the 256-user row lengths (4 prefix + history + 64
    candidates per user as one causal sequence each), H = 8, d = 128: queue builder plus attention
    kernel per call, timed with CUDA events; effective FLOPs = 4 d H per allowed pair,
    L (L + 1) / 2 pairs per user."""
    import torch
    import synth
    from candidate_isolated_jagged_b200 import jca, metrics
    n = synth.users256_history_lengths(0)
    b = synth.custom_batch(n + 68, prefix=0, n_cand=0, H=8, d=128, seed=0, name="users256_causal")
    B, T, H, d = b.B, b.T, b.H, b.d
    lengths = b.row_lengths.astype(np.int64)
    pairs = int((lengths * (lengths + 1) // 2).sum())
    flops = metrics.effective_flops(pairs, H, d)
    q, k, v = (t.to(dev) for t in (b.q, b.k, b.v))
    off = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int64, device=dev)
    out = torch.empty_like(q)
    ws = torch.empty(jca.jca_workspace_bytes(B, T, H, d), dtype=torch.uint8, device=dev)
    st = jca.new_status(dev)
    for _ in range(max(3, args.warmup)):
        jca.jagged_causal_attn_fwd(q, k, v, out, off, workspace=ws, status=st, stream=stream)
    n_it = max(10, min(args.steps, 100))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(n_it):
        jca.jagged_causal_attn_fwd(q, k, v, out, off, workspace=ws, status=st, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    jca.check_status(st, "causal")
    ms = e0.elapsed_time(e1) / n_it
    res = {"workload": "users256 row lengths as causal sequences (T=%d, H=%d, d=%d)" % (T, H, d),
           "ms": ms, "effective_tflops": flops / ms / 1e9,
           "pct_of_bf16_peak": 100 * flops / ms / 1e9 / peaks["bf16_tflops"],
           "allowed_pairs": pairs, "launches_per_call": 2, "launches_timed": 2 * n_it}
    del q, k, v, out, ws
    torch.cuda.empty_cache()
    return res


def run_ug_extras(args, dev, stream, peaks):
    """UG-Sep's masked cross-attention (the separated residual of a pyramid TokenMixer) on 16,384
    samples: 32 input tokens (16 U + 16 G) to 16 outputs (8 U + 8 G), one head of 128, with the
    residual added and a bf16 output. One kernel per call, timed with CUDA events over repeated
    calls; the inputs (about 460 MB) exceed L2. The op is bound by HBM: algorithmic bytes = Q, K,
    V and the residual read once plus the output written once."""
    import torch
    import synth
    from candidate_isolated_jagged_b200 import jca
    b = synth.ug_sep16k()
    B, To, Ti, H, d = b.B, b.T_out, b.T_in, b.H, b.d
    pairs_per_sample = b.c_u * b.n_u + (To - b.c_u) * Ti
    flops = 4.0 * d * H * pairs_per_sample * B
    byts = 2.0 * H * d * B * (3 * To + 2 * Ti)
    q, k, v, res = (t.to(dev) for t in (b.q, b.k, b.v, b.residual))
    out = torch.empty_like(q)
    st = jca.new_status(dev)
    for _ in range(max(3, args.warmup)):
        jca.ug_masked_cross_attn_fwd(q, k, v, out, b.c_u, b.n_u, residual=res, status=st,
                                     stream=stream)
    n_it = max(10, min(args.steps, 200))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(n_it):
        jca.ug_masked_cross_attn_fwd(q, k, v, out, b.c_u, b.n_u, residual=res, status=st,
                                     stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    jca.check_status(st, "ug")
    ms = e0.elapsed_time(e1) / n_it
    result = {
        "workload": "ug_sep16k: B=%d samples, T_in=%d (n=%d U), T_out=%d (c_u=%d U), H=%d, d=%d, "
                    "residual, bf16 out" % (B, Ti, b.n_u, To, b.c_u, H, d),
        "ms": ms, "samples_per_s": B / ms * 1e3, "effective_tflops": flops / ms / 1e9,
        "roofline": {"bound": "hbm", "achieved": byts / ms / 1e6, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": byts / ms / 1e6 / peaks["hbm_gbs"],
                     "algorithmic_bytes": byts},
        "launches_timed": n_it}
    del q, k, v, res, out
    torch.cuda.empty_cache()
    return result


def run_backward_extras(args, dev, stream, peaks):
    """The training path on the 256-user workload: the forward with its log-sum-exp, then the
    backward pass (plan, key-tile queue, row statistics, the dK/dV kernel and the dQ kernel), each
    timed with CUDA events over repeated calls. Effective backward FLOPs follow the usual
    flash-attention count, 2.5x the forward's (five d-deep products per allowed pair: the score,
    dP, dV, dK and dQ); the kernels here recompute the score and dP once more (seven products)."""
    import torch
    import synth
    from candidate_isolated_jagged_b200 import jca, metrics
    n_users = getattr(args, "users", 256)
    if n_users >= 256:
        b = synth.users256()
    else:   # the first n_users users of the same workload (smaller profiling captures)
        b = synth.custom_batch(synth.users256_history_lengths(0)[:n_users], prefix=4, n_cand=64,
                               H=8, d=128, seed=0, name="users256_head")
    B, T, H, d = b.B, b.T, b.H, b.d
    pairs = metrics.allowed_pairs_from_counts(b.prefix + b.hist_real, b.n_cand)
    fwd_flops = metrics.effective_flops(pairs, H, d)
    q, k, v = (t.to(dev) for t in (b.q, b.k, b.v))
    dout = synth.upstream_grad(b.q.shape, 15).to(dev)
    off = torch.tensor(np.concatenate([[0], np.cumsum(b.row_lengths)]), dtype=torch.int64,
                       device=dev)
    cs = torch.tensor(b.cand_start, dtype=torch.int64, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(T, H, dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    wsf = torch.empty(jca.jca_workspace_bytes(B, T, H, d), dtype=torch.uint8, device=dev)
    wsb = torch.empty(jca.jca_bwd_workspace_bytes(B, T, H, d), dtype=torch.uint8, device=dev)
    st = jca.new_status(dev)

    def fwd():
        jca.jagged_cand_attn_fwd_lse(q, k, v, out, lse, off, cs, None, workspace=wsf, status=st,
                                     stream=stream)

    def bwd():
        jca.jagged_cand_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, off, cs, None,
                                 workspace=wsb, status=st, stream=stream)

    for _ in range(max(3, args.warmup)):
        fwd()
        bwd()
    n = max(1, min(args.steps, 20))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    torch.cuda.synchronize(dev)
    ev[0].record(stream)
    for _ in range(n):
        fwd()
    ev[1].record(stream)
    for _ in range(n):
        bwd()
    ev[2].record(stream)
    torch.cuda.synchronize(dev)
    jca.check_status(st, "backward")
    f_ms = ev[0].elapsed_time(ev[1]) / n
    b_ms = ev[1].elapsed_time(ev[2]) / n
    bwd_flops = 2.5 * fwd_flops
    res = {
        "workload": "%s (%d users, T=%d, H=%d, d=%d), dO ~ N(0,1) seed 15, bf16 gradients" % (
            b.name, B, T, H, d),
        "fwd_lse_ms": f_ms, "fwd_lse_effective_tflops": fwd_flops / f_ms / 1e9,
        "bwd_ms": b_ms, "bwd_effective_tflops": bwd_flops / b_ms / 1e9,
        "bwd_pct_of_bf16_peak": 100 * bwd_flops / b_ms / 1e9 / peaks["bf16_tflops"],
        "bwd_executed_tflops": 3.5 * fwd_flops / b_ms / 1e9,
        "train_step_attention_ms": f_ms + b_ms,
        "launches_per_bwd": 6,
        "launches_timed": 2 * n,
    }
    del q, k, v, dout, out, lse, dq, dk, dv, wsf, wsb
    torch.cuda.empty_cache()
    return res


def run_seqpack_extras(args, dev, stream, peaks):
    """Training with candidate packing on the 256-user workload: every user's prefix + history
    first, then all candidates in one block (rows rearranged once on the host, as a data loader
    would pack them); the forward with its log-sum-exp and the backward through
    jagged_cand_attn_seqpack_fwd / _bwd, timed with CUDA events over repeated calls. FLOPs as for
    the serving-layout training path (backward: 2.5x the forward)."""
    import torch
    import synth
    from candidate_isolated_jagged_b200 import jca, metrics
    b = synth.users256()
    cs = np.asarray(b.cand_start, dtype=np.int64)
    L = np.asarray(b.row_lengths, dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(L)])
    perm = np.concatenate([np.arange(off[u], off[u] + cs[u]) for u in range(b.B)] +
                          [np.arange(off[u] + cs[u], off[u + 1]) for u in range(b.B)])
    hoff = torch.tensor(np.concatenate([[0], np.cumsum(cs)]), dtype=torch.int64, device=dev)
    coff = torch.tensor(np.concatenate([[0], np.cumsum(L - cs)]), dtype=torch.int64, device=dev)
    Th = int(cs.sum())
    p = torch.from_numpy(perm)
    q, k, v = (t[p].to(dev) for t in (b.q, b.k, b.v))
    dout = synth.upstream_grad(b.q.shape, 15)[p].to(dev)
    T, H, d = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(T, H, dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    wsf = torch.empty(jca.jca_seqpack_workspace_bytes(b.B, Th, T - Th, H, d), dtype=torch.uint8,
                      device=dev)
    wsb = torch.empty(jca.jca_seqpack_bwd_workspace_bytes(b.B, Th, T - Th, H, d),
                      dtype=torch.uint8, device=dev)
    st = jca.new_status(dev)
    fwd_flops = metrics.effective_flops(
        metrics.allowed_pairs_from_counts(b.prefix + b.hist_real, b.n_cand), H, d)

    def fwd():
        jca.jagged_cand_attn_seqpack_fwd(q, k, v, out, hoff, coff, None, lse, workspace=wsf,
                                         status=st, stream=stream, Th=Th)

    def bwd():
        jca.jagged_cand_attn_seqpack_bwd(q, k, v, out, dout, lse, dq, dk, dv, hoff, coff, None,
                                         workspace=wsb, status=st, stream=stream, Th=Th)

    for _ in range(max(3, args.warmup)):
        fwd()
        bwd()
    n = max(1, min(args.steps, 20))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    torch.cuda.synchronize(dev)
    ev[0].record(stream)
    for _ in range(n):
        fwd()
    ev[1].record(stream)
    for _ in range(n):
        bwd()
    ev[2].record(stream)
    torch.cuda.synchronize(dev)
    jca.check_status(st, "seqpack")
    f_ms = ev[0].elapsed_time(ev[1]) / n
    b_ms = ev[1].elapsed_time(ev[2]) / n
    res = {"workload": "users256 rearranged: %d history rows, then %d candidates in one block "
                       "(H=%d, d=%d), dO ~ N(0,1) seed 15" % (Th, T - Th, H, d),
           "fwd_lse_ms": f_ms, "fwd_lse_effective_tflops": fwd_flops / f_ms / 1e9,
           "bwd_ms": b_ms, "bwd_effective_tflops": 2.5 * fwd_flops / b_ms / 1e9,
           "bwd_pct_of_bf16_peak": 100 * 2.5 * fwd_flops / b_ms / 1e9 / peaks["bf16_tflops"],
           "launches_timed": 2 * n}
    del q, k, v, dout, out, lse, dq, dk, dv, wsf, wsb
    torch.cuda.empty_cache()
    return res


def run_stack_extras(args, dev, stream, peaks):
    """The layer stack on the 256-user rows: 8 layers (D = 1024, H = 8, d = 128) whose last 2 are
    candidate-only, with right-anchored RoPE, through jca_stack_fwd; and, for comparison, the same
    8 layers all run over whole rows (no candidate-only tail). Reported: ms per stack forward,
    useful TFLOP/s (projection GEMMs + effective attention FLOPs) and tokens/s."""
    import torch
    import synth
    from candidate_isolated_jagged_b200 import jca, metrics
    sb = synth.stack_users256()
    b = sb.batch
    T, D, H = b.T, sb.D, sb.H
    n1 = b.prefix + b.hist_real
    Nc, Th = int(b.n_cand.sum()), int(n1.sum())
    x = sb.x.to(dev)
    out = torch.empty_like(x)
    w = torch.stack([torch.stack(list(t)) for t in sb.weights]).to(dev)
    off = torch.tensor(np.concatenate([[0], np.cumsum(b.row_lengths)]), dtype=torch.int64,
                       device=dev)
    cs = torch.tensor(b.cand_start, dtype=torch.int64, device=dev)
    res = {"workload": ("users256 rows (T=%d, %d candidates, %d history tokens), D=%d, H=%d, "
                        "8 layers, RoPE history_end 8192" % (T, Nc, Th, D, H))}
    for name, n_co in (("cand_only_tail_2", sb.n_cand_only), ("all_full", 0)):
        ws = torch.empty(jca.jca_stack_workspace_bytes(b.B, T, Nc, Th, H, sb.d), dtype=torch.uint8,
                         device=dev)
        st = jca.new_status(dev)

        def fwd():
            jca.jca_stack_fwd(x, out, w, n_co, off, cs, None, Nc=Nc, Th=Th, H=H, history_end=8192,
                              workspace=ws, status=st, stream=stream)

        for _ in range(3):
            fwd()
        n = 10
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(n):
            fwd()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        jca.check_status(st, "stack " + name)
        ms = e0.elapsed_time(e1) / n
        fl = metrics.stack_flops(n1, b.n_cand, T, D, H, len(sb.weights), n_co)
        total = fl["gemm"] + fl["attention"]
        res[name] = {"ms": ms, "useful_tflops": total / ms / 1e9,
                     "pct_of_bf16_peak": 100 * total / ms / 1e9 / peaks["bf16_tflops"],
                     "gemm_tflop": fl["gemm"] / 1e12, "attention_tflop": fl["attention"] / 1e12,
                     "candidates_per_s": Nc / ms * 1e3, "launches_timed": n}
        del ws
    res["speedup_of_tail"] = res["all_full"]["ms"] / res["cand_only_tail_2"]["ms"]
    del x, out, w
    torch.cuda.empty_cache()
    return res


def run_cand_only_extras(args, dev, stream, peaks):
    """The candidate-only entry point on its two workloads: attention kernel time (CUDA events,
    mean over timed launches after one plan), effective TFLOP/s and algorithmic HBM GB/s."""
    import torch
    import oracle
    import synth
    from candidate_isolated_jagged_b200 import jca, metrics
    res = {}
    for name, make in (("cand_only256", synth.cand_only256), ("retrieval", synth.retrieval)):
        cb = make()
        coff = torch.tensor(oracle.offsets_from_lengths(cb.cand_counts), device=dev)
        hoff = torch.tensor(oracle.offsets_from_lengths(cb.hist_lengths), device=dev)
        cq, ck, cv, hk, hv = (t.to(dev) for t in (cb.cq, cb.ck, cb.cv, cb.hk, cb.hv))
        out = torch.empty(cq.shape, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(jca.jca_workspace_bytes(cb.B, cb.Nc, cb.H, cb.d), dtype=torch.uint8,
                         device=dev)
        st = jca.new_status(dev)
        jca.cand_only_attn_plan(coff, hoff, None, cb.Nc, cb.Th, cb.H, cb.d, ws, st, stream)
        for _ in range(max(3, args.warmup)):
            jca.cand_only_attn_run(cq, ck, cv, hk, hv, None, out, cb.B, ws, st, stream=stream)
        n = max(10, min(args.steps, 100))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(n):
            jca.cand_only_attn_run(cq, ck, cv, hk, hv, None, out, cb.B, ws, st, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        jca.check_status(st, name)
        ms = e0.elapsed_time(e1) / n
        pairs = int(np.sum(cb.cand_counts * (cb.hist_lengths + 1)))
        fl = metrics.effective_flops(pairs, cb.H, cb.d)
        byts = metrics.cand_only_bytes(cb.Nc, cb.Th, cb.H, cb.d)
        res[name] = {
            "kernel_ms": ms, "effective_tflops": fl / ms / 1e9,
            "pct_of_bf16_peak": 100 * fl / ms / 1e9 / peaks["bf16_tflops"],
            "candidates_per_s": cb.Nc / ms * 1e3,
            "roofline": {"bound": "hbm", "achieved": byts / ms / 1e6, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": byts / ms / 1e6 / peaks["hbm_gbs"],
                         "algorithmic_bytes_per_launch": byts},
            "launches_timed": n,
        }
        del cq, ck, cv, hk, hv, out, ws
        torch.cuda.empty_cache()
    return res


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-extras", action="store_true", help="skip the candidate-only workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the step's kernels one by one instead of replaying a CUDA graph")
    ap.add_argument("--cpu-sample-stride", type=int, default=4)
    ap.add_argument("--only", choices=["cand_only", "rope", "stack", "backward", "causal",
                                       "ug_sep", "configs", "seqpack"],
                    default=None,
                    help="run one extra section alone on one GPU and print its result (profiling)")
    ap.add_argument("--shard", choices=["replicas", "users"], default="replicas",
                    help="replicas: every rank runs its own 256-user batch; users: one global "
                         "batch split over the ranks by users (LPT), outputs stay sharded")
    ap.add_argument("--global-users", type=int, default=None,
                    help="--shard users: users in the global batch (default 256 per rank: weak "
                         "scaling; a fixed number makes it strong scaling)")
    ap.add_argument("--users", type=int, default=256,
                    help="--only backward: use the first N users of the 256-user workload")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.only is not None:
        import torch
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        fn = {"cand_only": run_cand_only_extras, "rope": run_rope_extras,
              "stack": run_stack_extras, "backward": run_backward_extras,
              "causal": run_causal_extras, "ug_sep": run_ug_extras,
              "configs": run_config_block, "seqpack": run_seqpack_extras}[args.only]
        print(json.dumps({args.only: fn(args, dev, torch.cuda.current_stream(dev), load_peaks())}),
              flush=True)
        return 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
