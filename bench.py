#!/usr/bin/env python
"""Throughput benchmark of the Longformer attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl b200|reference]

One step is one pass of the whole hot path (global-index compaction and mask
bitmaps, then band + global-column + global-row attention) over one batch of
synthetic inputs already resident in HBM, launched through the C ABI.  Steps
rotate over enough input sets that their total exceeds twice the L2 cache, and
run from a CUDA graph so the host does not limit the launch rate.  K timed
steps sit between a barrier plus device synchronisation on both sides; times
come from CUDA events, the maximum over ranks.  Under torchrun every rank runs
the same workload on its own GPU (independent (batch, head) work, no
collective on the data path: weak scaling).

Printed (rank 0, one JSON line): useful band+global TFLOP/s of the whole job,
tokens/s, the roofline of the attention kernel against the measured HBM peak,
the CPU oracle timed on this host, an end-to-end figure through the host-buffer
entry point, clocks sampled around the timed region.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "useful band+global attention TFLOP/s & tokens/s at n=4096,w=512 bf16, 1 B200"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# Kernel sources whose change invalidates a stored DRAM-traffic figure.
TRAFFIC_SOURCES = {
    "attn_fwd_kernel": ("lf_fwd.cu", "lf_sm100.cuh", "lf_device.cuh"),
    "attn_f32_kernel": ("lf_simt.cu", "lf_device.cuh"),
    "proj_kernel": ("lf_proj.cu", "lf_sm100.cuh", "lf_device.cuh"),
}


def kernel_source_digest(kernel: str) -> str:
    h = hashlib.sha256()
    for name in TRAFFIC_SOURCES[kernel]:
        with open(os.path.join(ROOT, "sparse_long_sequence_lf_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from a committed ncu
    capture (profiles/dram_traffic.json), or None when there is none or the
    kernel sources changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f).get(kernel, {}).get(workload)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("sources_sha256") != kernel_source_digest(kernel):
        return None
    return int(rec["dram_bytes_per_launch"])


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(value: float, device) -> float:
    """Maximum of a float over all ranks (identity on one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank: float, steps: int, world: int, max_ms: float) -> float:
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    return units_per_step_per_rank * steps * world / (max_ms * 1e-3)


class ClockSampler:
    """Samples SM clock, max clock and clock-event reasons through NVML."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.error = None
        self.max_mhz = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.h = None
            try:
                props = torch.cuda.get_device_properties(device_index)
                bus = "%08x:%02x:%02x.0" % (getattr(props, "pci_domain_id", 0),
                                             props.pci_bus_id, props.pci_device_id)
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
                self.bus = bus
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
                self.bus = f"index {device_index}"
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception as e:  # NVML missing: report, do not guess
            self.error = f"nvml unavailable: {e.__class__.__name__}"

    def _run(self):
        while not self._stop.is_set():
            try:
                sm = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = int(self._reasons(self.h))
                self.samples.append((sm, rs))
            except Exception as e:
                self.error = f"nvml sample failed: {e.__class__.__name__}"
                return
            time.sleep(self.period)

    def __enter__(self):
        if self.error is None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self, window: str):
        if self.error is not None and not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "error": self.error}
        loaded = [s for s in self.samples if not (s[1] & 0x1)] or self.samples
        reasons = set()
        for _, rs in loaded:
            for bit, name in self.REASONS.items():
                if rs & bit and bit != 0x1:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[0] for s in loaded), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(loaded), "window": window}


# --------------------------------------------------------------- GPU arm
def make_device_sets(wl, nsets, device, heads=None):
    """`nsets` input sets of the workload on the device; with heads=(h0, h1)
    only those heads of each full set (one problem split by heads)."""
    import torch
    from sparse_long_sequence_lf_b200.sharding import shard_inputs
    from sparse_long_sequence_lf_b200.workloads import make_inputs
    sets = []
    for s in range(nsets):
        x = make_inputs(wl, seed=wl.seed + 7919 * s)
        if heads is not None:
            x = shard_inputs(x, *heads)
        sets.append({k: (v.to(device) if torch.is_tensor(v) else v) for k, v in x.items()})
    return sets


def launches_per_step(wl, max_global):
    # prepare kernel + attention kernel; with global tokens fp32 adds its
    # global-row kernel, bf16/fp16 merge them inside the attention kernel up to
    # 8 chunks of 512 keys and add the merge kernel beyond
    if max_global == 0:
        return 2
    if wl.dtype == "f32":
        return 3
    return 2 if -(-wl.n // 512) <= 8 else 3


def run_gpu_arm(args, wl, world, rank, local):
    import torch
    import sparse_long_sequence_lf_b200 as lf
    from sparse_long_sequence_lf_b200 import accounting

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")

    # --shard heads: the ranks split one problem by heads (strong scaling);
    # otherwise every rank runs the whole workload (weak scaling).
    wl_full, heads, ranges = wl, None, None
    if args.shard == "heads" and world > 1:
        from sparse_long_sequence_lf_b200.sharding import head_ranges
        ranges = head_ranges(wl.H, world)
        heads = ranges[rank]
        wl = wl.with_(H=heads[1] - heads[0],
                      dilation=tuple(wl.dilation_list()[heads[0]:heads[1]]))
    x0 = make_device_sets(wl_full, 1, device, heads)[0]
    per_set = sum(t.numel() * t.element_size() for t in x0.values() if torch.is_tensor(t))
    per_set += x0["q"].numel() * x0["q"].element_size()          # output
    nsets = max(2, -(-2 * L2_BYTES // per_set))
    sets = [x0] + make_device_sets(wl_full.with_(seed=wl_full.seed + 1), nsets - 1, device, heads)
    outs = [torch.empty_like(s["q"]) for s in sets]
    max_global = max(int((s["global_mask"] != 0).sum(1).max()) if s["global_mask"] is not None
                     else 0 for s in sets)
    ws = lf.new_workspace(wl.B, wl.H, wl.n, max_global, device)
    stream = torch.cuda.Stream(device)

    def step(i):
        s = sets[i % nsets]
        lf.attention_forward(s["q"], s["k"], s["v"], s["qg"], s["kg"], s["vg"],
                             s["local_mask"], s["global_mask"], window=wl.window,
                             dilation=s["dilation"], causal=wl.causal, max_global=max_global,
                             out=outs[i % nsets], workspace=ws)

    def run_only(i):
        s = sets[i % nsets]
        lf.attention_run(s["q"], s["k"], s["v"], s["qg"], s["kg"], s["vg"], window=wl.window,
                         dilation=s["dilation"], causal=wl.causal, max_global=max_global,
                         out=outs[i % nsets], workspace=ws)

    def capture(fn, count, offset=0):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(count):
                fn(offset + i)
        return g

    # Eager warm-up (also builds the tensor-map cache), then the graphs.
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 1)):
            step(i)
    stream.synchronize()
    status = lf.workspace_status(ws, stream)
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    chunk = nsets * max(1, 64 // nsets)
    n_chunk = min(chunk, args.steps)           # steps in one replay of g_chunk
    g_chunk = capture(step, n_chunk)
    full, rem = divmod(args.steps, chunk) if args.steps >= chunk else (0, args.steps)
    g_rem = capture(step, rem) if (rem and full) else None
    if full == 0:
        g_chunk, full, g_rem = g_chunk, 1, None

    # Graphs replay on `stream`, the stream the CUDA events are recorded on.
    def replay(g):
        with torch.cuda.stream(stream):
            g.replay()

    def timed_steps():
        for _ in range(full):
            replay(g_chunk)
        if g_rem is not None:
            replay(g_rem)

    # Graph warm-up (W steps' worth, at least one replay).
    for _ in range(max(1, -(-args.warmup // chunk))):
        replay(g_chunk)
    stream.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        t_pad = time.time()
        while time.time() - t_pad < 0.5:           # same work before the timed region
            replay(g_chunk)
            stream.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        start.record(stream)
        timed_steps()
        end.record(stream)
        torch.cuda.synchronize(device)
        if world > 1:
            dist.barrier()
        t_pad = time.time()
        while time.time() - t_pad < 0.5:           # and after it
            replay(g_chunk)
            stream.synchronize()
    local_ms = start.elapsed_time(end)
    max_ms = reduce_max(local_ms, device)
    clocks = sampler.summary("timed region plus 0.5 s of the same graph on each side")

    # Distribution of the step time: every replay of the graph timed on its
    # own (events on the launching stream), at least 50 replays.
    step_dist = replay_distribution(replay, g_chunk, n_chunk, stream, device, samples=50)

    status = lf.workspace_status(ws, stream)
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")

    # Attention kernel alone (the dominant kernel), same rotation, graph replay.
    g_run = capture(run_only, chunk)
    for _ in range(2):
        replay(g_run)
    stream.synchronize()
    reps = max(1, -(-args.steps // chunk))
    ks, ke = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ks.record(stream)
    for _ in range(reps):
        replay(g_run)
    ke.record(stream)
    torch.cuda.synchronize(device)
    kernel_ms = ks.elapsed_time(ke) / (reps * chunk)
    kernel_dist = replay_distribution(replay, g_run, chunk, stream, device, samples=50)

    flops = accounting.useful_flops(wl)
    bytes_ = accounting.algorithmic_bytes(wl)
    ms_per_step = max_ms / args.steps
    if heads is None:
        value = whole_job_rate(flops, args.steps, world, max_ms) / 1e12
        tokens_per_s = whole_job_rate(accounting.tokens(wl), args.steps, world, max_ms)
    else:
        # One problem over all ranks: its units over the slowest rank's time.
        value = accounting.useful_flops(wl_full) * args.steps / (max_ms * 1e-3) / 1e12
        tokens_per_s = accounting.tokens(wl_full) * args.steps / (max_ms * 1e-3)
    shard_check = None
    if heads is not None:
        shard_check = check_head_shards(wl_full, sets[0], outs[0], ranges, max_global, ws,
                                        stream, device, rank, step)

    peaks, peak_kind = load_peaks()
    achieved_gbs = bytes_ / (kernel_ms * 1e-3) / 1e9
    kernel_tflops = flops / (kernel_ms * 1e-3) / 1e12
    kname = "attn_fwd_kernel" if wl.dtype != "f32" else "attn_f32_kernel"
    roofline = {
        "kernel": kname,
        "bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": peaks["hbm_gbs"],
        "unit": "GB/s", "frac": round(achieved_gbs / peaks["hbm_gbs"], 4),
        "traffic": stored_traffic(kname, wl.name) if heads is None else None,
        "peak_source": peak_kind,
        "kernel_us": round(kernel_ms * 1e3, 3), "algorithmic_bytes": bytes_,
        "useful_tflops": round(kernel_tflops, 1),
        "tensor_frac_of_measured_bf16": round(kernel_tflops / peaks["bf16_tflops"], 4),
        "kernel_us_dist": {k: (round(v * 1e3, 3) if k != "samples" else v)
                           for k, v in kernel_dist.items()},
    }

    if world > 1:
        dist.barrier()
    e2e = run_e2e(args, wl, device, stream, max_global)
    e2e_max_ms = reduce_max(e2e["ms_per_step"], device)
    e2e["value"] = round((whole_job_rate(flops, 1, world, e2e_max_ms) if heads is None else
                          accounting.useful_flops(wl_full) / (e2e_max_ms * 1e-3)) / 1e12, 4)
    e2e["ms_per_step"] = round(e2e_max_ms, 4)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_cpu_baseline(wl, budget_s=args.cpu_seconds)

    result = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True, "scaling": "weak" if heads is None else "strong",
        "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "tokens_per_s": round(tokens_per_s, 1),
        "config": workload_config(wl_full, world, heads_split=heads is not None),
        "timing": {"l2": f"{nsets} rotating input sets, {nsets * per_set / 2**20:.0f} MiB > 2x L2",
                   "launch": "CUDA graph of C-ABI calls",
                   "useful_gflop_per_step": round(flops / 1e9, 4),
                   "algorithmic_mb_per_step": round(bytes_ / 1e6, 3),
                   "step_ms_dist": step_dist},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step(wl, max_global) * args.steps,
        "clocks": clocks,
    }
    if shard_check is not None:
        result["shard_check"] = shard_check
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        del g_chunk, g_rem, g_run
        dist.destroy_process_group()


def replay_distribution(replay, graph, steps_per_replay, stream, device, samples=50):
    """Per-step time of `samples` replays of `graph`, each timed alone with
    CUDA events on `stream`: median, min and 90th percentile in ms."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(samples)]
    for a, b in evs:
        a.record(stream)
        replay(graph)
        b.record(stream)
    torch.cuda.synchronize(device)
    per_step = sorted(a.elapsed_time(b) / steps_per_replay for a, b in evs)
    p90 = per_step[min(len(per_step) - 1, int(round(0.9 * (len(per_step) - 1))))]
    return {"median": round(statistics.median(per_step), 6), "min": round(per_step[0], 6),
            "p90": round(p90, 6), "samples": samples}


def run_e2e(args, wl, device, stream, max_global):
    """Same metric through lf_attention_forward_host: pinned host inputs are
    copied in, the forward runs, the output is copied back, every step."""
    import torch
    import sparse_long_sequence_lf_b200 as lf
    from sparse_long_sequence_lf_b200 import accounting
    from sparse_long_sequence_lf_b200.workloads import make_inputs

    x = make_inputs(wl)
    pin = {k: (v.pin_memory() if torch.is_tensor(v) else v) for k, v in x.items()}
    out = torch.empty_like(pin["q"]).pin_memory()
    staging = torch.empty(lf.host_staging_size(pin["q"].dtype, wl.B, wl.H, wl.n),
                          dtype=torch.uint8, device=device)
    ws = lf.new_workspace(wl.B, wl.H, wl.n, max_global, device)

    def once():
        lf.attention_forward_host(pin["q"], pin["k"], pin["v"], pin["qg"], pin["kg"], pin["vg"],
                                  pin["local_mask"], pin["global_mask"], window=wl.window,
                                  dilation=pin["dilation"], causal=wl.causal,
                                  max_global=max_global, out=out, staging=staging,
                                  workspace=ws, stream=stream)

    for _ in range(3):
        once()
    steps = max(3, min(args.steps, args.e2e_steps))
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        once()
    e.record(stream)
    torch.cuda.synchronize(device)
    ms = s.elapsed_time(e) / steps
    # The bytes the call copies in: Q, K, V, the masks, and Kg, Vg and the
    # global rows of Qg when there are global tokens (lf_host_copy_bytes).
    h2d = lf.host_copy_bytes(pin["q"].dtype, wl.B, wl.H, wl.n, pin["local_mask"],
                             pin["global_mask"])
    d2h = out.numel() * out.element_size()
    return {"value": round(accounting.useful_flops(wl) / (ms * 1e-3) / 1e12, 4), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms, 4), "steps": steps,
            "path": "lf_attention_forward_host (pinned host buffers)"}


# ------------------------------------------------------ projection prologue
PROJ_METRIC = "projection prologue TFLOP/s (Q,K,V,Kg,Vg over all tokens, Qg over global tokens), 1 B200"


def projection_flops(wl, counts, max_global):
    hid = wl.H * wl.d
    g = sum(min(int(c), max_global) for c in counts)
    return 2.0 * wl.B * wl.n * hid * 5 * hid + 2.0 * g * hid * hid


def run_projection_arm(args, wl, world, rank, local):
    """One step = lf_qkv_projection on one batch of hidden states (the global
    index is computed once beforehand, as it is once per batch before the
    layer loop).  Tensor-bound: roofline against the measured dense peak."""
    import torch
    import sparse_long_sequence_lf_b200 as lf
    from sparse_long_sequence_lf_b200.workloads import make_layer_inputs

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    stream = torch.cuda.Stream(device)
    x0 = make_layer_inputs(wl)
    hid = wl.H * wl.d
    gm = x0["global_mask"]
    gm = (gm if gm is not None else torch.zeros((wl.B, wl.n), dtype=torch.uint8)).to(device)
    with torch.cuda.stream(stream):
        gidx, counts = lf.global_index(gm, stream=stream)
    stream.synchronize()
    max_global = int(counts.max().item())
    per_set = sum(t.numel() * t.element_size() for k, t in x0.items()
                  if torch.is_tensor(t) and k in ("x", "w", "bias", "wqg", "bqg"))
    per_set += 6 * wl.B * wl.H * wl.n * wl.d * x0["x"].element_size()
    nsets = max(2, -(-2 * L2_BYTES // per_set))
    sets = []
    for s_ in range(nsets):
        xs = make_layer_inputs(wl, seed=wl.seed + 7919 * s_) if s_ else x0
        d = {k: xs[k].to(device) for k in ("x", "w", "bias", "wqg", "bqg")}
        d["out"] = {k: torch.empty((wl.B, wl.H, wl.n, wl.d), dtype=xs["x"].dtype, device=device)
                    for k in ("q", "k", "v", "qg", "kg", "vg")}
        sets.append(d)

    def step(i):
        d = sets[i % nsets]
        lf.qkv_projection(d["x"], d["w"], d["bias"], d["wqg"], d["bqg"], gidx, counts, H=wl.H,
                          max_global=max_global, out=d["out"], stream=stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    chunk = nsets * max(1, 32 // nsets)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(chunk):
            step(i)
    reps = max(1, -(-args.steps // chunk))
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        t_pad = time.time()
        while time.time() - t_pad < 0.5:
            with torch.cuda.stream(stream):
                g.replay()
            stream.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        start.record(stream)
        for _ in range(reps):
            with torch.cuda.stream(stream):
                g.replay()
        end.record(stream)
        torch.cuda.synchronize(device)
        if world > 1:
            dist.barrier()
    steps = reps * chunk
    max_ms = reduce_max(start.elapsed_time(end), device)
    clocks = sampler.summary("timed region plus 0.5 s of the same graph before it")
    flops = projection_flops(wl, counts.cpu().tolist(), max_global)
    ms_per_step = max_ms / steps
    value = whole_job_rate(flops, steps, world, max_ms) / 1e12
    peaks, peak_kind = load_peaks()
    kernel_tflops = flops / (ms_per_step * 1e-3) / 1e12
    roofline = {"kernel": "proj_kernel", "bound": "tensor", "achieved": round(kernel_tflops, 1),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(kernel_tflops / peaks["bf16_tflops"], 4),
                "traffic": stored_traffic("proj_kernel", wl.name),
                "peak_source": peak_kind + " (bf16 dense; fp16 has the same nominal rate)"}

    # End to end: hidden states from pinned host memory in, six outputs back.
    pin_x = x0["x"].pin_memory()
    dev = sets[0]
    host_out = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in dev["out"].items()}
    xd = torch.empty_like(dev["x"])

    def e2e_once():
        with torch.cuda.stream(stream):
            xd.copy_(pin_x, non_blocking=True)
            lf.qkv_projection(xd, dev["w"], dev["bias"], dev["wqg"], dev["bqg"], gidx, counts,
                              H=wl.H, max_global=max_global, out=dev["out"], stream=stream)
            for k in host_out:
                host_out[k].copy_(dev["out"][k], non_blocking=True)
        stream.synchronize()

    for _ in range(3):
        e2e_once()
    e_steps = max(3, min(args.steps, args.e2e_steps))
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    es.record(stream)
    for _ in range(e_steps):
        e2e_once()
    ee.record(stream)
    torch.cuda.synchronize(device)
    e_ms = reduce_max(es.elapsed_time(ee) / e_steps, device)
    e2e = {"value": round(whole_job_rate(flops, 1, world, e_ms) / 1e12, 4), "unit": "TFLOP/s",
           "h2d_bytes_per_step": int(pin_x.numel() * pin_x.element_size()),
           "d2h_bytes_per_step": int(sum(t.numel() * t.element_size() for t in host_out.values())),
           "ms_per_step": round(e_ms, 4), "steps": e_steps,
           "path": "lf_qkv_projection with pinned host copies of x and the six outputs"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = run_projection_cpu_baseline(wl, counts.cpu().numpy(), gidx.cpu().numpy(),
                                          max_global, args.cpu_seconds)
    result = {
        "metric": PROJ_METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "op": "projection", "B": wl.B, "H": wl.H, "n": wl.n,
                   "hidden": hid, "global_rows": int(sum(min(int(c), max_global)
                                                         for c in counts.cpu().tolist())),
                   "global_batch": wl.B * world, "seq_len": wl.n,
                   "parallelism": f"independent replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"{nsets} rotating input sets, {nsets * per_set / 2**20:.0f} MiB > 2x L2",
                   "launch": "CUDA graph of C-ABI calls",
                   "useful_gflop_per_step": round(flops / 1e9, 4)},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": (2 if max_global > 0 else 1) * steps, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        del g
        dist.destroy_process_group()


OUT_METRIC = "output layer TFLOP/s (heads concatenated, output projection, bias, residual, LayerNorm), 1 B200"


def run_output_arm(args, wl, world, rank, local):
    """One step = lf_output_layer on one batch (GEMM 2 B n (H d)^2 FLOPs on the
    tensor cores, then a memory-bound LayerNorm).  Roofline: the step against
    the measured dense peak."""
    import torch
    import sparse_long_sequence_lf_b200 as lf
    from sparse_long_sequence_lf_b200.workloads import make_output_inputs

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    stream = torch.cuda.Stream(device)
    hid = wl.H * wl.d
    x0 = make_output_inputs(wl)
    per_set = sum(t.numel() * t.element_size() for t in x0.values())
    per_set += wl.B * wl.n * hid * (x0["attn"].element_size() + 4)
    nsets = max(2, -(-2 * L2_BYTES // per_set))
    ws = torch.empty(lf.output_workspace_size(wl.B, wl.n, wl.H), dtype=torch.uint8,
                     device=device)
    sets = []
    for s_ in range(nsets):
        xs = make_output_inputs(wl, seed=wl.seed + 7919 * s_) if s_ else x0
        d = {k: v.to(device) for k, v in xs.items()}
        d["out"] = torch.empty_like(d["residual"])
        sets.append(d)

    def step(i):
        d = sets[i % nsets]
        lf.output_layer(d["attn"], d["wo"], d["bo"], d["residual"], d["gamma"], d["beta"],
                        out=d["out"], workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    chunk = nsets * max(1, 32 // nsets)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(chunk):
            step(i)
    reps = max(1, -(-args.steps // chunk))
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        t_pad = time.time()
        while time.time() - t_pad < 0.5:
            with torch.cuda.stream(stream):
                g.replay()
            stream.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        start.record(stream)
        for _ in range(reps):
            with torch.cuda.stream(stream):
                g.replay()
        end.record(stream)
        torch.cuda.synchronize(device)
        if world > 1:
            dist.barrier()
    steps = reps * chunk
    max_ms = reduce_max(start.elapsed_time(end), device)
    clocks = sampler.summary("timed region plus 0.5 s of the same graph before it")
    flops = 2.0 * wl.B * wl.n * hid * hid
    ms_per_step = max_ms / steps
    value = whole_job_rate(flops, steps, world, max_ms) / 1e12
    peaks, peak_kind = load_peaks()
    tflops = flops / (ms_per_step * 1e-3) / 1e12
    roofline = {"kernel": "proj_kernel (residual mode) + layernorm_kernel", "bound": "tensor",
                "achieved": round(tflops, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(tflops / peaks["bf16_tflops"], 4), "traffic": None,
                "peak_source": peak_kind + " (bf16 dense; fp16 has the same nominal rate)"}

    # End to end: attention output and residual from pinned host memory in, the
    # normalised rows back.
    dev = sets[0]
    pin = {k: x0[k].pin_memory() for k in ("attn", "residual")}
    host_out = torch.empty_like(x0["residual"]).pin_memory()
    da, dr = torch.empty_like(dev["attn"]), torch.empty_like(dev["residual"])

    def e2e_once():
        with torch.cuda.stream(stream):
            da.copy_(pin["attn"], non_blocking=True)
            dr.copy_(pin["residual"], non_blocking=True)
            lf.output_layer(da, dev["wo"], dev["bo"], dr, dev["gamma"], dev["beta"],
                            out=dev["out"], workspace=ws, stream=stream)
            host_out.copy_(dev["out"], non_blocking=True)
        stream.synchronize()

    for _ in range(3):
        e2e_once()
    e_steps = max(3, min(args.steps, args.e2e_steps))
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    es.record(stream)
    for _ in range(e_steps):
        e2e_once()
    ee.record(stream)
    torch.cuda.synchronize(device)
    e_ms = reduce_max(es.elapsed_time(ee) / e_steps, device)
    e2e = {"value": round(whole_job_rate(flops, 1, world, e_ms) / 1e12, 4), "unit": "TFLOP/s",
           "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in pin.values())),
           "d2h_bytes_per_step": int(host_out.numel() * host_out.element_size()),
           "ms_per_step": round(e_ms, 4), "steps": e_steps,
           "path": "lf_output_layer with pinned host copies of attn, residual and the output"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import os
        import numpy as np
        from oracle.projection import output_layer as oracle_output_layer
        f = lambda t: t.double().numpy()
        rows = min(wl.n, 256)
        X = {k: f(v) for k, v in x0.items()}
        reps_, t0 = 0, time.perf_counter()
        while True:
            oracle_output_layer(X["attn"][:1, :, :rows], X["wo"], X["bo"], X["residual"][:1, :rows],
                                X["gamma"], X["beta"])
            reps_ += 1
            dt = time.perf_counter() - t0
            if dt > args.cpu_seconds or reps_ >= 1000:
                break
        cflops = 2.0 * rows * hid * hid
        cpu = {"value": round(cflops * reps_ / dt / 1e12, 6), "unit": "TFLOP/s",
               "cores": os.cpu_count(), "kind": "oracle",
               "sample": f"first {rows} tokens of batch 0, {reps_} repetition(s), {dt:.1f} s, "
                         "fp64 numpy oracle (BLAS threads)", "seconds": round(dt, 2)}
    result = {
        "metric": OUT_METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "op": "output", "B": wl.B, "H": wl.H, "n": wl.n,
                   "hidden": hid, "eps": 1e-5, "global_batch": wl.B * world, "seq_len": wl.n,
                   "parallelism": f"independent replicas x{world}" if world > 1 else "single GPU",
                   "l2": f"{nsets} rotating input sets, {nsets * per_set / 2**20:.0f} MiB > 2x L2",
                   "launch": "CUDA graph of C-ABI calls",
                   "useful_gflop_per_step": round(flops / 1e9, 4)},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": 2 * steps, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        del g
        dist.destroy_process_group()


BWD_METRIC = ("attention backward TFLOP/s (dq, dk, dv, dqg, dkg, dvg; 10*d flops per "
              "attended pair), 1 B200")


def run_backward_arm(args, wl, world, rank, local):
    """One step = lf_attention_backward over one batch (the forward's output
    and workspace prepared once beforehand).  The kernels run on the CUDA
    cores in fp32: the roofline is the fp32 FMA rate of the SMs at the
    sampled clock."""
    import torch
    import sparse_long_sequence_lf_b200 as lf
    from sparse_long_sequence_lf_b200 import accounting
    from sparse_long_sequence_lf_b200.workloads import make_inputs, make_output_grad

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    stream = torch.cuda.Stream(device)
    names = ("q", "k", "v", "qg", "kg", "vg")
    x0 = make_inputs(wl)
    mg = 0 if x0["global_mask"] is None else int((x0["global_mask"] != 0).sum(1).max())
    t_bytes = wl.B * wl.H * wl.n * wl.d * x0["q"].element_size()
    per_set = 14 * t_bytes
    nsets = max(2, -(-2 * L2_BYTES // per_set))
    sets = []
    with torch.cuda.stream(stream):
        for s_ in range(nsets):
            xs = make_inputs(wl, seed=wl.seed + 7919 * s_) if s_ else x0
            d = {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in xs.items()}
            d["ws"] = lf.new_workspace(wl.B, wl.H, wl.n, mg, device)
            kw = dict(window=wl.window, dilation=xs["dilation"], causal=wl.causal,
                      max_global=mg)
            # bf16 / fp16: the forward also keeps each row's log-sum-exp, which
            # the backward reads instead of recomputing (the training pair).
            d["lse"] = (torch.empty((wl.B, wl.H, wl.n), dtype=torch.float32, device=device)
                        if wl.dtype != "f32" and not args.no_lse else None)
            d["out"] = lf.attention_forward(*[d[nm] for nm in names], d["local_mask"],
                                            d["global_mask"], workspace=d["ws"], stream=stream,
                                            lse=d["lse"], **kw)
            d["dout"] = make_output_grad(wl, seed=wl.seed + 7919 * s_).to(device)
            d["grads"] = {nm: torch.empty_like(d["q"]) for nm in names}
            d["kw"] = kw
            sets.append(d)
    scratch = torch.empty(lf.backward_scratch_size(wl.B, wl.H, wl.n, mg), dtype=torch.uint8,
                          device=device)
    stream.synchronize()
    for d in sets:
        if lf.workspace_status(d["ws"]) != 0:
            raise RuntimeError("forward status not ok")

    def step(i):
        d = sets[i % nsets]
        lf.attention_backward(*[d[nm] for nm in names], d["out"], d["dout"],
                              workspace=d["ws"], grads=d["grads"], scratch=scratch,
                              lse=d["lse"], stream=stream, **d["kw"])

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    chunk = nsets * max(1, 8 // nsets)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(chunk):
            step(i)
    reps = max(1, -(-args.steps // chunk))
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        t_pad = time.time()
        while time.time() - t_pad < 0.5:
            with torch.cuda.stream(stream):
                g.replay()
            stream.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        start.record(stream)
        for _ in range(reps):
            with torch.cuda.stream(stream):
                g.replay()
        end.record(stream)
        torch.cuda.synchronize(device)
        if world > 1:
            dist.barrier()
    steps = reps * chunk
    max_ms = reduce_max(start.elapsed_time(end), device)
    clocks = sampler.summary("timed region plus 0.5 s of the same graph before it")
    flops = accounting.backward_flops(wl)
    ms_per_step = max_ms / steps
    value = whole_job_rate(flops, steps, world, max_ms) / 1e12
    tflops = flops / (ms_per_step * 1e-3) / 1e12
    if wl.dtype == "f32":
        # fp32: the CUDA-core kernels, bound by the fp32 FMA rate.
        mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965
        peak = accounting.FP32_FLOPS_PER_CLOCK * mhz * 1e6 / 1e12
        roofline = {"kernel": "bwd rows_kernel + keys_kernel (+ global-token kernels)",
                    "bound": "alu", "achieved": round(tflops, 2), "peak": round(peak, 1),
                    "unit": "TFLOP/s", "frac": round(tflops / peak, 4), "traffic": None,
                    "peak_source": f"derived: 148 SMs x 128 fp32 lanes x 2 flops x {mhz} MHz "
                                   "(median sampled SM clock)"}
    else:
        # bf16 / fp16: the tcgen05 band kernels (plus the CUDA-core global-token
        # kernels), against the measured dense tensor peak.
        peaks, peak_kind = load_peaks()
        roofline = {"kernel": "bwd_tc_kernel rows + keys sides (+ global-token kernels)",
                    "bound": "tensor", "achieved": round(tflops, 2),
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": round(tflops / peaks["bf16_tflops"], 4), "traffic": None,
                    "peak_source": peak_kind + " (bf16 dense; fp16 has the same nominal rate)"}

    # End to end through the host-buffer path: the eight inputs from pinned
    # host memory in, the six gradients back.
    dev = sets[0]
    ins = list(names) + ["out", "dout"]
    pin = {nm: (x0[nm] if nm in names else dev[nm].cpu()).pin_memory() for nm in ins}
    host_g = {nm: torch.empty_like(x0["q"]).pin_memory() for nm in names}
    stage = {nm: torch.empty_like(dev["q"]) for nm in ins}

    def e2e_once():
        with torch.cuda.stream(stream):
            for nm in ins:
                stage[nm].copy_(pin[nm], non_blocking=True)
            lf.attention_backward(*[stage[nm] for nm in names], stage["out"], stage["dout"],
                                  workspace=dev["ws"], grads=dev["grads"], scratch=scratch,
                                  stream=stream, **dev["kw"])
            for nm in names:
                host_g[nm].copy_(dev["grads"][nm], non_blocking=True)
        stream.synchronize()

    for _ in range(3):
        e2e_once()
    e_steps = max(3, min(args.steps, args.e2e_steps))
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    es.record(stream)
    for _ in range(e_steps):
        e2e_once()
    ee.record(stream)
    torch.cuda.synchronize(device)
    e_ms = reduce_max(es.elapsed_time(ee) / e_steps, device)
    e2e = {"value": round(whole_job_rate(flops, 1, world, e_ms) / 1e12, 4), "unit": "TFLOP/s",
           "h2d_bytes_per_step": 8 * t_bytes, "d2h_bytes_per_step": 6 * t_bytes,
           "ms_per_step": round(e_ms, 4), "steps": e_steps,
           "path": "lf_attention_backward with pinned host copies of the eight inputs and "
                   "the six gradients (masks prepared once)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import os
        from oracle import backward as obw
        sub = wl.with_(B=1, H=1, n=min(wl.n, 1024), pad_tail=())
        xs = make_inputs(sub)
        dsub = make_output_grad(sub)
        reps_, t0 = 0, time.perf_counter()
        while True:
            obw.backward(*[xs[nm] for nm in names], xs["local_mask"], xs["global_mask"], dsub,
                         window=sub.window, dilation=xs["dilation"], causal=sub.causal)
            reps_ += 1
            dt = time.perf_counter() - t0
            if dt > args.cpu_seconds or reps_ >= 100:
                break
        cflops = accounting.backward_flops(sub)
        cpu = {"value": round(cflops * reps_ / dt / 1e12, 6), "unit": "TFLOP/s",
               "cores": torch.get_num_threads(), "kind": "oracle",
               "sample": f"batch 0, head 0, first {sub.n} tokens, {reps_} repetition(s), "
                         f"{dt:.1f} s, fp64 dense-mask autograd oracle (torch CPU threads)",
               "seconds": round(dt, 2)}
    # rows + keys sides; with global tokens gcols, two global-row passes,
    # gfinal and gkeys
    launches = 7 if mg > 0 else 2
    result = {
        "metric": BWD_METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic",
        "config": {**workload_config(wl, world), "op": "backward",
                   "lse": "from the forward" if sets[0]["lse"] is not None else "recomputed",
                   "l2": f"{nsets} rotating input sets, {nsets * per_set / 2**20:.0f} MiB > 2x L2",
                   "launch": "CUDA graph of C-ABI calls",
                   "useful_gflop_per_step": round(flops / 1e9, 4)},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches * steps, "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        del g
        dist.destroy_process_group()


ENC_METRIC = ("Longformer encoder stack latency, ms per forward (projections, attention, "
              "output LayerNorm, GELU FFN per layer), 1 B200")
# FasterTransformer's fp16 encoder latencies on A100-80GB for this model
# (guide's benchmark table), keyed by (batch, seq_len): context, other hardware.
FT_A100_FP16_MS = {(1, 1024): 14, (1, 2048): 31, (1, 4096): 50, (8, 1024): 79, (8, 2048): 208,
                   (8, 4096): 369, (32, 1024): 305, (32, 2048): 820, (32, 4096): 823}


def encoder_flops(ew, counts):
    """Useful FLOPs of one stack forward: per layer the five projections over
    all tokens and Qg over the global rows, the attention, the output
    product and the two feed-forward products."""
    from sparse_long_sequence_lf_b200 import accounting
    wl = ew.attn
    hid = wl.H * wl.d
    tok = wl.B * wl.n
    per_layer = (2.0 * tok * hid * 5 * hid + 2.0 * sum(counts) * hid * hid
                 + accounting.useful_flops(wl) + 2.0 * tok * hid * hid
                 + 2 * 2.0 * tok * hid * ew.inter)
    return per_layer * ew.layers


def run_encoder_arm(args, ew, world, rank, local):
    """One step = one forward of the whole stack through lf_encoder_forward
    (masks prepared inside the call).  Roofline: the stack's useful FLOPs
    against the measured dense peak (its GEMMs dominate)."""
    import torch
    import sparse_long_sequence_lf_b200 as lf
    from sparse_long_sequence_lf_b200.workloads import make_encoder_inputs, make_masks

    wl = ew.attn
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    stream = torch.cuda.Stream(device)
    x0, layers = make_encoder_inputs(wl, ew.layers, ew.inter)
    local_m, glob_m = make_masks(wl)
    counts = [0] * wl.B if glob_m is None else [int(c) for c in (glob_m != 0).sum(1)]
    mg = max(counts)
    dev_layers = [{k: v.to(device) for k, v in lw.items()} for lw in layers]
    x = x0.to(device)
    lm = None if local_m is None else local_m.to(device)
    gm = None if glob_m is None else glob_m.to(device)
    out = torch.empty_like(x)
    ws = torch.empty(lf.encoder_workspace_size(wl.B, wl.n, wl.H, ew.inter, mg),
                     dtype=torch.uint8, device=device)
    weight_bytes = sum(t.numel() * t.element_size() for lw in dev_layers for t in lw.values())
    windows = [wl.window] * ew.layers

    def step():
        lf.encoder_forward(x, dev_layers, lm, gm, H=wl.H, windows=windows, max_global=mg,
                           out=out, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    if lf.workspace_status(ws) != 0:
        raise RuntimeError("encoder status not ok")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    with torch.cuda.stream(stream):
        g.replay()
    stream.synchronize()
    steps = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        start.record(stream)
        for _ in range(steps):
            with torch.cuda.stream(stream):
                g.replay()
        end.record(stream)
        torch.cuda.synchronize(device)
        if world > 1:
            dist.barrier()
    max_ms = reduce_max(start.elapsed_time(end), device)
    clocks = sampler.summary("timed region")
    ms = max_ms / steps
    flops = encoder_flops(ew, counts)
    tflops = flops / (ms * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    peak = peaks["bf16_tflops_sustained"]
    roofline = {"kernel": "whole stack (proj_kernel GEMMs dominate)", "bound": "tensor",
                "achieved": round(tflops, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(tflops / peak, 4), "traffic": None,
                "peak_source": peak_kind + " sustained (bf16 dense; fp16 has the same nominal "
                               "rate; the step runs for milliseconds)"}

    pin_x = x0.pin_memory()
    host_out = torch.empty_like(x0).pin_memory()
    xd = torch.empty_like(x)

    def e2e_once():
        with torch.cuda.stream(stream):
            xd.copy_(pin_x, non_blocking=True)
            lf.encoder_forward(xd, dev_layers, lm, gm, H=wl.H, windows=windows, max_global=mg,
                               out=out, workspace=ws, stream=stream)
            host_out.copy_(out, non_blocking=True)
        stream.synchronize()

    e2e_once()
    e_steps = max(3, min(steps, args.e2e_steps))
    es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    es.record(stream)
    for _ in range(e_steps):
        e2e_once()
    ee.record(stream)
    torch.cuda.synchronize(device)
    e_ms = reduce_max(es.elapsed_time(ee) / e_steps, device)
    e2e = {"value": round(e_ms, 4), "unit": "ms", "h2d_bytes_per_step":
           int(x0.numel() * x0.element_size()),
           "d2h_bytes_per_step": int(x0.numel() * x0.element_size()), "steps": e_steps,
           "path": "lf_encoder_forward with the input copied from pinned host memory and the "
                   "output copied back (weights resident)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import encoder as oenc
        w0 = {k: v.double().numpy() for k, v in layers[0].items()}
        # Sample: layer 0 over batch 0's first rows (every per-token cost is
        # linear in the tokens at a fixed window), scaled to the whole stack.
        rows = min(wl.n, 1024)
        sl = lambda m: None if m is None else m[:1, :rows].contiguous()
        t0 = time.perf_counter()
        oenc.encoder_layer(x0[:1, :rows].double().numpy(), w0, sl(local_m), sl(glob_m), H=wl.H,
                           window=wl.window)
        dt = time.perf_counter() - t0
        scale = ew.layers * wl.B * wl.n / rows
        cpu = {"value": round(dt * 1e3 * scale, 1), "unit": "ms", "cores": os.cpu_count(),
               "kind": "oracle",
               "sample": f"layer 0 on the first {rows} tokens of batch 0 timed once "
                         f"({dt:.1f} s, fp64 numpy products and the C attention oracle), "
                         f"scaled by {scale:g} to the whole stack"}
    ft = FT_A100_FP16_MS.get((wl.B, wl.n)) if wl.dtype == "f16" and ew.inter == 4096 \
        and wl.H == 16 and ew.layers == 24 and wl.window == 512 else None
    result = {
        "metric": ENC_METRIC, "value": round(ms, 4), "unit": "ms", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None if ft is None else round(ms / ft, 4),
        "dtype": wl.dtype, "data": "synthetic (random-init weights)",
        "config": {**workload_config(wl, world), "workload": ew.name, "op": "encoder",
                   "layers": ew.layers, "inter": ew.inter, "hidden": wl.H * wl.d,
                   "l2": f"weights {weight_bytes / 2**20:.0f} MiB per step > L2",
                   "launch": "CUDA graph of one lf_encoder_forward call",
                   "useful_tflop_per_step": round(flops / 1e12, 4),
                   "tflops": round(tflops, 1),
                   "vs_baseline_note": None if ft is None else
                   f"ms / FasterTransformer's {ft} ms on A100-80GB (guide's table; other "
                   "hardware, context only)"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": None, "clocks": clocks,
    }
    attn_launches = launches_per_step(wl, mg) - 1
    result["gpu_launches"] = steps * (1 + ew.layers * (1 + attn_launches + 2 + 3))
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        del g
        dist.destroy_process_group()


def run_projection_cpu_baseline(wl, counts, gidx, max_global, budget_s):
    """The fp64 projection oracle on the first tokens of batch 0 (a bounded
    sample), scaled to the metric's unit."""
    import numpy as np
    from oracle.projection import projection_forward
    from sparse_long_sequence_lf_b200.workloads import make_layer_inputs
    x = make_layer_inputs(wl)
    f = lambda t: t.double().numpy()
    X, W, Bi, Wg, Bg = f(x["x"]), f(x["w"]), f(x["bias"]), f(x["wqg"]), f(x["bqg"])
    hid = wl.H * wl.d
    rows = min(wl.n, 256)
    g0 = -np.ones((1, rows), dtype=np.int32)
    sel = [int(p) for p in gidx[0, :min(int(counts[0]), max_global)] if p < rows]
    g0[0, :len(sel)] = sel
    c0 = np.array([len(sel)], dtype=np.int32)
    flops = 2.0 * rows * hid * 5 * hid + 2.0 * len(sel) * hid * hid
    reps, t0 = 0, time.perf_counter()
    while True:
        projection_forward(X[:1, :rows], W, Bi, Wg, Bg, g0, c0, H=wl.H)
        reps += 1
        dt = time.perf_counter() - t0
        if dt > budget_s or reps >= 1000:
            break
    import os
    return {"value": round(flops * reps / dt / 1e12, 6), "unit": "TFLOP/s",
            "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"first {rows} tokens of batch 0, {reps} repetition(s), {dt:.1f} s, "
                      "fp64 numpy oracle (BLAS threads)",
            "seconds": round(dt, 2)}


# ------------------------------------------------------------- CPU oracle
def oracle_sample_plan(wl, budget_s):
    """Head count and repetitions of the oracle sample for a time budget."""
    import oracle
    from sparse_long_sequence_lf_b200 import accounting
    from sparse_long_sequence_lf_b200.workloads import make_inputs

    x = make_inputs(wl)
    # Calibrate on one head of every batch.
    t0 = time.perf_counter()
    run_oracle_heads(oracle, x, wl, 1)
    t1 = time.perf_counter() - t0
    heads = max(1, min(wl.H, int(budget_s / max(t1, 1e-3))))
    reps = 1
    if heads == wl.H:
        reps = max(1, int(budget_s / max(t1 * wl.H, 1e-3)))
    sub = wl.with_(H=heads, dilation=tuple(wl.dilation_list()[:heads]))
    return x, heads, reps, accounting.useful_flops(sub)


def run_oracle_heads(oracle, x, wl, heads):
    for b in range(wl.B):
        oracle.forward(x["q"], x["k"], x["v"], x["qg"], x["kg"], x["vg"], x["local_mask"],
                       x["global_mask"], window=wl.window, dilation=x["dilation"],
                       causal=wl.causal, bh_range=(b * wl.H, b * wl.H + heads))


def run_cpu_baseline(wl, budget_s=10.0):
    import oracle
    x, heads, reps, flops = oracle_sample_plan(wl, budget_s)
    # The thread count of the OpenMP run, read before the single-thread run
    # below sets the OpenMP default to one thread.
    cores = oracle.default().max_threads()
    t0 = time.perf_counter()
    for _ in range(reps):
        run_oracle_heads(oracle, x, wl, heads)
    dt = time.perf_counter() - t0
    single = run_cpu_single_thread(wl, x, budget_s=max(1.0, budget_s / 4))
    return {"value": round(flops * reps / dt / 1e12, 6), "unit": UNIT,
            "cores": cores, "kind": "oracle",
            "sample": f"{heads} of {wl.H} heads x {wl.B} batches, {reps} repetition(s), "
                      f"{dt:.1f} s, fp64 C oracle with OpenMP",
            "seconds": round(dt, 2), "single_thread": single}


def run_cpu_single_thread(wl, x, budget_s=2.5):
    """The oracle on one host thread, best of 3, on a block of rows of one
    head sized to about budget_s / 3 per run."""
    import oracle
    from sparse_long_sequence_lf_b200 import accounting

    def once(rows):
        t0 = time.perf_counter()
        oracle.forward(x["q"], x["k"], x["v"], x["qg"], x["kg"], x["vg"], x["local_mask"],
                       x["global_mask"], window=wl.window, dilation=x["dilation"],
                       causal=wl.causal, bh_range=(0, 1), row_range=(0, rows), threads=1)
        return time.perf_counter() - t0

    rows = min(wl.n, 256)
    t = once(rows)
    rows = max(1, min(wl.n, int(rows * (budget_s / 3) / max(t, 1e-4))))
    best = min(once(rows) for _ in range(3))
    flops = accounting.useful_flops_rows(wl, head=0, rows=(0, rows))
    return {"value": round(flops / best / 1e12, 6), "unit": UNIT, "cores": 1,
            "sample": f"rows 0..{rows} of batch 0 head 0, best of 3 ({best:.2f} s)"}


def workload_config(wl, world, heads_split=False):
    """The workload part of a bench line's config (both arms)."""
    if world == 1:
        par = "single GPU"
    elif heads_split:
        par = f"one problem, heads split over {world} GPUs"
    else:
        par = f"independent replicas x{world}"
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "n": wl.n, "d_head": wl.d,
            "window": wl.window, "dilation": wl.dilation_list(), "causal": wl.causal,
            "globals": wl.globals_kind, "pad_tail": list(wl.pad_tail),
            "global_batch": wl.B * (1 if heads_split else world), "seq_len": wl.n,
            "parallelism": par}


def check_head_shards(wl_full, set0, out0, ranges, max_global, ws, stream, device, rank, step):
    """After the timed region of a head-split run: every rank recomputes its
    heads of input set 0, the slices are all-gathered, and rank 0 compares
    them with the whole problem run on its own GPU.  The heads are
    independent, so the two must agree bit for bit."""
    import torch
    import sparse_long_sequence_lf_b200 as lf
    from sparse_long_sequence_lf_b200.sharding import gather_heads
    from sparse_long_sequence_lf_b200.workloads import make_inputs
    with torch.cuda.stream(stream):
        step(0)
    stream.synchronize()
    full = gather_heads(out0, ranges)
    verdict = None
    if rank == 0:
        x = {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in make_inputs(wl_full).items()}
        ws_full = lf.new_workspace(wl_full.B, wl_full.H, wl_full.n, max_global, device)
        ref = lf.attention_forward(x["q"], x["k"], x["v"], x["qg"], x["kg"], x["vg"],
                                   x["local_mask"], x["global_mask"], window=wl_full.window,
                                   dilation=x["dilation"], causal=wl_full.causal,
                                   max_global=max_global, workspace=ws_full)
        torch.cuda.synchronize(device)
        if not torch.equal(ref, full):
            raise RuntimeError("head-split output differs from the single-GPU output")
        verdict = f"gathered heads equal the single-GPU forward bit for bit ({len(ranges)} ranks)"
    return verdict


def run_reference_arm(args, wl, world, rank):
    """The oracle as the reference arm: each step a bounded sample (one or more
    heads) of the same workload on the host cores.  Rank 0 only."""
    if rank != 0:
        return
    import oracle
    budget_per_step = max(0.05, min(2.0, args.reference_seconds / max(1, args.steps + args.warmup)))
    x, heads, _, flops = oracle_sample_plan(wl, budget_per_step)
    for _ in range(args.warmup):
        run_oracle_heads(oracle, x, wl, heads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run_oracle_heads(oracle, x, wl, heads)
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    sample = f"{heads} of {wl.H} heads x {wl.B} batches per step, fp64 C oracle with OpenMP"
    cores = oracle.default().max_threads()
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, world),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    from sparse_long_sequence_lf_b200.workloads import HEADLINE, WORKLOADS
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=HEADLINE)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-seconds", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-lse", action="store_true",
                    help="--op backward: recompute the rows' log-sum-exp instead of taking it "
                         "from the forward")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="under torchrun: every rank runs the whole workload (replicas, weak "
                         "scaling) or the ranks split one problem by heads (strong scaling)")
    ap.add_argument("--encoder", default=None,
                    help="encoder stack of --op encoder (default: the 24-layer fp16 model)")
    ap.add_argument("--op", choices=["attention", "projection", "output", "backward", "encoder"],
                    default="attention",
                    help="attention: the hot path (default); projection: the Q/K/V/Kg/Vg/Qg "
                         "prologue; output: the output projection + LayerNorm; backward: the "
                         "attention backward, on the workload's shape; encoder: a whole "
                         "encoder stack (--encoder)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_env()
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 needs torchrun with N processes")
    wl = WORKLOADS[args.workload]
    if args.shard == "heads" and world > wl.H:
        ap.error("--shard heads needs at most H ranks")
    if args.shard == "heads" and args.op != "attention":
        ap.error("--shard heads applies to the attention op")
    if args.impl == "reference":
        run_reference_arm(args, wl, world, rank)
        return
    if args.op in ("projection", "output"):
        if wl.dtype == "f32":
            ap.error("the projection and output layers run on bf16 / fp16 workloads")
        (run_projection_arm if args.op == "projection" else run_output_arm)(
            args, wl, world, rank, local)
        return
    if args.op == "backward":
        run_backward_arm(args, wl, world, rank, local)
        return
    if args.op == "encoder":
        from sparse_long_sequence_lf_b200.workloads import ENCODER_HEADLINE, ENCODER_WORKLOADS
        run_encoder_arm(args, ENCODER_WORKLOADS[args.encoder or ENCODER_HEADLINE], world, rank,
                        local)
        return
    run_gpu_arm(args, wl, world, rank, local)


if __name__ == "__main__":
    main()
