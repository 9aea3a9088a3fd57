#!/usr/bin/env python
"""Throughput of RIPE verify-attention on B200: KV GB/s, query-rows/s and the
fraction of the HBM roofline.

One step = one verify of the Huginn-shaped workload over its 4 recurrent layers
(R=32 loop planes, H=55 heads, d=96, T=1024 committed positions, W=64 window,
k=4 draft tokens verified at all 32 depths: 128 query rows per head), i.e. four
ripe_verify_attn_all_depths calls through the C ABI.  The store holds two such
sequences and steps alternate between them, so 552 MB of distinct KV separate
two reads of the same bytes (the L2 holds 126 MB): inputs larger than L2.

Multi-GPU: one process per GPU (torchrun), each rank verifies its own sequences;
no data-path collective ("scaling": "weak").  The step time is the max over ranks.

--impl reference times the fp64 CPU oracle (the reference arm of this project)
on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from depth_planed_kv_b200 import synth as S  # noqa: E402

METRIC = "RIPE verify-attn KV GB/s + query-rows/s (1×B200), % of HBM roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM = 6650.0
PROFILES_DIR = os.path.join(ROOT, "profiles")


def algorithmic_bytes(wl, T, ws, branches, with_lse=True):
    """Bytes the method must move for one verify call of one layer.

    Per sequence: plane R K+V of every position read at plane R (all T if some
    branch is at depth R, else the min(ws,T) outside the window); K+V of each
    distinct queried depth r < R over the window positions; block K+V, Q and O of
    every row; the fp32 LSE of every row if requested.  Metadata and partial
    results are not counted.
    """
    es = 2 if wl.bf16 else 4
    row = wl.H * wl.d * es
    total = 0
    for s in range(len(T)):
        A = min(ws[s], T[s])
        mine = [b for b in branches if b.seq == s]
        depths = {b.depth for b in mine}
        deep_pos = T[s] if wl.R in depths else A
        total += 2 * deep_pos * row
        total += 2 * (T[s] - A) * row * len([r for r in depths if r < wl.R])
        nrows = sum(b.ntok for b in mine)
        total += nrows * row * 4  # Q, Kblk, Vblk read; O written
        if with_lse:
            total += nrows * wl.H * 4
    return total


def measured_peak():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for name in sorted(os.listdir(os.path.join(ROOT, "depth_planed_kv_b200", "csrc"))):
        with open(os.path.join(ROOT, "depth_planed_kv_b200", "csrc", name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def traffic_for(workload: str):
    """ncu DRAM bytes (read + write) per launch of the dominant kernel, if a summary
    under profiles/ records them for this workload on the current kernel source.

    A summary carries one line of the form
    ``traffic: workload=<name> source_hash=<hash> dram_bytes_per_launch=<int>``.
    """
    want = kernel_source_hash()
    try:
        names = sorted(os.listdir(PROFILES_DIR))
    except OSError:
        return None
    for name in names:
        if not name.endswith((".md", ".txt")):
            continue
        with open(os.path.join(PROFILES_DIR, name)) as f:
            for line in f:
                line = line.strip().strip("`")
                if not line.startswith("traffic:"):
                    continue
                kv = dict(x.split("=", 1) for x in line[len("traffic:"):].split() if "=" in x)
                if kv.get("workload") == workload and kv.get("source_hash") == want:
                    return int(kv["dram_bytes_per_launch"])
    return None


class ClockSampler:
    """Polls NVML for SM clock and throttle reasons on this GPU while running."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, dev_index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nvml = pynvml
        except Exception as e:  # no NVML: report nothing rather than guess
            self.error = str(e)

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for k, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def cpu_baseline(wl, budget_s=10.0):
    """The fp64 oracle, as it stands, on a bounded sample of the workload: the
    whole Huginn step in (layer, 11-head) blocks, repeated until about budget_s
    seconds of oracle time (input generation excluded)."""
    from oracle import oracle as OR
    from depth_planed_kv_b200.synth_rows import all_depth_rows, seq_planes
    T, ws = wl.ctx, wl.ctx - wl.W
    br = S.all_depth_branches(1, wl.R, wl.k)
    blocks = []
    for l in range(wl.layers):
        for h0 in range(0, wl.H, 11):
            heads = np.arange(h0, min(h0 + 11, wl.H))
            sub = S.Workload(wl.name, 1, wl.R, len(heads), wl.d, wl.W, wl.k, 1, T, wl.decay, wl.seed,
                             wl.dtype, wl.Tmax, wl.kmax)
            blocks.append((seq_planes(wl, l, 0, T, ws, heads=heads),
                           all_depth_rows(wl, l, 1, [0], wl.k, heads=heads),
                           algorithmic_bytes(sub, [T], [ws], br), len(heads)))
    done_bytes, done_rows, spent, n = 0, 0, 0.0, 0
    while spent < budget_s:
        view, (table, Q, Kb, Vb), nbytes, nh = blocks[n % len(blocks)]
        t0 = time.perf_counter()
        OR.verify([view], table, Q, Kb, Vb, 1 / math.sqrt(wl.d))
        spent += time.perf_counter() - t0
        done_bytes += nbytes
        done_rows += Q.shape[0] * nh
        n += 1
    return {"value": done_bytes / spent / 1e9, "unit": "GB/s", "cores": OR.num_threads(), "kind": "oracle",
            "sample": "fp64 oracle (deep/window/block partials) over the whole 4-layer Huginn step in "
                      "(layer, 11-head) blocks: %d blocks = %.2f steps in %.1f s" % (n, n / len(blocks), spent),
            "query_rows_per_s": done_rows / spent}


# ---------------------------------------------------------------- multi-rank host logic
# One process per GPU; ranks verify disjoint sequences (their own synthetic stores)
# and exchange nothing on the data path: NCCL (gloo on CPU) serves only the barrier
# and the max-over-ranks step time.

def shard_seed(seed: int, rank: int) -> int:
    """Seed of the synthetic store of `rank` (each rank holds different sequences)."""
    return seed + 17 * rank


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's time: every rank calls this, in the same order."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(bytes_per_step_per_rank: float, world: int, steps: int, ms_max: float) -> float:
    """GB/s of all ranks together over the slowest rank's time (weak scaling)."""
    return bytes_per_step_per_rank * world * steps / (ms_max / 1e3) / 1e9


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = S.huginn()
    from oracle import oracle as OR
    from depth_planed_kv_b200.synth_rows import all_depth_rows, seq_planes
    T, ws = wl.ctx, wl.ctx - wl.W
    heads = np.arange(0, 4)
    br = S.all_depth_branches(1, wl.R, wl.k)
    sub = S.Workload(wl.name, 1, wl.R, len(heads), wl.d, wl.W, wl.k, 1, T, wl.decay, wl.seed, wl.dtype,
                     wl.Tmax, wl.kmax)
    per_step = algorithmic_bytes(sub, [T], [ws], br)
    views, probs = [], []
    for l in range(wl.layers):
        views.append(seq_planes(wl, l, 0, T, ws, heads=heads))
        probs.append(all_depth_rows(wl, l, 1, [0], wl.k, heads=heads))

    def step(i):
        l = i % wl.layers
        table, Q, Kb, Vb = probs[l]
        OR.verify([views[l]], table, Q, Kb, Vb, 1 / math.sqrt(wl.d))

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    value = per_step * args.steps / dt / 1e9
    rows = 128 * len(heads) * args.steps / dt
    sample = "fp64 oracle on heads 0-3 of one layer per step (layers in turn) of the Huginn workload"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": wl.name, "sample": "4 of 55 heads, 1 of 4 layers per step"},
        "query_rows_per_s": rows,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": OR.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ripe", choices=["ripe", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    warmup = max(args.warmup, 3)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from depth_planed_kv_b200 import build as B
    B.build()
    from depth_planed_kv_b200.ripe import RipeCache, launch_count
    from depth_planed_kv_b200.synth_rows import all_depth_rows

    wl = S.huginn()
    nrep = 2
    cache = RipeCache(wl.layers, wl.R, wl.H, wl.d, wl.W, wl.Tmax, nrep, wl.kmax, torch.bfloat16)
    cache.ripe_synth_fill(list(range(nrep)), [wl.ctx] * nrep, shard_seed(wl.seed, rank),
                          S.coef_table(wl.decay, wl.R))
    ids = [torch.tensor([s], dtype=torch.int32, device="cuda") for s in range(nrep)]
    for s in range(nrep):
        cache.ripe_evict(ids[s])
    shape = (1, wl.k, wl.R, wl.H, wl.d)
    host_in, dev_in = [], []
    for s in range(nrep):
        hl, dl = [], []
        for l in range(wl.layers):
            _, Q, Kb, Vb = all_depth_rows(wl, l, 1, [s], wl.k)
            trip = [torch.from_numpy(x.reshape(shape)).to(torch.bfloat16).pin_memory() for x in (Q, Kb, Vb)]
            hl.append(trip)
            dl.append([t.cuda() for t in trip])
        host_in.append(hl)
        dev_in.append(dl)
    O = [torch.empty(shape, dtype=torch.bfloat16, device="cuda") for _ in range(wl.layers)]
    lse = [torch.empty(shape[:-1], dtype=torch.float32, device="cuda") for _ in range(wl.layers)]
    O_host = [torch.empty(shape, dtype=torch.bfloat16).pin_memory() for _ in range(wl.layers)]
    lse_host = [torch.empty(shape[:-1], dtype=torch.float32).pin_memory() for _ in range(wl.layers)]
    stream = torch.cuda.current_stream()
    T, ws = wl.ctx, wl.ctx - wl.W
    br = S.all_depth_branches(1, wl.R, wl.k)
    bytes_layer = algorithmic_bytes(wl, [T], [ws], br)
    bytes_step = bytes_layer * wl.layers
    rows_step = wl.k * wl.R * wl.H * wl.layers

    def step(i, ev=None):
        s = i % nrep
        for l in range(wl.layers):
            if ev is not None:
                ev[l][0].record(stream)
            q, kb, vb = dev_in[s][l]
            cache.ripe_verify_attn_all_depths(l, ids[s], wl.k, q, kb, vb, O[l], lse[l])
            if ev is not None:
                ev[l][1].record(stream)

    def step_e2e(i):
        s = i % nrep
        for l in range(wl.layers):
            for hsrc, ddst in zip(host_in[s][l], dev_in[s][l]):
                ddst.copy_(hsrc, non_blocking=True)
            q, kb, vb = dev_in[s][l]
            cache.ripe_verify_attn_all_depths(l, ids[s], wl.k, q, kb, vb, O[l], lse[l])
            O_host[l].copy_(O[l], non_blocking=True)
            lse_host[l].copy_(lse[l], non_blocking=True)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()


    for i in range(warmup):
        step(i)
    assert cache.ripe_get_device_error() == 0
    # Per-call events inside the timed region (one record before and after each call).
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(wl.layers)]
           for _ in range(min(args.steps, 500))]
    # A second of identical untimed steps first, so the clock samples reflect steady load.
    sampler = ClockSampler(local)
    with sampler:
        t_end = time.time() + 1.0
        i = 0
        while time.time() < t_end:
            step(i)
            i += 1
            if i % 200 == 0:
                torch.cuda.synchronize()
        barrier()
        n0 = launch_count()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        n1 = launch_count()
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world, "cuda")
    # Kernel duration for the roofline: a separate pass with an event pair around every
    # call (events between calls stop consecutive calls from overlapping, so this pass
    # is not the step time).
    barrier()
    nev = min(args.steps, 500)
    for i in range(nev):
        step(i, evs[i])
    torch.cuda.synchronize()
    call_ms = statistics.mean(evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(nev)
                              for l in range(wl.layers))

    # End to end through the public call with host buffers: H2D inputs, verify, D2H outputs.
    barrier()
    for i in range(warmup):
        step_e2e(i)
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(args.steps):
        step_e2e(i)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, "cuda")

    value = whole_job_rate(bytes_step, world, args.steps, ms_max)
    e2e_value = whole_job_rate(bytes_step, world, args.steps, e2e_ms)
    peak, peak_kind = measured_peak()
    # Average launch duration over the timed region: consecutive calls overlap their
    # prologues (programmatic dependent launch), so the region divided by its launches
    # is the per-launch time the step sustains; an isolated call takes call_ms.
    launch_ms = ms_max / (args.steps * wl.layers)
    achieved = bytes_layer / (launch_ms / 1e3) / 1e9
    h2d = sum(t.numel() * t.element_size() for l in range(wl.layers) for t in host_in[0][l])
    d2h = sum(O_host[l].numel() * 2 + lse_host[l].numel() * 4 for l in range(wl.layers))
    tr = traffic_for(wl.name)
    out = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "layers": wl.layers, "R": wl.R, "H": wl.H, "d": wl.d, "T": wl.ctx,
                   "W": wl.W, "k": wl.k, "rows_per_head": wl.k * wl.R,
                   "l2": "inputs larger than L2: 2 sequences x 4 layers alternated, 552 MB between reuses",
                   "algorithmic_bytes_per_step": bytes_step},
        "query_rows_per_s": rows_step * world * args.steps / (ms_max / 1e3),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": tr, "peak_source": peak_kind,
                     "kernel": "verify_kernel: one ripe_verify_attn_all_depths call (one layer); CUDA events "
                               "on its stream around the timed region / launches",
                     "isolated_call_us": call_ms * 1e3},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(n1 - n0),
        "clocks": dict(sampler.summary(), window="1 s of identical steps before and through the timed region"),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))
    cache.close()


if __name__ == "__main__":
    main()
