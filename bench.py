#!/usr/bin/env python
"""Throughput of RIPE verify-attention on B200: KV GB/s, query-rows/s and the
fraction of the HBM roofline, one JSON line per workload.

Workloads (seeded synthetic stores; the pages' own benchmarks need trained
weights and datasets, which these shapes stand in for):
  huginn (default): the Huginn-shaped step -- 4 recurrent layers, R=32 loop
      planes, H=55 heads, d=96, T=1024, W=64, k=4 draft tokens verified at all 32
      depths (128 query rows per head): four ripe_verify_attn_all_depths calls.
      The store holds two such sequences and steps alternate between them, so
      552 MB of distinct KV separate two reads of the same bytes (the L2 holds
      126 MB): inputs larger than L2.
  sweep_W{0,4,64,256,1024}: the same step with other windows (W=0 deepest plane
      only, W=1024 the full cache).
  loopspec_mixed: 64 sequences, contexts U[512,4096], a main branch at depth 32,
      a draft branch at U[4,16] and with probability 0.3 a fallback at U[16,28],
      8 tokens each, H=32, d=128: one ripe_verify_attn call over the branch list.
  long_ctx: 16 sequences at T=32768, W=128, k=8 at all 32 depths, H=32, d=128;
      a step is ripe_verify_attn_all_depths, then ripe_append of U[1,8] accepted
      tokens per sequence (their planes are the verified block's) and ripe_evict.

`value` is timed on the device with inputs resident; `e2e` times the same calls
with the inputs copied from pinned host memory and the outputs read back every
step (copies on their own streams, overlapped with the neighbouring calls).

Multi-GPU: one process per GPU (torchrun), each rank verifies its own sequences;
no data-path collective ("scaling": "weak").  The step time is the max over ranks.

--impl reference times the fp64 CPU oracle (the reference arm of this project)
on a bounded sample of the Huginn workload on the host cores.
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
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILES_DIR = os.path.join(ROOT, "profiles")
MUFU_PER_CLK_SM = 16  # ex2 results per clock per SM (CUDA throughput table, compute capability 10.0)


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


def measured_peaks():
    """The driver's measured peaks ({key: value}, "measured"), else the recipe's fallback."""
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        out = {k: float(p[k]) for k in FALLBACK if k in p}
        if "hbm_gbs" in out:
            return {**FALLBACK, **out}, "measured"
    except Exception:
        pass
    return dict(FALLBACK), "fallback"


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


# ---------------------------------------------------------------- oracle baselines

def oracle_rate(blocks, budget_s):
    """Time the fp64 oracle, as it stands, over (oracle inputs, algorithmic bytes,
    query rows) blocks in turn until about budget_s seconds of oracle time."""
    from oracle import oracle as OR
    done_bytes, done_rows, spent, n = 0, 0, 0.0, 0
    while spent < budget_s:
        views, (table, Q, Kb, Vb), nbytes, nrows, scale = blocks[n % len(blocks)]
        t0 = time.perf_counter()
        OR.verify(views, table, Q, Kb, Vb, scale)
        spent += time.perf_counter() - t0
        done_bytes += nbytes
        done_rows += nrows
        n += 1
    return done_bytes / spent / 1e9, done_rows / spent, n, spent, OR.num_threads()


def all_depth_blocks(wl, T, ws, layers, head_block, max_blocks=None):
    """Oracle inputs of an all-depths step in (layer, head-block) pieces."""
    from depth_planed_kv_b200.synth_rows import all_depth_rows, seq_planes
    br = S.all_depth_branches(1, wl.R, wl.k)
    blocks = []
    for l in range(layers):
        for h0 in range(0, wl.H, head_block):
            heads = np.arange(h0, min(h0 + head_block, wl.H))
            sub = S.Workload(wl.name, 1, wl.R, len(heads), wl.d, wl.W, wl.k, 1, T, wl.decay, wl.seed, wl.dtype,
                             wl.Tmax, wl.kmax)
            blocks.append(([seq_planes(wl, l, 0, T, ws, heads=heads)], all_depth_rows(wl, l, 1, [0], wl.k, heads=heads),
                           algorithmic_bytes(sub, [T], [ws], br), wl.k * wl.R * len(heads), 1 / math.sqrt(wl.d)))
            if max_blocks is not None and len(blocks) >= max_blocks:
                return blocks
    return blocks


def cpu_baseline(wl, budget_s=10.0):
    """The fp64 oracle, as it stands, on a bounded sample of the Huginn step: the
    whole step in (layer, 11-head) blocks, repeated until about budget_s seconds of
    oracle time (input generation excluded)."""
    T, ws = wl.ctx, wl.ctx - wl.W
    blocks = all_depth_blocks(wl, T, ws, wl.layers, 11)
    v, rows, n, spent, cores = oracle_rate(blocks, budget_s)
    return {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": "fp64 oracle (deep/window/block partials) over the whole 4-layer Huginn step in "
                      "(layer, 11-head) blocks: %d blocks = %.2f steps in %.1f s" % (n, n / len(blocks), spent),
            "query_rows_per_s": rows}


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


# ---------------------------------------------------------------- GPU workloads
# A workload holds its cache, its inputs (pinned host copies and device copies, one
# set per layer of each of `nrep` alternating problems), its outputs, and:
#   call(s, l): the library call(s) of layer l of problem s (device inputs);
#   post(i): calls after the layers of step i (store maintenance), or None;
#   nbytes(i), nrows(i): algorithmic bytes and query rows (x heads) of step i.

class Work:
    def __init__(self, name, config, cache, layers, nrep):
        self.name, self.config, self.cache, self.layers, self.nrep = name, config, cache, layers, nrep
        self.host_in, self.dev_in, self.outs, self.outs_host = [], [], [], []
        self.post = None
        self.steps = None        # fixed timed step count (None: --steps)
        self.warmup = None       # fixed warm-up count (None: --warmup, at least 3)
        self.preroll = True      # run ~1 s of untimed steps first (identical, store unchanged)
        self.verify_events = False  # time each verify inside the timed region (roofline)
        self.extra = {}

    def step(self, i, ev=None):
        s = i % self.nrep
        for l in range(self.layers):
            if ev is not None:
                ev[l][0].record()
            self.call(s, l, self.dev_in[s][l])
            if ev is not None:
                ev[l][1].record()
        if self.post is not None:
            self.post(i)


def pinned_pair(x, dtype):
    import torch
    h = torch.from_numpy(np.ascontiguousarray(x)).to(dtype).pin_memory()
    return h, h.cuda()


def make_all_depths_work(wl, name, rank, nrep=2, layers=None, lse=True):
    """An all-depths step (every layer, k tokens at all R depths) on nrep alternating
    single-sequence problems."""
    import torch
    from depth_planed_kv_b200.ripe import RipeCache
    from depth_planed_kv_b200.synth_rows import all_depth_rows
    layers = wl.layers if layers is None else layers
    cache = RipeCache(layers, wl.R, wl.H, wl.d, wl.W, wl.Tmax, nrep, wl.kmax, torch.bfloat16)
    cache.ripe_synth_fill(list(range(nrep)), [wl.ctx] * nrep, shard_seed(wl.seed, rank), S.coef_table(wl.decay, wl.R))
    ids = [torch.tensor([s], dtype=torch.int32, device="cuda") for s in range(nrep)]
    for s in range(nrep):
        cache.ripe_evict(ids[s])
    shape = (1, wl.k, wl.R, wl.H, wl.d)
    T, ws = wl.ctx, max(0, wl.ctx - wl.W)
    per_layer = algorithmic_bytes(wl, [T], [ws], S.all_depth_branches(1, wl.R, wl.k), with_lse=lse)
    wk = Work(name, {"workload": name, "layers": layers, "R": wl.R, "H": wl.H, "d": wl.d, "T": wl.ctx,
                     "W": wl.W, "k": wl.k, "rows_per_head": wl.k * wl.R}, cache, layers, nrep)
    for s in range(nrep):
        hl, dl = [], []
        for l in range(layers):
            _, Q, Kb, Vb = all_depth_rows(wl, l, 1, [s], wl.k)
            pairs = [pinned_pair(x.reshape(shape), torch.bfloat16) for x in (Q, Kb, Vb)]
            hl.append([p[0] for p in pairs])
            dl.append([p[1] for p in pairs])
        wk.host_in.append(hl)
        wk.dev_in.append(dl)
    for l in range(layers):
        o = [torch.empty(shape, dtype=torch.bfloat16, device="cuda")]
        if lse:
            o.append(torch.empty(shape[:-1], dtype=torch.float32, device="cuda"))
        wk.outs.append(o)
        wk.outs_host.append([torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in o])

    def call(s, l, din):
        q, kb, vb = din
        o = wk.outs[l]
        cache.ripe_verify_attn_all_depths(l, ids[s], wl.k, q, kb, vb, o[0], o[1] if lse else None)

    wk.call = call
    wk.nbytes = lambda i: per_layer * layers
    wk.nrows = lambda i: wl.k * wl.R * wl.H * layers
    wk.bytes_per_launch = per_layer
    wk.config["l2"] = "inputs larger than L2: %d sequences x %d layers alternated, %.0f MB between reuses" % (
        nrep, layers, nrep * per_layer * layers / 1e6)
    wk.config["algorithmic_bytes_per_step"] = per_layer * layers
    return wk


def make_mixed_work(rank):
    """The LoopSpec mixed-depth branch list: one ripe_verify_attn call per step."""
    import torch
    from depth_planed_kv_b200.ripe import RipeCache, branch_table
    from depth_planed_kv_b200.synth_rows import branch_rows
    wl = S.mixed()
    ctx, branches = S.mixed_structure(wl)
    cache = RipeCache(1, wl.R, wl.H, wl.d, wl.W, wl.Tmax, wl.nseq, wl.kmax, torch.bfloat16)
    cache.ripe_synth_fill(list(range(wl.nseq)), [int(t) for t in ctx], shard_seed(wl.seed, rank),
                          S.coef_table(wl.decay, wl.R))
    cache.ripe_evict(torch.arange(wl.nseq, dtype=torch.int32, device="cuda"))
    table, Q, Kb, Vb = branch_rows(wl, 0, branches, list(range(wl.nseq)))
    tb = branch_table([tuple(t) for t in table])
    ws = np.maximum(ctx - wl.W, 0)
    nbytes = algorithmic_bytes(wl, [int(t) for t in ctx], [int(w) for w in ws], branches)
    wk = Work("loopspec_mixed", {"workload": "loopspec_mixed_64seq", "layers": 1, "R": wl.R, "H": wl.H, "d": wl.d,
                                 "W": wl.W, "k": wl.k, "sequences": wl.nseq, "branches": len(branches),
                                 "ctx": "U[512,4096] (seed %d), total %d" % (wl.seed, int(ctx.sum())),
                                 "l2": "inputs larger than L2: %.0f MB per call" % (nbytes / 1e6),
                                 "algorithmic_bytes_per_step": nbytes}, cache, 1, 1)
    pairs = [pinned_pair(x, torch.bfloat16) for x in (Q, Kb, Vb)]
    wk.host_in = [[[p[0] for p in pairs]]]
    wk.dev_in = [[[p[1] for p in pairs]]]
    o = [torch.empty(Q.shape, dtype=torch.bfloat16, device="cuda"), torch.empty(Q.shape[:2], device="cuda")]
    wk.outs = [o]
    wk.outs_host = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in o]]

    def call(s, l, din):
        cache.ripe_verify_attn(0, tb, len(table), din[0], din[1], din[2], o[0], o[1])

    wk.call = call
    wk.nbytes = lambda i: nbytes
    wk.nrows = lambda i: Q.shape[0] * wl.H
    wk.bytes_per_launch = nbytes
    return wk


def make_long_work(rank, peaks, small=False):
    """Long context: verify all depths of 16 sequences at T=32768, then append U[1,8]
    accepted tokens per sequence (their planes are the verified block's) and evict;
    16 timed steps, the contexts grow.  `small`: 6 sequences at T=8192, the case
    the profiler captures."""
    import torch
    from depth_planed_kv_b200.ripe import RipeCache, ripe_cache_bytes
    from depth_planed_kv_b200.synth_rows import all_depth_rows
    wl = S.long_context_small() if small else S.long_context()
    B, R, H, d, k = wl.nseq, wl.R, wl.H, wl.d, wl.k
    cache = RipeCache(1, R, H, d, wl.W, wl.Tmax, B, wl.kmax, torch.bfloat16)
    cache.ripe_synth_fill(list(range(B)), [wl.ctx] * B, shard_seed(wl.seed, rank), S.coef_table(wl.decay, R))
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    cache.ripe_evict(ids)
    _, Q, Kb, Vb = all_depth_rows(wl, 0, B, list(range(B)), k)
    shape = (B, k, R, H, d)
    rng = np.random.default_rng(wl.seed)
    n_acc = rng.integers(1, 9, size=(64, B)).astype(np.int32)   # per step, per sequence
    T = np.full(B, wl.ctx, dtype=np.int64)
    lens = [T.copy()]
    for i in range(64):
        T = T + n_acc[i]
        lens.append(T.copy())
    wk = Work("long_ctx", {"workload": wl.name, "layers": 1, "R": R, "H": H, "d": d, "T": wl.ctx,
                           "W": wl.W, "k": k, "sequences": B,
                           "step": "verify all depths + append U[1,8] accepted tokens + evict; contexts grow",
                           "l2": "inputs larger than L2: %.1f GB store" %
                                 (ripe_cache_bytes(1, R, H, d, wl.W, wl.Tmax, B, wl.kmax, torch.bfloat16) / 1e9)},
              cache, 1, 1)
    pairs = [pinned_pair(x.reshape(shape), torch.bfloat16) for x in (Q, Kb, Vb)]
    nacc_h, nacc_d = pinned_pair(n_acc, torch.int32)
    wk.host_in = [[[p[0] for p in pairs] + [nacc_h]]]
    wk.dev_in = [[[p[1] for p in pairs] + [nacc_d]]]
    o = [torch.empty(shape, dtype=torch.bfloat16, device="cuda"), torch.empty(shape[:-1], device="cuda")]
    wk.outs = [o]
    wk.outs_host = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in o]]
    Kb5 = wk.dev_in[0][0][1].view(1, B, k, R, H, d)
    Vb5 = wk.dev_in[0][0][2].view(1, B, k, R, H, d)
    br = S.all_depth_branches(B, R, k)
    es = 2

    def verify_bytes(i):
        Ts = [int(t) for t in lens[i]]
        return algorithmic_bytes(wl, Ts, [max(0, t - wl.W) for t in Ts], br)

    def call(s, l, din):
        cache.ripe_verify_attn_all_depths(0, ids, k, din[0], din[1], din[2], o[0], o[1])

    def post(i):
        nd = wk.dev_in[0][0][3]
        cache.ripe_append(ids, nd[i % 64], Kb5, Vb5)
        cache.ripe_evict(ids)

    wk.call = call
    wk.post = post
    # The store holds Tmax = ctx + 512 positions and a step appends up to 8 tokens per
    # sequence: 3 warm-up + 16 timed steps, then 3 + 16 more end to end, is 38 <= 64.
    wk.steps = 16
    wk.warmup = 3
    wk.preroll = False
    wk.verify_events = True
    # bytes of a step: the verify's, plus the append's (read the accepted tokens'
    # R planes, write them to the store)
    wk.nbytes = lambda i: verify_bytes(i) + int(n_acc[i % 64].sum()) * R * H * d * es * 2 * 2
    wk.nrows = lambda i: B * k * R * H
    wk.verify_bytes = verify_bytes
    wk.flops = lambda i: sum(4 * k * R * max(0, int(t) - wl.W) * d * H for t in lens[i])   # deep QK^T + PV
    wk.exps = lambda i: sum(k * R * max(0, int(t) - wl.W) * H for t in lens[i])
    return wk


def run_work(wk, args, world, rank, local, peaks, peak_kind):
    """Time one workload; returns its JSON object."""
    import torch
    from depth_planed_kv_b200.ripe import launch_count
    stream = torch.cuda.current_stream()
    steps = wk.steps or args.steps
    warmup = wk.warmup or max(args.warmup, 3)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    i0 = 0
    for i in range(warmup):
        wk.step(i0 + i)
    i0 += warmup
    err = wk.cache.ripe_get_device_error()
    assert err == 0, "device error %d in warm-up" % err
    ev = None
    if wk.verify_events:
        ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(wk.layers)]
              for _ in range(steps)]
    sampler = ClockSampler(local)
    with sampler:
        if wk.preroll:  # identical untimed calls first, so the clock samples reflect steady load
            t_end = time.time() + 1.0
            j = 0
            while time.time() < t_end:
                wk.step(j)
                j += 1
                if j % 200 == 0:
                    torch.cuda.synchronize()
        barrier()
        n0 = launch_count()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            wk.step(i0 + i, ev[i] if ev is not None else None)
        e1.record(stream)
        torch.cuda.synchronize()
        n1 = launch_count()
    timed = range(i0, i0 + steps)
    i0 += steps
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, world, "cuda")
    nbytes = sum(wk.nbytes(i) for i in timed)
    nrows = sum(wk.nrows(i) for i in timed)
    value = nbytes * world / (ms_max / 1e3) / 1e9
    launches = steps * wk.layers
    if ev is not None:
        verify_ms = [ev[i][l][0].elapsed_time(ev[i][l][1]) for i in range(steps) for l in range(wk.layers)]
        launch_ms = statistics.mean(verify_ms)
        achieved = statistics.mean(wk.verify_bytes(i) for i in timed) / (launch_ms / 1e3) / 1e9
        isolated = None
    else:
        # The region divided by its launches: consecutive calls overlap their
        # prologues (programmatic dependent launch), so this is the per-launch time
        # the step sustains.  An isolated call (an event pair around every call,
        # which stops the overlap) is timed in a separate pass.
        launch_ms = ms_max / launches
        achieved = wk.bytes_per_launch / (launch_ms / 1e3) / 1e9
        barrier()
        nev = min(steps, 200)
        evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(wk.layers)] for _ in range(nev)]
        for i in range(nev):
            wk.step(i, evs[i])
        torch.cuda.synchronize()
        isolated = statistics.mean(evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(nev)
                                   for l in range(wk.layers)) * 1e3
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic_for(wk.config["workload"]),
            "peak_source": peak_kind,
            "kernel": "the verify call (one ripe_verify_attn* call: the persistent kernel and its merge kernel, or the cluster kernel, as the call is routed); CUDA events on their stream"}
    if isolated is not None:
        roof["isolated_call_us"] = isolated
    clocks = dict(sampler.summary(), window="1 s of identical steps before and through the timed region"
                  if wk.preroll else "the timed region")
    if hasattr(wk, "flops"):
        sm_mhz = clocks.get("sm_mhz") or 1965.0
        t_s = launch_ms / 1e3
        fl = statistics.mean(wk.flops(i) for i in timed) / t_s / 1e12
        ex = statistics.mean(wk.exps(i) for i in timed) / t_s
        mufu_peak = MUFU_PER_CLK_SM * torch.cuda.get_device_properties(local).multi_processor_count * sm_mhz * 1e6
        roof["tensor"] = {"achieved": fl, "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                          "frac": fl / peaks["bf16_tflops_sustained"],
                          "note": "deep-plane QK^T and PV flops (4 rows*keys*d per head) over the verify time"}
        roof["mufu"] = {"achieved": ex / 1e12, "peak": mufu_peak / 1e12, "unit": "Tex2/s",
                        "frac": ex / mufu_peak,
                        "note": "one ex2 per deep score; peak = 16 ex2/clk/SM x SMs x median SM clock"}
        roof["binding"] = max(("hbm", roof["frac"]), ("tensor", roof["tensor"]["frac"]),
                              ("mufu", roof["mufu"]["frac"]), key=lambda x: x[1])[0]

    # End to end through the same calls: every step copies its inputs from pinned
    # host memory and reads its outputs back, on copy streams ordered by events so
    # that the copies of one layer overlap the verify of its neighbours.
    barrier()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    mk = lambda: torch.cuda.Event()
    loaded = [[mk() for _ in range(wk.layers)] for _ in range(wk.nrep)]
    consumed = [[mk() for _ in range(wk.layers)] for _ in range(wk.nrep)]
    written = [mk() for _ in range(wk.layers)]
    drained = [mk() for _ in range(wk.layers)]
    for evl in consumed + [drained]:
        for e in evl:
            e.record(stream)

    def step_e2e(i):
        s = i % wk.nrep
        for l in range(wk.layers):
            h2d_s.wait_event(consumed[s][l])
            with torch.cuda.stream(h2d_s):
                for h, dv in zip(wk.host_in[s][l], wk.dev_in[s][l]):
                    dv.copy_(h, non_blocking=True)
                loaded[s][l].record(h2d_s)
            stream.wait_event(loaded[s][l])
            stream.wait_event(drained[l])
            wk.call(s, l, wk.dev_in[s][l])
            consumed[s][l].record(stream)
            written[l].record(stream)
            d2h_s.wait_event(written[l])
            with torch.cuda.stream(d2h_s):
                for dv, h in zip(wk.outs[l], wk.outs_host[l]):
                    h.copy_(dv, non_blocking=True)
                drained[l].record(d2h_s)
        if wk.post is not None:
            wk.post(i)

    e2e_steps = steps
    for i in range(warmup):
        step_e2e(i0 + i)
    i0 += warmup
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for evl in consumed:
        for e in evl:
            e.record(stream)
    for i in range(e2e_steps):
        step_e2e(i0 + i)
    for e in drained:
        stream.wait_event(e)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_bytes = sum(wk.nbytes(i) for i in range(i0, i0 + e2e_steps))
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, "cuda")
    h2d = sum(t.numel() * t.element_size() for l in range(wk.layers) for t in wk.host_in[0][l])
    d2h = sum(t.numel() * t.element_size() for l in range(wk.layers) for t in wk.outs_host[l])
    err = wk.cache.ripe_get_device_error()
    assert err == 0, "device error %d" % err
    out = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": ms_max / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic", "config": wk.config,
        "query_rows_per_s": nrows * world / (ms_max / 1e3),
        "roofline": roof,
        "e2e": {"value": e2e_bytes * world / (e2e_ms / 1e3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "copies": "H2D and D2H on their own streams, event-ordered"},
        "gpu_launches": int(n1 - n0),
        "clocks": clocks,
    }
    out.update(wk.extra)
    return out


WORKLOADS = ["huginn"] + ["sweep_W%d" % w for w in S.SWEEP_W] + ["loopspec_mixed", "long_ctx"]


def build_work(name, rank, peaks):
    if name == "huginn":
        return make_all_depths_work(S.huginn(), "huginn_T1024_W64_k4", rank)
    if name.startswith("sweep_W"):
        W = int(name[len("sweep_W"):])
        return make_all_depths_work(S.sweep(W), "sweep_T1024_W%d_k4" % W, rank)
    if name == "loopspec_mixed":
        return make_mixed_work(rank)
    if name == "long_ctx":
        return make_long_work(rank, peaks)
    if name == "long_ctx_small":
        return make_long_work(rank, peaks, small=True)
    raise ValueError(name)


def sampled_cpu_baseline(name, budget_s):
    """The oracle on a bounded sample of a non-default workload (for its line)."""
    from depth_planed_kv_b200.synth_rows import branch_rows, seq_planes
    if name.startswith("sweep_W"):
        wl = S.sweep(int(name[len("sweep_W"):]))
        blocks = all_depth_blocks(wl, wl.ctx, max(0, wl.ctx - wl.W), 1, 11)
        sample = "layer 0 of the step in 11-head blocks"
    elif name == "loopspec_mixed":
        wl = S.mixed()
        ctx, branches = S.mixed_structure(wl)
        blocks = []
        heads = np.arange(4)
        for s in range(0, wl.nseq, 8):
            mine = [b for b in branches if b.seq == s]
            sub = [S.BranchSpec(0, b.depth, b.ntok, b.qslot, b.bslot) for b in mine]
            T = int(ctx[s])
            ws = max(0, T - wl.W)
            w4 = S.Workload(wl.name, 1, wl.R, 4, wl.d, wl.W, wl.k, 1, T, wl.decay, wl.seed, wl.dtype, wl.Tmax, wl.kmax)
            blocks.append(([seq_planes(wl, 0, s, T, ws, heads=heads)], branch_rows(wl, 0, sub, [s], heads=heads),
                           algorithmic_bytes(w4, [T], [ws], sub), sum(b.ntok for b in sub) * 4, 1 / math.sqrt(wl.d)))
        sample = "heads 0-3 of every 8th sequence"
    elif name == "long_ctx":
        wl = S.long_context()
        one = S.Workload(wl.name, 1, wl.R, wl.H, wl.d, wl.W, wl.k, 1, wl.ctx, wl.decay, wl.seed, wl.dtype,
                         wl.Tmax, wl.kmax)
        blocks = all_depth_blocks(one, wl.ctx, wl.ctx - wl.W, 1, 1, max_blocks=2)
        sample = "heads 0 and 1 of sequence 0 (verify only)"
    else:
        return None
    v, rows, n, spent, cores = oracle_rate(blocks, budget_s)
    return {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": "fp64 oracle on %s: %d blocks in %.1f s" % (sample, n, spent), "query_rows_per_s": rows}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ripe", choices=["ripe", "reference"])
    ap.add_argument("--workload", default="huginn", choices=WORKLOADS + ["all", "long_ctx_small"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
        return

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

    peaks, peak_kind = measured_peaks()
    names = WORKLOADS if args.workload == "all" else [args.workload]
    for name in names:
        wk = build_work(name, rank, peaks)
        out = run_work(wk, args, world, rank, local, peaks, peak_kind)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            if name == "huginn":
                out["cpu_baseline"] = cpu_baseline(S.huginn())
            else:
                out["cpu_baseline"] = sampled_cpu_baseline(name, 5.0)
        wk.cache.close()
        del wk
        torch.cuda.empty_cache()
        if rank == 0:
            print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
