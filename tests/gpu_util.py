"""GPU-side test helpers: build a store for a workload through the C ABI and
gather the oracle's answer for a sample of (sequence, head) units."""
from __future__ import annotations

import math

import numpy as np
import torch

from depth_planed_kv_b200 import synth as S
from oracle import oracle as OR
from tests.util import all_depth_rows, branch_rows, errors, seq_planes

TOL = {"bf16": (2e-2, 1e-2), "f32": (1e-5, 1e-5)}  # (max abs, max row-normwise rel)


def torch_dtype(wl):
    return torch.bfloat16 if wl.bf16 else torch.float32


def make_cache(wl, nseq=None, Tmax=None):
    from depth_planed_kv_b200.ripe import RipeCache
    return RipeCache(wl.layers, wl.R, wl.H, wl.d, wl.W, Tmax or wl.Tmax, nseq or wl.nseq, wl.kmax,
                     torch_dtype(wl))


def fill(cache, wl, ctx):
    """Synthetic store of every sequence: T = ctx[s] positions, then evict."""
    ids = list(range(len(ctx)))
    cache.ripe_synth_fill(ids, [int(t) for t in ctx], wl.seed, S.coef_table(wl.decay, wl.R))
    cache.ripe_evict(torch.tensor(ids, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()


def to_dev(x, wl):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=torch_dtype(wl))


def check(got: np.ndarray, ref: np.ndarray, wl, what=""):
    a, r = errors(got, ref)
    tol_a, tol_r = TOL[wl.dtype]
    assert a <= tol_a and r <= tol_r, "%s: max abs %.3g (tol %.1g), max rel %.3g (tol %.1g)" % (
        what, a, tol_a, r, tol_r)
    return a, r


def oracle_units(wl, layer, ctx, ws, branches, seq_sample, head_sample, mode=1):
    """Oracle outputs for the branches of the sampled sequences, restricted to
    the sampled heads.  Returns {branch index: (O [ntok][nh][d], lse [ntok][nh])}."""
    local = {s: i for i, s in enumerate(seq_sample)}
    seqs = [seq_planes(wl, layer, s, int(ctx[s]), int(ws[s]), heads=head_sample) for s in seq_sample]
    sel = [(bi, b) for bi, b in enumerate(branches) if b.seq in local]
    sub = [S.BranchSpec(local[b.seq], b.depth, b.ntok, b.qslot, b.bslot) for _, b in sel]
    table, Q, Kb, Vb = branch_rows(wl, layer, sub, seq_sample, heads=head_sample)
    O, lse = OR.verify(seqs, table, Q, Kb, Vb, 1 / math.sqrt(wl.d), mode)
    out = {}
    for (bi, b), t in zip(sel, table):
        out[bi] = (O[t[3]:t[3] + t[2]], lse[t[3]:t[3] + t[2]])
    return out
