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


def make_cache(wl, nseq=None, Tmax=None, kernel=0):
    """kernel: which sm_100a kernel serves all-depths calls (0 auto, 1 persistent,
    2 cluster)."""
    from depth_planed_kv_b200.ripe import RipeCache
    cache = RipeCache(wl.layers, wl.R, wl.H, wl.d, wl.W, Tmax or wl.Tmax, nseq or wl.nseq, wl.kmax,
                      torch_dtype(wl))
    if kernel:
        cache.ripe_cache_set_all_depths_kernel(kernel)
    return cache


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


def run_all_depths(cache, wl, layer, nseq, k, seqs=None, ctx_len=None, with_lse=True):
    seqs = list(range(nseq)) if seqs is None else seqs
    table, Q, Kb, Vb = all_depth_rows(wl, layer, nseq, seqs, k)
    shape = (nseq, k, wl.R, wl.H, wl.d)
    q, kb, vb = (to_dev(x.reshape(shape), wl) for x in (Q, Kb, Vb))
    O = torch.full(shape, float("nan"), dtype=torch_dtype(wl), device="cuda")
    lse = torch.full((nseq, k, wl.R, wl.H), float("nan"), device="cuda") if with_lse else None
    ids = torch.tensor(seqs, dtype=torch.int32, device="cuda")
    cache.ripe_verify_attn_all_depths(layer, ids, k, q, kb, vb, O, lse, ctx_len=ctx_len)
    torch.cuda.synchronize()
    O = O.float().cpu().numpy().reshape(nseq * k * wl.R, wl.H, wl.d)
    lse = lse.cpu().numpy().reshape(nseq * k * wl.R, wl.H) if with_lse else None
    return table, O, lse, (Q, Kb, Vb)


def oracle_all_depths(wl, layer, nseq, k, T, ws, seqs=None, heads=None, mode=1):
    seqs = list(range(nseq)) if seqs is None else seqs
    views = [seq_planes(wl, layer, s, T[i], ws[i], heads=heads) for i, s in enumerate(seqs)]
    table, Q, Kb, Vb = all_depth_rows(wl, layer, nseq, seqs, k, heads=heads)
    return OR.verify(views, table, Q, Kb, Vb, 1 / math.sqrt(wl.d), mode)


def check_lse(got, ref):
    assert np.abs(got - ref).max() < 2e-3, np.abs(got - ref).max()
