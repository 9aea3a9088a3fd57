"""Loop-by-loop verification and the prelude/coda layers of a looped model
(RIPE abstract, first sentence: R planes per recurrent layer; LoopSpec article on
the layers before and after the loop).

* A looped model produces the draft block's keys and values at depth r only after
  its r-th loop, so it verifies one depth per launch: R calls of ripe_verify_attn
  with the depth-r branch of each sequence, the block planes of depth r supplied
  just before the r-th call.  Each call's rows equal the all-depths call's rows of
  that depth (and the fp64 oracle).
* Prelude and coda layers run once per token: their caches are single-plane stores
  (R = 1).  With the recurrent layers' RIPE store, the live planes of the whole
  2/4/2 stack are the closed form's fraction of the full cache -- 11.9 % at
  T = 1024, W = 64, R = 32 -- counted from the stores' own lengths and window starts.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from depth_planed_kv_b200.synth_rows import all_depth_rows, seq_planes
from oracle import oracle as OR
from tests.gpu_util import check, fill, make_cache, to_dev

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_one_depth_per_launch_equals_all_depths(dtype):
    from depth_planed_kv_b200.ripe import branch_table
    d = 96 if dtype == "bf16" else 32
    wl = S.Workload("loops", 1, 8, 3, d, 32, 4, 1, 400, 0.88, 1401, dtype, 500, 4)
    R, k, H = wl.R, wl.k, wl.H
    cache = make_cache(wl)
    fill(cache, wl, [wl.ctx])
    table, Q, Kb, Vb = all_depth_rows(wl, 0, 1, [0], k)
    shape = (1, k, R, H, d)
    O_all = torch.empty(shape, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32, device="cuda")
    ids = torch.tensor([0], dtype=torch.int32, device="cuda")
    cache.ripe_verify_attn_all_depths(0, ids, k, to_dev(Q.reshape(shape), wl), to_dev(Kb.reshape(shape), wl),
                                      to_dev(Vb.reshape(shape), wl), O_all)
    O_all = O_all.float().cpu().numpy().reshape(k * R, H, d)
    ref, _ = OR.verify([seq_planes(wl, 0, 0, wl.ctx, wl.ctx - wl.W)], table, Q, Kb, Vb, 1 / math.sqrt(d))
    check(O_all, ref, wl, "all depths")
    for r in range(1, R + 1):
        rows = np.arange(k) * R + r - 1          # this depth's rows in the all-depths layout
        q, kb, vb = (to_dev(x[rows], wl) for x in (Q, Kb, Vb))   # block planes of loop r only
        o = torch.empty_like(q)
        cache.ripe_verify_attn(0, branch_table([(0, r, k, 0, 1)]), 1, q, kb, vb, o)
        o = o.float().cpu().numpy()
        check(o, ref[rows], wl, "depth %d" % r)
        check(o, O_all[rows], wl, "depth %d vs all depths" % r)
    assert cache.ripe_get_device_error() == 0
    cache.close()


def test_prelude_recurrent_coda_stack_memory_fraction():
    from depth_planed_kv_b200.ripe import RipeCache
    g = json.load(open(os.path.join(GOLDEN, "memory_fraction.json")))
    T, W, R = g["T"], g["W"], g["R"]
    n_pre, n_rec, n_coda = g["n_prelude"], g["n_recurrent"], g["n_coda"]
    H, d, kmax = 1, 64, 4
    rec = RipeCache(n_rec, R, H, d, W, T + kmax, 1, kmax, torch.bfloat16)
    single = RipeCache(n_pre + n_coda, 1, H, d, 0, T + kmax, 1, kmax, torch.bfloat16)
    ids = torch.tensor([0], dtype=torch.int32, device="cuda")
    for c, r in ((rec, R), (single, 1)):
        c.ripe_synth_fill([0], [T], 5, S.coef_table(0.88, r))
        c.ripe_evict(ids)
    # live planes per layer and head: every position's deepest plane, plus planes
    # 1..R-1 of the positions still in the window (ws <= p < len)
    live = 0
    for c, layers, r in ((rec, n_rec, R), (single, n_pre + n_coda, 1)):
        ln, ws = c.ripe_read_meta()
        live += layers * (int(ln[0]) + (int(ln[0]) - min(int(ws[0]), int(ln[0]))) * (r - 1))
    full = (n_pre + n_coda) * T + n_rec * R * T
    frac = live / full
    assert round(100 * frac, g["printed_decimals"]) == g["printed_percent"]
    assert frac == pytest.approx(OR.memory_fraction(T, W, R, n_rec, n_pre, n_coda), abs=1e-15)
    rec.close()
    single.close()
