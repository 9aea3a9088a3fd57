"""The per-query sliding-window verify on the GPU against the fp64 oracle's
sliding reading (RIPE abstract, fifth sentence, read per query): windows longer
and shorter than the draft block (W < k reads older draft tokens at plane R, from
their depth-R rows), W = 0, ragged contexts, one and two M tiles; and the BI4
property on the GPU: with W >= k the depth-R rows' block planes reach no shallower
row, bit for bit."""
import math

import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from depth_planed_kv_b200.synth_rows import all_depth_rows, seq_planes
from oracle import oracle as OR
from tests.gpu_util import check, check_lse, fill, make_cache, to_dev

pytestmark = pytest.mark.gpu


def _run(cache, wl, nseq, Q, Kb, Vb):
    shape = (nseq, wl.k, wl.R, wl.H, wl.d)
    O = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full(shape[:-1], float("nan"), device="cuda")
    ids = torch.arange(nseq, dtype=torch.int32, device="cuda")
    cache.ripe_verify_attn_all_depths_sliding(0, ids, wl.k, to_dev(Q.reshape(shape), wl),
                                              to_dev(Kb.reshape(shape), wl), to_dev(Vb.reshape(shape), wl), O, lse)
    torch.cuda.synchronize()
    n = nseq * wl.k * wl.R
    return O.float().cpu().numpy().reshape(n, wl.H, wl.d), lse.cpu().numpy().reshape(n, wl.H)


@pytest.mark.parametrize("d,R,k,W", [(96, 8, 4, 16), (96, 8, 4, 2), (64, 8, 12, 5), (64, 16, 8, 0),
                                     (128, 32, 8, 3)])
def test_sliding_matches_oracle(d, R, k, W):
    wl = S.Workload("slide_d%d_W%d" % (d, W), 1, R, 2, d, W, k, 3, None, 0.88, 1501, "bf16", 700, k)
    ctx = np.array([600, 37, 2])
    cache = make_cache(wl)
    assert cache.ripe_cache_verify_path() == 1
    fill(cache, wl, ctx)
    table, Q, Kb, Vb = all_depth_rows(wl, 0, 3, [0, 1, 2], k)
    O, lse = _run(cache, wl, 3, Q, Kb, Vb)
    views = [seq_planes(wl, 0, s, int(ctx[s]), max(0, int(ctx[s]) - W)) for s in range(3)]
    ref, ref_lse = OR.verify_sliding(views, table, Q, Kb, Vb, W, 1 / math.sqrt(d))
    check(O, ref, wl, "sliding d=%d W=%d" % (d, W))
    check_lse(lse, ref_lse)
    assert cache.ripe_get_device_error() == 0
    cache.close()


@pytest.mark.parametrize("W,k", [(4, 4), (3, 4)])
def test_sliding_block_independence_on_gpu(W, k):
    wl = S.Workload("slide_bi4", 1, 8, 2, 96, W, k, 1, 300, 0.88, 1502, "bf16", 400, k)
    R = wl.R
    cache = make_cache(wl)
    fill(cache, wl, [wl.ctx])
    table, Q, Kb, Vb = all_depth_rows(wl, 0, 1, [0], k)
    O, _ = _run(cache, wl, 1, Q, Kb, Vb)
    Kp, Vp = Kb.copy(), Vb.copy()
    rng = np.random.default_rng(4)
    for j in range(k):
        Kp[j * R + R - 1] = S.round_bf16(Kp[j * R + R - 1] + rng.standard_normal(Kp[0].shape).astype(np.float32))
        Vp[j * R + R - 1] = S.round_bf16(Vp[j * R + R - 1] + rng.standard_normal(Vp[0].shape).astype(np.float32))
    O2, _ = _run(cache, wl, 1, Q, Kp, Vp)
    shallow = [j * R + r - 1 for j in range(k) for r in range(1, R)]
    assert (not np.array_equal(O[shallow], O2[shallow])) == (W < k)
    cache.close()
