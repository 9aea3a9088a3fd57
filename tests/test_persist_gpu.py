"""The persistent all-depths kernel against the fp64 oracle: several sequences
with ragged contexts (deep items and window units spread over the grid), one and
two 128-row M tiles, slices of fewer than eight tokens, contexts inside the window,
empty windows, many deep items per CTA, the context-length override, repeated
calls (the merge order is fixed), and calls of the cluster kernel and over fewer
sequences in between (both kernels share the cache's scratch)."""
import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from tests.gpu_util import check, check_lse, fill, make_cache, oracle_all_depths, run_all_depths

pytestmark = pytest.mark.gpu


def _verify_and_check(wl, ctx, heads=None, ctx_len=None, reps=1):
    cache = make_cache(wl, nseq=len(ctx), kernel=1)
    assert cache.ripe_cache_verify_path() == 1
    fill(cache, wl, ctx)
    nseq = len(ctx)
    T = [int(t) for t in (ctx if ctx_len is None else np.minimum(ctx, ctx_len))]
    ws = [max(0, int(t) - wl.W) for t in ctx]
    cl = None if ctx_len is None else torch.tensor(ctx_len, dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(reps):
        _, O, lse, _ = run_all_depths(cache, wl, 0, nseq, wl.k, ctx_len=cl)
        outs.append((O, lse))
    hs = np.arange(wl.H) if heads is None else np.asarray(heads)
    ref, ref_lse = oracle_all_depths(wl, 0, nseq, wl.k, T, ws, heads=hs)
    for O, lse in outs:
        check(O[:, hs], ref, wl, wl.name)
        check_lse(lse[:, hs], ref_lse)
    for O, lse in outs[1:]:
        assert np.array_equal(O, outs[0][0]) and np.array_equal(lse, outs[0][1])
    assert cache.ripe_get_device_error() == 0
    cache.close()


@pytest.mark.parametrize("d", [64, 96, 128])
def test_ragged_sequences_one_m_tile(d):
    # contexts: deep + window, inside the window (no deep region), empty
    wl = S.Workload("p_ragged_d%d" % d, 1, 4, 3, d, 16, 4, 4, None, 0.88, 1201, "bf16", 700, 4)
    _verify_and_check(wl, np.array([650, 77, 9, 0]), reps=2)


@pytest.mark.parametrize("d,R,k", [(128, 32, 8), (96, 16, 12), (64, 40, 5)])
def test_two_m_tiles_and_partial_slices(d, R, k):
    # k*R > 128 rows per sequence: two M tiles; k = 12 and 5 give slices of 4 and 5 tokens
    wl = S.Workload("p_mt2_d%d" % d, 1, R, 2, d, 40, k, 2, None, 0.88, 1202, "bf16", 1200, k)
    _verify_and_check(wl, np.array([1100, 333]))


@pytest.mark.parametrize("W", [0, 1, 64, 4096])
def test_window_extremes(W):
    # W = 0: no window keys (block only); W >= T: no deep region (a slice's only arrival)
    wl = S.Workload("p_w%d" % W, 1, 8, 2, 96, W, 4, 2, None, 0.88, 1203, "bf16", 5000, 4)
    _verify_and_check(wl, np.array([700, 129]))


def test_many_deep_items_per_cta():
    # 24 sequences x 16 heads: more deep items than SMs, several per CTA
    wl = S.Workload("p_many", 1, 32, 16, 128, 128, 8, 24, None, 0.88, 1204, "bf16", 2200, 8)
    rng = np.random.default_rng(3)
    ctx = rng.integers(0, 2100, size=24)
    ctx[5] = 2100
    _verify_and_check(wl, ctx, heads=[0, 7, 15])


def test_context_override_and_repeats():
    wl = S.Workload("p_ctx", 1, 32, 4, 96, 64, 4, 3, None, 0.88, 1205, "bf16", 1200, 4)
    ctx = np.array([1100, 500, 64])
    _verify_and_check(wl, ctx, ctx_len=np.array([900, 500, 30]), reps=3)


@pytest.mark.parametrize("W", [0, 4])
def test_many_window_units_per_cta(W):
    # The 55-head, 32-depth shape with a small window: the planner puts many window
    # units on each CTA, so the stage ring's producer warps run far apart.
    wl = S.Workload("p_units_w%d" % W, 1, 32, 55, 96, W, 4, 1, None, 0.88, 1206, "bf16", 1088, 4)
    _verify_and_check(wl, np.array([1024]), heads=[0, 17, 54], reps=2)


def test_interleaved_kernels_and_subsets():
    # Persistent and cluster-kernel calls alternate on one cache (they share its
    # scratch), over all three sequences or fewer.
    wl = S.Workload("p_mix", 1, 32, 6, 96, 64, 4, 3, None, 0.88, 1207, "bf16", 1200, 4)
    cache = make_cache(wl, nseq=3, kernel=1)
    ctx = np.array([1100, 700, 80])
    fill(cache, wl, ctx)
    ws = [max(0, int(t) - wl.W) for t in ctx]
    ref, ref_lse = oracle_all_depths(wl, 0, 3, wl.k, [int(t) for t in ctx], ws)
    rows = wl.k * wl.R
    for kern, n in [(1, 3), (2, 3), (1, 3), (1, 1), (2, 2), (1, 3), (1, 2), (1, 3)]:
        cache.ripe_cache_set_all_depths_kernel(kern)
        _, O, lse, _ = run_all_depths(cache, wl, 0, n, wl.k)
        check(O, ref[: n * rows], wl, "kernel %d, %d sequences" % (kern, n))
        check_lse(lse, ref_lse[: n * rows])
    assert cache.ripe_get_device_error() == 0
    cache.close()
