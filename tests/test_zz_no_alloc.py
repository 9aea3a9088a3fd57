"""ripe_verify_attn_noalloc: verify for callers that cannot allocate device memory.

Such callers exist: a serving stack that has reserved nearly all of HBM for its
own pools, code that enqueues work while a stream is captured into a CUDA graph,
or a latency-bound path that cannot pay cudaMalloc's device synchronisation.
The entry point keeps its partial results in the library's fixed device array;
its outputs must match the allocating entry point's, call after call.

This file is collected last so that a failure here stops a -x run only after
every other test has run.
"""
import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from tests.gpu_util import TOL, fill, make_cache, to_dev
from tests.util import branch_rows, errors

pytestmark = pytest.mark.gpu


def _problem(wl, layer, branches, nseq):
    from depth_planed_kv_b200.ripe import branch_table
    table, Q, Kb, Vb = branch_rows(wl, layer, branches, list(range(nseq)))
    return branch_table([tuple(t) for t in table]), len(table), to_dev(Q, wl), to_dev(Kb, wl), to_dev(Vb, wl)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_allocating_entry_point_on_consecutive_calls(dtype):
    wl = S.Workload("noalloc", 2, 8, 4, 64, 16, 8, 2, None, 0.81, 404, dtype, 512, 8)
    cache = make_cache(wl)
    fill(cache, wl, [300, 77])
    sets = [
        (0, [S.BranchSpec(0, 8, 8, 0, 0), S.BranchSpec(0, 3, 8, 1, 1), S.BranchSpec(1, 8, 5, 0, 0)]),
        (1, [S.BranchSpec(0, 8, 6, 0, 0), S.BranchSpec(1, 8, 8, 0, 0), S.BranchSpec(1, 5, 8, 1, 1),
             S.BranchSpec(1, 6, 3, 2, 2)]),
    ]
    tol_abs, tol_rel = TOL[dtype]
    for layer, branches in sets:  # two calls in a row, different problems
        tb, nb, Q, Kb, Vb = _problem(wl, layer, branches, 2)
        ref = torch.full(Q.shape, float("nan"), dtype=Q.dtype, device="cuda")
        ref_lse = torch.full(Q.shape[:2], float("nan"), device="cuda")
        cache.ripe_verify_attn(layer, tb, nb, Q, Kb, Vb, ref, ref_lse)
        got = torch.full_like(ref, float("nan"))
        got_lse = torch.full_like(ref_lse, float("nan"))
        rc, used = cache.ripe_verify_attn_noalloc(layer, tb, nb, Q, Kb, Vb, got, got_lse)
        torch.cuda.synchronize()
        assert rc == 0 and 0 < used <= 32 << 20
        a, r = errors(got.float().cpu().numpy(), ref.float().cpu().numpy())
        assert a <= tol_abs and r <= tol_rel, (a, r)
        assert np.abs(got_lse.cpu().numpy() - ref_lse.cpu().numpy()).max() <= 1e-5
    assert cache.ripe_get_device_error() == 0
    cache.close()


def test_noalloc_halves_the_split_count_until_its_scratch_fits():
    """A call whose first plan (8 deep splits: one sequence, two heads) needs more
    than the fixed 32 MiB, but fits with fewer, longer splits: it runs with the
    halved plan and matches the allocating entry point.  (Only the fused kernel's
    plan can need this: the CUDA-core plan's split count already falls as the
    rows grow.)"""
    from depth_planed_kv_b200.ripe import branch_table
    wl = S.Workload("noalloc_halve", 1, 4, 2, 64, 16, 141, 1, None, 0.88, 406, "bf16", 512, 141)
    cache = make_cache(wl)
    assert cache.ripe_cache_verify_path() == 1
    fill(cache, wl, [300])
    branches = [S.BranchSpec(0, 1 + i % 4, 141, i % 3, i % 2) for i in range(64)]   # 9024 rows
    tb, nb, Q, Kb, Vb = _problem(wl, 0, branches, 1)
    first_plan = Q.shape[0] * wl.H * 9 * (2 + wl.d) * 4     # 8 splits + the window partial
    assert first_plan > 32 << 20
    tol_abs, tol_rel = TOL["bf16"]
    for _ in range(2):
        ref = torch.full(Q.shape, float("nan"), dtype=Q.dtype, device="cuda")
        cache.ripe_verify_attn(0, tb, nb, Q, Kb, Vb, ref)
        got = torch.full_like(ref, float("nan"))
        rc, used = cache.ripe_verify_attn_noalloc(0, tb, nb, Q, Kb, Vb, got)
        torch.cuda.synchronize()
        assert rc == 0 and used <= 32 << 20 and used < first_plan
        a, r = errors(got.float().cpu().numpy(), ref.float().cpu().numpy())
        assert a <= tol_abs and r <= tol_rel, (a, r)
    assert cache.ripe_get_device_error() == 0
    cache.close()


def test_noalloc_refuses_calls_beyond_its_fixed_scratch():
    from depth_planed_kv_b200.ripe import RIPE_ERR_CAPACITY, branch_table
    wl = S.Workload("noalloc_big", 1, 4, 32, 128, 8, 64, 1, 64, 0.88, 5, "bf16", 128, 64)
    cache = make_cache(wl)
    fill(cache, wl, [64])
    nb = 40
    rows = [(0, 1 + i % 4, 64, 64 * i, 1) for i in range(nb)]       # 2560 rows x 32 heads
    tb = branch_table(rows)
    Q = torch.zeros(64 * nb, wl.H, wl.d, dtype=torch.bfloat16, device="cuda")
    O = torch.full_like(Q, 7.0)
    rc, need = cache.ripe_verify_attn_noalloc(0, tb, nb, Q, Q, Q, O, check=False)
    torch.cuda.synchronize()
    assert rc == RIPE_ERR_CAPACITY and need > 32 << 20
    assert torch.all(O == 7.0)  # nothing was launched
    cache.close()
