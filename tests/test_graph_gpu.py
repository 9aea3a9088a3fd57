"""A decode step captured once into a CUDA graph and replayed while the
sequences grow.

One step verifies k draft tokens at all R depths for every layer
(ripe_verify_attn_all_depths), then appends the accepted tokens with all their
planes (ripe_append) and evicts down to W full-depth positions (ripe_evict).
The step runs once eagerly, is captured, and is replayed.  Before each replay
the host writes the step's new K/V into the captured input buffers, drawn from
the counter-based generator at the positions they are appended to, as a model
would produce them; every stored value then equals the generator's value for its
(plane, position), so the oracle's view of the store after any number of steps
comes straight from the generator.

The lengths grow past what a plan made for the lengths at capture time covers:
for these shapes such a plan splits the deep region into 8 chunks of 64 keys
(512 keys), and the last replays have deep regions of up to 524 keys.  Captured
launches are planned for the cache's capacity instead, so every replay must
match the oracle, and an eager call after the replays as well (a captured
append leaves the host's length bound at the capacity).
"""
import math

import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from oracle import oracle as OR
from tests.gpu_util import TOL, check, fill, make_cache, to_dev, torch_dtype
from tests.util import all_depth_rows, seq_planes

pytestmark = pytest.mark.gpu

T0 = [500, 470]   # committed lengths before the eager step
N_ACC = [4, 3]    # tokens each sequence accepts per step
REPLAYS = 10


def _new_kv(wl, T, kmax_in):
    """[layers][nseq][kmax_in][R][H][d] K and V of positions T[s] .. T[s]+N_ACC[s]-1."""
    coef = S.coef_table(wl.decay, wl.R)
    out = []
    for kv in (0, 1):
        x = np.zeros((wl.layers, len(T), kmax_in, wl.R, wl.H, wl.d), np.float32)
        for l in range(wl.layers):
            for s in range(len(T)):
                pos = T[s] + np.arange(N_ACC[s])
                p = S.planes(wl.seed, kv, l, s, np.arange(wl.H), np.arange(1, wl.R + 1), pos, wl.d, wl.R,
                             coef, wl.bf16)                       # [H][R][n][d]
                x[l, s, :N_ACC[s]] = np.transpose(p, (2, 1, 0, 3))
        out.append(x)
    return out


def _check_step(wl, O, lse, T):
    """Every output of one step against the oracle at lengths T (ws = T - W)."""
    nseq, k = len(T), wl.k
    for l in range(wl.layers):
        views = [seq_planes(wl, l, s, T[s], T[s] - wl.W) for s in range(nseq)]
        table, Q, Kb, Vb = all_depth_rows(wl, l, nseq, list(range(nseq)), k)
        ref, ref_lse = OR.verify(views, table, Q, Kb, Vb, 1 / math.sqrt(wl.d))
        got = O[l].float().cpu().numpy().reshape(ref.shape)
        check(got, ref, wl, "layer %d at T=%s" % (l, T))
        assert np.abs(lse[l].cpu().numpy().reshape(ref_lse.shape) - ref_lse).max() < 2e-3


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_captured_step_replays_exactly_as_sequences_grow(dtype):
    wl = S.Workload("graph_step", 2, 4, 4, 64, 16, 4, 2, None, 0.88, 2024, dtype, 640, 4)
    nseq, k, R, H, d = wl.nseq, wl.k, wl.R, wl.H, wl.d
    cache = make_cache(wl)
    fill(cache, wl, T0)
    ids = torch.arange(nseq, dtype=torch.int32, device="cuda")
    n_acc = torch.tensor(N_ACC, dtype=torch.int32, device="cuda")
    shape = (nseq, k, R, H, d)
    qkv = []
    for l in range(wl.layers):
        _, Q, Kb, Vb = all_depth_rows(wl, l, nseq, list(range(nseq)), k)
        qkv.append([to_dev(x.reshape(shape), wl) for x in (Q, Kb, Vb)])
    O = [torch.full(shape, float("nan"), dtype=torch_dtype(wl), device="cuda") for _ in range(wl.layers)]
    lse = [torch.full(shape[:4], float("nan"), device="cuda") for _ in range(wl.layers)]
    Knew = torch.zeros((wl.layers, nseq, wl.kmax, R, H, d), dtype=torch_dtype(wl), device="cuda")
    Vnew = torch.zeros_like(Knew)

    def load_new_kv(T):
        kn, vn = _new_kv(wl, T, wl.kmax)
        Knew.copy_(to_dev(kn, wl))
        Vnew.copy_(to_dev(vn, wl))

    def step():
        for l in range(wl.layers):
            q, kb, vb = qkv[l]
            cache.ripe_verify_attn_all_depths(l, ids, k, q, kb, vb, O[l], lse[l])
        cache.ripe_append(ids, n_acc, Knew, Vnew)
        cache.ripe_evict(ids)

    T = list(T0)
    # One eager step (first launches configure the kernels), then the capture.
    load_new_kv(T)
    step()
    torch.cuda.synchronize()
    _check_step(wl, O, lse, T)
    T = [t + n for t, n in zip(T, N_ACC)]
    cache.ripe_reserve_workspace(nseq * k * R)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(REPLAYS):
        load_new_kv(T)
        g.replay()
        torch.cuda.synchronize()
        _check_step(wl, O, lse, T)
        T = [t + n for t, n in zip(T, N_ACC)]
        length, ws = cache.ripe_read_meta()
        assert list(length[:nseq]) == T and list(ws[:nseq]) == [t - wl.W for t in T]
    assert max(T) - wl.W - N_ACC[0] > 512  # the last replays read past a capture-time plan
    # An eager call after the replays plans from the host's bound, which the
    # captured append left at the capacity.
    for l in range(wl.layers):
        q, kb, vb = qkv[l]
        cache.ripe_verify_attn_all_depths(l, ids, k, q, kb, vb, O[l], lse[l])
    torch.cuda.synchronize()
    _check_step(wl, O, lse, T)
    assert cache.ripe_get_device_error() == 0
    del g
    cache.close()
