"""Rollback to the confirmed prefix on the GPU (LoopSpec article, section on the
second branch): after speculative appends, evicts and a truncate, the GPU verify
matches the fp64 oracle over the oracle's store model, and the store metadata
matches it exactly."""
import math

import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from oracle import oracle as OR
from tests.gpu_util import TOL, check

pytestmark = pytest.mark.gpu


def _vals(rng, shape, bf16):
    x = rng.standard_normal(shape).astype(np.float32)
    return S.round_bf16(x) if bf16 else x


@pytest.mark.parametrize("kernel", [1, 2])   # all-depths calls: persistent / cluster kernel
@pytest.mark.parametrize("dtype,d,W,kmax", [
    (torch.bfloat16, 64, 16, 4),   # fused sm_100a kernels, W >= block
    (torch.bfloat16, 128, 3, 8),   # fused kernels, W < block
    (torch.float32, 16, 5, 4),     # CUDA-core kernels
])
def test_verify_after_rollback_matches_oracle(dtype, d, W, kmax, kernel):
    from depth_planed_kv_b200.ripe import RipeCache
    bf16 = dtype == torch.bfloat16
    wl = S.Workload("rollback", 1, 4, 2, d, W, kmax, 2, None, 0.88, 0, "bf16" if bf16 else "f32", 256, kmax)
    L, R, H, B, Tmax = 1, wl.R, wl.H, 2, wl.Tmax
    cache = RipeCache(L, R, H, d, W, Tmax, B, kmax, dtype)
    cache.ripe_cache_set_all_depths_kernel(kernel)
    model = OR.OracleStore(L, R, H, d, W, Tmax, B, kmax, np.float32)
    rng = np.random.default_rng(7 + d + W)
    ids = np.array([0, 1], np.int32)
    dev = lambda a: torch.from_numpy(np.asarray(a, np.int32)).cuda()
    tens = lambda a: torch.from_numpy(a).to(device="cuda", dtype=dtype).contiguous()

    def append(n, kin):
        K, V = _vals(rng, (L, 2, kin, R, H, d), bf16), _vals(rng, (L, 2, kin, R, H, d), bf16)
        cache.ripe_append(dev(ids), dev(n), tens(K), tens(V))
        model.append(ids, n, K, V)

    append([90, 61], 90)
    cache.ripe_evict(dev(ids))
    model.evict(ids)
    scale = 1 / math.sqrt(d)
    k = 3
    for step in range(6):
        n = rng.integers(1, kmax + 1, size=2).astype(np.int32)
        append(n, kmax)
        cache.ripe_evict(dev(ids))
        model.evict(ids)
        new_len = (model.length[ids] - n + rng.integers(0, n + 1)).astype(np.int32)
        cache.ripe_truncate(dev(ids), dev(new_len))
        model.truncate(ids, new_len)
        ln, ws, rf = cache.ripe_read_meta(with_rfloor=True)
        assert np.array_equal(ln, model.length) and np.array_equal(ws, model.wstart)
        assert np.array_equal(rf, model.rfloor)
        # All depths of k fresh draft tokens for both sequences.
        nrows = 2 * k * R
        Q, Kb, Vb = (_vals(rng, (nrows, H, d), bf16) for _ in range(3))
        O = torch.full((nrows, H, d), float("nan"), dtype=dtype, device="cuda")
        cache.ripe_verify_attn_all_depths(0, dev(ids), k, tens(Q), tens(Kb), tens(Vb), O)
        torch.cuda.synchronize()
        table = np.array([(s, r, k, s * k * R + r - 1, R) for s in range(2) for r in range(1, R + 1)], np.int32)
        ref, _ = OR.verify([model.plane_view(0, b) for b in range(B)], table, Q, Kb, Vb, scale)
        check(O.float().cpu().numpy(), ref, wl, "step %d" % step)
    assert cache.ripe_get_device_error() == 0
    cache.close()
