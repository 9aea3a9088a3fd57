"""Branch forks on the GPU (LoopSpec article, deployment section: a KV cache per
branch, rejected continuations deleted): a fork reads its parent's deep prefix and
then its own positions.  After forking and appending a branch's tokens, verify on
the fork -- persistent kernel (all depths), cluster kernel (branch list) and
CUDA-core kernels (fp32) -- matches the fp64 oracle over the oracle's store model,
and the parent's results are unchanged; releasing the fork empties it."""
import math

import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from oracle import oracle as OR
from tests.gpu_util import check

pytestmark = pytest.mark.gpu


def _vals(rng, shape, bf16):
    x = rng.standard_normal(shape).astype(np.float32)
    return S.round_bf16(x) if bf16 else x


@pytest.mark.parametrize("dtype,d,T0,kernel", [(torch.bfloat16, 96, 300, 1), (torch.bfloat16, 96, 300, 2),
                                               (torch.bfloat16, 64, 130, 1), (torch.bfloat16, 64, 130, 2),
                                               (torch.float32, 16, 200, 0)])
def test_verify_on_a_fork_matches_oracle(dtype, d, T0, kernel):
    from depth_planed_kv_b200.ripe import RipeCache, branch_table
    bf16 = dtype == torch.bfloat16
    L, R, H, W, kmax, Tmax, B = 1, 4, 2, 16, 4, 400, 4
    wl = S.Workload("fork", L, R, H, d, W, kmax, B, None, 0.88, 0, "bf16" if bf16 else "f32", Tmax, kmax)
    cache = RipeCache(L, R, H, d, W, Tmax, B, kmax, dtype)
    if kernel:
        cache.ripe_cache_set_all_depths_kernel(kernel)   # 1 persistent, 2 cluster
    model = OR.OracleStore(L, R, H, d, W, Tmax, B, kmax, np.float32)
    rng = np.random.default_rng(d + T0)
    dev = lambda a: torch.from_numpy(np.asarray(a, np.int32)).cuda()
    tens = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)

    K, V = _vals(rng, (L, 1, T0, R, H, d), bf16), _vals(rng, (L, 1, T0, R, H, d), bf16)
    cache.ripe_append(dev([1]), dev([T0]), tens(K), tens(V))
    model.append([1], [T0], K, V)
    cache.ripe_evict(dev([1]))
    model.evict([1])
    cache.ripe_fork(dev([1]), dev([3]))
    model.fork([1], [3])
    for step in range(3):
        n = int(rng.integers(1, kmax + 1))
        K, V = _vals(rng, (L, 1, kmax, R, H, d), bf16), _vals(rng, (L, 1, kmax, R, H, d), bf16)
        cache.ripe_append(dev([3]), dev([n]), tens(K), tens(V))
        model.append([3], [n], K, V)
        cache.ripe_evict(dev([3]))
        model.evict([3])
    fb, fp = cache.ripe_read_forks()
    assert fb[3] == 1 and fp[3] == T0 // 64 * 64
    scale = 1 / math.sqrt(d)
    k = 3
    for seq in (3, 1):   # the fork, then its parent
        nrows = k * R
        Q, Kb, Vb = (_vals(rng, (nrows, H, d), bf16) for _ in range(3))
        table = np.array([(seq, r, k, r - 1, R) for r in range(1, R + 1)], np.int32)
        ref, _ = OR.verify([model.plane_view(0, b) for b in range(B)], table, Q, Kb, Vb, scale)
        O = torch.full((nrows, H, d), float("nan"), dtype=dtype, device="cuda")
        cache.ripe_verify_attn_all_depths(0, dev([seq]), k, tens(Q), tens(Kb), tens(Vb), O)
        O2 = torch.full_like(O, float("nan"))
        cache.ripe_verify_attn(0, branch_table([tuple(t) for t in table]), R, tens(Q), tens(Kb), tens(Vb), O2)
        torch.cuda.synchronize()
        check(O.float().cpu().numpy(), ref, wl, "all depths seq %d" % seq)
        check(O2.float().cpu().numpy(), ref, wl, "branch list seq %d" % seq)
    assert cache.ripe_get_device_error() == 0
    cache.ripe_cache_reset(dev([3]))
    fb, fp = cache.ripe_read_forks()
    ln, _ = cache.ripe_read_meta()
    assert fb[3] == 3 and fp[3] == 0 and ln[3] == 0
    cache.close()
