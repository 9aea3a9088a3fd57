"""RIPE store on the GPU against the oracle's store model, byte for byte."""
import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from oracle import oracle as OR

pytestmark = pytest.mark.gpu


def bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.view(torch.int32).cpu().numpy().view(np.uint32)
    return t.cpu().numpy()


def compare_store(cache, model, what=""):
    buf = cache.buffers()
    torch.cuda.synchronize()
    for name, ref in (("kdeep", model.kdeep), ("vdeep", model.vdeep), ("kwin", model.kwin), ("vwin", model.vwin)):
        got = bits(buf[name])
        assert np.array_equal(got, ref), "%s: %s differs at %d elements" % (what, name, int((got != ref).sum()))
    ln, ws, rf = cache.ripe_read_meta(with_rfloor=True)
    assert np.array_equal(ln, model.length), (what, ln, model.length)
    assert np.array_equal(ws, model.wstart), (what, ws, model.wstart)
    assert np.array_equal(rf, model.rfloor), (what, rf, model.rfloor)
    fb, fp = cache.ripe_read_forks()
    assert np.array_equal(fp, model.fpos), (what, fp, model.fpos)
    assert np.array_equal(fb[fp > 0], model.base[fp > 0]), (what, fb, model.base)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("W", [0, 3, 8])
def test_append_evict_truncate_bit_exact(dtype, W):
    from depth_planed_kv_b200.ripe import RipeCache
    L, R, H, d, Tmax, B, kmax = 2, 4, 3, 16, 200, 5, 6
    cache = RipeCache(L, R, H, d, W, Tmax, B, kmax, dtype)
    np_t = np.uint16 if dtype == torch.bfloat16 else np.uint32
    model = OR.OracleStore(L, R, H, d, W, Tmax, B, kmax, np_t)
    rng = np.random.default_rng(100 + W)
    dev = lambda a: torch.from_numpy(np.asarray(a, np.int32)).cuda()
    for step in range(60):
        op = rng.integers(0, 11)
        ids = rng.choice(B, size=rng.integers(1, B + 1), replace=False).astype(np.int32)
        if op == 10:
            # forks: a parent and a distinct child (sometimes a fork of a fork, flagged)
            pc = rng.choice(B, size=2, replace=False).astype(np.int32)
            cache.ripe_fork(dev(pc[:1]), dev(pc[1:]))
            model.fork(pc[:1], pc[1:])
            compare_store(cache, model, "step %d fork %s" % (step, pc))
            continue
        if op < 6:
            kin = int(rng.choice([1, 2, kmax, 2 * (W + kmax) + 3, 70]))
            n = rng.integers(0, kin + 1, size=len(ids)).astype(np.int32)
            vals = torch.randn(2, L, len(ids), kin, R, H, d).to(dtype).cuda()
            K, V = vals[0].contiguous(), vals[1].contiguous()
            cache.ripe_append(dev(ids), dev(n), K, V)
            model.append(ids, n, bits(K), bits(V))
        elif op < 8:
            cache.ripe_evict(dev(ids))
            model.evict(ids)
        elif op < 9:
            nl = rng.integers(0, Tmax, size=len(ids)).astype(np.int32)
            cache.ripe_truncate(dev(ids), dev(nl))
            model.truncate(ids, nl)
        else:
            cache.ripe_cache_reset(dev(ids))
            model.reset(ids)
        compare_store(cache, model, "step %d op %d" % (step, op))
    err = cache.ripe_get_device_error()
    assert (err != 0) == model.flagged
    cache.close()


def test_capacity_overflow_is_flagged_and_skipped():
    from depth_planed_kv_b200.ripe import RipeCache
    cache = RipeCache(1, 2, 1, 8, 4, 10, 2, 8, torch.float32)
    K = torch.ones(1, 2, 8, 2, 1, 8, device="cuda")
    ids = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    cache.ripe_append(ids, torch.tensor([8, 3], dtype=torch.int32, device="cuda"), K, K)
    cache.ripe_append(ids, torch.tensor([5, 3], dtype=torch.int32, device="cuda"), K, K)  # seq 0 overflows
    ln, _ = cache.ripe_read_meta()
    assert list(ln[:2]) == [8, 6]
    from depth_planed_kv_b200.ripe import RIPE_OK
    assert cache.ripe_get_device_error() == 2
    assert cache.ripe_get_device_error() == 0  # cleared by the read
    bad = torch.tensor([5], dtype=torch.int32, device="cuda")
    cache.ripe_evict(bad)
    assert cache.ripe_get_device_error() == 1
    cache.close()


@pytest.mark.parametrize("dtype,R,H,d,W,kmax,T", [
    (torch.float32, 4, 3, 16, 8, 4, 48),
    (torch.bfloat16, 5, 2, 32, 6, 3, 70),
    (torch.bfloat16, 3, 2, 96, 0, 4, 5),
])
def test_synthetic_fill_equals_append_of_generator_planes(dtype, R, H, d, W, kmax, T):
    """The fill kernel's generator equals the documented NumPy generator, and its
    store state equals one ripe_append of all T positions with all planes."""
    from depth_planed_kv_b200.ripe import RipeCache
    seed, decay, L, B, seq = 77, 0.88, 2, 4, 2
    a = RipeCache(L, R, H, d, W, T + 8, B, kmax, dtype)
    b = RipeCache(L, R, H, d, W, T + 8, B, kmax, dtype)
    coef = S.coef_table(decay, R)
    a.ripe_synth_fill([seq], [T], seed, coef)
    bf = dtype == torch.bfloat16
    K = np.zeros((L, 1, T, R, H, d), np.float32)
    V = np.zeros_like(K)
    for l in range(L):
        kp = S.planes(seed, 0, l, seq, range(H), np.arange(1, R + 1), np.arange(T), d, R, coef, bf)
        vp = S.planes(seed, 1, l, seq, range(H), np.arange(1, R + 1), np.arange(T), d, R, coef, bf)
        K[l, 0] = np.transpose(kp, (2, 1, 0, 3))
        V[l, 0] = np.transpose(vp, (2, 1, 0, 3))
    ids = torch.tensor([seq], dtype=torch.int32, device="cuda")
    b.ripe_append(ids, torch.tensor([T], dtype=torch.int32, device="cuda"),
                  torch.from_numpy(K).to(dtype).cuda(), torch.from_numpy(V).to(dtype).cuda())
    torch.cuda.synchronize()
    ba, bb = a.buffers(), b.buffers()
    for name in ("kdeep", "vdeep", "kwin", "vwin", "len", "ws", "rfloor"):
        assert np.array_equal(bits(ba[name]), bits(bb[name])), name
    a.close()
    b.close()
