"""The long-context step at full size, as a step: 16 sequences at T=32768, W=128,
k=8 tokens at all 32 depths (H=32, d=128); each step verifies, appends U[1,8]
accepted tokens per sequence (the planes the verify read for them) and evicts.
After three steps the store metadata equals the expected lengths exactly, and the
third verify, which reads positions appended by the first two, matches the fp64
oracle on sampled (sequence, head) units."""
import math

import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from depth_planed_kv_b200.synth_rows import all_depth_rows
from oracle import oracle as OR
from tests.gpu_util import check, check_lse

pytestmark = pytest.mark.gpu


def _sample_view(wl, seq, head, steps_n, Kb, Vb):
    """The oracle's view of sequence `seq`, head `head` after the appended steps:
    positions below the context from the generator, later ones from the block
    planes each step appended (tokens 0..n-1 of the verified block)."""
    R, d = wl.R, wl.d
    coef = S.coef_table(wl.decay, R)
    T0 = wl.ctx
    T = T0 + int(sum(steps_n))
    ws = T - wl.W
    pos = np.arange(T0)
    kd = [S.planes(wl.seed, 0, 0, seq, [head], [R], pos, d, R, coef, True)[0, 0]]
    vd = [S.planes(wl.seed, 1, 0, seq, [head], [R], pos, d, R, coef, True)[0, 0]]
    # block planes of this sequence: [k][R][d] for the head
    kb = Kb[seq][:, :, head]
    vb = Vb[seq][:, :, head]
    app_k, app_v = [], []
    for n in steps_n:
        app_k.append(kb[:n])
        app_v.append(vb[:n])
    app_k = np.concatenate(app_k)      # [appended][R][d]
    app_v = np.concatenate(app_v)
    kd.append(app_k[:, R - 1])
    vd.append(app_v[:, R - 1])
    Kd = np.concatenate(kd)[None]
    Vd = np.concatenate(vd)[None]
    # window planes 1..R-1 of positions ws..T-1
    kw = np.zeros((1, R - 1, T - ws, d), np.float32)
    vw = np.zeros_like(kw)
    old = np.arange(ws, T0)
    if len(old):
        kw[0, :, :len(old)] = S.planes(wl.seed, 0, 0, seq, [head], np.arange(1, R), old, d, R, coef, True)[0]
        vw[0, :, :len(old)] = S.planes(wl.seed, 1, 0, seq, [head], np.arange(1, R), old, d, R, coef, True)[0]
    new = np.arange(max(ws, T0), T) - T0
    kw[0, :, len(old):] = np.transpose(app_k[new][:, :R - 1], (1, 0, 2))
    vw[0, :, len(old):] = np.transpose(app_v[new][:, :R - 1], (1, 0, 2))
    return {"T": T, "ws": ws, "R": R, "Kd": Kd, "Vd": Vd, "Kw": kw, "Vw": vw}


def test_long_context_three_steps():
    from depth_planed_kv_b200.ripe import RipeCache
    wl = S.long_context()
    B, R, H, d, k = wl.nseq, wl.R, wl.H, wl.d, wl.k
    cache = RipeCache(1, R, H, d, wl.W, wl.Tmax, B, wl.kmax, torch.bfloat16)
    cache.ripe_synth_fill(list(range(B)), [wl.ctx] * B, wl.seed, S.coef_table(wl.decay, R))
    ids = torch.arange(B, dtype=torch.int32, device="cuda")
    cache.ripe_evict(ids)
    _, Q, Kb, Vb = all_depth_rows(wl, 0, B, list(range(B)), k)
    shape = (B, k, R, H, d)
    q, kb, vb = (torch.from_numpy(x.reshape(shape)).to(torch.bfloat16).cuda() for x in (Q, Kb, Vb))
    O = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(shape[:-1], device="cuda")
    rng = np.random.default_rng(wl.seed)
    n_acc = rng.integers(1, 9, size=(3, B)).astype(np.int32)
    for step in range(3):
        cache.ripe_verify_attn_all_depths(0, ids, k, q, kb, vb, O, lse)
        if step < 2:
            cache.ripe_append(ids, torch.from_numpy(n_acc[step]).cuda(), kb.view(1, B, k, R, H, d),
                              vb.view(1, B, k, R, H, d))
            cache.ripe_evict(ids)
    torch.cuda.synchronize()
    ln, ws, rf = cache.ripe_read_meta(with_rfloor=True)
    T_exp = wl.ctx + n_acc[0] + n_acc[1]
    assert np.array_equal(ln, T_exp) and np.array_equal(ws, T_exp - wl.W)
    assert np.array_equal(rf, T_exp - wl.W - wl.kmax)
    assert cache.ripe_get_device_error() == 0
    O = O.float().cpu().numpy().reshape(B, k * R, H, d)
    lse = lse.cpu().numpy().reshape(B, k * R, H)
    Kb5 = Kb.reshape(shape)
    Vb5 = Vb.reshape(shape)
    table = np.array([(0, r, k, r - 1, R) for r in range(1, R + 1)], np.int32)
    for seq, head in [(3, 5), (14, 30)]:
        view = _sample_view(wl, seq, head, [n_acc[0][seq], n_acc[1][seq]], Kb5, Vb5)
        qs = Q.reshape(shape)[seq][:, :, head:head + 1].reshape(k * R, 1, d)
        kbs = Kb5[seq][:, :, head:head + 1].reshape(k * R, 1, d)
        vbs = Vb5[seq][:, :, head:head + 1].reshape(k * R, 1, d)
        ref, ref_lse = OR.verify([view], table, qs, kbs, vbs, 1 / math.sqrt(d))
        check(O[seq][:, head:head + 1], ref, wl, "seq %d head %d" % (seq, head))
        check_lse(lse[seq][:, head:head + 1], ref_lse)
    cache.close()
