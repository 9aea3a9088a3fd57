"""Pins of the fp64 oracle against facts outside itself (CPU only).

Each test names what it pins: a value the pages print, an identity the pages
state, a library routine (torch SDPA in fp64), a closed form, or brute force.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from oracle import oracle as OR
from tests.util import all_depth_rows, branch_rows, seq_planes

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small(R=4, H=2, d=16, W=8, k=4, decay=0.88, seed=7, dtype="f32"):
    return S.Workload("t", 1, R, H, d, W, k, 1, None, decay, seed, dtype, 256, k)


def run_oracle(wl, T, ws, k, mode=1, layer=0, seq=3, nseq=1):
    seqs = [seq_planes(wl, layer, seq + s, T, ws) for s in range(nseq)]
    table, Q, Kb, Vb = all_depth_rows(wl, layer, nseq, [seq + s for s in range(nseq)], k)
    O, lse = OR.verify(seqs, table, Q, Kb, Vb, 1 / math.sqrt(wl.d), mode)
    return O, lse, (seqs, table, Q, Kb, Vb)


def sdpa_row(q, keys, vals, scale):
    """torch SDPA in fp64 on an explicitly gathered key list (library routine)."""
    qt = torch.from_numpy(np.asarray(q, np.float64)).view(1, 1, 1, -1)
    kt = torch.from_numpy(np.asarray(keys, np.float64)).view(1, 1, len(keys), -1)
    vt = torch.from_numpy(np.asarray(vals, np.float64)).view(1, 1, len(vals), -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return o.view(-1).numpy()


def full_planes(wl, layer, seq, T):
    """Every plane 1..R of every position 0..T-1: [H][R][T][d] (the full cache)."""
    coef = S.coef_table(wl.decay, wl.R)
    k = S.planes(wl.seed, 0, layer, seq, range(wl.H), np.arange(1, wl.R + 1), np.arange(T), wl.d,
                 wl.R, coef, wl.bf16)
    v = S.planes(wl.seed, 1, layer, seq, range(wl.H), np.arange(1, wl.R + 1), np.arange(T), wl.d,
                 wl.R, coef, wl.bf16)
    return k, v


# --- P1: the page's memory figure --------------------------------------------------

def test_memory_fraction_matches_printed_value():
    g = json.load(open(os.path.join(GOLDEN, "memory_fraction.json")))
    f = OR.memory_fraction(g["T"], g["W"], g["R"], g["n_recurrent"], g["n_prelude"], g["n_coda"])
    assert round(100 * f, g["printed_decimals"]) == g["printed_percent"]


def test_memory_fraction_limits_and_store_count():
    # W >= T keeps everything; the store model's live-plane count equals the model.
    assert OR.memory_fraction(1024, 1024, 32, 4, 2, 2) == 1.0
    assert OR.memory_fraction(1024, 4096, 32, 4, 2, 2) == 1.0
    # W = 0 keeps one plane per position per layer
    assert OR.memory_fraction(1024, 0, 32, 4, 2, 2) == pytest.approx(8 / (4 + 4 * 32))
    for W in (0, 4, 64, 256, 1024):
        st = OR.OracleStore(1, 32, 1, 8, W, 1024 + 8, 1, 8, np.float32)
        K = np.zeros((1, 1, 1024, 32, 1, 8), np.float32)
        st.append([0], [1024], K, K)
        st.evict([0])
        live = st.live_planes(0)
        assert live / (32 * 1024) == pytest.approx(OR.memory_fraction(1024, W, 32, 1))


# --- P5: brute force, the library routine, closed forms ----------------------------

def test_naive_and_region_agree():
    wl = small()
    for T, ws in [(48, 40), (48, 0), (48, 48), (48, 60), (0, 0), (5, 2), (1, 1)]:
        O0, l0, _ = run_oracle(wl, T, ws, 4, mode=0, nseq=2)
        O1, l1, _ = run_oracle(wl, T, ws, 4, mode=1, nseq=2)
        assert np.abs(O0 - O1).max() < 1e-13
        assert np.abs(l0 - l1).max() < 1e-12


def test_against_torch_sdpa_on_gathered_keys():
    wl = small(R=5, H=3, d=8)
    T, ws, k = 20, 13, 3
    O, lse, (seqs, table, Q, Kb, Vb) = run_oracle(wl, T, ws, k)
    kf, vf = full_planes(wl, 0, 3, T)
    scale = 1 / math.sqrt(wl.d)
    for (seq, r, n, row0, stride) in table:
        for j in range(n):
            row = row0 + j * stride
            for h in range(wl.H):
                keys = [kf[h, (r if p >= ws else wl.R) - 1, p] for p in range(T)]
                vals = [vf[h, (r if p >= ws else wl.R) - 1, p] for p in range(T)]
                keys += [Kb[row0 + jj * stride, h] for jj in range(j + 1)]
                vals += [Vb[row0 + jj * stride, h] for jj in range(j + 1)]
                ref = sdpa_row(Q[row, h], keys, vals, scale)
                assert np.abs(O[row, h] - ref).max() < 1e-13


def test_pure_python_brute_force():
    wl = small(R=3, H=1, d=4, W=2, k=2, seed=11)
    T, ws, k = 5, 3, 2
    O, lse, (seqs, table, Q, Kb, Vb) = run_oracle(wl, T, ws, k)
    kf, vf = full_planes(wl, 0, 3, T)
    scale = 1 / math.sqrt(wl.d)
    for (seq, r, n, row0, stride) in table:
        for j in range(n):
            row = row0 + j * stride
            q = [float(x) for x in Q[row, 0]]
            keys, vals = [], []
            for p in range(T):
                plane = r if p >= ws else wl.R
                keys.append([float(x) for x in kf[0, plane - 1, p]])
                vals.append([float(x) for x in vf[0, plane - 1, p]])
            for jj in range(j + 1):
                keys.append([float(x) for x in Kb[row0 + jj * stride, 0]])
                vals.append([float(x) for x in Vb[row0 + jj * stride, 0]])
            s = [scale * sum(a * b for a, b in zip(q, kk)) for kk in keys]
            e = [math.exp(x) for x in s]
            z = sum(e)
            o = [sum(e[t] * vals[t][c] for t in range(len(e))) / z for c in range(wl.d)]
            assert max(abs(O[row, 0, c] - o[c]) for c in range(wl.d)) < 1e-12
            assert abs(lse[row, 0] - math.log(z)) < 1e-12


def test_closed_forms():
    wl = small()
    T, ws, k = 30, 26, 4
    O, lse, (seqs, table, Q, Kb, Vb) = run_oracle(wl, T, ws, k)
    scale = 1 / math.sqrt(wl.d)
    # single key: empty prefix, first token sees only itself -> o = v, lse = s
    O1, l1 = OR.verify([dict(seqs[0], T=0, ws=0, Kd=seqs[0]["Kd"][:, :0], Vd=seqs[0]["Vd"][:, :0],
                             Kw=seqs[0]["Kw"][:, :, :0], Vw=seqs[0]["Vw"][:, :, :0])],
                       table, Q, Kb, Vb, scale)
    for (seq, r, n, row0, stride) in table:
        assert np.array_equal(O1[row0], Vb[row0].astype(np.float64))
        np.testing.assert_allclose(l1[row0], scale * np.sum(Q[row0].astype(np.float64)
                                                            * Kb[row0], axis=-1), rtol=0, atol=1e-14)
    # equal scores (q = 0): o = mean of the visible values, lse = ln(#keys)
    Oz, lz = OR.verify(seqs, table, np.zeros_like(Q), Kb, Vb, scale)
    kd_v = seqs[0]["Vd"].astype(np.float64)
    kw_v = seqs[0]["Vw"].astype(np.float64)
    for (seq, r, n, row0, stride) in table:
        for j in range(n):
            row = row0 + j * stride
            vis = [kd_v[:, p] if (p < ws or r == wl.R) else kw_v[:, r - 1, p - ws] for p in range(T)]
            vis += [Vb[row0 + jj * stride].astype(np.float64) for jj in range(j + 1)]
            np.testing.assert_allclose(Oz[row], np.mean(vis, axis=0), rtol=0, atol=1e-14)
            np.testing.assert_allclose(lz[row], math.log(T + j + 1), rtol=0, atol=1e-14)
    # V == 1 everywhere: every output is exactly 1 up to rounding (rows sum to 1)
    ones = lambda a: np.ones_like(a)
    s1 = [dict(seqs[0], Vd=ones(seqs[0]["Vd"]), Vw=ones(seqs[0]["Vw"]))]
    O_1, _ = OR.verify(s1, table, Q, Kb, ones(Vb), scale)
    assert np.abs(O_1 - 1).max() < 1e-14


# --- P2 / P3: the window identities --------------------------------------------------

@pytest.mark.parametrize("R", [1, 4])
def test_window_covering_context_is_full_cache(R):
    wl = small(R=R, H=2, d=8)
    T, k = 24, 3
    O, _, (seqs, table, Q, Kb, Vb) = run_oracle(wl, T, 0, k)  # ws = 0: all positions in window
    kf, vf = full_planes(wl, 0, 3, T)
    scale = 1 / math.sqrt(wl.d)
    for (seq, r, n, row0, stride) in table:
        for j in range(n):
            row = row0 + j * stride
            for h in range(wl.H):
                keys = list(kf[h, r - 1]) + [Kb[row0 + jj * stride, h] for jj in range(j + 1)]
                vals = list(vf[h, r - 1]) + [Vb[row0 + jj * stride, h] for jj in range(j + 1)]
                assert np.abs(O[row, h] - sdpa_row(Q[row, h], keys, vals, scale)).max() <= 1e-13


def test_zero_window_is_deepest_plane_only():
    wl = small(R=4, H=2, d=8)
    T, k = 24, 3
    O, _, (seqs, table, Q, Kb, Vb) = run_oracle(wl, T, T, k)  # ws = T: nothing in window
    kf, vf = full_planes(wl, 0, 3, T)
    scale = 1 / math.sqrt(wl.d)
    for (seq, r, n, row0, stride) in table:
        for j in range(n):
            row = row0 + j * stride
            for h in range(wl.H):
                keys = list(kf[h, wl.R - 1]) + [Kb[row0 + jj * stride, h] for jj in range(j + 1)]
                vals = list(vf[h, wl.R - 1]) + [Vb[row0 + jj * stride, h] for jj in range(j + 1)]
                assert np.abs(O[row, h] - sdpa_row(Q[row, h], keys, vals, scale)).max() <= 1e-13


def test_single_plane_is_ordinary_causal_attention():
    wl = small(R=1, H=2, d=8)
    T, k = 17, 4
    O, _, (seqs, table, Q, Kb, Vb) = run_oracle(wl, T, 9, k)
    kf, vf = full_planes(wl, 0, 3, T)
    scale = 1 / math.sqrt(wl.d)
    q = torch.from_numpy(Q.astype(np.float64)).permute(1, 0, 2)[None]            # [1,H,k,d]
    kk = torch.from_numpy(np.concatenate([kf[:, 0], np.transpose(Kb, (1, 0, 2))], 1).astype(np.float64))[None]
    vv = torch.from_numpy(np.concatenate([vf[:, 0], np.transpose(Vb, (1, 0, 2))], 1).astype(np.float64))[None]
    mask = torch.ones(k, T + k, dtype=torch.bool).tril(diagonal=T)
    ref = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, attn_mask=mask, scale=scale)
    assert np.abs(O - ref[0].permute(1, 0, 2).numpy()).max() <= 1e-13


# --- P6: block independence ---------------------------------------------------------

def test_rows_ignore_other_depths_and_later_tokens():
    wl = small(R=4, H=2, d=8)
    T, ws, k = 20, 12, 4
    O, lse, (seqs, table, Q, Kb, Vb) = run_oracle(wl, T, ws, k)
    R = wl.R
    j0, r0 = 1, 2
    Kp, Vp = Kb.copy(), Vb.copy()
    rng = np.random.default_rng(0)
    for j in range(k):
        for r in range(1, R + 1):
            if r != r0 or j > j0:
                row = j * R + (r - 1)
                Kp[row] += rng.standard_normal(Kp[row].shape).astype(np.float32)
                Vp[row] += rng.standard_normal(Vp[row].shape).astype(np.float32)
    O2, l2 = OR.verify(seqs, table, Q, Kp, Vp, 1 / math.sqrt(wl.d))
    for j in range(j0 + 1):
        row = j * R + (r0 - 1)
        assert np.array_equal(O[row], O2[row]) and np.array_equal(lse[row], l2[row])
    assert not np.array_equal(O, O2)


@pytest.mark.parametrize("W", [4, 6, 16])
def test_batched_equals_one_token_at_a_time(W):
    """Verifying k tokens in one call == k calls of one token, where tokens 0..j-1
    were appended with all R planes (no evict) before token j."""
    wl = small(R=4, H=2, d=8, W=W, k=4)
    T, k, R = 21, 4, 4
    seq = 3
    coef = S.coef_table(wl.decay, R)
    st = OR.OracleStore(1, R, wl.H, wl.d, W, 64, 8, k, np.float64)
    allp = np.arange(T)
    K = np.transpose(S.planes(wl.seed, 0, 0, seq, range(wl.H), np.arange(1, R + 1), allp, wl.d, R,
                              coef, False), (2, 1, 0, 3))[None, None]     # [1][1][T][R][H][d]
    V = np.transpose(S.planes(wl.seed, 1, 0, seq, range(wl.H), np.arange(1, R + 1), allp, wl.d, R,
                              coef, False), (2, 1, 0, 3))[None, None]
    st.append([seq], [T], K, V)
    st.evict([seq])
    scale = 1 / math.sqrt(wl.d)
    table, Q, Kb, Vb = all_depth_rows(wl, 0, 1, [seq], k)
    views = [st.plane_view(0, b) for b in range(8)]
    tb = table.copy()
    tb[:, 0] = seq
    Ob, lb = OR.verify(views, tb, Q, Kb, Vb, scale)
    Kblk = Kb.reshape(k, R, wl.H, wl.d)
    Vblk = Vb.reshape(k, R, wl.H, wl.d)
    for j in range(k):
        s2 = OR.OracleStore(1, R, wl.H, wl.d, W, 64, 8, k, np.float64)
        s2.append([seq], [T], K, V)
        s2.evict([seq])
        if j:
            s2.append([seq], [j], Kblk[None, None, :j], Vblk[None, None, :j])
        v2 = [s2.plane_view(0, b) for b in range(8)]
        for r in range(1, R + 1):
            row = j * R + (r - 1)
            one = np.array([[seq, r, 1, 0, 1]], np.int32)
            O1, l1 = OR.verify(v2, one, Q[row:row + 1], Kb[row:row + 1], Vb[row:row + 1], scale)
            assert np.abs(O1[0] - Ob[row]).max() <= 1e-13
            assert np.abs(l1[0] - lb[row]).max() <= 1e-12


@pytest.mark.parametrize("W,k", [(4, 4), (8, 4), (3, 4), (1, 8)])
def test_accepted_block_keeps_all_planes_iff_window_covers_it(W, k):
    R, H, d = 4, 2, 8
    st = OR.OracleStore(1, R, H, d, W, 64, 2, k, np.float64)
    rng = np.random.default_rng(1)
    K0 = rng.standard_normal((1, 1, 10, R, H, d))
    st.append([1], [10], K0, K0)
    st.evict([1])
    Kb = rng.standard_normal((1, 1, k, R, H, d))
    Vb = rng.standard_normal((1, 1, k, R, H, d))
    st.append([1], [k], Kb, Vb)
    st.evict([1])
    T, ws = int(st.length[1]), int(st.wstart[1])
    for t in range(k):
        p = 10 + t
        live = p >= ws
        assert live == (t >= k - W)
        assert np.array_equal(st.kdeep[0, 1, :, p], Kb[0, 0, t, R - 1])
        if live:
            slot = p % st.Wcap
            assert np.array_equal(st.kwin[0, 1, :, :, slot], np.swapaxes(Kb[0, 0, t, :R - 1], 0, 1))
            assert np.array_equal(st.vwin[0, 1, :, :, slot], np.swapaxes(Vb[0, 0, t, :R - 1], 0, 1))


@pytest.mark.parametrize("W,k", [(4, 4), (64, 4), (8, 8), (3, 4), (1, 4), (7, 8)])
def test_sliding_reading_block_independent_iff_window_covers_block(W, k):
    deep = OR.sliding_block_reads_deepest(W, k)
    assert (not deep.any()) == (W >= k)


# --- P7: the generator's planes approach the deepest one as the page says -------

@pytest.mark.parametrize("key", ["huginn_per_loop", "raven_per_loop"])
def test_generator_decay(key):
    decay = json.load(open(os.path.join(GOLDEN, "plane_decay.json")))[key]
    R = 32
    coef = S.coef_table(decay, R)
    P = S.planes(5, 0, 0, 0, range(4), np.arange(1, R + 1), np.arange(256), 64, R, coef, False)
    dist = np.sqrt(((P - P[:, R - 1:R]) ** 2).sum(axis=(0, 2, 3)))
    ratios = dist[0:R - 2] / dist[1:R - 1]   # distance to plane R shrinks by `decay` per loop
    assert np.all(np.abs(ratios - decay) < 0.02)


# --- rollback to the confirmed prefix (LoopSpec article, section on the second branch) -----

def _block(rng, L, n, R, H, d):
    return rng.standard_normal((L, 1, n, R, H, d)), rng.standard_normal((L, 1, n, R, H, d))


def _all_depth_verify(st, seq, rng, R, H, d, k=3):
    """Verify k fresh draft tokens at every depth over sequence seq of store st."""
    nrows = k * R
    Q = rng.standard_normal((nrows, H, d))
    Kb = rng.standard_normal((nrows, H, d))
    Vb = rng.standard_normal((nrows, H, d))
    table = np.array([(seq, r, k, r - 1, R) for r in range(1, R + 1)], np.int32)
    views = [st.plane_view(0, b) for b in range(st.Bmax)]
    return OR.verify(views, table, Q, Kb, Vb, 1 / math.sqrt(d))


@pytest.mark.parametrize("W,kmax", [(8, 4), (4, 4), (2, 4), (0, 3), (1, 6), (16, 8)])
def test_rollback_returns_to_confirmed_prefix(W, kmax):
    """Decode steps that append a speculative block (all planes), evict, then roll
    back to the accepted length leave a store that verifies exactly like one that
    only ever appended the accepted tokens (append + evict per step).  Covers
    windows longer and shorter than the speculative block (W >= n and W < n)."""
    L, R, H, d, Tmax, B, seq = 1, 4, 2, 8, 200, 3, 1
    rng = np.random.default_rng(1000 + 10 * W + kmax)
    spec = OR.OracleStore(L, R, H, d, W, Tmax, B, kmax, np.float64)
    conf = OR.OracleStore(L, R, H, d, W, Tmax, B, kmax, np.float64)
    K0, V0 = _block(rng, L, 23, R, H, d)
    for st in (spec, conf):
        st.append([seq], [23], K0, V0)   # prefill: more than Wcap positions
        st.evict([seq])
    for step in range(12):
        n = int(rng.integers(1, kmax + 1))
        acc = int(rng.integers(0, n + 1))
        K, V = _block(rng, L, n, R, H, d)
        spec.append([seq], [n], K, V)
        spec.evict([seq])
        T_conf = int(conf.length[seq]) + acc
        spec.truncate([seq], [T_conf])
        conf.append([seq], [acc], K, V)  # the accepted tokens are the first acc of the block
        conf.evict([seq])
        assert int(spec.length[seq]) == int(conf.length[seq]) == T_conf
        assert int(spec.wstart[seq]) == int(conf.wstart[seq]), (step, spec.wstart[seq], conf.wstart[seq])
        vs, vc = spec.plane_view(0, seq), conf.plane_view(0, seq)
        for key in ("Kd", "Vd", "Kw", "Vw"):
            assert np.array_equal(vs[key], vc[key]), (step, key)
        s = int(rng.integers(0, 2 ** 31))
        Os, ls = _all_depth_verify(spec, seq, np.random.default_rng(s), R, H, d)
        Oc, lc = _all_depth_verify(conf, seq, np.random.default_rng(s), R, H, d)
        assert np.abs(Os - Oc).max() <= 1e-13 and np.abs(ls - lc).max() <= 1e-13


def test_rollback_deeper_than_ring_keeps_only_intact_positions():
    """Rolling back more than kmax positions: the rejected tokens overwrote ring
    slots of confirmed positions, which then read at the deepest plane only.  Every
    position left in the window still holds its own planes (the state is valid),
    and the window is as long as the ring allows."""
    L, R, H, d, W, kmax, Tmax, seq = 1, 3, 2, 4, 4, 2, 64, 0
    rng = np.random.default_rng(5)
    st = OR.OracleStore(L, R, H, d, W, Tmax, 1, kmax, np.float64)
    K0, V0 = _block(rng, L, 12, R, H, d)
    st.append([seq], [12], K0, V0)
    st.evict([seq])
    for _ in range(3):   # 3 * kmax = 6 speculative positions, ring capacity Wcap = 6
        K, V = _block(rng, L, kmax, R, H, d)
        st.append([seq], [kmax], K, V)
        st.evict([seq])
    st.truncate([seq], [12])
    T, ws, rf = int(st.length[seq]), int(st.wstart[seq]), int(st.rfloor[seq])
    assert T == 12 and rf == 12 and ws == 12   # every slot of 8..11 was overwritten
    # A shorter rollback: positions 12..13 kept, 14..17 rejected.
    st2 = OR.OracleStore(L, R, H, d, W, Tmax, 1, kmax, np.float64)
    st2.append([seq], [12], K0, V0)
    st2.evict([seq])
    blocks = [_block(rng, L, kmax, R, H, d) for _ in range(3)]
    for K, V in blocks:
        st2.append([seq], [kmax], K, V)
        st2.evict([seq])
    st2.truncate([seq], [14])
    T, ws = int(st2.length[seq]), int(st2.wstart[seq])
    assert T == 14 and ws == 18 - st2.Wcap == 12   # positions 10, 11 overwritten by 16, 17
    view = st2.plane_view(0, seq)
    for i, p in enumerate(range(ws, T)):
        t = p - 12
        K, V = blocks[t // kmax]
        assert np.array_equal(view["Kw"][:, :, i], np.swapaxes(K[0, 0, t % kmax, :R - 1], 0, 1))


def test_rollback_past_window_start_and_noop():
    L, R, H, d, W, kmax, seq = 1, 2, 1, 4, 3, 2, 0
    rng = np.random.default_rng(6)
    st = OR.OracleStore(L, R, H, d, W, 64, 1, kmax, np.float64)
    K0, V0 = _block(rng, L, 10, R, H, d)
    st.append([seq], [10], K0, V0)
    st.evict([seq])
    before = (int(st.length[seq]), int(st.wstart[seq]), int(st.rfloor[seq]))
    st.truncate([seq], [10])
    st.truncate([seq], [50])
    assert (int(st.length[seq]), int(st.wstart[seq]), int(st.rfloor[seq])) == before
    st.truncate([seq], [2])            # below the ring floor: empty window
    assert (int(st.length[seq]), int(st.wstart[seq]), int(st.rfloor[seq])) == (2, 2, 2)


# --- the sliding-window reading (the RIPE abstract's fifth sentence, per query) -----

def _sliding(wl, T, ws, k, W, seq=3, layer=0):
    views = [seq_planes(wl, layer, seq, T, ws)]
    table, Q, Kb, Vb = all_depth_rows(wl, layer, 1, [seq], k)
    O, lse = OR.verify_sliding(views, table, Q, Kb, Vb, W, 1 / math.sqrt(wl.d))
    return O, lse, (views, table, Q, Kb, Vb)


def test_sliding_window_covering_everything_is_full_cache():
    wl = small(R=4, H=2, d=8)
    T, k = 20, 3
    O, _, (views, table, Q, Kb, Vb) = _sliding(wl, T, 0, k, W=T + k + 5)
    kf, vf = full_planes(wl, 0, 3, T)
    scale = 1 / math.sqrt(wl.d)
    for (seq, r, n, row0, stride) in table:
        for j in range(n):
            row = row0 + j * stride
            for h in range(wl.H):
                keys = list(kf[h, r - 1]) + [Kb[row0 + jj * stride, h] for jj in range(j + 1)]
                vals = list(vf[h, r - 1]) + [Vb[row0 + jj * stride, h] for jj in range(j + 1)]
                assert np.abs(O[row, h] - sdpa_row(Q[row, h], keys, vals, scale)).max() <= 1e-13


def test_sliding_zero_window_reads_the_deepest_plane_only():
    """W = 0: every committed position and every draft token, the query's own
    included, at plane R (a draft token's plane R is its depth-R row)."""
    wl = small(R=4, H=2, d=8)
    T, k = 20, 3
    R = wl.R
    O, _, (views, table, Q, Kb, Vb) = _sliding(wl, T, T, k, W=0)
    kf, vf = full_planes(wl, 0, 3, T)
    scale = 1 / math.sqrt(wl.d)
    for (seq, r, n, row0, stride) in table:
        for j in range(n):
            row = row0 + j * stride
            for h in range(wl.H):
                keys = list(kf[h, R - 1]) + [Kb[jj * R + R - 1, h] for jj in range(j + 1)]
                vals = list(vf[h, R - 1]) + [Vb[jj * R + R - 1, h] for jj in range(j + 1)]
                assert np.abs(O[row, h] - sdpa_row(Q[row, h], keys, vals, scale)).max() <= 1e-13


def test_sliding_pure_python_brute_force():
    wl = small(R=3, H=1, d=4, W=2, k=3, seed=11)
    T, ws, k, W, R = 6, 3, 3, 2, 3
    O, lse, (views, table, Q, Kb, Vb) = _sliding(wl, T, ws, k, W)
    kf, vf = full_planes(wl, 0, 3, T)
    scale = 1 / math.sqrt(wl.d)
    for (seq, r, n, row0, stride) in table:
        for j in range(n):
            row = row0 + j * stride
            q = [float(x) for x in Q[row, 0]]
            keys, vals = [], []
            for p in range(T):
                plane = r if (p >= T + j - W + 1 and p >= ws) else R
                keys.append([float(x) for x in kf[0, plane - 1, p]])
                vals.append([float(x) for x in vf[0, plane - 1, p]])
            for jj in range(j + 1):
                src = row0 + jj * stride if jj >= j - W + 1 else jj * R + R - 1
                keys.append([float(x) for x in Kb[src, 0]])
                vals.append([float(x) for x in Vb[src, 0]])
            s = [scale * sum(a * b for a, b in zip(q, kk)) for kk in keys]
            e = [math.exp(x) for x in s]
            z = sum(e)
            o = [sum(e[t] * vals[t][c] for t in range(len(e))) / z for c in range(wl.d)]
            assert max(abs(O[row, 0, c] - o[c]) for c in range(wl.d)) < 1e-12
            assert abs(lse[row, 0] - math.log(z)) < 1e-12


@pytest.mark.parametrize("W,k", [(4, 4), (6, 4), (3, 4), (1, 4)])
def test_sliding_block_independence_iff_window_covers_block(W, k):
    """BI4 as a computation: the depth-R rows' block planes reach a depth-r < R row
    only through draft tokens read at plane R, which happens iff W < k."""
    wl = small(R=4, H=2, d=8, W=W, k=k)
    T, R = 20, wl.R
    O, _, (views, table, Q, Kb, Vb) = _sliding(wl, T, T - W, k, W)
    Kp, Vp = Kb.copy(), Vb.copy()
    rng = np.random.default_rng(2)
    for j in range(k):
        Kp[j * R + R - 1] += rng.standard_normal(Kp[0].shape).astype(np.float32)
        Vp[j * R + R - 1] += rng.standard_normal(Vp[0].shape).astype(np.float32)
    O2, _ = OR.verify_sliding(views, table, Q, Kp, Vp, W, 1 / math.sqrt(wl.d))
    shallow = [j * R + r - 1 for j in range(k) for r in range(1, R)]
    changed = not np.array_equal(O[shallow], O2[shallow])
    assert changed == (W < k)
    assert changed == bool(OR.sliding_block_reads_deepest(W, k).any())


# --- branch forks (LoopSpec article, deployment section: a KV cache per branch) -----

@pytest.mark.parametrize("T0,W,kmax", [(130, 8, 4), (64, 16, 8), (5, 4, 4), (200, 0, 3)])
def test_fork_equals_a_store_that_appended_the_branch(T0, W, kmax):
    """A fork that appends its branch's tokens reads exactly what a store that
    appended the parent's tokens and then the branch's would read; the parent is
    untouched; releasing the fork empties it."""
    L, R, H, d, Tmax, B = 1, 4, 2, 8, 400, 4
    rng = np.random.default_rng(T0 + W)
    st = OR.OracleStore(L, R, H, d, W, Tmax, B, kmax, np.float64)
    ref = OR.OracleStore(L, R, H, d, W, Tmax, B, kmax, np.float64)
    K0, V0 = _block(rng, L, T0, R, H, d)
    for s in (st, ref):
        s.append([0], [T0], K0, V0)
        s.evict([0])
    parent_before = {k: v.copy() for k, v in st.plane_view(0, 0).items() if isinstance(v, np.ndarray)}
    st.fork([0], [2])
    assert not st.flagged
    for step in range(3):
        n = int(rng.integers(1, kmax + 1))
        K, V = _block(rng, L, n, R, H, d)
        st.append([2], [n], K, V)
        st.evict([2])
        ref.append([0], [n], K, V)
        ref.evict([0])
        vs, vr = st.plane_view(0, 2), ref.plane_view(0, 0)
        assert vs["T"] == vr["T"] and vs["ws"] == vr["ws"]
        for key in ("Kd", "Vd", "Kw", "Vw"):
            assert np.array_equal(vs[key], vr[key]), (step, key)
        s1 = int(rng.integers(0, 2 ** 31))
        Os, _ = _all_depth_verify(st, 2, np.random.default_rng(s1), R, H, d)
        Or, _ = _all_depth_verify(ref, 0, np.random.default_rng(s1), R, H, d)
        assert np.array_equal(Os[:], Or[:])
    after = st.plane_view(0, 0)
    for k, v in parent_before.items():
        assert np.array_equal(after[k], v)
    st.reset([2])
    assert st.length[2] == 0 and st.base[2] == 2 and st.fpos[2] == 0


def test_fork_rules():
    L, R, H, d = 1, 3, 1, 4
    st = OR.OracleStore(L, R, H, d, 4, 300, 4, 4, np.float64)
    rng = np.random.default_rng(9)
    K0, V0 = _block(rng, L, 150, R, H, d)
    st.append([0], [150], K0, V0)
    st.fork([0], [1])
    assert not st.flagged and st.fpos[1] == 128 and st.base[1] == 0
    st.fork([1], [2])                  # a fork of a fork
    assert st.flagged
    st.flagged = False
    st.truncate([1], [100])            # below the fork position
    assert st.flagged and st.length[1] == 150
    st.flagged = False
    st.truncate([1], [140])            # above it: an ordinary rollback
    assert not st.flagged and st.length[1] == 140
