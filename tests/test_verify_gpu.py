"""Verify-attention on the GPU against the fp64 oracle, on the five workloads,
their edge cases and the method's invariants.  Every call goes through the C ABI."""
import math

import numpy as np
import pytest
import torch

from depth_planed_kv_b200 import synth as S
from oracle import oracle as OR
from tests.gpu_util import (TOL, check, check_lse, fill, make_cache, oracle_all_depths, oracle_units,
                            run_all_depths, to_dev, torch_dtype)
from tests.util import all_depth_rows, branch_rows, errors, seq_planes

pytestmark = pytest.mark.gpu


# --- the tiny fp32 workload: every element -----------------------------------------

def test_tiny_f32_all_depths():
    wl = S.tiny()
    cache = make_cache(wl)
    fill(cache, wl, [wl.ctx])
    _, O, lse, _ = run_all_depths(cache, wl, 0, 1, wl.k)
    ref, ref_lse = oracle_all_depths(wl, 0, 1, wl.k, [wl.ctx], [wl.ctx - wl.W])
    check(O, ref, wl, "tiny")
    assert np.abs(lse - ref_lse).max() < 1e-5
    assert cache.ripe_get_device_error() == 0


# --- Huginn-shaped: all heads of two layers ----------------------------------------

@pytest.fixture(scope="module")
def huginn_cache():
    wl = S.huginn()
    cache = make_cache(wl)
    fill(cache, wl, [wl.ctx])
    yield wl, cache
    cache.close()


@pytest.mark.parametrize("layer", [0, 3])
def test_huginn_all_heads(huginn_cache, layer):
    wl, cache = huginn_cache
    _, O, lse, _ = run_all_depths(cache, wl, layer, 1, wl.k)
    heads = np.arange(wl.H) if layer == 0 else np.array([0, 17, 54])
    ref, ref_lse = oracle_all_depths(wl, layer, 1, wl.k, [wl.ctx], [wl.ctx - wl.W], heads=heads)
    check(O[:, heads], ref, wl, "huginn layer %d" % layer)
    check_lse(lse[:, heads], ref_lse)
    assert cache.ripe_get_device_error() == 0


def test_huginn_values_all_one_give_ones(huginn_cache):
    """Rows sum to 1: with every value vector equal to 1 the output is 1."""
    wl, cache = huginn_cache
    buf = cache.buffers()
    saved = (buf["vdeep"][1].clone(), buf["vwin"][1].clone())
    buf["vdeep"][1].fill_(1.0)
    buf["vwin"][1].fill_(1.0)
    table, Q, Kb, Vb = all_depth_rows(wl, 1, 1, [0], wl.k)
    shape = (1, wl.k, wl.R, wl.H, wl.d)
    O = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    cache.ripe_verify_attn_all_depths(1, torch.tensor([0], dtype=torch.int32, device="cuda"), wl.k,
                                      to_dev(Q.reshape(shape), wl), to_dev(Kb.reshape(shape), wl),
                                      torch.ones(shape, dtype=torch.bfloat16, device="cuda"), O)
    torch.cuda.synchronize()
    buf["vdeep"][1].copy_(saved[0])
    buf["vwin"][1].copy_(saved[1])
    assert torch.all(O.float() == 1.0)


def test_huginn_rows_ignore_other_depths_and_later_tokens(huginn_cache):
    """Block independence on the GPU: perturbing block planes at other depths, or
    later tokens, leaves a row's output bitwise unchanged."""
    wl, cache = huginn_cache
    table, O, lse, (Q, Kb, Vb) = run_all_depths(cache, wl, 2, 1, wl.k)
    R, k = wl.R, wl.k
    j0, r0 = 1, 7
    rng = np.random.default_rng(3)
    Kp, Vp = Kb.copy(), Vb.copy()
    for j in range(k):
        for r in range(1, R + 1):
            if r != r0 or j > j0:
                row = j * R + r - 1
                Kp[row] = S.round_bf16(Kp[row] + rng.standard_normal(Kp[row].shape).astype(np.float32))
                Vp[row] = S.round_bf16(Vp[row] + rng.standard_normal(Vp[row].shape).astype(np.float32))
    shape = (1, k, R, wl.H, wl.d)
    O2 = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    cache.ripe_verify_attn_all_depths(2, torch.tensor([0], dtype=torch.int32, device="cuda"), k,
                                      to_dev(Q.reshape(shape), wl), to_dev(Kp.reshape(shape), wl),
                                      to_dev(Vp.reshape(shape), wl), O2)
    torch.cuda.synchronize()
    O2 = O2.float().cpu().numpy().reshape(k * R, wl.H, wl.d)
    for j in range(j0 + 1):
        row = j * R + r0 - 1
        assert np.array_equal(O[row], O2[row])
    assert not np.array_equal(O, O2)


# --- window sweep at the Huginn shape ---------------------------------------------

@pytest.mark.parametrize("kernel", [1, 2])   # persistent / cluster kernel
@pytest.mark.parametrize("W", S.SWEEP_W)
def test_window_sweep(W, kernel):
    wl = S.sweep(W)
    wl.layers = 1
    cache = make_cache(wl, kernel=kernel)
    fill(cache, wl, [wl.ctx])
    _, O, lse, _ = run_all_depths(cache, wl, 0, 1, wl.k)
    heads = np.array([0, 9, 31, 54])
    ws = max(0, wl.ctx - W)
    ref, ref_lse = oracle_all_depths(wl, 0, 1, wl.k, [wl.ctx], [ws], heads=heads)
    check(O[:, heads], ref, wl, "sweep W=%d" % W)
    check_lse(lse[:, heads], ref_lse)
    cache.close()


# --- LoopSpec mixed-depth branch list ----------------------------------------------

def test_loopspec_mixed_batch():
    wl = S.mixed()
    ctx, branches = S.mixed_structure(wl)
    cache = make_cache(wl)
    fill(cache, wl, ctx)
    table, Q, Kb, Vb = branch_rows(wl, 0, branches, list(range(wl.nseq)))
    from depth_planed_kv_b200.ripe import branch_table
    tb = branch_table([tuple(t) for t in table])
    O = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full(Q.shape[:2], float("nan"), device="cuda")
    cache.ripe_verify_attn(0, tb, len(table), to_dev(Q, wl), to_dev(Kb, wl), to_dev(Vb, wl), O, lse)
    torch.cuda.synchronize()
    O = O.float().cpu().numpy()
    lse = lse.cpu().numpy()
    ws = np.maximum(ctx - wl.W, 0)
    seq_sample = [0, 5, 17, 40, 63]
    heads = np.array([0, 13, 31])
    ref = oracle_units(wl, 0, ctx, ws, branches, seq_sample, heads)
    for bi, (ro, rl) in ref.items():
        t = table[bi]
        check(O[t[3]:t[3] + t[2]][:, heads], ro, wl, "branch %d" % bi)
        check_lse(lse[t[3]:t[3] + t[2]][:, heads], rl)
    assert cache.ripe_get_device_error() == 0
    cache.close()


# --- long context: sampled units of the full-size launch -----------------------------

def test_long_context_sampled_units():
    wl = S.long_context()
    cache = make_cache(wl)
    fill(cache, wl, [wl.ctx] * wl.nseq)
    _, O, lse, _ = run_all_depths(cache, wl, 0, wl.nseq, wl.k)
    R, k = wl.R, wl.k
    for s, heads in [(0, [0]), (11, [19]), (15, [31])]:
        ref, ref_lse = oracle_all_depths(wl, 0, 1, k, [wl.ctx], [wl.ctx - wl.W], seqs=[s], heads=heads)
        rows = slice(s * k * R, (s + 1) * k * R)
        check(O[rows][:, heads], ref, wl, "long seq %d" % s)
        check_lse(lse[rows][:, heads], ref_lse)
    cache.close()


# --- edge cases ------------------------------------------------------------------

@pytest.mark.parametrize("T,W", [(0, 4), (1, 0), (5, 64), (37, 7), (200, 0), (200, 300)])
def test_edge_contexts_f32(T, W):
    wl = S.Workload("edge", 1, 3, 2, 16, W, 5, 2, T, 0.88, 31, "f32", 512, 5)
    cache = make_cache(wl)
    fill(cache, wl, [T, max(T - 1, 0)])
    _, O, lse, _ = run_all_depths(cache, wl, 0, 2, wl.k)
    Ts = [T, max(T - 1, 0)]
    ws = [max(0, t - W) for t in Ts]
    ref, ref_lse = oracle_all_depths(wl, 0, 2, wl.k, Ts, ws)
    check(O, ref, wl, "T=%d W=%d" % (T, W))
    assert np.abs(lse - ref_lse).max() < 1e-5
    cache.close()


def test_ragged_branches_and_long_blocks_bf16():
    """Branches of 0..37 tokens (more than one row chunk), mixed depths, ragged
    contexts, and the ctx_len override below the committed length."""
    wl = S.Workload("ragged", 1, 6, 3, 64, 9, 37, 3, None, 0.81, 55, "bf16", 400, 37)
    ctx = np.array([300, 17, 0])
    cache = make_cache(wl)
    fill(cache, wl, ctx)
    branches = [S.BranchSpec(0, 6, 37, 0, 0), S.BranchSpec(0, 2, 5, 1, 1), S.BranchSpec(1, 3, 0, 2, 2),
                S.BranchSpec(1, 6, 19, 0, 0), S.BranchSpec(1, 1, 1, 3, 3), S.BranchSpec(2, 4, 16, 1, 1),
                S.BranchSpec(2, 6, 17, 0, 0)]
    table, Q, Kb, Vb = branch_rows(wl, 0, branches, [0, 1, 2])
    from depth_planed_kv_b200.ripe import branch_table
    tb = branch_table([tuple(t) for t in table])
    ctx_len = torch.tensor([250, 17, 0], dtype=torch.int32, device="cuda")
    O = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full(Q.shape[:2], float("nan"), device="cuda")
    cache.ripe_verify_attn(0, tb, len(table), to_dev(Q, wl), to_dev(Kb, wl), to_dev(Vb, wl), O, lse,
                           ctx_len=ctx_len)
    torch.cuda.synchronize()
    O = O.float().cpu().numpy()
    ws = np.maximum(ctx - wl.W, 0)
    T_eff = np.array([250, 17, 0])
    views = [seq_planes(wl, 0, s, int(T_eff[s]), int(ws[s])) for s in range(3)]
    ref, ref_lse = OR.verify(views, table, Q, Kb, Vb, 1 / math.sqrt(wl.d))
    check(O, ref, wl, "ragged")
    assert np.abs(lse.cpu().numpy() - ref_lse).max() < 2e-3
    assert cache.ripe_get_device_error() == 0
    cache.close()


def test_batched_equals_one_token_at_a_time_gpu():
    """k tokens verified in one call == k calls of one token with tokens 0..j-1
    committed by ripe_append (all planes) before token j."""
    wl = S.Workload("bi2", 1, 4, 2, 32, 6, 4, 1, 40, 0.88, 9, "f32", 64, 4)
    R, k = wl.R, wl.k
    cache = make_cache(wl)
    fill(cache, wl, [wl.ctx])
    table, O, lse, (Q, Kb, Vb) = run_all_depths(cache, wl, 0, 1, k)
    Kblk = torch.from_numpy(Kb.reshape(1, 1, k, R, wl.H, wl.d)).cuda()
    Vblk = torch.from_numpy(Vb.reshape(1, 1, k, R, wl.H, wl.d)).cuda()
    from depth_planed_kv_b200.ripe import branch_table
    ids = torch.tensor([0], dtype=torch.int32, device="cuda")
    for j in range(k):
        c2 = make_cache(wl)
        fill(c2, wl, [wl.ctx])
        if j:
            c2.ripe_append(ids, torch.tensor([j], dtype=torch.int32, device="cuda"),
                           Kblk[:, :, :j].contiguous(), Vblk[:, :, :j].contiguous())
        for r in range(1, R + 1):
            row = j * R + r - 1
            o1 = torch.empty(1, wl.H, wl.d, device="cuda")
            c2.ripe_verify_attn(0, branch_table([(0, r, 1, 0, 1)]), 1, to_dev(Q[row:row + 1], wl),
                                to_dev(Kb[row:row + 1], wl), to_dev(Vb[row:row + 1], wl), o1)
            torch.cuda.synchronize()
            a, rel = errors(o1.cpu().numpy()[0], O[row])
            assert a <= 1e-5 and rel <= 1e-5
        c2.close()
    cache.close()


@pytest.mark.parametrize("d", [64, 96, 128])
def test_many_rows_per_sequence_branch_list(d):
    """More than 128 query rows for one sequence (several row tiles of the deep
    kernel), next to a sequence with few rows."""
    wl = S.Workload("rows", 1, 8, 3, d, 16, 60, 2, None, 0.88, 61, "bf16", 700, 60)
    ctx = np.array([650, 130])
    cache = make_cache(wl)
    fill(cache, wl, ctx)
    branches = [S.BranchSpec(0, 8, 60, 0, 0), S.BranchSpec(0, 2, 60, 1, 1), S.BranchSpec(0, 5, 37, 2, 2),
                S.BranchSpec(1, 8, 9, 0, 0), S.BranchSpec(1, 4, 3, 1, 1)]
    table, Q, Kb, Vb = branch_rows(wl, 0, branches, [0, 1])
    from depth_planed_kv_b200.ripe import branch_table
    O = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full(Q.shape[:2], float("nan"), device="cuda")
    cache.ripe_verify_attn(0, branch_table([tuple(t) for t in table]), len(table), to_dev(Q, wl),
                           to_dev(Kb, wl), to_dev(Vb, wl), O, lse)
    torch.cuda.synchronize()
    ws = np.maximum(ctx - wl.W, 0)
    views = [seq_planes(wl, 0, s, int(ctx[s]), int(ws[s])) for s in range(2)]
    ref, ref_lse = OR.verify(views, table, Q, Kb, Vb, 1 / math.sqrt(wl.d))
    check(O.float().cpu().numpy(), ref, wl, "many rows d=%d" % d)
    check_lse(lse.cpu().numpy(), ref_lse)
    assert cache.ripe_get_device_error() == 0
    cache.close()


def test_all_depths_more_than_256_rows():
    """k*R = 9*32 = 288 rows per sequence and head: two 128-row M tiles per CTA
    plus a second row tile."""
    wl = S.Workload("k9", 1, 32, 2, 128, 32, 9, 2, 300, 0.88, 71, "bf16", 400, 9)
    cache = make_cache(wl)
    fill(cache, wl, [300, 211])
    _, O, lse, _ = run_all_depths(cache, wl, 0, 2, wl.k)
    ref, ref_lse = oracle_all_depths(wl, 0, 2, wl.k, [300, 211], [300 - 32, 211 - 32])
    check(O, ref, wl, "k=9 all depths")
    check_lse(lse, ref_lse)
    assert cache.ripe_get_device_error() == 0
    cache.close()
