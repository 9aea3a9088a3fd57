"""Seeded inputs arranged into the layouts the C ABI and the fp64 oracle take.

Nothing here computes attention or touches the store: it calls the generator in
``synth`` and places its values into row layouts -- the all-depths
[nseq][k][R][H][d] rows, a branch list's contiguous rows, and the logical view of
one sequence's store that the oracle reads (plane R of positions 0..T-1, planes
1..R-1 of the positions from min(ws,T) on).  The benchmark, the smoke check and
the tests share it so that the GPU and the oracle see the same values.
"""
from __future__ import annotations

import numpy as np

from depth_planed_kv_b200 import synth as S


def seq_planes(wl: S.Workload, layer: int, seq: int, T: int, ws: int, heads=None):
    """The oracle's view of one sequence's store, drawn straight from the generator.

    Plane R of positions 0..T-1 and planes 1..R-1 of positions min(ws,T)..T-1.
    """
    heads = np.arange(wl.H) if heads is None else np.asarray(heads)
    coef = S.coef_table(wl.decay, wl.R)
    lo = min(ws, T)
    pos = np.arange(T)
    kd = S.planes(wl.seed, 0, layer, seq, heads, [wl.R], pos, wl.d, wl.R, coef, wl.bf16)[:, 0]
    vd = S.planes(wl.seed, 1, layer, seq, heads, [wl.R], pos, wl.d, wl.R, coef, wl.bf16)[:, 0]
    wpos = np.arange(lo, T)
    planes = np.arange(1, wl.R)
    if len(planes) and len(wpos):
        kw = S.planes(wl.seed, 0, layer, seq, heads, planes, wpos, wl.d, wl.R, coef, wl.bf16)
        vw = S.planes(wl.seed, 1, layer, seq, heads, planes, wpos, wl.d, wl.R, coef, wl.bf16)
    else:
        kw = np.zeros((len(heads), max(wl.R - 1, 0), len(wpos), wl.d), np.float32)
        vw = kw.copy()
    return {"T": T, "ws": ws, "R": wl.R, "Kd": kd, "Vd": vd, "Kw": kw, "Vw": vw}


def branch_rows(wl: S.Workload, layer: int, branches, seqs_global, heads=None):
    """Q, Kblk, Vblk [nrows][H][d] and the int branch table for a branch list.

    ``branches`` are synth.BranchSpec with ``seq`` the local sequence index;
    ``seqs_global[seq]`` is the sequence id the generator is keyed on.  Rows of
    a branch are contiguous, branches in list order (row_stride 1).
    """
    heads = np.arange(wl.H) if heads is None else np.asarray(heads)
    coef = S.coef_table(wl.decay, wl.R)
    nrows = sum(b.ntok for b in branches)
    Q = np.zeros((nrows, len(heads), wl.d), np.float32)
    Kb = np.zeros_like(Q)
    Vb = np.zeros_like(Q)
    table = np.zeros((len(branches), 5), np.int32)
    row = 0
    for i, b in enumerate(branches):
        g = int(seqs_global[b.seq])
        toks = np.arange(b.ntok)
        Q[row:row + b.ntok] = S.queries(wl.seed, layer, b.qslot, g, heads, toks, wl.d, wl.bf16)
        bp = S.block_positions(b.bslot, b.ntok)
        kb = S.planes(wl.seed, 0, layer, g, heads, [b.depth], bp, wl.d, wl.R, coef, wl.bf16)
        vb = S.planes(wl.seed, 1, layer, g, heads, [b.depth], bp, wl.d, wl.R, coef, wl.bf16)
        Kb[row:row + b.ntok] = np.transpose(kb[:, 0], (1, 0, 2))
        Vb[row:row + b.ntok] = np.transpose(vb[:, 0], (1, 0, 2))
        table[i] = (b.seq, b.depth, b.ntok, row, 1)
        row += b.ntok
    return table, Q, Kb, Vb


def all_depth_rows(wl: S.Workload, layer: int, nseq: int, seqs_global, k: int, heads=None):
    """All-depths layout [nseq][k][R][H][d] flattened to rows, and its branch table.

    Row of (sequence s, token j, depth r) = (s*k + j)*R + (r-1); branch (s, r)
    has row0 = s*k*R + r-1 and row_stride R.
    """
    heads = np.arange(wl.H) if heads is None else np.asarray(heads)
    coef = S.coef_table(wl.decay, wl.R)
    R, d = wl.R, wl.d
    Q = np.zeros((nseq, k, R, len(heads), d), np.float32)
    Kb = np.zeros_like(Q)
    Vb = np.zeros_like(Q)
    toks = np.arange(k)
    bp = S.block_positions(0, k)
    for s in range(nseq):
        g = int(seqs_global[s])
        kb = S.planes(wl.seed, 0, layer, g, heads, np.arange(1, R + 1), bp, d, R, coef, wl.bf16)
        vb = S.planes(wl.seed, 1, layer, g, heads, np.arange(1, R + 1), bp, d, R, coef, wl.bf16)
        Kb[s] = np.transpose(kb, (2, 1, 0, 3))
        Vb[s] = np.transpose(vb, (2, 1, 0, 3))
        for r in range(1, R + 1):
            Q[s, :, r - 1] = S.queries(wl.seed, layer, r - 1, g, heads, toks, d, wl.bf16)
    table = np.array([(s, r, k, s * k * R + (r - 1), R) for s in range(nseq) for r in range(1, R + 1)],
                     dtype=np.int32)
    nrows = nseq * k * R
    return (table, Q.reshape(nrows, len(heads), d), Kb.reshape(nrows, len(heads), d),
            Vb.reshape(nrows, len(heads), d))
