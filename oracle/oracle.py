"""fp64 CPU oracle for RIPE verify-attention, the RIPE store and its memory model.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline use this package; the product library never imports it and shares no
code with it.

Sources (each function names the passage it follows):
  * the RIPE abstract (zhuanzhiai.com mirror): R KV planes per recurrent layer;
    the RIPE store (deepest plane everywhere, all planes in a window of recent
    positions); 11.9 % of the full cache at W=64, T=1024 on Huginn; windows at
    least as long as the draft block make batched verification block-independent;
  * the LoopSpec article (rit.work): branches at different recurrent depths in
    one batched call; rollback to the confirmed prefix.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ripe_oracle.c")
_LIB = os.path.join(_HERE, "libripe_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, fp64, OpenMP over independent (branch, head) units)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        lib.oracle_verify.argtypes = [ctypes.c_int] * 4 + [P] * 8 + [ctypes.c_int, P, ctypes.c_int,
                                                                     P, P, P, ctypes.c_double,
                                                                     ctypes.c_int, P, P]
        lib.oracle_verify.restype = ctypes.c_int
        lib.oracle_verify_sliding.argtypes = [ctypes.c_int] * 5 + [P] * 8 + [ctypes.c_int, P, ctypes.c_int,
                                                                             P, P, P, ctypes.c_double, P, P]
        lib.oracle_verify_sliding.restype = ctypes.c_int
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _pack(seqs, Q, Kb, Vb):
    """The flat arrays oracle_verify* take: per-sequence views concatenated."""
    Q = np.ascontiguousarray(Q, dtype=np.float64)
    Kb = np.ascontiguousarray(Kb, dtype=np.float64)
    Vb = np.ascontiguousarray(Vb, dtype=np.float64)
    nrows, H, d = Q.shape
    R = None
    deep_k, deep_v, win_k, win_v, deep_off, win_off = [], [], [], [], [], []
    dpos = wpos = 0
    for s in seqs:
        T, ws = int(s["T"]), int(s["ws"])
        lo = min(ws, T)
        kd = np.ascontiguousarray(s["Kd"], dtype=np.float64)
        assert kd.shape == (H, T, d), (kd.shape, (H, T, d))
        deep_k.append(kd.ravel()); deep_v.append(np.ascontiguousarray(s["Vd"], dtype=np.float64).ravel())
        deep_off.append(dpos); dpos += kd.size
        kw = s.get("Kw")
        if kw is not None and kw.size:
            kw = np.ascontiguousarray(kw, dtype=np.float64)
            assert kw.shape[0] == H and kw.shape[2] == T - lo and kw.shape[3] == d
            R = kw.shape[1] + 1 if R is None else R
            win_k.append(kw.ravel()); win_v.append(np.ascontiguousarray(s["Vw"], dtype=np.float64).ravel())
            win_off.append(wpos); wpos += kw.size
        else:
            win_off.append(wpos)
    R = int(seqs[0]["R"]) if R is None else R
    for s in seqs:
        assert int(s.get("R", R)) == R
    cat = lambda xs: np.concatenate(xs) if xs else np.zeros(1)
    return dict(Q=Q, Kb=Kb, Vb=Vb, H=H, d=d, R=R, nrows=nrows,
                Kd=cat(deep_k), Vd=cat(deep_v), Kw=cat(win_k), Vw=cat(win_v),
                T=np.array([int(s["T"]) for s in seqs], dtype=np.int64),
                ws=np.array([int(s["ws"]) for s in seqs], dtype=np.int64),
                do=np.array(deep_off, dtype=np.int64), wo=np.array(win_off, dtype=np.int64))


def verify_sliding(seqs: Sequence[Dict], branches: np.ndarray, Q: np.ndarray, Kb: np.ndarray,
                   Vb: np.ndarray, W: int, scale: float):
    """Verify-attention under the per-query sliding-window reading (the RIPE
    abstract's fifth sentence read per query): draft token j at position T + j sees
    positions T+j-W+1 .. T+j at its own depth r -- committed positions among them
    only if the store still holds their planes (p >= ws) -- and everything older at
    the deepest plane R; an older draft token's plane R is its depth-R row.
    ``branches`` must be the all-depths form (row0 = s*k*R + r - 1, row_stride R).
    Same inputs and outputs as ``verify`` otherwise; the definition is evaluated
    directly (all scores of a row, one softmax)."""
    lib = _load()
    a = _pack(seqs, Q, Kb, Vb)
    br = np.ascontiguousarray(branches, dtype=np.int32).reshape(-1, 5)
    O = np.zeros((a["nrows"], a["H"], a["d"]), dtype=np.float64)
    lse = np.zeros((a["nrows"], a["H"]), dtype=np.float64)
    rc = lib.oracle_verify_sliding(len(seqs), a["H"], a["d"], a["R"], int(W), _ptr(a["T"]), _ptr(a["ws"]),
                                   _ptr(a["do"]), _ptr(a["Kd"]), _ptr(a["Vd"]), _ptr(a["wo"]), _ptr(a["Kw"]),
                                   _ptr(a["Vw"]), br.shape[0], _ptr(br), a["nrows"], _ptr(a["Q"]), _ptr(a["Kb"]),
                                   _ptr(a["Vb"]), float(scale), _ptr(O), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_verify_sliding rejected its arguments (code %d)" % rc)
    return O, lse


def verify(seqs: Sequence[Dict], branches: np.ndarray, Q: np.ndarray, Kb: np.ndarray,
           Vb: np.ndarray, scale: float, mode: int = 1):
    """Verify-attention of every branch row over its sequence's RIPE store.

    ``seqs[b]`` holds ``T`` (committed length), ``ws`` (window start), ``Kd``/``Vd``
    (plane R, [H][T][d]) and ``Kw``/``Vw`` (planes 1..R-1 of positions
    min(ws,T)..T-1, [H][R-1][T-min(ws,T)][d]).  ``branches`` is an int array
    [nbranch][5] = (seq, depth 1..R, ntok, row0, row_stride).  Q, Kb, Vb are
    [nrows][H][d].  Returns (O [nrows][H][d], lse [nrows][H]) in fp64; rows not
    named by any branch are left at zero.

    mode 0 evaluates the definition directly (all scores of a row, one softmax);
    mode 1 evaluates it as deep-region, window-region and block partials merged
    by their maxima.
    """
    lib = _load()
    Q = np.ascontiguousarray(Q, dtype=np.float64)
    Kb = np.ascontiguousarray(Kb, dtype=np.float64)
    Vb = np.ascontiguousarray(Vb, dtype=np.float64)
    nrows, H, d = Q.shape
    R = None
    deep_k, deep_v, win_k, win_v, deep_off, win_off = [], [], [], [], [], []
    dpos = wpos = 0
    for s in seqs:
        T, ws = int(s["T"]), int(s["ws"])
        lo = min(ws, T)
        kd = np.ascontiguousarray(s["Kd"], dtype=np.float64)
        assert kd.shape == (H, T, d), (kd.shape, (H, T, d))
        deep_k.append(kd.ravel()); deep_v.append(np.ascontiguousarray(s["Vd"], dtype=np.float64).ravel())
        deep_off.append(dpos); dpos += kd.size
        kw = s.get("Kw")
        if kw is not None and kw.size:
            kw = np.ascontiguousarray(kw, dtype=np.float64)
            assert kw.shape[0] == H and kw.shape[2] == T - lo and kw.shape[3] == d
            R = kw.shape[1] + 1 if R is None else R
            win_k.append(kw.ravel()); win_v.append(np.ascontiguousarray(s["Vw"], dtype=np.float64).ravel())
            win_off.append(wpos); wpos += kw.size
        else:
            win_off.append(wpos)
    R = int(seqs[0]["R"]) if R is None else R
    for s in seqs:
        assert int(s.get("R", R)) == R
    cat = lambda xs: np.concatenate(xs) if xs else np.zeros(1)
    Kd, Vd, Kw, Vw = cat(deep_k), cat(deep_v), cat(win_k), cat(win_v)
    br = np.ascontiguousarray(branches, dtype=np.int32).reshape(-1, 5)
    T_arr = np.array([int(s["T"]) for s in seqs], dtype=np.int64)
    ws_arr = np.array([int(s["ws"]) for s in seqs], dtype=np.int64)
    do = np.array(deep_off, dtype=np.int64)
    wo = np.array(win_off, dtype=np.int64)
    O = np.zeros((nrows, H, d), dtype=np.float64)
    lse = np.zeros((nrows, H), dtype=np.float64)
    rc = lib.oracle_verify(len(seqs), H, d, R, _ptr(T_arr), _ptr(ws_arr), _ptr(do), _ptr(Kd),
                           _ptr(Vd), _ptr(wo), _ptr(Kw), _ptr(Vw), br.shape[0], _ptr(br), nrows,
                           _ptr(Q), _ptr(Kb), _ptr(Vb), float(scale), int(mode), _ptr(O), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_verify rejected its arguments (code %d)" % rc)
    return O, lse


# -----------------------------------------------------------------------------
# Memory model of the RIPE store (the RIPE abstract: 11.9 % of the full cache's
# memory for a 64-position window at a 1024-token context on Huginn).
# -----------------------------------------------------------------------------

def memory_fraction(T: int, W: int, R: int, n_recurrent: int, n_prelude: int = 0,
                    n_coda: int = 0) -> float:
    """KV planes kept by RIPE over the planes of the full cache.

    Non-recurrent (prelude and coda) layers hold one plane per position either
    way; each recurrent layer holds the deepest plane for the T - W' positions
    outside the window and all R planes for the W' = min(W, T) inside it, against
    R planes for all T positions in the full cache.
    """
    Wp = min(W, T)
    ripe = (n_prelude + n_coda) * T + n_recurrent * ((T - Wp) + Wp * R)
    full = (n_prelude + n_coda) * T + n_recurrent * R * T
    return ripe / full


# -----------------------------------------------------------------------------
# Store model: the documented GPU layout, written out with NumPy indexing.
# -----------------------------------------------------------------------------

class OracleStore:
    """Host model of the RIPE store, for byte-exact checks of append and evict.

    Layout (the RIPE abstract's store: deepest plane everywhere, all planes in a
    window kept as a ring buffer):
      kdeep/vdeep [L][Bmax][H][Tmax][d]         plane R of every appended position
      kwin/vwin   [L][Bmax][H][R-1][Wcap][d]    planes 1..R-1; position p in slot
                                                p mod Wcap, Wcap = W + kmax
      length[b], wstart[b]                      committed length T_b, window start
      rfloor[b]                                 ring floor (below)
    Positions ws_b <= p < T_b are live in the ring.

    append(seq b, n): positions T_b..T_b+n-1 get plane R in kdeep; of those, the
    last min(n, Wcap) get planes 1..R-1 in the ring; T_b += n; then ws_b rises to
    T_b - Wcap if more than Wcap positions would be live.  Sequences whose
    T_b + n exceeds Tmax, or with n outside [0, kmax_in], are skipped and flagged.
    evict(seq b): ws_b = max(ws_b, T_b - W): positions leaving the window keep only
    their deepest plane, which kdeep already holds.

    Ring floor rf_b: the lowest position whose ring slots still hold its own
    planes 1..R-1 (positions below it were overwritten by later positions, or
    never written by a long prefill).  append raises it to T_b - Wcap like ws_b,
    but evict leaves it alone, so rf_b <= ws_b always.

    truncate(seq b, T'): rollback to the confirmed prefix (LoopSpec article,
    section on the second branch: a rejected early draft discards the dependent
    work and decoding resumes from the confirmed prefix).  The target state is
    the one a store that only ever saw the confirmed tokens reaches after its
    evict at the confirmed length, as far as the ring still holds the planes:
      T_b  = min(T_b, T')
      rf_b = min(rf_b, T_b)
      ws_b = min(ws_b, max(T_b - W, rf_b))
    Positions that were evicted only because the rejected tokens pushed the
    window forward come back into the window; positions whose ring slots the
    rejected tokens overwrote cannot (with Wcap = W + kmax that happens only when
    more than kmax positions are rolled back).  A truncate to T' >= T_b changes
    nothing.  A fork cannot be truncated below its fork position (flagged,
    skipped): release it instead.

    Branch forks (LoopSpec article, section on deployment: a KV cache per branch,
    rejected continuations deleted).  fork(parent p -> child c) gives slot c the
    parent's state without copying its deep prefix: base[c] = p and fpos[c] =
    floor64(T_p) (a multiple of 64, the deep tile), so positions below fpos[c] are
    read from p's deep plane; the child gets its own copies of p's deep rows
    fpos..T_p-1 and of p's whole ring, and its own len/ws/rfloor.  Appends to c
    then write c's own rows.  While c lives, p must keep its deep rows below
    fpos[c] (no truncate below it).  Only a sequence that is not itself a fork can
    be forked (else flagged, skipped).  release(c) frees the slot: len = ws =
    rfloor = 0, base = itself, fpos = 0.
    """

    def __init__(self, L, R, H, d, W, Tmax, Bmax, kmax, np_dtype):
        self.L, self.R, self.H, self.d, self.W = L, R, H, d, W
        self.Tmax, self.Bmax, self.kmax = Tmax, Bmax, kmax
        self.Wcap = W + kmax
        self.kdeep = np.zeros((L, Bmax, H, Tmax, d), dtype=np_dtype)
        self.vdeep = np.zeros_like(self.kdeep)
        self.kwin = np.zeros((L, Bmax, H, max(R - 1, 0), self.Wcap, d), dtype=np_dtype)
        self.vwin = np.zeros_like(self.kwin)
        self.length = np.zeros(Bmax, dtype=np.int32)
        self.wstart = np.zeros(Bmax, dtype=np.int32)
        self.rfloor = np.zeros(Bmax, dtype=np.int32)
        self.base = np.arange(Bmax, dtype=np.int32)
        self.fpos = np.zeros(Bmax, dtype=np.int32)
        self.flagged = False

    def reset(self, seq_ids):
        """Empty the listed slots (a fork is released: it no longer reads its parent)."""
        for b in seq_ids:
            self.length[b] = 0
            self.wstart[b] = 0
            self.rfloor[b] = 0
            self.base[b] = b
            self.fpos[b] = 0

    def fork(self, parent_ids, child_ids):
        for p, c in zip(parent_ids, child_ids):
            p, c = int(p), int(c)
            if not (0 <= p < self.Bmax and 0 <= c < self.Bmax) or p == c or self.base[p] != p:
                self.flagged = True
                continue
            T = int(self.length[p])
            f = T // 64 * 64
            self.kdeep[:, c, :, f:T] = self.kdeep[:, p, :, f:T]
            self.vdeep[:, c, :, f:T] = self.vdeep[:, p, :, f:T]
            self.kwin[:, c] = self.kwin[:, p]
            self.vwin[:, c] = self.vwin[:, p]
            self.length[c] = T
            self.wstart[c] = self.wstart[p]
            self.rfloor[c] = self.rfloor[p]
            self.base[c] = p
            self.fpos[c] = f

    def append(self, seq_ids, n_acc, K, V):
        """K, V: [L][nseq][kmax_in][R][H][d]; plane index r-1 along axis 3."""
        kmax_in = K.shape[2]
        for i, b in enumerate(seq_ids):
            n = int(n_acc[i])
            T = int(self.length[b])
            if n < 0 or n > kmax_in or T + n > self.Tmax or b < 0 or b >= self.Bmax:
                self.flagged = True
                continue
            for t in range(n):
                p = T + t
                self.kdeep[:, b, :, p, :] = K[:, i, t, self.R - 1]
                self.vdeep[:, b, :, p, :] = V[:, i, t, self.R - 1]
                if t >= n - self.Wcap and self.R > 1:
                    slot = p % self.Wcap
                    # K[:, i, t, :R-1] is [L][R-1][H][d]; the ring is [L][H][R-1][d]
                    self.kwin[:, b, :, :, slot, :] = np.swapaxes(K[:, i, t, : self.R - 1], 1, 2)
                    self.vwin[:, b, :, :, slot, :] = np.swapaxes(V[:, i, t, : self.R - 1], 1, 2)
            self.length[b] = T + n
            self.wstart[b] = max(int(self.wstart[b]), T + n - self.Wcap)
            self.rfloor[b] = max(int(self.rfloor[b]), T + n - self.Wcap)

    def evict(self, seq_ids):
        for b in seq_ids:
            self.wstart[b] = max(int(self.wstart[b]), int(self.length[b]) - self.W)

    def truncate(self, seq_ids, new_len):
        for i, b in enumerate(seq_ids):
            if int(new_len[i]) < 0 or (self.base[b] != b and int(new_len[i]) < int(self.fpos[b])):
                self.flagged = True
                continue
            T = min(int(self.length[b]), int(new_len[i]))
            rf = min(int(self.rfloor[b]), T)
            self.length[b] = T
            self.rfloor[b] = rf
            self.wstart[b] = min(int(self.wstart[b]), max(T - self.W, rf))

    def plane_view(self, layer: int, b: int):
        """What a verify reads for sequence b: the oracle's logical input dict (a
        fork's deep positions below its fork position come from its parent)."""
        T, ws = int(self.length[b]), int(self.wstart[b])
        lo = min(ws, T)
        pos = np.arange(lo, T)
        slots = pos % self.Wcap
        f, base = min(int(self.fpos[b]), T), int(self.base[b])
        kd = np.concatenate([self.kdeep[layer, base, :, :f, :], self.kdeep[layer, b, :, f:T, :]], axis=1)
        vd = np.concatenate([self.vdeep[layer, base, :, :f, :], self.vdeep[layer, b, :, f:T, :]], axis=1)
        return {
            "T": T, "ws": ws, "R": self.R, "Kd": kd, "Vd": vd,
            "Kw": self.kwin[layer, b][:, :, slots, :], "Vw": self.vwin[layer, b][:, :, slots, :],
        }

    def live_planes(self, b: int) -> int:
        """Planes per recurrent layer and head that the store holds for sequence b."""
        T, ws = int(self.length[b]), int(self.wstart[b])
        return T + max(0, T - max(ws, 0)) * (self.R - 1)


# -----------------------------------------------------------------------------
# The block-independence claim of the RIPE abstract, under a per-query sliding
# window: a query at draft position j (position T+j) sees the W most recent
# positions T+j-W+1 .. T+j at its own depth, everything older at the deepest
# plane.  Returns, for each (j, j') with j' <= j, whether block token j' would be
# read at the deepest plane -- a plane the batched pass has not computed yet.
# -----------------------------------------------------------------------------

def sliding_block_reads_deepest(W: int, k: int) -> np.ndarray:
    out = np.zeros((k, k), dtype=bool)
    for j in range(k):
        for jj in range(j + 1):
            out[j, jj] = (jj < j + 1 - W)
    return out
