"""Seeded synthetic inputs for RIPE verify-attention.

This module holds the workload shapes and the input generator, and nothing of
the method itself: no attention, no store layout, no window rule.  Both sides of
every parity check draw their inputs here (the fp64 oracle through NumPy, the
GPU store through the library's fill kernel, which restates the same generator).

Generator (counter-based, so any element can be produced on its own):

* ``mix64`` is the SplitMix64 output function (Steele, Lea and Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014): add the golden-ratio
  increment, then two xor-shift-multiply rounds and a final xor-shift.
* A stream key is ``mix64(seed * 2**16 + tag)``; element ``idx`` of the stream
  is ``mix64(key + idx)`` (64-bit wrap-around).
* A 64-bit word becomes one approximately standard-normal value by summing its
  four 16-bit fields (Irwin-Hall, n=4: mean 131070, variance (2**32-1)/3),
  centring in integers, converting to fp32 (exact) and multiplying once by the
  fp32 constant ``INV_SD`` = fl32(1/sqrt((2**32-1)/3)).  The support is bounded
  at +-3.46 sigma, which is immaterial for attention inputs.
* ``idx`` packs logical coordinates into fixed bit fields, independent of any
  tensor shape: layer (6 bits) | plane (6) | sequence (10) | head (8) |
  position (20) | channel (10).

Synthetic planes (the RIPE abstract, sentence on geometric approach): the
deepest plane R is ~N(0,1); plane r < R adds independent noise scaled by
decay**(R-r) (0.88 per loop for Huginn, 0.81 for Raven).  Arithmetic: the
coefficient table is fl32(decay**(R-r)) computed on the host in fp64, the value
is fl32(fl32(c*e) + z) with no fused multiply-add, then rounded to bf16
(round-to-nearest-even) for bf16 workloads.

Draft-block tokens are fresh positions: token j of query slot s lives at the
virtual position ``BLOCK_POS0 + 1024*s + j`` of its sequence (beyond any real
context), and its plane r follows the same rule as a stored position.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
MUL1 = np.uint64(0xBF58476D1CE4E5B9)
MUL2 = np.uint64(0x94D049BB133111EB)
INV_SD = np.uint32(0x37DDB3D7).view(np.float32)  # fl32(1/sqrt((2**32-1)/3))

TAG_DEEP_K, TAG_DEEP_V, TAG_NOISE_K, TAG_NOISE_V, TAG_Q = 1, 2, 3, 4, 5
BLOCK_POS0 = 1 << 19

_SH_C, _SH_P, _SH_H, _SH_S, _SH_R, _SH_L = 0, 10, 30, 38, 48, 54


def mix64(x: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on uint64 arrays (wrap-around arithmetic)."""
    with np.errstate(over="ignore"):
        z = (x + GOLDEN).astype(np.uint64)
        z = (z ^ (z >> np.uint64(30))) * MUL1
        z = (z ^ (z >> np.uint64(27))) * MUL2
        return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tag: int) -> np.uint64:
    return mix64(np.array([(seed << 16) + tag], dtype=np.uint64))[0]


def pack_index(layer, plane, seq, head, pos, chan) -> np.ndarray:
    """Broadcast the logical coordinates into the fixed 60-bit counter."""
    u = lambda a: np.asarray(a, dtype=np.uint64)
    return ((u(layer) << np.uint64(_SH_L)) | (u(plane) << np.uint64(_SH_R))
            | (u(seq) << np.uint64(_SH_S)) | (u(head) << np.uint64(_SH_H))
            | (u(pos) << np.uint64(_SH_P)) | (u(chan) << np.uint64(_SH_C)))


def normal_from_bits(bits: np.ndarray) -> np.ndarray:
    """Irwin-Hall (n=4) approximately standard-normal fp32 values."""
    m = np.uint64(0xFFFF)
    s = ((bits & m) + ((bits >> np.uint64(16)) & m) + ((bits >> np.uint64(32)) & m)
         + (bits >> np.uint64(48))).astype(np.int64) - 131070
    return s.astype(np.float32) * INV_SD


def normals(seed: int, tag: int, idx: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return normal_from_bits(mix64(stream_key(seed, tag) + idx.astype(np.uint64)))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 (ties to even), returned as fp32 holding the bf16 value."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def coef_table(decay: float, R: int) -> np.ndarray:
    """c[r-1] = fl32(decay**(R-r)) for r = 1..R (c[R-1] = 1, never used for noise)."""
    return np.array([decay ** (R - r) for r in range(1, R + 1)], dtype=np.float64).astype(np.float32)


def planes(seed: int, kv: int, layer: int, seq: int, heads, plane_ids, positions, d: int,
           R: int, coef: np.ndarray, bf16: bool) -> np.ndarray:
    """Values of K (kv=0) or V (kv=1) planes -> fp32 array [heads][planes][positions][d].

    ``plane_ids`` are depths r in 1..R; r == R gives the deepest plane itself.
    """
    heads = np.asarray(heads, dtype=np.int64)
    plane_ids = np.asarray(plane_ids, dtype=np.int64)
    positions = np.asarray(positions, dtype=np.int64)
    h = heads[:, None, None, None]
    r = plane_ids[None, :, None, None]
    p = positions[None, None, :, None]
    c = np.arange(d, dtype=np.int64)[None, None, None, :]
    z = normals(seed, TAG_DEEP_K + kv, pack_index(layer, 0, seq, h, p, c))
    z = np.broadcast_to(z, (len(heads), len(plane_ids), len(positions), d))
    e = normals(seed, TAG_NOISE_K + kv, pack_index(layer, r, seq, h, p, c))
    cf = coef[plane_ids - 1].astype(np.float32)[None, :, None, None]
    noisy = (cf * e).astype(np.float32) + z  # two fp32 roundings, no fma
    out = np.where(r == R, z, noisy).astype(np.float32)
    return round_bf16(out) if bf16 else out


def queries(seed: int, layer: int, slot: int, seq: int, heads, tokens, d: int, bf16: bool) -> np.ndarray:
    """Q rows -> fp32 array [tokens][heads][d]."""
    heads = np.asarray(heads, dtype=np.int64)
    tokens = np.asarray(tokens, dtype=np.int64)
    idx = pack_index(layer, slot, seq, heads[None, :, None], tokens[:, None, None],
                     np.arange(d, dtype=np.int64)[None, None, :])
    q = normals(seed, TAG_Q, idx)
    return round_bf16(q) if bf16 else q


def block_positions(slot: int, ntok: int) -> np.ndarray:
    return BLOCK_POS0 + 1024 * slot + np.arange(ntok, dtype=np.int64)


# ----------------------------------------------------------------------------
# Workload shapes (the five configurations the pages' workloads are quoted on)
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    layers: int
    R: int
    H: int
    d: int
    W: int
    k: int
    nseq: int
    ctx: Optional[int]          # fixed context length (None: drawn per sequence)
    decay: float
    seed: int
    dtype: str                  # "bf16" | "f32"
    Tmax: int
    kmax: int
    mixed: bool = False         # LoopSpec-style branch list instead of all depths
    ctx_range: Optional[tuple] = None

    @property
    def bf16(self) -> bool:
        return self.dtype == "bf16"


def tiny() -> Workload:
    return Workload("tiny_f32", 1, 4, 2, 16, 8, 4, 1, 48, 0.88, 1000, "f32", 48 + 16, 4)


def huginn(W: int = 64, seed: int = 1001, layers: int = 4) -> Workload:
    return Workload("huginn_T1024_W%d_k4" % W, layers, 32, 55, 96, W, 4, 1, 1024, 0.88, seed,
                    "bf16", 1024 + 64, 4)


def sweep(W: int) -> Workload:
    return huginn(W=W, seed=1002)


SWEEP_W = (0, 4, 64, 256, 1024)


def mixed() -> Workload:
    return Workload("loopspec_mixed_64seq", 1, 32, 32, 128, 64, 8, 64, None, 0.81, 1003, "bf16",
                    4096 + 64, 8, mixed=True, ctx_range=(512, 4096))


def long_context() -> Workload:
    return Workload("long_ctx_B16_T32768", 1, 32, 32, 128, 128, 8, 16, 32768, 0.88, 1004, "bf16",
                    32768 + 512, 8)


def long_context_small() -> Workload:
    """The long-context step at 6 sequences x 8192 (about 2.2 GB of store): a
    case small enough for a full profiler capture of the same kernels."""
    return Workload("long_ctx_B6_T8192", 1, 32, 32, 128, 128, 8, 6, 8192, 0.88, 1005, "bf16",
                    8192 + 512, 8)


@dataclasses.dataclass
class BranchSpec:
    seq: int
    depth: int
    ntok: int
    qslot: int     # query slot of the generator
    bslot: int     # draft-block slot of the generator (0 main, 1 draft, 2 fallback)


def mixed_structure(wl: Workload):
    """Per-sequence contexts and the LoopSpec branch list (host-side draws, PCG64).

    Integer uniforms are inclusive: ctx in [512, 4096], draft depth in [4, 16],
    fallback (probability 0.3) depth in [16, 28]; the main branch is at depth R.
    """
    rng = np.random.default_rng(wl.seed)
    lo, hi = wl.ctx_range
    ctx = rng.integers(lo, hi + 1, size=wl.nseq)
    branches: List[BranchSpec] = []
    for s in range(wl.nseq):
        branches.append(BranchSpec(s, wl.R, wl.k, 0, 0))
        branches.append(BranchSpec(s, int(rng.integers(4, 17)), wl.k, 1, 1))
        if rng.random() < 0.3:
            branches.append(BranchSpec(s, int(rng.integers(16, 29)), wl.k, 2, 2))
    return ctx.astype(np.int64), branches


def all_depth_branches(nseq: int, R: int, k: int) -> List[BranchSpec]:
    """All k draft tokens at every depth.

    Branch (s, r) uses query slot r-1 (the query differs per depth) and block
    slot 0: the same k draft tokens, seen at their plane r.
    """
    return [BranchSpec(s, r, k, r - 1, 0) for s in range(nseq) for r in range(1, R + 1)]


def context_lengths(wl: Workload) -> np.ndarray:
    if wl.mixed:
        return mixed_structure(wl)[0]
    return np.full(wl.nseq, wl.ctx, dtype=np.int64)
