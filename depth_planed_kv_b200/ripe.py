"""ctypes binding of libripe (include/ripe.h).

Argument marshalling only: every step of the verify path runs in libripe's CUDA
kernels.  Importing this module loads ``libripe.so`` from this directory and
raises ``ImportError`` if it has not been built (``python -m
depth_planed_kv_b200.build``); there is no fallback implementation.

Function names follow the C ABI.  Tensors are torch CUDA tensors; their data
pointers and the current torch stream are passed through unchanged.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libripe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libripe.so is not built at %s; run `python -m depth_planed_kv_b200.build`" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

RIPE_OK = 0
RIPE_ERR_INVALID_ARG = 1
RIPE_ERR_CAPACITY = 2
RIPE_ERR_UNALIGNED = 3
RIPE_ERR_OOM = 4
RIPE_ERR_CUDA = 5
RIPE_ERR_DEVICE = 6
RIPE_ERR_UNSUPPORTED = 7
RIPE_ERR_CAPTURING = 8
RIPE_BF16 = 0
RIPE_F32 = 1
DEVERR_NAMES = {0: "none", 1: "seq_range", 2: "capacity", 3: "count", 4: "ctx", 5: "branch", 6: "timeout",
                7: "fork"}

_P = ctypes.c_void_p
_I = ctypes.c_int


class ripe_branch_t(ctypes.Structure):
    _fields_ = [("seq", ctypes.c_int32), ("depth", ctypes.c_int32), ("ntok", ctypes.c_int32),
                ("row0", ctypes.c_int32), ("row_stride", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 3)]


def _sig(name, args, res=ctypes.c_int):
    f = getattr(_lib, name)
    f.argtypes = args
    f.restype = res
    return f


_sig("ripe_cache_bytes", [_I] * 9 + [ctypes.POINTER(ctypes.c_size_t)])
_sig("ripe_cache_create", [_I] * 9 + [_P, ctypes.POINTER(_P)])
_sig("ripe_cache_destroy", [_P])
_sig("ripe_cache_reset", [_P, _P, _I, _P])
_sig("ripe_append", [_P, _P, _P, _I, _P, _P, _I, _P])
_sig("ripe_evict", [_P, _P, _I, _P])
_sig("ripe_truncate", [_P, _P, _P, _I, _P])
_sig("ripe_fork", [_P, _P, _P, _I, _P])
_sig("ripe_read_forks", [_P, _P, _P, _P])
_sig("ripe_verify_attn", [_P, _I, _P, _I, _I, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P])
_sig("ripe_verify_attn_all_depths", [_P, _I, _P, _I, _I, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P])
_sig("ripe_verify_attn_all_depths_sliding", [_P, _I, _P, _I, _I, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P])
_sig("ripe_verify_attn_noalloc", [_P, _I, _P, _I, _I, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P,
                                  ctypes.POINTER(ctypes.c_size_t)])
_sig("ripe_reserve_workspace", [_P, _I])
_sig("ripe_synth_fill", [_P, _P, _P, _I, ctypes.c_uint64, _P, _P])
_sig("ripe_cache_verify_path", [_P, ctypes.POINTER(_I)])
_sig("ripe_cache_set_all_depths_kernel", [_P, _I])
_sig("ripe_debug_stall_next_verify", [_P, ctypes.c_longlong])
_sig("ripe_accept", [_I, _I, _I, _P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P, _P])
_sig("ripe_cache_buffers", [_P] + [ctypes.POINTER(_P)] * 7)
_sig("ripe_read_meta", [_P, _P, _P, _P, _P])
_sig("ripe_get_device_error", [_P, _P, _P])
_sig("ripe_launch_count", [], ctypes.c_uint64)
_sig("ripe_error_string", [_I], ctypes.c_char_p)
_sig("ripe_last_error", [], ctypes.c_char_p)

EXPORTED = ["ripe_cache_bytes", "ripe_cache_create", "ripe_cache_destroy", "ripe_cache_reset",
            "ripe_append", "ripe_evict", "ripe_truncate", "ripe_fork", "ripe_read_forks", "ripe_verify_attn",
            "ripe_verify_attn_all_depths", "ripe_verify_attn_all_depths_sliding", "ripe_verify_attn_noalloc", "ripe_reserve_workspace",
            "ripe_synth_fill", "ripe_cache_verify_path", "ripe_cache_set_all_depths_kernel",
            "ripe_debug_stall_next_verify", "ripe_accept",
            "ripe_cache_buffers", "ripe_read_meta", "ripe_get_device_error", "ripe_launch_count",
            "ripe_error_string", "ripe_last_error"]


class RipeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.ripe_error_string(status).decode()
        detail = (_lib.ripe_last_error() or b"").decode()
        super().__init__("%s: %s (%d)%s" % (where, msg, status, (": " + detail) if detail else ""))


def _check(status: int, where: str):
    if status != RIPE_OK:
        raise RipeError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return RIPE_BF16
    if dtype == torch.float32:
        return RIPE_F32
    raise ValueError("unsupported dtype %s" % dtype)


def launch_count() -> int:
    return int(_lib.ripe_launch_count())


def ripe_accept(zp: torch.Tensor, zq: torch.Tensor, zf: Optional[torch.Tensor], x1: torch.Tensor,
                x2: Optional[torch.Tensor], u: torch.Tensor, temperature: float, stream=None):
    """LoopSpec acceptance of [nseq][k] draft positions.  zp, zq, zf: float32
    [nseq][k][V] logits (zf None: no fallback); x1, x2: int32 [nseq][k]; u: float32
    [nseq][k][3].  Returns (n_accepted, token, path) as int32 [nseq] tensors."""
    nseq, k, V = zp.shape
    for t in (zp, zq) + ((zf,) if zf is not None else ()):
        assert t.dtype == torch.float32 and t.is_contiguous() and t.shape == zp.shape
    assert x1.dtype == torch.int32 and u.dtype == torch.float32 and u.shape == (nseq, k, 3)
    out = [torch.empty(nseq, dtype=torch.int32, device=zp.device) for _ in range(3)]
    _check(_lib.ripe_accept(nseq, k, V, _ptr(zp), _ptr(zq), _ptr(zf), _ptr(x1), _ptr(x2), _ptr(u),
                            ctypes.c_float(temperature), _ptr(out[0]), _ptr(out[1]), _ptr(out[2]),
                            _stream(stream)), "ripe_accept")
    return tuple(out)


def ripe_cache_bytes(layers, R, H, d, W, Tmax, max_seqs, kmax, dtype=torch.bfloat16) -> int:
    out = ctypes.c_size_t()
    _check(_lib.ripe_cache_bytes(layers, R, H, d, W, Tmax, max_seqs, kmax, _dtype_code(dtype),
                                 ctypes.byref(out)), "ripe_cache_bytes")
    return out.value


class RipeCache:
    """Owner of one ripe_cache_t; methods mirror the C entry points."""

    def __init__(self, layers, R, H, d, W, Tmax, max_seqs, kmax, dtype=torch.bfloat16,
                 dev_mem: Optional[torch.Tensor] = None):
        self.layers, self.R, self.H, self.d, self.W = layers, R, H, d, W
        self.Tmax, self.max_seqs, self.kmax, self.dtype = Tmax, max_seqs, kmax, dtype
        self.Wcap = W + kmax
        self._mem = dev_mem  # keep a caller-provided buffer alive
        h = ctypes.c_void_p()
        _check(_lib.ripe_cache_create(layers, R, H, d, W, Tmax, max_seqs, kmax, _dtype_code(dtype),
                                      _ptr(dev_mem), ctypes.byref(h)), "ripe_cache_create")
        self.handle = h

    def close(self):
        if self.handle:
            _check(_lib.ripe_cache_destroy(self.handle), "ripe_cache_destroy")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # --- store -----------------------------------------------------------------
    def ripe_cache_reset(self, seq_ids: torch.Tensor, stream=None):
        _check(_lib.ripe_cache_reset(self.handle, _ptr(seq_ids), seq_ids.numel(), _stream(stream)),
               "ripe_cache_reset")

    def ripe_append(self, seq_ids: torch.Tensor, n_acc: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                    stream=None):
        """K, V: [layers][nseq][kmax_in][R][H][d] in the cache dtype."""
        assert K.is_contiguous() and V.is_contiguous() and K.dtype == self.dtype and V.dtype == self.dtype
        assert K.shape == V.shape and K.dim() == 6 and K.shape[0] == self.layers and K.shape[3] == self.R
        assert K.shape[4] == self.H and K.shape[5] == self.d and K.shape[1] == seq_ids.numel()
        assert seq_ids.dtype == torch.int32 and n_acc.dtype == torch.int32
        _check(_lib.ripe_append(self.handle, _ptr(seq_ids), _ptr(n_acc), seq_ids.numel(), _ptr(K), _ptr(V),
                                K.shape[2], _stream(stream)), "ripe_append")

    def ripe_evict(self, seq_ids: torch.Tensor, stream=None):
        _check(_lib.ripe_evict(self.handle, _ptr(seq_ids), seq_ids.numel(), _stream(stream)), "ripe_evict")

    def ripe_truncate(self, seq_ids: torch.Tensor, new_len: torch.Tensor, stream=None):
        _check(_lib.ripe_truncate(self.handle, _ptr(seq_ids), _ptr(new_len), seq_ids.numel(),
                                  _stream(stream)), "ripe_truncate")

    def ripe_fork(self, parent_ids: torch.Tensor, child_ids: torch.Tensor, stream=None):
        """Each child becomes a fork of its parent (device int32 ids)."""
        _check(_lib.ripe_fork(self.handle, _ptr(parent_ids), _ptr(child_ids), parent_ids.numel(),
                              _stream(stream)), "ripe_fork")

    def ripe_read_forks(self, stream=None):
        """(fbase, fpos) of every sequence, as host int32 arrays."""
        import numpy as np
        fb = np.zeros(self.max_seqs, np.int32)
        fp = np.zeros(self.max_seqs, np.int32)
        _check(_lib.ripe_read_forks(self.handle, fb.ctypes.data_as(_P), fp.ctypes.data_as(_P), _stream(stream)),
               "ripe_read_forks")
        return fb, fp

    def ripe_synth_fill(self, seq_ids, T, seed: int, coef, stream=None):
        """Host lists/arrays: seq_ids, T (per sequence); coef: float[R]."""
        n = len(seq_ids)
        ids = (ctypes.c_int32 * n)(*[int(x) for x in seq_ids])
        ts = (ctypes.c_int32 * n)(*[int(x) for x in T])
        cf = (ctypes.c_float * self.R)(*[float(x) for x in coef])
        _check(_lib.ripe_synth_fill(self.handle, ids, ts, n, ctypes.c_uint64(seed), cf, _stream(stream)),
               "ripe_synth_fill")

    def ripe_reserve_workspace(self, max_rows: int):
        _check(_lib.ripe_reserve_workspace(self.handle, max_rows), "ripe_reserve_workspace")

    # --- verify ----------------------------------------------------------------
    def ripe_verify_attn(self, layer: int, branches: torch.Tensor, nbranch: int, Q: torch.Tensor,
                         Kblk: torch.Tensor, Vblk: torch.Tensor, O: torch.Tensor,
                         lse: Optional[torch.Tensor] = None, ctx_len: Optional[torch.Tensor] = None,
                         scale: float = 0.0, stream=None):
        """branches: device int32 tensor [nbranch][8] (ripe_branch_t rows)."""
        nrows = Q.shape[0]
        _check(_lib.ripe_verify_attn(self.handle, layer, _ptr(branches), nbranch, nrows, _ptr(Q),
                                     _ptr(Kblk), _ptr(Vblk), _ptr(ctx_len), ctypes.c_float(scale),
                                     _ptr(O), _ptr(lse), _stream(stream)), "ripe_verify_attn")

    def ripe_verify_attn_noalloc(self, layer: int, branches: torch.Tensor, nbranch: int, Q: torch.Tensor,
                                 Kblk: torch.Tensor, Vblk: torch.Tensor, O: torch.Tensor,
                                 lse: Optional[torch.Tensor] = None, ctx_len: Optional[torch.Tensor] = None,
                                 scale: float = 0.0, stream=None, check: bool = True):
        """Same as ripe_verify_attn, with the library's fixed scratch instead of an
        allocation.  Returns (status, scratch bytes used or needed)."""
        need = ctypes.c_size_t()
        rc = _lib.ripe_verify_attn_noalloc(self.handle, layer, _ptr(branches), nbranch, Q.shape[0], _ptr(Q),
                                           _ptr(Kblk), _ptr(Vblk), _ptr(ctx_len), ctypes.c_float(scale),
                                           _ptr(O), _ptr(lse), _stream(stream), ctypes.byref(need))
        if check:
            _check(rc, "ripe_verify_attn_noalloc")
        return rc, need.value

    def ripe_verify_attn_all_depths(self, layer: int, seq_ids: torch.Tensor, k: int, Q: torch.Tensor,
                                    Kblk: torch.Tensor, Vblk: torch.Tensor, O: torch.Tensor,
                                    lse: Optional[torch.Tensor] = None,
                                    ctx_len: Optional[torch.Tensor] = None, scale: float = 0.0,
                                    stream=None):
        """Q, Kblk, Vblk, O: [nseq][k][R][H][d]; lse: [nseq][k][R][H]."""
        _check(_lib.ripe_verify_attn_all_depths(self.handle, layer, _ptr(seq_ids), seq_ids.numel(), k,
                                                _ptr(Q), _ptr(Kblk), _ptr(Vblk), _ptr(ctx_len),
                                                ctypes.c_float(scale), _ptr(O), _ptr(lse),
                                                _stream(stream)), "ripe_verify_attn_all_depths")

    def ripe_verify_attn_all_depths_sliding(self, layer: int, seq_ids: torch.Tensor, k: int, Q: torch.Tensor,
                                            Kblk: torch.Tensor, Vblk: torch.Tensor, O: torch.Tensor,
                                            lse: Optional[torch.Tensor] = None,
                                            ctx_len: Optional[torch.Tensor] = None, scale: float = 0.0,
                                            stream=None):
        """The all-depths call under the per-query sliding window (same layouts)."""
        _check(_lib.ripe_verify_attn_all_depths_sliding(self.handle, layer, _ptr(seq_ids), seq_ids.numel(), k,
                                                        _ptr(Q), _ptr(Kblk), _ptr(Vblk), _ptr(ctx_len),
                                                        ctypes.c_float(scale), _ptr(O), _ptr(lse),
                                                        _stream(stream)), "ripe_verify_attn_all_depths_sliding")

    # --- inspection ------------------------------------------------------------
    def ripe_debug_stall_next_verify(self, cycles: int):
        """Test hook: the next persistent-kernel verify waits `cycles` on a barrier
        nothing signals, so its bounded wait runs out (RIPE_DEVERR_TIMEOUT)."""
        _check(_lib.ripe_debug_stall_next_verify(self.handle, int(cycles)), "ripe_debug_stall_next_verify")

    ALL_DEPTHS_AUTO, ALL_DEPTHS_PERSISTENT, ALL_DEPTHS_CLUSTER = 0, 1, 2

    def ripe_cache_set_all_depths_kernel(self, kernel: int):
        """Which sm_100a kernel serves the all-depths verify (0 auto, 1 persistent,
        2 cluster); the sliding form always runs in the persistent kernel."""
        _check(_lib.ripe_cache_set_all_depths_kernel(self.handle, int(kernel)), "ripe_cache_set_all_depths_kernel")

    def ripe_cache_verify_path(self) -> int:
        """1: the fused sm_100a kernel serves verify; 0: the CUDA-core kernels."""
        out = ctypes.c_int()
        _check(_lib.ripe_cache_verify_path(self.handle, ctypes.byref(out)), "ripe_cache_verify_path")
        return out.value

    def buffers(self):
        """Torch views of the store parts (device memory owned by the cache)."""
        ptrs = [ctypes.c_void_p() for _ in range(7)]
        _check(_lib.ripe_cache_buffers(self.handle, *[ctypes.byref(p) for p in ptrs]), "ripe_cache_buffers")
        es = 2 if self.dtype == torch.bfloat16 else 4
        deep_shape = (self.layers, self.max_seqs, self.H, self.Tmax, self.d)
        ring_shape = (self.layers, self.max_seqs, self.H, max(self.R - 1, 0), self.Wcap, self.d)
        mk = lambda p, shape, dt: _from_ptr(p.value, shape, dt)
        return {"kdeep": mk(ptrs[0], deep_shape, self.dtype), "vdeep": mk(ptrs[1], deep_shape, self.dtype),
                "kwin": mk(ptrs[2], ring_shape, self.dtype), "vwin": mk(ptrs[3], ring_shape, self.dtype),
                "len": mk(ptrs[4], (self.max_seqs,), torch.int32),
                "ws": mk(ptrs[5], (self.max_seqs,), torch.int32),
                "rfloor": mk(ptrs[6], (self.max_seqs,), torch.int32)}

    def ripe_read_meta(self, stream=None, with_rfloor=False):
        """(len, ws) -- or (len, ws, rfloor) -- of every sequence, as host int32 arrays."""
        import numpy as np
        ln = np.zeros(self.max_seqs, np.int32)
        ws = np.zeros(self.max_seqs, np.int32)
        rf = np.zeros(self.max_seqs, np.int32)
        _check(_lib.ripe_read_meta(self.handle, ln.ctypes.data_as(_P), ws.ctypes.data_as(_P),
                                   rf.ctypes.data_as(_P), _stream(stream)), "ripe_read_meta")
        return (ln, ws, rf) if with_rfloor else (ln, ws)

    def ripe_get_device_error(self, stream=None) -> int:
        code = ctypes.c_int32()
        _check(_lib.ripe_get_device_error(self.handle, ctypes.byref(code), _stream(stream)),
               "ripe_get_device_error")
        return code.value


def _from_ptr(ptr: int, shape, dtype):
    """A torch tensor aliasing device memory the library owns (no copy)."""
    n = 1
    for s in shape:
        n *= s
    if n == 0:
        return torch.empty(shape, dtype=dtype, device="cuda")
    es = torch.tensor([], dtype=dtype).element_size()
    arr = _CudaArray(ptr, n * es)
    t = torch.as_tensor(arr, device="cuda").view(dtype)
    return t[: n].view(shape)


class _CudaArray:
    """Minimal __cuda_array_interface__ wrapper so torch can alias a device pointer."""

    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (ptr, False),
                                         "version": 3, "strides": None}


def branch_table(rows, device="cuda") -> torch.Tensor:
    """int32 [n][8] device tensor of ripe_branch_t from (seq, depth, ntok, row0, row_stride) tuples."""
    import numpy as np
    arr = np.zeros((len(rows), 8), np.int32)
    for i, r in enumerate(rows):
        arr[i, :5] = r[:5]
    return torch.from_numpy(arr).to(device)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
