"""The C ABI library loads and exports every entry point include/ripe.h declares;
host-side size and argument logic (no GPU needed)."""
import ctypes
import os
import re

import pytest

from oracle import oracle as OR

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ripe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ripe_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_entry_point():
    from depth_planed_kv_b200 import build as B
    B.build()
    from depth_planed_kv_b200 import ripe
    names = declared_functions()
    assert len(names) >= 17
    lib = ctypes.CDLL(ripe.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) <= set(ripe.EXPORTED)


def test_error_strings_and_codes():
    from depth_planed_kv_b200 import ripe
    for code in range(9):
        assert ripe._lib.ripe_error_string(code)
    assert ripe._lib.ripe_error_string(0) == b"ok"


def test_cache_bytes_matches_layout_and_memory_model():
    from depth_planed_kv_b200 import ripe
    import torch
    L, R, H, d, W, T, B, k = 4, 32, 55, 96, 64, 1024, 1, 4
    n = ripe.ripe_cache_bytes(L, R, H, d, W, T, B, k, torch.bfloat16)
    r256 = lambda x: (x + 255) // 256 * 256
    deep = r256(L * B * H * T * d * 2)
    ring = r256(L * B * H * (R - 1) * (W + k) * d * 2)
    assert n == 2 * deep + 2 * ring + 5 * r256(4 * B) + 256   # len, ws, rfloor, fbase, fpos, error word
    # stored planes per (layer, head): T + (W+kmax)(R-1); the live part is T + W(R-1)
    live = T + W * (R - 1)
    assert live / (R * T) == pytest.approx(OR.memory_fraction(T, W, R, 1))


@pytest.mark.parametrize("args,code", [
    ((0, 4, 2, 16, 8, 64, 1, 4), 1),     # layers
    ((1, 0, 2, 16, 8, 64, 1, 4), 1),     # R
    ((1, 65, 2, 16, 8, 64, 1, 4), 1),
    ((1, 4, 2, 12, 8, 64, 1, 4), 3),     # d*2 not a multiple of 16 (bf16)
    ((1, 4, 2, 256, 8, 64, 1, 4), 7),    # d above the library's kernels
    ((1, 4, 2, 16, -1, 64, 1, 4), 1),    # W
    ((1, 4, 2, 16, 8, 64, 0, 4), 1),     # max_seqs
    ((1, 4, 2, 16, 8, 64, 1, 0), 1),     # kmax
])
def test_invalid_sizes_rejected_on_host(args, code):
    from depth_planed_kv_b200 import ripe
    out = ctypes.c_size_t()
    rc = ripe._lib.ripe_cache_bytes(*args, ripe.RIPE_BF16, ctypes.byref(out))
    assert rc == code
    assert ripe._lib.ripe_last_error()


def test_null_cache_rejected():
    from depth_planed_kv_b200 import ripe
    assert ripe._lib.ripe_evict(None, None, 0, None) == ripe.RIPE_ERR_INVALID_ARG
    assert ripe._lib.ripe_verify_attn(None, 0, None, 0, 0, None, None, None, None, 0.0, None, None,
                                      None) == ripe.RIPE_ERR_INVALID_ARG
