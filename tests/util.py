"""Shared test helpers.

The input-arranging helpers live in the package (``depth_planed_kv_b200.synth_rows``)
so that the benchmark does not depend on the test tree; they are re-exported here.
"""
from __future__ import annotations

import numpy as np

from depth_planed_kv_b200.synth_rows import all_depth_rows, branch_rows, seq_planes  # noqa: F401


def errors(got: np.ndarray, ref: np.ndarray):
    """(max abs error, max row-normwise relative error) over [..., d] outputs."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = np.abs(got - ref)
    abs_err = float(diff.max()) if diff.size else 0.0
    denom = np.maximum(np.abs(ref).max(axis=-1), 1e-6)
    rel = float((diff.max(axis=-1) / denom).max()) if diff.size else 0.0
    return abs_err, rel
