"""The multi-rank path of bench.py on CPU: two gloo ranks, world size 2.

Ranks verify disjoint sequences (their own synthetic stores, seeded per rank) with
no data-path exchange; the only collectives are the barrier and the max over ranks
of the step time, taken by every rank in the same order.  The sequences a rank
verifies give the same result as verifying them alone (checked with the fp64
oracle on a tiny workload), and the whole-job rate uses the slowest rank's time.
"""
import contextlib
import importlib.util
import io
import json
import os
import socket
import sys
import types

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _tiny_shard_output(seed):
    """fp64 oracle output of the tiny all-depths workload on the store seeded `seed`."""
    import dataclasses
    import math
    sys.path.insert(0, ROOT)
    from depth_planed_kv_b200 import synth as S
    from oracle import oracle as OR
    from tests.util import all_depth_rows, seq_planes
    wl = dataclasses.replace(S.tiny(), seed=seed)
    views = [seq_planes(wl, 0, 0, wl.ctx, wl.ctx - wl.W)]
    table, Q, Kb, Vb = all_depth_rows(wl, 0, 1, [0], wl.k)
    out, _ = OR.verify(views, table, Q, Kb, Vb, 1 / math.sqrt(wl.d))
    return out


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench = _bench()
        local_ms = 10.0 + 5.0 * rank  # the ranks' own step times
        ms_max = bench.max_over_ranks(local_ms, world, "cpu")
        dist.barrier()
        seed = bench.shard_seed(1000, rank)
        out = _tiny_shard_output(seed)
        # The reference arm: only rank 0 runs and prints; the others return at once.
        printed = io.StringIO()
        if rank != 0:
            args = types.SimpleNamespace(gpus=world, steps=1, warmup=0)
            with contextlib.redirect_stdout(printed):
                bench.run_reference(args)
        dist.barrier()
        np.save(os.path.join(out_dir, "out%d.npy" % rank), out)
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump({"ms_max": ms_max, "seed": seed, "printed": printed.getvalue(),
                       "rate": bench.whole_job_rate(1e9, world, 10, ms_max)}, f)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    info = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    # Every rank sees the slowest rank's time.
    assert [i["ms_max"] for i in info] == [15.0, 15.0]
    # Whole-job rate: all ranks' bytes over the slowest time.
    assert info[0]["rate"] == pytest.approx(1e9 * 2 * 10 / 0.015 / 1e9)
    # Disjoint shards: different stores, and each rank's result is the result of
    # verifying its sequences alone (no exchange between ranks).
    assert info[0]["seed"] != info[1]["seed"]
    outs = [np.load(tmp_path / ("out%d.npy" % r)) for r in range(world)]
    for r in range(world):
        np.testing.assert_array_equal(outs[r], _tiny_shard_output(info[r]["seed"]))
    assert not np.array_equal(outs[0], outs[1])
    # Reference arm on rank 1: no output.
    assert info[1]["printed"] == ""
