"""The bounded-wait error path, run without any fault: a test hook makes the
softmax warps of the persistent kernel wait on a barrier that nothing signals,
with a limit of about a millisecond.  The wait runs out, the call reports
RIPE_DEVERR_TIMEOUT through the device error word (the kernel lets its copies and
tensor-core operations in flight finish and returns), and the next call on the
same cache is exact again."""
import numpy as np
import pytest

from depth_planed_kv_b200 import synth as S
from tests.gpu_util import check, check_lse, fill, make_cache, oracle_all_depths, run_all_depths

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_next_call_is_exact():
    from depth_planed_kv_b200.ripe import RIPE_OK
    wl = S.Workload("timeout", 1, 4, 3, 64, 16, 4, 2, None, 0.88, 1301, "bf16", 600, 4)
    ctx = np.array([500, 130])
    cache = make_cache(wl, kernel=1)   # the hook stalls the persistent kernel
    assert cache.ripe_cache_verify_path() == 1
    fill(cache, wl, ctx)
    ws = [int(t) - wl.W for t in ctx]
    ref, ref_lse = oracle_all_depths(wl, 0, 2, wl.k, [int(t) for t in ctx], ws)
    cache.ripe_debug_stall_next_verify(2_000_000)   # ~1 ms at the B200's clock
    run_all_depths(cache, wl, 0, 2, wl.k)
    assert cache.ripe_get_device_error() == 6        # RIPE_DEVERR_TIMEOUT
    for _ in range(2):
        _, O, lse, _ = run_all_depths(cache, wl, 0, 2, wl.k)
        check(O, ref, wl, "after the timeout")
        check_lse(lse, ref_lse)
        assert cache.ripe_get_device_error() == RIPE_OK
    cache.close()
