"""Failure detection of the library's kernels, exercised without a fault.

Every wait inside a kernel is bounded: a wait that runs out sets a bit in the
sticky device error word and the kernel unwinds (warp-uniformly) instead of
hanging. tg_selftest_wait_timeout runs that path on purpose with a short
limit, on the two kinds of wait the library has: the shared-memory mbarrier
of the TMA / tensor-core pipelines and the grid barrier of the cooperative
decode kernel. Each test checks that the call returns, that the error word
reports the timeout, and that a normal call afterwards runs and is exact.
Nothing here traps, faults or waits without a limit.
"""

import time

import numpy as np
import pytest
import torch

from oracle import tokengate_oracle as ref

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")

LIMIT_NS = 2_000_000  # 2 ms


def _normal_call_is_exact():
    rng = np.random.default_rng(7)
    s = rng.standard_normal(10_000).astype(np.float32)
    prot = np.zeros(s.size, np.uint8)
    prot[-32:] = 1
    got = tg.tg_topk_select(torch.from_numpy(s).cuda(), torch.from_numpy(prot).cuda(), 777)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), ref.topk_select(s, prot, 777))


@pytest.mark.parametrize("mode", [0, 2], ids=["mbarrier", "grid_barrier"])
def test_wait_that_never_completes_gives_up_and_reports(mode):
    tg.tg_device_error(clear=True)
    t0 = time.perf_counter()
    res = tg.tg_selftest_wait_timeout(mode, LIMIT_NS)
    elapsed = time.perf_counter() - t0
    if mode == 0:
        assert res == [0, 0, 0, 0]  # every warp gave up, together
    else:
        assert res[0] == 0
    assert elapsed < 5.0  # bounded by the limit, not by a hang
    assert tg.tg_device_error() & 1  # bit value 1: a bounded wait ran out
    tg.tg_device_error(clear=True)
    assert tg.tg_device_error() == 0
    _normal_call_is_exact()
    assert tg.tg_device_error() == 0


def test_wait_that_completes_reports_nothing():
    tg.tg_device_error(clear=True)
    assert tg.tg_selftest_wait_timeout(1, LIMIT_NS) == [1, 1, 1, 1]
    assert tg.tg_device_error() == 0


def test_selftest_validates_its_arguments():
    with pytest.raises(tg.TokenGateError):
        tg.tg_selftest_wait_timeout(3, LIMIT_NS)
    with pytest.raises(tg.TokenGateError):
        tg.tg_selftest_wait_timeout(0, 10)  # below the 1 us floor
