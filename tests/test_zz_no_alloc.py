"""The allocation-free selection entry point against the workspace one.

tg_topk_select_noalloc serves callers that can pass the library only their
inputs and outputs -- e.g. code embedded in a host application that keeps
the GPU's memory in its own pool, or a loop that must not call
cudaMalloc/cudaFree because they can synchronise the device. Its scratch is a
static device array inside the library, shared by every call on the device.

This file is collected last so that a run stopping at the first failure has
run every other test first. It calls the C entry point directly (ctypes),
twice in a row with different sizes: the second call must not see the
first call's leftovers in the shared array.
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")


def _noalloc_c(scores, protect, k):
    """Direct C-ABI call of tg_topk_select_noalloc on the current stream."""
    n = scores.shape[0]
    out = torch.full((k,), -7, dtype=torch.int32, device=scores.device)
    st = torch.cuda.current_stream().cuda_stream
    status = tg._lib.tg_topk_select_noalloc(
        ctypes.c_void_p(scores.data_ptr()),
        ctypes.c_void_p(protect.data_ptr()) if protect is not None else None,
        ctypes.c_int64(n), ctypes.c_int64(k), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(st))
    assert status == tg.TG_OK, tg.tg_status_string(status)
    return out


def _case(seed, n, k, n_protect):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal(n).astype(np.float32)
    s[rng.integers(0, n, n // 20)] = np.float32(0.5)  # ties straddling the cut
    prot = np.zeros(n, np.uint8)
    prot[n - n_protect:] = 1
    return torch.from_numpy(s).cuda(), torch.from_numpy(prot).cuda()


def test_noalloc_select_matches_workspace_select_on_two_calls():
    tg.tg_device_error(clear=True)
    # first call: a large problem fills the shared scratch (many chunks)
    s1, p1 = _case(1, 300_000, 40_000, 128)
    got1 = _noalloc_c(s1, p1, 40_000)
    # second call right after: a smaller problem on the same scratch
    s2, p2 = _case(2, 5_003, 611, 17)
    got2 = _noalloc_c(s2, p2, 611)
    want1 = tg.tg_topk_select(s1, p1, 40_000)
    want2 = tg.tg_topk_select(s2, p2, 611)
    torch.cuda.synchronize()
    # index sets are integer results: the tolerance is exact equality
    assert torch.equal(got1, want1)
    assert torch.equal(got2, want2)
    assert tg.tg_device_error() == 0


def test_noalloc_select_rejects_n_above_its_limit():
    limit = tg.SELECT_NOALLOC_MAX_N
    bogus = ctypes.c_void_p(4096)  # rejected before any launch
    assert tg._lib.tg_topk_select_noalloc(bogus, None, ctypes.c_int64(limit + 1),
                                          ctypes.c_int64(10), bogus, None) == \
        tg.TG_ERR_UNSUPPORTED
    with pytest.raises(ValueError, match="allocation-free limit"):
        tg.tg_topk_select_noalloc(torch.zeros(limit + 1, device="cuda"), None, 10)
