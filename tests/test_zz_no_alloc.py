"""The allocation-free selection entry point against the oracle and the
workspace one.

tg_topk_select_noalloc serves callers that can pass the library only their
inputs and outputs -- e.g. code embedded in a host application that keeps
the GPU's memory in its own pool, or a loop that must not call
cudaMalloc/cudaFree because they can synchronise the device. Its scratch is a
static device array inside the library, shared by every call on the device.

This file is collected last so that a run stopping at the first failure has
run every other test first. It calls the C entry point directly (ctypes),
twice in a row with different sizes: the second call must not see the
first call's leftovers in the shared array. Index sets are integer results,
so every comparison is exact equality.
"""

import ctypes
import json
import os

import numpy as np
import pytest
import torch

from oracle import tokengate_oracle as ref

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "select_handworked.json")


def _noalloc_c(scores, protect, k, n=None):
    """Direct C-ABI call of tg_topk_select_noalloc on the current stream;
    returns (status, kept_idx)."""
    n = scores.shape[0] if n is None else n
    out = torch.full((k,), -7, dtype=torch.int32, device=scores.device)
    st = torch.cuda.current_stream().cuda_stream
    status = tg._lib.tg_topk_select_noalloc(
        ctypes.c_void_p(scores.data_ptr()),
        ctypes.c_void_p(protect.data_ptr()) if protect is not None else None,
        ctypes.c_int64(n), ctypes.c_int64(k), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(st))
    return status, out


def _ok(scores, protect, k):
    status, out = _noalloc_c(scores, protect, k)
    assert status == tg.TG_OK, tg.tg_status_string(status)
    return out


def _case(seed, n, k, n_protect):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal(n).astype(np.float32)
    s[rng.integers(0, n, n // 20)] = np.float32(0.5)  # ties straddling the cut
    prot = np.zeros(n, np.uint8)
    prot[n - n_protect:] = 1
    return s, prot


def _dev(s, prot):
    return torch.from_numpy(s).cuda(), torch.from_numpy(prot).cuda()


def test_noalloc_select_matches_oracle_and_workspace_select_on_two_calls():
    tg.tg_device_error(clear=True)
    # first call: a large problem fills the shared scratch (many chunks)
    s1, p1 = _case(1, 300_000, 40_000, 128)
    got1 = _ok(*_dev(s1, p1), 40_000)
    # second call right after: a smaller problem on the same scratch
    s2, p2 = _case(2, 5_003, 611, 17)
    got2 = _ok(*_dev(s2, p2), 611)
    want1 = tg.tg_topk_select(*_dev(s1, p1), 40_000)
    want2 = tg.tg_topk_select(*_dev(s2, p2), 611)
    torch.cuda.synchronize()
    assert np.array_equal(got1.cpu().numpy(), ref.topk_select(s1, p1, 40_000))
    assert np.array_equal(got2.cpu().numpy(), ref.topk_select(s2, p2, 611))
    assert torch.equal(got1, want1)
    assert torch.equal(got2, want2)
    assert tg.tg_device_error() == 0


def test_noalloc_select_hand_derived_fixture():
    """The hand-worked selection (ties, -0/+0, +-inf, NaN, one protected
    token) at every budget of the fixture, calls back to back."""
    g = json.load(open(GOLDEN))
    s = np.array([float(v) for v in g["scores"]], dtype=np.float32)
    prot = np.array(g["protect"], dtype=np.uint8)
    sd, pd = _dev(s, prot)
    for case in g["cases"]:
        got = _ok(sd, pd, case["k"])
        torch.cuda.synchronize()
        assert got.cpu().tolist() == case["kept"], case


def test_noalloc_select_more_protected_than_k_fills_minus_one():
    """More protected tokens than k is a budget error known only on the
    device: kept_idx is filled with -1. A valid call afterwards on the same
    scratch is exact again."""
    s, prot = _case(3, 4_096, 100, 300)
    got = _ok(*_dev(s, prot), 100)
    torch.cuda.synchronize()
    assert (got.cpu().numpy() == -1).all()
    s, prot = _case(4, 4_096, 400, 300)
    got = _ok(*_dev(s, prot), 400)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), ref.topk_select(s, prot, 400))


def test_noalloc_select_limit_is_the_documented_one():
    """The Python constant is the C limit: n at the limit runs (and is
    exact), one more is rejected before any launch."""
    limit = tg.SELECT_NOALLOC_MAX_N
    s, prot = _case(5, limit, limit // 3, 128)
    status, got = _noalloc_c(*_dev(s, prot), limit // 3)
    assert status == tg.TG_OK
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), ref.topk_select(s, prot, limit // 3))
    bogus = ctypes.c_void_p(4096)  # rejected before any launch
    assert tg._lib.tg_topk_select_noalloc(bogus, None, ctypes.c_int64(limit + 1),
                                          ctypes.c_int64(10), bogus, None) == \
        tg.TG_ERR_UNSUPPORTED
    with pytest.raises(ValueError, match="allocation-free limit"):
        tg.tg_topk_select_noalloc(torch.zeros(limit + 1, device="cuda"), None, 10)
    assert tg.tg_device_error() == 0
