"""GPU parity of selection and compaction against the oracle (bit-exact).

Selection must return exactly the oracle's kept index set on the same fp32
scores, for the full sweep of sizes (N in {8K, 32K, 128K}, K/N in
{1/16 .. 1}, 128 protected tokens, tie blocks, +-0 and +-inf), plus edge
cases: tiny and ragged N, K = P, K = N, all ties, NaN, misaligned inputs.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import tokengate_oracle as ref

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")


def _select(s32: np.ndarray, prot, k):
    sd = torch.from_numpy(s32).cuda()
    pd = None if prot is None else torch.from_numpy(prot).cuda()
    out = tg.tg_topk_select(sd, pd, k)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _check(s32, prot, k):
    got = _select(s32, prot, k)
    want = ref.topk_select(s32, prot, k)
    assert np.array_equal(got, want), (len(s32), k, np.setdiff1d(got, want)[:5],
                                       np.setdiff1d(want, got)[:5])


@pytest.fixture(autouse=True)
def _no_device_errors():
    tg.tg_device_error(clear=True)
    yield
    assert tg.tg_device_error() == 0


@pytest.mark.parametrize("n", [1, 7, 100, 2047, 2048, 2049, 5000, 8195])
def test_select_small_and_ragged(n):
    rng = np.random.default_rng(n)
    s = rng.standard_normal(n).astype(np.float32)
    s[rng.integers(0, n, max(1, n // 10))] = np.float32(0.25)  # ties
    prot = (rng.random(n) < 0.05).astype(np.uint8)
    p = int(prot.sum())
    for k in sorted({max(p, 1), min(n, p + 1), max(p, 1) + (n - max(p, 1)) // 3, n}):
        _check(s, prot, k)
    _check(s, None, max(1, n // 2))


@pytest.mark.parametrize("n,k", synth.sweep_points())
def test_select_sweep_full_size(n, k):
    rng = synth.rng_for(synth.SWEEP_SEED + n + k)
    s = synth.sweep_scores(n, rng)
    prot = synth.protect_tail(n, synth.SWEEP_PROTECT)
    _check(s, prot, k)


@pytest.mark.parametrize("n", synth.SWEEP_N)
def test_select_threshold_inside_tie_block(n):
    k, p = n // 8, synth.SWEEP_PROTECT
    s = synth.scores_threshold_in_tie(n, k, p, synth.rng_for(7 + n))
    _check(s, synth.protect_tail(n, p), k)


def test_select_special_values_and_all_ties():
    rng = np.random.default_rng(3)
    n = 3000
    pool = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1.0, -1.0], dtype=np.float32)
    s = pool[rng.integers(0, pool.size, n)]
    for k in (1, 10, 1500, 2999, 3000):
        _check(s, None, k)
    _check(np.zeros(n, np.float32), None, 777)
    _check(np.full(n, np.nan, np.float32), None, 5)
    _check(np.full(n, -np.inf, np.float32), synth.protect_tail(n, 9), 9)


def test_select_misaligned_inputs():
    rng = np.random.default_rng(4)
    n = 10001
    base = torch.from_numpy(rng.standard_normal(n + 1).astype(np.float32)).cuda()
    pbase = torch.zeros(n + 3, dtype=torch.uint8, device="cuda")
    pbase[-40:] = 1
    s = base[1:]  # 4-byte aligned, not 16
    pr = pbase[3:]
    k = 1234
    got = tg.tg_topk_select(s, pr, k).cpu().numpy()
    want = ref.topk_select(s.cpu().numpy(), pr.cpu().numpy(), k)
    assert np.array_equal(got, want)


def test_select_too_many_protected_flags_on_device():
    n, k = 5000, 100
    s = torch.randn(n, device="cuda")
    prot = torch.zeros(n, dtype=torch.uint8, device="cuda")
    prot[:101] = 1
    ws = torch.zeros(tg.tg_workspace_size(tg.TG_OP_TOPK_SELECT, n=n), dtype=torch.uint8,
                     device="cuda")
    out = tg.tg_topk_select(s, prot, k, ws=ws)
    torch.cuda.synchronize()
    assert (out.cpu() == -1).all()
    assert int(ws[:4].view(torch.int32)[0]) == tg.TG_ERR_BUDGET
    # the same workspace is reset by the next good call
    prot[:] = 0
    tg.tg_topk_select(s, prot, k, ws=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32)[0]) == 0


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 2048), (torch.bfloat16, 64),
                                     (torch.float32, 256), (torch.float32, 4)])
def test_compact_exact(dtype, d):
    rng = np.random.default_rng(d)
    n, k = 3001, 777
    x = torch.from_numpy(rng.standard_normal((n, d)).astype(np.float32)).to("cuda", dtype)
    s = torch.from_numpy(rng.standard_normal(n).astype(np.float32)).cuda()
    idx = np.sort(rng.choice(n, k, replace=False)).astype(np.int32)
    idx_d = torch.from_numpy(idx).cuda()
    xo, po, so = tg.tg_compact(x, idx_d, scores=s)
    torch.cuda.synchronize()
    assert torch.equal(xo, x[idx_d.long()])
    assert np.array_equal(po.cpu().numpy(), idx)
    assert torch.equal(so, s[idx_d.long()])
    pos_in = torch.arange(100, 100 + n, dtype=torch.int32, device="cuda")
    _, po2, _ = tg.tg_compact(x, idx_d, pos_in=pos_in)
    assert np.array_equal(po2.cpu().numpy(), idx + 100)


@pytest.mark.parametrize("n,k", [(8192, 512), (32768, 8192), (131072, 65536)])
def test_select_then_compact_full_size(n, k):
    rng = synth.rng_for(n + 1)
    s = synth.sweep_scores(n, rng)
    prot = synth.protect_tail(n, 128)
    x = torch.randn(n, synth.SWEEP_D, device="cuda", dtype=torch.bfloat16)
    sd, pd = torch.from_numpy(s).cuda(), torch.from_numpy(prot).cuda()
    idx = tg.tg_topk_select(sd, pd, k)
    xo, po, so = tg.tg_compact(x, idx, scores=sd)
    torch.cuda.synchronize()
    want = ref.topk_select(s, prot, k)
    assert np.array_equal(idx.cpu().numpy(), want)
    wl = torch.from_numpy(want.astype(np.int64)).cuda()
    assert torch.equal(xo, x[wl]) and torch.equal(so, sd[wl])
