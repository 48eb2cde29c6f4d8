"""GPU parity of the multi-budget prefill (tg_prefill_multi).

One request at several budgets: the layers below the gate and the scores run
once, then each budget gets its own selection, compaction and upper layers.
Each budget's result must equal tg_prefill at that budget bit for bit (the
same kernels on the same data), and the oracle (teacher-forced with the GPU's
kept sets) within the bf16 tolerance.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import tokengate_oracle as ref
from tests._helpers import STORE, assert_close, build_models, host64

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")


@pytest.fixture(autouse=True)
def _no_device_errors():
    tg.tg_device_error(clear=True)
    yield
    assert tg.tg_device_error() == 0


def _setup(gate_layer, seed, n=300, n_layers=3, qk_norm=True):
    w = synth.shrink(synth.QWEN_LAYER_16K, name="multi", n=n, k=100, d=256, hq=4, hkv=2, dh=128,
                     f=64, inter=256, n_layers=n_layers, gate_layer=gate_layer, n_protect=10,
                     qk_norm=qk_norm, seed=seed, salient_frac=0.02)
    rng = synth.rng_for(w.seed)
    model, om = build_models(w, rng, torch.bfloat16)
    x = torch.from_numpy(synth.hidden_states(w, rng)).to("cuda", torch.bfloat16)
    prot_np = synth.protect_tail(w.n, w.n_protect)
    return w, model, om, x, prot_np


@pytest.mark.parametrize("gate_layer", [-1, 0, 1])
def test_multi_budget_equals_single_budget_runs(gate_layer):
    w, model, om, x, prot_np = _setup(gate_layer, 60 + gate_layer)
    prot = torch.from_numpy(prot_np).cuda()
    ks = [17, 100, 129, 300]
    sc = torch.empty(w.n, device="cuda")
    outs, kept, _ = tg.tg_prefill_multi(model, x, prot, ks, gate_layer, scores=sc)
    torch.cuda.synchronize()
    for b, k in enumerate(ks):
        sc1 = torch.empty(w.n, device="cuda")
        out1, kept1, _ = tg.tg_prefill(model, x, prot, k, gate_layer, scores=sc1)
        torch.cuda.synchronize()
        assert torch.equal(kept[b], kept1), k
        assert torch.equal(outs[b], out1), k
        assert torch.equal(sc, sc1)
    # the sets nest and K = N keeps every row
    for a, b in zip(kept, kept[1:]):
        assert set(a.tolist()) <= set(b.tolist())
    assert kept[-1].tolist() == list(range(w.n))


def test_multi_budget_against_the_oracle():
    w, model, om, x, prot_np = _setup(1, 64)
    prot = torch.from_numpy(prot_np).cuda()
    ks = [40, 150]
    sc = torch.empty(w.n, device="cuda")
    outs, kept, _ = tg.tg_prefill_multi(model, x, prot, ks, 1, scores=sc)
    torch.cuda.synchronize()
    scores = sc.cpu().numpy()
    kept_np = [t.cpu().numpy() for t in kept]
    for b, k in enumerate(ks):
        assert np.array_equal(kept_np[b], ref.topk_select(scores, prot_np, k))
    res = ref.prefill_budgets(host64(x), prot_np, ks, om, 1, store=STORE[torch.bfloat16],
                              kept_sets=kept_np, fold_norms=model.fold_norms)
    for b, r in enumerate(res):
        assert_close(scores, r.scores, torch.bfloat16, "scores")
        assert_close(outs[b], r.out, torch.bfloat16, f"out k={ks[b]}")


def test_multi_budget_order_and_repeats():
    w, model, om, x, prot_np = _setup(0, 65)
    prot = torch.from_numpy(prot_np).cuda()
    outs, kept, _ = tg.tg_prefill_multi(model, x, prot, [250, 30, 250, 30], 0)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[2]) and torch.equal(kept[0], kept[2])
    assert torch.equal(outs[1], outs[3]) and torch.equal(kept[1], kept[3])
