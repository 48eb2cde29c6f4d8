"""GPU parity of the batched prefill (tg_prefill_batch): requests of
different lengths, each with its own budget and protected span, packed back
to back. Reading: a batch is, by definition, each request's own gated
prefill (positions restart at 0 in every request). On the GPU each request's
kept set, scores and output equal tg_prefill on that request alone bit for
bit (the same kernels on the same rows), and the oracle, teacher-forced with
the GPU's kept set, within the bf16 tolerance.
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


def _setup(gate_layer, seed, lens, n_layers=3):
    w = synth.shrink(synth.QWEN_LAYER_16K, name="batch", n=max(lens), k=64, d=256, hq=4, hkv=2,
                     dh=128, f=64, inter=256, n_layers=n_layers, gate_layer=gate_layer,
                     n_protect=8, qk_norm=True, seed=seed, salient_frac=0.02)
    rng = synth.rng_for(w.seed)
    model, om = build_models(w, rng, torch.bfloat16)
    xs = [rng.standard_normal((n, w.d)).astype(np.float32) for n in lens]
    x = torch.from_numpy(np.concatenate(xs)).to("cuda", torch.bfloat16)
    prots = [synth.protect_tail(n, min(8, n)) for n in lens]
    return w, model, om, x, prots


@pytest.mark.parametrize("gate_layer", [-1, 0, 1])
def test_batch_equals_each_request_alone(gate_layer):
    lens, ks = [300, 129, 517, 64], [100, 129, 200, 17]
    w, model, om, x, prots = _setup(gate_layer, 70 + gate_layer, lens)
    prot = torch.from_numpy(np.concatenate(prots)).cuda()
    sc = torch.empty(sum(lens), device="cuda")
    out, kept, _ = tg.tg_prefill_batch(model, x, prot, lens, ks, gate_layer, scores=sc)
    torch.cuda.synchronize()
    r0 = k0 = 0
    for n, k in zip(lens, ks):
        sc1 = torch.empty(n, device="cuda")
        out1, kept1, _ = tg.tg_prefill(model, x[r0:r0 + n].contiguous(), prot[r0:r0 + n].contiguous(),
                                       k, gate_layer, scores=sc1)
        torch.cuda.synchronize()
        assert torch.equal(kept[k0:k0 + k], kept1), (n, k)
        assert torch.equal(sc[r0:r0 + n], sc1), (n, k)
        assert torch.equal(out[k0:k0 + k], out1), (n, k)
        r0 += n
        k0 += k


def test_batch_against_the_oracle():
    lens, ks = [200, 333], [80, 150]
    w, model, om, x, prots = _setup(1, 75, lens)
    prot = torch.from_numpy(np.concatenate(prots)).cuda()
    sc = torch.empty(sum(lens), device="cuda")
    out, kept, _ = tg.tg_prefill_batch(model, x, prot, lens, ks, 1, scores=sc)
    torch.cuda.synchronize()
    scores, kept_np, xh = sc.cpu().numpy(), kept.cpu().numpy(), host64(x)
    r0 = k0 = 0
    for b, (n, k) in enumerate(zip(lens, ks)):
        kb = kept_np[k0:k0 + k]
        assert np.array_equal(kb, ref.topk_select(scores[r0:r0 + n], prots[b], k))
        res = ref.prefill(xh[r0:r0 + n], prots[b], k, om, 1, store=STORE[torch.bfloat16],
                          kept_idx=kb, fold_norms=model.fold_norms)
        assert_close(scores[r0:r0 + n], res.scores, torch.bfloat16, f"scores request {b}")
        assert_close(out[k0:k0 + k], res.out, torch.bfloat16, f"out request {b}")
        r0 += n
        k0 += k


def test_batch_of_one_is_tg_prefill():
    lens, ks = [257], [99]
    w, model, om, x, prots = _setup(0, 76, lens)
    prot = torch.from_numpy(prots[0]).cuda()
    out, kept, _ = tg.tg_prefill_batch(model, x, prot, lens, ks, 0)
    out1, kept1, _ = tg.tg_prefill(model, x, prot, 99, 0)
    torch.cuda.synchronize()
    assert torch.equal(kept, kept1) and torch.equal(out, out1)
