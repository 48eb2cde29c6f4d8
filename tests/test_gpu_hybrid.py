"""GPU parity of a hybrid stack's gated prefill (Gated DeltaNet layers and
full-attention layers, the gate at either kind of layer).

In a hybrid model most layers are Gated DeltaNet layers; the scorer reads
the post-mixer residual of the gate layer whichever kind it is, the gate bias
applies only to the attention layers above the gate, and the Gated DeltaNet
layers above the gate run their mixer over the kept rows in order (Tencent
Cloud article on TokenGate, section "门控位置影响剪枝效果", figure 5).

tg_prefill is compared with the oracle's hybrid_prefill layer by layer,
teacher-forced at every tensor the library stores between kernels (the
layer taps): each layer starts from the GPU's own input; a Gated DeltaNet
layer's input projection, its mixer output (from the GPU's stored
projection: the recurrence can amplify a one-ulp difference of its input
where a head's output is small before the gated norm), then its residual
(from the GPU's mixer output), an attention layer's k/v, output and residual
likewise, then the FFN output from the GPU's residual. Every element is held
to 2e-2 + 1e-2 |ref| (bf16). The mixer's carried conv rows and final state
(the layer's KV outputs) are compared at the same bound.
"""

from collections.abc import Sequence

import numpy as np
import pytest
import torch

import synth
from oracle import gated_deltanet_oracle as gdn
from oracle import tokengate_oracle as ref
from tests._helpers import assert_close, boundary_flips, host64

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")
BF16 = torch.bfloat16
rb = ref.round_bf16


@pytest.fixture(autouse=True)
def _no_device_errors():
    tg.tg_device_error(clear=True)
    yield
    assert tg.tg_device_error() == 0


class HostLayers(Sequence):
    """The device layers as oracle layers (attention Layer or GdnStackLayer),
    converted to float64 on access, one cached."""

    def __init__(self, w, layers):
        self.w, self.layers, self.cache = w, layers, (None, None)

    def __len__(self):
        return len(self.layers)

    def __getitem__(self, i):
        if self.cache[0] != i:
            lp = self.layers[i]
            g = lambda k: host64(lp[k]) if k in lp else None  # noqa: E731
            if "gdn" in lp:
                gp = lp["gdn_params"]
                mp = gdn.MixerParams(conv_w=host64(gp["conv_w"]), A_log=host64(gp["A_log"]),
                                     dt_bias=host64(gp["dt_bias"]), norm_w=host64(gp["norm_w"]),
                                     eps=self.w.base.eps)
                lw = gdn.GdnStackLayer(norm=g("attn_norm"), w_in=g("w_in"), mixer=mp,
                                       w_out=g("w_out"), hk=self.w.hk, hv=self.w.hv,
                                       dk=self.w.dk, dv=self.w.dv, ffn_norm=g("ffn_norm"),
                                       w_gate_up=g("w_gate_up"), w_down=g("w_down"))
            else:
                lw = ref.Layer(attn_norm=g("attn_norm"), wqkv=g("wqkv"), wo=g("wo"),
                               ffn_norm=g("ffn_norm"), w_gate_up=g("w_gate_up"),
                               w_down=g("w_down"), q_norm=g("q_norm"), k_norm=g("k_norm"),
                               gain=g("gain"), tau=g("tau"))
            self.cache = (i, lw)
        return self.cache[1]


def _models(w):
    b = w.base
    p = synth.torch_hybrid_params(w, seed=b.seed, device="cuda")
    for lp in p["layers"]:
        if "gdn_params" in lp:
            gp = lp["gdn_params"]
            lp["gdn"] = tg.GdnLayer(w.hk, w.hv, w.dk, w.dv, gp["conv_w"], gp["A_log"],
                                    gp["dt_bias"], gp["norm_w"], eps=b.eps)
    score = {k: p[k] for k in ("score_norm", "score_w1", "score_b1", "score_w2", "score_b2")}
    model = tg.Model(n_heads_q=b.hq, n_heads_kv=b.hkv, head_dim=b.dh, layers=p["layers"],
                     score=score, final_norm=p["final_norm"], eps=b.eps, rope_base=b.rope_base)
    om = ref.Model(d_model=b.d, n_heads_q=b.hq, n_heads_kv=b.hkv, head_dim=b.dh,
                   layers=HostLayers(w, p["layers"]), final_norm=host64(p["final_norm"]),
                   score_norm=host64(score["score_norm"]), score_w1=host64(score["score_w1"]),
                   score_b1=host64(score["score_b1"]), score_w2=host64(score["score_w2"]),
                   score_b2=host64(score["score_b2"]), eps=b.eps, rope_base=b.rope_base)
    return model, om


def _run(w, model, x, prot, gate):
    b = w.base
    C = 2 * w.hk * w.dk + w.hv * w.dv
    kv, taps = [], []
    for li, kind in enumerate(w.kinds):
        rows = b.n if li <= gate else b.k
        if kind == "gdn":
            kv.append((torch.empty(w.W - 1, C, device="cuda", dtype=BF16),
                       torch.empty(w.hv, w.dv, w.dk, device="cuda", dtype=torch.float32)))
            width = w.hv * w.dv
        else:
            kv.append((torch.empty(rows, b.hkv, b.dh, device="cuda", dtype=BF16),
                       torch.empty(rows, b.hkv, b.dh, device="cuda", dtype=BF16)))
            width = b.hq * b.dh
        hrows = b.n if li < gate else b.k
        t = {"attn_out": torch.empty(rows, width, device="cuda", dtype=BF16),
             "resid": torch.empty(rows, b.d, device="cuda", dtype=BF16),
             "hidden": torch.empty(hrows, b.d, device="cuda", dtype=BF16)}
        if kind == "gdn":
            t["mixer_in"] = torch.empty(rows, C + w.hv * w.dv + 2 * w.hv, device="cuda",
                                        dtype=BF16)
        taps.append(t)
    scores = torch.empty(b.n, device="cuda")
    out, kept, _ = tg.tg_prefill(model, x, torch.from_numpy(prot).cuda(), b.k, gate,
                                 scores=scores, kv=kv, taps=taps)
    torch.cuda.synchronize()
    return out, kept.cpu().numpy(), scores.cpu().numpy(), kv, taps


def _check_stack(w, gate):
    b = w.base
    model, om = _models(w)
    x = synth.torch_hidden_states(b, seed=b.seed + 1000, device="cuda")
    prot = synth.protect_tail(b.n, b.n_protect)
    out, kept, scores, kv, taps = _run(w, model, x, prot, gate)
    assert np.array_equal(kept, ref.topk_select(scores, prot, b.k))
    s_k = scores[kept].astype(np.float64)
    h_in = host64(x)
    # folded norms (the model's default): a norm whose rows a residual GEMM
    # just wrote runs on the folded weight; a Gated DeltaNet input projection
    # never does
    fold = model.fold_norms
    fresh = False
    if gate < 0:  # the gate before the stack: the scorer reads x, the layers see x[kept]
        s_ref = ref.round_fp32(ref.score(h_in, om.score_norm, om.eps, om.score_w1, om.score_b1,
                                         om.score_w2, om.score_b2, rb))
        assert_close(scores, s_ref, BF16, "scores")
        h_in = h_in[kept]
    for li, kind in enumerate(w.kinds):
        lw = om.layers[li]
        below = li <= gate
        pos = np.arange(b.n) if below else kept
        what = f"layer {li} ({kind})"
        mix_gpu = host64(taps[li]["attn_out"])
        if kind == "gdn":
            C = 2 * w.hk * w.dk + w.hv * w.dv
            y = rb(ref.rmsnorm(h_in, lw.norm, b.eps))
            proj_gpu = host64(taps[li]["mixer_in"])
            assert_close(proj_gpu, rb(y @ lw.w_in.T), BF16, f"input projection {what}")
            proj = proj_gpu  # the mixer from the GPU's stored projection
            res = gdn.gated_deltanet(proj[:, :C], proj[:, C:C + w.hv * w.dv],
                                     proj[:, C + w.hv * w.dv:C + w.hv * w.dv + w.hv],
                                     proj[:, C + w.hv * w.dv + w.hv:], lw.mixer, w.hk, w.hv,
                                     w.dk, w.dv, store=rb)
            assert_close(mix_gpu, res.y, BF16, f"mixer output {what}")
            assert_close(kv[li][0], res.conv_state, BF16, f"conv rows {what}")
            assert_close(kv[li][1], res.S, BF16, f"state {what}")
            r = rb(h_in + mix_gpu @ lw.w_out.T)
        else:
            q, k_o, v_o = ref.project_qkv(h_in, lw, om, pos, rb, fold and fresh)
            assert_close(kv[li][0], k_o, BF16, f"k {what}")
            assert_close(kv[li][1], v_o, BF16, f"v {what}")
            o = rb(ref.gated_attention(q, host64(kv[li][0]), host64(kv[li][1]), pos,
                                       None if below else s_k, None if below else lw.gain,
                                       None if below else lw.tau))
            assert_close(mix_gpu, o.reshape(o.shape[0], -1), BF16, f"attention output {what}")
            r = rb(h_in + mix_gpu @ lw.wo.T)
        r_gpu = host64(taps[li]["resid"])
        assert_close(r_gpu, r, BF16, f"post-mixer residual {what}")
        fresh = True
        if li == gate:
            s_ref = ref.round_fp32(ref.score(r_gpu, om.score_norm, om.eps, om.score_w1,
                                             om.score_b1, om.score_w2, om.score_b2, rb, fold))
            assert_close(scores, s_ref, BF16, "scores")
            flips, near = boundary_flips(s_ref.astype(np.float32), kept, prot, b.k, 2e-2, 1e-2)
            assert near, flips
            r_gpu = r_gpu[kept]  # the compacted rows keep their row sums
        h_gpu = host64(taps[li]["hidden"])
        assert_close(h_gpu, ref.ffn_sublayer(r_gpu, lw, om, rb, fold and fresh), BF16,
                     f"hidden {what}")
        fresh = True
        h_in = h_gpu
    assert_close(out, rb(ref.rmsnorm(h_in, om.final_norm, om.eps)), BF16, "out")


SMALL = synth.HybridWorkload(
    synth.Workload("hybrid_small", "bf16", n=600, k=150, d=512, hq=4, hkv=2, dh=128, f=64,
                   inter=512, n_layers=5, gate_layer=-1, n_protect=8, seed=61, qk_norm=True,
                   w_std=0.04),  # gate_layer -1: every attention layer draws a gain and tau
    kinds=("gdn", "attn", "gdn", "gdn", "attn"), hk=4, hv=16, dk=64, dv=32, W=4)


@pytest.mark.parametrize("gate", [-1, 0, 1, 2])
def test_small_hybrid_stack_gate_at_either_kind_of_layer(gate):
    """Gate before the stack, at a Gated DeltaNet layer (0, 2) and at an
    attention layer (1)."""
    _check_stack(SMALL, gate)


@pytest.mark.slow
@pytest.mark.parametrize("gate", [1, 2])
def test_qwen35_like_hybrid_stack(gate):
    """Qwen3.5-2B-like hybrid stack at d_model 2048 (three Gated DeltaNet
    layers to one attention layer, 8 layers), N = 4096, K = 1024, the gate
    at layer 1 or 2 (both Gated DeltaNet layers)."""
    _check_stack(synth.HYBRID_4K, gate)
