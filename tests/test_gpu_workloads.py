"""GPU parity at the benchmark workloads' sizes.

* 28-layer Qwen3-1.7B-shaped gated prefill (qk-norm, gate at layer 1),
  checked per layer and teacher-forced at every tensor the library stores
  between kernels. For each layer the oracle starts from the GPU's own input
  of that layer and checks, in turn:
    - the layer's k and v (its KV cache) from that input;
    - the attention output (tg_prefill's attn_out tap) from the GPU's k, v;
    - the post-attention residual (resid tap) from the GPU's attention output;
    - at the gate layer, the scores from the GPU's residual;
    - the layer's output (hidden tap) from the GPU's residual.
  Each comparison thus covers one stage's arithmetic and its one rounding to
  bf16, and every element is held to |gpu - ref| <= 2e-2 + 1e-2 |ref| with no
  exceptions. The kept set is checked bit-exactly on the GPU's scores.
  - at a reduced N=4096, K=512 (every other shape unchanged): every row;
  - at the full N=32768 with K = 2048, 4096 and 8192, and the dense run
    (K = N, no gate bias) the speedups are measured against: sampled rows,
    attention keys and values taken from the GPU's KV cache of the layer.
* long-context gated attention layer: N=131072 -> K=4096, in full.

Weights are drawn on the device (seeded), so host and device see the same
bf16 values.
"""

from collections.abc import Sequence

import numpy as np
import pytest
import torch

import synth
from oracle import tokengate_oracle as ref
from tests._helpers import assert_close, boundary_flips, host64

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

tg = pytest.importorskip("learned_token_pruning_score_b200")
BF16 = torch.bfloat16
rb = ref.round_bf16


@pytest.fixture(autouse=True)
def _no_device_errors():
    tg.tg_device_error(clear=True)
    yield
    assert tg.tg_device_error() == 0


class HostLayers(Sequence):
    """The device layers as oracle Layers, converted to float64 on access
    (one layer cached: the oracle walks them in order)."""

    def __init__(self, layers):
        self.layers = layers
        self.cache = (None, None)

    def __len__(self):
        return len(self.layers)

    def __getitem__(self, i):
        if self.cache[0] != i:
            lp = self.layers[i]
            g = lambda k: host64(lp[k]) if k in lp else None  # noqa: E731
            self.cache = (i, ref.Layer(attn_norm=g("attn_norm"), wqkv=g("wqkv"), wo=g("wo"),
                                       ffn_norm=g("ffn_norm"), w_gate_up=g("w_gate_up"),
                                       w_down=g("w_down"), q_norm=g("q_norm"), k_norm=g("k_norm"),
                                       gain=g("gain"), tau=g("tau")))
        return self.cache[1]


def _models(w, dense=False):
    p = synth.torch_model_params(w, seed=w.seed, device="cuda")
    if dense:  # the dense baseline: the same weights without the gate bias
        p["layers"] = [{k: v for k, v in lp.items() if k not in ("gain", "tau")}
                       for lp in p["layers"]]
    score = {k: p[k] for k in ("score_norm", "score_w1", "score_b1", "score_w2", "score_b2")}
    model = tg.Model(n_heads_q=w.hq, n_heads_kv=w.hkv, head_dim=w.dh, layers=p["layers"],
                     score=score, final_norm=p["final_norm"], eps=w.eps, rope_base=w.rope_base)
    om = ref.Model(d_model=w.d, n_heads_q=w.hq, n_heads_kv=w.hkv, head_dim=w.dh,
                   layers=HostLayers(p["layers"]), final_norm=host64(p["final_norm"]),
                   score_norm=host64(score["score_norm"]), score_w1=host64(score["score_w1"]),
                   score_b1=host64(score["score_b1"]), score_w2=host64(score["score_w2"]),
                   score_b2=host64(score["score_b2"]), eps=w.eps, rope_base=w.rope_base)
    return model, om


def _run_gpu(w, model, x, prot, with_taps=False):
    kv, taps = [], []
    for li in range(w.n_layers):
        rows = w.n if li <= w.gate_layer else w.k
        kv.append((torch.empty(rows, w.hkv, w.dh, device="cuda", dtype=BF16),
                   torch.empty(rows, w.hkv, w.dh, device="cuda", dtype=BF16)))
        hrows = w.n if li < w.gate_layer else w.k
        taps.append({"attn_out": torch.empty(rows, w.hq * w.dh, device="cuda", dtype=BF16),
                     "resid": torch.empty(rows, w.d, device="cuda", dtype=BF16),
                     "hidden": torch.empty(hrows, w.d, device="cuda", dtype=BF16)})
    scores = torch.empty(w.n, device="cuda")
    out, kept, _ = tg.tg_prefill(model, x, torch.from_numpy(prot).cuda(), w.k, w.gate_layer,
                                 scores=scores, kv=kv, taps=taps if with_taps else None)
    torch.cuda.synchronize()
    return out, kept.cpu().numpy(), scores.cpu().numpy(), kv, taps


def _check_scores(r_gpu, om, scores_gpu, what, fold):
    s_ref = ref.round_fp32(ref.score(r_gpu, om.score_norm, om.eps, om.score_w1, om.score_b1,
                                     om.score_w2, om.score_b2, rb, fold))
    assert_close(scores_gpu, s_ref, BF16, what)
    return s_ref


def test_prefill_28_layers_reduced_n_per_layer():
    w = synth.shrink(synth.QWEN_PREFILL_32K, n=4096, k=512)
    model, om = _models(w)
    x = synth.torch_hidden_states(w, seed=w.seed + 1000, device="cuda")
    prot = synth.protect_tail(w.n, w.n_protect)
    out, kept, scores, kv, taps = _run_gpu(w, model, x, prot, with_taps=True)
    assert np.array_equal(kept, ref.topk_select(scores, prot, w.k))
    pos_n = np.arange(w.n)
    s_k = scores[kept].astype(np.float64)
    h_in = host64(x)
    # folded norms (the default): every norm whose rows a residual GEMM just
    # wrote (the compacted rows keep their row sums), i.e. all but layer 0's
    # attention norm
    fold = model.fold_norms
    for li in range(w.n_layers):
        lw = om.layers[li]
        dense = li <= w.gate_layer
        pos = pos_n if dense else kept
        rows = pos.size
        q, k_o, v_o = ref.project_qkv(h_in, lw, om, pos, rb, fold and li > 0)
        assert_close(kv[li][0], k_o, BF16, f"k layer {li}")
        assert_close(kv[li][1], v_o, BF16, f"v layer {li}")
        o = rb(ref.gated_attention(q, host64(kv[li][0]), host64(kv[li][1]), pos,
                                   None if dense else s_k, None if dense else lw.gain,
                                   None if dense else lw.tau))
        o_gpu = host64(taps[li]["attn_out"])
        assert_close(o_gpu, o.reshape(rows, -1), BF16, f"attention output layer {li}")
        r = rb(h_in + o_gpu @ lw.wo.T)
        r_gpu = host64(taps[li]["resid"])
        assert_close(r_gpu, r, BF16, f"post-attention residual layer {li}")
        if li == w.gate_layer:
            s_ref = _check_scores(r_gpu, om, scores, "scores", fold)
            flips, near = boundary_flips(s_ref.astype(np.float32), kept, prot, w.k, 2e-2, 1e-2)
            assert near, flips
            r_gpu = r_gpu[kept]
        h_gpu = host64(taps[li]["hidden"])
        assert_close(h_gpu, ref.ffn_sublayer(r_gpu, lw, om, rb, fold), BF16,
                     f"hidden layer {li}")
        h_in = h_gpu  # teacher forcing: the next layer reads the GPU's output
    assert_close(out, rb(ref.rmsnorm(h_in, om.final_norm, om.eps)), BF16, "out")


def _attn_row(h, lw, m, pos_q, k_cache, v_cache, pos_k, s_k, gain, tau, want_k, want_v, o_gpu,
              r_gpu, what, fold):
    """One token through one layer's attention sub-layer, teacher-forced:
    its q, k, v from the GPU's input row h (k, v checked against the GPU's
    cache row), its attention output from the GPU's cached keys/values
    [0..its own row] (checked against o_gpu), its residual from o_gpu
    (checked against r_gpu)."""
    q, k, v = ref.project_qkv(h[None], lw, m, np.array([pos_q]), rb, fold)
    assert_close(want_k, k[0], BF16, f"k {what}")
    assert_close(want_v, v[0], BF16, f"v {what}")
    o = rb(ref.gated_attention_rows(q, np.array([pos_q]), k_cache, v_cache, pos_k, s_k, gain,
                                    tau))
    assert_close(o_gpu, o.reshape(-1), BF16, f"attention output {what}")
    r = rb(h + o_gpu @ lw.wo.T)
    assert_close(r_gpu, r, BF16, f"post-attention residual {what}")


FULL_SIZE_CASES = [pytest.param(k, False, id=f"k{k}") for k in synth.PREFILL_32K_BUDGETS] + \
    [pytest.param(synth.QWEN_PREFILL_32K.n, True, id="dense")]


@pytest.mark.parametrize("k,dense", FULL_SIZE_CASES)
def test_prefill_28_layers_full_size_sampled_rows(k, dense):
    """N=32768, 28 layers, gate at layer 1, at each budget of the workload
    and in the dense run (K = N, no gate bias)."""
    w = synth.shrink(synth.QWEN_PREFILL_32K, k=k)
    model, om = _models(w, dense=dense)
    x = synth.torch_hidden_states(w, seed=w.seed + 1000, device="cuda")
    prot = synth.protect_tail(w.n, w.n_protect)
    out, kept, scores, kv, taps = _run_gpu(w, model, x, prot, with_taps=True)
    # the kept set is exactly the selection of the GPU's scores
    assert np.array_equal(kept, ref.topk_select(scores, prot, w.k))
    if dense:
        assert np.array_equal(kept, np.arange(w.n))
    rng = np.random.default_rng(11 + k)
    kept_set = set(kept.tolist())
    pruned = np.array(sorted(set(range(w.n)) - kept_set), dtype=np.int64)
    sample_kept = sorted({int(kept[-1]), int(kept[0]), int(kept[1])} |
                         set(rng.choice(kept[:-w.n_protect], 4, replace=False).tolist()) |
                         {int(np.nonzero(prot)[0][3])})
    sample_pruned = sorted(rng.choice(pruned, 3, replace=False).tolist()) if pruned.size else []
    tokens = sample_kept + sample_pruned
    row_of = {int(t): r for r, t in enumerate(kept)}
    s_kept = scores[kept].astype(np.float64)
    fold = model.fold_norms  # all norms but layer 0's attention
    rows = lambda t_, idx: host64(t_[torch.as_tensor(idx, device="cuda")])  # noqa: E731
    xin = dict(zip(tokens, rows(x, tokens)))
    for li in range(w.n_layers):
        lw = om.layers[li]
        tp = taps[li]
        if li <= w.gate_layer:  # every sampled token, keys 0..t
            kc, vc = host64(kv[li][0]), host64(kv[li][1])
            hin = xin if li == 0 else dict(zip(tokens, rows(taps[li - 1]["hidden"], tokens)))
            o_gpu = dict(zip(tokens, rows(tp["attn_out"], tokens)))
            r_gpu = dict(zip(tokens, rows(tp["resid"], tokens)))
            for t in tokens:
                what = f"layer {li} token {t}"
                _attn_row(hin[t], lw, om, t, kc[: t + 1], vc[: t + 1], np.arange(t + 1), None,
                          None, None, kc[t], vc[t], o_gpu[t], r_gpu[t], what, fold and li > 0)
                if li < w.gate_layer:
                    want = rows(tp["hidden"], [t])[0]
                    assert_close(want, ref.ffn_sublayer(r_gpu[t][None], lw, om, rb, fold)[0],
                                 BF16, f"hidden {what}")
                    continue
                # the gate layer: score of the GPU's post-attention residual, then
                # its FFN on the kept rows
                _check_scores(r_gpu[t][None], om, scores[t:t + 1], f"score token {t}", fold)
                if t in kept_set:
                    want = rows(tp["hidden"], [row_of[t]])[0]
                    assert_close(want, ref.ffn_sublayer(r_gpu[t][None], lw, om, rb, fold)[0],
                                 BF16, f"hidden layer {li} kept row {row_of[t]}")
            del kc, vc
            continue
        rk_list = [row_of[t] for t in sample_kept]
        hin = dict(zip(sample_kept, rows(taps[li - 1]["hidden"], rk_list)))
        o_gpu = dict(zip(sample_kept, rows(tp["attn_out"], rk_list)))
        r_gpu = dict(zip(sample_kept, rows(tp["resid"], rk_list)))
        want_out = dict(zip(sample_kept, rows(tp["hidden"], rk_list)))
        kc_all, vc_all = host64(kv[li][0]), host64(kv[li][1])
        for t in sample_kept:
            rk = row_of[t]
            kc, vc = kc_all[: rk + 1], vc_all[: rk + 1]
            what = f"layer {li} kept row {rk}"
            _attn_row(hin[t], lw, om, t, kc, vc, kept[: rk + 1], None if dense else
                      s_kept[: rk + 1], lw.gain, lw.tau, kc[rk], vc[rk], o_gpu[t], r_gpu[t],
                      what, fold)
            assert_close(want_out[t], ref.ffn_sublayer(r_gpu[t][None], lw, om, rb, fold)[0],
                         BF16, f"hidden {what}")
        del kc_all, vc_all
    last = rows(taps[-1]["hidden"], [row_of[t] for t in sample_kept])
    final = rb(ref.rmsnorm(last, om.final_norm, om.eps))
    assert_close(rows(out, [row_of[t] for t in sample_kept]), final, BF16, "out sampled rows")


def test_long_context_gated_layer_128k():
    """N=131072 -> K=4096 (last 256 protected), one attention-only gated
    layer with Qwen3-1.7B heads: scorer + select + compact + gated attention."""
    w = synth.LONG_128K
    rng = synth.rng_for(w.seed)
    p = synth.model_params(w, rng)
    dev = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)  # noqa: E731
    lp = p["layers"][0]
    layer_d = {k: dev(v, BF16 if v.ndim == 2 else torch.float32) for k, v in lp.items()}
    score = {k: dev(p[k], BF16 if p[k].ndim == 2 else torch.float32)
             for k in ("score_norm", "score_w1", "score_b1", "score_w2", "score_b2")}
    model = tg.Model(n_heads_q=w.hq, n_heads_kv=w.hkv, head_dim=w.dh, layers=[layer_d],
                     score=score, final_norm=dev(p["final_norm"], torch.float32))
    g = lambda k: host64(layer_d[k]) if k in layer_d else None  # noqa: E731
    om = ref.Model(d_model=w.d, n_heads_q=w.hq, n_heads_kv=w.hkv, head_dim=w.dh,
                   layers=[ref.Layer(attn_norm=g("attn_norm"), wqkv=g("wqkv"), wo=g("wo"),
                                     ffn_norm=g("ffn_norm"), w_gate_up=None, w_down=None,
                                     gain=g("gain"), tau=g("tau"))],
                   final_norm=host64(model.final_norm),
                   score_norm=host64(score["score_norm"]), score_w1=host64(score["score_w1"]),
                   score_b1=host64(score["score_b1"]), score_w2=host64(score["score_w2"]),
                   score_b2=host64(score["score_b2"]))
    x = dev(synth.hidden_states(w, rng), BF16)
    prot = synth.protect_tail(w.n, w.n_protect)
    out, kept, scores, kv, _ = _run_gpu(w, model, x, prot)
    assert np.array_equal(kept, ref.topk_select(scores, prot, w.k))
    res = ref.prefill(host64(x), prot, w.k, om, -1, store=rb, kept_idx=kept,
                      fold_norms=model.fold_norms)
    assert_close(scores, res.scores, BF16, "scores")
    assert_close(kv[0][0], res.kv[0][0], BF16, "k")
    assert_close(kv[0][1], res.kv[0][1], BF16, "v")
    assert_close(out, res.out, BF16, "out")
