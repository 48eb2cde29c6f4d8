"""GPU parity of the full gated prefill (tg_prefill) against the oracle.

The oracle is teacher-forced with the GPU's kept set, so a near-tie at the
K-th score cannot cascade; the kept set itself is checked bit-exactly as
oracle_select(gpu_scores) == gpu_kept, and the oracle's own-score kept set
may differ only at near-threshold tokens (zero differences allowed in fp32).
"""

import numpy as np
import pytest
import torch

import synth
from oracle import tokengate_oracle as ref
from tests._helpers import STORE, TOL, assert_close, boundary_flips, build_models, host64

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")

DT = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(autouse=True)
def _no_device_errors():
    tg.tg_device_error(clear=True)
    yield
    assert tg.tg_device_error() == 0


def _run(w, want_kv=True, seed=None, fold_norms=True):
    dtype = DT[w.dtype]
    rng = synth.rng_for(w.seed if seed is None else seed)
    model, om = build_models(w, rng, dtype, fold_norms)
    x_np = synth.hidden_states(w, rng)
    x = torch.from_numpy(x_np).to("cuda", dtype)
    prot_np = synth.protect_tail(w.n, w.n_protect)
    prot = torch.from_numpy(prot_np).cuda()
    scores = torch.empty(w.n, device="cuda")
    kv = None
    if want_kv:
        kv = []
        for li in range(w.n_layers):
            rows = w.n if li <= w.gate_layer else w.k
            kv.append((torch.empty(rows, w.hkv, w.dh, device="cuda", dtype=dtype),
                       torch.empty(rows, w.hkv, w.dh, device="cuda", dtype=dtype)))
    out, kept, _ = tg.tg_prefill(model, x, prot, w.k, w.gate_layer, scores=scores, kv=kv)
    torch.cuda.synchronize()
    return dict(model=model, om=om, x=x, prot=prot_np, out=out, kept=kept.cpu().numpy(),
                scores=scores.cpu().numpy(), kv=kv, dtype=dtype)


def _check_against_oracle(w, r):
    dtype = r["dtype"]
    # 1. the kept set is the exact selection of the GPU's own scores
    assert np.array_equal(r["kept"], ref.topk_select(r["scores"], r["prot"], w.k))
    # 2. teacher-forced oracle run
    res = ref.prefill(host64(r["x"]), r["prot"], w.k, r["om"], w.gate_layer,
                      store=STORE[dtype], kept_idx=r["kept"], fold_norms=r["model"].fold_norms)
    assert_close(r["scores"], res.scores, dtype, "scores")
    assert_close(r["out"], res.out, dtype, "out")
    if r["kv"] is not None:
        for li, ((kg, vg), (ko, vo)) in enumerate(zip(r["kv"], res.kv)):
            assert kg.shape[0] == ko.shape[0]
            assert_close(kg, ko, dtype, f"k cache layer {li}")
            assert_close(vg, vo, dtype, f"v cache layer {li}")
    # 3. the oracle's own-score selection differs only at near-ties
    atol, rtol = TOL[dtype]
    flips, near = boundary_flips(res.scores, r["kept"], r["prot"], w.k, atol, rtol)
    assert near, f"{flips} kept-set differences away from the threshold"
    if dtype == torch.float32:
        assert flips == 0
    return res


def test_tiny_fp32_gated_block():
    """The tiny fp32 gated block: N 512, d 256, 4/2 heads of 64, K 128, the
    last 16 tokens protected; checked to 1e-4."""
    _check_against_oracle(synth.TINY_F32, _run(synth.TINY_F32))


@pytest.mark.parametrize("fold_norms", [True, False])
@pytest.mark.parametrize("qk_norm", [False, True])
@pytest.mark.parametrize("gate_layer", [-1, 0, 1])
def test_small_bf16_stack(qk_norm, gate_layer, fold_norms):
    """fold_norms: the RMSNorms after a residual GEMM folded into the next
    projection (its weight times the norm weight, its accumulator rows over
    the rms), or the norm kernel before every projection."""
    w = synth.shrink(synth.QWEN_LAYER_16K, name="small", n=300, k=100, d=256, hq=4, hkv=2, dh=128,
                     f=64, inter=256, n_layers=3, gate_layer=gate_layer, n_protect=10,
                     qk_norm=qk_norm, seed=40 + gate_layer, salient_frac=0.02)
    _check_against_oracle(w, _run(w, fold_norms=fold_norms))


@pytest.mark.parametrize("rows,cols", [(3, 8), (17, 2048), (5, 13), (1, 1)])
def test_fold_norm_weight_is_exact(rows, cols):
    """W_g = bf16(W . diag(g)): one product and one round-to-nearest-even per
    element (the vector path for cols % 8 == 0, the scalar one otherwise)."""
    gen = torch.Generator(device="cuda").manual_seed(rows * 1000 + cols)
    w = (torch.randn(rows, cols, device="cuda", generator=gen) * 3).to(torch.bfloat16)
    g = torch.rand(cols, device="cuda", generator=gen) * 2 - 0.5
    out = tg.tg_fold_norm_weight(w, g)
    torch.cuda.synchronize()
    assert torch.equal(out, (w.float() * g).to(torch.bfloat16))


def test_small_fp32_stack():
    w = synth.shrink(synth.TINY_F32, name="small32", n=200, k=64, n_layers=3, gate_layer=1,
                     n_protect=8, qk_norm=True, seed=77)
    _check_against_oracle(w, _run(w))


def test_gated_equals_dense_when_all_kept():
    """K = N with gain 0 and tau 1 above the gate is the dense prefill: on the
    GPU the two runs use the same kernels and agree bit for bit."""
    w = synth.shrink(synth.QWEN_LAYER_16K, name="dense_eq", n=256, k=256, d=256, hq=4, hkv=2,
                     dh=128, f=64, inter=256, n_layers=3, gate_layer=0, n_protect=4, seed=5)
    rng = synth.rng_for(w.seed)
    model, _ = build_models(w, rng, torch.bfloat16)
    for lw in model.layers:
        lw.pop("gain", None)
        lw.pop("tau", None)
    model = tg.Model(n_heads_q=w.hq, n_heads_kv=w.hkv, head_dim=w.dh, layers=model.layers,
                     score=model.score, final_norm=model.final_norm)
    x = torch.randn(w.n, w.d, device="cuda", dtype=torch.bfloat16)
    out_g, kept, _ = tg.tg_prefill(model, x, None, w.n, 0)
    out_d, _, _ = tg.tg_prefill(model, x, None, w.n, w.n_layers - 1)
    torch.cuda.synchronize()
    assert np.array_equal(kept.cpu().numpy(), np.arange(w.n))
    assert torch.equal(out_g, out_d)


@pytest.mark.parametrize("n", [16684, 700])
def test_prefill_from_host_memory_equals_device_input(n):
    """tg_prefill_host (x in pinned host memory) gives tg_prefill's results
    bit for bit: above 8192 rows the copy is chunked and layer 0's norm, QKV
    projection and attention run per chunk as the rows land (n = 16684: four
    whole 4096-row chunks and a ragged one); below, one copy then the same
    path."""
    w = synth.shrink(synth.QWEN_LAYER_16K, name="host_in", n=n, k=n // 5, d=256, hq=4, hkv=2,
                     dh=128, f=64, inter=256, n_layers=3, gate_layer=1, n_protect=16, seed=81,
                     qk_norm=True)
    rng = synth.rng_for(w.seed)
    model, _ = build_models(w, rng, torch.bfloat16)
    x = torch.from_numpy(synth.hidden_states(w, rng)).to("cuda", torch.bfloat16)
    prot = torch.from_numpy(synth.protect_tail(w.n, w.n_protect)).cuda()

    def kvs():
        return [(torch.zeros(w.n if li <= w.gate_layer else w.k, w.hkv, w.dh, device="cuda",
                             dtype=torch.bfloat16),
                 torch.zeros(w.n if li <= w.gate_layer else w.k, w.hkv, w.dh, device="cuda",
                             dtype=torch.bfloat16)) for li in range(w.n_layers)]
    kv_d, kv_h = kvs(), kvs()
    sc_d = torch.empty(w.n, device="cuda")
    sc_h = torch.empty(w.n, device="cuda")
    out_d, kept_d, _ = tg.tg_prefill(model, x, prot, w.k, w.gate_layer, scores=sc_d, kv=kv_d)
    x_host = x.cpu().pin_memory()
    out_h, kept_h, _ = tg.tg_prefill_host(model, x_host, prot, w.k, w.gate_layer, scores=sc_h,
                                          kv=kv_h)
    torch.cuda.synchronize()
    assert torch.equal(kept_h, kept_d)
    assert torch.equal(sc_h, sc_d)
    assert torch.equal(out_h, out_d)
    for (kd, vd), (kh, vh) in zip(kv_d, kv_h):
        assert torch.equal(kh, kd) and torch.equal(vh, vd)


def test_pruned_tokens_make_no_upper_kv():
    w = synth.shrink(synth.QWEN_LAYER_16K, name="kvrows", n=300, k=60, d=256, hq=4, hkv=2, dh=128,
                     f=64, inter=256, n_layers=3, gate_layer=0, n_protect=6, seed=9)
    r = _run(w)
    assert [kv[0].shape[0] for kv in r["kv"]] == [300, 60, 60]
    # upper KV rows are exactly the kept tokens' (teacher-forced) projections
    _check_against_oracle(w, r)


@pytest.mark.slow
def test_qwen_gated_layer_16k():
    """One Qwen3-1.7B-shaped gated layer: N 16384 -> K 2048, d 2048, 16/8 heads
    of 128, scorer 2048->256->1, SwiGLU 6144, last 64 protected, 1% salient."""
    _check_against_oracle(synth.QWEN_LAYER_16K, _run(synth.QWEN_LAYER_16K))
