"""GPU parity of the decode step over the pruned cache (tg_decode_step)
against the oracle's decode_step, on seeded synthetic caches that both
sides consume (no GPU output feeds the oracle).

Tolerance |d| <= 2e-2 + 1e-2 |ref| on the bf16 output and on the k/v rows the
step appends to every layer's cache.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import tokengate_oracle as ref
from tests._helpers import assert_close, build_models, dev, host64

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")


@pytest.fixture(autouse=True)
def _no_device_errors():
    tg.tg_device_error(clear=True)
    yield
    assert tg.tg_device_error() == 0


def _run(w, seed, generated=0, bias=True, extra_rows=1):
    rng = synth.rng_for(seed)
    model, om = build_models(w, rng, torch.bfloat16)
    st = synth.decode_state(w, rng, generated)
    kv, cache_o = [], []
    for (k, v), t in zip(st["caches"], st["lens"]):
        kc = torch.zeros(t + extra_rows, w.hkv, w.dh, dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        kc[:t] = dev(k, torch.bfloat16)
        vc[:t] = dev(v, torch.bfloat16)
        kv.append((kc, vc))
        cache_o.append((host64(kc[:t]), host64(vc[:t])))
    x = dev(st["x"], torch.bfloat16)
    scores = torch.from_numpy(st["scores"]).cuda() if bias else None
    kept = torch.from_numpy(st["kept_idx"]).cuda() if bias else None
    out = tg.tg_decode_step(model, x, st["pos"], w.gate_layer, kv, st["lens"], scores=scores,
                            kept_idx=kept)
    torch.cuda.synchronize()
    kept_scores = st["scores"][st["kept_idx"]].astype(np.float64) if bias else None
    if not bias:
        kept_scores = np.full(max(w.k, 1), np.inf)  # logsigmoid(inf) = 0: no bias
    want, new_kv = ref.decode_step(host64(x), st["pos"], om, w.gate_layer, cache_o, kept_scores)
    assert_close(out[0], want, torch.bfloat16, "decode out")
    for li, ((kc, vc), t, (kn, vn)) in enumerate(zip(kv, st["lens"], new_kv)):
        assert_close(kc[t], kn, torch.bfloat16, f"layer {li} appended k")
        assert_close(vc[t], vn, torch.bfloat16, f"layer {li} appended v")
        # rows before the new one are untouched, the row after it too
        assert torch.equal(kc[:t], dev(st["caches"][li][0], torch.bfloat16))
        if extra_rows > 1:
            assert torch.count_nonzero(kc[t + 1:]) == 0


SMALL = synth.Workload("decode_small", "bf16", n=300, k=100, d=256, hq=4, hkv=2, dh=128, f=64,
                       inter=512, n_layers=3, gate_layer=0, n_protect=16, seed=0, qk_norm=True)


@pytest.mark.parametrize("gate_layer", [-1, 0, 1, 2])
def test_decode_small_gate_positions(gate_layer):
    _run(synth.shrink(SMALL, gate_layer=gate_layer), 10 + gate_layer, generated=3)


def test_decode_no_qk_norm_mha_and_wide_gqa():
    _run(synth.shrink(SMALL, qk_norm=False), 21)
    _run(synth.shrink(SMALL, hq=2, hkv=2), 22)          # group of 1
    _run(synth.shrink(SMALL, hq=8, hkv=1, d=512), 23)   # group of 8


def test_decode_without_gate_bias():
    _run(SMALL, 24, bias=False)


def test_decode_ragged_and_tiny_caches():
    # caches of 1..few rows, lengths not a multiple of any split or vector size
    _run(synth.shrink(SMALL, n=17, k=5, n_protect=2, gate_layer=0), 25, generated=0)
    _run(synth.shrink(SMALL, n=1, k=1, n_protect=1, gate_layer=-1), 26, generated=0)
    _run(synth.shrink(SMALL, n=1000, k=333, n_protect=16), 27, generated=7, extra_rows=4)


def test_decode_no_ffn_layers():
    _run(synth.shrink(SMALL, inter=0), 28)


def test_decode_qwen_shapes_dense_and_gated_caches():
    """Qwen3-1.7B widths (d 2048, 16/8 x 128, SwiGLU 6144), the gate at layer
    0: a 32768-row dense cache below, 4096-row gated caches above."""
    w = synth.shrink(synth.QWEN_PREFILL_32K, n_layers=3, gate_layer=0)
    _run(w, 29, generated=5)


def test_decode_matches_one_more_token_of_prefill_on_gpu():
    """GPU against GPU: a dense prefill of N tokens followed by decoding token
    N gives (within bf16 tolerance) token N's row of a dense prefill of N + 1
    tokens, and the same cache rows."""
    w = synth.shrink(SMALL, n=257, k=257, n_protect=8, gate_layer=2)  # every layer at/below the gate
    rng = synth.rng_for(30)
    model, _ = build_models(w, rng, torch.bfloat16)
    x = dev(rng.standard_normal((w.n + 1, w.d)), torch.bfloat16)
    prot = torch.from_numpy(synth.protect_tail(w.n, w.n_protect)).cuda()
    kv = [(torch.zeros(w.n + 1, w.hkv, w.dh, dtype=torch.bfloat16, device="cuda"),
           torch.zeros(w.n + 1, w.hkv, w.dh, dtype=torch.bfloat16, device="cuda"))
          for _ in range(w.n_layers)]
    tg.tg_prefill(model, x[:w.n], prot, w.n, w.gate_layer, kv=kv)
    out = tg.tg_decode_step(model, x[w.n], w.n, w.gate_layer, kv, [w.n] * w.n_layers)
    prot1 = torch.from_numpy(synth.protect_tail(w.n + 1, w.n_protect)).cuda()
    kv1 = [(torch.empty_like(a), torch.empty_like(b)) for a, b in kv]
    full, _, _ = tg.tg_prefill(model, x, prot1, w.n + 1, w.gate_layer, kv=kv1)
    torch.cuda.synchronize()
    assert_close(out[0], host64(full[-1]), torch.bfloat16, "decode vs prefill(N+1)")
    for (kc, vc), (k1, v1) in zip(kv, kv1):
        assert_close(kc[w.n], host64(k1[w.n]), torch.bfloat16, "k row")
        assert_close(vc[w.n], host64(v1[w.n]), torch.bfloat16, "v row")
