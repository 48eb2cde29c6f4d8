"""Shared test helpers: tolerances, host<->device conversion, and model
construction from the seeded synthetic parameters (the same values go to the
CUDA library and to the oracle)."""

from __future__ import annotations

import numpy as np
import torch

from oracle import tokengate_oracle as ref

# Parity tolerances: |gpu - ref| <= ATOL + RTOL * |ref| elementwise.
TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-4, 1e-4)}
STORE = {torch.bfloat16: ref.round_bf16, torch.float32: ref.round_fp32}


def dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float32))).to(
        device="cuda", dtype=dtype)


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(gpu, want, dtype, what=""):
    g = host64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    w = np.asarray(want, dtype=np.float64)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    atol, rtol = TOL[dtype]
    diff = np.abs(g - w)
    bad = ~(diff <= atol + rtol * np.abs(w))
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, diff, -1)), diff.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                             f"worst at {i}: gpu={g[i]!r} ref={w[i]!r}; max|d|={diff.max():.3e}")


def device_params(params: dict, dtype):
    """numpy float32 params -> device tensors: 2-D matrices in `dtype`, 1-D
    vectors (norm weights, biases, w2, gain, tau) in fp32."""
    out = {}
    for k, v in params.items():
        if isinstance(v, np.ndarray):
            out[k] = dev(v, dtype if v.ndim == 2 else torch.float32)
    return out


def build_models(w, rng, dtype, fold_norms=True):
    """(library Model, oracle Model) holding identical values."""
    import learned_token_pruning_score_b200 as tg
    import synth

    p = synth.model_params(w, rng)
    layers_d = [device_params(lp, dtype) for lp in p["layers"]]
    score_d = device_params({k: p[k] for k in ("score_norm", "score_w1", "score_b1", "score_w2",
                                               "score_b2")}, dtype)
    final_d = dev(p["final_norm"])
    m = tg.Model(n_heads_q=w.hq, n_heads_kv=w.hkv, head_dim=w.dh, layers=layers_d, score=score_d,
                 final_norm=final_d, eps=w.eps, rope_base=w.rope_base, fold_norms=fold_norms)
    o_layers = []
    for ld in layers_d:
        g = lambda k: host64(ld[k]) if k in ld else None  # noqa: E731
        o_layers.append(ref.Layer(attn_norm=g("attn_norm"), wqkv=g("wqkv"), wo=g("wo"),
                                  ffn_norm=g("ffn_norm"), w_gate_up=g("w_gate_up"),
                                  w_down=g("w_down"), q_norm=g("q_norm"), k_norm=g("k_norm"),
                                  gain=g("gain"), tau=g("tau")))
    om = ref.Model(d_model=w.d, n_heads_q=w.hq, n_heads_kv=w.hkv, head_dim=w.dh, layers=o_layers,
                   final_norm=host64(final_d), score_norm=host64(score_d["score_norm"]),
                   score_w1=host64(score_d["score_w1"]), score_b1=host64(score_d["score_b1"]),
                   score_w2=host64(score_d["score_w2"]), score_b2=host64(score_d["score_b2"]),
                   eps=w.eps, rope_base=w.rope_base)
    return m, om


def boundary_flips(oracle_scores32, gpu_kept, protect, k, atol, rtol):
    """Tokens where the oracle's own kept set differs from the GPU's, and
    whether every such token's score lies within tolerance of the K-th
    threshold (a near-tie that rounding may legitimately flip)."""
    own = set(ref.topk_select(oracle_scores32, protect, k).tolist())
    gpu = set(np.asarray(gpu_kept).tolist())
    diff = sorted(own ^ gpu)
    if not diff:
        return 0, True
    s = np.asarray(oracle_scores32, np.float64)
    kept_un = [i for i in own if not protect[i]]
    thr = min(s[kept_un]) if kept_un else np.inf
    near = all(abs(s[i] - thr) <= 2 * (atol + rtol * abs(thr)) for i in diff)
    return len(diff), near
