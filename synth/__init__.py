"""Seeded synthetic inputs for the gated-prefill workloads.

This module only draws random numbers (numpy PCG64 on the host, or a seeded
torch generator on the device for the multi-gigabyte weight sets). It holds
none of the method's arithmetic; the CUDA path and the oracle both consume
what it produces.

The pages measure on public task suites (code completion, multi-hop QA,
multi-document summarisation, medical extraction, needle-in-a-haystack) at
contexts of 16K-128K tokens with a protected question span at the end. None
of those datasets is used: these draws stand in for them, taking only their
scale and structure.
"""

from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Dict, List, Optional, Tuple

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str  # "f32" or "bf16"
    n: int  # tokens entering the gate
    k: int  # tokens kept
    d: int  # d_model
    hq: int
    hkv: int
    dh: int
    f: int  # scorer hidden width
    inter: int  # SwiGLU intermediate width (0 = attention sub-layer only)
    n_layers: int
    gate_layer: int  # -1: gate before layer 0 (every layer is an upper layer)
    n_protect: int  # protected tokens at the end of the prompt
    seed: int
    qk_norm: bool = False
    salient_frac: float = 0.0  # fraction of rows scaled by `salient_scale`
    salient_scale: float = 4.0
    rope_base: float = 1e6
    eps: float = 1e-6
    w_std: float = 0.02


# The five workloads. Sizes follow Qwen3-1.7B (d 2048, 16 query / 8 KV heads,
# head dim 128, SwiGLU 6144, 28 layers, RoPE base 1e6).
TINY_F32 = Workload("tiny_f32_gated_block", "f32", n=512, k=128, d=256, hq=4, hkv=2, dh=64,
                    f=64, inter=512, n_layers=1, gate_layer=-1, n_protect=16, seed=0)
QWEN_LAYER_16K = Workload("qwen3_1p7b_gated_layer_n16k_k2k", "bf16", n=16384, k=2048, d=2048,
                          hq=16, hkv=8, dh=128, f=256, inter=6144, n_layers=1, gate_layer=-1,
                          n_protect=64, seed=1, salient_frac=0.01)
SWEEP_D = 2048
SWEEP_N = (8192, 32768, 131072)
SWEEP_FRAC = (16, 8, 4, 2, 1)  # K = N / frac
SWEEP_PROTECT = 128
SWEEP_SEED = 2
QWEN_PREFILL_32K = Workload("qwen3_1p7b_prefill_n32k", "bf16", n=32768, k=4096, d=2048, hq=16,
                            hkv=8, dh=128, f=256, inter=6144, n_layers=28, gate_layer=1,
                            n_protect=128, seed=3, qk_norm=True)
PREFILL_32K_BUDGETS = (2048, 4096, 8192)
LONG_128K = Workload("long_context_gated_attn_n128k_k4k", "bf16", n=131072, k=4096, d=2048,
                     hq=16, hkv=8, dh=128, f=256, inter=0, n_layers=1, gate_layer=-1,
                     n_protect=256, seed=4)

WORKLOADS: Dict[str, Workload] = {w.name: w for w in (TINY_F32, QWEN_LAYER_16K,
                                                      QWEN_PREFILL_32K, LONG_128K)}


def shrink(w: Workload, **kw) -> Workload:
    """A smaller copy of a workload (same structure, other sizes)."""
    return replace(w, **kw)


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def hidden_states(w: Workload, rng: np.random.Generator) -> np.ndarray:
    """[n, d] float32 ~ N(0, 1); a `salient_frac` share of rows (chosen
    uniformly without replacement) is multiplied by `salient_scale`."""
    x = rng.standard_normal((w.n, w.d), dtype=np.float32)
    if w.salient_frac > 0:
        m = max(1, int(round(w.salient_frac * w.n)))
        rows = rng.choice(w.n, size=m, replace=False)
        x[rows] *= np.float32(w.salient_scale)
    return x


def protect_tail(n: int, p: int) -> np.ndarray:
    """uint8 mask with the last p tokens protected (the question span)."""
    m = np.zeros(n, dtype=np.uint8)
    if p > 0:
        m[n - p:] = 1
    return m


def layer_params(w: Workload, rng: np.random.Generator, upper: bool) -> Dict[str, np.ndarray]:
    """One layer's parameters as float32 arrays (weights N(0, w_std), norms 1,
    gain U(0, 2), tau U(0.5, 1.5) for an upper layer)."""
    s = np.float32(w.w_std)
    qkv_rows = (w.hq + 2 * w.hkv) * w.dh
    p = {
        "attn_norm": np.ones(w.d, np.float32),
        "wqkv": rng.standard_normal((qkv_rows, w.d), dtype=np.float32) * s,
        "wo": rng.standard_normal((w.d, w.hq * w.dh), dtype=np.float32) * s,
        "ffn_norm": np.ones(w.d, np.float32),
    }
    if w.inter > 0:
        p["w_gate_up"] = rng.standard_normal((2 * w.inter, w.d), dtype=np.float32) * s
        p["w_down"] = rng.standard_normal((w.d, w.inter), dtype=np.float32) * s
    if w.qk_norm:
        p["q_norm"] = np.ones(w.dh, np.float32)
        p["k_norm"] = np.ones(w.dh, np.float32)
    if upper:
        p["gain"] = rng.uniform(0.0, 2.0, w.hq).astype(np.float32)
        p["tau"] = rng.uniform(0.5, 1.5, w.hq).astype(np.float32)
    return p


def scorer_params(w: Workload, rng: np.random.Generator) -> Dict[str, np.ndarray]:
    s = np.float32(w.w_std)
    return {
        "score_norm": np.ones(w.d, np.float32),
        "score_w1": rng.standard_normal((w.f, w.d), dtype=np.float32) * s,
        "score_b1": np.zeros(w.f, np.float32),
        "score_w2": rng.standard_normal(w.f, dtype=np.float32) * s,
        "score_b2": np.zeros(1, np.float32),
    }


def model_params(w: Workload, rng: np.random.Generator) -> Dict[str, object]:
    layers = [layer_params(w, rng, upper=(li > w.gate_layer)) for li in range(w.n_layers)]
    out: Dict[str, object] = {"layers": layers, "final_norm": np.ones(w.d, np.float32)}
    out.update(scorer_params(w, rng))
    return out


def sweep_scores(n: int, rng: np.random.Generator, tie_block: int = 64,
                 tie_frac: float = 0.10, n_specials: int = 8) -> np.ndarray:
    """fp32 N(0,1) scores; about `tie_frac` of the `tie_block`-token blocks are
    overwritten by one repeated value, and a few entries become +-0 and
    +-inf."""
    s = rng.standard_normal(n, dtype=np.float32)
    nb = n // tie_block
    if nb > 0:
        blocks = rng.choice(nb, size=max(1, int(tie_frac * nb)), replace=False)
        for b in blocks:
            s[b * tie_block:(b + 1) * tie_block] = np.float32(rng.standard_normal())
    specials = np.array([0.0, -0.0, np.inf, -np.inf], dtype=np.float32)
    pos = rng.choice(n, size=min(n, n_specials), replace=False)
    s[pos] = specials[np.arange(pos.size) % 4]
    return s


def scores_threshold_in_tie(n: int, k: int, p: int, rng: np.random.Generator,
                            tie_len: int = 64, cut: int = 20) -> np.ndarray:
    """Scores built so that the K-th kept unprotected token falls inside a tie
    block: exactly k - p - cut unprotected tokens score in [1, 2), one block
    of `tie_len` unprotected tokens scores exactly 0.5, the rest score in
    [-2, 0.4). Protected tokens (the last p) score in [-2, 0.4) too."""
    assert k - p - cut >= 0 and n - p >= k - p - cut + tie_len
    s = rng.uniform(-2.0, 0.4, n).astype(np.float32)
    unprot = n - p
    start = int(rng.integers(0, unprot - tie_len + 1))
    tie = np.arange(start, start + tie_len)
    s[tie] = np.float32(0.5)
    rest = np.setdiff1d(np.arange(unprot), tie)
    high = rng.choice(rest, size=k - p - cut, replace=False)
    s[high] = rng.uniform(1.0, 2.0, high.size).astype(np.float32)
    return s


def sweep_points() -> List[Tuple[int, int]]:
    return [(n, n // f) for n in SWEEP_N for f in SWEEP_FRAC]


def torch_model_params(w: Workload, seed: int, device: str = "cuda"):
    """Device-side draws of a full model for sizes whose host generation
    would take minutes (28 layers of d 2048). Same distributions as
    `model_params`; values come from a seeded torch generator on `device`,
    already in the model dtype."""
    import torch

    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    g = torch.Generator(device=device)
    g.manual_seed(seed)

    def normal(*shape):
        t = torch.empty(*shape, device=device, dtype=torch.float32)
        t.normal_(0.0, w.w_std, generator=g)
        return t.to(dt)

    def ones(n):
        return torch.ones(n, device=device, dtype=torch.float32)

    def unif(n, lo, hi):
        t = torch.empty(n, device=device, dtype=torch.float32)
        return t.uniform_(lo, hi, generator=g)

    layers = []
    for li in range(w.n_layers):
        p = {"attn_norm": ones(w.d), "wqkv": normal((w.hq + 2 * w.hkv) * w.dh, w.d),
             "wo": normal(w.d, w.hq * w.dh), "ffn_norm": ones(w.d)}
        if w.inter > 0:
            p["w_gate_up"] = normal(2 * w.inter, w.d)
            p["w_down"] = normal(w.d, w.inter)
        if w.qk_norm:
            p["q_norm"] = ones(w.dh)
            p["k_norm"] = ones(w.dh)
        if li > w.gate_layer:
            p["gain"] = unif(w.hq, 0.0, 2.0)
            p["tau"] = unif(w.hq, 0.5, 1.5)
        layers.append(p)
    out = {"layers": layers, "final_norm": ones(w.d), "score_norm": ones(w.d),
           "score_w1": normal(w.f, w.d), "score_b1": torch.zeros(w.f, device=device),
           "score_w2": normal(w.f).float(), "score_b2": torch.zeros(1, device=device)}
    return out


def torch_hidden_states(w: Workload, seed: int, device: str = "cuda"):
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.empty(w.n, w.d, device=device, dtype=torch.float32)
    x.normal_(0.0, 1.0, generator=g)
    if w.salient_frac > 0:
        m = max(1, int(round(w.salient_frac * w.n)))
        rows = torch.randperm(w.n, generator=g, device=device)[:m]
        x[rows] *= w.salient_scale
    return x.to(torch.bfloat16 if w.dtype == "bf16" else torch.float32)


def decode_state(w: Workload, rng: np.random.Generator, generated: int = 0) -> Dict[str, object]:
    """Inputs of one decode step after a prefill of w.n tokens that kept w.k,
    with `generated` tokens decoded since: per-layer caches of N(0, 1)
    float32 keys and values (w.n + generated rows at or below the gate,
    w.k + generated above), gate scores [w.n] ~ N(0, 2^2), an ascending kept
    set of w.k tokens that holds the protected tail, the new token's hidden
    state [d] ~ N(0, 1), and its position w.n + generated."""
    lens = [(w.n if li <= w.gate_layer else w.k) + generated for li in range(w.n_layers)]
    caches = [(rng.standard_normal((t, w.hkv, w.dh), dtype=np.float32),
               rng.standard_normal((t, w.hkv, w.dh), dtype=np.float32)) for t in lens]
    scores = (rng.standard_normal(w.n) * 2.0).astype(np.float32)
    tail = np.arange(w.n - w.n_protect, w.n)
    rest = rng.choice(w.n - w.n_protect, size=w.k - w.n_protect, replace=False)
    kept = np.sort(np.concatenate([rest, tail])).astype(np.int32)
    x = rng.standard_normal(w.d, dtype=np.float32)
    return {"lens": lens, "caches": caches, "scores": scores, "kept_idx": kept, "x": x,
            "pos": w.n + generated}


# ---------------------------------------------------------------- hybrid models
@dataclass(frozen=True)
class GdnWorkload:
    """A Gated DeltaNet layer's token mixer over T tokens (the kept tokens of
    a gated prefill; n is what the same layer sees without the gate)."""
    name: str
    dtype: str
    T: int
    n: int
    hk: int
    hv: int
    dk: int
    dv: int
    W: int
    seed: int
    eps: float = 1e-6


# Linear-attention layer of a hybrid model at d_model 2048 (Qwen3-Next-style
# shape: 16 key and 16 value heads of dim 128, convolution width 4); the
# pages give the hybrid model's name but not its sizes. K = 4096 of N = 32768.
GDN_LAYER_32K = GdnWorkload("hybrid_gdn_mixer_n32k_k4k", "bf16", T=4096, n=32768, hk=16, hv=16,
                            dk=128, dv=128, W=4, seed=5)


def gdn_params(w: GdnWorkload, rng: np.random.Generator) -> Dict[str, np.ndarray]:
    """float32 mixer parameters: conv_w [C, W] ~ U(+-1/sqrt(W)); A_log =
    log U(1, 16); dt_bias ~ U(-7, -2); norm_w ~ 1 + 0.1 N(0, 1)."""
    C = 2 * w.hk * w.dk + w.hv * w.dv
    lim = 1.0 / np.sqrt(w.W)
    return {
        "conv_w": rng.uniform(-lim, lim, (C, w.W)).astype(np.float32),
        "A_log": np.log(rng.uniform(1.0, 16.0, w.hv)).astype(np.float32),
        "dt_bias": rng.uniform(-7.0, -2.0, w.hv).astype(np.float32),
        "norm_w": (1.0 + 0.1 * rng.standard_normal(w.dv)).astype(np.float32),
    }


def gdn_inputs(w: GdnWorkload, rng: np.random.Generator, T: Optional[int] = None
               ) -> Dict[str, np.ndarray]:
    """float32 projection outputs for T tokens (default w.T): qkv [T, C],
    z [T, hv dv], a and b [T, hv], all ~ N(0, 1)."""
    T = w.T if T is None else T
    C = 2 * w.hk * w.dk + w.hv * w.dv
    return {
        "qkv": rng.standard_normal((T, C), dtype=np.float32),
        "z": rng.standard_normal((T, w.hv * w.dv), dtype=np.float32),
        "a": rng.standard_normal((T, w.hv), dtype=np.float32),
        "b": rng.standard_normal((T, w.hv), dtype=np.float32),
    }


@dataclass(frozen=True)
class HybridWorkload:
    """A hybrid decoder stack: `kinds` gives each layer's token mixer
    ("gdn": Gated DeltaNet, "attn": full attention); the attention layers
    use `base`'s heads and every layer `base`'s FFN; the Gated DeltaNet
    layers have hk / hv heads of dim dk / dv and convolution width W."""
    base: Workload
    kinds: Tuple[str, ...]
    hk: int
    hv: int
    dk: int
    dv: int
    W: int


# Qwen3.5-2B-like hybrid stack: three Gated DeltaNet layers to one
# full-attention layer, d_model 2048 (the pages name the model and its gate
# positions, layers 1 to 3, but not its sizes; the Qwen3-Next-style mixer
# shape and Qwen3-1.7B-style attention heads stand in). N = 4096, K = 1024.
HYBRID_4K = HybridWorkload(
    Workload("hybrid_qwen35_like_n4k_k1k", "bf16", n=4096, k=1024, d=2048, hq=16, hkv=8, dh=128,
             f=256, inter=6144, n_layers=8, gate_layer=1, n_protect=64, seed=6, qk_norm=True),
    kinds=("gdn", "gdn", "gdn", "attn", "gdn", "gdn", "gdn", "attn"),
    hk=16, hv=16, dk=128, dv=128, W=4)


def torch_hybrid_params(w: HybridWorkload, seed: int, device: str = "cuda"):
    """Device-side draws of a hybrid stack, like `torch_model_params`: the
    attention layers as there; a Gated DeltaNet layer has attn_norm (the
    norm before the mixer) = 1, w_in [C + hv dv + 2 hv, d] and w_out
    [d, hv dv] ~ N(0, w_std), and fp32 mixer parameters conv_w [C, W] ~
    U(+-1/sqrt(W)), A_log = log U(1, 16), dt_bias ~ U(-7, -2) and norm_w ~
    1 + 0.1 N(0, 1) (C = 2 hk dk + hv dv)."""
    import math

    import torch

    b = w.base
    p = torch_model_params(b, seed, device)
    g = torch.Generator(device=device)
    g.manual_seed(seed + 7919)
    dt = torch.bfloat16 if b.dtype == "bf16" else torch.float32
    C = 2 * w.hk * w.dk + w.hv * w.dv

    def normal(*shape, std=b.w_std):
        t = torch.empty(*shape, device=device, dtype=torch.float32)
        return t.normal_(0.0, std, generator=g)

    def unif(shape, lo, hi):
        t = torch.empty(*shape, device=device, dtype=torch.float32)
        return t.uniform_(lo, hi, generator=g)

    for li, kind in enumerate(w.kinds):
        if kind != "gdn":
            continue
        lp = p["layers"][li]
        for key in ("wqkv", "wo", "q_norm", "k_norm", "gain", "tau"):
            lp.pop(key, None)
        lp["w_in"] = normal(C + w.hv * w.dv + 2 * w.hv, b.d).to(dt)
        lp["w_out"] = normal(b.d, w.hv * w.dv).to(dt)
        lim = 1.0 / math.sqrt(w.W)
        lp["gdn_params"] = {"conv_w": unif((C, w.W), -lim, lim),
                            "A_log": torch.log(unif((w.hv,), 1.0, 16.0)),
                            "dt_bias": unif((w.hv,), -7.0, -2.0),
                            "norm_w": 1.0 + 0.1 * normal(w.dv, std=1.0)}
    return p
