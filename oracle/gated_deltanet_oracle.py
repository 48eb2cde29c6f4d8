"""Gated DeltaNet mixer over the kept tokens -- the oracle.

TEST INFRASTRUCTURE. A plain, slow, obviously correct float64 (numpy)
restatement of the token mixer that hybrid models run in their linear
layers. Only the test suite, the package's smoke check and the benchmark's
CPU baseline leg may import it; the CUDA library never calls it and shares no
code, table or constant with it.

Source: Tencent Cloud developer article "TokenGate：端到端可训练的 Token 剪枝机制，
让大模型 Prefill 提速 11.3 倍" [TC], section "门控位置影响剪枝效果" (with its
figure 5). In the hybrid Qwen3.5-2B most layers are Gated DeltaNet layers and
only some are full attention. The scorer reads hidden states, so the gate may
sit at a Gated DeltaNet layer. The token-gated logit bias applies only in the
full-attention layers above the gate; a Gated DeltaNet layer above the gate
has no logits and simply runs on the kept tokens.

The pages name the layer type but do not define it. Its computation is the
published gated delta rule (Yang, Kautz and Hatamizadeh, "Gated Delta
Networks: Improving Mamba2 with Delta Rule", ICLR 2025), in the layer shape
of the Qwen3-Next / Qwen3.5 family. Readings (listed with the others in the
design notes):

  G1  The kept tokens, in ascending original order, are the layer's input
      sequence. The short convolution and the recurrence run over that
      sequence; a pruned token leaves no trace in either.
  G2  Mixer inputs are the outputs of the layer's input projections, per
      token: qkv = [q (hk*dk) | k (hk*dk) | v (hv*dv)] before the
      convolution, the output gate z (hv*dv), and the decay and write-strength
      inputs a, b (hv each).
  G3  Short convolution: causal, depthwise, width W over the qkv channels,
      followed by SiLU. Rows before the first token come from a carried conv
      state (the last W-1 input rows of the previous call), else are zero.
  G4  q and k are L2-normalised per head, x / sqrt(sum x^2 + 1e-6); q is then
      scaled by dk^-1/2.
  G5  Per token and value head: g = -exp(A_log) * softplus(a + dt_bias),
      alpha = exp(g) in (0, 1]; beta = sigmoid(b).
  G6  Value head h reads key head floor(h / (hv / hk)).
  G7  State S (dv x dk per value head), starting from a carried state or
      zero:  S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
      output o_t = S_t q_t.
  G8  Output: y = RMSNorm(o) * w * SiLU(z) per value head (RMS over dv),
      stored in the call's dtype. The final S is returned in fp32.
  G9  Rounding points: the inputs as given, the stored output y (dtype) and
      the returned states (conv state in the input dtype, S in fp32).
      Everything between is float64 here.
  G10, G11  A Gated DeltaNet layer of a stack, and the gated forward of a
      hybrid stack (below, with hybrid_prefill).

G2-G8 agree with the Qwen3.5 Gated DeltaNet layer in the transformers
library; the pins check the two against each other on the same weights.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np

from .tokengate_oracle import round_fp32, sigmoid, silu

F64 = np.float64
L2_EPS = 1e-6


# ---------------------------------------------------------------------------
# G3: the short causal convolution
# ---------------------------------------------------------------------------
def causal_conv_silu(x, w, conv_state=None) -> Tuple[np.ndarray, np.ndarray]:
    """y[t, c] = SiLU(sum_{i<W} w[c, i] * xx[t + i, c]) where xx is x with the
    W-1 carried rows (or zeros) in front; also returns xx's last W-1 rows.

    x [T, C], w [C, W], conv_state [W-1, C] or None."""
    x = np.asarray(x, dtype=F64)
    w = np.asarray(w, dtype=F64)
    T, C = x.shape
    W = w.shape[1]
    prev = np.zeros((W - 1, C)) if conv_state is None else np.asarray(conv_state, dtype=F64)
    xx = np.concatenate([prev, x], axis=0)
    y = np.zeros((T, C))
    for t in range(T):
        for i in range(W):
            y[t] += w[:, i] * xx[t + i]
    return silu(y), xx[T:].copy()


# ---------------------------------------------------------------------------
# G4, G5: normalisation, decay and write strength
# ---------------------------------------------------------------------------
def l2_normalize(x, eps: float = L2_EPS) -> np.ndarray:
    """x / sqrt(sum x^2 + eps) over the last axis."""
    x = np.asarray(x, dtype=F64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def softplus(x) -> np.ndarray:
    """log(1 + exp(x)), stable for large |x|."""
    x = np.asarray(x, dtype=F64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def decay_and_strength(a, b, A_log, dt_bias) -> Tuple[np.ndarray, np.ndarray]:
    """(g, beta): g = -exp(A_log) softplus(a + dt_bias) (log of the decay
    alpha), beta = sigmoid(b). a, b [T, hv]; A_log, dt_bias [hv]."""
    g = -np.exp(np.asarray(A_log, dtype=F64)) * softplus(np.asarray(a, dtype=F64) +
                                                          np.asarray(dt_bias, dtype=F64))
    return g, sigmoid(b)


# ---------------------------------------------------------------------------
# G7: the gated delta rule
# ---------------------------------------------------------------------------
def gated_delta_rule(q, k, v, g, beta, S0=None) -> Tuple[np.ndarray, np.ndarray]:
    """Token-by-token recurrence of G7, per value head.

    q, k [T, H, dk] (already mapped to value heads), v [T, H, dv], g, beta
    [T, H], S0 [H, dv, dk] or None. Returns o [T, H, dv] and S_T."""
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    v = np.asarray(v, dtype=F64)
    T, H, dk = k.shape
    dv = v.shape[2]
    S = np.zeros((H, dv, dk)) if S0 is None else np.array(S0, dtype=F64)
    alpha = np.exp(np.asarray(g, dtype=F64))
    beta = np.asarray(beta, dtype=F64)
    eye = np.eye(dk)
    o = np.zeros((T, H, dv))
    for t in range(T):
        for h in range(H):
            kt = k[t, h]
            S[h] = alpha[t, h] * S[h] @ (eye - beta[t, h] * np.outer(kt, kt)) \
                + beta[t, h] * np.outer(v[t, h], kt)
            o[t, h] = S[h] @ q[t, h]
    return o, S


# ---------------------------------------------------------------------------
# G8: the gated output norm
# ---------------------------------------------------------------------------
def gated_rmsnorm(o, z, w, eps) -> np.ndarray:
    """RMSNorm(o) * w * SiLU(z) over the last axis."""
    o = np.asarray(o, dtype=F64)
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o * r * np.asarray(w, dtype=F64) * silu(z)


# ---------------------------------------------------------------------------
# The whole mixer (G1-G9)
# ---------------------------------------------------------------------------
@dataclass
class MixerParams:
    conv_w: np.ndarray   # [2 hk dk + hv dv, W]
    A_log: np.ndarray    # [hv]
    dt_bias: np.ndarray  # [hv]
    norm_w: np.ndarray   # [dv]
    eps: float = 1e-6


@dataclass
class MixerResult:
    y: np.ndarray           # [T, hv * dv], rounded by `store`
    conv_state: np.ndarray  # [W - 1, C], rounded by `store`
    S: np.ndarray           # [hv, dv, dk], rounded to fp32
    o: np.ndarray           # [T, hv, dv] float64, before the output norm


def gated_deltanet(qkv, z, a, b, p: MixerParams, hk: int, hv: int, dk: int, dv: int,
                   conv_state=None, S0=None, store=round_fp32) -> MixerResult:
    """The Gated DeltaNet mixer over one token sequence (the kept tokens,
    reading G1): conv + SiLU (G3), L2 norm (G4), decay and strength (G5),
    the gated delta rule (G6, G7), the gated output norm (G8)."""
    qkv = np.asarray(qkv, dtype=F64)
    T = qkv.shape[0]
    assert qkv.shape[1] == 2 * hk * dk + hv * dv and hv % hk == 0
    c, conv_out = causal_conv_silu(qkv, p.conv_w, conv_state)
    qh = c[:, :hk * dk].reshape(T, hk, dk)
    kh = c[:, hk * dk:2 * hk * dk].reshape(T, hk, dk)
    vh = c[:, 2 * hk * dk:].reshape(T, hv, dv)
    qh = l2_normalize(qh) / np.sqrt(dk)
    kh = l2_normalize(kh)
    grp = hv // hk
    qv = qh[:, np.arange(hv) // grp]
    kv = kh[:, np.arange(hv) // grp]
    g, beta = decay_and_strength(a, b, p.A_log, p.dt_bias)
    o, S = gated_delta_rule(qv, kv, vh, g, beta, S0)
    y = gated_rmsnorm(o, np.asarray(z, dtype=F64).reshape(T, hv, dv), p.norm_w, p.eps)
    return MixerResult(y=store(y.reshape(T, hv * dv)), conv_state=store(conv_out),
                       S=round_fp32(S), o=o)


def mixer_flops(T: int, hk: int, hv: int, dk: int, dv: int, W: int) -> float:
    """Algorithmic floating-point operations of the mixer (multiply-adds
    counted as 2): the recurrence's S.k, S.q and rank-1 update
    (3 * 2 dv dk per token and value head) plus the convolution
    (2 W per channel and token); normalisations and gates are O(T H d)."""
    C = 2 * hk * dk + hv * dv
    return float(T) * (hv * 6.0 * dv * dk + 2.0 * W * C)


def sample_mixer(qkv, z, a, b, p: MixerParams, hk: int, hv: int, dk: int, dv: int,
                 heads, store=round_fp32) -> np.ndarray:
    """y restricted to the value heads in `heads` (the recurrence of each
    value head is independent), for checking large runs one head at a time.
    Returns [T, len(heads), dv]."""
    qkv = np.asarray(qkv, dtype=F64)
    T = qkv.shape[0]
    grp = hv // hk
    W = p.conv_w.shape[1]
    out = []
    for h in heads:
        kh_ = h // grp
        cols = np.concatenate([np.arange(kh_ * dk, (kh_ + 1) * dk),
                               hk * dk + np.arange(kh_ * dk, (kh_ + 1) * dk),
                               2 * hk * dk + np.arange(h * dv, (h + 1) * dv)])
        c, _ = causal_conv_silu(qkv[:, cols], np.asarray(p.conv_w)[cols].reshape(-1, W))
        qh = l2_normalize(c[:, :dk]) / np.sqrt(dk)
        kh = l2_normalize(c[:, dk:2 * dk])
        vh = c[:, 2 * dk:]
        g, beta = decay_and_strength(np.asarray(a)[:, h:h + 1], np.asarray(b)[:, h:h + 1],
                                     np.asarray(p.A_log)[h:h + 1],
                                     np.asarray(p.dt_bias)[h:h + 1])
        o, _ = gated_delta_rule(qh[:, None], kh[:, None], vh[:, None], g, beta)
        zz = np.asarray(z, dtype=F64).reshape(T, hv, dv)[:, h:h + 1]
        out.append(gated_rmsnorm(o, zz, p.norm_w, p.eps)[:, 0])
    return store(np.stack(out, axis=1))


# ---------------------------------------------------------------------------
# A hybrid stack with the gate (G10, G11)
# ---------------------------------------------------------------------------
#  G10 A Gated DeltaNet layer is r = x + W_out . mixer(W_in . RMSNorm(x)) (no
#      projection biases; W_in's rows give qkv, then z, then a, then b),
#      followed by the same SwiGLU FFN sub-layer as an attention layer.
#      Rounding points as the attention layers': the normed rows, the
#      projections, the mixer output and the residual are stored.
#  G11 In a hybrid stack gated at layer L, layers below L run over all N
#      tokens; layer L runs its token mixer (attention or Gated DeltaNet) over
#      all N tokens and the scorer reads the post-mixer residual; the kept
#      rows continue into layer L's FFN and every layer above. Attention
#      layers above the gate use the token-gated logits; Gated DeltaNet
#      layers above it run their mixer on the kept rows in order (G1).
@dataclass
class GdnStackLayer:
    norm: np.ndarray                   # [d]
    w_in: np.ndarray                   # [C + hv dv + 2 hv, d]
    mixer: MixerParams
    w_out: np.ndarray                  # [d, hv dv]
    hk: int
    hv: int
    dk: int
    dv: int
    ffn_norm: Optional[np.ndarray] = None
    w_gate_up: Optional[np.ndarray] = None
    w_down: Optional[np.ndarray] = None


def gdn_sublayer(x, lw: GdnStackLayer, eps: float, store=round_fp32):
    """r = x + W_out . mixer(W_in . RMSNorm(x)) over the rows of x (one
    sequence), and the mixer's final (conv rows, S)."""
    from .tokengate_oracle import rmsnorm
    x = np.asarray(x, dtype=F64)
    T = x.shape[0]
    C = 2 * lw.hk * lw.dk + lw.hv * lw.dv
    y = store(rmsnorm(x, lw.norm, eps))
    proj = store(y @ np.asarray(lw.w_in, dtype=F64).T)
    qkv = proj[:, :C]
    z = proj[:, C:C + lw.hv * lw.dv]
    a = proj[:, C + lw.hv * lw.dv:C + lw.hv * lw.dv + lw.hv]
    b = proj[:, C + lw.hv * lw.dv + lw.hv:]
    res = gated_deltanet(qkv, z, a, b, lw.mixer, lw.hk, lw.hv, lw.dk, lw.dv, store=store)
    r = store(x + res.y @ np.asarray(lw.w_out, dtype=F64).T)
    assert r.shape == (T, x.shape[1])
    return r, (res.conv_state, res.S)


def hybrid_prefill(x, protect, k: int, m, gate_layer: int, store=round_fp32, kept_idx=None,
                   fold_norms: bool = False):
    """The gated forward of a hybrid stack (G11). m is a tokengate_oracle
    Model whose layers are attention Layers or GdnStackLayers. Returns a
    PrefillResult; kv holds, per layer, the attention (k, v) or the Gated
    DeltaNet (conv rows, S). fold_norms: as in tokengate_oracle.prefill (R7b);
    a Gated DeltaNet layer's input projection is never folded."""
    from .tokengate_oracle import (PrefillResult, attention_sublayer, compact, ffn_sublayer,
                                   score, topk_select)

    def mix(h, lw, pos, s, gated, fresh):
        if isinstance(lw, GdnStackLayer):
            return gdn_sublayer(h, lw, m.eps, store)
        fold = fold_norms and fresh
        if gated:
            return attention_sublayer(h, lw, m, pos, s, lw.gain, lw.tau, store, fold)
        return attention_sublayer(h, lw, m, pos, None, None, None, store, fold)

    x = store(np.asarray(x, dtype=F64))
    n = x.shape[0]
    pos = np.arange(n, dtype=np.int32)
    kv = []
    h = x
    fresh = False  # rows just written by a residual GEMM (R7b)
    for li in range(max(gate_layer, 0)):
        r, st = mix(h, m.layers[li], pos, None, False, fresh)
        kv.append(st)
        h = ffn_sublayer(r, m.layers[li], m, store, fold_norms)
        fresh = True
    if gate_layer >= 0:
        r, st = mix(h, m.layers[gate_layer], pos, None, False, fresh)
        kv.append(st)
        fresh = True
    else:
        r = h
    s = round_fp32(score(r, m.score_norm, m.eps, m.score_w1, m.score_b1, m.score_w2,
                         m.score_b2, store, fold_norms and fresh))
    idx = topk_select(s.astype(np.float32), protect, k) if kept_idx is None \
        else np.asarray(kept_idx, dtype=np.int32)
    x_k, pos_k, s_k = compact(r, idx, pos, s)  # rows keep their freshness
    if gate_layer >= 0:
        h = ffn_sublayer(x_k, m.layers[gate_layer], m, store, fold_norms and fresh)
        fresh = fresh or m.layers[gate_layer].w_gate_up is not None
    else:
        h = x_k
    for li in range(gate_layer + 1, len(m.layers)):
        r, st = mix(h, m.layers[li], pos_k, s_k, True, fresh)
        kv.append(st)
        h = ffn_sublayer(r, m.layers[li], m, store, fold_norms)
        fresh = True
    from .tokengate_oracle import rmsnorm
    out = h if m.final_norm is None else store(rmsnorm(h, m.final_norm, m.eps))
    return PrefillResult(out=out, kept_idx=idx, scores=s.astype(np.float32), kv=kv,
                         gate_residual=r if gate_layer < 0 else None)
