"""TokenGate gated prefill -- the oracle.

TEST INFRASTRUCTURE. This module is a plain, slow, obviously correct CPU
restatement of what the gated-prefill path computes, in float64 (numpy).
Only the test suite, the package's smoke check and the benchmark's CPU
baseline leg may import it. The CUDA library never calls it and shares no
code, table or constant with it.

Sources (web pages about the TokenGate paper, cited by title and section):

  [TC]  Tencent Cloud developer article "TokenGate：端到端可训练的 Token 剪枝机制，
        让大模型 Prefill 提速 11.3 倍"
  [FW]  farwalk.ai news item "Researchers from Stanford and Berkeley propose
        TokenGate, using learnable pruning to speed up long-context Prefill by
        up to about 11x"
  [HF]  Hugging Face paper page mirror "TokenGate：通过学习式 Token 剪枝让 LLM
        实现快速且节省内存的预填充", abstract
  [AI]  ai.866data.com article "让大模型学会"略读"：TokenGate如何破解长上下文推理
        的效率困局"

Mechanism, as the pages give it:
  * N tokens go through layers below the gate layer L unchanged; at layer L,
    after attention, a small MLP scores every token from its post-attention
    residual, a top-K selector keeps K of them, and only those continue into
    layer L's feed-forward network and the layers above; pruned tokens make
    no KV there ([TC] "TokenGate 提前筛选 Token"; [AI] "可学习剪枝的机制设计";
    [FW] "论文的方法").
  * The question span (and decode tokens) can never be pruned ([TC] same
    section; [AI] same section).
  * Above the gate the kept tokens' scores enter the attention logits as a
    bias, with a learnable per-head gain and a per-head temperature ([TC]
    "门控机制为评分网络建立梯度路径"; [AI] "可学习剪枝的机制设计"; [HF] abstract).
  * Layers at and below the gate keep the full-prompt KV ([TC]
    "TokenGate 的工程验证仍有限").

Readings where the pages are silent (each one is listed in the design notes):
  R1  Scorer = RMSNorm -> Linear(d->F) -> SiLU -> Linear(F->1); eps 1e-6.
  R2  The bias algebra: logit_ij = (q_i.k_j) / (sqrt(dh) * tau_h)
      + gain_h * logsigmoid(s_j), masked to pos_j <= pos_i. Gain and tau are
      per query head; tau divides only the q.k term; the bias applies to every
      kept key, the diagonal and protected keys included.
  R3  Budget K counts the protected tokens: exactly K are kept, and more than
      K protected tokens is an error. Ranking is (score descending, index
      ascending); -0.0 equals +0.0; NaN ranks below -inf. Output ascending.
  R4  RoPE: rotate-half pairing (i, i + dh/2), theta_i = base^(-2i/dh), angle
      pos * theta_i evaluated in float64, at each kept token's original
      position.
  R5  GQA: query head h reads KV head floor(h / (Hq / Hkv)).
  R6  Backbone layer (Qwen3 shape): pre-RMSNorm, fused QKV without bias,
      optional per-head RMSNorm on q and k before RoPE (qk-norm), causal
      attention, output projection + residual, pre-RMSNorm SwiGLU FFN +
      residual, final RMSNorm of the kept rows.
  R7  Rounding points: a tensor that a GPU kernel stores in the compute
      dtype (bf16 or fp32) is rounded to it here at the same place: the
      input, each RMSNorm output fed to a GEMM, q/k/v after projection,
      q/k after qk-norm + RoPE, the attention output, every residual-stream
      value, the SwiGLU product, and the final output. Everything between
      two rounding points is float64. Scores are stored as float32.
  R8  Decode: the t-th generated token has position N + t; above the gate
      its logits over the cached keys follow R2, with the kept prompt tokens'
      scores as the bias and no bias (logsigmoid = 0) on generated tokens'
      keys; tau applies to every key.
  R7b Folded RMSNorm (an implementation form of R6, not from the pages):
      RMSNorm(x; g) . W^T = (x / rms(x)) . (W diag g)^T in real arithmetic.
      When the library runs a projection with the folded weight
      W_g = W diag(g) (stored once, in the compute dtype), the normed row is
      never stored, so by R7 the rounding point moves from the normed row
      to W_g. It does so where the norm's input rows were just written by a
      residual GEMM (`fresh` below; the compaction gathers the rows' sums of
      squares with them): every norm but the stack's input and a Gated
      DeltaNet layer's input projection.
  R9  Backward: the gradients of the gated attention with respect to q, k,
      v, the gate scores s, the per-head gain and the per-head temperature,
      for an upstream gradient of its output. The pages give only the path
      (loss -> upper attention -> gate scores -> scorer); the formulas are
      the plain chain rule of R2. Rounding to the storage dtype passes
      gradients straight through.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, List, Optional, Sequence

import numpy as np

F64 = np.float64

# ---------------------------------------------------------------------------
# Storage rounding (R7)
# ---------------------------------------------------------------------------


def round_fp32(x) -> np.ndarray:
    """Round to IEEE binary32 (round-to-nearest-even) and return float64."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=F64).astype(np.float32).astype(F64)


def round_bf16(x) -> np.ndarray:
    """Round to bfloat16 and return float64.

    bfloat16 is the upper half of a binary32 word. The value is first
    rounded to binary32 (as a kernel accumulating in fp32 holds it), then the
    low 16 bits are dropped with round-to-nearest-even: add 0x7FFF plus the
    lowest kept bit, then truncate. NaN stays NaN; values past the largest
    bfloat16 round to infinity.
    """
    a = np.asarray(x, dtype=F64).astype(np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + keep_lsb) & np.uint64(0xFFFF0000)
    out = u.astype(np.uint32).view(np.float32).astype(F64)
    out = np.where(np.isnan(a), np.nan, out)
    return out


def identity(x) -> np.ndarray:
    return np.asarray(x, dtype=F64)


STORE = {"bf16": round_bf16, "f32": round_fp32, "f64": identity}

# ---------------------------------------------------------------------------
# Elementary functions
# ---------------------------------------------------------------------------


def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2) + eps) * gamma over the last axis (R1, R6)."""
    x = np.asarray(x, dtype=F64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(gamma, dtype=F64)


def norm_project(x, gamma, w, eps: float, store, fold: bool = False) -> np.ndarray:
    """RMSNorm(x; gamma) . w^T, unrounded. fold=False: the normed rows are a
    stored GEMM operand (R7): store(RMSNorm(x)) . w^T. fold=True (R7b): the
    folded weight is the stored operand: (x / rms(x)) . store(w diag gamma)^T."""
    w = np.asarray(w, dtype=F64)
    if not fold:
        return store(rmsnorm(x, gamma, eps)) @ w.T
    x = np.asarray(x, dtype=F64)
    inv_rms = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return (x * inv_rms) @ store(w * np.asarray(gamma, dtype=F64)).T


def sigmoid(x) -> np.ndarray:
    """1 / (1 + exp(-x)), written as exp(x) / (1 + exp(x)) for x < 0 so
    that no exponential overflows and small values keep full precision."""
    x = np.asarray(x, dtype=F64)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def silu(x) -> np.ndarray:
    x = np.asarray(x, dtype=F64)
    return x * sigmoid(x)


def logsigmoid(x) -> np.ndarray:
    """log(sigmoid(x)) = min(x, 0) - log1p(exp(-|x|)), stable for all x."""
    x = np.asarray(x, dtype=F64)
    return np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))


# ---------------------------------------------------------------------------
# Step a2: the scorer ([TC] "TokenGate 提前筛选 Token"; [AI] "可学习剪枝的机制设计")
# ---------------------------------------------------------------------------


def score(r, norm_w, eps, w1, b1, w2, b2, store: Callable = round_bf16,
          fold: bool = False) -> np.ndarray:
    """Importance score of each token from its post-attention residual.

    s_t = w2 . SiLU(W1 . RMSNorm(r_t) + b1) + b2   (R1)

    r: [N, d]; w1: [F, d]; b1: [F] or None; w2: [F]; b2: scalar or None.
    The normalised rows are rounded by `store` (they are a GEMM operand), or
    with fold the folded weight is (R7b). Returns float64 scores; a caller
    that needs the stored value rounds them to float32.
    """
    h = norm_project(r, norm_w, w1, eps, store, fold)
    if b1 is not None:
        h = h + np.asarray(b1, dtype=F64)
    s = silu(h) @ np.asarray(w2, dtype=F64).reshape(-1)
    if b2 is not None:
        s = s + float(np.asarray(b2, dtype=F64).reshape(-1)[0])
    return s


# ---------------------------------------------------------------------------
# Step a3: top-K selection with protected tokens (R3)
# ([TC] "TokenGate 提前筛选 Token": top-K keeps K tokens, designated tokens are
#  un-prunable; [AI] "可学习剪枝的机制设计": the question part is never pruned)
# ---------------------------------------------------------------------------


class BudgetError(ValueError):
    """Raised when k < 1, k > n, or more than k tokens are protected."""


def topk_select(scores32, protect, k: int) -> np.ndarray:
    """Indices (int32, ascending) of the kept tokens.

    Every protected token is kept. The remaining k - P slots go to the
    unprotected tokens ranked by (score descending, index ascending), with
    NaN below every number and -0.0 equal to +0.0 (plain float comparison
    already treats the two zeros as equal).
    """
    s = np.asarray(scores32, dtype=np.float32)
    n = s.shape[0]
    if not (1 <= k <= n):
        raise BudgetError(f"k={k} outside [1, n={n}]")
    prot = np.zeros(n, dtype=bool) if protect is None else np.asarray(protect).astype(bool)
    p = int(prot.sum())
    if p > k:
        raise BudgetError(f"{p} protected tokens exceed the budget k={k}")
    cand = np.nonzero(~prot)[0]
    sv = s[cand].astype(F64)
    is_nan = np.isnan(sv)
    neg = np.where(is_nan, 0.0, -sv)
    # np.lexsort sorts by the LAST key first: NaN flag (False first), then
    # -score ascending (= score descending), then index ascending.
    order = np.lexsort((cand, neg, is_nan))
    chosen = cand[order[: k - p]]
    kept = np.sort(np.concatenate([np.nonzero(prot)[0], chosen]))
    return kept.astype(np.int32)


# ---------------------------------------------------------------------------
# Step a4: compaction ([TC] "TokenGate 提前筛选 Token"; [FW] "论文的方法")
# ---------------------------------------------------------------------------


def compact(x, kept_idx, pos=None, scores=None):
    """Gather the kept rows, their original positions and their scores."""
    idx = np.asarray(kept_idx, dtype=np.int64)
    x_out = np.asarray(x)[idx]
    pos_out = idx.astype(np.int32) if pos is None else np.asarray(pos)[idx].astype(np.int32)
    s_out = None if scores is None else np.asarray(scores)[idx]
    return x_out, pos_out, s_out


# ---------------------------------------------------------------------------
# RoPE at original positions (R4)
# ---------------------------------------------------------------------------


def rope(x, pos, base: float) -> np.ndarray:
    """Rotate-half RoPE of x [T, H, dh] at integer positions pos [T]."""
    x = np.asarray(x, dtype=F64)
    dh = x.shape[-1]
    half = dh // 2
    i = np.arange(half, dtype=F64)
    theta = float(base) ** (-2.0 * i / dh)
    ang = np.asarray(pos, dtype=F64)[:, None] * theta[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1 = x[..., :half]
    x2 = x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ---------------------------------------------------------------------------
# Step a7: token-gated causal GQA attention (R2, R5)
# ([TC] "门控机制为评分网络建立梯度路径": scores of kept tokens enter the later
#  attention and re-weight it; per-head learnable gain and temperature scaling;
#  [AI] "可学习剪枝的机制设计": the score becomes a bias on the attention logits)
# ---------------------------------------------------------------------------


def gated_attention_rows(q, pos_q, k, v, pos_k, s, gain, tau) -> np.ndarray:
    """Token-gated attention of query rows q [Tq, Hq, dh] at positions pos_q
    over keys k/v [Tk, Hkv, dh] at positions pos_k (R2, R5):

    l_ij = (q_i . k_j) / (sqrt(dh) * tau_h) + gain_h * logsigmoid(s_j), pos_j <= pos_i

    s: [Tk] gate scores of the keys or None (no bias); gain/tau: [Hq] or None
    (gain 0, tau 1). Pruned keys are simply absent from k/v.
    """
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    v = np.asarray(v, dtype=F64)
    tq, hq, dh = q.shape
    tk, hkv = k.shape[0], k.shape[1]
    group = hq // hkv
    gain = np.zeros(hq) if gain is None else np.asarray(gain, dtype=F64)
    tau = np.ones(hq) if tau is None else np.asarray(tau, dtype=F64)
    key_bias = np.zeros(tk) if s is None else logsigmoid(s)
    pq = np.asarray(pos_q, dtype=np.int64)
    pk = np.asarray(pos_k, dtype=np.int64)
    allowed = pk[None, :] <= pq[:, None]  # [query i, key j]
    out = np.empty((tq, hq, dh), dtype=F64)
    for h in range(hq):
        g = h // group
        logits = (q[:, h, :] @ k[:, g, :].T) / (math.sqrt(dh) * tau[h])
        logits = logits + gain[h] * key_bias[None, :]
        logits = np.where(allowed, logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        w = np.exp(logits - m)
        w = w / w.sum(axis=1, keepdims=True)
        out[:, h, :] = w @ v[:, g, :]
    return out


def gated_attention(q, k, v, pos, s, gain, tau) -> np.ndarray:
    """o_i = sum_j softmax_j(l_ij) v_j over kept keys with pos_j <= pos_i,
    for the kept rows themselves as queries (q, k, v share positions pos)."""
    return gated_attention_rows(q, pos, k, v, pos, s, gain, tau)


def gated_attn_prefill(q, k, v, pos, s, gain, tau, rope_base, store=round_bf16):
    """The standalone gated-attention call: RoPE q and k at the original
    positions (stored rotated), then token-gated attention; output stored."""
    qr = store(rope(q, pos, rope_base))
    kr = store(rope(k, pos, rope_base))
    return store(gated_attention(qr, kr, np.asarray(v, dtype=F64), pos, s, gain, tau))


# ---------------------------------------------------------------------------
# Gated-attention backward (R9). The pages' point about the gate: the top-K
# choice itself is discrete, but the kept tokens' scores stay in the
# differentiable graph through the upper layers' attention bias, so the task
# loss reaches the scorer along loss -> upper attention -> gate scores ->
# scorer, and the per-head gain and temperature are learned with it ([TC]
# "门控机制为评分网络建立梯度路径"; [AI] "可学习剪枝的机制设计").
# ---------------------------------------------------------------------------


def gated_attention_lse(q, k, pos, s, gain, tau) -> np.ndarray:
    """lse[h, i] = log sum_{pos_j <= pos_i} exp(l_ij) with the logits of R2
    (q and k as they enter the logits). The forward's softmax normaliser,
    which its backward takes instead of recomputing it."""
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    t, hq, dh = q.shape
    group = hq // k.shape[1]
    gain_v = np.zeros(hq) if gain is None else np.asarray(gain, dtype=F64)
    tau_v = np.ones(hq) if tau is None else np.asarray(tau, dtype=F64)
    b = np.zeros(t) if s is None else logsigmoid(s)
    p = np.asarray(pos, dtype=np.int64)
    allowed = p[None, :] <= p[:, None]
    out = np.empty((hq, t))
    for h in range(hq):
        g = h // group
        logits = (q[:, h, :] @ k[:, g, :].T) / (math.sqrt(dh) * tau_v[h]) + gain_v[h] * b[None, :]
        logits = np.where(allowed, logits, -np.inf)
        m = logits.max(axis=1)
        out[h] = m + np.log(np.exp(logits - m[:, None]).sum(axis=1))
    return out


def gated_attention_grads(q, k, v, pos, s, gain, tau, dout, on_head=None):
    """Gradients of o = gated_attention(q, k, v, pos, s, gain, tau) for the
    upstream gradient dout [T, Hq, dh] (q and k as they enter the logits,
    i.e. already rotated). Returns (dq, dk, dv, ds, dgain, dtau), float64.

    With a_ij = (q_i . k_j) / (sqrt(dh) tau_h) and b_j = logsigmoid(s_j):
      l_ij = a_ij + gain_h b_j (pos_j <= pos_i), P = softmax_j(l), o_i = sum_j P_ij v_j
      dP_ij = dout_i . v_j
      dl_ij = P_ij (dP_ij - sum_j' P_ij' dP_ij')          (softmax Jacobian)
      dq_i  = sum_j dl_ij k_j / (sqrt(dh) tau_h)
      dk_j  = sum_{h in group} sum_i dl_ij q_i / (sqrt(dh) tau_h)
      dv_j  = sum_{h in group} sum_i P_ij dout_i
      dgain_h = sum_ij dl_ij b_j
      dtau_h  = -sum_ij dl_ij a_ij / tau_h                 (d a_ij / d tau_h = -a_ij / tau_h)
      ds_j  = sigmoid(-s_j) sum_h gain_h sum_i dl_ij       (d logsigmoid(x)/dx = sigmoid(-x))
    s None means no bias: ds is None and dgain is zero; gain/tau None mean
    0 and 1 (dgain and dtau are still returned). on_head, if given, is called
    as on_head(h, g, P, dl, dP) with each head's [T, T] matrices (tests use
    them to bound the effect of storage roundings).
    """
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    v = np.asarray(v, dtype=F64)
    dout = np.asarray(dout, dtype=F64)
    t, hq, dh = q.shape
    hkv = k.shape[1]
    group = hq // hkv
    gain_v = np.zeros(hq) if gain is None else np.asarray(gain, dtype=F64)
    tau_v = np.ones(hq) if tau is None else np.asarray(tau, dtype=F64)
    b = np.zeros(t) if s is None else logsigmoid(s)
    p = np.asarray(pos, dtype=np.int64)
    allowed = p[None, :] <= p[:, None]  # [query i, key j]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dgain = np.zeros(hq)
    dtau = np.zeros(hq)
    key_sum = np.zeros(t)  # sum_h gain_h sum_i dl_ij
    for h in range(hq):
        g = h // group
        c = 1.0 / (math.sqrt(dh) * tau_v[h])
        a = (q[:, h, :] @ k[:, g, :].T) * c
        logits = np.where(allowed, a + gain_v[h] * b[None, :], -np.inf)
        w = np.exp(logits - logits.max(axis=1, keepdims=True))
        w = w / w.sum(axis=1, keepdims=True)
        dp = dout[:, h, :] @ v[:, g, :].T
        dl = w * (dp - (w * dp).sum(axis=1, keepdims=True))
        if on_head is not None:
            on_head(h, g, w, dl, dp)
        dq[:, h, :] = c * (dl @ k[:, g, :])
        dk[:, g, :] += c * (dl.T @ q[:, h, :])
        dv[:, g, :] += w.T @ dout[:, h, :]
        col = dl.sum(axis=0)
        dgain[h] = col @ b
        dtau[h] = -(dl * np.where(allowed, a, 0.0)).sum() / tau_v[h]
        key_sum += gain_v[h] * col
    ds = None if s is None else sigmoid(-np.asarray(s, dtype=F64)) * key_sum
    return dq, dk, dv, ds, dgain, dtau


def gated_attn_backward(q, k, v, pos, s, gain, tau, rope_base, dout, store=round_bf16):
    """The standalone backward call, for the inputs of gated_attn_prefill
    (q and k un-rotated): q and k are rotated and stored as in the forward,
    the gradients are taken there, and those of q and k are rotated back
    (RoPE at position p is orthogonal, so its transpose is RoPE at -p; the
    storage rounding passes gradients straight through). dq, dk, dv are
    stored in the compute dtype; ds, dgain, dtau as float32."""
    qr = store(rope(q, pos, rope_base))
    kr = store(rope(k, pos, rope_base))
    dqr, dkr, dv, ds, dgain, dtau = gated_attention_grads(
        qr, kr, np.asarray(v, dtype=F64), pos, s, gain, tau, dout)
    neg = -np.asarray(pos, dtype=np.int64)
    dq = store(rope(dqr, neg, rope_base))
    dk = store(rope(dkr, neg, rope_base))
    return (dq, dk, store(dv), None if ds is None else round_fp32(ds), round_fp32(dgain),
            round_fp32(dtau))


def attention_backward_flops(t: int, hq: int, dh: int) -> float:
    """Algorithmic FLOPs of the causal attention backward: the five
    [t x t x dh] products (S and dP recomputed, dV, dK, dQ), 2.5 times the
    forward's 4 * dh * hq * t (t + 1) / 2."""
    return 2.5 * attention_flops(t, hq, dh)


# ---------------------------------------------------------------------------
# Backbone layer pieces (R6) and the full stack
# ---------------------------------------------------------------------------


@dataclass
class Layer:
    attn_norm: np.ndarray  # [d]
    wqkv: np.ndarray  # [(hq + 2 hkv) dh, d]: Wq rows, then Wk, then Wv
    wo: np.ndarray  # [d, hq dh]
    ffn_norm: np.ndarray  # [d]
    w_gate_up: Optional[np.ndarray]  # [2 I, d]: W_gate rows then W_up rows; None = no FFN
    w_down: Optional[np.ndarray]  # [d, I]
    q_norm: Optional[np.ndarray] = None  # [dh] (qk-norm on when given)
    k_norm: Optional[np.ndarray] = None
    gain: Optional[np.ndarray] = None  # [hq], used only above the gate
    tau: Optional[np.ndarray] = None  # [hq]


@dataclass
class Model:
    d_model: int
    n_heads_q: int
    n_heads_kv: int
    head_dim: int
    layers: List[Layer]
    final_norm: Optional[np.ndarray]
    score_norm: np.ndarray
    score_w1: np.ndarray
    score_b1: Optional[np.ndarray]
    score_w2: np.ndarray
    score_b2: Optional[np.ndarray]
    eps: float = 1e-6
    rope_base: float = 1e6


def project_qkv(x, lw: Layer, m: Model, pos, store, fold: bool = False):
    """Rows x [t, d] -> q [t, Hq, dh] and k [t, Hkv, dh] (qk-norm, then RoPE at
    pos, stored) and v [t, Hkv, dh] (stored) (R4, R6, R7; fold: R7b)."""
    t = x.shape[0]
    hq, hkv, dh = m.n_heads_q, m.n_heads_kv, m.head_dim
    qkv = store(norm_project(x, lw.attn_norm, lw.wqkv, m.eps, store, fold))
    q = qkv[:, : hq * dh].reshape(t, hq, dh)
    k = qkv[:, hq * dh : (hq + hkv) * dh].reshape(t, hkv, dh)
    v = qkv[:, (hq + hkv) * dh :].reshape(t, hkv, dh)
    if lw.q_norm is not None:
        q = rmsnorm(q, lw.q_norm, m.eps)
        k = rmsnorm(k, lw.k_norm, m.eps)
    return store(rope(q, pos, m.rope_base)), store(rope(k, pos, m.rope_base)), v


def attention_sublayer(x, lw: Layer, m: Model, pos, s, gain, tau, store, fold: bool = False):
    """r = x + Wo . attn(RoPE(qk-norm(W_qkv . RMSNorm(x)))) and the layer's KV."""
    t = x.shape[0]
    q, k, v = project_qkv(x, lw, m, pos, store, fold)
    o = store(gated_attention(q, k, v, pos, s, gain, tau))
    r = store(x + o.reshape(t, m.n_heads_q * m.head_dim) @ np.asarray(lw.wo, dtype=F64).T)
    return r, (k, v)


def ffn_sublayer(x, lw: Layer, m: Model, store, fold: bool = False):
    """x + W_down . (SiLU(W_gate . y) * (W_up . y)), y = RMSNorm(x)."""
    if lw.w_gate_up is None:
        return x
    inter = lw.w_gate_up.shape[0] // 2
    gu = norm_project(x, lw.ffn_norm, lw.w_gate_up, m.eps, store, fold)
    h = store(silu(gu[:, :inter]) * gu[:, inter:])
    return store(x + h @ np.asarray(lw.w_down, dtype=F64).T)


@dataclass
class PrefillResult:
    out: np.ndarray  # [K, d] final (normed) hidden states of the kept rows
    kept_idx: np.ndarray  # [K] int32 ascending
    scores: np.ndarray  # [N] float32 gate scores
    kv: list = field(default_factory=list)  # per layer (k, v): N rows at/below gate, K above
    gate_residual: Optional[np.ndarray] = None  # [N, d] the scorer's input


def prefill(x, protect, k: int, m: Model, gate_layer: int, store=round_bf16,
            kept_idx=None, fold_norms: bool = False) -> PrefillResult:
    """The three-stage gated forward ([TC] "TokenGate 提前筛选 Token";
    [FW] "论文的方法"; [AI] "可学习剪枝的机制设计").

    gate_layer = L >= 0: layers < L run over all N tokens; layer L runs its
    attention over all N tokens, then the scorer reads its post-attention
    residual, the selector keeps k tokens, and layer L's FFN and every layer
    above run over the kept tokens only, with token-gated attention.
    gate_layer = -1 puts the gate before layer 0 (the scorer reads the input
    hidden states) so that every layer is an upper layer.

    kept_idx, when given, replaces the oracle's own selection (teacher
    forcing): the later stages then consume exactly that kept set.

    fold_norms (R7b): a norm whose input rows come straight from a residual
    GEMM (`fresh`) rounds the folded weight instead of the normed rows.
    """
    x = store(np.asarray(x, dtype=F64))
    n = x.shape[0]
    pos = np.arange(n, dtype=np.int32)
    kv = []
    h = x
    fresh = False  # the input rows were not written by a residual GEMM
    for li in range(max(gate_layer, 0)):
        r, kvl = attention_sublayer(h, m.layers[li], m, pos, None, None, None, store,
                                    fold_norms and fresh)
        kv.append(kvl)
        h = ffn_sublayer(r, m.layers[li], m, store, fold_norms)
        fresh = True
    if gate_layer >= 0:
        lw = m.layers[gate_layer]
        r, kvl = attention_sublayer(h, lw, m, pos, None, None, None, store, fold_norms and fresh)
        kv.append(kvl)
        fresh = True
    else:
        r = h
    s = round_fp32(score(r, m.score_norm, m.eps, m.score_w1, m.score_b1, m.score_w2,
                         m.score_b2, store, fold_norms and fresh))
    idx = topk_select(s.astype(np.float32), protect, k) if kept_idx is None \
        else np.asarray(kept_idx, dtype=np.int32)
    x_k, pos_k, s_k = compact(r, idx, pos, s)  # rows keep their freshness (R7b)
    if gate_layer >= 0:
        lw = m.layers[gate_layer]
        h = ffn_sublayer(x_k, lw, m, store, fold_norms and fresh)
        fresh = fresh or lw.w_gate_up is not None
    else:
        h = x_k
    for li in range(gate_layer + 1, len(m.layers)):
        lw = m.layers[li]
        r, kvl = attention_sublayer(h, lw, m, pos_k, s_k, lw.gain, lw.tau, store,
                                    fold_norms and fresh)
        kv.append(kvl)
        h = ffn_sublayer(r, lw, m, store, fold_norms)
        fresh = True
    out = h if m.final_norm is None else store(rmsnorm(h, m.final_norm, m.eps))
    return PrefillResult(out=out, kept_idx=idx, scores=s.astype(np.float32), kv=kv,
                         gate_residual=r if gate_layer < 0 else None)


def prefill_budgets(x, protect, ks, m: Model, gate_layer: int, store=round_bf16,
                    kept_sets=None, fold_norms: bool = False) -> List[PrefillResult]:
    """The gated forward of one request at several budgets: by definition the
    single-budget forward at each k of ks (one trained gate serves every
    budget, [AI] "可学习剪枝的机制设计"). kept_sets, when given, teacher-forces
    each budget's kept set."""
    return [prefill(x, protect, k, m, gate_layer, store,
                    None if kept_sets is None else kept_sets[b], fold_norms)
            for b, k in enumerate(ks)]


def decode_step(x, pos: int, m: Model, gate_layer: int, cache, kept_scores=None,
                store=round_bf16):
    """One generated token through every layer, after a gated prefill.

    Generated tokens are never pruned ([TC] "TokenGate 提前筛选 Token"), so
    the token runs every layer and appends its k/v to every layer's cache.
    Layers at and below the gate hold the full prompt's KV, layers above only
    the kept tokens' KV ([TC] "TokenGate 的工程验证仍有限"). In decoding the
    gate bias fixed at prefill is an additive mask over the cached keys (same
    section), so an upper layer's logits are those of R2 with the kept prompt
    tokens' scores; the generated tokens' keys carry no bias (R8).

    x [d]: the token's input hidden state; pos: its position (the prompt is
    0..N-1, so the t-th generated token has pos N + t).
    cache: per layer (k [T_l, Hkv, dh] post-RoPE, v [T_l, Hkv, dh]): T_l =
    N + t at or below the gate, K + t above, rows in position order, every one
    earlier than pos. kept_scores [K]: gate scores of the kept prompt tokens,
    which are rows 0..K-1 of every upper cache.
    Returns (out [d] final-normed, [(k_new [Hkv, dh], v_new [Hkv, dh]) per layer]).
    """
    h = store(np.asarray(x, dtype=F64).reshape(1, -1))
    p = np.array([pos], dtype=np.int64)
    new_kv = []
    for li, lw in enumerate(m.layers):
        kc, vc = cache[li]
        q, k, v = project_qkv(h, lw, m, p, store)
        k_all = np.concatenate([np.asarray(kc, dtype=F64), k])
        v_all = np.concatenate([np.asarray(vc, dtype=F64), v])
        before = np.full(k_all.shape[0], pos, dtype=np.int64)  # every key is visible
        if li > gate_layer:
            ks = np.asarray(kept_scores, dtype=F64)
            s_all = np.concatenate([ks, np.full(k_all.shape[0] - ks.size, np.inf)])  # logsig(inf) = 0
            o = gated_attention_rows(q, p, k_all, v_all, before, s_all, lw.gain, lw.tau)
        else:
            o = gated_attention_rows(q, p, k_all, v_all, before, None, None, None)
        o = store(o)
        r = store(h + o.reshape(1, -1) @ np.asarray(lw.wo, dtype=F64).T)
        h = ffn_sublayer(r, lw, m, store)
        new_kv.append((k[0], v[0]))
    out = h if m.final_norm is None else store(rmsnorm(h, m.final_norm, m.eps))
    return out[0], new_kv


def decode_bytes(m: Model, lens, elem: int = 2) -> int:
    """Algorithmic HBM bytes of one decode step: every weight matrix read
    once, every cached k/v row read once (lens[l] rows before the step), the
    new k/v rows written."""
    hkv, dh = m.n_heads_kv, m.head_dim
    total = 0
    for lw, t in zip(m.layers, lens):
        for w in (lw.wqkv, lw.wo, lw.w_gate_up, lw.w_down):
            if w is not None:
                total += int(np.asarray(w).size) * elem
        total += (2 * t + 2) * hkv * dh * elem
    return total


def gated_layer_forward(x_k, pos_k, s_k, lw: Layer, m: Model, store=round_bf16,
                        fold_norms: bool = False):
    """One upper (gated) layer over already-compacted rows: attention + FFN
    (the FFN's input rows come from the attention's residual GEMM, R7b)."""
    r, kv = attention_sublayer(np.asarray(x_k, dtype=F64), lw, m, pos_k, s_k,
                               lw.gain, lw.tau, store)
    return ffn_sublayer(r, lw, m, store, fold_norms), kv


# ---------------------------------------------------------------------------
# Algorithmic work counts (used by the benchmark's roofline denominators)
# ---------------------------------------------------------------------------


def attention_flops(t: int, hq: int, dh: int) -> float:
    """Causal attention FLOPs over t rows: 4 * dh * hq * t (t + 1) / 2."""
    return 4.0 * dh * hq * t * (t + 1) / 2.0


def select_compact_bytes(n: int, k: int, d: int, elem: int = 2) -> int:
    """Bytes select+compact must move: scores + mask read, indices written,
    kept rows read and written, positions and scores of kept rows written."""
    return 4 * n + n + 4 * k + 2 * k * d * elem + 8 * k


__all__: Sequence[str] = [
    "round_bf16", "round_fp32", "identity", "STORE", "rmsnorm", "silu", "sigmoid",
    "logsigmoid", "score", "BudgetError", "topk_select", "compact", "rope",
    "gated_attention", "gated_attention_rows", "gated_attn_prefill", "Layer", "Model", "attention_sublayer",
    "ffn_sublayer", "prefill", "PrefillResult", "gated_layer_forward",
    "attention_flops", "select_compact_bytes",
]
