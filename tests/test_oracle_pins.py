"""Pins for the oracle: checks against things other than the oracle itself.

Each test ties one oracle function to a closed form, a brute-force count, an
invariant the method implies, a hand-derived fixture, or a library routine
(torch, scipy, Hugging Face transformers) that computes the same special
case. A plausible slip anywhere in the oracle (a dropped term, a wrong sign,
a transposed operand, a wrong head mapping) fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import tokengate_oracle as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32(vals):
    return np.array([float(v) for v in vals], dtype=np.float32)


# ---------------------------------------------------------------- rounding


def test_round_bf16_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        [0.0, -0.0, 1.0, -1.0, 3.0e38, 3.4e38, -3.4e38, 1e-40, -1e-40, np.inf, -np.inf],
        # exact halfway cases between bf16 neighbours, both parities
        [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 2.0 ** -130 * 1.5],
    ]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = ref.round_bf16(x)
    assert np.array_equal(got, want)
    assert np.isnan(ref.round_bf16(np.array([np.nan], np.float32)))[0]


def test_round_fp32_is_binary32():
    x = np.array([1.0 + 2.0 ** -30, math.pi, 1e-50, 1e50])
    got = ref.round_fp32(x)
    assert got[0] == 1.0 and got[1] == float(np.float32(math.pi))
    assert got[2] == 0.0 and np.isinf(got[3])


# ---------------------------------------------------------------- elementary


def test_rmsnorm_closed_form_and_scale_invariance():
    c, d, eps = 3.0, 16, 1e-6
    x = np.full((1, d), c)
    g = np.linspace(0.5, 1.5, d)
    y = ref.rmsnorm(x, g, eps)
    assert np.allclose(y, c / math.sqrt(c * c + eps) * g, rtol=0, atol=1e-15)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, d))
    assert np.allclose(ref.rmsnorm(7.0 * x, g, 0.0), ref.rmsnorm(x, g, 0.0), atol=1e-13)
    # library routine
    want = torch.nn.functional.rms_norm(torch.from_numpy(x), (d,), torch.from_numpy(g), eps)
    assert np.allclose(ref.rmsnorm(x, g, eps), want.numpy(), atol=1e-13)


def test_silu_sigmoid_logsigmoid_match_scipy():
    from scipy import special

    x = np.linspace(-800, 800, 4001)
    assert np.allclose(ref.sigmoid(x), special.expit(x), rtol=1e-13, atol=1e-300)
    assert np.allclose(ref.silu(x), x * special.expit(x), rtol=1e-13, atol=1e-300)
    assert np.allclose(ref.logsigmoid(x), special.log_expit(x), rtol=1e-13, atol=1e-13)
    assert ref.logsigmoid(np.array([0.0]))[0] == pytest.approx(-math.log(2.0), abs=1e-16)


# ---------------------------------------------------------------- scorer


def test_scorer_reduces_to_silu_of_dot_when_f_is_one():
    rng = np.random.default_rng(2)
    n, d = 9, 32
    x = rng.standard_normal((n, d))
    w1 = rng.standard_normal((1, d))
    g = rng.uniform(0.5, 1.5, d)
    got = ref.score(x, g, 1e-6, w1, None, np.ones(1), None, store=ref.identity)
    y = torch.nn.functional.rms_norm(torch.from_numpy(x), (d,), torch.from_numpy(g), 1e-6)
    want = torch.nn.functional.silu(y @ torch.from_numpy(w1[0]))
    assert np.allclose(got, want.numpy(), atol=1e-13)


def test_scorer_biases_and_scale_invariance():
    rng = np.random.default_rng(3)
    n, d, f = 11, 24, 6
    x = rng.standard_normal((n, d))
    g = np.ones(d)
    w1 = rng.standard_normal((f, d))
    b1 = rng.standard_normal(f)
    w2 = rng.standard_normal(f)
    b2 = np.array([0.25])
    s = ref.score(x, g, 0.0, w1, b1, w2, b2, store=ref.identity)
    # salient rows (4x norm) score like their unscaled direction
    s4 = ref.score(4.0 * x, g, 0.0, w1, b1, w2, b2, store=ref.identity)
    assert np.allclose(s, s4, atol=1e-12)
    # torch composition of the same layers
    tx = torch.from_numpy(x)
    y = torch.nn.functional.rms_norm(tx, (d,), torch.from_numpy(g), 0.0)
    h = torch.nn.functional.linear(y, torch.from_numpy(w1), torch.from_numpy(b1))
    want = torch.nn.functional.linear(torch.nn.functional.silu(h), torch.from_numpy(w2)[None],
                                      torch.from_numpy(b2))[:, 0]
    assert np.allclose(s, want.numpy(), atol=1e-12)


# ---------------------------------------------------------------- select


def _brute_force_select(s32, prot, k):
    """Token i is kept iff protected, or fewer than k - P unprotected tokens
    beat it, where j beats i when key_j > key_i or (key_j == key_i and j < i)
    and NaN sits below every number. Quadratic rank count, no sort."""
    n = len(s32)
    p = int(sum(prot))

    def beats(j, i):
        a, b = float(s32[j]), float(s32[i])
        na, nb = math.isnan(a), math.isnan(b)
        if na and nb:
            return j < i
        if na:
            return False
        if nb:
            return True
        return a > b or (a == b and j < i)

    kept = []
    for i in range(n):
        if prot[i]:
            kept.append(i)
            continue
        rank = sum(1 for j in range(n) if not prot[j] and j != i and beats(j, i))
        if rank < k - p:
            kept.append(i)
    return np.array(kept, dtype=np.int32)


def test_select_handworked_fixture():
    with open(os.path.join(GOLDEN, "select_handworked.json")) as fh:
        fx = json.load(fh)
    s = _f32(fx["scores"])
    assert math.copysign(1.0, s[1]) < 0  # the fixture really holds -0.0
    prot = np.array(fx["protect"], dtype=np.uint8)
    for case in fx["cases"]:
        got = ref.topk_select(s, prot, case["k"])
        assert got.tolist() == case["kept"], case


@pytest.mark.parametrize("seed", range(40))
def test_select_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 48))
    pool = _f32([0.0, -0.0, 1.0, -1.0, 0.5, np.inf, -np.inf, np.nan, 2.0, -3.0])
    mode = seed % 3
    if mode == 0:
        s = rng.standard_normal(n).astype(np.float32)
    elif mode == 1:
        s = pool[rng.integers(0, pool.size, n)]
    else:
        s = rng.integers(-2, 3, n).astype(np.float32)  # heavy ties
    prot = (rng.random(n) < 0.2).astype(np.uint8)
    p = int(prot.sum())
    for k in sorted({max(p, 1), max(p, 1) + (n - max(p, 1)) // 2, n}):
        if k < 1 or k > n:
            continue
        assert ref.topk_select(s, prot, k).tolist() == _brute_force_select(s, prot, k).tolist()


def test_select_invariants_and_edges():
    rng = np.random.default_rng(7)
    n, k = 300, 70
    s = rng.standard_normal(n).astype(np.float32)
    s[50:90] = np.float32(0.75)  # a tie block
    prot = np.zeros(n, np.uint8)
    prot[-16:] = 1
    idx = ref.topk_select(s, prot, k)
    assert idx.size == k and np.all(np.diff(idx) > 0)
    assert set(np.nonzero(prot)[0]) <= set(idx.tolist())
    kept_un = [i for i in idx if not prot[i]]
    drop_un = [i for i in range(n) if i not in set(idx.tolist()) and not prot[i]]
    assert min(s[kept_un]) >= max(s[drop_un])
    # equal keys straddling the cut: the kept ones have the lower indices
    thr = min(s[kept_un])
    kt = [i for i in kept_un if s[i] == thr]
    dt = [i for i in drop_un if s[i] == thr]
    if kt and dt:
        assert max(kt) < min(dt)
    # K = N keeps everything; P = K keeps exactly the protected tokens
    assert ref.topk_select(s, prot, n).tolist() == list(range(n))
    assert ref.topk_select(s, prot, 16).tolist() == list(range(n - 16, n))
    # all ties: the lowest indices win
    assert ref.topk_select(np.zeros(10, np.float32), None, 4).tolist() == [0, 1, 2, 3]
    # all -0/+0 mixed is one tie class
    z = _f32(["-0.0", 0.0, "-0.0", 0.0, "-0.0"])
    assert ref.topk_select(z, None, 2).tolist() == [0, 1]
    with pytest.raises(ref.BudgetError):
        ref.topk_select(s, prot, 15)  # P > K
    with pytest.raises(ref.BudgetError):
        ref.topk_select(s, prot, 0)
    with pytest.raises(ref.BudgetError):
        ref.topk_select(s, prot, n + 1)


def test_synthetic_tie_threshold_fixture():
    """The sweep's forced-tie case puts the K-th kept token inside the tie
    block; only the lowest-index members of the block survive."""
    import synth

    rng = synth.rng_for(5)
    n, k, p = 4096, 512, 128
    s = synth.scores_threshold_in_tie(n, k, p, rng)
    prot = synth.protect_tail(n, p)
    idx = ref.topk_select(s, prot, k)
    tie = np.nonzero(s == np.float32(0.5))[0]
    tie = tie[tie < n - p]
    kept_tie = sorted(set(idx.tolist()) & set(tie.tolist()))
    assert len(kept_tie) == 20 and kept_tie == tie[:20].tolist()


# ---------------------------------------------------------------- compact


def test_compact_is_a_gather():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((20, 5))
    s = rng.standard_normal(20).astype(np.float32)
    idx = np.array([1, 4, 5, 19], np.int32)
    xo, po, so = ref.compact(x, idx, None, s)
    for r, i in enumerate(idx):
        assert np.array_equal(xo[r], x[i]) and po[r] == i and so[r] == s[i]
    pos = np.arange(100, 120)
    _, po2, _ = ref.compact(x, idx, pos, None)
    assert po2.tolist() == [101, 104, 105, 119]


# ---------------------------------------------------------------- RoPE


def test_rope_relative_position_and_norm():
    rng = np.random.default_rng(9)
    dh = 16
    q = rng.standard_normal((1, 1, dh))
    k = rng.standard_normal((1, 1, dh))

    def dot_at(pq, pk):
        return float(np.sum(ref.rope(q, np.array([pq]), 1e4) * ref.rope(k, np.array([pk]), 1e4)))

    assert dot_at(7, 3) == pytest.approx(dot_at(104, 100), abs=1e-12)
    assert dot_at(50, 50) == pytest.approx(float(np.sum(q * k)), abs=1e-12)
    xr = ref.rope(q, np.array([12345]), 1e6)
    assert np.linalg.norm(xr) == pytest.approx(np.linalg.norm(q), rel=1e-14)
    assert np.allclose(ref.rope(q, np.array([0]), 1e6), q, atol=0)


def test_rope_two_dim_closed_form():
    # dh = 2: one pair, theta_0 = 1 -> a plain rotation by `pos` radians
    x = np.array([[[1.0, 0.0]]])
    got = ref.rope(x, np.array([3]), 1e6)[0, 0]
    assert np.allclose(got, [math.cos(3.0), math.sin(3.0)], atol=1e-15)


def test_rope_matches_transformers_rotary():
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb

    rng = np.random.default_rng(10)
    t, h, dh, base = 6, 2, 8, 1e6
    x = rng.standard_normal((t, h, dh))
    pos = np.array([0, 3, 7, 100, 1000, 131071])
    inv = 1.0 / (base ** (torch.arange(0, dh, 2, dtype=torch.float64) / dh))
    ang = torch.from_numpy(pos).double()[:, None] * inv[None, :]
    emb = torch.cat([ang, ang], dim=-1)
    cos, sin = emb.cos()[None], emb.sin()[None]
    tx = torch.from_numpy(x).permute(1, 0, 2)[None]  # [1, h, t, dh]
    want, _ = apply_rotary_pos_emb(tx, tx, cos, sin)
    want = want[0].permute(1, 0, 2).numpy()
    assert np.allclose(ref.rope(x, pos, base), want, atol=1e-12)


# ---------------------------------------------------------------- gated attention


def _qkv(seed, t=13, hq=4, hkv=2, dh=8):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((t, hq, dh)), rng.standard_normal((t, hkv, dh)),
            rng.standard_normal((t, hkv, dh)))


def _sdpa(q, k, v, scale=None, mask=None, causal=False):
    tq = torch.from_numpy(q).permute(1, 0, 2)[None]
    tk = torch.from_numpy(k).permute(1, 0, 2)[None]
    tv = torch.from_numpy(v).permute(1, 0, 2)[None]
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, attn_mask=mask, is_causal=causal, scale=scale, enable_gqa=True)
    return out[0].permute(1, 0, 2).numpy()


def test_gated_attention_reduces_to_causal_sdpa():
    q, k, v = _qkv(11)
    t = q.shape[0]
    got = ref.gated_attention(q, k, v, np.arange(t), None, None, None)
    assert np.allclose(got, _sdpa(q, k, v, causal=True), atol=1e-12)
    # K = N with gain 0 and tau 1 and any scores: still plain attention
    s = np.random.default_rng(1).standard_normal(t)
    got0 = ref.gated_attention(q, k, v, np.arange(t), s, np.zeros(4), np.ones(4))
    assert np.allclose(got0, _sdpa(q, k, v, causal=True), atol=1e-12)


def test_gated_attention_matches_sdpa_with_additive_bias():
    q, k, v = _qkv(12, t=17, hq=6, hkv=3, dh=16)
    t, hq, dh = q.shape
    rng = np.random.default_rng(2)
    s = rng.standard_normal(t) * 3
    gain = rng.uniform(0, 2, hq)
    tau = rng.uniform(0.5, 1.5, hq)
    pos = np.sort(rng.choice(1000, t, replace=False))
    got = ref.gated_attention(q, k, v, pos, s, gain, tau)
    causal = torch.from_numpy(pos[None, :] <= pos[:, None])
    lsig = torch.nn.functional.logsigmoid(torch.from_numpy(s))
    for h in range(hq):
        mask = torch.where(causal, gain[h] * lsig[None, :], torch.tensor(-math.inf,
                           dtype=torch.float64))
        g = h // (hq // 3)
        want = _sdpa(q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1],
                     scale=1.0 / (math.sqrt(dh) * tau[h]), mask=mask)
        assert np.allclose(got[:, h], want[:, 0], atol=1e-12), h


def test_gated_attention_constant_scores_shift_invariance():
    q, k, v = _qkv(13)
    t = q.shape[0]
    tau = np.array([0.6, 0.9, 1.2, 1.4])
    a = ref.gated_attention(q, k, v, np.arange(t), np.full(t, -1.3), np.full(4, 1.7), tau)
    b = ref.gated_attention(q, k, v, np.arange(t), None, None, tau)
    assert np.allclose(a, b, atol=1e-12)


def test_gated_attention_gain_one_is_multiplicative_sigmoid():
    q, k, v = _qkv(14, t=9, hq=2, hkv=1, dh=4)
    t, hq, dh = q.shape
    s = np.random.default_rng(3).standard_normal(t) * 2
    tau = np.array([0.7, 1.3])
    got = ref.gated_attention(q, k, v, np.arange(t), s, np.ones(hq), tau)
    for h in range(hq):
        for i in range(t):
            w = np.array([(1.0 / (1.0 + math.exp(-s[j]))) *
                          math.exp(float(q[i, h] @ k[j, 0]) / (math.sqrt(dh) * tau[h]))
                          for j in range(i + 1)])
            o = (w[:, None] * v[: i + 1, 0]).sum(0) / w.sum()
            assert np.allclose(got[i, h], o, atol=1e-12)


def test_gated_attention_tau_equals_scaling_q_and_first_row():
    q, k, v = _qkv(15)
    t = q.shape[0]
    tau = np.array([0.5, 0.8, 1.1, 1.5])
    a = ref.gated_attention(q, k, v, np.arange(t), None, None, tau)
    b = ref.gated_attention(q / tau[None, :, None], k, v, np.arange(t), None, None, None)
    assert np.allclose(a, b, atol=1e-12)
    # the first kept row sees only itself: o_0 = v_0 of its KV head
    assert np.allclose(a[0, 0], v[0, 0]) and np.allclose(a[0, 3], v[0, 1])


def test_gated_attention_causal_by_original_position():
    # ascending distinct positions: masking by position = masking by row index
    q, k, v = _qkv(16)
    t = q.shape[0]
    pos = np.cumsum(np.random.default_rng(4).integers(1, 50, t))
    assert np.allclose(ref.gated_attention(q, k, v, pos, None, None, None),
                       ref.gated_attention(q, k, v, np.arange(t), None, None, None), atol=1e-13)


# ---------------------------------------------------------------- gated attention backward


def _bwd_case(seed, t=6, hq=4, hkv=2, dh=8):
    rng = np.random.default_rng(seed)
    q, k, v = _qkv(seed, t=t, hq=hq, hkv=hkv, dh=dh)
    pos = np.sort(rng.choice(60, t, replace=False))
    s = rng.standard_normal(t) * 2
    gain = rng.uniform(0.2, 2.0, hq)
    tau = rng.uniform(0.5, 1.5, hq)
    dout = rng.standard_normal((t, hq, dh))
    return q, k, v, pos, s, gain, tau, dout


def test_attention_backward_matches_finite_differences():
    # Central differences of the (separately pinned) fp64 forward, RoPE
    # included, for every input element: a dropped term, a wrong sign or a
    # transposed operand anywhere in the backward fails here.
    q, k, v, pos, s, gain, tau, dout = _bwd_case(21)
    base = 1e4
    ident = ref.identity

    def loss(q_, k_, v_, s_, g_, t_):
        o = ref.gated_attn_prefill(q_, k_, v_, pos, s_, g_, t_, base, store=ident)
        return float((o * dout).sum())

    args = [q, k, v, s, gain, tau]
    got = ref.gated_attn_backward(q, k, v, pos, s, gain, tau, base, dout, store=ident)
    eps = 1e-6
    for a_idx, g in enumerate(got):
        fd = np.zeros_like(args[a_idx])
        flat = fd.reshape(-1)
        for e in range(flat.size):
            plus = [x.copy() for x in args]
            minus = [x.copy() for x in args]
            plus[a_idx].reshape(-1)[e] += eps
            minus[a_idx].reshape(-1)[e] -= eps
            flat[e] = (loss(*plus) - loss(*minus)) / (2 * eps)
        assert np.allclose(g, fd, rtol=1e-6, atol=1e-7), a_idx


def test_attention_backward_matches_torch_autograd():
    # torch autograd through SDPA with the gate bias as an additive mask and
    # tau folded into q (fp64 on the CPU): a library derivative of the same
    # forward, for all six gradients.
    q, k, v, pos, s, gain, tau, dout = _bwd_case(22, t=11, hq=6, hkv=3, dh=16)
    t, hq, dh = q.shape
    got = ref.gated_attention_grads(q, k, v, pos, s, gain, tau, dout)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    ts, tg, tt = (torch.tensor(x, requires_grad=True) for x in (s, gain, tau))
    causal = torch.from_numpy(pos[None, :] <= pos[:, None])
    lsig = torch.nn.functional.logsigmoid(ts)
    outs = []
    for h in range(hq):
        g = h // (hq // 3)
        mask = torch.where(causal, tg[h] * lsig[None, :],
                           torch.tensor(-math.inf, dtype=torch.float64))
        qh = tq[:, h] / tt[h]  # [t, dh]
        o = torch.nn.functional.scaled_dot_product_attention(
            qh[None, None], tk[:, g][None, None], tv[:, g][None, None], attn_mask=mask,
            scale=1.0 / math.sqrt(dh))
        outs.append(o[0, 0])
    out = torch.stack(outs, dim=1)
    (out * torch.from_numpy(dout)).sum().backward()
    for mine, theirs in zip(got, (tq.grad, tk.grad, tv.grad, ts.grad, tg.grad, tt.grad)):
        assert np.allclose(mine, theirs.numpy(), rtol=1e-9, atol=1e-11)


def test_attention_lse_closed_forms():
    q, k, v, pos, s, gain, tau, dout = _bwd_case(24, t=10)
    # q = 0 and no bias: every visible logit is 0, so lse_i = log(i + 1)
    lse0 = ref.gated_attention_lse(np.zeros_like(q), k, pos, None, gain, tau)
    assert np.allclose(lse0, np.log(np.arange(1, 11))[None, :], atol=1e-14)
    # q = 0 with the bias: lse_i = log sum_{j <= i} sigmoid(s_j)^gain_h
    lse1 = ref.gated_attention_lse(np.zeros_like(q), k, pos, s, gain, tau)
    sig = 1.0 / (1.0 + np.exp(-s))
    want = np.log(np.cumsum(sig[None, :] ** gain[:, None], axis=1))
    assert np.allclose(lse1, want, atol=1e-13)
    # the first row sees only itself: lse_0 = l_00
    lse = ref.gated_attention_lse(q, k, pos, s, gain, tau)
    for h in range(4):
        l00 = q[0, h] @ k[0, h // 2] / (math.sqrt(8) * tau[h]) + gain[h] * math.log(sig[0])
        assert lse[h, 0] == pytest.approx(l00, abs=1e-13)


def test_attention_backward_invariants_and_degenerate_cases():
    q, k, v, pos, s, gain, tau, dout = _bwd_case(23, t=9)
    # constant scores: each head's key sums of dl vanish (softmax rows sum to
    # one), so sum_j ds_j = 0 and dgain = 0
    sc = np.full(len(pos), 0.7)
    _, _, _, ds, dgain, _ = ref.gated_attention_grads(q, k, v, pos, sc, gain, tau, dout)
    assert abs(ds.sum()) < 1e-12 and np.all(np.abs(dgain) < 1e-12)
    # tau divides the q.k term only: dtau_h = -(1/tau_h) sum_i q_i . dq_i
    dq, _, _, _, _, dtau = ref.gated_attention_grads(q, k, v, pos, s, gain, tau, dout)
    assert np.allclose(dtau, -np.einsum("thd,thd->h", q, dq) / tau, atol=1e-12)
    # no bias: nothing flows to s, and gain has no effect
    _, _, _, ds0, dgain0, _ = ref.gated_attention_grads(q, k, v, pos, None, gain, tau, dout)
    assert ds0 is None and np.all(dgain0 == 0.0)
    # one token: o_0 = v_0, so dv_0 = sum over the group of dout_0 and all
    # other gradients are zero
    dq1, dk1, dv1, ds1, dg1, dt1 = ref.gated_attention_grads(
        q[:1], k[:1], v[:1], pos[:1], s[:1], gain, tau, dout[:1])
    assert np.allclose(dv1[0, 0], dout[0, 0] + dout[0, 1]) and np.allclose(dv1[0, 1],
                                                                           dout[0, 2] + dout[0, 3])
    for z in (dq1, dk1, ds1, dg1, dt1):
        assert np.all(np.abs(z) < 1e-12)


# ---------------------------------------------------------------- full stack


def _tiny_model(seed, qk_norm, n_layers=3, d=64, hq=4, hkv=2, dh=16, inter=96, f=8):
    rng = np.random.default_rng(seed)
    layers = []
    for _ in range(n_layers):
        layers.append(ref.Layer(
            attn_norm=rng.uniform(0.5, 1.5, d), wqkv=rng.standard_normal(((hq + 2 * hkv) * dh, d)) * 0.1,
            wo=rng.standard_normal((d, hq * dh)) * 0.1, ffn_norm=rng.uniform(0.5, 1.5, d),
            w_gate_up=rng.standard_normal((2 * inter, d)) * 0.1,
            w_down=rng.standard_normal((d, inter)) * 0.1,
            q_norm=rng.uniform(0.5, 1.5, dh) if qk_norm else None,
            k_norm=rng.uniform(0.5, 1.5, dh) if qk_norm else None))
    return ref.Model(d_model=d, n_heads_q=hq, n_heads_kv=hkv, head_dim=dh, layers=layers,
                     final_norm=rng.uniform(0.5, 1.5, d), score_norm=np.ones(d),
                     score_w1=rng.standard_normal((f, d)), score_b1=None,
                     score_w2=rng.standard_normal(f), score_b2=None, eps=1e-6, rope_base=1e6)


def _hf_model(m: ref.Model, qk_norm: bool):
    """The same weights in a Hugging Face Qwen3 (qk-norm) or Llama model."""
    from transformers import LlamaConfig, LlamaModel, Qwen3Config, Qwen3Model

    d, hq, hkv, dh = m.d_model, m.n_heads_q, m.n_heads_kv, m.head_dim
    inter = m.layers[0].w_gate_up.shape[0] // 2
    common = dict(vocab_size=8, hidden_size=d, intermediate_size=inter,
                  num_hidden_layers=len(m.layers), num_attention_heads=hq,
                  num_key_value_heads=hkv, head_dim=dh, rms_norm_eps=m.eps,
                  max_position_embeddings=4096, attention_bias=False, hidden_act="silu")
    if qk_norm:
        cfg = Qwen3Config(rope_theta=m.rope_base, **common)
        cfg.rope_parameters = {"rope_type": "default", "rope_theta": m.rope_base}
        model = Qwen3Model(cfg)
    else:
        cfg = LlamaConfig(rope_theta=m.rope_base, mlp_bias=False, **common)
        cfg.rope_parameters = {"rope_type": "default", "rope_theta": m.rope_base}
        model = LlamaModel(cfg)
    cfg._attn_implementation = "eager"
    model = model.double().eval()
    T = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float64))
    with torch.no_grad():
        for lw, hl in zip(m.layers, model.layers):
            a = hl.self_attn
            a.q_proj.weight.copy_(T(lw.wqkv[: hq * dh]))
            a.k_proj.weight.copy_(T(lw.wqkv[hq * dh: (hq + hkv) * dh]))
            a.v_proj.weight.copy_(T(lw.wqkv[(hq + hkv) * dh:]))
            a.o_proj.weight.copy_(T(lw.wo))
            if qk_norm:
                a.q_norm.weight.copy_(T(lw.q_norm))
                a.k_norm.weight.copy_(T(lw.k_norm))
            hl.input_layernorm.weight.copy_(T(lw.attn_norm))
            hl.post_attention_layernorm.weight.copy_(T(lw.ffn_norm))
            hl.mlp.gate_proj.weight.copy_(T(lw.w_gate_up[:inter]))
            hl.mlp.up_proj.weight.copy_(T(lw.w_gate_up[inter:]))
            hl.mlp.down_proj.weight.copy_(T(lw.w_down))
        model.norm.weight.copy_(T(m.final_norm))
    return model


@pytest.mark.parametrize("qk_norm", [True, False])
@pytest.mark.parametrize("gate_layer", [0, 1, -1])
def test_dense_stack_matches_transformers(qk_norm, gate_layer):
    """K = N with gain 0 and tau 1 is a plain decoder stack: the oracle's
    gated prefill must equal a Qwen3 (qk-norm) / Llama model's forward."""
    m = _tiny_model(20 + qk_norm, qk_norm)
    n = 21
    x = np.random.default_rng(5).standard_normal((n, m.d_model))
    res = ref.prefill(x, ref_protect(n, 3), n, m, gate_layer, store=ref.identity)
    assert res.kept_idx.tolist() == list(range(n))
    hf = _hf_model(m, qk_norm)
    with torch.no_grad():
        out = hf(inputs_embeds=torch.from_numpy(x)[None]).last_hidden_state[0].numpy()
    # transformers evaluates RMSNorm and the rotary tables in float32 even in
    # a float64 model, so agreement is at float32 level (measured ~5e-7 on
    # values up to ~5); a wrong sign, index or operand would differ by O(0.1).
    assert np.allclose(res.out, out, rtol=0, atol=2e-6)
    # KV rows: N at or below the gate; above it K (= N here)
    assert all(kk.shape[0] == n for kk, _ in res.kv)


def ref_protect(n, p):
    m = np.zeros(n, np.uint8)
    m[n - p:] = 1
    return m


def test_folded_norm_projection():
    """R7b: (x / rms(x)) . (W diag g)^T is RMSNorm(x; g) . W^T. In exact
    arithmetic the two forms agree to rounding; with bf16 storage the folded
    form rounds W g instead of the normed rows, so the two differ by at most
    one bf16 rounding of either operand, and the folded form keeps RMSNorm's
    scale invariance."""
    rng = np.random.default_rng(41)
    x = rng.standard_normal((9, 64)) * rng.uniform(0.1, 10, (9, 1))
    g = rng.uniform(0.2, 3.0, 64)
    w = rng.standard_normal((24, 64)) * 0.1
    a = ref.norm_project(x, g, w, 1e-6, ref.identity, fold=True)
    b = ref.norm_project(x, g, w, 1e-6, ref.identity, fold=False)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-13)
    assert np.allclose(b, ref.rmsnorm(x, g, 1e-6) @ w.T, rtol=1e-12, atol=1e-13)
    af = ref.norm_project(x, g, w, 0.0, ref.round_bf16, fold=True)
    bf = ref.norm_project(x, g, w, 0.0, ref.round_bf16, fold=False)
    mag = np.abs(ref.rmsnorm(x, g, 0.0)) @ np.abs(w).T
    assert np.all(np.abs(af - a) <= 2.0 ** -8 * mag + 1e-12)
    assert np.all(np.abs(bf - a) <= 2.0 ** -8 * mag + 1e-12)
    assert np.allclose(ref.norm_project(7.0 * x, g, w, 0.0, ref.round_bf16, fold=True), af,
                       rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("gate_layer", [1, -1])
def test_prefill_with_folded_norms_is_the_same_map(gate_layer):
    """R7b only moves rounding points: with exact storage the folded-norm
    forward equals the plain one, for an attention stack and a hybrid one."""
    from oracle import gated_deltanet_oracle as gdn
    m = _tiny_model(33, True, n_layers=3)
    rng = np.random.default_rng(8)
    for lw in m.layers:
        lw.gain = rng.uniform(0, 2, m.n_heads_q)
        lw.tau = rng.uniform(0.5, 1.5, m.n_heads_q)
    n, k = 30, 11
    x = rng.standard_normal((n, m.d_model))
    prot = ref_protect(n, 3)
    a = ref.prefill(x, prot, k, m, gate_layer, store=ref.identity, fold_norms=True)
    b = ref.prefill(x, prot, k, m, gate_layer, store=ref.identity)
    assert np.array_equal(a.kept_idx, b.kept_idx)
    assert np.allclose(a.out, b.out, rtol=0, atol=1e-10)
    assert np.allclose(a.scores, b.scores, rtol=0, atol=1e-6)
    c = gdn.hybrid_prefill(x, prot, k, m, gate_layer, store=ref.identity, fold_norms=True)
    assert np.array_equal(c.kept_idx, b.kept_idx)
    assert np.allclose(c.out, b.out, rtol=0, atol=1e-10)


def test_pruned_tokens_make_no_upper_kv_and_kept_set_drives_upper_layers():
    m = _tiny_model(30, True, n_layers=4)
    rng = np.random.default_rng(6)
    for lw in m.layers:
        lw.gain = rng.uniform(0, 2, m.n_heads_q)
        lw.tau = rng.uniform(0.5, 1.5, m.n_heads_q)
    n, k, L = 40, 12, 1
    x = rng.standard_normal((n, m.d_model))
    prot = ref_protect(n, 4)
    res = ref.prefill(x, prot, k, m, L, store=ref.identity)
    assert res.kept_idx.size == k and set(range(n - 4, n)) <= set(res.kept_idx.tolist())
    assert [kk.shape[0] for kk, _ in res.kv] == [n, n, k, k]
    # the upper layers see only the kept rows: rerunning them from the compacted
    # residual reproduces the output, and upper KV rows are projections of it
    x_all = x
    h = x_all
    pos = np.arange(n)
    r0, _ = ref.attention_sublayer(h, m.layers[0], m, pos, None, None, None, ref.identity)
    h = ref.ffn_sublayer(r0, m.layers[0], m, ref.identity)
    r1, _ = ref.attention_sublayer(h, m.layers[1], m, pos, None, None, None, ref.identity)
    xk, pk, sk = ref.compact(r1, res.kept_idx, pos, res.scores.astype(np.float64))
    h = ref.ffn_sublayer(xk, m.layers[1], m, ref.identity)
    for li in (2, 3):
        h, kv = ref.gated_layer_forward(h, pk, sk, m.layers[li], m, ref.identity)
        assert np.allclose(kv[0], res.kv[li][0])
    assert np.allclose(ref.rmsnorm(h, m.final_norm, m.eps), res.out, atol=1e-12)


def test_budgets_nest_and_share_the_below_gate_pass():
    # one request at several budgets: the scores do not depend on k, the kept
    # sets nest (a larger budget keeps every token a smaller one keeps: the
    # ranking is the same), the protected tokens are in every set, and K = N
    # keeps everything
    m = _tiny_model(31, qk_norm=True, n_layers=3)
    n = 40
    rng = np.random.default_rng(32)
    x = rng.standard_normal((n, m.d_model))
    prot = ref_protect(n, 4)
    ks = [6, 13, 27, n]
    res = ref.prefill_budgets(x, prot, ks, m, 1)
    for r in res[1:]:
        assert np.array_equal(r.scores, res[0].scores)
    for a, b in zip(res, res[1:]):
        assert set(a.kept_idx.tolist()) <= set(b.kept_idx.tolist())
    for r in res:
        assert set(np.nonzero(prot)[0].tolist()) <= set(r.kept_idx.tolist())
    assert res[-1].kept_idx.tolist() == list(range(n))
    # the budget-independent part (layers below the gate, the gate layer's
    # attention) gives every budget the same below-gate KV
    for r in res[1:]:
        for (k0, v0), (k1, v1) in zip(res[0].kv[:2], r.kv[:2]):
            assert np.array_equal(k0, k1) and np.array_equal(v0, v1)


def test_work_counts():
    assert ref.attention_flops(2048, 16, 128) == pytest.approx(17.19e9, rel=1e-3)
    assert ref.select_compact_bytes(131072, 65536, 2048) == pytest.approx(538e6, rel=2e-3)


# ---------------------------------------------------------------- decode step


def _hf_cache(kv):
    from transformers import DynamicCache

    cache = DynamicCache()
    for li, (k, v) in enumerate(kv):
        cache.update(torch.from_numpy(np.ascontiguousarray(k)).permute(1, 0, 2)[None].contiguous(),
                     torch.from_numpy(np.ascontiguousarray(v)).permute(1, 0, 2)[None].contiguous(),
                     li)
    return cache


@pytest.mark.parametrize("store", [ref.identity, ref.round_bf16])
def test_decode_step_equals_prefill_of_one_more_token(store):
    """Incremental decoding is full recomputation: with every layer at or
    below the gate (K = N), prefilling N tokens and decoding token N gives
    token N's row of a prefill over N + 1 tokens, and the decoded k/v rows
    are that prefill's last cache rows."""
    m = _tiny_model(40, True, n_layers=3)
    n, last = 17, 2
    x = np.random.default_rng(7).standard_normal((n + 1, m.d_model))
    res = ref.prefill(x[:n], ref_protect(n, 3), n, m, last, store=store)
    out, new_kv = ref.decode_step(x[n], n, m, last, res.kv, None, store=store)
    full = ref.prefill(x, ref_protect(n + 1, 3), n + 1, m, last, store=store)
    tol = 1e-12 if store is ref.identity else 0.0
    assert np.max(np.abs(out - full.out[-1])) <= tol
    for (k_new, v_new), (k_full, v_full) in zip(new_kv, full.kv):
        assert np.max(np.abs(k_new - k_full[-1])) <= tol
        assert np.max(np.abs(v_new - v_full[-1])) <= tol


@pytest.mark.parametrize("qk_norm", [True, False])
def test_decode_step_matches_transformers_kv_cache(qk_norm):
    """The oracle's decode over a prefill's cache against a Hugging Face
    model stepping one token with the same cache (past_key_values)."""
    m = _tiny_model(41 + qk_norm, qk_norm, n_layers=3)
    n = 15
    x = np.random.default_rng(8).standard_normal((n + 1, m.d_model))
    res = ref.prefill(x[:n], ref_protect(n, 2), n, m, len(m.layers) - 1, store=ref.identity)
    out, _ = ref.decode_step(x[n], n, m, len(m.layers) - 1, res.kv, None, store=ref.identity)
    hf = _hf_model(m, qk_norm)
    with torch.no_grad():
        o = hf(inputs_embeds=torch.from_numpy(x[n:n + 1])[None], past_key_values=_hf_cache(res.kv),
               position_ids=torch.tensor([[n]]), use_cache=True).last_hidden_state[0, -1].numpy()
    assert np.allclose(out, o, rtol=0, atol=2e-6)  # float32-level, as the prefill pin


def test_decode_gate_bias_matches_transformers_additive_mask():
    """Above the gate, the kept prompt keys carry gain * logsigmoid(s_j) and
    the generated token's own key carries none: with one gain for every head
    and layer and tau = 1 that is an additive attention mask, which a Hugging
    Face model applies to the logits as given."""
    m = _tiny_model(43, True, n_layers=3)
    rng = np.random.default_rng(9)
    gain = 0.7
    for lw in m.layers:
        lw.gain = np.full(m.n_heads_q, gain)
        lw.tau = np.ones(m.n_heads_q)
    n, k = 15, 7
    x = rng.standard_normal((n + 1, m.d_model))
    res = ref.prefill(x[:n], ref_protect(n, 2), n, m, len(m.layers) - 1, store=ref.identity)
    kept = np.sort(rng.choice(n, k, replace=False))
    kv = [(kk[kept], vv[kept]) for kk, vv in res.kv]  # every layer above the gate
    ks = rng.standard_normal(k) * 2
    out, _ = ref.decode_step(x[n], n, m, -1, kv, ks, store=ref.identity)
    mask = np.concatenate([gain * np.log(1.0 / (1.0 + np.exp(-ks))), [0.0]])
    hf = _hf_model(m, True)
    with torch.no_grad():
        o = hf(inputs_embeds=torch.from_numpy(x[n:n + 1])[None], past_key_values=_hf_cache(kv),
               position_ids=torch.tensor([[n]]), attention_mask=torch.from_numpy(mask)[None, None, None],
               use_cache=True).last_hidden_state[0, -1].numpy()
    assert np.allclose(out, o, rtol=0, atol=2e-6)
    # and the bias matters: without it the output moves by O(0.1)
    plain, _ = ref.decode_step(x[n], n, m, -1, kv, np.full(k, np.inf), store=ref.identity)
    assert np.max(np.abs(plain - out)) > 1e-2
