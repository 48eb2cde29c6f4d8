"""Pins of the Gated DeltaNet oracle to facts outside it.

Each test checks the oracle against something it does not compute itself: a
closed form of a special case, a library routine, automatic differentiation,
the whole-sequence solution of the recurrence by one triangular solve, or an
invariant (splitting a sequence across calls). A plausible slip (a
transposed state, a decay applied to the wrong term, an off-by-one in the
convolution window, a wrong head mapping) fails at least one of them.
"""

import numpy as np
import pytest
import scipy.signal
import torch

from oracle import gated_deltanet_oracle as gdn

RNG = np.random.default_rng(1234)


def _orthonormal(n, d, rng):
    q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    return q[:n]


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_write_with_full_strength_is_read_back_exactly():
    # beta = 1 and a unit key: S_t k_t = alpha S(k - k k^T k) + v = v, whatever
    # the decay and the previous state; so querying with the key just written
    # returns its value.
    T, H, dk, dv = 9, 2, 16, 8
    k = _unit(RNG.standard_normal((T, H, dk)))
    v = RNG.standard_normal((T, H, dv))
    g = -RNG.uniform(0, 1, (T, H))
    beta = np.ones((T, H))
    S0 = RNG.standard_normal((H, dv, dk))
    o, _ = gdn.gated_delta_rule(k, k, v, g, beta, S0)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


def test_recall_with_orthonormal_keys():
    # No decay, full strength, orthonormal keys: the state is sum_j v_j k_j^T
    # and reads each stored value back exactly.
    T, dk, dv = 12, 16, 5
    K = _orthonormal(T, dk, RNG)
    V = RNG.standard_normal((T, dv))
    _, S = gdn.gated_delta_rule(K[:, None], K[:, None], V[:, None], np.zeros((T, 1)),
                                np.ones((T, 1)))
    np.testing.assert_allclose(S[0], V.T @ K, atol=1e-12)
    np.testing.assert_allclose(S[0] @ K.T, V.T, atol=1e-12)


def test_orthogonal_keys_reduce_to_gated_linear_attention():
    # With mutually orthogonal keys the correction term S_{t-1} k_t vanishes,
    # so o_t = sum_{j<=t} exp(G_t - G_j) beta_j (k_j . q_t) v_j with G the
    # running sum of g: a masked quadratic form computed here with matrices.
    T, dk, dv = 10, 16, 6
    K = _orthonormal(T, dk, RNG)
    Q = RNG.standard_normal((T, dk))
    V = RNG.standard_normal((T, dv))
    g = -RNG.uniform(0.0, 0.7, T)
    beta = RNG.uniform(0.1, 1.0, T)
    G = np.cumsum(g)
    D = np.tril(np.exp(G[:, None] - G[None, :]))
    want = (D * (Q @ K.T) * beta[None, :]) @ V
    o, _ = gdn.gated_delta_rule(Q[:, None], K[:, None], V[:, None], g[:, None], beta[:, None])
    np.testing.assert_allclose(o[:, 0], want, rtol=1e-12, atol=1e-12)


def test_update_is_one_gradient_step_on_the_recall_loss():
    # The delta rule is one step of size beta on 0.5 |S' k - v|^2 from the
    # decayed state S' = alpha S: the gradient comes from autograd here.
    dk, dv = 12, 7
    S0 = RNG.standard_normal((1, dv, dk))
    k = _unit(RNG.standard_normal((1, 1, dk)))
    v = RNG.standard_normal((1, 1, dv))
    g, beta = np.array([[-0.3]]), np.array([[0.45]])
    _, S1 = gdn.gated_delta_rule(np.zeros((1, 1, dk)), k, v, g, beta, S0)
    Sp = torch.tensor(np.exp(-0.3) * S0[0], dtype=torch.float64, requires_grad=True)
    loss = 0.5 * ((Sp @ torch.tensor(k[0, 0]) - torch.tensor(v[0, 0])) ** 2).sum()
    loss.backward()
    want = (Sp - 0.45 * Sp.grad).detach().numpy()
    np.testing.assert_allclose(S1[0], want, rtol=1e-12, atol=1e-12)


def test_zero_strength_only_decays_the_state():
    T, H, dk, dv = 7, 3, 8, 4
    q = RNG.standard_normal((T, H, dk))
    k = _unit(RNG.standard_normal((T, H, dk)))
    v = RNG.standard_normal((T, H, dv))
    g = -RNG.uniform(0, 0.5, (T, H))
    S0 = RNG.standard_normal((H, dv, dk))
    o, S = gdn.gated_delta_rule(q, k, v, g, np.zeros((T, H)), S0)
    G = np.cumsum(g, axis=0)
    want = np.exp(G)[:, :, None] * np.einsum("hij,thj->thi", S0, q)
    np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, np.exp(G[-1])[:, None, None] * S0, rtol=1e-12)


def _chunk_solution(q, k, v, g, beta, S0):
    """The recurrence of one head solved for a whole sequence at once: with
    G the running sum of g and d_t = beta_t (v_t - alpha_t S_{t-1} k_t), the
    d_t satisfy (I + A) D = diag(beta) (V - diag(e^G) K S0^T), where
    A_tj = beta_t e^(G_t - G_j) (k_t . k_j) for j < t; then
    o_t = e^G_t S0 q_t + sum_{j<=t} e^(G_t - G_j) (k_j . q_t) d_j."""
    G = np.cumsum(g)
    E = np.exp(G[:, None] - G[None, :])
    A = np.tril(beta[:, None] * E * (k @ k.T), -1)
    rhs = beta[:, None] * (v - np.exp(G)[:, None] * (k @ S0.T))
    D = np.linalg.solve(np.eye(len(g)) + A, rhs)
    o = np.exp(G)[:, None] * (q @ S0.T) + (np.tril(E) * (q @ k.T)) @ D
    S = np.exp(G[-1]) * S0 + (np.exp(G[-1] - G)[:, None] * D).T @ k
    return o, S


def test_recurrence_equals_the_whole_sequence_solution():
    T, dk, dv = 40, 16, 12
    q = RNG.standard_normal((T, dk))
    k = _unit(RNG.standard_normal((T, dk)))
    v = RNG.standard_normal((T, dv))
    g = -RNG.uniform(0.0, 0.4, T)
    beta = RNG.uniform(0.0, 1.0, T)
    S0 = RNG.standard_normal((dv, dk))
    want_o, want_S = _chunk_solution(q, k, v, g, beta, S0)
    o, S = gdn.gated_delta_rule(q[:, None], k[:, None], v[:, None], g[:, None], beta[:, None],
                                S0[None])
    np.testing.assert_allclose(o[:, 0], want_o, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(S[0], want_S, rtol=1e-10, atol=1e-10)


def test_convolution_matches_a_library_filter():
    T, C, W = 23, 5, 4
    x = RNG.standard_normal((T, C))
    w = RNG.standard_normal((C, W))
    prev = RNG.standard_normal((W - 1, C))
    y, state = gdn.causal_conv_silu(x, w, prev)
    xx = np.concatenate([prev, x])
    for c in range(C):
        pre = scipy.signal.lfilter(w[c, ::-1], [1.0], xx[:, c])[W - 1:]
        np.testing.assert_allclose(y[:, c], pre / (1.0 + np.exp(-pre)), rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(state, xx[-(W - 1):])
    # no carried rows = zeros before the first token
    y0, _ = gdn.causal_conv_silu(x, w)
    pre0 = scipy.signal.lfilter(w[0, ::-1], [1.0], x[:, 0])
    np.testing.assert_allclose(y0[:, 0], pre0 / (1.0 + np.exp(-pre0)), rtol=1e-12, atol=1e-12)
    # fewer tokens than the window: the state keeps older carried rows
    _, st2 = gdn.causal_conv_silu(x[:1], w, prev)
    np.testing.assert_array_equal(st2, np.concatenate([prev[1:], x[:1]]))


def test_decay_strength_and_norm_closed_forms():
    g, beta = gdn.decay_and_strength(np.array([[0.0, 50.0]]), np.array([[0.0, -3.0]]),
                                     np.array([0.0, np.log(2.0)]), np.array([0.0, 0.0]))
    np.testing.assert_allclose(g[0, 0], -np.log(2.0), rtol=1e-15)   # alpha = 1/2
    np.testing.assert_allclose(g[0, 1], -2.0 * (50.0 + np.log1p(np.exp(-50.0))), rtol=1e-15)
    np.testing.assert_allclose(beta[0], [0.5, 1.0 / (1.0 + np.exp(3.0))], rtol=1e-15)
    x = RNG.standard_normal((4, 64)) * 10
    np.testing.assert_allclose(gdn.l2_normalize(x, 0.0), x / np.linalg.norm(x, axis=1)[:, None],
                               rtol=1e-14)
    # RMSNorm of a constant vector c is sign(c) / sqrt(1 + eps / c^2)
    c, eps = -0.25, 1e-3
    y = gdn.gated_rmsnorm(np.full((1, 8), c), np.full((1, 8), 40.0), np.full(8, 2.0), eps)
    np.testing.assert_allclose(y, -2.0 * 40.0 / (1 + np.exp(-40.0)) / np.sqrt(1 + eps / c**2),
                               rtol=1e-14)
    assert np.all(gdn.gated_rmsnorm(np.ones((1, 4)), np.zeros((1, 4)), np.ones(4), eps) == 0)


def _mixer_inputs(T, hk, hv, dk, dv, W, rng):
    C = 2 * hk * dk + hv * dv
    qkv = rng.standard_normal((T, C))
    z = rng.standard_normal((T, hv * dv))
    a = rng.standard_normal((T, hv))
    b = rng.standard_normal((T, hv))
    p = gdn.MixerParams(conv_w=rng.standard_normal((C, W)) * 0.5,
                        A_log=np.log(rng.uniform(1, 16, hv)), dt_bias=rng.standard_normal(hv) * 0.5,
                        norm_w=rng.uniform(0.5, 1.5, dv), eps=1e-6)
    return qkv, z, a, b, p


def test_split_calls_with_carried_state_equal_one_call():
    T, hk, hv, dk, dv, W = 19, 1, 2, 8, 6, 4
    qkv, z, a, b, p = _mixer_inputs(T, hk, hv, dk, dv, W, RNG)
    ident = lambda x: np.asarray(x, dtype=np.float64)
    full = gdn.gated_deltanet(qkv, z, a, b, p, hk, hv, dk, dv, store=ident)
    for cut in (1, 2, 11):
        r1 = gdn.gated_deltanet(qkv[:cut], z[:cut], a[:cut], b[:cut], p, hk, hv, dk, dv,
                                store=ident)
        r2 = gdn.gated_deltanet(qkv[cut:], z[cut:], a[cut:], b[cut:], p, hk, hv, dk, dv,
                                conv_state=r1.conv_state, S0=r1.S, store=ident)
        np.testing.assert_allclose(np.concatenate([r1.y, r2.y]), full.y, rtol=1e-6, atol=1e-7)
        np.testing.assert_array_equal(r2.conv_state, full.conv_state)


def test_head_mapping_and_per_head_sampling():
    # Value heads 2h and 2h+1 read key head h: swapping the two value heads'
    # channels (v, z, a, b) swaps their outputs. The per-head sampler, which
    # slices the inputs its own way, agrees with the whole mixer.
    T, hk, hv, dk, dv, W = 13, 2, 4, 8, 4, 4
    qkv, z, a, b, p = _mixer_inputs(T, hk, hv, dk, dv, W, RNG)
    p.A_log = np.full(hv, 0.3)
    p.dt_bias = np.full(hv, -0.2)
    ident = lambda x: np.asarray(x, dtype=np.float64)
    base = gdn.gated_deltanet(qkv, z, a, b, p, hk, hv, dk, dv, store=ident)
    perm = np.array([1, 0, 2, 3])
    vcols = 2 * hk * dk + np.concatenate([np.arange(h * dv, (h + 1) * dv) for h in perm])
    qkv2 = qkv.copy()
    qkv2[:, 2 * hk * dk:] = qkv[:, vcols]
    p2 = gdn.MixerParams(conv_w=p.conv_w.copy(), A_log=p.A_log, dt_bias=p.dt_bias,
                         norm_w=p.norm_w, eps=p.eps)
    p2.conv_w[2 * hk * dk:] = p.conv_w[vcols]
    z2 = z.reshape(T, hv, dv)[:, perm].reshape(T, -1)
    sw = gdn.gated_deltanet(qkv2, z2, a[:, perm], b[:, perm], p2, hk, hv, dk, dv, store=ident)
    np.testing.assert_allclose(sw.y.reshape(T, hv, dv), base.y.reshape(T, hv, dv)[:, perm],
                               rtol=1e-12, atol=1e-12)
    # moving a value head to the other key group changes its output
    perm_x = np.array([2, 1, 0, 3])
    vcols_x = 2 * hk * dk + np.concatenate([np.arange(h * dv, (h + 1) * dv) for h in perm_x])
    qkv3 = qkv.copy()
    qkv3[:, 2 * hk * dk:] = qkv[:, vcols_x]
    p3 = gdn.MixerParams(conv_w=p.conv_w.copy(), A_log=p.A_log, dt_bias=p.dt_bias,
                         norm_w=p.norm_w, eps=p.eps)
    p3.conv_w[2 * hk * dk:] = p.conv_w[vcols_x]
    z3 = z.reshape(T, hv, dv)[:, perm_x].reshape(T, -1)
    x3 = gdn.gated_deltanet(qkv3, z3, a[:, perm_x], b[:, perm_x], p3, hk, hv, dk, dv, store=ident)
    assert not np.allclose(x3.y.reshape(T, hv, dv)[:, 0], base.y.reshape(T, hv, dv)[:, 2])
    for heads in ([0], [3, 1]):
        s = gdn.sample_mixer(qkv, z, a, b, p, hk, hv, dk, dv, heads, store=ident)
        np.testing.assert_allclose(s, base.y.reshape(T, hv, dv)[:, heads], rtol=1e-12,
                                   atol=1e-12)


@pytest.mark.parametrize("T", [0, 1])
def test_degenerate_lengths(T):
    hk, hv, dk, dv, W = 1, 1, 4, 4, 4
    qkv, z, a, b, p = _mixer_inputs(max(T, 1), hk, hv, dk, dv, W, RNG)
    qkv, z, a, b = qkv[:T], z[:T], a[:T], b[:T]
    S0 = RNG.standard_normal((hv, dv, dk))
    prev = RNG.standard_normal((W - 1, qkv.shape[1]))
    r = gdn.gated_deltanet(qkv, z, a, b, p, hk, hv, dk, dv, conv_state=prev, S0=S0,
                           store=lambda x: np.asarray(x, dtype=np.float64))
    assert r.y.shape == (T, hv * dv)
    if T == 0:
        np.testing.assert_array_equal(r.conv_state, prev)
        np.testing.assert_allclose(r.S, S0, rtol=1e-7)


def test_mixer_matches_the_qwen3_5_layer_in_transformers():
    # The pages' hybrid model is Qwen3.5; transformers ships its Gated DeltaNet
    # layer, whose portable path (no fused kernels installed) solves the
    # recurrence in 64-token chunks in fp32. The same weights through the
    # oracle's token-by-token recurrence must agree to fp32 rounding. This
    # checks the readings G2-G8 (channel order, conv orientation, the L2-norm
    # eps and q scale, the decay and strength formulas, the value-to-key head
    # map and the gated norm) against the model's own code.
    mq = pytest.importorskip("transformers.models.qwen3_5.modeling_qwen3_5")
    from transformers.models.qwen3_5.configuration_qwen3_5 import Qwen3_5TextConfig
    if mq.is_fast_path_available:
        pytest.skip("fused kernels installed: the portable path is not the one that runs")
    d, hk, hv, dk, dv, W, T = 48, 2, 4, 16, 8, 4, 70
    cfg = Qwen3_5TextConfig(hidden_size=d, linear_num_key_heads=hk, linear_num_value_heads=hv,
                            linear_key_head_dim=dk, linear_value_head_dim=dv,
                            linear_conv_kernel_dim=W, rms_norm_eps=1e-6, hidden_act="silu",
                            num_hidden_layers=1)
    torch.manual_seed(0)
    layer = mq.Qwen3_5GatedDeltaNet(cfg, layer_idx=0).double().eval()
    with torch.no_grad():
        for p_ in layer.parameters():
            p_.copy_(torch.randn_like(p_) * 0.3)
        layer.A_log.copy_(torch.log(torch.rand(hv, dtype=torch.float64) * 15 + 1))
        layer.dt_bias.copy_(torch.randn(hv, dtype=torch.float64) - 2)
        layer.norm.weight.copy_(1 + 0.1 * torch.randn(dv, dtype=torch.float64))
    x = torch.randn(1, T, d, dtype=torch.float64)
    with torch.no_grad():
        want = layer(x)[0].numpy()
    npw = lambda m: m.weight.detach().numpy()
    xs = x[0].numpy()
    p = gdn.MixerParams(conv_w=layer.conv1d.weight.detach().numpy()[:, 0, :],
                        A_log=layer.A_log.detach().numpy(), dt_bias=layer.dt_bias.detach().numpy(),
                        norm_w=layer.norm.weight.detach().numpy(), eps=1e-6)
    r = gdn.gated_deltanet(xs @ npw(layer.in_proj_qkv).T, xs @ npw(layer.in_proj_z).T,
                           xs @ npw(layer.in_proj_a).T, xs @ npw(layer.in_proj_b).T, p,
                           hk, hv, dk, dv, store=lambda v: np.asarray(v, dtype=np.float64))
    got = r.y @ npw(layer.out_proj).T
    scale = np.abs(want).max()
    np.testing.assert_allclose(got, want, rtol=1e-4, atol=1e-5 * scale)


# ---------------------------------------------------------------- hybrid stacks
def _gdn_stack_layer(rng, d, hk=1, hv=2, dk=8, dv=8, W=4, inter=32):
    C = 2 * hk * dk + hv * dv
    return gdn.GdnStackLayer(
        norm=rng.uniform(0.5, 1.5, d), w_in=rng.standard_normal((C + hv * dv + 2 * hv, d)) * 0.2,
        mixer=gdn.MixerParams(conv_w=rng.uniform(-0.5, 0.5, (C, W)),
                              A_log=np.log(rng.uniform(1, 16, hv)),
                              dt_bias=rng.uniform(-4, -1, hv), norm_w=rng.uniform(0.5, 1.5, dv)),
        w_out=rng.standard_normal((d, hv * dv)) * 0.2, hk=hk, hv=hv, dk=dk, dv=dv,
        ffn_norm=rng.uniform(0.5, 1.5, d), w_gate_up=rng.standard_normal((2 * inter, d)) * 0.1,
        w_down=rng.standard_normal((d, inter)) * 0.1)


def _hybrid_model(seed, kinds, d=64):
    from tests.test_oracle_pins import _tiny_model
    m = _tiny_model(seed, True, n_layers=len(kinds), d=d)
    rng = np.random.default_rng(seed + 1000)
    for i, kind in enumerate(kinds):
        if kind == "gdn":
            m.layers[i] = _gdn_stack_layer(rng, d)
        else:
            m.layers[i].gain = rng.uniform(0, 2, m.n_heads_q)
            m.layers[i].tau = rng.uniform(0.5, 1.5, m.n_heads_q)
    return m


def test_hybrid_with_attention_layers_only_is_the_gated_prefill():
    from oracle import tokengate_oracle as ref
    m = _hybrid_model(50, ["attn", "attn", "attn"])
    x = RNG.standard_normal((40, m.d_model))
    prot = np.zeros(40, dtype=np.uint8)
    prot[-3:] = 1
    for gate in (-1, 0, 1):
        a = gdn.hybrid_prefill(x, prot, 17, m, gate, store=ref.round_bf16)
        b = ref.prefill(x, prot, 17, m, gate, store=ref.round_bf16)
        np.testing.assert_array_equal(a.kept_idx, b.kept_idx)
        np.testing.assert_array_equal(a.out, b.out)


def test_gated_deltanet_layers_above_the_gate_see_only_the_kept_rows():
    # Gate before layer 0 in a Gated DeltaNet-only stack: every layer runs on
    # the kept rows, in order, with no positions or bias, so the result is
    # the ungated stack applied to just those rows (reading G1).
    from oracle import tokengate_oracle as ref
    m = _hybrid_model(51, ["gdn", "gdn"])
    x = RNG.standard_normal((30, m.d_model))
    prot = np.zeros(30, dtype=np.uint8)
    res = gdn.hybrid_prefill(x, prot, 12, m, -1)
    h = ref.round_fp32(x)[res.kept_idx]  # the forward stores its input first
    for lw in m.layers:
        r, _ = gdn.gdn_sublayer(h, lw, m.eps)
        h = ref.ffn_sublayer(r, lw, m, ref.round_fp32)
    h = ref.round_fp32(ref.rmsnorm(h, m.final_norm, m.eps))
    np.testing.assert_allclose(res.out, h, rtol=1e-12, atol=1e-12)
    # and a pruned row's input changes nothing above the gate
    pruned = np.setdiff1d(np.arange(30), res.kept_idx)[0]
    x2 = x.copy()
    x2[pruned] *= 3.0
    res2 = gdn.hybrid_prefill(x2, prot, 12, m, -1, kept_idx=res.kept_idx)
    np.testing.assert_array_equal(res2.out, res.out)


def test_hybrid_keeping_every_token_without_bias_is_the_ungated_stack():
    # K = N with gain 0 (and tau 1): the gate selects everything and adds
    # nothing, so the gated hybrid forward equals the plain layer-by-layer
    # forward, whichever layer (attention or Gated DeltaNet) holds the gate.
    from oracle import tokengate_oracle as ref
    m = _hybrid_model(52, ["gdn", "attn", "gdn", "attn"])
    for lw in m.layers:
        if not isinstance(lw, gdn.GdnStackLayer):
            lw.gain = np.zeros(m.n_heads_q)
            lw.tau = np.ones(m.n_heads_q)
    n = 24
    x = RNG.standard_normal((n, m.d_model))
    pos = np.arange(n, dtype=np.int32)
    h = ref.round_fp32(x)
    for lw in m.layers:
        if isinstance(lw, gdn.GdnStackLayer):
            r, _ = gdn.gdn_sublayer(h, lw, m.eps)
        else:
            r, _ = ref.attention_sublayer(h, lw, m, pos, None, None, None, ref.round_fp32)
        h = ref.ffn_sublayer(r, lw, m, ref.round_fp32)
    want = ref.round_fp32(ref.rmsnorm(h, m.final_norm, m.eps))
    for gate in (-1, 0, 1, 2):
        res = gdn.hybrid_prefill(x, np.zeros(n, dtype=np.uint8), n, m, gate)
        np.testing.assert_array_equal(res.kept_idx, np.arange(n))
        np.testing.assert_allclose(res.out, want, rtol=1e-12, atol=1e-12)


def test_gated_deltanet_sublayer_reads_its_projection_slices():
    # Zero output-gate rows (z) make the mixer's output exactly zero, so the
    # sub-layer is the identity; zeroing any other slice does not.
    rng = np.random.default_rng(53)
    d = 32
    lw = _gdn_stack_layer(rng, d)
    C = 2 * lw.hk * lw.dk + lw.hv * lw.dv
    x = rng.standard_normal((9, d))
    lw.w_in[C:C + lw.hv * lw.dv] = 0.0
    r, _ = gdn.gdn_sublayer(x, lw, 1e-6, store=lambda v: np.asarray(v, dtype=np.float64))
    np.testing.assert_array_equal(r, x)
    lw2 = _gdn_stack_layer(np.random.default_rng(53), d)
    lw2.w_in[C + lw2.hv * lw2.dv:] = 0.0  # a = b = 0 only
    r2, _ = gdn.gdn_sublayer(x, lw2, 1e-6, store=lambda v: np.asarray(v, dtype=np.float64))
    assert not np.allclose(r2, x)
