"""Parity of the gated-attention backward (tg_gated_attn_forward's lse and
tg_gated_attn_backward) with the oracle, on the same seeded bf16 inputs.

Tolerance for the gradients, per element, from the arithmetic of the
kernels. They round P and dS to bf16 (unit roundoff u = 2^-8) as
tensor-core operands, and the D_i = dout_i . o_i they use carries the
forward's bf16 P of its P.V product. To first order, with the oracle's own P,
dl and dP = dout . v^T of each head (c_h = 1 / (sqrt(dh) tau_h)):
  e_i  = u sum_j P_ij |dP_ij|                               (error of D_i)
  dq'  : c_h (u |dl| |k'| + e P |k'|)                      (rotated frame)
  dk'  : sum_h c_h (u |dl|^T |q'| + (P e)^T |q'|)
  dv   : sum_h u P^T |dout|
  C_hj : sum_i P_ij e_i   -> ds: sigmoid(-s) sum_h |g_h| C-bound, dgain: |b| . C-bound
  dtau : (1 / tau_h) sum_i |q'_i| . dq'-bound
dq and dk are rotated back (|cos x + sin y| <= |x| + |y| per pair). The test
allows twice that (second-order terms, the approximate exp2, fp32 sums), plus
the two bf16 output roundings (2^-7 |ref|). A per-element bound alone is
loose on rows with thousands of keys, so the RMS of the error must also stay
below 1e-2 of the RMS of the reference (at least 1e-3: gradients that vanish
exactly, like every gradient but dv of a single row), which catches
systematic slips.
"""

import math

import numpy as np
import pytest
import torch

from oracle import tokengate_oracle as ref
from tests._helpers import dev, host64

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")


@pytest.fixture(autouse=True)
def _no_device_errors():
    tg.tg_device_error(clear=True)
    yield
    assert tg.tg_device_error() == 0


def _inputs(t, hq, hkv, seed, bias=True, sparse_pos=True, max_pos=131072):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((t, hq, 128)).astype(np.float32)
    k = rng.standard_normal((t, hkv, 128)).astype(np.float32)
    v = rng.standard_normal((t, hkv, 128)).astype(np.float32)
    dout = rng.standard_normal((t, hq, 128)).astype(np.float32)
    if sparse_pos:
        pos = np.sort(rng.choice(max(max_pos, t), t, replace=False)).astype(np.int32)
    else:
        pos = np.arange(t, dtype=np.int32)
    s = (rng.standard_normal(t) * 2).astype(np.float32) if bias else None
    gain = rng.uniform(0, 2, hq).astype(np.float32) if bias else None
    tau = rng.uniform(0.5, 1.5, hq).astype(np.float32) if bias else None
    bf = torch.bfloat16
    d = dict(q=dev(q, bf), k=dev(k, bf), v=dev(v, bf), dout=dev(dout, bf),
             pos=torch.from_numpy(pos).cuda(), s=None if s is None else dev(s),
             gain=None if gain is None else dev(gain), tau=None if tau is None else dev(tau))
    h = dict(q=host64(d["q"]), k=host64(d["k"]), v=host64(d["v"]), dout=host64(d["dout"]),
             pos=pos, s=s, gain=gain, tau=tau)
    return d, h


def _gpu_fwd_bwd(d, base=1e6, f32=True):
    out, lse, o32 = tg.tg_gated_attn_forward(d["q"], d["k"], d["v"], d["pos"], d["s"], d["gain"],
                                             d["tau"], rope_base=base, want_f32=f32)
    grads = tg.tg_gated_attn_backward(d["q"], d["k"], d["v"], d["pos"], out, lse, d["dout"],
                                      d["s"], d["gain"], d["tau"], rope_base=base, out_f32=o32)
    torch.cuda.synchronize()
    return out, lse, grads


def _reference_with_bounds(h, base=1e6, heads=None, kv=None):
    """Oracle gradients (stored as the kernels store them) and their
    per-element error budgets; heads/kv restrict to a KV group's sub-problem."""
    q, k, v, dout = h["q"], h["k"], h["v"], h["dout"]
    gain, tau = h["gain"], h["tau"]
    if heads is not None:
        q, dout, k, v = q[:, heads], dout[:, heads], k[:, kv], v[:, kv]
        gain = None if gain is None else gain[heads]
        tau = None if tau is None else tau[heads]
    pos, s = h["pos"], h["s"]
    t, hq, dh = q.shape
    u = 2.0 ** -8
    qr = ref.round_bf16(ref.rope(q, pos, base))
    kr = ref.round_bf16(ref.rope(k, pos, base))
    tau_v = np.ones(hq) if tau is None else np.asarray(tau, np.float64)
    gain_v = np.zeros(hq) if gain is None else np.asarray(gain, np.float64)
    bq = np.zeros_like(qr)
    bk = np.zeros_like(kr)
    bv = np.zeros_like(kr)
    bc = np.zeros((hq, t))

    def on_head(hh, g, P, dl, dp):
        c = 1.0 / (math.sqrt(dh) * tau_v[hh])
        e = u * (P * np.abs(dp)).sum(axis=1)
        adl = np.abs(dl)
        ak, aq = np.abs(kr[:, g]), np.abs(qr[:, hh])
        bq[:, hh] = c * (u * (adl @ ak) + e[:, None] * (P @ ak))
        bk[:, g] += c * (u * (adl.T @ aq) + (P * e[:, None]).T @ aq)
        bv[:, g] += u * (P.T @ np.abs(dout[:, hh]))
        bc[hh] = (P * e[:, None]).sum(axis=0)

    grads = ref.gated_attention_grads(qr, kr, v, pos, s, gain, tau, dout, on_head=on_head)

    def back(b):  # bound through the transposed rotation of each (d, d+64) pair
        half = b.shape[-1] // 2
        pair = b[..., :half] + b[..., half:]
        return np.concatenate([pair, pair], axis=-1)

    neg = -np.asarray(pos, dtype=np.int64)
    want = [ref.round_bf16(ref.rope(grads[0], neg, base)),
            ref.round_bf16(ref.rope(grads[1], neg, base)), ref.round_bf16(grads[2]),
            None if grads[3] is None else ref.round_fp32(grads[3]),
            ref.round_fp32(grads[4]), ref.round_fp32(grads[5])]
    bound = [back(bq), back(bk), bv,
             None if s is None else ref.sigmoid(-np.asarray(s, np.float64)) * (np.abs(gain_v) @ bc),
             (np.zeros(hq) if s is None else bc @ np.abs(ref.logsigmoid(s))),
             np.einsum("thd,thd->h", np.abs(qr), bq) / tau_v]
    return want, bound


def assert_within_budget(gpu, want, budget, what):
    g = host64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    w = np.asarray(want, dtype=np.float64)
    assert g.shape == w.shape, (what, g.shape, w.shape)
    assert np.all(np.isfinite(g)), what
    d = np.abs(g - w)
    rms = math.sqrt(float(np.mean(w * w))) if w.size else 0.0
    lim = 2.0 * budget + 2.0 ** -7 * np.abs(w) + 1e-6 * max(rms, 1e-3)
    bad = d > lim
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, d / lim, -1)), d.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside the budget; worst at "
                             f"{i}: gpu={g[i]!r} ref={w[i]!r} budget={lim[i]:.3e}")
    if d.size <= 64:  # per-head scalars (dgain, dtau): the budget per element only
        return
    rms_err = math.sqrt(float(np.mean(d * d))) if d.size else 0.0
    assert rms_err <= 1e-2 * max(rms, 1e-3), f"{what}: rms error {rms_err:.3e} vs rms {rms:.3e}"


def _check_case(t, hq, hkv, seed, bias=True, sparse_pos=True, max_pos=131072):
    d, h = _inputs(t, hq, hkv, seed, bias, sparse_pos, max_pos)
    out, lse, (dq, dk, dv, ds, dgain, dtau) = _gpu_fwd_bwd(d)
    qr = ref.round_bf16(ref.rope(h["q"], h["pos"], 1e6))
    kr = ref.round_bf16(ref.rope(h["k"], h["pos"], 1e6))
    want_lse = ref.gated_attention_lse(qr, kr, h["pos"], h["s"], h["gain"], h["tau"])
    # lse: fp32 softmax statistics; the gate bias enters the tensor-core
    # product as a bf16 hi/lo pair (about 2^-16 of |gain * logsigmoid(s)|) and
    # a quarter of the exponentials use a degree-3 polynomial (7.5e-5
    # relative), so the bound is absolute, in natural-log units
    err = np.max(np.abs(host64(lse) - want_lse))
    assert err <= 5e-4, f"lse t={t}: max |d| = {err:.3e}"
    want, budget = _reference_with_bounds(h)
    for name, g, r, b in zip(("dq", "dk", "dv", "ds", "dgain", "dtau"),
                             (dq, dk, dv, ds, dgain, dtau), want, budget):
        if r is None:
            assert g is None, name
            continue
        assert_within_budget(g, r, b, f"{name} t={t} h={hq}/{hkv}")


@pytest.mark.parametrize("t", [1, 100, 128, 129, 300, 700])
def test_attn_backward_ragged(t):
    _check_case(t, 4, 2, 100 + t)


def test_attn_backward_no_bias_dense_positions():
    _check_case(400, 4, 2, 7, bias=False, sparse_pos=False)


def test_attn_backward_mha_and_wide_gqa():
    _check_case(260, 3, 3, 8)
    _check_case(260, 8, 1, 9)


def test_attn_backward_qwen_heads_k2048():
    # one gated layer of the 16K-token workload: 2048 kept rows, 16 / 8 heads
    _check_case(2048, 16, 8, 10, max_pos=16384)


def test_attn_backward_reduces_to_plain_attention_gradients():
    # gain 0, tau 1, positions 0..t-1: torch autograd of causal SDPA in fp64
    # over the same (rotated) operands gives dq', dk', dv
    t, hq, hkv = 200, 4, 2
    d, h = _inputs(t, hq, hkv, 11, bias=False, sparse_pos=False)
    out, lse, (dq, dk, dv, ds, dgain, dtau) = _gpu_fwd_bwd(d)
    assert ds is None and np.all(host64(dgain) == 0.0)
    qr = torch.tensor(ref.round_bf16(ref.rope(h["q"], h["pos"], 1e6)), requires_grad=True)
    kr = torch.tensor(ref.round_bf16(ref.rope(h["k"], h["pos"], 1e6)), requires_grad=True)
    vv = torch.tensor(h["v"], requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(
        qr.permute(1, 0, 2)[None], kr.permute(1, 0, 2)[None], vv.permute(1, 0, 2)[None],
        is_causal=True, enable_gqa=True)[0].permute(1, 0, 2)
    (o * torch.from_numpy(h["dout"])).sum().backward()
    neg = -h["pos"].astype(np.int64)
    _, budget = _reference_with_bounds(h)
    assert_within_budget(dq, ref.rope(qr.grad.numpy(), neg, 1e6), budget[0], "dq vs autograd")
    assert_within_budget(dk, ref.rope(kr.grad.numpy(), neg, 1e6), budget[1], "dk vs autograd")
    assert_within_budget(dv, vv.grad.numpy(), budget[2], "dv vs autograd")


def test_attn_backward_deterministic():
    d, _ = _inputs(333, 4, 2, 12)
    _, _, a = _gpu_fwd_bwd(d)
    _, _, b = _gpu_fwd_bwd(d)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_attn_backward_full_size_sampled_heads():
    # K = 4096 kept rows, 16 / 8 heads (the gated layers of the 32K-token
    # workload): the oracle computes KV group 0 (query heads 0 and 1) whole
    # (its dk, dv and the two heads' dq, dgain, dtau depend on no other head)
    t, hq, hkv = 4096, 16, 8
    d, h = _inputs(t, hq, hkv, 13, max_pos=32768)
    out, lse, (dq, dk, dv, ds, dgain, dtau) = _gpu_fwd_bwd(d)
    sub = [0, 1]
    want, budget = _reference_with_bounds(h, heads=sub, kv=[0])
    assert_within_budget(dq[:, sub], want[0], budget[0], "dq heads 0-1")
    assert_within_budget(dk[:, :1], want[1], budget[1], "dk group 0")
    assert_within_budget(dv[:, :1], want[2], budget[2], "dv group 0")
    assert_within_budget(dgain[sub], want[4], budget[4], "dgain heads 0-1")
    assert_within_budget(dtau[sub], want[5], budget[5], "dtau heads 0-1")
    # ds sums over all 16 heads (not computed by the oracle here): finite
    assert torch.isfinite(ds).all()


def test_attn_backward_from_the_bf16_output():
    # Without the fp32 output, D_i = dout_i . o_i comes from the bf16 output:
    # dv (no D) is bit-identical, and every other gradient moves by what the
    # output's rounding (|delta o| <= 2^-9 |o| elementwise) does through D:
    # |delta D_i| <= 2^-9 sum_d |dout_id| |o_id| =: e_i, so each dl_ij moves
    # by at most P_ij e_i, and dq_i by at most c_h e_i max_j |k'_j|; the
    # bound below also allows one bf16 rounding of the result.
    t, hq, hkv = 300, 4, 2
    d, _ = _inputs(t, hq, hkv, 15)
    out, lse, o32 = tg.tg_gated_attn_forward(d["q"], d["k"], d["v"], d["pos"], d["s"], d["gain"],
                                             d["tau"], rope_base=1e6)
    args = (d["q"], d["k"], d["v"], d["pos"], out, lse, d["dout"], d["s"], d["gain"], d["tau"])
    a = tg.tg_gated_attn_backward(*args, rope_base=1e6, out_f32=o32)
    b = tg.tg_gated_attn_backward(*args, rope_base=1e6)
    torch.cuda.synchronize()
    assert torch.equal(a[2], b[2])
    e = (2.0 ** -9) * (d["dout"].float().abs() * o32.abs()).sum(-1)  # [t, hq]
    kmax = float(d["k"].float().abs().max()) * 1.01  # RoPE keeps |k'|_2; bound per element loosely
    c = 1.0 / (math.sqrt(128) * d["tau"])
    bound_q = (c[None, :] * e * kmax * math.sqrt(128))[..., None]
    dq_a, dq_b = a[0].float(), b[0].float()
    assert torch.all((dq_a - dq_b).abs() <= bound_q + 2.0 ** -8 * dq_a.abs()), "dq"


def test_attn_backward_constant_scores():
    # constant s: every head's per-key sums of dl add up to zero over the keys
    # (softmax rows sum to one), so sum_j ds_j and dgain vanish
    t, hq, hkv = 300, 4, 2
    d, h = _inputs(t, hq, hkv, 14)
    d["s"] = torch.full((t,), -0.8, device="cuda")
    _, _, (dq, dk, dv, ds, dgain, dtau) = _gpu_fwd_bwd(d)
    dsh = host64(ds)
    assert abs(dsh.sum()) <= 1e-3 * np.abs(dsh).sum()
    h["s"] = np.full(t, -0.8)
    want, budget = _reference_with_bounds(h)
    assert_within_budget(ds, want[3], budget[3], "ds constant scores")
    scale = float(np.abs(want[3]).sum())
    assert np.all(np.abs(host64(dgain)) <= 1e-3 * scale)


# ---------------------------------------------------------------- fp32 (CUDA cores)


def _inputs_f32(t, hq, hkv, dh, seed, bias=True):
    rng = np.random.default_rng(seed)
    arrs = [rng.standard_normal((t, hq, dh)), rng.standard_normal((t, hkv, dh)),
            rng.standard_normal((t, hkv, dh)), rng.standard_normal((t, hq, dh))]
    pos = np.sort(rng.choice(max(4096, t), t, replace=False)).astype(np.int32)
    s = (rng.standard_normal(t) * 2).astype(np.float32) if bias else None
    gain = rng.uniform(0, 2, hq).astype(np.float32) if bias else None
    tau = rng.uniform(0.5, 1.5, hq).astype(np.float32) if bias else None
    dq_, dk_, dv_, do_ = (dev(x) for x in arrs)
    d = dict(q=dq_, k=dk_, v=dv_, dout=do_, pos=torch.from_numpy(pos).cuda(),
             s=None if s is None else dev(s), gain=None if gain is None else dev(gain),
             tau=None if tau is None else dev(tau))
    h = dict(q=host64(dq_), k=host64(dk_), v=host64(dv_), dout=host64(do_), pos=pos, s=s,
             gain=gain, tau=tau)
    return d, h


@pytest.mark.parametrize("t,dh,bias", [(1, 64, True), (37, 64, True), (128, 128, True),
                                       (200, 64, False), (300, 128, True)])
def test_attn_backward_fp32(t, dh, bias):
    # fp32 end to end: the gradients match the oracle to the fp32 tolerance
    # (1e-4, the absolute term scaled by the tensor's RMS as in the bf16 case)
    d, h = _inputs_f32(t, 4, 2, dh, 900 + t + dh, bias)
    out, lse, o32 = tg.tg_gated_attn_forward(d["q"], d["k"], d["v"], d["pos"], d["s"], d["gain"],
                                             d["tau"], rope_base=1e6)
    assert o32 is None
    grads = tg.tg_gated_attn_backward(d["q"], d["k"], d["v"], d["pos"], out, lse, d["dout"],
                                      d["s"], d["gain"], d["tau"], rope_base=1e6)
    torch.cuda.synchronize()
    qr = ref.round_fp32(ref.rope(h["q"], h["pos"], 1e6))
    kr = ref.round_fp32(ref.rope(h["k"], h["pos"], 1e6))
    want_lse = ref.gated_attention_lse(qr, kr, h["pos"], h["s"], h["gain"], h["tau"])
    assert np.max(np.abs(host64(lse) - want_lse)) <= 1e-4
    want = ref.gated_attn_backward(h["q"], h["k"], h["v"], h["pos"], h["s"], h["gain"], h["tau"],
                                   1e6, h["dout"], store=ref.round_fp32)
    for name, g, r in zip(("dq", "dk", "dv", "ds", "dgain", "dtau"), grads, want):
        if r is None:
            assert g is None, name
            continue
        gg, rr = host64(g), np.asarray(r, dtype=np.float64)
        rms = math.sqrt(float(np.mean(rr * rr))) if rr.size else 0.0
        bad = np.abs(gg - rr) > 1e-4 * max(rms, 1e-3) + 1e-4 * np.abs(rr)
        assert not bad.any(), (name, t, dh, float(np.abs(gg - rr).max()), rms)
