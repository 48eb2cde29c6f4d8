"""GPU parity of the Gated DeltaNet mixer (tg_gated_deltanet) with the oracle.

The mixer runs a hybrid model's linear-attention layer over the kept tokens.
The oracle takes the same seeded inputs, rounded to the call's dtype, in
float64. Tolerances: bf16 outputs within the bf16 bound used throughout
(2e-2 + 1e-2 |ref|); fp32 outputs within 1e-4 + 1e-4 |ref|. The fp32 state
S (dv x dk per value head) within 1e-4 + 1e-3 |ref|: the recurrence is
fp32 with fused multiply-adds, the oracle float64, and each step's rounding
(~6e-8 relative) decays with alpha (I - beta k k^T), whose eigenvalues lie
in [0, 1].
"""

import numpy as np
import pytest
import torch

import synth
from oracle import gated_deltanet_oracle as gdn
from tests._helpers import STORE, assert_close, host64

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")


@pytest.fixture(autouse=True)
def _no_device_errors():
    tg.tg_device_error(clear=True)
    yield
    assert tg.tg_device_error() == 0


def _setup(T, hk, hv, dk, dv, W, dtype, seed, carried=False):
    w = synth.GdnWorkload("test", "bf16", T=T, n=T, hk=hk, hv=hv, dk=dk, dv=dv, W=W, seed=seed)
    rng = synth.rng_for(seed)
    p = synth.gdn_params(w, rng)
    x = synth.gdn_inputs(w, rng)
    C = 2 * hk * dk + hv * dv
    conv_in = rng.standard_normal((W - 1, C), dtype=np.float32) if carried else None
    s_in = (0.3 * rng.standard_normal((hv, dv, dk), dtype=np.float32)) if carried else None
    dev = {k: torch.from_numpy(v).to("cuda", dtype) for k, v in x.items()}
    layer = tg.GdnLayer(hk, hv, dk, dv, *(torch.from_numpy(p[k]).cuda()
                                          for k in ("conv_w", "A_log", "dt_bias", "norm_w")),
                        eps=w.eps)
    conv_in_d = None if conv_in is None else torch.from_numpy(conv_in).to("cuda", dtype)
    s_in_d = None if s_in is None else torch.from_numpy(s_in).cuda()
    # the oracle sees exactly the values the device holds
    host = {k: host64(v) for k, v in dev.items()}
    om = gdn.MixerParams(conv_w=p["conv_w"].astype(np.float64), A_log=p["A_log"].astype(np.float64),
                         dt_bias=p["dt_bias"].astype(np.float64),
                         norm_w=p["norm_w"].astype(np.float64), eps=w.eps)
    ref_in = dict(conv_state=None if conv_in_d is None else host64(conv_in_d),
                  S0=None if s_in is None else s_in.astype(np.float64))
    return layer, dev, conv_in_d, s_in_d, host, om, ref_in


def _check_state(gpu, want):
    """The carried state is an fp32 output whatever the call's dtype: it is
    held to the fp32 tolerance, |gpu - ref| <= 1e-4 + 1e-4 |ref|."""
    assert_close(gpu, want, torch.float32, "state")


@pytest.mark.parametrize("T", [1, 31, 32, 33, 200, 517])
def test_mixer_matches_oracle_bf16(T):
    hk, hv, dk, dv, W = 2, 4, 128, 128, 4
    layer, x, _, _, host, om, _ = _setup(T, hk, hv, dk, dv, W, torch.bfloat16, 70 + T)
    y, conv_out, s_out = tg.tg_gated_deltanet(layer, x["qkv"], x["z"], x["a"], x["b"])
    torch.cuda.synchronize()
    r = gdn.gated_deltanet(host["qkv"], host["z"], host["a"], host["b"], om, hk, hv, dk, dv,
                           store=STORE[torch.bfloat16])
    assert_close(y, r.y, torch.bfloat16, "y")
    assert np.array_equal(host64(conv_out), r.conv_state)
    _check_state(s_out, r.S)


@pytest.mark.parametrize("hk,hv,dk,dv,W,T", [(2, 2, 64, 64, 3, 300), (1, 3, 64, 32, 4, 97),
                                             (1, 2, 128, 256, 2, 70), (2, 2, 128, 96, 1, 45)])
def test_mixer_matches_oracle_fp32_with_carried_state(hk, hv, dk, dv, W, T):
    layer, x, conv_in, s_in, host, om, ref_in = _setup(T, hk, hv, dk, dv, W, torch.float32,
                                                       80 + T, carried=True)
    y, conv_out, s_out = tg.tg_gated_deltanet(layer, x["qkv"], x["z"], x["a"], x["b"],
                                              conv_in=conv_in if W > 1 else None,
                                              state_in=s_in)
    torch.cuda.synchronize()
    r = gdn.gated_deltanet(host["qkv"], host["z"], host["a"], host["b"], om, hk, hv, dk, dv,
                           conv_state=ref_in["conv_state"] if W > 1 else None, S0=ref_in["S0"],
                           store=STORE[torch.float32])
    assert_close(y, r.y, torch.float32, "y")
    if W > 1:
        assert np.array_equal(host64(conv_out), r.conv_state)
    else:
        assert conv_out is None
    _check_state(s_out, r.S)


def test_zero_tokens_pass_the_state_through():
    hk, hv, dk, dv, W = 1, 2, 128, 64, 4
    layer, x, conv_in, s_in, *_ = _setup(5, hk, hv, dk, dv, W, torch.bfloat16, 90, carried=True)
    e = {k: v[:0] for k, v in x.items()}
    y, conv_out, s_out = tg.tg_gated_deltanet(layer, e["qkv"], e["z"], e["a"], e["b"],
                                              conv_in=conv_in, state_in=s_in)
    torch.cuda.synchronize()
    assert y.shape == (0, hv * dv)
    assert torch.equal(conv_out, conv_in) and torch.equal(s_out, s_in)
    # fewer tokens than the window keeps the older carried rows
    y1, conv1, _ = tg.tg_gated_deltanet(layer, x["qkv"][:1], x["z"][:1], x["a"][:1], x["b"][:1],
                                        conv_in=conv_in, state_in=s_in)
    torch.cuda.synchronize()
    assert torch.equal(conv1, torch.cat([conv_in[1:], x["qkv"][:1]]))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_split_calls_equal_one_call(dtype):
    # The carried conv rows are the inputs themselves and S is carried in
    # fp32. A split on a 32-token chunk boundary takes exactly the
    # arithmetic of one call (bit for bit); a split inside a chunk regroups
    # the chunked solve, so it agrees to rounding.
    T, hk, hv, dk, dv, W = 300, 2, 4, 128, 128, 4
    layer, x, *_ = _setup(T, hk, hv, dk, dv, W, dtype, 91)
    y, conv, s = tg.tg_gated_deltanet(layer, x["qkv"], x["z"], x["a"], x["b"])
    for cut in (32, 256, 1, 100):
        y1, c1, s1 = tg.tg_gated_deltanet(layer, *(x[k][:cut] for k in ("qkv", "z", "a", "b")))
        y2, c2, s2 = tg.tg_gated_deltanet(layer, *(x[k][cut:] for k in ("qkv", "z", "a", "b")),
                                          conv_in=c1, state_in=s1)
        torch.cuda.synchronize()
        assert torch.equal(c2, conv), cut
        if cut % 32 == 0:
            assert torch.equal(torch.cat([y1, y2]), y), cut
            assert torch.equal(s2, s), cut
        else:
            assert_close(torch.cat([y1, y2]), host64(y), dtype, f"y split at {cut}")
            _check_state(s2, host64(s))


def test_in_place_state_and_determinism():
    T, hk, hv, dk, dv, W = 150, 1, 2, 64, 128, 4
    layer, x, conv_in, s_in, *_ = _setup(T, hk, hv, dk, dv, W, torch.bfloat16, 92, carried=True)
    y, conv, s = tg.tg_gated_deltanet(layer, x["qkv"], x["z"], x["a"], x["b"], conv_in=conv_in,
                                      state_in=s_in)
    s_buf = s_in.clone()
    y2, _, s2 = tg.tg_gated_deltanet(layer, x["qkv"], x["z"], x["a"], x["b"], conv_in=conv_in,
                                     state_in=s_buf, state_out=s_buf)
    torch.cuda.synchronize()
    assert s2.data_ptr() == s_buf.data_ptr()
    assert torch.equal(y, y2) and torch.equal(s, s_buf)


def test_full_size_sampled_heads():
    # The workload's own sizes (4096 kept tokens, 16 + 16 heads of dim 128);
    # value heads are independent, so two of them are checked in full
    # against the oracle, one head at a time.
    w = synth.GDN_LAYER_32K
    rng = synth.rng_for(w.seed)
    p = synth.gdn_params(w, rng)
    x = synth.gdn_inputs(w, rng)
    dev = {k: torch.from_numpy(v).to("cuda", torch.bfloat16) for k, v in x.items()}
    layer = tg.GdnLayer(w.hk, w.hv, w.dk, w.dv, *(torch.from_numpy(p[k]).cuda()
                                                  for k in ("conv_w", "A_log", "dt_bias",
                                                            "norm_w")), eps=w.eps)
    y, _, _ = tg.tg_gated_deltanet(layer, dev["qkv"], dev["z"], dev["a"], dev["b"],
                                   want_state=False)
    torch.cuda.synchronize()
    host = {k: host64(v) for k, v in dev.items()}
    om = gdn.MixerParams(conv_w=p["conv_w"].astype(np.float64), A_log=p["A_log"].astype(np.float64),
                         dt_bias=p["dt_bias"].astype(np.float64),
                         norm_w=p["norm_w"].astype(np.float64), eps=w.eps)
    heads = [0, w.hv - 1]
    want = gdn.sample_mixer(host["qkv"], host["z"], host["a"], host["b"], om, w.hk, w.hv, w.dk,
                            w.dv, heads, store=STORE[torch.bfloat16])
    got = y.view(w.T, w.hv, w.dv)[:, heads]
    assert_close(got, want, torch.bfloat16, "y (sampled heads)")


def test_repeated_keys_full_strength_and_extreme_decay():
    # The per-chunk solve at its worst conditioning: (nearly) the same key at
    # every token with beta ~ 1, one value head with no decay (alpha = 1) and
    # one whose decay underflows fp32 (alpha ~ e^-80) within a chunk.
    T, hk, hv, dk, dv, W = 150, 1, 2, 64, 64, 4
    layer, x, _, _, host, om, _ = _setup(T, hk, hv, dk, dv, W, torch.float32, 93)
    C = 2 * hk * dk + hv * dv
    qkv = x["qkv"].clone()
    qkv[:, dk:2 * dk] = qkv[0, dk:2 * dk]  # constant k channels: the same key after W-1 tokens
    b = torch.full_like(x["b"], 8.0)
    layer.A_log.copy_(torch.tensor([0.0, float(np.log(16.0))]))
    layer.dt_bias.copy_(torch.tensor([-30.0, 5.0]))
    y, _, s_out = tg.tg_gated_deltanet(layer, qkv, x["z"], x["a"], b)
    torch.cuda.synchronize()
    om.A_log = np.array([0.0, np.log(16.0)])
    om.dt_bias = np.array([-30.0, 5.0])
    r = gdn.gated_deltanet(host64(qkv), host["z"], host["a"], host64(b), om, hk, hv, dk, dv,
                           store=STORE[torch.float32])
    assert qkv.shape[1] == C
    assert_close(y, r.y, torch.float32, "y")
    _check_state(s_out, r.S)
