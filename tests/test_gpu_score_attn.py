"""GPU parity of the scorer and the token-gated attention against the oracle.

bf16 runs the tensor-core kernels (tcgen05), fp32 the SIMT kernels. Inputs
are the same device values on both sides; tolerance |d| <= atol + rtol*|ref|
with (2e-2, 1e-2) for bf16 and (1e-4, 1e-4) for fp32.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import tokengate_oracle as ref
from tests._helpers import STORE, assert_close, dev, host64

pytestmark = pytest.mark.gpu

tg = pytest.importorskip("learned_token_pruning_score_b200")


@pytest.fixture(autouse=True)
def _no_device_errors():
    tg.tg_device_error(clear=True)
    yield
    assert tg.tg_device_error() == 0


def _score_case(n, d, f, dtype, seed, salient=0.0, bias=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d)).astype(np.float32)
    if salient:
        rows = rng.choice(n, max(1, int(salient * n)), replace=False)
        x[rows] *= 4
    g = rng.uniform(0.5, 1.5, d).astype(np.float32)
    w1 = (rng.standard_normal((f, d)) * 0.02).astype(np.float32)
    b1 = (rng.standard_normal(f) * 0.1).astype(np.float32) if bias else None
    w2 = (rng.standard_normal(f) * 0.02).astype(np.float32)
    b2 = np.array([0.05], np.float32) if bias else None
    xd, w1d = dev(x, dtype), dev(w1, dtype)
    s = tg.tg_score(xd, dev(g), w1d, dev(w2), b1=None if b1 is None else dev(b1),
                    b2=None if b2 is None else dev(b2))
    torch.cuda.synchronize()
    want = ref.score(host64(xd), g, 1e-6, host64(w1d), b1, w2, b2, store=STORE[dtype])
    assert_close(s, want, dtype, "scores")


@pytest.mark.parametrize("n", [1, 127, 1000])
def test_score_bf16(n):
    _score_case(n, 2048, 256, torch.bfloat16, n)


def test_score_bf16_narrow_hidden_and_no_bias():
    _score_case(333, 512, 64, torch.bfloat16, 5, bias=False)


def test_score_bf16_config_shape():
    # 16K tokens x 2048 -> 256 -> 1, 1% salient rows at 4x norm
    _score_case(16384, 2048, 256, torch.bfloat16, 11, salient=0.01)


def test_score_fp32_tiny_config():
    _score_case(512, 256, 64, torch.float32, 0)


def _attn_case(t, hq, hkv, dh, dtype, seed, bias=True, sparse_pos=True, max_pos=131072):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((t, hq, dh)).astype(np.float32)
    k = rng.standard_normal((t, hkv, dh)).astype(np.float32)
    v = rng.standard_normal((t, hkv, dh)).astype(np.float32)
    if sparse_pos:
        pos = np.sort(rng.choice(max(max_pos, t), t, replace=False)).astype(np.int32)
    else:
        pos = np.arange(t, dtype=np.int32)
    s = (rng.standard_normal(t) * 2).astype(np.float32) if bias else None
    gain = rng.uniform(0, 2, hq).astype(np.float32) if bias else None
    tau = rng.uniform(0.5, 1.5, hq).astype(np.float32) if bias else None
    qd, kd, vd = dev(q, dtype), dev(k, dtype), dev(v, dtype)
    out = tg.tg_gated_attn_prefill(
        qd, kd, vd, torch.from_numpy(pos).cuda(), None if s is None else dev(s),
        None if gain is None else dev(gain), None if tau is None else dev(tau), rope_base=1e6)
    torch.cuda.synchronize()
    want = ref.gated_attn_prefill(host64(qd), host64(kd), host64(vd), pos, s, gain, tau, 1e6,
                                  store=STORE[dtype])
    assert_close(out, want, dtype, f"attn t={t}")


@pytest.mark.parametrize("t", [1, 100, 128, 129, 300, 1000])
def test_attn_bf16_ragged(t):
    _attn_case(t, 4, 2, 128, torch.bfloat16, t)


def test_attn_bf16_no_bias_dense_positions():
    _attn_case(700, 4, 2, 128, torch.bfloat16, 3, bias=False, sparse_pos=False)


def test_attn_bf16_mha_and_wide_gqa():
    _attn_case(260, 3, 3, 128, torch.bfloat16, 4)
    _attn_case(260, 8, 1, 128, torch.bfloat16, 5)


def test_attn_bf16_qwen_heads_k2048():
    # the gated layer of the 16K-token workload: K = 2048 rows, 16 / 8 heads
    _attn_case(2048, 16, 8, 128, torch.bfloat16, 6, max_pos=16384)


@pytest.mark.parametrize("t", [512, 1024, 1536])
def test_attn_bf16_qwen_heads_short_sequences(t):
    """Short sequences run a table schedule in which long query tiles are
    split across CTAs (parts merged by the last one to finish): 16 / 8 heads
    at lengths whose schedules split tiles into 2 to 4 parts."""
    _attn_case(t, 16, 8, 128, torch.bfloat16, 20 + t, max_pos=4 * t)


def test_attn_bf16_split_schedule_is_deterministic():
    """Which part of a split query tile finishes last varies from run to run;
    the merge takes the parts in a fixed order, so the bits do not."""
    rng = np.random.default_rng(31)
    t, hq, hkv = 2048, 16, 8
    q = dev(rng.standard_normal((t, hq, 128)), torch.bfloat16)
    k = dev(rng.standard_normal((t, hkv, 128)), torch.bfloat16)
    v = dev(rng.standard_normal((t, hkv, 128)), torch.bfloat16)
    pos = torch.from_numpy(np.sort(rng.choice(8 * t, t, replace=False)).astype(np.int32)).cuda()
    s = dev(rng.standard_normal(t) * 2)
    gain = dev(rng.uniform(0, 2, hq))
    tau = dev(rng.uniform(0.5, 1.5, hq))
    runs = [tg.tg_gated_attn_forward(q, k, v, pos, s, gain, tau) for _ in range(3)]
    torch.cuda.synchronize()
    for out, lse, o32 in runs[1:]:
        assert torch.equal(out, runs[0][0])
        assert torch.equal(lse, runs[0][1])
        assert torch.equal(o32, runs[0][2])


@pytest.mark.parametrize("dh", [64, 128])
def test_attn_fp32(dh):
    _attn_case(128, 4, 2, dh, torch.float32, 7 + dh, max_pos=512)
    _attn_case(37, 2, 1, dh, torch.float32, 8 + dh, bias=False)


def test_attn_reduces_to_causal_attention_when_gain_zero_tau_one():
    """K = N, gain 0, tau 1: the kernel equals plain causal attention
    (torch SDPA in fp64 on the same rotated inputs)."""
    t, hq, hkv, dh = 400, 4, 2, 128
    rng = np.random.default_rng(9)
    q = dev(rng.standard_normal((t, hq, dh)), torch.bfloat16)
    k = dev(rng.standard_normal((t, hkv, dh)), torch.bfloat16)
    v = dev(rng.standard_normal((t, hkv, dh)), torch.bfloat16)
    pos = torch.arange(t, dtype=torch.int32, device="cuda")
    s = dev(rng.standard_normal(t))
    out = tg.tg_gated_attn_prefill(q, k, v, pos, s, torch.zeros(hq, device="cuda"),
                                   torch.ones(hq, device="cuda"))
    torch.cuda.synchronize()
    qr = ref.round_bf16(ref.rope(host64(q), np.arange(t), 1e6))
    kr = ref.round_bf16(ref.rope(host64(k), np.arange(t), 1e6))
    tq = torch.from_numpy(qr).permute(1, 0, 2)[None]
    tk = torch.from_numpy(kr).permute(1, 0, 2)[None]
    tv = torch.from_numpy(host64(v)).permute(1, 0, 2)[None]
    want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True,
                                                            enable_gqa=True)
    assert_close(out, want[0].permute(1, 0, 2).numpy(), torch.bfloat16, "sdpa")


@pytest.mark.parametrize("m,n,k", [(1, 256, 64), (127, 2048, 2048), (1000, 4096, 2048),
                                   (300, 2048, 6144), (4096, 288, 520),
                                   (4000, 1824, 520), (8192, 2048, 2048)])
@pytest.mark.parametrize("residual", [False, True])
def test_linear_bf16(m, n, k, residual):
    """The tcgen05 GEMM against a float64 product of the same bf16 values
    (ragged m, k not a multiple of 64, n not a multiple of 256). The last two
    shapes fill more than one wave of pair tiles, the first of them with a
    ragged last column block."""
    rng = np.random.default_rng(m + n + k)
    x = dev(rng.standard_normal((m, k)), torch.bfloat16)
    w = dev(rng.standard_normal((n, k)) * 0.02, torch.bfloat16)
    r = dev(rng.standard_normal((m, n)), torch.bfloat16) if residual else None
    y = tg.tg_linear(x, w, residual=r)
    torch.cuda.synchronize()
    want = host64(x) @ host64(w).T + (host64(r) if residual else 0.0)
    assert_close(y, ref.round_bf16(want), torch.bfloat16, f"linear {m}x{n}x{k}")


def test_linear_fp32_and_in_place_residual():
    rng = np.random.default_rng(5)
    x = dev(rng.standard_normal((77, 96)))
    w = dev(rng.standard_normal((40, 96)))
    y = dev(rng.standard_normal((77, 40)))
    y0 = host64(y)
    tg.tg_linear(x, w, residual=y, y=y)
    torch.cuda.synchronize()
    assert_close(y, host64(x) @ host64(w).T + y0, torch.float32, "fp32 linear")
