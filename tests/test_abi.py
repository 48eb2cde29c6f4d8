"""The C ABI on the host: the library loads, exports every declared symbol,
sizes workspaces, and rejects bad arguments before launching anything.

None of these calls reaches a kernel: each one fails host-side validation,
so they run on a machine without a GPU.
"""

import ctypes
import os
import re

import pytest
import torch

import learned_token_pruning_score_b200 as tg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tokengate.h")
BOGUS = ctypes.c_void_p(4096)  # never dereferenced: every call below fails validation first


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tg_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert {"tg_score", "tg_topk_select", "tg_compact", "tg_gated_attn_prefill",
            "tg_prefill", "tg_workspace_size", "tg_status_string"} <= set(names)
    lib = ctypes.CDLL(tg.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version():
    assert tg.tg_status_string(tg.TG_OK) == "ok"
    for s in range(1, 6):
        assert len(tg.tg_status_string(s)) > 3
    assert "sm_100a" in tg.tg_version()


def test_workspace_sizes():
    a = tg.tg_workspace_size(tg.TG_OP_TOPK_SELECT, n=8192)
    b = tg.tg_workspace_size(tg.TG_OP_TOPK_SELECT, n=131072)
    assert 0 < a < b
    assert tg.tg_workspace_size(tg.TG_OP_COMPACT, n=10, k=5) == 0
    s1 = tg.tg_workspace_size(tg.TG_OP_GATED_ATTN, k=2048, n_heads_q=16, n_heads_kv=8,
                              head_dim=128, dtype=tg.TG_BF16)
    # q, k, V^T (bf16) and the per-key bias
    assert s1 >= 2048 * 16 * 128 * 2 + 2048 * 8 * 128 * 2 * 2 + 2048 * 4
    p = dict(d_model=2048, n_heads_q=16, n_heads_kv=8, head_dim=128, d_score=256, d_ffn=6144,
             n_layers=28, gate_layer=1, dtype=tg.TG_BF16)
    assert tg.tg_workspace_size(tg.TG_OP_PREFILL, n=32768, k=4096, **p) > \
        tg.tg_workspace_size(tg.TG_OP_PREFILL, n=16384, k=4096, **p)


def test_select_validation():
    f = tg._topk
    assert f(None, None, 10, 5, BOGUS, BOGUS, 1 << 20, None) == tg.TG_ERR_INVALID_ARG
    assert f(BOGUS, None, 10, 0, BOGUS, BOGUS, 1 << 20, None) == tg.TG_ERR_BUDGET
    assert f(BOGUS, None, 10, 11, BOGUS, BOGUS, 1 << 20, None) == tg.TG_ERR_BUDGET
    assert f(BOGUS, None, 10, 5, BOGUS, BOGUS, 4, None) == tg.TG_ERR_WORKSPACE
    assert f(BOGUS, None, 10, 5, BOGUS, None, 1 << 20, None) == tg.TG_ERR_WORKSPACE


def test_compact_validation():
    f = tg._compact
    assert f(BOGUS, None, None, BOGUS, 10, 11, 64, tg.TG_BF16, BOGUS, BOGUS, None, None) == \
        tg.TG_ERR_BUDGET
    # 6 bf16 = 12-byte rows cannot be copied in 16-byte vectors
    assert f(BOGUS, None, None, BOGUS, 10, 5, 6, tg.TG_BF16, BOGUS, BOGUS, None, None) == \
        tg.TG_ERR_UNSUPPORTED
    assert f(BOGUS, None, None, BOGUS, 10, 5, 64, 7, BOGUS, BOGUS, None, None) == \
        tg.TG_ERR_UNSUPPORTED
    # scores_out requested without scores
    assert f(BOGUS, None, None, BOGUS, 10, 5, 64, tg.TG_BF16, BOGUS, BOGUS, BOGUS, None) == \
        tg.TG_ERR_INVALID_ARG
    unaligned = ctypes.c_void_p(4096 + 2)
    assert f(unaligned, None, None, BOGUS, 10, 5, 64, tg.TG_BF16, BOGUS, BOGUS, None, None) == \
        tg.TG_ERR_INVALID_ARG


def test_score_validation():
    f = tg._score
    args = [BOGUS, 100, 2048, 256, BOGUS, 1e-6, BOGUS, None, BOGUS, None]
    assert f(*args, tg.TG_BF16, BOGUS, BOGUS, 16, None) == tg.TG_ERR_WORKSPACE
    a2 = list(args)
    a2[3] = 512  # F > 256 is not built for bf16
    assert f(*a2, tg.TG_BF16, BOGUS, BOGUS, 1 << 30, None) == tg.TG_ERR_UNSUPPORTED
    a3 = list(args)
    a3[0] = None
    assert f(*a3, tg.TG_BF16, BOGUS, BOGUS, 1 << 30, None) == tg.TG_ERR_INVALID_ARG


def test_attention_validation():
    f = tg._attn
    base = [BOGUS, BOGUS, BOGUS, BOGUS, None, None, None, 128]
    assert f(*base, 4, 2, 64, 1e6, tg.TG_BF16, BOGUS, BOGUS, 1 << 30, None) == \
        tg.TG_ERR_UNSUPPORTED  # bf16 head_dim 64 is not built
    assert f(*base, 4, 3, 128, 1e6, tg.TG_BF16, BOGUS, BOGUS, 1 << 30, None) == \
        tg.TG_ERR_INVALID_ARG  # hq % hkv != 0
    assert f(*base, 4, 2, 128, 1e6, tg.TG_BF16, BOGUS, BOGUS, 64, None) == tg.TG_ERR_WORKSPACE
    assert f(*base, 4, 2, 96, 1e6, tg.TG_F32, BOGUS, BOGUS, 1 << 30, None) == \
        tg.TG_ERR_UNSUPPORTED


def test_attention_forward_lse_and_backward_validation():
    fwd = tg._attn_fwd
    base = [BOGUS, BOGUS, BOGUS, BOGUS, None, None, None, 128, 4, 2, 128, 1e6]
    assert fwd(*base, tg.TG_BF16, BOGUS, None, None, BOGUS, 1 << 30, None) == \
        tg.TG_ERR_INVALID_ARG  # no lse
    assert fwd(*base, tg.TG_BF16, BOGUS, BOGUS, ctypes.c_void_p(4096 + 4), BOGUS, 1 << 30,
               None) == tg.TG_ERR_INVALID_ARG  # misaligned fp32 output
    assert fwd(*base, tg.TG_F32, BOGUS, BOGUS, BOGUS, BOGUS, 1 << 30, None) == \
        tg.TG_ERR_INVALID_ARG  # fp32: the output is already fp32, no second copy
    assert fwd(*base, tg.TG_BF16, BOGUS, BOGUS, None, BOGUS, 64, None) == tg.TG_ERR_WORKSPACE
    bwd = tg._attn_bwd
    need = tg.tg_workspace_size(tg.TG_OP_GATED_ATTN_BWD, k=128, n_heads_q=4, n_heads_kv=2,
                                head_dim=128, dtype=tg.TG_BF16)
    # rotated q and k, the RoPE table and the per-row vectors
    assert need >= 128 * 128 * 2 * (4 + 2) + 64 * 128 * 8 + 3 * 4 * 128 * 4
    outs = [BOGUS, BOGUS, BOGUS, BOGUS, BOGUS, BOGUS]  # dq, dk, dv, ds, dgain, dtau

    def call(dt=tg.TG_BF16, dh=128, hq=4, hkv=2, s=BOGUS, out=BOGUS, o=outs, ws=BOGUS,
             ws_bytes=1 << 30, o32=None):
        return bwd(BOGUS, BOGUS, BOGUS, BOGUS, s, None, None, 128, hq, hkv, dh, 1e6, dt, out,
                   o32, BOGUS, BOGUS, *o, ws, ws_bytes, None)

    assert call(dt=tg.TG_F32, dh=96) == tg.TG_ERR_UNSUPPORTED
    assert call(dt=tg.TG_F32, o32=BOGUS) == tg.TG_ERR_INVALID_ARG  # fp32 takes no fp32 copy
    assert call(dt=7) == tg.TG_ERR_UNSUPPORTED
    assert call(dh=64) == tg.TG_ERR_UNSUPPORTED  # bf16 needs head_dim 128
    need32 = tg.tg_workspace_size(tg.TG_OP_GATED_ATTN_BWD, k=128, n_heads_q=4, n_heads_kv=2,
                                  head_dim=64, dtype=tg.TG_F32)
    assert call(dt=tg.TG_F32, dh=64, ws_bytes=need32 - 1) == tg.TG_ERR_WORKSPACE
    assert call(hkv=3) == tg.TG_ERR_INVALID_ARG  # hq % hkv != 0
    assert call(out=None) == tg.TG_ERR_INVALID_ARG
    assert call(s=None) == tg.TG_ERR_INVALID_ARG  # ds asked for without scores
    assert call(ws=ctypes.c_void_p(4096 + 8)) == tg.TG_ERR_INVALID_ARG  # misaligned workspace
    assert call(ws_bytes=need - 1) == tg.TG_ERR_WORKSPACE


def _bogus_model(**over):
    layers = (tg.TgLayer * 2)()
    for i in range(2):
        for name, _ in tg.TgLayer._fields_:
            setattr(layers[i], name, 4096)
        layers[i].q_norm = None
        layers[i].k_norm = None
        layers[i].gdn = None  # attention layers
    m = tg.TgModel(tg.TG_BF16, 2, 2048, 16, 8, 128, 6144, 256, 1e-6, 1e6, layers, 4096, 4096,
                   4096, None, 4096, None)
    for k, v in over.items():
        setattr(m, k, v)
    return m, layers


def _prefill(model, n, k, gate, ws_bytes):
    return tg._prefill(model, BOGUS, None, n, k, gate, BOGUS, BOGUS, None, None, None, BOGUS,
                       ws_bytes, None)


def test_prefill_multi_validation():
    m, keep = _bogus_model()
    big = 1 << 40

    def call(ks, n=1000, outs=None, ws_bytes=big):
        nb = len(ks)
        ks_c = (ctypes.c_int64 * max(nb, 1))(*ks)
        o = outs if outs is not None else [BOGUS] * max(nb, 1)
        outs_c = (ctypes.c_void_p * max(nb, 1))(*[x.value if x is not None else None for x in o])
        kept_c = (ctypes.c_void_p * max(nb, 1))(*([BOGUS.value] * max(nb, 1)))
        return tg._prefill_multi(ctypes.byref(m), BOGUS, None, n, ks_c, nb, 1, outs_c, kept_c,
                                 None, BOGUS, ws_bytes, None)

    assert call([]) == tg.TG_ERR_INVALID_ARG  # no budgets
    assert call([10] * 65) == tg.TG_ERR_INVALID_ARG  # more than TG_MAX_BUDGETS
    assert call([100, 1001]) == tg.TG_ERR_BUDGET  # k > n
    assert call([100, 0]) == tg.TG_ERR_BUDGET
    assert call([100, 200], outs=[BOGUS, None]) == tg.TG_ERR_INVALID_ARG
    p = dict(d_model=2048, n_heads_q=16, n_heads_kv=8, head_dim=128, d_score=256, d_ffn=6144,
             n_layers=2, gate_layer=1, dtype=tg.TG_BF16)
    need = tg.tg_workspace_size(tg.TG_OP_PREFILL, n=1000, k=500, **p)
    assert call([100, 500], ws_bytes=need - 1) == tg.TG_ERR_WORKSPACE


def test_prefill_validation():
    m, keep = _bogus_model()
    big = 1 << 40
    assert _prefill(ctypes.byref(m), 1000, 0, 1, big) == tg.TG_ERR_BUDGET
    assert _prefill(ctypes.byref(m), 1000, 1001, 1, big) == tg.TG_ERR_BUDGET
    assert _prefill(ctypes.byref(m), 1000, 100, 2, big) == tg.TG_ERR_INVALID_ARG  # gate past stack
    assert _prefill(ctypes.byref(m), 1000, 100, 1, 16) == tg.TG_ERR_WORKSPACE
    m2, keep2 = _bogus_model(head_dim=64)
    assert _prefill(ctypes.byref(m2), 1000, 100, 1, big) == tg.TG_ERR_UNSUPPORTED
    m3, keep3 = _bogus_model(d_ffn=6100)  # SwiGLU width must be a multiple of 128 in bf16
    assert _prefill(ctypes.byref(m3), 1000, 100, 1, big) == tg.TG_ERR_UNSUPPORTED
    assert _prefill(None, 1000, 100, 1, big) == tg.TG_ERR_INVALID_ARG
    keep[0].k_norm = 4096  # q_norm and k_norm come together
    assert _prefill(ctypes.byref(m), 1000, 100, 1, big) == tg.TG_ERR_INVALID_ARG


def test_prefill_validation_folded_norm_weights():
    """The optional folded-norm weights: bf16 models only, 16-byte aligned
    (they are TMA operands), and the FFN one only beside an FFN."""
    big = 1 << 40
    m, keep = _bogus_model()
    keep[1].wqkv_g = 4096 + 8
    assert _prefill(ctypes.byref(m), 1000, 100, 1, big) == tg.TG_ERR_INVALID_ARG
    m, keep = _bogus_model()
    keep[0].w_gate_up_g = 4096 + 2
    assert _prefill(ctypes.byref(m), 1000, 100, 1, big) == tg.TG_ERR_INVALID_ARG
    m, keep = _bogus_model(score_w1_g=4096 + 4)
    assert _prefill(ctypes.byref(m), 1000, 100, 1, big) == tg.TG_ERR_INVALID_ARG
    m, keep = _bogus_model(dtype=tg.TG_F32)
    assert _prefill(ctypes.byref(m), 1000, 100, 1, big) == tg.TG_ERR_UNSUPPORTED
    m, keep = _bogus_model(dtype=tg.TG_F32)
    for i in range(2):
        keep[i].wqkv_g = keep[i].w_gate_up_g = None
    assert _prefill(ctypes.byref(m), 1000, 100, 1, 16) == tg.TG_ERR_WORKSPACE  # valid otherwise


def test_prefill_host_validation():
    m, keep = _bogus_model()
    big = 1 << 40
    f = tg._prefill_host

    def call(x=BOGUS, n=1000, k=100, gate=1, ws_bytes=big, out=BOGUS):
        return f(ctypes.byref(m), x, None, n, k, gate, out, BOGUS, None, None, BOGUS, ws_bytes,
                 None)

    assert call(x=None) == tg.TG_ERR_INVALID_ARG
    assert call(out=None) == tg.TG_ERR_INVALID_ARG
    assert call(out=ctypes.c_void_p(4096 + 2)) == tg.TG_ERR_INVALID_ARG
    assert call(k=0) == tg.TG_ERR_BUDGET
    assert call(gate=2) == tg.TG_ERR_INVALID_ARG
    assert call(ws_bytes=16) == tg.TG_ERR_WORKSPACE


def test_fold_norm_weight_validation():
    f = tg._fold
    w, g, out = 4096, 1 << 20, 1 << 24
    assert f(None, g, 2, 8, out, None) == tg.TG_ERR_INVALID_ARG
    assert f(w, None, 2, 8, out, None) == tg.TG_ERR_INVALID_ARG
    assert f(w, g, 2, 8, None, None) == tg.TG_ERR_INVALID_ARG
    assert f(w, g, 0, 8, out, None) == tg.TG_ERR_INVALID_ARG
    assert f(w, g, 2, 0, out, None) == tg.TG_ERR_INVALID_ARG
    assert f(w, g, 2, 8, w + 16, None) == tg.TG_ERR_INVALID_ARG  # out overlaps w (32 bytes)
    assert f(w, g, 2, 8, w, None) == tg.TG_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="exercises the no-device error path")
def test_device_error_without_a_device_is_a_cuda_error():
    with pytest.raises(tg.TokenGateError) as ei:
        tg.tg_device_error()
    assert ei.value.status == tg.TG_ERR_CUDA


def _decode(model, kv, lens, gate=1, pos=1000, scores=None, n=0, kept=None, k_kept=0, ws_bytes=1 << 30,
            x=BOGUS, out=BOGUS):
    return tg._decode(model, x, pos, gate, kv, lens, scores, n, kept, k_kept, out, BOGUS, ws_bytes,
                      None)


def _bogus_kv(n_layers=2, **over):
    kv = (tg.TgKV * n_layers)()
    for i in range(n_layers):
        kv[i].k, kv[i].v = 4096, 8192
    lens = (ctypes.c_int64 * n_layers)(1000, 100)
    return kv, lens


def test_decode_validation():
    m, keep = _bogus_model()
    kv, lens = _bogus_kv()
    big = 1 << 30
    need = tg.tg_workspace_size(tg.TG_OP_DECODE, k=100, d_model=2048, n_heads_q=16, n_heads_kv=8,
                                head_dim=128, d_ffn=6144, dtype=tg.TG_BF16)
    assert 0 < need < big
    assert _decode(None, kv, lens) == tg.TG_ERR_INVALID_ARG
    assert _decode(ctypes.byref(m), None, lens) == tg.TG_ERR_INVALID_ARG
    assert _decode(ctypes.byref(m), kv, None) == tg.TG_ERR_INVALID_ARG
    assert _decode(ctypes.byref(m), kv, lens, gate=2) == tg.TG_ERR_INVALID_ARG   # gate past the stack
    assert _decode(ctypes.byref(m), kv, lens, pos=-1) == tg.TG_ERR_INVALID_ARG
    # bias inputs: kept_idx needed, k_kept within [1, n]
    assert _decode(ctypes.byref(m), kv, lens, scores=BOGUS, n=1000, kept=None, k_kept=100) == \
        tg.TG_ERR_INVALID_ARG
    assert _decode(ctypes.byref(m), kv, lens, scores=BOGUS, n=1000, kept=BOGUS, k_kept=0) == \
        tg.TG_ERR_BUDGET
    assert _decode(ctypes.byref(m), kv, lens, scores=BOGUS, n=1000, kept=BOGUS, k_kept=1001) == \
        tg.TG_ERR_BUDGET
    # an upper cache shorter than the kept prompt rows
    assert _decode(ctypes.byref(m), kv, lens, gate=0, scores=BOGUS, n=1000, kept=BOGUS,
                   k_kept=200) == tg.TG_ERR_INVALID_ARG
    assert _decode(ctypes.byref(m), kv, lens, ws_bytes=16) == tg.TG_ERR_WORKSPACE
    unaligned = ctypes.c_void_p(4096 + 2)
    assert _decode(ctypes.byref(m), kv, lens, x=unaligned) == tg.TG_ERR_INVALID_ARG
    kv[1].v = None
    assert _decode(ctypes.byref(m), kv, lens) == tg.TG_ERR_INVALID_ARG
    kv, lens = _bogus_kv()
    m2, keep2 = _bogus_model(head_dim=64)
    assert _decode(ctypes.byref(m2), kv, lens) == tg.TG_ERR_UNSUPPORTED
    m3, keep3 = _bogus_model(n_heads_q=24, n_heads_kv=8)  # GQA group of 3
    assert _decode(ctypes.byref(m3), kv, lens) == tg.TG_ERR_UNSUPPORTED
    m4, keep4 = _bogus_model(dtype=tg.TG_F32)
    assert _decode(ctypes.byref(m4), kv, lens) == tg.TG_ERR_UNSUPPORTED


def test_prefill_batch_validation():
    m, keep = _bogus_model()
    big = 1 << 40

    def call(cu, ks, model=None, ws_bytes=big):
        nb = len(ks)
        cu_c = (ctypes.c_int64 * len(cu))(*cu)
        ks_c = (ctypes.c_int64 * max(nb, 1))(*(ks or [0]))
        mm = model if model is not None else m
        return tg._prefill_batch(ctypes.byref(mm), BOGUS, None, cu_c, ks_c, nb, 1, BOGUS, BOGUS,
                                 None, BOGUS, ws_bytes, None)

    assert call([0], []) == tg.TG_ERR_INVALID_ARG  # empty batch
    assert call([1, 300], [10]) == tg.TG_ERR_INVALID_ARG  # cu_n[0] != 0
    assert call([0, 300, 300], [10, 10]) == tg.TG_ERR_INVALID_ARG  # an empty request
    assert call([0, 300, 400], [10, 101]) == tg.TG_ERR_BUDGET  # k > n
    assert call([0, 300, 400], [10, 0]) == tg.TG_ERR_BUDGET
    m32, keep32 = _bogus_model(dtype=tg.TG_F32)
    assert call([0, 300], [10], model=m32) == tg.TG_ERR_UNSUPPORTED
    cu = (ctypes.c_int64 * 3)(0, 300, 429)
    ks = (ctypes.c_int64 * 2)(100, 129)
    need = tg._prefill_batch_ws(ctypes.byref(m), cu, ks, 2)
    # the padded layout: 384 + 256 all-token rows, 128 + 256 kept rows
    p = dict(d_model=2048, n_heads_q=16, n_heads_kv=8, head_dim=128, d_score=256, d_ffn=6144,
             n_layers=2, gate_layer=1, dtype=tg.TG_BF16)
    assert need >= tg.tg_workspace_size(tg.TG_OP_PREFILL, n=640, k=384, **p)
    assert call([0, 300, 429], [100, 129], ws_bytes=need - 1) == tg.TG_ERR_WORKSPACE
    bad = (ctypes.c_int64 * 2)(100, 300)
    assert tg._prefill_batch_ws(ctypes.byref(m), cu, bad, 2) == 0


def _gdn_layer(hk=2, hv=4, dk=128, dv=128, W=4, eps=1e-6, ptrs=True):
    p = BOGUS.value if ptrs else None
    return tg.TgGdnLayer(hk, hv, dk, dv, W, p, p, p, p, eps)


def test_gated_deltanet_validation():
    f = tg._gdn
    L = _gdn_layer()
    need = tg._gdn_ws(ctypes.byref(L), 100)
    assert need > 0
    # the workspace holds the fp32 operands and the output before its norm
    assert need >= 4 * 100 * (2 * 2 * 128 + 4 * 128 + 4 * 128) + 2 * 4 * 4 * 128 * 36
    assert tg._gdn_ws(ctypes.byref(L), 0) == 0 or tg._gdn_ws(ctypes.byref(L), 0) < need
    ws = ctypes.c_void_p(1 << 20)

    def call(layer=L, T=100, dtype=tg.TG_BF16, conv_in=None, conv_out=None, s_in=None, s_out=None,
             ws_=ws, nbytes=need, ptr=BOGUS):
        return f(ctypes.byref(layer) if layer is not None else None, ptr, ptr, ptr, ptr, T, dtype,
                 conv_in, conv_out, s_in, s_out, ptr, ws_, nbytes, None)

    assert call(layer=None) == tg.TG_ERR_INVALID_ARG
    assert call(T=-1) == tg.TG_ERR_INVALID_ARG
    assert call(ptr=None) == tg.TG_ERR_INVALID_ARG
    assert call(dtype=7) == tg.TG_ERR_UNSUPPORTED
    assert call(layer=_gdn_layer(hk=3, hv=4)) == tg.TG_ERR_INVALID_ARG
    assert call(layer=_gdn_layer(W=0)) == tg.TG_ERR_INVALID_ARG
    assert call(layer=_gdn_layer(W=5)) == tg.TG_ERR_INVALID_ARG
    assert call(layer=_gdn_layer(eps=float("nan"))) == tg.TG_ERR_INVALID_ARG
    assert call(layer=_gdn_layer(ptrs=False)) == tg.TG_ERR_INVALID_ARG
    assert call(layer=_gdn_layer(dk=96)) == tg.TG_ERR_UNSUPPORTED
    assert call(layer=_gdn_layer(dv=48)) == tg.TG_ERR_UNSUPPORTED
    assert call(layer=_gdn_layer(dv=512)) == tg.TG_ERR_UNSUPPORTED
    assert call(nbytes=need - 1) == tg.TG_ERR_WORKSPACE
    assert call(ws_=None) == tg.TG_ERR_WORKSPACE
    assert call(ws_=ctypes.c_void_p((1 << 20) + 8)) == tg.TG_ERR_INVALID_ARG
    # overlapping carried state: conv rows always, S unless exactly in place
    base = 1 << 24
    assert call(conv_in=base, conv_out=base + 64) == tg.TG_ERR_INVALID_ARG
    assert call(s_in=base, s_out=base + 4) == tg.TG_ERR_INVALID_ARG
    names = [tg._kernel_name(i).decode() for i in (20, 21, 22, 23, 24, 25)]
    assert names == ["gdn_prep", "gdn_chunk", "gdn_recur", "gdn_out", "fold_norm", "unknown"]


def test_selftest_wait_validation():
    f = tg._selftest_wait
    assert f(3, 2_000_000, BOGUS, None, 0, None) == tg.TG_ERR_INVALID_ARG  # no such mode
    assert f(0, 10, BOGUS, None, 0, None) == tg.TG_ERR_INVALID_ARG  # limit below 1 us
    assert f(0, 2_000_000_000, BOGUS, None, 0, None) == tg.TG_ERR_INVALID_ARG  # above 1 s
    assert f(0, 2_000_000, None, None, 0, None) == tg.TG_ERR_INVALID_ARG  # no result buffer
    assert f(2, 2_000_000, BOGUS, None, 0, None) == tg.TG_ERR_WORKSPACE  # barrier words


def test_prefill_validation_hybrid_layers():
    """A Gated DeltaNet layer (hybrid stack): the mixer's sizes, the input
    projection's width (a multiple of 32 for the tensor-core GEMM) and the
    dtype are checked on the host."""
    m, keep = _bogus_model()
    big = 1 << 40
    gdn = tg.TgGdnLayer(4, 16, 64, 32, 4, 4096, 4096, 4096, 4096, 1e-6)  # width 1568 = 49 * 32
    keep[0].gdn = ctypes.addressof(gdn)
    assert tg._prefill_ws(ctypes.byref(m), 1000, 100) > \
        tg.tg_workspace_size(tg.TG_OP_PREFILL, n=1000, k=100, d_model=2048, n_heads_q=16,
                             n_heads_kv=8, head_dim=128, d_score=256, d_ffn=6144, n_layers=2,
                             gate_layer=1, dtype=tg.TG_BF16)
    assert _prefill(ctypes.byref(m), 1000, 100, 1, 16) == tg.TG_ERR_WORKSPACE  # passes validation
    bad = tg.TgGdnLayer(4, 16, 96, 32, 4, 4096, 4096, 4096, 4096, 1e-6)  # dk 96
    keep[0].gdn = ctypes.addressof(bad)
    assert _prefill(ctypes.byref(m), 1000, 100, 1, big) == tg.TG_ERR_UNSUPPORTED
    odd = tg.TgGdnLayer(2, 4, 64, 64, 4, 4096, 4096, 4096, 4096, 1e-6)  # width 520
    keep[0].gdn = ctypes.addressof(odd)
    assert _prefill(ctypes.byref(m), 1000, 100, 1, big) == tg.TG_ERR_UNSUPPORTED
    keep[0].gdn = ctypes.addressof(gdn)
    keep[0].w_in = None
    assert _prefill(ctypes.byref(m), 1000, 100, 1, big) == tg.TG_ERR_INVALID_ARG
    m32, keep32 = _bogus_model(dtype=tg.TG_F32)
    keep32[1].gdn = ctypes.addressof(gdn)
    assert _prefill(ctypes.byref(m32), 1000, 100, 1, big) == tg.TG_ERR_UNSUPPORTED
