"""Python binding of libtokengate, the B200 (sm_100a) gated-prefill library.

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch supplies device memory (tensors, workspaces) and streams. The names
mirror the C ABI in include/tokengate.h.

The shared library is built in-tree (``python
learned_token_pruning_score_b200/_build.py``); importing this package without
it raises ImportError -- there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtokengate.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is not built; run `python learned_token_pruning_score_b200/_build.py`")

_lib = ctypes.CDLL(LIB_PATH)

# ----------------------------------------------------------------- ABI types

TG_OK, TG_ERR_INVALID_ARG, TG_ERR_UNSUPPORTED, TG_ERR_BUDGET, TG_ERR_WORKSPACE, TG_ERR_CUDA = range(6)
TG_F32, TG_BF16 = 0, 1
(TG_OP_SCORE, TG_OP_TOPK_SELECT, TG_OP_COMPACT, TG_OP_GATED_ATTN, TG_OP_PREFILL, TG_OP_DECODE,
 TG_OP_GATED_ATTN_BWD) = range(7)

_c_i32, _c_i64, _c_f32, _c_p, _c_sz = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                       ctypes.c_void_p, ctypes.c_size_t)


class TgShape(ctypes.Structure):
    _fields_ = [("n", _c_i64), ("k", _c_i64), ("d_model", _c_i32), ("n_heads_q", _c_i32),
                ("n_heads_kv", _c_i32), ("head_dim", _c_i32), ("d_score", _c_i32),
                ("d_ffn", _c_i32), ("n_layers", _c_i32), ("gate_layer", _c_i32),
                ("dtype", ctypes.c_int)]


class TgLayer(ctypes.Structure):
    _fields_ = [(n, _c_p) for n in ("attn_norm", "wqkv", "q_norm", "k_norm", "wo", "ffn_norm",
                                    "w_gate_up", "w_down", "gain", "tau", "gdn", "w_in", "w_out",
                                    "wqkv_g", "w_gate_up_g")]


class TgModel(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("n_layers", _c_i32), ("d_model", _c_i32),
                ("n_heads_q", _c_i32), ("n_heads_kv", _c_i32), ("head_dim", _c_i32),
                ("d_ffn", _c_i32), ("d_score", _c_i32), ("norm_eps", _c_f32),
                ("rope_base", _c_f32), ("layers", ctypes.POINTER(TgLayer)),
                ("final_norm", _c_p), ("score_norm", _c_p), ("score_w1", _c_p),
                ("score_b1", _c_p), ("score_w2", _c_p), ("score_b2", _c_p),
                ("score_w1_g", _c_p)]


class TgKV(ctypes.Structure):
    _fields_ = [("k", _c_p), ("v", _c_p)]


class TgLayerTaps(ctypes.Structure):
    _fields_ = [("attn_out", _c_p), ("resid", _c_p), ("hidden", _c_p), ("mixer_in", _c_p)]


class TgGdnLayer(ctypes.Structure):
    _fields_ = [("n_heads_k", _c_i32), ("n_heads_v", _c_i32), ("head_dim_k", _c_i32),
                ("head_dim_v", _c_i32), ("conv_width", _c_i32), ("conv_w", _c_p),
                ("A_log", _c_p), ("dt_bias", _c_p), ("norm_w", _c_p), ("norm_eps", _c_f32)]


class TgTraceRecord(ctypes.Structure):
    _fields_ = [("kernel", _c_i32), ("layer", _c_i32), ("rows", _c_i64), ("ms", _c_f32),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_ci = ctypes.c_int
_workspace_size = _sig("tg_workspace_size", _c_sz, _ci, ctypes.POINTER(TgShape))
_score = _sig("tg_score", _ci, _c_p, _c_i64, _c_i32, _c_i32, _c_p, _c_f32, _c_p, _c_p, _c_p, _c_p,
              _ci, _c_p, _c_p, _c_sz, _c_p)
_topk = _sig("tg_topk_select", _ci, _c_p, _c_p, _c_i64, _c_i64, _c_p, _c_p, _c_sz, _c_p)
_linear = _sig("tg_linear", _ci, _c_p, _c_p, _c_p, _c_i64, _c_i32, _c_i32, _ci, _c_p, _c_p)
_fold = _sig("tg_fold_norm_weight", _ci, _c_p, _c_p, _c_i64, _c_i64, _c_p, _c_p)
_topk_noalloc = _sig("tg_topk_select_noalloc", _ci, _c_p, _c_p, _c_i64, _c_i64, _c_p, _c_p)
_compact = _sig("tg_compact", _ci, _c_p, _c_p, _c_p, _c_p, _c_i64, _c_i64, _c_i32, _ci, _c_p,
                _c_p, _c_p, _c_p)
_attn = _sig("tg_gated_attn_prefill", _ci, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i64,
             _c_i32, _c_i32, _c_i32, _c_f32, _ci, _c_p, _c_p, _c_sz, _c_p)
_attn_fwd = _sig("tg_gated_attn_forward", _ci, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i64,
                 _c_i32, _c_i32, _c_i32, _c_f32, _ci, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p)
_attn_bwd = _sig("tg_gated_attn_backward", _ci, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_i64,
                 _c_i32, _c_i32, _c_i32, _c_f32, _ci, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p,
                 _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p)
_prefill = _sig("tg_prefill", _ci, ctypes.POINTER(TgModel), _c_p, _c_p, _c_i64, _c_i64, _c_i32,
                _c_p, _c_p, _c_p, ctypes.POINTER(TgKV), ctypes.POINTER(TgLayerTaps), _c_p,
                _c_sz, _c_p)
_prefill_ws = _sig("tg_prefill_workspace_size", _c_sz, ctypes.POINTER(TgModel), _c_i64, _c_i64)
_prefill_host = _sig("tg_prefill_host", _ci, ctypes.POINTER(TgModel), _c_p, _c_p, _c_i64, _c_i64,
                     _c_i32, _c_p, _c_p, _c_p, ctypes.POINTER(TgKV), _c_p, _c_sz, _c_p)
_prefill_multi = _sig("tg_prefill_multi", _ci, ctypes.POINTER(TgModel), _c_p, _c_p, _c_i64,
                      ctypes.POINTER(_c_i64), _c_i32, _c_i32, ctypes.POINTER(_c_p),
                      ctypes.POINTER(_c_p), _c_p, _c_p, _c_sz, _c_p)
_prefill_batch_ws = _sig("tg_prefill_batch_workspace_size", _c_sz, ctypes.POINTER(TgModel),
                         ctypes.POINTER(_c_i64), ctypes.POINTER(_c_i64), _c_i32)
_prefill_batch = _sig("tg_prefill_batch", _ci, ctypes.POINTER(TgModel), _c_p, _c_p,
                      ctypes.POINTER(_c_i64), ctypes.POINTER(_c_i64), _c_i32, _c_i32, _c_p, _c_p,
                      _c_p, _c_p, _c_sz, _c_p)
_decode = _sig("tg_decode_step", _ci, ctypes.POINTER(TgModel), _c_p, _c_i64, _c_i32,
               ctypes.POINTER(TgKV), ctypes.POINTER(_c_i64), _c_p, _c_i64, _c_p, _c_i64, _c_p, _c_p,
               _c_sz, _c_p)
_gdn_ws = _sig("tg_gated_deltanet_workspace_size", _c_sz, ctypes.POINTER(TgGdnLayer), _c_i64)
_gdn = _sig("tg_gated_deltanet", _ci, ctypes.POINTER(TgGdnLayer), _c_p, _c_p, _c_p, _c_p, _c_i64,
            _ci, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p)
_status_string = _sig("tg_status_string", ctypes.c_char_p, _ci)
_last_cuda_error = _sig("tg_last_cuda_error", _ci)
_device_error = _sig("tg_device_error", _ci, ctypes.POINTER(ctypes.c_uint32), _ci)
_version = _sig("tg_version", ctypes.c_char_p)
_selftest_wait = _sig("tg_selftest_wait_timeout", _ci, _c_i32, _c_i64, _c_p, _c_p, _c_sz, _c_p)
_trace_start = _sig("tg_trace_start", _ci, _c_i32)
_trace_stop = _sig("tg_trace_stop", _c_i32, ctypes.POINTER(TgTraceRecord), _c_i32)
_kernel_name = _sig("tg_kernel_name", ctypes.c_char_p, _c_i32)


class TokenGateError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = f"{where}: {tg_status_string(status)}"
        if status == TG_ERR_CUDA:
            msg += f" (cudaError {_last_cuda_error()})"
        super().__init__(msg)
        self.status = status


def _check(status: int, where: str) -> None:
    if status != TG_OK:
        raise TokenGateError(status, where)


# ----------------------------------------------------------------- helpers


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TG_BF16
    if t.dtype == torch.float32:
        return TG_F32
    raise ValueError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libtokengate must be contiguous")
    return t.data_ptr()


def _stream(stream, device) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ws(nbytes: int, device, ws: Optional[torch.Tensor]) -> torch.Tensor:
    if ws is None:
        return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    if ws.numel() * ws.element_size() < nbytes:
        raise ValueError(f"workspace too small: {ws.numel() * ws.element_size()} < {nbytes}")
    return ws


def tg_status_string(status: int) -> str:
    return _status_string(status).decode()


def tg_version() -> str:
    return _version().decode()


def tg_workspace_size(op: int, n=0, k=0, d_model=0, n_heads_q=0, n_heads_kv=0, head_dim=0,
                      d_score=0, d_ffn=0, n_layers=0, gate_layer=0, dtype=TG_BF16) -> int:
    s = TgShape(n, k, d_model, n_heads_q, n_heads_kv, head_dim, d_score, d_ffn, n_layers,
                gate_layer, dtype)
    return int(_workspace_size(op, ctypes.byref(s)))


def tg_device_error(clear: bool = False) -> int:
    w = ctypes.c_uint32(0)
    _check(_device_error(ctypes.byref(w), int(clear)), "tg_device_error")
    return int(w.value)


def tg_selftest_wait_timeout(mode: int, limit_ns: int, device="cuda", stream=None) -> List[int]:
    """Runs the failure-detection self-test (mode 0: an mbarrier wait that
    never completes; 1: one that does; 2: the decode kernel's grid barrier,
    never reached) and returns the per-wait results (1 = completed, 0 = gave
    up after limit_ns). Synchronises the stream."""
    res = torch.full((4,), -1, dtype=torch.int32, device=device)
    ws = torch.zeros(16, dtype=torch.uint8, device=device)
    _check(_selftest_wait(int(mode), int(limit_ns), _ptr(res), _ptr(ws), ws.numel(),
                          _stream(stream, res.device)), "tg_selftest_wait_timeout")
    torch.cuda.synchronize(res.device)
    return res.cpu().tolist()


def tg_trace_start(capacity: int = 65536) -> None:
    """Bracket every library kernel launched from this thread with CUDA events."""
    _check(_trace_start(capacity), "tg_trace_start")


def tg_trace_stop() -> List[dict]:
    """Stop tracing; one dict per traced launch: kernel, layer, rows, ms,
    flops, bytes (algorithmic work of the launch)."""
    cap = 1 << 20
    buf = (TgTraceRecord * cap)()
    n = _trace_stop(buf, cap)
    if n < 0:
        raise TokenGateError(-n, "tg_trace_stop")
    return [dict(kernel=_kernel_name(r.kernel).decode(), layer=r.layer, rows=r.rows, ms=r.ms,
                 flops=r.flops, bytes=r.bytes) for r in buf[:n]]


# ----------------------------------------------------------------- the calls


def tg_score(x, norm_w, w1, w2, b1=None, b2=None, eps: float = 1e-6, scores=None, ws=None,
             stream=None) -> torch.Tensor:
    n, d = x.shape
    f = w1.shape[0]
    if scores is None:
        scores = torch.empty(n, dtype=torch.float32, device=x.device)
    dt = _dt(x)
    need = tg_workspace_size(TG_OP_SCORE, n=n, d_model=d, d_score=f, dtype=dt)
    ws = _ws(need, x.device, ws)
    _check(_score(_ptr(x), n, d, f, _ptr(norm_w), eps, _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), dt,
                  _ptr(scores), _ptr(ws), ws.numel(), _stream(stream, x.device)), "tg_score")
    return scores


def tg_topk_select(scores, protect, k: int, kept_idx=None, ws=None, stream=None) -> torch.Tensor:
    n = scores.shape[0]
    if kept_idx is None:
        kept_idx = torch.empty(k, dtype=torch.int32, device=scores.device)
    need = tg_workspace_size(TG_OP_TOPK_SELECT, n=n)
    ws = _ws(need, scores.device, ws)
    _check(_topk(_ptr(scores), _ptr(protect), n, k, _ptr(kept_idx), _ptr(ws), ws.numel(),
                 _stream(stream, scores.device)), "tg_topk_select")
    return kept_idx


def tg_linear(x, w, residual=None, y=None, stream=None) -> torch.Tensor:
    """y = x . w^T (+ residual): x [m, k], w [n, k] (nn.Linear layout)."""
    m, k = x.shape
    n = w.shape[0]
    if y is None:
        y = torch.empty(m, n, dtype=x.dtype, device=x.device)
    _check(_linear(_ptr(x), _ptr(w), _ptr(residual), m, n, k, _dt(x), _ptr(y),
                   _stream(stream, x.device)), "tg_linear")
    return y


def tg_fold_norm_weight(w, g, out=None, stream=None) -> torch.Tensor:
    """W_g = bf16(W . diag(g)): w [rows, cols] bf16, g [cols] fp32 (the weight
    of the RMSNorm in front of the projection w)."""
    rows, cols = w.shape
    if out is None:
        out = torch.empty_like(w)
    _check(_fold(_ptr(w), _ptr(g), rows, cols, _ptr(out), _stream(stream, w.device)),
           "tg_fold_norm_weight")
    return out


SELECT_NOALLOC_MAX_N = 1 << 20


def tg_topk_select_noalloc(scores, protect, k: int, kept_idx=None, stream=None) -> torch.Tensor:
    """tg_topk_select with no workspace: the library keeps this call's scratch
    in a static device array (n <= SELECT_NOALLOC_MAX_N). For callers that can
    pass only inputs and outputs. Calls that overlap on the GPU share that
    array and race; the first call on a device should precede stream capture."""
    n = scores.shape[0]
    if n > SELECT_NOALLOC_MAX_N:
        raise ValueError(f"n={n} exceeds the allocation-free limit {SELECT_NOALLOC_MAX_N}; "
                         "use tg_topk_select with a workspace")
    if kept_idx is None:
        kept_idx = torch.empty(k, dtype=torch.int32, device=scores.device)
    _check(_topk_noalloc(_ptr(scores), _ptr(protect), n, k, _ptr(kept_idx),
                         _stream(stream, scores.device)), "tg_topk_select_noalloc")
    return kept_idx


def tg_compact(x, kept_idx, pos_in=None, scores=None, x_out=None, pos_out=None, scores_out=None,
               stream=None):
    n, d = x.shape
    k = kept_idx.shape[0]
    if x_out is None:
        x_out = torch.empty(k, d, dtype=x.dtype, device=x.device)
    if pos_out is None:
        pos_out = torch.empty(k, dtype=torch.int32, device=x.device)
    if scores is not None and scores_out is None:
        scores_out = torch.empty(k, dtype=torch.float32, device=x.device)
    _check(_compact(_ptr(x), _ptr(pos_in), _ptr(scores), _ptr(kept_idx), n, k, d, _dt(x),
                    _ptr(x_out), _ptr(pos_out), _ptr(scores_out), _stream(stream, x.device)),
           "tg_compact")
    return x_out, pos_out, scores_out


def tg_gated_attn_prefill(q, k, v, pos, s=None, gain=None, tau=None, rope_base: float = 1e6,
                          out=None, ws=None, stream=None) -> torch.Tensor:
    t, hq, dh = q.shape
    hkv = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    dt = _dt(q)
    need = tg_workspace_size(TG_OP_GATED_ATTN, k=t, n_heads_q=hq, n_heads_kv=hkv, head_dim=dh,
                             dtype=dt)
    ws = _ws(need, q.device, ws)
    _check(_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), _ptr(s), _ptr(gain), _ptr(tau), t, hq, hkv,
                 dh, rope_base, dt, _ptr(out), _ptr(ws), ws.numel(), _stream(stream, q.device)),
           "tg_gated_attn_prefill")
    return out


def tg_gated_attn_forward(q, k, v, pos, s=None, gain=None, tau=None, rope_base: float = 1e6,
                          out=None, lse=None, out_f32=None, want_f32: bool = True, ws=None,
                          stream=None):
    """tg_gated_attn_prefill plus the per-row log-sum-exp [hq, t] and (when
    want_f32) the output before rounding [t, hq, dh] fp32, both of which
    tg_gated_attn_backward takes. Returns (out, lse, out_f32 or None)."""
    t, hq, dh = q.shape
    hkv = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(hq, t, dtype=torch.float32, device=q.device)
    if out_f32 is None and want_f32 and q.dtype == torch.bfloat16:
        out_f32 = torch.empty(t, hq, dh, dtype=torch.float32, device=q.device)
    dt = _dt(q)
    need = tg_workspace_size(TG_OP_GATED_ATTN, k=t, n_heads_q=hq, n_heads_kv=hkv, head_dim=dh,
                             dtype=dt)
    ws = _ws(need, q.device, ws)
    _check(_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), _ptr(s), _ptr(gain), _ptr(tau), t, hq,
                     hkv, dh, rope_base, dt, _ptr(out), _ptr(lse), _ptr(out_f32), _ptr(ws),
                     ws.numel(), _stream(stream, q.device)), "tg_gated_attn_forward")
    return out, lse, out_f32


def tg_gated_attn_backward(q, k, v, pos, out, lse, dout, s=None, gain=None, tau=None,
                           rope_base: float = 1e6, out_f32=None, dq=None, dk=None, dv=None,
                           ds=None, dgain=None, dtau=None, want_ds: bool = True, ws=None,
                           stream=None):
    """Gradients (dq, dk, dv, ds, dgain, dtau) of tg_gated_attn_forward for dout.
    ds is None when s is None (or want_ds is False)."""
    t, hq, dh = q.shape
    hkv = k.shape[1]
    dev = q.device
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ds is None and s is not None and want_ds:
        ds = torch.empty(t, dtype=torch.float32, device=dev)
    dgain = torch.empty(hq, dtype=torch.float32, device=dev) if dgain is None else dgain
    dtau = torch.empty(hq, dtype=torch.float32, device=dev) if dtau is None else dtau
    need = tg_workspace_size(TG_OP_GATED_ATTN_BWD, k=t, n_heads_q=hq, n_heads_kv=hkv,
                             head_dim=dh, dtype=_dt(q))
    ws = _ws(need, dev, ws)
    _check(_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), _ptr(s), _ptr(gain), _ptr(tau), t, hq,
                     hkv, dh, rope_base, _dt(q), _ptr(out), _ptr(out_f32), _ptr(lse), _ptr(dout),
                     _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds), _ptr(dgain), _ptr(dtau), _ptr(ws),
                     ws.numel(), _stream(stream, dev)), "tg_gated_attn_backward")
    return dq, dk, dv, ds, dgain, dtau


@dataclass
class GdnLayer:
    """Parameters of a Gated DeltaNet layer's token mixer (fp32 device
    tensors) plus the ctypes view tg_gated_deltanet takes: conv_w [C, W],
    A_log [hv], dt_bias [hv], norm_w [dv], with C = 2 hk dk + hv dv."""

    n_heads_k: int
    n_heads_v: int
    head_dim_k: int
    head_dim_v: int
    conv_w: torch.Tensor
    A_log: torch.Tensor
    dt_bias: torch.Tensor
    norm_w: torch.Tensor
    eps: float = 1e-6

    def __post_init__(self):
        self.conv_width = self.conv_w.shape[1]
        self.channels = 2 * self.n_heads_k * self.head_dim_k + self.n_heads_v * self.head_dim_v
        self.c = TgGdnLayer(self.n_heads_k, self.n_heads_v, self.head_dim_k, self.head_dim_v,
                            self.conv_width, _ptr(self.conv_w), _ptr(self.A_log),
                            _ptr(self.dt_bias), _ptr(self.norm_w), self.eps)


def tg_gated_deltanet_workspace_size(layer: GdnLayer, T: int) -> int:
    return int(_gdn_ws(ctypes.byref(layer.c), T))


def tg_gated_deltanet(layer: GdnLayer, qkv, z, a, b, conv_in=None, state_in=None,
                      want_state: bool = True, y=None, conv_out=None, state_out=None, ws=None,
                      stream=None):
    """The Gated DeltaNet mixer over the T rows of qkv [T, C], z [T, hv dv],
    a, b [T, hv] (one dtype, bf16 or fp32). Returns (y, conv_out, state_out);
    the last two are None when want_state is False and none is passed."""
    T = qkv.shape[0]
    dev = qkv.device
    hv, dv, dk = layer.n_heads_v, layer.head_dim_v, layer.head_dim_k
    y = torch.empty(T, hv * dv, dtype=qkv.dtype, device=dev) if y is None else y
    if want_state and conv_out is None and layer.conv_width > 1:
        conv_out = torch.empty(layer.conv_width - 1, layer.channels, dtype=qkv.dtype, device=dev)
    if want_state and state_out is None:
        state_out = torch.empty(hv, dv, dk, dtype=torch.float32, device=dev)
    ws = _ws(tg_gated_deltanet_workspace_size(layer, T), dev, ws)
    _check(_gdn(ctypes.byref(layer.c), _ptr(qkv), _ptr(z), _ptr(a), _ptr(b), T, _dt(qkv),
                _ptr(conv_in), _ptr(conv_out), _ptr(state_in), _ptr(state_out), _ptr(y),
                _ptr(ws), ws.numel(), _stream(stream, dev)), "tg_gated_deltanet")
    return y, conv_out, state_out


@dataclass
class Model:
    """Device tensors of a decoder stack plus the ctypes view tg_prefill takes.

    layers: one dict per layer with keys attn_norm, wqkv, wo, ffn_norm,
    w_gate_up, w_down (optional), q_norm/k_norm (optional), gain/tau
    (optional; used above the gate). Matrices in the model dtype, vectors fp32.
    A hybrid model's Gated DeltaNet layer has instead of wqkv/wo the keys gdn
    (a GdnLayer: the mixer's parameters), w_in [C + hv dv + 2 hv, d] and
    w_out [d, hv dv]; attn_norm is then the norm before the mixer.

    fold_norms (bf16): also keep wqkv, w_gate_up and score_w1 with the weight
    of the RMSNorm in front of each folded in (tg_fold_norm_weight, made once
    here), so that tg_prefill skips the norm kernels whose input rows come
    straight from a residual GEMM.
    """

    n_heads_q: int
    n_heads_kv: int
    head_dim: int
    layers: List[Dict[str, torch.Tensor]]
    score: Dict[str, torch.Tensor]  # score_norm, score_w1, score_w2, score_b1?, score_b2?
    final_norm: Optional[torch.Tensor] = None
    eps: float = 1e-6
    rope_base: float = 1e6
    fold_norms: bool = True

    def __post_init__(self):
        w = next(lw["wqkv"] if "wqkv" in lw else lw["w_in"] for lw in self.layers)
        self.dtype = _dt(w)
        self.d_model = w.shape[1]
        gu = next((lw["w_gate_up"] for lw in self.layers if lw.get("w_gate_up") is not None),
                  None)
        self.d_ffn = 0 if gu is None else gu.shape[0] // 2
        self.d_score = self.score["score_w1"].shape[0]
        fold = self.fold_norms and self.dtype == TG_BF16
        self.fold_norms = fold  # what the model does (folding is bf16 only)
        # folded-norm weights, kept beside the layer dicts (which stay as given)
        self._folded = [{} for _ in self.layers]
        if fold:
            for lw, fw in zip(self.layers, self._folded):
                if lw.get("wqkv") is not None and lw.get("gdn") is None:
                    fw["wqkv_g"] = tg_fold_norm_weight(lw["wqkv"], lw["attn_norm"])
                if lw.get("w_gate_up") is not None:
                    fw["w_gate_up_g"] = tg_fold_norm_weight(lw["w_gate_up"], lw["ffn_norm"])
            self._score_w1_g = tg_fold_norm_weight(self.score["score_w1"],
                                                   self.score["score_norm"])
        else:
            self._score_w1_g = None
        arr = (TgLayer * len(self.layers))()
        for i, lw in enumerate(self.layers):
            for name, _ in TgLayer._fields_:
                if name == "gdn":
                    g = lw.get("gdn")
                    arr[i].gdn = None if g is None else ctypes.addressof(g.c)
                elif name in ("wqkv_g", "w_gate_up_g"):
                    setattr(arr[i], name, _ptr(self._folded[i].get(name)))
                else:
                    setattr(arr[i], name, _ptr(lw.get(name)))
        self._layers_c = arr
        self.c = TgModel(self.dtype, len(self.layers), self.d_model, self.n_heads_q,
                         self.n_heads_kv, self.head_dim, self.d_ffn, self.d_score, self.eps,
                         self.rope_base, arr, _ptr(self.final_norm),
                         _ptr(self.score["score_norm"]), _ptr(self.score["score_w1"]),
                         _ptr(self.score.get("score_b1")), _ptr(self.score["score_w2"]),
                         _ptr(self.score.get("score_b2")), _ptr(self._score_w1_g))

    def decode_workspace_size(self, k_kept: int) -> int:
        return tg_workspace_size(TG_OP_DECODE, k=k_kept, d_model=self.d_model,
                                 n_heads_q=self.n_heads_q, n_heads_kv=self.n_heads_kv,
                                 head_dim=self.head_dim, d_ffn=self.d_ffn, dtype=self.dtype)

    def workspace_size(self, n: int, k: int, gate_layer: int) -> int:
        return int(_prefill_ws(ctypes.byref(self.c), n, k))


def tg_decode_step(model: Model, x, pos: int, gate_layer: int, kv: Sequence, lens: Sequence[int],
                   scores=None, kept_idx=None, out=None, ws=None, stream=None):
    """One generated token through every layer after a gated prefill.

    x [d] or [1, d] bf16; kv: per-layer (k_cache, v_cache) [cap, hkv, dh]
    bf16 with room for the new row; lens: per-layer rows before this step (the
    token's k/v go to row lens[l]; the caller advances lens). scores [n] /
    kept_idx [k] from tg_prefill give the upper layers' gate bias (None: no
    bias). Returns out [1, d]."""
    d = x.shape[-1]
    if out is None:
        out = torch.empty(1, d, dtype=x.dtype, device=x.device)
    k_kept = 0 if kept_idx is None else int(kept_idx.numel())
    ws = _ws(model.decode_workspace_size(k_kept), x.device, ws)
    kv_c = (TgKV * len(model.layers))()
    for i, (kc, vc) in enumerate(kv):
        kv_c[i].k, kv_c[i].v = _ptr(kc), _ptr(vc)
    lens_c = (_c_i64 * len(model.layers))(*[int(t) for t in lens])
    n_scores = 0 if scores is None else int(scores.numel())
    _check(_decode(ctypes.byref(model.c), _ptr(x), int(pos), gate_layer, kv_c, lens_c,
                   _ptr(scores), n_scores, _ptr(kept_idx), k_kept, _ptr(out), _ptr(ws),
                   ws.numel(), _stream(stream, x.device)), "tg_decode_step")
    return out


def tg_prefill_host(model: Model, x_host, protect, k: int, gate_layer: int, device=None,
                    out=None, kept_idx=None, scores=None, kv: Optional[Sequence] = None, ws=None,
                    stream=None):
    """tg_prefill with x_host [n, d] a CPU tensor (pinned for the copy to
    overlap layer 0); protect, out, kept_idx, scores and kv on the device.
    Returns (out [k, d], kept_idx [k], scores [n] or None)."""
    if x_host.is_cuda:
        raise ValueError("x_host must be a host (CPU) tensor; use tg_prefill for device input")
    n, d = x_host.shape
    dev = torch.device(device) if device is not None else (
        protect.device if protect is not None else torch.device("cuda", torch.cuda.current_device()))
    if out is None:
        out = torch.empty(k, d, dtype=x_host.dtype, device=dev)
    if kept_idx is None:
        kept_idx = torch.empty(k, dtype=torch.int32, device=dev)
    ws = _ws(model.workspace_size(n, k, gate_layer), dev, ws)
    kv_c = None
    if kv is not None:
        kv_c = (TgKV * len(model.layers))()
        for i, pair in enumerate(kv):
            if pair is not None:
                kv_c[i].k, kv_c[i].v = _ptr(pair[0]), _ptr(pair[1])
    _check(_prefill_host(ctypes.byref(model.c), _ptr(x_host), _ptr(protect), n, k,
                         gate_layer, _ptr(out), _ptr(kept_idx), _ptr(scores), kv_c, _ptr(ws),
                         ws.numel(), _stream(stream, dev)), "tg_prefill_host")
    return out, kept_idx, scores


def tg_prefill(model: Model, x, protect, k: int, gate_layer: int, out=None, kept_idx=None,
               scores=None, kv: Optional[Sequence] = None, taps: Optional[Sequence] = None,
               ws=None, stream=None):
    """Returns (out [k, d], kept_idx [k], scores [n] or None).

    kv: per-layer (k_cache, v_cache) tensors or None entries. taps: per-layer
    dicts (or None) with any of the keys attn_out ([rows, hq*dh], the
    attention output before the output projection), resid ([rows, d], the
    residual stream after the attention sub-layer) and hidden (the layer's
    output: [n, d] below the gate, [k, d] at and above it); rows = n at and
    below the gate, k above it."""
    n, d = x.shape
    if out is None:
        out = torch.empty(k, d, dtype=x.dtype, device=x.device)
    if kept_idx is None:
        kept_idx = torch.empty(k, dtype=torch.int32, device=x.device)
    ws = _ws(model.workspace_size(n, k, gate_layer), x.device, ws)
    kv_c = None
    if kv is not None:
        kv_c = (TgKV * len(model.layers))()
        for i, pair in enumerate(kv):
            if pair is not None:
                kv_c[i].k, kv_c[i].v = _ptr(pair[0]), _ptr(pair[1])
    taps_c = None
    if taps is not None:
        taps_c = (TgLayerTaps * len(model.layers))()
        for i, t in enumerate(taps):
            if t:
                taps_c[i].attn_out = _ptr(t.get("attn_out"))
                taps_c[i].resid = _ptr(t.get("resid"))
                taps_c[i].hidden = _ptr(t.get("hidden"))
                taps_c[i].mixer_in = _ptr(t.get("mixer_in"))
    _check(_prefill(ctypes.byref(model.c), _ptr(x), _ptr(protect), n, k, gate_layer, _ptr(out),
                    _ptr(kept_idx), _ptr(scores), kv_c, taps_c, _ptr(ws), ws.numel(),
                    _stream(stream, x.device)), "tg_prefill")
    return out, kept_idx, scores


def tg_prefill_multi(model: Model, x, protect, ks: Sequence[int], gate_layer: int, outs=None,
                     kept_idx=None, scores=None, ws=None, stream=None):
    """The gated prefill at several budgets of one request: the layers below
    the gate and the scores run once. Returns (outs, kept_idx, scores), the
    first two lists with one tensor per budget."""
    n, d = x.shape
    nb = len(ks)
    if outs is None:
        outs = [torch.empty(k, d, dtype=x.dtype, device=x.device) for k in ks]
    if kept_idx is None:
        kept_idx = [torch.empty(k, dtype=torch.int32, device=x.device) for k in ks]
    ws = _ws(model.workspace_size(n, max(ks), gate_layer), x.device, ws)
    ks_c = (_c_i64 * nb)(*ks)
    outs_c = (_c_p * nb)(*[_ptr(t) for t in outs])
    kept_c = (_c_p * nb)(*[_ptr(t) for t in kept_idx])
    _check(_prefill_multi(ctypes.byref(model.c), _ptr(x), _ptr(protect), n, ks_c, nb, gate_layer,
                          outs_c, kept_c, _ptr(scores), _ptr(ws), ws.numel(),
                          _stream(stream, x.device)), "tg_prefill_multi")
    return outs, kept_idx, scores


def tg_prefill_batch(model: Model, x, protect, lens: Sequence[int], ks: Sequence[int],
                     gate_layer: int, out=None, kept_idx=None, scores=None, ws=None, stream=None):
    """The gated prefill of len(lens) requests packed back to back in x
    (request b: lens[b] rows, budget ks[b]). Returns (out [sum ks, d],
    kept_idx [sum ks] (request-local indices), scores [sum lens] or None),
    each request's rows after the previous ones'."""
    d = x.shape[1]
    nb = len(lens)
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + int(n))
    if cu[-1] != x.shape[0]:
        raise ValueError("sum of lens must equal x's rows")
    cu_c = (_c_i64 * (nb + 1))(*cu)
    ks_c = (_c_i64 * nb)(*[int(k) for k in ks])
    tot_k = int(sum(ks))
    if out is None:
        out = torch.empty(tot_k, d, dtype=x.dtype, device=x.device)
    if kept_idx is None:
        kept_idx = torch.empty(tot_k, dtype=torch.int32, device=x.device)
    need = _prefill_batch_ws(ctypes.byref(model.c), cu_c, ks_c, nb)
    if need == 0:
        raise ValueError("invalid batch sizes")
    ws = _ws(need, x.device, ws)
    _check(_prefill_batch(ctypes.byref(model.c), _ptr(x), _ptr(protect), cu_c, ks_c, nb,
                          gate_layer, _ptr(out), _ptr(kept_idx), _ptr(scores), _ptr(ws),
                          ws.numel(), _stream(stream, x.device)), "tg_prefill_batch")
    return out, kept_idx, scores


__all__ = [
    "tg_score", "tg_linear", "tg_fold_norm_weight", "tg_prefill_host", "tg_topk_select", "tg_topk_select_noalloc", "SELECT_NOALLOC_MAX_N", "tg_compact", "tg_gated_attn_prefill", "tg_gated_attn_forward", "tg_gated_attn_backward", "tg_prefill", "tg_prefill_multi", "tg_prefill_batch", "tg_decode_step",
    "tg_workspace_size", "tg_status_string", "tg_device_error", "tg_version", "Model",
    "tg_selftest_wait_timeout",
    "TokenGateError", "LIB_PATH", "tg_trace_start", "tg_trace_stop", "TG_OK", "TG_ERR_INVALID_ARG", "TG_ERR_UNSUPPORTED",
    "TG_ERR_BUDGET", "TG_ERR_WORKSPACE", "TG_ERR_CUDA", "TG_F32", "TG_BF16", "TG_OP_SCORE",
    "TG_OP_TOPK_SELECT", "TG_OP_COMPACT", "TG_OP_GATED_ATTN", "TG_OP_PREFILL", "TG_OP_DECODE",
    "TG_OP_GATED_ATTN_BWD", "GdnLayer", "tg_gated_deltanet", "tg_gated_deltanet_workspace_size",
]
