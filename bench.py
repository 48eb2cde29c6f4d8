#!/usr/bin/env python
"""Benchmark of the gated prefill on B200.

Default workload: the 28-layer Qwen3-1.7B-shaped gated prefill in bf16 at
batch 1 -- N = 32768 tokens, gate at layer 1, K = 4096 kept tokens, the last
128 protected, qk-norm on, seeded random weights and N(0,1) hidden states in
place of the embedding lookup. One step = one tg_prefill call: every stage
of the path (dense layers over N, scorer, select, compact, gated layers over
K, final norm).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    python bench.py --sweep      # select+compact sweep, the 16K and 128K layers alone
    python bench.py --case attn|attn_bwd|layer|gemm|decode|gdn|score|select [--rows R]
                                 # one kernel family alone: the commands the ncu
                                 # summaries under profiles/ were captured with

Prints one JSON line (rank 0). `value` = tokens/s (N / TTFT) summed over the
ranks; ranks run independent replicas (the path has no exchange step).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "gated-prefill tokens/s (N/TTFT) at N=32K"
UNIT = "tokens/s"
WORKLOAD = synth.QWEN_PREFILL_32K
HEADLINE_K = 4096
SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
# library kernels behind one traced record (the rest: one each). The select
# is one cluster launch up to 131072 tokens, else five kernels; a copy is a
# cudaMemcpyAsync, not a kernel of the library.
LAUNCHES_PER_RECORD = {"rope_prep": 2, "copy": 0}
SELECT_ONE_LAUNCH_MAX_N = 131072


def launches_of(rec) -> int:
    if rec["kernel"] == "select":
        return 1 if rec["rows"] <= SELECT_ONE_LAUNCH_MAX_N else 5
    return LAUNCHES_PER_RECORD.get(rec["kernel"], 1)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"],
                    bf16_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ----------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi sampled every 100 ms while the timed region runs."""

    def __init__(self, gpu_index: int):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={SMI_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, reasons, mx = [], set(), None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for nm, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- helpers


def kernel_source_hash(name: str) -> str:
    """First 12 hex digits of the sha256 of the kernel's source file and the
    device header it includes."""
    files = {"attention_tc": "k_attn_tc.cu", "gemm_tc": "k_gemm_tc.cu"}
    key = "gemm_tc" if name.startswith("gemm_tc") else name
    f = files.get(key)
    if f is None:
        return ""
    h = hashlib.sha256()
    for part in (f, "tg_device.cuh"):
        with open(os.path.join(ROOT, "learned_token_pruning_score_b200", "csrc", part), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def traffic_from_profiles(kernel: str, source: str, workload: str):
    """dram bytes per launch of `kernel` (a kernel family's launches in the
    workload, e.g. attention_tc_gated) from the committed ncu summary, or
    None if absent or taken on another revision of the source of the family
    `source`."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash(source)
    if not want:
        return None
    with open(path) as fh:
        for line in fh:
            if line.startswith("#") or not line.strip():
                continue
            kv = dict(tok.split("=", 1) for tok in line.split() if "=" in tok)
            if kv.get("kernel") == kernel and kv.get("workload") == workload and \
                    kv.get("src") == want:
                return float(kv["dram_bytes_per_launch"])
    return None


def build_model(tg, torch, w, device):
    p = synth.torch_model_params(w, seed=w.seed, device=device)
    score = {k: p[k] for k in ("score_norm", "score_w1", "score_b1", "score_w2", "score_b2")}
    return tg.Model(n_heads_q=w.hq, n_heads_kv=w.hkv, head_dim=w.dh, layers=p["layers"],
                    score=score, final_norm=p["final_norm"], eps=w.eps, rope_base=w.rope_base)


def kv_buffers(torch, w, k, device, extra_rows=0):
    """Per-layer KV caches: n rows at/below the gate, k rows above, plus
    `extra_rows` of room for generated tokens."""
    out = []
    for li in range(w.n_layers):
        rows = (w.n if li <= w.gate_layer else k) + extra_rows
        out.append((torch.empty(rows, w.hkv, w.dh, dtype=torch.bfloat16, device=device),
                    torch.empty(rows, w.hkv, w.dh, dtype=torch.bfloat16, device=device)))
    return out


def decode_step_bytes(w, lens):
    """Algorithmic HBM bytes of one decode step: every weight matrix once,
    every cached k/v row once, the new k/v rows written (bf16)."""
    per_layer_w = 2 * ((w.hq + 2 * w.hkv) * w.dh * w.d + w.d * w.hq * w.dh +
                       (3 * w.inter * w.d if w.inter else 0))
    kv = sum((2 * t + 2) * w.hkv * w.dh * 2 for t in lens)
    return w.n_layers * per_layer_w + kv


def decode_bench(tg, torch, model, w, kk, dense, steps, warmup, device, stream, pk):
    """Prefill the prompt (gated at budget kk, or dense), then decode
    warmup + steps tokens back to back over the caches it wrote. Returns the
    timed steps' ms per token and the per-kernel split of a traced step."""
    extra = warmup + steps + 1
    kvb = kv_buffers(torch, w, w.n if dense else kk, device, extra_rows=extra)
    x = synth.torch_hidden_states(w, seed=w.seed + 2000, device=str(device))
    prot = torch.zeros(w.n, dtype=torch.uint8, device=device)
    prot[w.n - w.n_protect:] = 1
    k = w.n if dense else kk
    scores = torch.empty(w.n, dtype=torch.float32, device=device)
    _, kept, _ = tg.tg_prefill(model, x, prot, k, w.gate_layer, scores=scores, kv=kvb, stream=stream)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed + 3000)
    toks = torch.randn(extra, w.d, device=device, generator=g).to(torch.bfloat16)
    lens0 = [(w.n if (dense or li <= w.gate_layer) else kk) for li in range(w.n_layers)]
    out = torch.empty(1, w.d, dtype=torch.bfloat16, device=device)
    ws = torch.empty(model.decode_workspace_size(k), dtype=torch.uint8, device=device)
    sc, ki = (None, None) if dense else (scores, kept)

    def step(i):
        tg.tg_decode_step(model, toks[i], w.n + i, w.gate_layer, kvb, [t + i for t in lens0],
                          scores=sc, kept_idx=ki, out=out, ws=ws, stream=stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(warmup, warmup + steps):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    tg.tg_trace_start(1 << 12)
    step(warmup + steps)
    torch.cuda.synchronize()
    tr = tg.tg_trace_stop()
    by = {}
    for r in tr:
        e = by.setdefault(r["kernel"], {"ms": 0.0, "bytes": 0.0, "launches": 0})
        e["ms"] += r["ms"]
        e["bytes"] += r["bytes"]
        e["launches"] += 1
    for e in by.values():
        e["gbs"] = e["bytes"] / (e["ms"] / 1e3) / 1e9 if e["ms"] > 0 else 0.0
    mid = [t + warmup + steps // 2 for t in lens0]
    nbytes = decode_step_bytes(w, mid)
    res = {"ms_per_token": ms, "tokens_per_s": 1e3 / ms, "bytes_per_step": nbytes,
           "gbs": nbytes / (ms / 1e3) / 1e9, "hbm_frac": nbytes / (ms / 1e3) / 1e9 / pk["hbm"],
           "cache_rows": {"at_or_below_gate": lens0[0], "above_gate": lens0[-1]},
           "steps": steps, "warmup": warmup, "launches_per_step": len(tr), "by_kernel": by}
    del kvb, ws, x, toks
    torch.cuda.empty_cache()
    return res


def dense_model(tg, model):
    layers = [{k: v for k, v in lw.items() if k not in ("gain", "tau")} for lw in model.layers]
    return tg.Model(n_heads_q=model.n_heads_q, n_heads_kv=model.n_heads_kv,
                    head_dim=model.head_dim, layers=layers, score=model.score,
                    final_norm=model.final_norm, eps=model.eps, rope_base=model.rope_base)


# ----------------------------------------------------------------- oracle CPU leg


def oracle_sample(seconds: float, rows: int = 2048):
    """Times the oracle on a bounded sample of the workload: one gated upper
    layer (attention + SwiGLU, the workload's shapes) over `rows` kept rows,
    repeated until `seconds` elapse. Returns (FLOP/s, sample description,
    threads used)."""
    from oracle import tokengate_oracle as ref

    w = WORKLOAD
    rng = synth.rng_for(w.seed)
    lp = synth.layer_params(w, rng, upper=True)
    lw = ref.Layer(attn_norm=lp["attn_norm"], wqkv=ref.round_bf16(lp["wqkv"]),
                   wo=ref.round_bf16(lp["wo"]), ffn_norm=lp["ffn_norm"],
                   w_gate_up=ref.round_bf16(lp["w_gate_up"]), w_down=ref.round_bf16(lp["w_down"]),
                   q_norm=lp["q_norm"], k_norm=lp["k_norm"], gain=lp["gain"], tau=lp["tau"])
    m = ref.Model(d_model=w.d, n_heads_q=w.hq, n_heads_kv=w.hkv, head_dim=w.dh, layers=[lw],
                  final_norm=None, score_norm=np.ones(w.d), score_w1=np.zeros((1, w.d)),
                  score_b1=None, score_w2=np.zeros(1), score_b2=None)
    x = ref.round_bf16(rng.standard_normal((rows, w.d)))
    pos = np.sort(rng.choice(w.n, rows, replace=False)).astype(np.int32)
    s = rng.standard_normal(rows).astype(np.float32)
    flops_one = layer_flops(w, rows)
    t0 = time.perf_counter()
    reps = 0
    while True:
        ref.gated_layer_forward(x, pos, s, lw, m)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info

        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # noqa: BLE001
        threads = os.cpu_count() or 1
    desc = (f"oracle gated upper layer (Qwen3-1.7B shapes, {rows} rows) x{reps} in {dt:.1f} s; "
            f"TTFT extrapolated by algorithmic FLOPs of the full workload")
    return flops_one * reps / dt, desc, threads, dt


def layer_flops(w, t, with_ffn=True):
    qkv = (w.hq + 2 * w.hkv) * w.dh
    f = 2.0 * t * w.d * qkv + 4.0 * w.dh * w.hq * t * (t + 1) / 2 + 2.0 * t * w.hq * w.dh * w.d
    if with_ffn:
        f += 2.0 * t * w.d * 2 * w.inter + 2.0 * t * w.inter * w.d
    return f


def workload_flops(w, k):
    n, L = w.n, w.gate_layer
    f = L * layer_flops(w, n) + layer_flops(w, n, with_ffn=False)
    f += 2.0 * n * w.d * w.f  # scorer
    f += 2.0 * k * w.d * 3 * w.inter  # gate layer's FFN on K
    f += (w.n_layers - L - 1) * layer_flops(w, k)
    return f


# ----------------------------------------------------------------- reference arm


def config_of(w, k, args, world):
    """The workload's config dict, the same for both arms."""
    return {"workload": w.name, "n": w.n, "k": k, "layers": w.n_layers,
            "gate_layer": w.gate_layer, "d_model": w.d, "heads": f"{w.hq}/{w.hkv}x{w.dh}",
            "ffn": w.inter, "scorer": w.f, "protected": w.n_protect, "qk_norm": w.qk_norm,
            "kv_cache_out": not args.no_kv, "parallelism": f"replicas x{world}",
            "l2": "flushed between timed steps (256 MB write); inputs > L2"}


def run_reference(args, rank, world):
    """The oracle on the host cores. Each step times a bounded sample of the
    workload (one gated upper layer over 1024 kept rows) and extrapolates the
    whole workload's TTFT from its FLOP rate by algorithmic FLOPs: `value`
    is that extrapolated tokens/s (mean over the steps), `ms_per_step` the
    wall time each step's sample actually took."""
    if rank != 0:
        return 0
    w = WORKLOAD
    per_step, step_ms = [], []
    desc = ""
    threads = 1
    for i in range(args.warmup + args.steps):
        rate, desc, threads, dt = oracle_sample(seconds=0.0, rows=1024)
        if i >= args.warmup:
            per_step.append(w.n / (workload_flops(w, HEADLINE_K) / rate))
            step_ms.append(dt * 1e3)
    value = statistics.mean(per_step)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": statistics.mean(step_ms),
        "extrapolated_ttft_ms": 1000.0 * w.n / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, HEADLINE_K, args, world),
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(ms: float, dist=None, device=None) -> float:
    """The slowest rank's device time. Every rank calls this at the same
    point of the run (one all-reduce, MAX); without a process group it
    returns `ms` unchanged."""
    if dist is None:
        return ms
    import torch

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replicas_throughput(tokens_per_step: int, steps: int, world: int, total_ms: float) -> float:
    """Whole-job tokens/s of `world` independent replicas, each running
    `steps` steps of `tokens_per_step` tokens, over the slowest rank's time."""
    return world * tokens_per_step * steps / (total_ms / 1000.0)


# ----------------------------------------------------------------- our arm


def run_ours(args, rank, world, local_rank):
    import torch

    import learned_token_pruning_score_b200 as tg

    dist = None
    if world > 1:
        import torch.distributed as dist  # noqa: F811
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    w = WORKLOAD
    k = args.budget
    pk = peaks()
    model = build_model(tg, torch, w, device)
    x = synth.torch_hidden_states(w, seed=w.seed + 1000 + rank, device=str(device))
    prot = torch.zeros(w.n, dtype=torch.uint8, device=device)
    prot[w.n - w.n_protect:] = 1
    out = torch.empty(k, w.d, dtype=torch.bfloat16, device=device)
    kept = torch.empty(k, dtype=torch.int32, device=device)
    scores = torch.empty(w.n, dtype=torch.float32, device=device)
    ws = torch.empty(model.workspace_size(w.n, k, w.gate_layer), dtype=torch.uint8, device=device)
    kv = None if args.no_kv else kv_buffers(torch, w, k, device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # > 126 MB L2
    stream = torch.cuda.current_stream(device)
    tg.tg_device_error(clear=True)

    def step():
        tg.tg_prefill(model, x, prot, k, w.gate_layer, out=out, kept_idx=kept, scores=scores,
                      kv=kv, ws=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    def barrier():
        if dist is not None:
            dist.barrier()

    # ---- timed region: device time of each step with events on the
    # launching stream; L2 flushed between steps (outside the events). The
    # steps run twice: first plain (the throughput), then with every library
    # launch bracketed by its own event pair (the per-kernel durations of the
    # roofline; those events add a few microseconds between launches, so the
    # traced steps are not the throughput).
    def timed_steps(traced):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        if traced:
            tg.tg_trace_start(1 << 16)
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            torch.cuda.nvtx.range_push("tg_step")
            step()
            torch.cuda.nvtx.range_pop()
            stops[i].record(stream)
        torch.cuda.synchronize()
        trace = tg.tg_trace_stop() if traced else None
        barrier()
        return sum(a.elapsed_time(b) for a, b in zip(starts, stops)), trace

    clocks = ClockSampler(device.index if device.index is not None else 0)
    t_wall = time.perf_counter()
    plain_ms, _ = timed_steps(traced=False)
    wall = time.perf_counter() - t_wall
    traced_ms, trace = timed_steps(traced=True)
    clk = clocks.stop()
    total_ms = max_over_ranks(plain_ms, dist, device)
    traced_ms = max_over_ranks(traced_ms, dist, device)
    ms_per_step = total_ms / args.steps
    value = replicas_throughput(w.n, args.steps, world, total_ms)
    err_word = tg.tg_device_error()

    # ---- per-kernel breakdown from the trace (timed steps only)
    per = {}
    for r in trace:
        key = r["kernel"]
        if r["kernel"] == "attention_tc":
            key = "attention_tc_dense" if r["layer"] <= w.gate_layer else "attention_tc_gated"
        e = per.setdefault(key, {"ms": 0.0, "flops": 0.0, "bytes": 0.0, "launches": 0,
                                 "records": 0})
        e["ms"] += r["ms"]
        e["flops"] += r["flops"]
        e["bytes"] += r["bytes"]
        e["launches"] += launches_of(r)
        e["records"] += 1
    traced_ms = sum(e["ms"] for e in per.values())
    by_kernel = {}
    for key, e in sorted(per.items(), key=lambda kv: -kv[1]["ms"]):
        d = {"ms_per_step": e["ms"] / args.steps, "share": e["ms"] / traced_ms,
             "launches_per_step": e["launches"] / args.steps}
        if e["flops"] > 0:
            d["tflops"] = e["flops"] / (e["ms"] / 1e3) / 1e12
        else:
            d["gbs"] = e["bytes"] / (e["ms"] / 1e3) / 1e9
        by_kernel[key] = d
    # roofline of every traced kernel (the attention split into the dense
    # launches below the gate and the gated ones above it); the dominant one
    # (largest device time per step) is the line's `roofline`. Each launch
    # lasts at most a few ms inside a ~24 ms step, so the denominators are
    # the measured burst figures (bf16_tflops, hbm_gbs).
    def roofline_of(key, e):
        tensor = e["flops"] > 0
        ach = (e["flops"] if tensor else e["bytes"]) / (e["ms"] / 1e3) / (1e12 if tensor else 1e9)
        peak = pk["bf16"] if tensor else pk["hbm"]
        n_l = max(1, e["records"])
        base = "attention_tc" if key.startswith("attention_tc") else key
        return {"bound": "tensor" if tensor else "hbm", "kernel": key, "achieved": ach,
                "peak": peak, "unit": "TFLOP/s" if tensor else "GB/s", "frac": ach / peak,
                "peak_source": f"{pk['source']} ({'bf16_tflops' if tensor else 'hbm_gbs'}, burst)",
                "traffic": traffic_from_profiles(key, base, w.name),
                "algorithmic_per_launch": (e["flops"] if tensor else e["bytes"]) / n_l,
                "launches": n_l, "ms_per_step": e["ms"] / args.steps}

    rooflines = {key: roofline_of(key, e) for key, e in per.items()
                 if e["ms"] > 0 and (e["flops"] > 0 or e["bytes"] > 0)}
    dom = max(rooflines, key=lambda kk: rooflines[kk]["ms_per_step"])
    roofline = rooflines[dom]
    att_g = per.get("attention_tc_gated", {})
    att_d = per.get("attention_tc_dense", {})
    sel = per.get("select", {"ms": 0, "bytes": 0})
    cmp_ = per.get("compact", {"ms": 0, "bytes": 0})

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        x_host = x.cpu().pin_memory()
        prot_host = prot.cpu().pin_memory()
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        kept_host = torch.empty(kept.shape, dtype=kept.dtype).pin_memory()
        prot_dev = torch.empty_like(prot)

        # the input stays in pinned host memory: tg_prefill_host copies it in
        # chunks that overlap layer 0's projection and attention
        def e2e_step():
            prot_dev.copy_(prot_host, non_blocking=True)
            tg.tg_prefill_host(model, x_host, prot_dev, k, w.gate_layer, out=out, kept_idx=kept,
                               scores=scores, kv=kv, ws=ws, stream=stream)
            out_host.copy_(out, non_blocking=True)
            kept_host.copy_(kept, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
        h2d = x.numel() * x.element_size() + prot.numel()
        d2h = out.numel() * out.element_size() + kept.numel() * 4
        e2e = {"value": replicas_throughput(w.n, args.steps, world, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms / args.steps}

    # ---- other budgets, dense baseline and peak memory (not timed region;
    # single-GPU runs only: the replicas of a multi-GPU run report the headline)
    extras = {}
    if not args.quick and world == 1:
        def ttft(mdl, kk, reps=5):
            # peak memory of one prefill: weights + input + outputs (incl. KV
            # cache) + workspace, all allocated by the caller
            torch.cuda.synchronize()
            torch.cuda.reset_peak_memory_stats(device)
            o = torch.empty(kk, w.d, dtype=torch.bfloat16, device=device)
            ki = torch.empty(kk, dtype=torch.int32, device=device)
            kvb = None if args.no_kv else kv_buffers(torch, w, kk, device)
            wsz = torch.empty(mdl.workspace_size(w.n, kk, w.gate_layer), dtype=torch.uint8,
                              device=device)
            tg.tg_prefill(mdl, x, prot, kk, w.gate_layer, out=o, kept_idx=ki, kv=kvb, ws=wsz)
            torch.cuda.synchronize()
            # back to back like the headline steps (an idle gap before each
            # step would let the clocks recover and flatter the number)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(reps)]
            for a, b in evs:
                flush.zero_()
                a.record(stream)
                tg.tg_prefill(mdl, x, prot, kk, w.gate_layer, out=o, kept_idx=ki, kv=kvb, ws=wsz)
                b.record(stream)
            torch.cuda.synchronize()
            ms = [a.elapsed_time(b) for a, b in evs]
            # one more, traced: the attention kernels' own durations
            flush.zero_()
            tg.tg_trace_start(1 << 14)
            tg.tg_prefill(mdl, x, prot, kk, w.gate_layer, out=o, kept_idx=ki, kv=kvb, ws=wsz)
            torch.cuda.synchronize()
            tr = tg.tg_trace_stop()
            mem = torch.cuda.max_memory_allocated(device)
            del o, ki, wsz, kvb
            att = {}
            for name, sel in (("gated", lambda r: r["layer"] > w.gate_layer),
                              ("dense", lambda r: r["layer"] <= w.gate_layer)):
                rs = [r for r in tr if r["kernel"] == "attention_tc" and sel(r)]
                if rs:
                    tf = sum(r["flops"] for r in rs) / (sum(r["ms"] for r in rs) / 1e3) / 1e12
                    att[f"attn_{name}_tflops"] = tf
                    att[f"attn_{name}_frac_of_burst_peak"] = tf / pk["bf16"]
            return statistics.median(ms), mem, att

        del ws, kv
        torch.cuda.empty_cache()
        for kk in synth.PREFILL_32K_BUDGETS:
            t_ms, mem, att = ttft(model, kk)
            extras[f"gated_k{kk}"] = {"ttft_ms": t_ms, "tokens_per_s": w.n / (t_ms / 1e3),
                                      "tflop": workload_flops(w, kk) / 1e12,
                                      "peak_mem_gb": mem / 1e9, **att}
        t_ms, mem, att = ttft(dense_model(tg, model), w.n)
        extras["dense"] = {"ttft_ms": t_ms, "tokens_per_s": w.n / (t_ms / 1e3),
                           "tflop": workload_flops(w, w.n) / 1e12, "peak_mem_gb": mem / 1e9,
                           **att}
        for kk in synth.PREFILL_32K_BUDGETS:
            g = extras[f"gated_k{kk}"]
            g["ttft_speedup_vs_dense"] = extras["dense"]["ttft_ms"] / g["ttft_ms"]
            g["peak_mem_reduction_vs_dense"] = extras["dense"]["peak_mem_gb"] / g["peak_mem_gb"]
        # one request at all three budgets: the below-gate pass and the scores
        # once (tg_prefill_multi) against three single-budget prefills, both
        # without KV outputs, L2 flushed before each timed call
        ks = list(synth.PREFILL_32K_BUDGETS)
        outs_m = [torch.empty(kk, w.d, dtype=torch.bfloat16, device=device) for kk in ks]
        kept_m = [torch.empty(kk, dtype=torch.int32, device=device) for kk in ks]
        ws_m = torch.empty(model.workspace_size(w.n, max(ks), w.gate_layer), dtype=torch.uint8,
                           device=device)

        def run_multi():
            tg.tg_prefill_multi(model, x, prot, ks, w.gate_layer, outs=outs_m, kept_idx=kept_m,
                                ws=ws_m)

        def run_singles():
            for kk, o, ki in zip(ks, outs_m, kept_m):
                tg.tg_prefill(model, x, prot, kk, w.gate_layer, out=o, kept_idx=ki, ws=ws_m)

        mb = {}
        for name, fn in (("multi", run_multi), ("singles", run_singles)):
            fn()
            torch.cuda.synchronize()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(5)]
            for a, b in evs:
                flush.zero_()
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
            mb[name] = statistics.median([a.elapsed_time(b) for a, b in evs])
        extras["multi_budget"] = {"budgets": ks, "ms": mb["multi"],
                                  "separate_prefills_ms": mb["singles"],
                                  "speedup_vs_separate": mb["singles"] / mb["multi"],
                                  "tokens_per_s": w.n / (mb["multi"] / 1e3)}
        del outs_m, kept_m, ws_m
        # four requests of N/4 rows (budget K/4 each, the last 128 rows of
        # each protected) in one batched call against four separate prefills
        nb = 4
        lens = [w.n // nb] * nb
        ks_b = [k // nb] * nb
        prot_b = torch.zeros(w.n, dtype=torch.uint8, device=device)
        for b in range(nb):
            prot_b[(b + 1) * lens[b] - w.n_protect:(b + 1) * lens[b]] = 1
        out_b = torch.empty(sum(ks_b), w.d, dtype=torch.bfloat16, device=device)
        kept_b = torch.empty(sum(ks_b), dtype=torch.int32, device=device)
        ws_b = torch.empty(max(model.workspace_size(w.n + 128 * nb, k + 128 * nb, w.gate_layer),
                               1), dtype=torch.uint8, device=device)

        def run_batch():
            tg.tg_prefill_batch(model, x, prot_b, lens, ks_b, w.gate_layer, out=out_b,
                                kept_idx=kept_b, ws=ws_b)

        def run_each():
            r0 = k0 = 0
            for n_r, k_r in zip(lens, ks_b):
                tg.tg_prefill(model, x[r0:r0 + n_r], prot_b[r0:r0 + n_r], k_r, w.gate_layer,
                              out=out_b[k0:k0 + k_r], kept_idx=kept_b[k0:k0 + k_r], ws=ws_b)
                r0 += n_r
                k0 += k_r

        bt = {}
        for name, fn in (("batch", run_batch), ("each", run_each)):
            fn()
            torch.cuda.synchronize()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(5)]
            for a, b in evs:
                flush.zero_()
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
            bt[name] = statistics.median([a.elapsed_time(b) for a, b in evs])
        extras["batched"] = {"requests": nb, "rows_per_request": lens[0],
                             "budget_per_request": ks_b[0], "ms": bt["batch"],
                             "separate_prefills_ms": bt["each"],
                             "speedup_vs_separate": bt["each"] / bt["batch"],
                             "tokens_per_s": w.n / (bt["batch"] / 1e3)}
        del out_b, kept_b, ws_b
        # decode over the pruned cache (next to the dense cache) after the prefill
        dec = decode_bench(tg, torch, model, w, k, False, 64, 8, device, stream, pk)
        dec_d = decode_bench(tg, torch, dense_model(tg, model), w, w.n, True, 64, 8, device,
                             stream, pk)
        dec["dense_ms_per_token"] = dec_d["ms_per_token"]
        dec["dense_gbs"] = dec_d["gbs"]
        dec["dense_hbm_frac"] = dec_d["hbm_frac"]
        dec["speedup_vs_dense"] = dec_d["ms_per_token"] / dec["ms_per_token"]
        extras["decode"] = {"workload": f"{w.name} + decode (K={k}, batch 1)", **dec}
        # backward of one gated attention layer over the K kept rows (the
        # gradient path to the scorer, gain and temperature)
        bwd = attn_backward_bench(tg, torch, w.hq, w.hkv, w.dh, k, 20, device)
        bwd["frac_of_burst_bf16"] = bwd["tflops_algorithmic"] / pk["bf16"]
        extras["attn_backward"] = {"workload": f"one gated attention layer, K={k} rows, "
                                               f"{w.hq}/{w.hkv} heads x {w.dh}", **bwd}
        # a hybrid model's Gated DeltaNet layer above the gate runs its mixer
        # on the kept tokens only
        extras["gated_deltanet"] = gdn_bench(tg, torch, device, 20)
        # the gated-attention kernel alone at each budget, with and without
        # the gate bias
        extras["attention_budgets"] = attention_budget_bench(
            tg, torch, w, device, flush, pk, synth.PREFILL_32K_BUDGETS)
        # the Qwen3-1.7B single gated layer at N=16384, K=2048 (per stage)
        extras["layer_16k"] = single_layer_bench(tg, torch, synth.QWEN_LAYER_16K, device,
                                                 flush, pk)
        # select + compact over the sweep points
        extras["select_compact_sweep"] = sweep_bench(tg, torch, device, flush, pk)
        # the long-context gated sub-layer: N=131072 -> K=4096
        extras["long_context_128k"] = single_layer_bench(tg, torch, synth.LONG_128K, device,
                                                         flush, pk, reps=5)

    # ---- CPU baseline: the oracle, rank 0 only, N = 1
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        rate, desc, threads, _ = oracle_sample(seconds=args.cpu_seconds)
        cpu_tps = w.n / (workload_flops(w, k) / rate)
        cpu = {"value": cpu_tps, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc, "extrapolated": True}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded random weights and N(0,1) hidden states)",
            "config": config_of(w, k, args, world),
            "ttft_ms": ms_per_step,
            "traced_ms_per_step": traced_ms / args.steps,
            "tflop_per_step": workload_flops(w, k) / 1e12,
            "model_tflops": workload_flops(w, k) / (ms_per_step / 1e3) / 1e12,
            "roofline": roofline,
            "attn_gated_tflops": att_g and att_g["flops"] / (att_g["ms"] / 1e3) / 1e12,
            "attn_dense_tflops": att_d and att_d["flops"] / (att_d["ms"] / 1e3) / 1e12,
            "attn_gated_frac_of_burst_peak": att_g and
            att_g["flops"] / (att_g["ms"] / 1e3) / 1e12 / pk["bf16"],
            "rooflines": rooflines,
            "select_compact_gbs": (sel["bytes"] + cmp_["bytes"]) /
            max(1e-9, (sel["ms"] + cmp_["ms"]) / 1e3) / 1e9,
            "by_kernel": by_kernel,
            "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(sum(e["launches"] for e in per.values())),
            "clocks": clk, "wall_s_timed": wall, "device_error_word": err_word,
            "extras": extras,
        }
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- the other workloads


def _events_median(torch, fn, reps, flush, stream):
    """Median device ms of `reps` calls of fn (CUDA events on `stream`), L2
    flushed before each call (outside the events), after one untimed call.
    A spin kernel queued before each timed call keeps the GPU busy while the
    host enqueues the call, so a short call's events see its device time,
    not the host's launch latency."""
    fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for a, b in evs:
        if flush is not None:
            flush.zero_()
        torch.cuda._sleep(200000)  # ~0.1 ms: longer than the host's enqueue of fn
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.median([a.elapsed_time(b) for a, b in evs])


def _traced(tg, torch, fn, reps, flush):
    """Per-kernel totals of `reps` traced calls (each launch bracketed by its
    own events), divided by reps: {kernel: {ms, flops, bytes, launches}}."""
    tg.tg_trace_start(1 << 16)
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        fn()
    torch.cuda.synchronize()
    out = {}
    for r in tg.tg_trace_stop():
        e = out.setdefault(r["kernel"], {"ms": 0.0, "flops": 0.0, "bytes": 0.0, "launches": 0})
        e["ms"] += r["ms"] / reps
        e["flops"] += r["flops"] / reps
        e["bytes"] += r["bytes"] / reps
        e["launches"] += launches_of(r) / reps
    return out


def select_compact_bytes(n, k, d, elem=2):
    """Algorithmic bytes of select + compact: scores (4N) and mask (N) read,
    indices written (4K), kept rows read and written (2 K d elem), positions
    and scores of the kept rows written (8K)."""
    return 4 * n + n + 4 * k + 2 * k * d * elem + 8 * k


def sweep_bench(tg, torch, device, flush, pk, reps=10, points=None):
    """Select + compact over the sweep points (seeded fp32 N(0,1) scores with
    exact-tie blocks and a few +-0 / +-inf, the last 128 protected, bf16 rows
    of d 2048): median us, algorithmic GB/s and fraction of the measured HBM
    copy bandwidth, L2 flushed before each call."""
    res = []
    x_all = torch.randn(max(synth.SWEEP_N), synth.SWEEP_D, device=device, dtype=torch.bfloat16)
    for n, k in (points or synth.sweep_points()):
        rng = synth.rng_for(synth.SWEEP_SEED)
        s = torch.from_numpy(synth.sweep_scores(n, rng)).to(device)
        prot = torch.from_numpy(synth.protect_tail(n, synth.SWEEP_PROTECT)).to(device)
        x = x_all[:n]
        idx = torch.empty(k, dtype=torch.int32, device=device)
        xo = torch.empty(k, synth.SWEEP_D, device=device, dtype=torch.bfloat16)
        po = torch.empty(k, dtype=torch.int32, device=device)
        so = torch.empty(k, dtype=torch.float32, device=device)
        ws = torch.empty(tg.tg_workspace_size(tg.TG_OP_TOPK_SELECT, n=n), dtype=torch.uint8,
                         device=device)
        stream = torch.cuda.current_stream(device)

        def once():
            tg.tg_topk_select(s, prot, k, kept_idx=idx, ws=ws, stream=stream)
            tg.tg_compact(x, idx, scores=s, x_out=xo, pos_out=po, scores_out=so, stream=stream)

        for _ in range(2):
            once()
        t = _events_median(torch, once, reps, flush, stream)
        sel_ms = _events_median(
            torch, lambda: tg.tg_topk_select(s, prot, k, kept_idx=idx, ws=ws, stream=stream),
            reps, flush, stream)
        byt = select_compact_bytes(n, k, synth.SWEEP_D)
        gbs = byt / (t / 1e3) / 1e9
        res.append({"n": n, "k": k, "us": t * 1e3, "select_us": sel_ms * 1e3, "bytes": byt,
                    "gbs": gbs, "frac_hbm": gbs / pk["hbm"]})
        del s, prot, idx, xo, po, so, ws
    del x_all
    torch.cuda.empty_cache()
    return res


STAGE_OF = {"rmsnorm": "rmsnorm", "gemm_tc_score": "scorer", "select": "select",
            "compact": "compact", "rope_table": "tables", "gemm_tc_qkv": "qkv_proj",
            "attention_tc": "attention", "gemm_tc_residual": "o_proj+down_proj",
            "gemm_tc_swiglu": "gate_up_proj", "copy": "copy"}


def single_layer_bench(tg, torch, w, device, flush, pk, reps=10, dense_too=True):
    """One gated layer gated before it (tg_prefill, gate_layer -1): scorer over
    the N input rows, select, compact, then the layer over the K kept rows.
    Reports the step's median ms, per-stage ms from a traced run, the
    attention's TFLOP/s, the scorer's GB/s (its algorithmic bytes: the N rows
    read once, the weights, the scores written), and the same layer dense
    over all N rows (no gate bias)."""
    model = build_model(tg, torch, w, device)
    x = synth.torch_hidden_states(w, seed=w.seed, device=str(device))
    prot = torch.zeros(w.n, dtype=torch.uint8, device=device)
    prot[w.n - w.n_protect:] = 1
    stream = torch.cuda.current_stream(device)

    def measure(mdl, kk):
        o = torch.empty(kk, w.d, dtype=torch.bfloat16, device=device)
        ki = torch.empty(kk, dtype=torch.int32, device=device)
        wsz = torch.empty(mdl.workspace_size(w.n, kk, -1), dtype=torch.uint8, device=device)
        run = lambda: tg.tg_prefill(mdl, x, prot, kk, -1, out=o, kept_idx=ki, ws=wsz,  # noqa: E731
                                    stream=stream)
        ms = _events_median(torch, run, reps, flush, stream)
        tr = _traced(tg, torch, run, reps, flush)
        stages = {}
        for kern, e in tr.items():
            st_ = STAGE_OF.get(kern, kern)
            stages[st_] = stages.get(st_, 0.0) + e["ms"]
        att = tr.get("attention_tc")
        r = {"ms": ms, "stages_ms": stages, "launches": sum(e["launches"] for e in tr.values())}
        if att:
            tf = att["flops"] / (att["ms"] / 1e3) / 1e12
            r.update(attention_tflops=tf, attention_frac_of_burst_bf16=tf / pk["bf16"])
        del o, ki, wsz
        return r, tr

    g, tr = measure(model, w.k)
    # the scorer: its RMSNorm (first rmsnorm launch of the call) and the
    # scorer GEMM; algorithmic bytes = the rows read once + W1 + the scores
    rows_b = w.n * w.d * 2
    sc_bytes = rows_b + w.f * w.d * 2 + 4 * w.n
    rms_ms = _traced_first(tg, torch, lambda: tg.tg_prefill(
        model, x, prot, w.k, -1, stream=stream), "rmsnorm", flush)
    sc_ms = tr.get("gemm_tc_score", {"ms": 0.0})["ms"]
    g["scorer_ms"] = rms_ms + sc_ms
    g["scorer_gbs"] = sc_bytes / ((rms_ms + sc_ms) / 1e3) / 1e9
    g["scorer_frac_hbm"] = g["scorer_gbs"] / pk["hbm"]
    sel = tr.get("select", {"ms": 0.0})["ms"] + tr.get("compact", {"ms": 0.0})["ms"]
    g["select_compact_us"] = sel * 1e3
    res = {"workload": w.name, "n": w.n, "k": w.k, "gated": g}
    if dense_too:
        d, _ = measure(dense_model(tg, model), w.n)
        res["dense"] = d
        res["speedup_vs_dense"] = d["ms"] / g["ms"]
    del model, x, prot
    torch.cuda.empty_cache()
    return res


def _traced_first(tg, torch, fn, kernel, flush, reps=5):
    """Median device ms of the first launch of `kernel` in a traced call of
    fn, over `reps` calls."""
    ms = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        tg.tg_trace_start(1 << 12)
        fn()
        torch.cuda.synchronize()
        first = [r["ms"] for r in tg.tg_trace_stop() if r["kernel"] == kernel]
        ms.append(first[0] if first else 0.0)
    return statistics.median(ms)


def attention_budget_bench(tg, torch, w, device, flush, pk, budgets, reps=10):
    """The gated-attention kernel alone at each budget: K kept rows of an
    N-token prompt (ascending positions drawn from 0..N-1), Qwen3-1.7B heads,
    with the gate bias (scores ~N(0, 2^2), gain U(0,2), tau U(0.5,1.5)) and
    without it (plain causal attention over the same rows). Traced attention
    kernel time (median launch), algorithmic TFLOP/s and fraction of the
    measured burst bf16 peak."""
    stream = torch.cuda.current_stream(device)
    res = {}
    for kk in budgets:
        g = torch.Generator(device=device).manual_seed(100 + kk)
        q = torch.randn(kk, w.hq, w.dh, device=device, generator=g).to(torch.bfloat16)
        k_ = torch.randn(kk, w.hkv, w.dh, device=device, generator=g).to(torch.bfloat16)
        v = torch.randn(kk, w.hkv, w.dh, device=device, generator=g).to(torch.bfloat16)
        pos = torch.sort(torch.randperm(w.n, device=device, generator=g)[:kk]).values
        pos = pos.to(torch.int32)
        s = torch.randn(kk, device=device, generator=g) * 2
        gain = torch.rand(w.hq, device=device, generator=g) * 2
        tau = torch.rand(w.hq, device=device, generator=g) + 0.5
        out = torch.empty_like(q)
        ws = torch.empty(tg.tg_workspace_size(tg.TG_OP_GATED_ATTN, k=kk, n_heads_q=w.hq,
                                              n_heads_kv=w.hkv, head_dim=w.dh),
                         dtype=torch.uint8, device=device)
        flops = 4.0 * w.dh * w.hq * kk * (kk + 1) / 2
        r = {}
        for name, args_ in (("bias", (s, gain, tau)), ("no_bias", (None, None, None))):
            run = lambda a=args_: tg.tg_gated_attn_prefill(q, k_, v, pos, *a, out=out,  # noqa
                                                           ws=ws, stream=stream)
            run()
            torch.cuda.synchronize()
            tg.tg_trace_start(1 << 12)
            for _ in range(reps):
                flush.zero_()
                run()
            torch.cuda.synchronize()
            ms = statistics.median([t["ms"] for t in tg.tg_trace_stop()
                                    if t["kernel"] == "attention_tc"])
            tf = flops / (ms / 1e3) / 1e12
            r[name] = {"us": ms * 1e3, "tflops": tf, "frac_of_burst_bf16": tf / pk["bf16"]}
        r["bias_cost"] = r["bias"]["us"] / r["no_bias"]["us"]
        res[f"k{kk}"] = r
        del q, k_, v, pos, s, out, ws
    return res


def run_sweep(args):
    """The select+compact sweep, the 16K single layer and the 128K
    long-context layer alone, one JSON line each."""
    import torch

    import learned_token_pruning_score_b200 as tg

    device = torch.device("cuda", 0)
    pk = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    for r in sweep_bench(tg, torch, device, flush, pk, reps=args.steps):
        print(json.dumps({"sweep": "select+compact", **r}), flush=True)
    print(json.dumps(single_layer_bench(tg, torch, synth.QWEN_LAYER_16K, device, flush, pk)),
          flush=True)
    print(json.dumps(single_layer_bench(tg, torch, synth.LONG_128K, device, flush, pk, reps=5)),
          flush=True)
    print(json.dumps(attention_budget_bench(tg, torch, WORKLOAD, device, flush, pk,
                                            synth.PREFILL_32K_BUDGETS)), flush=True)
    assert tg.tg_device_error() == 0
    return 0


# ----------------------------------------------------------------- attention backward


def attn_backward_bench(tg, torch, hq, hkv, dh, t, steps, device, bias=True, warmup=3):
    """tg_gated_attn_backward over t kept rows (positions spread over 8t, gate
    bias on): median ms per call of `steps` calls (CUDA events, inputs resident),
    algorithmic TFLOP/s (the five causal [t x t x dh] products: 2.5 times the
    forward's FLOPs), and a traced per-kernel split."""
    g = torch.Generator(device=device).manual_seed(5)
    q = torch.randn(t, hq, dh, device=device, dtype=torch.bfloat16, generator=g)
    kk = torch.randn(t, hkv, dh, device=device, dtype=torch.bfloat16, generator=g)
    v = torch.randn(t, hkv, dh, device=device, dtype=torch.bfloat16, generator=g)
    dout = torch.randn(t, hq, dh, device=device, dtype=torch.bfloat16, generator=g)
    pos = torch.sort(torch.randperm(8 * t, device=device, generator=g)[:t]).values.to(torch.int32)
    s = torch.randn(t, device=device, generator=g) * 2 if bias else None
    gain = torch.rand(hq, device=device, generator=g) * 2 if bias else None
    tau = torch.rand(hq, device=device, generator=g) + 0.5 if bias else None
    out, lse, o32 = tg.tg_gated_attn_forward(q, kk, v, pos, s, gain, tau)
    grads = [torch.empty_like(q), torch.empty_like(kk), torch.empty_like(v),
             torch.empty(t, device=device) if bias else None,
             torch.empty(hq, device=device), torch.empty(hq, device=device)]
    ws = torch.empty(tg.tg_workspace_size(tg.TG_OP_GATED_ATTN_BWD, k=t, n_heads_q=hq,
                                          n_heads_kv=hkv, head_dim=dh),
                     dtype=torch.uint8, device=device)

    def run():
        tg.tg_gated_attn_backward(q, kk, v, pos, out, lse, dout, s, gain, tau, out_f32=o32,
                                  dq=grads[0],
                                  dk=grads[1], dv=grads[2], ds=grads[3], dgain=grads[4],
                                  dtau=grads[5], want_ds=bias, ws=ws)

    for _ in range(warmup):
        run()
    ms = []
    for _ in range(steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        run()
        b.record()
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    tg.tg_trace_start()
    for _ in range(steps):
        run()
    torch.cuda.synchronize()
    tr = tg.tg_trace_stop()
    split = {}
    for r in tr:
        e = split.setdefault(r["kernel"], {"ms": 0.0, "flops": 0.0})
        e["ms"] += r["ms"] / steps
        e["flops"] += r["flops"] / steps
    for e in split.values():
        e["tflops_executed"] = e["flops"] / (e["ms"] / 1e3) / 1e12 if e["flops"] else None
        del e["flops"]
    fwd_flops = 4.0 * dh * hq * t * (t + 1) / 2.0
    med = statistics.median(ms)
    return {"ms": med, "tflops_algorithmic": 2.5 * fwd_flops / (med / 1e3) / 1e12,
            "kernels": split, "heads": [hq, hkv], "bias": bias}


# fp32 FMA rate of the CUDA cores, from the unit counts and the maximum SM
# clock (148 SMs x 128 FP32 lanes x 2 flops x 1.965 GHz); no measured figure
# exists for it, so fractions against it say "of nominal".
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def gdn_bench(tg, torch, device, steps, warmup=3):
    """tg_gated_deltanet of a hybrid model's linear-attention layer over the
    K kept tokens, next to the same mixer over all N tokens (the layer without
    the gate): median ms per call (CUDA events, inputs resident), the
    per-kernel split, and the recurrence's fp32 rate against the nominal
    CUDA-core FMA rate (it runs on CUDA cores in fp32: no tensor-core path)."""
    w = synth.GDN_LAYER_32K
    rng = synth.rng_for(w.seed)
    p = synth.gdn_params(w, rng)
    layer = tg.GdnLayer(w.hk, w.hv, w.dk, w.dv, *(torch.from_numpy(p[k]).to(device)
                                                  for k in ("conv_w", "A_log", "dt_bias",
                                                            "norm_w")), eps=w.eps)
    res = {"workload": f"{w.name}: {w.hk}/{w.hv} heads x {w.dk}/{w.dv}, conv {w.W}",
           "dtype": "bf16 in/out, fp32 state"}
    for name, T in (("gated", w.T), ("dense", w.n)):
        g = torch.Generator(device=device).manual_seed(11)
        C = 2 * w.hk * w.dk + w.hv * w.dv
        x = [torch.randn(T, n, device=device, generator=g).to(torch.bfloat16)
             for n in (C, w.hv * w.dv, w.hv, w.hv)]
        y = torch.empty(T, w.hv * w.dv, dtype=torch.bfloat16, device=device)
        s_out = torch.empty(w.hv, w.dv, w.dk, dtype=torch.float32, device=device)
        ws = torch.empty(tg.tg_gated_deltanet_workspace_size(layer, T), dtype=torch.uint8,
                         device=device)

        def run():
            tg.tg_gated_deltanet(layer, *x, y=y, state_out=s_out, want_state=False, ws=ws)

        for _ in range(warmup):
            run()
        ms = []
        for _ in range(steps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            run()
            b.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        tg.tg_trace_start()
        for _ in range(steps):
            run()
        torch.cuda.synchronize()
        split = {}
        for r in tg.tg_trace_stop():
            e = split.setdefault(r["kernel"], {"ms": 0.0, "flops": 0.0})
            e["ms"] += r["ms"] / steps
            e["flops"] += r["flops"] / steps
        rec = split.get("gdn_recur", {"ms": 0.0, "flops": 0.0})
        tf = rec["flops"] / (rec["ms"] / 1e3) / 1e12 if rec["ms"] else None
        for e in split.values():
            del e["flops"]
        res[name] = {"tokens": T, "ms": statistics.median(ms),
                     "tokens_per_s": T / (statistics.median(ms) / 1e3), "kernels": split,
                     "recur_tflops_fp32": tf,
                     "recur_frac_of_nominal_fp32": tf and tf / FP32_FMA_TFLOPS}
        del x, y, ws
    res["speedup_vs_dense"] = res["dense"]["ms"] / res["gated"]["ms"]
    return res


# ----------------------------------------------------------------- profiling cases


def run_case(args):
    """Small, repeatable invocations of one kernel family: the commands that
    the ncu summaries under profiles/ were captured with, and the timings
    they quote. Not part of the default bench line.

    attn:     tg_gated_attn_prefill over `rows` rows, Qwen3-1.7B heads
              (16/8 x 128), gate bias on (--no-bias: plain causal) -- the
              attention kernel (plus its RoPE prep).
    attn_bwd: tg_gated_attn_forward + tg_gated_attn_backward at those heads.
    layer:    tg_prefill of a 2-layer Qwen3-1.7B-shaped model, gate at layer 0,
              N = rows, K = rows / 8 -- every GEMM epilogue, select and compact.
    gemm:     the prefill's projection shapes through tg_linear, next to
              torch.matmul (cuBLAS) on the same operands, timed interleaved.
    decode:   a 2-layer Qwen3-1.7B-shaped model gated at layer 0 (N = rows,
              K = rows / 8, at least 128): prefill, then `steps` decode steps.
    gdn:      the Gated DeltaNet mixer over `rows` kept tokens.
    score:    tg_score over `rows` rows (d_model 2048, 256 hidden).
    select:   tg_topk_select then tg_compact of `rows` sweep-style scores.
    """
    import torch

    import learned_token_pruning_score_b200 as tg

    device = torch.device("cuda", 0)
    torch.manual_seed(0)
    w = WORKLOAD
    t = args.rows
    if args.case == "gemm":
        # the prefill's projection shapes: tg_linear (tcgen05) next to
        # torch.matmul (cuBLAS) on the same operands, interleaved
        shapes = [("qkv", 4096, 2048), ("o_proj", 2048, 2048), ("gate_up", 12288, 2048),
                  ("down", 2048, 6144)]
        for name, n, kdim in shapes:
            x = torch.randn(t, kdim, device=device, dtype=torch.bfloat16)
            wt = torch.randn(n, kdim, device=device, dtype=torch.bfloat16) * 0.02
            y = torch.empty(t, n, device=device, dtype=torch.bfloat16)
            res = {}
            for _ in range(3):
                for impl in ("tg_linear", "cublas"):
                    f = (lambda: tg.tg_linear(x, wt, y=y)) if impl == "tg_linear" else \
                        (lambda: torch.matmul(x, wt.t(), out=y))
                    f()
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record()
                    for _ in range(args.steps):
                        f()
                    b.record()
                    torch.cuda.synchronize()
                    res.setdefault(impl, []).append(a.elapsed_time(b) / args.steps)
            fl = 2.0 * t * n * kdim
            print(json.dumps({"case": "gemm", "shape": name, "m": t, "n": n, "k": kdim,
                              **{f"{i}_tflops": fl / (statistics.median(v) / 1e3) / 1e12
                                 for i, v in res.items()}}), flush=True)
        return 0
    if args.case == "decode":
        # a 2-layer Qwen3-1.7B-shaped model, gate at layer 0: one layer with an
        # N-row cache, one with a K-row cache; `steps` decode steps after the prefill
        wl = synth.shrink(w, n=t, k=max(128, t // 8), n_layers=2, gate_layer=0)
        model = build_model(tg, torch, wl, device)
        res = decode_bench(tg, torch, model, wl, wl.k, False, args.steps, 3, device,
                           torch.cuda.current_stream(device), peaks())
        assert tg.tg_device_error() == 0
        print(json.dumps({"case": "decode", "rows": t, "steps": args.steps,
                          "ms_per_token": res["ms_per_token"], "gbs": res["gbs"]}))
        return 0
    if args.case == "select":
        # tg_topk_select then tg_compact of `rows` sweep-style scores, K = rows / 8
        n, kk = t, max(1, t // 8)
        rng = synth.rng_for(synth.SWEEP_SEED)
        s = torch.from_numpy(synth.sweep_scores(n, rng)).to(device)
        prot = torch.from_numpy(synth.protect_tail(n, synth.SWEEP_PROTECT)).to(device)
        x = torch.randn(n, synth.SWEEP_D, device=device, dtype=torch.bfloat16)
        idx = torch.empty(kk, dtype=torch.int32, device=device)
        ws = torch.empty(tg.tg_workspace_size(tg.TG_OP_TOPK_SELECT, n=n), dtype=torch.uint8,
                         device=device)
        for _ in range(args.steps):
            tg.tg_topk_select(s, prot, kk, kept_idx=idx, ws=ws)
            tg.tg_compact(x, idx, scores=s)
        torch.cuda.synchronize()
        assert tg.tg_device_error() == 0
        print(json.dumps({"case": "select", "rows": t, "k": kk, "reps": args.steps}))
        return 0
    if args.case == "score":
        # tg_score over `rows` rows of d_model 2048 into the 256-wide scorer
        x = torch.randn(t, w.d, device=device, dtype=torch.bfloat16)
        nw = torch.ones(w.d, device=device)
        w1 = (torch.randn(w.f, w.d, device=device) * 0.02).to(torch.bfloat16)
        w2 = torch.randn(w.f, device=device) * 0.02
        sc = torch.empty(t, device=device)
        ws = torch.empty(tg.tg_workspace_size(tg.TG_OP_SCORE, n=t, d_model=w.d, d_score=w.f,
                                              dtype=tg.TG_BF16), dtype=torch.uint8, device=device)
        for _ in range(args.steps):
            tg.tg_score(x, nw, w1, w2, scores=sc, ws=ws)
        torch.cuda.synchronize()
        assert tg.tg_device_error() == 0
        print(json.dumps({"case": "score", "rows": t, "reps": args.steps}))
        return 0
    if args.case == "attn_bwd":
        res = attn_backward_bench(tg, torch, w.hq, w.hkv, w.dh, t, args.steps, device,
                                  bias=not args.no_bias)
        assert tg.tg_device_error() == 0
        print(json.dumps({"case": "attn_bwd", "rows": t, "steps": args.steps, **res}))
        return 0
    if args.case == "gdn":
        # tg_gated_deltanet over `rows` tokens, the hybrid-layer mixer's shape
        gw = synth.GDN_LAYER_32K
        p = synth.gdn_params(gw, synth.rng_for(gw.seed))
        layer = tg.GdnLayer(gw.hk, gw.hv, gw.dk, gw.dv,
                            *(torch.from_numpy(p[k]).to(device)
                              for k in ("conv_w", "A_log", "dt_bias", "norm_w")), eps=gw.eps)
        C = 2 * gw.hk * gw.dk + gw.hv * gw.dv
        x = [torch.randn(t, n, device=device).to(torch.bfloat16)
             for n in (C, gw.hv * gw.dv, gw.hv, gw.hv)]
        for _ in range(args.steps):
            tg.tg_gated_deltanet(layer, *x, want_state=False)
        torch.cuda.synchronize()
        assert tg.tg_device_error() == 0
        print(json.dumps({"case": "gdn", "rows": t, "reps": args.steps}))
        return 0
    if args.case == "attn":
        q = torch.randn(t, w.hq, w.dh, device=device, dtype=torch.bfloat16)
        kk = torch.randn(t, w.hkv, w.dh, device=device, dtype=torch.bfloat16)
        v = torch.randn(t, w.hkv, w.dh, device=device, dtype=torch.bfloat16)
        pos = torch.arange(t, dtype=torch.int32, device=device)
        s = None if args.no_bias else torch.randn(t, device=device)
        gain = None if args.no_bias else torch.rand(w.hq, device=device) * 2
        tau = None if args.no_bias else torch.rand(w.hq, device=device) + 0.5
        out = torch.empty_like(q)
        ws = torch.empty(tg.tg_workspace_size(tg.TG_OP_GATED_ATTN, k=t, n_heads_q=w.hq,
                                              n_heads_kv=w.hkv, head_dim=w.dh),
                         dtype=torch.uint8, device=device)
        run = lambda: tg.tg_gated_attn_prefill(q, kk, v, pos, s, gain, tau, out=out, ws=ws)  # noqa: E731
    else:
        wl = synth.shrink(w, n=t, k=max(128, t // 8), n_layers=2, gate_layer=0)
        model = build_model(tg, torch, wl, device)
        x = synth.torch_hidden_states(wl, seed=1, device=str(device))
        ws = torch.empty(model.workspace_size(wl.n, wl.k, 0), dtype=torch.uint8, device=device)
        out = torch.empty(wl.k, wl.d, dtype=torch.bfloat16, device=device)
        kept = torch.empty(wl.k, dtype=torch.int32, device=device)
        run = lambda: tg.tg_prefill(model, x, None, wl.k, 0, out=out, kept_idx=kept, ws=ws)  # noqa: E731
    for _ in range(args.steps):
        run()
    torch.cuda.synchronize()
    assert tg.tg_device_error() == 0
    print(json.dumps({"case": args.case, "rows": t, "reps": args.steps}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--budget", type=int, default=HEADLINE_K)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-kv", action="store_true", help="do not write the KV cache outputs")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--quick", action="store_true", help="skip the other budgets / dense run")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--case", choices=["attn", "attn_bwd", "layer", "gemm", "decode", "gdn", "score",
                                       "select"],
                    default=None,
                    help="run one kernel family's small case (the profiles/ captures) instead "
                         "of the bench line")
    ap.add_argument("--rows", type=int, default=32768)
    ap.add_argument("--no-bias", action="store_true",
                    help="attn case: plain causal attention (as the layers below the gate)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.sweep:
        return run_sweep(args)
    if args.case:
        return run_case(args)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
