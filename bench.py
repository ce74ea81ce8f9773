#!/usr/bin/env python
"""Benchmark of the Llama-3-8B-shape decoder on B200: prefill + greedy decode tokens/s.

One step = the whole hot path over one batch of the workload
"llama3-8b-bf16-b1-p2048-g256": prefill of a 2048-token prompt (batch 1), then
256 greedy decode steps feeding back the argmax, on seeded random bf16 weights
of the Llama-3-8B architecture (32 layers, dim 4096, 32/8 heads, FFN 14336,
vocab 128256). Inputs are resident in HBM when the timed region starts.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --workload NAME [--steps K] [--warmup W] [--fused]   # another seeded workload

For N > 1 run under torch.distributed.run: every rank runs an independent
replica on its own GPU (the decoder has no exchange step), times are the max
over ranks, and value is the tokens of all ranks / that time.
Prints one JSON line on rank 0.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "llama3-8b-bf16-b1-p2048-g256"
METRIC = "decode & prefill tokens/s at Llama-3-8B shape, 1 B200; % of HBM/tensor roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks(path=None):
    """The roofline denominators: the measured HBM copy bandwidth (GB/s) and bf16 GEMM
    rates (TF/s) when MEASURED_PEAKS.json holds them as numbers, else the fallback."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            peaks = {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops")}
            peaks["bf16_tflops_sustained"] = float(d.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
            if min(peaks.values()) > 0:
                return peaks, "measured"
        except (OSError, ValueError, TypeError, KeyError, AttributeError):
            pass
    return dict(PEAKS_FALLBACK), "fallback"


# ---------------------------------------------------------------- algorithmic work
def work_model(shape, B, T, S_decode_mean):
    """Algorithmic FLOPs of the prefill and bytes of one decode step."""
    D, H, Hk, d, F, V, L = (shape.dim, shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.ffn_hidden,
                            shape.vocab, shape.n_layers)
    lin_params = L * (D * (H + 2 * Hk) * d + H * d * D + 3 * D * F)
    prefill_flops = 2 * B * T * lin_params + L * B * (4 * H * d * T * T / 2) + 2 * B * D * V
    w_bytes = 2 * (lin_params + V * D)
    kv_bytes = L * B * 2 * Hk * d * 2 * S_decode_mean
    kinds_bytes = {  # one decode launch, B rows
        "qkv": 2 * D * (H + 2 * Hk) * d, "wo": 2 * H * d * D, "w13": 2 * 2 * F * D, "w2": 2 * F * D,
        "head": 2 * V * D, "attn": B * 2 * Hk * d * 2 * S_decode_mean,
        "step": w_bytes + kv_bytes,  # the fused decode step: every weight and the cache, once
    }
    kinds_flops = {"qkv": 2 * B * T * D * (H + 2 * Hk) * d, "wo": 2 * B * T * H * d * D, "w13": 2 * B * T * 2 * F * D,
                   "w2": 2 * B * T * F * D, "attn": B * 4 * H * d * T * T / 2}
    return prefill_flops, w_bytes + kv_bytes, kinds_bytes, kinds_flops


# ---------------------------------------------------------------- replicas
# With N > 1 every rank runs its own replica of the whole workload on its own GPU;
# the ranks meet only to line up the timed region and to take the slowest rank's
# time. These helpers take the process group torch.distributed already holds
# (nccl on GPUs, gloo in the CPU tests) and the device its tensors live on.
def replica_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def replica_max(x: float, world: int, device) -> float:
    """The largest x over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, steps: int, units_per_step: float, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * steps * units_per_step / max_seconds


# ---------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in rows]
        smax = float(rows[0][2])
        loaded = [s for s, r in zip(sm, rows) if float(r[3] or 0) > 300] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3] or 0) for r in rows)}


# ---------------------------------------------------------------- CPU oracle sample
def oracle_sample(shape, seed, prompt_len, decode_steps, budget_s=20.0):
    """Time the fp64 oracle on one decoder layer of the workload and extrapolate.

    Sample: layer 0 at full width; a prefill of Ts prompt tokens and a decode step
    against a cache of prompt_len positions; the lm_head on a vocab slice. The
    whole-step time is estimated as n_layers * (prompt_len * t_prefill_token +
    decode_steps * t_decode) + (decode_steps + 1) * t_head. Attention cost of the
    full prompt is underestimated by timing a shorter prefill (stated in `sample`).
    """
    import numpy as np
    import torch
    import oracle as O
    import seeded_inputs as S
    t0 = time.time()
    one = shape.replace(n_layers=1, has_embed_and_head=False)
    lw = S.make_layer_weights(one, seed, 0)
    orc = O.OracleModel(one, {}, [lw], batch=1)
    orc.layer(0)  # widen the layer's weights once (not timed)
    Ts = 512
    h = S.make_hidden(seed, 1, Ts, shape.dim, tag="oracle-sample").numpy()
    t = time.perf_counter()
    orc.forward_hidden(h)
    t_prefill_tok = (time.perf_counter() - t) / Ts
    # decode against a prompt_len cache
    g = np.random.default_rng(0)
    orc.set_cache(0, 0, g.standard_normal((prompt_len, shape.n_kv_heads, shape.head_dim)),
                  g.standard_normal((prompt_len, shape.n_kv_heads, shape.head_dim)))
    n_dec = 0
    t = time.perf_counter()
    while n_dec < 10 and time.perf_counter() - t < budget_s / 2:
        orc.forward_hidden(h[:, :1])
        n_dec += 1
    t_decode = (time.perf_counter() - t) / n_dec
    rows = 8192
    Wslice = np.random.default_rng(1).standard_normal((rows, shape.dim))
    x = np.random.default_rng(2).standard_normal(shape.dim)
    t = time.perf_counter()
    O.argmax_first(x @ Wslice.T)
    t_head = (time.perf_counter() - t) * shape.vocab / rows
    est = shape.n_layers * (prompt_len * t_prefill_tok + decode_steps * t_decode) + (decode_steps + 1) * t_head
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=os.cpu_count())
    except Exception:
        cores = os.cpu_count()
    return {
        "value": (prompt_len + decode_steps) / est, "unit": "tokens/s", "cores": int(cores), "kind": "oracle",
        "sample": (f"fp64 oracle, layer 0 of 32 at full width: prefill of {Ts} tokens and {n_dec} decode "
                   f"steps against a {prompt_len}-position cache, lm_head on {rows} of {shape.vocab} rows; "
                   f"extrapolated to the full step ({prompt_len} prefill + {decode_steps} decode tokens, "
                   f"{shape.n_layers} layers; prefill attention of the full prompt underestimated)"),
        "estimated_step_s": est, "wall_s": time.time() - t0,
    }


def run_reference(args, rank):
    """--impl reference: the CPU oracle as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    import seeded_inputs as S
    w = S.WORKLOADS[WORKLOAD]
    vals = []
    last = None
    for i in range(args.warmup + args.steps):
        r = oracle_sample(w.shape, w.seed, w.prompt_len, w.decode_steps, budget_s=8.0)
        if i >= args.warmup:
            vals.append(r["value"])
        last = r
    v = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * (w.prompt_len + w.decode_steps) / v,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,0.02) weights, N(0,1) hidden states)",
            "config": {"workload": WORKLOAD, "batch": w.batch, "prompt_len": w.prompt_len,
                       "decode_steps": w.decode_steps},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": last["cores"], "kind": "oracle",
                             "sample": last["sample"]},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- ncu traffic record
def ncu_traffic(kind):
    """DRAM bytes per launch of a kernel kind from the committed ncu summary, if its
    sources are unchanged since the counters were taken (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(kind)
    if not rec:
        return None
    h = hashlib.sha256()
    for f in rec["sources"]:
        h.update(open(os.path.join(ROOT, "llama_decoder_forward_fwd_b200", "csrc", f), "rb").read())
    if h.hexdigest()[:16] != rec["source_sha"]:
        return None  # the kernel changed since the counters were taken
    return rec["dram_bytes_per_launch"]


# ---------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch

    import llama_decoder_forward_fwd_b200 as L
    import seeded_inputs as S

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = S.WORKLOADS[WORKLOAD]
    shape, B, T, G = w.shape, w.batch, w.prompt_len, w.decode_steps
    peaks, peak_src = load_peaks()

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        cpu = oracle_sample(shape, w.seed, T, G)  # before the first GPU call

    glob, layers = S.make_weights(shape, w.seed, device=dev)
    stream = torch.cuda.Stream(device=dev)
    extra = (L.LLM_FLAG_FUSED_DECODE if args.fused else 0) | (L.LLM_FLAG_PDL if args.pdl else 0)
    model = L.Model(shape, glob, layers, max_batch=B, max_tokens=B * T,
                    flags=extra | (0 if args.no_graph else L.LLM_FLAG_CUDA_GRAPH), stream=stream, device=dev)
    prompt = S.make_tokens(w.seed, B, T, shape.vocab).to(dev)
    gen = torch.zeros(G + 1, B, dtype=torch.int32, device=dev)

    def one_step(ev=None):
        L.llm_kv_cache_reset(model.h)
        L.llm_prefill(model.h, prompt, gen[0])
        if ev is not None:
            ev.record(stream)
        for i in range(G):
            L.llm_decode_step(model.h, gen[i], gen[i + 1])

    def barrier():
        replica_barrier(world)

    def max_over_ranks(x):
        return replica_max(x, world, dev)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize(dev)

    # ---- timed region (device time, CUDA events on the model's stream) ----
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        for k in range(args.steps):
            starts[k].record(stream)
            one_step(mids[k])
            ends[k].record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    pre_ms = [s.elapsed_time(m) for s, m in zip(starts, mids)]
    dec_ms = [m.elapsed_time(e) for m, e in zip(mids, ends)]
    total_s = max_over_ranks(sum(step_ms) / 1e3)
    clocks = clk.summary()
    L.llm_synchronize(model.h)
    tokens_per_step = B * (T + G)
    value = replica_throughput(world, args.steps, tokens_per_step, total_s)

    S_mean = T + G / 2
    prefill_flops, decode_bytes, kbytes, kflops = work_model(shape, B, T, S_mean)
    pre_s = max_over_ranks(statistics.mean(pre_ms) / 1e3)
    dec_s = max_over_ranks(statistics.mean(dec_ms) / 1e3)
    prefill = {"tok_s": B * T / pre_s, "ms": pre_s * 1e3, "tflops": prefill_flops / pre_s / 1e12,
               "frac_of_bf16_peak": prefill_flops / pre_s / 1e12 / peaks["bf16_tflops"],
               "peak_tflops": peaks["bf16_tflops"], "peak_kind": f"{peak_src} burst"}
    decode = {"tok_s": B * G / dec_s, "ms_per_token": dec_s * 1e3 / G,
              "gbs": decode_bytes * G / dec_s / 1e9,
              "frac_of_hbm": decode_bytes * G / dec_s / 1e9 / peaks["hbm_gbs"], "peak_gbs": peaks["hbm_gbs"],
              "bytes_per_step": decode_bytes}

    # ---- e2e: host buffers through the public API, copies inside the timed region ----
    host_prompt = prompt.cpu().pin_memory()
    host_out = torch.empty_like(gen, device="cpu").pin_memory()
    dprompt = torch.empty_like(prompt)
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    for k in range(args.steps):
        e_s[k].record(stream)
        with torch.cuda.stream(stream):
            dprompt.copy_(host_prompt, non_blocking=True)
        L.llm_kv_cache_reset(model.h)
        L.llm_prefill(model.h, dprompt, gen[0])
        for i in range(G):
            L.llm_decode_step(model.h, gen[i], gen[i + 1])
        with torch.cuda.stream(stream):
            host_out.copy_(gen, non_blocking=True)
        e_e[k].record(stream)
    torch.cuda.synchronize(dev)
    e2e_s = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e)) / 1e3)
    e2e = {"value": replica_throughput(world, args.steps, tokens_per_step, e2e_s), "unit": "tokens/s",
           "h2d_bytes_per_step": host_prompt.numel() * 4, "d2h_bytes_per_step": host_out.numel() * 4}

    # ---- per-kernel CUDA-event timing of one step (roofline of the dominant kernel) ----
    tm = L.Model(shape, model.glob, model.layers, max_batch=B, max_tokens=B * T,
                 flags=extra | L.LLM_FLAG_KERNEL_TIMING | L.LLM_FLAG_CUDA_GRAPH, stream=stream, device=dev)
    gen2 = torch.zeros_like(gen)
    L.llm_prefill(tm.h, prompt, gen2[0])
    kt_pre = L.llm_kernel_times(tm.h, reset=True)
    for i in range(G):
        L.llm_decode_step(tm.h, gen2[i], gen2[i + 1])
    kt_dec = L.llm_kernel_times(tm.h, reset=True)
    tm.free()
    fused = kt_dec["step"][1] > 0  # decode steps ran as one launch each
    shares = {}
    for name, (ms, n) in kt_pre.items():
        if n:
            shares["prefill/" + name] = (ms, n)
    for name, (ms, n) in kt_dec.items():
        if n:
            shares["decode/" + name] = (ms, n)
    tot = sum(ms for ms, _ in shares.values())
    dom = max(shares, key=lambda k: shares[k][0])
    ms, n = shares[dom]
    avg_s = ms / n / 1e3
    phase, kind = dom.split("/")
    if phase == "decode" and kind in kbytes:
        achieved = kbytes[kind] / avg_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": ncu_traffic("decode/" + kind),
                "kernel": dom, "bytes_per_launch": kbytes[kind], "avg_launch_us": avg_s * 1e6,
                "launches": n, "peak_source": f"{peak_src} hbm_gbs"}
    else:
        per = kflops.get(kind, 0)
        achieved = per / avg_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": ncu_traffic(dom), "kernel": dom,
                "flops_per_launch": per, "avg_launch_us": avg_s * 1e6, "launches": n,
                "peak_source": f"{peak_src} bf16_tflops (burst)"}
    kernel_table = {k: {"ms": round(v[0], 3), "launches": v[1], "share": round(v[0] / tot, 4)}
                    for k, v in sorted(shares.items(), key=lambda kv: -kv[1][0])}
    model.free()
    workloads = None
    if world == 1 and not args.no_workloads:
        # after the timed region: the headline weights go, each workload brings its own
        del glob, layers, model, tm
        torch.cuda.empty_cache()
        workloads = workloads_block()

    if rank != 0:
        return
    line = {
        "impl": "ours", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_s * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,0.02) bf16 weights of the Llama-3-8B architecture, uniform token ids",
        "config": {"workload": WORKLOAD, "batch": B, "prompt_len": T, "decode_steps": G,
                   "layers": shape.n_layers, "dim": shape.dim, "vocab": shape.vocab,
                   "l2": "inputs larger than L2: every step streams 16 GB of weights",
                   "cuda_graph_decode": not args.no_graph, "decode_kernel": "fused step" if fused else "layerwise", "pdl": bool(args.pdl),
                   "parallelism": f"replicas x{world}"},
        "prefill": prefill, "decode": decode, "roofline": roof, "kernels": kernel_table,
        "cpu_baseline": ({k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample")} if cpu else None),
        "e2e": e2e,
        "gpu_launches": args.steps * ((5 * shape.n_layers + 2) +
                                      G * (1 if fused else 5 * shape.n_layers + 2)),
        "clocks": clocks,
    }
    if workloads is not None:
        line["workloads"] = workloads
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- the other workloads
def run_workload(args):
    """The --workload command: one JSON line for that workload."""
    print(json.dumps(measure_workload(args.workload, args.steps, args.warmup, args.fused, args.no_graph)), flush=True)


# the other workloads, summarised in the headline line (decode and prefill at each one's own sizes)
OTHER_WORKLOADS = ("llama3-8b-bf16-b16-kv4k8k-g128", "llama2-7b-mha-bf16-b8-p1024-g256",
                   "llama3-8b-bf16-b1-kv8k-g128", "llama3-8b-mqa-bf16-b1-p2048-g256")


def workloads_block(steps=1, warmup=1):
    """Compact decode (and prefill) numbers of OTHER_WORKLOADS, one pass each after a warm-up."""
    import torch
    out = {}
    for name in OTHER_WORKLOADS:
        d = measure_workload(name, steps, warmup, fused=False, no_graph=False, kernel_times=False)
        rec = {"batch": d["config"]["batch"], "decode_steps": d["config"]["decode_steps"],
               "decode_tok_s": round(d["decode"]["tok_s"], 1),
               "decode_ms_per_step": round(d["decode"]["ms_per_step"], 4),
               "decode_frac_of_hbm": round(d["decode"]["frac_of_hbm"], 4)}
        if d["config"]["input"] == "kv_prefilled":
            rec["cache_lengths"] = d["config"]["cache_lengths"]
        if "prefill" in d:
            rec["prompt_len"] = d["config"]["prompt_len"]
            rec["prefill_tok_s"] = round(d["prefill"]["tok_s"], 1)
            rec["prefill_frac_of_bf16_peak"] = round(d["prefill"]["frac_of_bf16_peak"], 4)
        out[name] = rec
        torch.cuda.empty_cache()
    return out


def measure_workload(name, steps, warmup, fused=False, no_graph=False, kernel_times=True):
    """Prefill and decode throughput of a workload other than the headline one (one GPU).

    Token workloads: a prefill of the prompt, then greedy decode steps (CUDA
    graphs). Hidden-state workloads: the layer stack on N(0,1) hidden states, then
    hidden-state decode steps. Pre-filled-cache workloads: N(0,1) keys and values
    written straight into the cache at the seeded ragged lengths (drawn on the
    device: timing only, parity is the tests'), then decode steps.
    """
    import torch

    import llama_decoder_forward_fwd_b200 as L
    import seeded_inputs as S

    w = S.WORKLOADS[name]
    shape, B, T, G = w.shape, w.batch, w.prompt_len, w.decode_steps
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    glob, layers = S.make_weights(shape, w.seed, device=dev)
    stream = torch.cuda.Stream(device=dev)
    graph = w.input_kind != "hidden" and not no_graph
    flags = (L.LLM_FLAG_CUDA_GRAPH if graph else 0) | (L.LLM_FLAG_FUSED_DECODE if fused else 0)
    mt = B * T if T else B
    model = L.Model(shape, glob, layers, max_batch=B, max_tokens=mt, flags=flags, stream=stream, device=dev)
    D, Hk, d, Ln = shape.dim, shape.n_kv_heads, shape.head_dim, shape.n_layers
    if w.input_kind == "kv_prefilled":
        lens = S.make_kv_prefill(shape, w.seed, B, *w.kv_len_range, layers=[])[0].tolist()
    else:
        lens = [T] * B
    tok0 = S.make_tokens(w.seed, B, max(T, 1), shape.vocab).to(dev)
    hid = S.make_hidden(w.seed, B, T, D).to(dev) if w.input_kind == "hidden" else None
    out_h = torch.empty_like(hid) if hid is not None else None
    x1 = S.make_hidden(w.seed, B, 1, D, tag="decode")[:, 0].contiguous().to(dev) if hid is not None else None
    o1 = torch.empty_like(x1) if x1 is not None else None
    gen = torch.zeros(G + 1, B, dtype=torch.int32, device=dev)
    gen[0] = S.make_tokens(w.seed, B, 1, shape.vocab, tag="decode0")[:, 0].to(dev)  # read by cache-only decode

    def prefill():
        L.llm_kv_cache_reset(model.h)
        if w.input_kind == "tokens":
            L.llm_prefill(model.h, tok0, gen[0])
        elif w.input_kind == "hidden":
            L.llm_prefill_hidden(model.h, hid, out_h)
        else:
            L.llm_kv_cache_set_lens(model.h, lens)

    def decode():
        for i in range(G):
            if w.input_kind == "hidden":
                L.llm_decode_step_hidden(model.h, x1, o1)
            else:
                L.llm_decode_step(model.h, gen[i], gen[i + 1])

    if w.input_kind == "kv_prefilled":
        kc, vc = model.kv_cache_tensors()
        kc.normal_()
        vc.normal_()
        torch.cuda.synchronize(dev)
    for _ in range(warmup):
        prefill()
        decode()
    torch.cuda.synchronize(dev)
    pre_ms, dec_ms = [], []
    with ClockSampler(0) as clk:
        for _ in range(steps):
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(stream)
            prefill()
            e1.record(stream)
            decode()
            e2.record(stream)
            torch.cuda.synchronize(dev)
            pre_ms.append(e0.elapsed_time(e1))
            dec_ms.append(e1.elapsed_time(e2))
    L.llm_synchronize(model.h)
    model.free()
    kt = {}
    if kernel_times:
        # per-kernel decode time: a second pass with the library's CUDA-event timing
        tm = L.Model(shape, model.glob, model.layers, max_batch=B, max_tokens=mt,
                     flags=flags | L.LLM_FLAG_KERNEL_TIMING, stream=stream, device=dev)
        model = tm
        if w.input_kind == "kv_prefilled":
            kc, vc = model.kv_cache_tensors()
            kc.normal_()
            vc.normal_()
            torch.cuda.synchronize(dev)
        for rep in range(2):  # the first pass captures the graphs
            prefill()
            L.llm_kernel_times(model.h, reset=True)
            decode()
            kt = L.llm_kernel_times(model.h, reset=True)
        model.free()
    # algorithmic work: every weight once per decode step, each sequence's cache once
    head = shape.has_embed_and_head
    S_mean = sum(lens) / B + G / 2
    prefill_flops, _, kind_bytes, _ = work_model(shape, B, T, S_mean)
    kernels = {k: {"ms_per_step": ms / G, "launches_per_step": n / G,
                   "gbs": (kind_bytes[k] * n / G) / (ms / G) / 1e6 if k in kind_bytes and ms else None}
               for k, (ms, n) in kt.items() if n}
    lin_params = Ln * (D * (shape.n_heads + 2 * Hk) * d + shape.n_heads * d * D + 3 * D * shape.ffn_hidden)
    esz = 2 if shape.dtype == "bf16" else 4
    if not head:
        prefill_flops -= 2 * B * D * shape.vocab
    step_bytes = esz * (lin_params + (shape.vocab * D if head else 0)) + Ln * B * 2 * Hk * d * esz * S_mean
    dec_s = statistics.median(dec_ms) / 1e3
    line = {"impl": "ours", "workload": w.name, "metric": "decode tokens/s; % of measured HBM (and prefill % of bf16 peak)",
            "n_gpus": 1, "steps": steps, "warmup": warmup, "dtype": shape.dtype, "data": "synthetic",
            "config": {"workload": w.name, "batch": B, "prompt_len": T, "decode_steps": G, "input": w.input_kind,
                       "cache_lengths": [min(lens), max(lens)], "cuda_graph_decode": graph,
                       "decode_kernel": "fused step" if fused else "layerwise"},
            "decode": {"tok_s": B * G / dec_s, "ms_per_step": dec_s * 1e3 / G, "gbs": step_bytes * G / dec_s / 1e9,
                       "frac_of_hbm": step_bytes * G / dec_s / 1e9 / peaks["hbm_gbs"], "bytes_per_step": step_bytes,
                       "peak_gbs": peaks["hbm_gbs"], "peak_source": peak_src, "kernels": kernels},
            "clocks": clk.summary()}
    if w.input_kind != "kv_prefilled":
        pre_s = statistics.median(pre_ms) / 1e3
        line["prefill"] = {"tok_s": B * T / pre_s, "ms": pre_s * 1e3, "tflops": prefill_flops / pre_s / 1e12,
                           "frac_of_bf16_peak": (prefill_flops / pre_s / 1e12 / peaks["bf16_tflops"]
                                                 if shape.dtype == "bf16" else None)}
    line["value"] = line["decode"]["tok_s"]
    line["unit"] = "tokens/s"
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="leave out the compact block of the other workloads' numbers (single GPU only)")
    ap.add_argument("--pdl", action="store_true",
                    help="programmatic dependent launch between consecutive kernels")
    ap.add_argument("--fused", action="store_true",
                    help="decode each step as the fused single-launch kernel instead of one launch per "
                         "projection and attention")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="another workload of seeded_inputs.WORKLOADS: prefill and decode throughput on one GPU "
                         "(the default is the headline benchmark)")
    args = ap.parse_args()
    if args.workload != WORKLOAD:
        if args.impl == "ours":
            run_workload(args)
        elif int(os.environ.get("RANK", "0")) == 0:
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm times the headline workload only"}))
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
