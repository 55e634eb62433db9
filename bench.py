#!/usr/bin/env python
"""Benchmark of masked block-diffusion generation at batch 1 on B200.

One step = prefill of the prompt (causal, into the KV cache) + for each canvas:
denoising passes until the canvas is full (bidirectional canvas pass, LM-head
confidence, commit) + append of the finished canvas to the KV cache. Default
workload: the 26B-parameter MoE (30 layers, d 2816, 128 experts top-8), prompt 4096,
one 256-position canvas, confidence threshold 0.9 with the step-budget floor, at most
48 passes. Synthetic data: seeded random-init weights N(0, 0.02) and uniform prompt
tokens. The 48 GB of weights exceed the 126 MB L2, so no flush is needed between
steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). Under torchrun every rank runs its own replica
(independent requests, weak scaling); the time is the max over ranks.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "committed tokens/s and denoise passes/s at batch 1; % of bf16 tensor-core peak"
TIMING_STRIDE = 6   # kernel timing brackets layers 0, 6, 12, ... of each pass
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
GEMM_SOURCE = os.path.join(ROOT, "masked_block_diffusion_b200", "csrc", "gemm_tc.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "moe_gate_up_gemm_moe26b.md")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c3-moe26b-canvas")
    ap.add_argument("--batch", type=int, default=0, help="requests per GPU (default: the workload's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    # profiling runs only (smaller captures); the reported workload never uses them
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling)")
    ap.add_argument("--max-steps", type=int, default=0, help="override the step budget (profiling)")
    ap.add_argument("--timing-all", action="store_true", help="time every kernel group (diagnostic)")
    return ap.parse_args()


def resolve_workload(args):
    from dataclasses import replace
    from synth import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.layers:
        w = replace(w, model=w.model.with_layers(args.layers), name=f"{w.name}-{args.layers}L")
    if args.max_steps:
        w = replace(w, max_steps=args.max_steps, name=f"{w.name}-{args.max_steps}steps")
    return w


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_config(w, n_gpus, batch=None):
    return {
        "workload": f"{w.name}: prompt {w.prefix}, {w.n_canvases} canvas(es) of {w.model.canvas}, "
                    f"{w.model.name} ({w.model.n_layers} layers, d {w.model.d_model}, "
                    f"{w.model.n_experts} experts top-{w.model.top_k}, vocab {w.model.vocab})",
        "prefix": w.prefix,
        "canvas": w.model.canvas,
        "n_canvases": w.n_canvases,
        "batch_per_gpu": batch or w.batch,
        "policy": (f"top-{w.k}" if w.policy == "topk" else f"threshold {w.tau} + step-budget floor"),
        "max_steps": w.max_steps,
        "parallelism": "replicas" if n_gpus == 1 else f"replicas x{n_gpus} (independent requests)",
        "l2": "inputs larger than L2 (48 GB of weights streamed per pass)",
    }


# ------------------------------------------------------------------ algorithmic work

def pass_flops(cfg, T, P, R):
    """Algorithmic flops of one canvas pass over T tokens with prefix P and R masked rows."""
    d, F, hd = cfg.d_model, cfg.ffn_dim, cfg.head_dim
    k = 1 if cfg.dense else cfg.top_k
    lin = 2 * T * d * (cfg.q_dim + 2 * cfg.kv_dim) + 2 * T * cfg.q_dim * d   # QKV, O
    lin += 2 * T * k * 3 * F * d                                              # experts
    if not cfg.dense:
        lin += 2 * T * d * cfg.n_experts                                      # router
    attn = 4 * T * (P + cfg.canvas) * cfg.n_heads * hd
    return cfg.n_layers * (lin + attn) + 2 * R * d * cfg.vocab


def gate_up_bytes(cfg, T):
    """Algorithmic HBM bytes of one grouped gate/up GEMM launch (one layer, T tokens):
    every expert's gate and up rows (bf16), the gathered token rows as a bf16 hi/lo
    pair, and the SwiGLU output written as a hi/lo pair."""
    E = max(1, cfg.n_experts)
    k = 1 if cfg.dense else cfg.top_k
    N = T * k
    return E * 2 * cfg.ffn_dim * cfg.d_model * 2 + N * cfg.d_model * 4 + N * cfg.ffn_dim * 4


def recorded_traffic():
    """Per-launch DRAM bytes of the gate/up GEMM from the committed ncu summary, if the
    kernel source is unchanged since the capture; else None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    txt = open(TRAFFIC_FILE).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"gemm_source_sha256:\s*([0-9a-f]+)", txt)
    if not m or not h:
        return None
    cur = hashlib.sha256(open(GEMM_SOURCE, "rb").read()).hexdigest()
    return float(m.group(1)) if h.group(1) == cur else None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU baseline (oracle)

def oracle_sample(w, passes_per_canvas, reps=1):
    """Times the oracle on a bounded sample of the workload and scales it to one step.

    Sample: one full-width layer of the model (fresh seeded weights of the same shapes),
    run as causal prefill over the prompt and as one bidirectional canvas pass over the
    cached prompt, plus the LM head with confidence over the canvas rows. One step is
    then n_layers * (prefill layer + (passes + 1) * canvas layer) + passes * LM head per
    canvas. Weight generation is input setup and is not timed.
    """
    import numpy as np
    import threadpoolctl
    from oracle import OracleModel, lm_head_conf
    from synth import gen_weights, prompt_tokens

    cfg = w.model.with_layers(1)
    W = gen_weights(cfg, threads=os.cpu_count() or 8)
    m = OracleModel(cfg, W)
    prompt = prompt_tokens(cfg.vocab, w.prompt_seed, w.prefix)
    C = cfg.canvas
    canvas = np.full(C, cfg.mask_id)
    mask = np.ones(C, bool)
    times = []
    S = passes_per_canvas
    for _ in range(reps):
        t0 = time.perf_counter()
        m.prefill(0, prompt)
        t1 = time.perf_counter()
        x, _, _ = m._canvas_forward(0, canvas, mask)
        t2 = time.perf_counter()
        lm_head_conf(x, m.final_norm, m.head, cfg.mask_id, cfg.rms_eps)
        t3 = time.perf_counter()
        t_pre, t_pass, t_head = t1 - t0, t2 - t1, t3 - t2
        L = w.model.n_layers
        step = L * t_pre + w.n_canvases * (L * (S + 1) * t_pass + S * t_head)
        times.append((step, t3 - t0))
    threads = max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()] or [1])
    sample = (f"oracle (numpy fp64) on one full-width layer of {w.model.name}: causal prefill of "
              f"{w.prefix} tokens, one canvas pass of {C} positions over that prefix, LM head over "
              f"{C} rows; scaled to {w.model.n_layers} layers x ({S} passes + append) per canvas, "
              f"x{w.n_canvases} canvas(es), + prefill")
    return times, threads, sample


def expected_passes(w):
    """Passes per canvas of the workload's schedule: top-k fills the canvas in C / k
    passes; with random weights the confidences never reach the 0.9 threshold, so the
    step-budget floor runs every one of the max_steps passes."""
    return w.model.canvas // w.k if w.policy == "topk" else w.max_steps


# ------------------------------------------------------------------ distributed plumbing

def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    from masked_block_diffusion_b200.replicas import max_over_ranks as _max
    return float(v) if world == 1 else _max(v, "cuda")


def prefill_flops(cfg, n):
    d, F, hd = cfg.d_model, cfg.ffn_dim, cfg.head_dim
    k = 1 if cfg.dense else cfg.top_k
    lin = 2 * n * d * (cfg.q_dim + 2 * cfg.kv_dim) + 2 * n * cfg.q_dim * d + 2 * n * k * 3 * F * d
    if not cfg.dense:
        lin += 2 * n * d * cfg.n_experts
    attn = 2 * n * n * cfg.n_heads * hd          # causal: half of 4 n^2 H hd
    return cfg.n_layers * (lin + attn)


# ------------------------------------------------------------------ our arm

def run_ours(args):
    import numpy as np
    import torch
    from masked_block_diffusion_b200 import Denoiser, DllmError, binding, make_policy
    from synth import WORKLOADS, prompt_tokens
    from synth.device import device_blob

    world, rank, local = dist_setup()
    w = resolve_workload(args)
    cfg = w.model
    C = cfg.canvas
    Bq = args.batch or w.batch   # independent requests on this GPU
    max_ctx = w.prefix + w.n_canvases * C
    blob = device_blob(cfg)
    den = Denoiser(cfg, blob, max_ctx=max_ctx, max_batch=Bq)
    del blob
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    h, st = den.h, den.stream
    # requests of this rank: seeds prompt_seed + global request id
    prompt_np = np.stack([prompt_tokens(cfg.vocab, w.prompt_seed + rank * Bq + r, w.prefix) for r in range(Bq)])
    d_prompt = torch.from_numpy(prompt_np).cuda()
    d_canvas = torch.empty((Bq, C), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    pol = make_policy(w.policy, w.k, w.tau, w.floor)
    # the two grouped expert GEMMs are timed inside the graph (--timing-all: every kernel group)
    # every TIMING_STRIDE-th layer is bracketed with events: few enough event nodes that
    # the timed pass runs close to an untimed one, every kind still sampled each pass
    binding.dllm_set_timing(h, ((1 << binding.DLLM_TIMING_KINDS) - 1 if args.timing_all
                                else (1 << binding.DLLM_TIMING_GATE_UP) | (1 << binding.DLLM_TIMING_DOWN))
                            | (TIMING_STRIDE << binding.DLLM_TIMING_STRIDE_SHIFT))

    def step(gen_events=None):
        for r in range(Bq):
            binding.dllm_reset(h, r)
            binding.dllm_prefill(h, r, d_prompt[r].data_ptr(), w.prefix)
        passes = 0
        for _ in range(w.n_canvases):
            if gen_events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(st)
            code, steps = binding.dllm_generate_block(h, Bq, w.max_steps, pol, d_canvas.data_ptr())
            if code != 0:
                raise DllmError(code, "dllm_generate_block", binding.dllm_last_error(h))
            if gen_events is not None:
                e1 = torch.cuda.Event(enable_timing=True)
                e1.record(st)
                gen_events.append((e0, e1))
            passes += max(steps)
            binding.dllm_append_kv(h, Bq, 0)
        return passes

    for _ in range(args.warmup):
        step()
    st.synchronize()
    barrier(world)
    binding.dllm_timing_read(h, reset=True)
    launches0 = binding.dllm_launch_count(h)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    gen_events = []
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_start.record(st)
    passes = 0
    for _ in range(args.steps):
        passes += step(gen_events)
    t_stop.record(st)
    st.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()
    launches = binding.dllm_launch_count(h) - launches0
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_stop), world)
    gen_ms = sum(a.elapsed_time(b) for a, b in gen_events)
    kms, kn, kbytes = binding.dllm_timing_read(h, reset=True)
    barrier(world)

    from masked_block_diffusion_b200.replicas import aggregate_rate
    value = aggregate_rate(args.steps * w.n_canvases * C * Bq, world, elapsed_ms / 1e3)
    passes_per_canvas = passes / (args.steps * w.n_canvases)
    peaks, peak_src = load_peaks()

    # dominant kernel: the grouped gate/up GEMM (expert weights streamed from HBM)
    GU, DN = binding.DLLM_TIMING_GATE_UP, binding.DLLM_TIMING_DOWN
    if kn[GU] == 0 or kms[GU] <= 0:
        raise RuntimeError("no gate/up GEMM launch was timed")
    gu_ms = kms[GU] / kn[GU]
    gu_bytes = kbytes[GU] / kn[GU]          # mean algorithmic bytes per launch (routed experts)
    achieved = kbytes[GU] / (kms[GU] / 1e3) / 1e9
    peak_hbm = float(peaks["hbm_gbs"])
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak_hbm, "unit": "GB/s",
                "frac": round(achieved / peak_hbm, 4), "traffic": recorded_traffic(),
                "kernel": "grouped expert gate/up GEMM + SwiGLU (tcgen05, one launch per layer)",
                "bytes_per_launch": round(gu_bytes), "bytes_per_launch_all_experts": gate_up_bytes(cfg, C * Bq),
                "avg_launch_ms": round(gu_ms, 5), "launches_timed": kn[GU],
                "bytes_note": "weights of the experts each launch routed to + token pair rows + SwiGLU output",
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else "fallback"}
    dn_ms = max(1e-9, kms[DN] / max(1, kn[DN]))
    dn_gbs = kbytes[DN] / max(1e-9, kms[DN] / 1e3) / 1e9

    step_flops = Bq * prefill_flops(cfg, w.prefix) + w.n_canvases * (
        passes_per_canvas * pass_flops(cfg, C * Bq, w.prefix, C * Bq) + pass_flops(cfg, C * Bq, w.prefix, 0))
    tc_peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    step_tc = step_flops / (elapsed_ms / args.steps / 1e3) / (tc_peak * 1e12)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(elapsed_ms / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random-init weights N(0,0.02), uniform prompt tokens)",
        "config": workload_config(w, world, Bq),
        "passes_per_s": round(world * passes / (gen_ms / 1e3), 2) if gen_ms > 0 else None,
        "passes_per_canvas": passes_per_canvas,
        "denoise_ms_per_pass": round(gen_ms / max(1, passes), 4),
        "step_tc_frac": round(step_tc, 4),
        "step_tc_note": (f"algorithmic flops per step / step time / sustained bf16 peak {tc_peak} TFLOP/s "
                         f"({peak_src}); batch 1 is HBM-bound on expert weights"),
        "roofline": roofline,
        "down_gemm": {"avg_launch_ms": round(dn_ms, 5), "achieved_gbs": round(dn_gbs, 1),
                      "bytes_per_launch": round(kbytes[DN] / max(1, kn[DN]))},
        "experts_routed_per_layer": round((kbytes[GU] / kn[GU] - Bq * C * cfg.top_k * (cfg.d_model + cfg.ffn_dim) * 4)
                                          / (2 * cfg.ffn_dim * cfg.d_model * 2), 2),
        "gpu_launches": int(launches),
        # mean bracketed launch time x launches per pass (n_layers, or 1 for the LM head)
        "kernel_ms_per_pass": {binding.TIMING_NAMES[k]: round(kms[k] / kn[k] * (
                                   1 if k == binding.DLLM_TIMING_HEAD else cfg.n_layers), 4)
                               for k in range(binding.DLLM_TIMING_KINDS) if kn[k]},
        "timing_layer_stride": TIMING_STRIDE,
        "clocks": clk,
    }

    if not args.no_e2e:
        prompts = np.ascontiguousarray(prompt_np)
        toks = np.zeros((Bq, w.n_canvases * C), dtype=np.int32)
        stp = np.zeros((Bq * w.n_canvases,), dtype=np.int32)
        binding.dllm_set_timing(h, 0)
        for _ in range(max(1, args.warmup)):
            binding.dllm_generate(h, Bq, prompts.ctypes.data, w.prefix, w.n_canvases, w.max_steps, pol,
                                  toks.ctypes.data, stp.ctypes.data)
        barrier(world)
        t0 = time.perf_counter()
        e_passes = 0
        for _ in range(args.steps):
            binding.dllm_generate(h, Bq, prompts.ctypes.data, w.prefix, w.n_canvases, w.max_steps, pol,
                                  toks.ctypes.data, stp.ctypes.data)
            e_passes += int(stp.reshape(Bq, w.n_canvases).max(axis=0).sum())
        t1 = time.perf_counter()
        e_s = max_over_ranks(t1 - t0, world)
        out["e2e"] = {"value": round(world * args.steps * w.n_canvases * C * Bq / e_s, 2), "unit": UNIT,
                      "h2d_bytes_per_step": int(prompts.nbytes),
                      "d2h_bytes_per_step": int(toks.nbytes + 4 * Bq * e_passes // args.steps),
                      "api": "dllm_generate (host prompt in, host tokens out)"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        times, threads, sample = oracle_sample(w, passes_per_canvas, reps=1)
        out["cpu_baseline"] = {"value": round(w.n_canvases * C / times[0][0], 5), "unit": UNIT, "cores": threads,
                               "kind": "oracle", "sample": sample,
                               "sample_seconds": round(times[0][1], 2)}
    den.close()
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ reference arm

def run_reference(args):
    """The oracle (plain numpy CPU code), timed on the host cores on a bounded sample of
    the same workload per step; rank 0 only."""
    from synth import WORKLOADS
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = resolve_workload(args)
    C = w.model.canvas
    times, threads, sample = oracle_sample(w, expected_passes(w), reps=args.warmup + args.steps)
    steps = [t[0] for t in times[args.warmup:]]
    step_s = statistics.mean(steps)
    value = w.n_canvases * C / step_s
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded random-init weights N(0,0.02), uniform prompt tokens)",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
