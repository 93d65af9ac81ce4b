"""Benchmark: Llama-2-7B-shaped low-rank decoder, greedy decode on a dense KV
cache with per-layer CUDA-graph replay.

Workload (one "step"): prefill a batch of B prompts of 2048 synthetic tokens
into the contiguous bf16 KV cache, then 128 greedy decode steps.  32 layers,
hidden 4096, 32 heads of 128, SwiGLU 11008, vocab 32000, every projection
factorized at retention 0.6 (rank 1216 for 4096x4096, 1792 for
4096<->11008), random-init seeded weights.  The metric is decode tokens/s
(whole job, all GPUs); prefill tokens/s is reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B]
    python bench.py --impl reference ...   (the CPU oracle, timed on host cores)

For N > 1 the script runs under torchrun: every rank serves its own replica
(independent sequences, no collective on the data path); times are the max
over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
PROMPT = 2048
DECODE_STEPS = 128
METRIC = "low-rank 7B decode tok/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["decode7b", "linear-sweep", "bert", "mixed-rank",
                                           "long-decode", "prefill-attn", "retention", "shared-basis"],
                    default="decode7b",
                    help="decode7b (default): the headline line; the others print one JSON "
                         "line per measured case of the isolated-linear sweep, the BERT-shaped "
                         "encoder, the mixed-rank model and decode over long histories "
                         "(1 GPU)")
    ap.add_argument("--layers", type=int, default=32,
                    help="decoder layers (default 32; fewer only for small profiling cases)")
    ap.add_argument("--no-l2-discard", action="store_true",
                    help="leave prefill rank activations to the normal L2 write-back (control "
                         "for measuring what discarding them saves)")
    ap.add_argument("--profile-step", action="store_true",
                    help="after warm-up, run the workload's unit of work once inside an NVTX "
                         "range 'profile_step' (for an ncu capture) and exit: decode7b one "
                         "prefill and two decode steps, bert one forward, prefill-attn one "
                         "rank-1216 layer prefill with the query formed in the attention kernel")
    return ap.parse_args()


# ------------------------------------------------------------ peaks ------

def max_over_ranks(values, world: int, device):
    """Element-wise max of per-rank timings over all ranks (every rank gets
    the result); a no-op for one rank."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units of all ranks per second, over the slowest rank's time."""
    return world * units_per_rank / (ms / 1e3)


TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "ncu_traffic_decode_layers_fused.txt")


def ncu_traffic(kernel: str, layers: int):
    """DRAM bytes per launch of the fused decode kernel from the committed ncu
    record (key: value lines: the kernel source's sha1, the layers the
    captured launch covered, dram__bytes_read.sum and dram__bytes_write.sum),
    scaled per layer to `layers`; None for other kernels or when the kernel
    source has changed since the capture."""
    import hashlib
    if kernel != "decode_layers_fused":
        return None
    src = os.path.join(ROOT, "rank_transformer_b200", "csrc", "decode_fused.cu")
    try:
        rec = {}
        for line in open(TRAFFIC_RECORD):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                rec[k.strip()] = v.strip()
        sha = hashlib.sha1(open(src, "rb").read()).hexdigest()
        if rec.get("kernel_source_sha1") != sha:
            return None
        per_layer = (float(rec["dram__bytes_read.sum"]) + float(rec["dram__bytes_write.sum"])) / \
            float(rec["layers_launched"])
    except (OSError, KeyError, ValueError):
        return None
    return per_layer * layers


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


# ----------------------------------------------------------- clocks ------

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region
    runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# -------------------------------------------------------- CPU oracle ------

def oracle_decode_sample(budget_s: float = 12.0, context: int = PROMPT):
    """Time the CPU oracle on a bounded sample of the decode workload: one
    7B-shaped low-rank layer (rank 1216 / 1792) decoding single tokens at a
    2048-token history, plus the 4096x32000 head, then scale to 32 layers.
    Returns (tok/s, cores, sample description)."""
    import numpy as np

    sys.path.insert(0, ROOT)
    from oracle import flashsvd_oracle as oracle
    from rank_transformer_b200 import synth

    rng = synth.rng_for(0)
    d, H, f = 4096, 32, 11008
    w = oracle.widen_layer(synth.decoder_layer_weights(rng, d, f, 1216, 1792))
    k_hist = oracle.from_bf16(synth.normal_bf16(rng, (1, context, H, 128)))
    v_hist = oracle.from_bf16(synth.normal_bf16(rng, (1, context, H, 128)))
    W_lm = oracle.from_bf16(synth.normal_bf16(rng, (d, 32000), d ** -0.5))
    g = np.ones(d)
    x = oracle.from_bf16(synth.normal_bf16(rng, (1, d)))
    t0 = time.perf_counter()
    oracle.lm_head(x, g, W_lm)
    t_head = time.perf_counter() - t0
    n, t_layer = 0, 0.0
    while t_layer < budget_s or n < 2:
        t0 = time.perf_counter()
        oracle.decoder_layer_decode(x, w, H, k_hist, v_hist, [context])
        t_layer += time.perf_counter() - t0
        n += 1
    per_token = 32 * t_layer / n + t_head
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = (f"{n} single-token decode steps of one 7B-shaped layer at context {context} "
              f"(+1 head GEMV), scaled to 32 layers; numpy float64")
    return 1.0 / per_token, cores, sample


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_decode_sample(budget_s=1.0)
    vals = []
    t_start = time.perf_counter()
    for _ in range(args.steps):
        v, cores, sample = oracle_decode_sample(budget_s=4.0)
        vals.append(v)
    wall = time.perf_counter() - t_start
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * wall / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "llama2-7b-shaped low-rank decoder, rho=0.6, B=1, ctx 2048, "
                               "greedy decode (oracle sample)", "batch": 1},
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------- ours -------

def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    sys.path.insert(0, ROOT)
    from rank_transformer_b200 import flashsvd as fs
    from rank_transformer_b200.model import LLAMA7B, DecoderModel

    B = args.batch
    import dataclasses
    cfg = dataclasses.replace(LLAMA7B, layers=args.layers)
    S_max = PROMPT + DECODE_STEPS
    fs.init(local, max_tokens=B * PROMPT, max_rank=2368, max_hidden=cfg.d, max_ffn=cfg.f)
    if args.no_l2_discard:
        fs.set_l2_discard(False)
    model = DecoderModel(cfg, B, S_max, seed=1234 + rank)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(99 + rank)
    prompt = torch.randint(0, cfg.vocab, (B, PROMPT), generator=gen, device="cuda",
                           dtype=torch.int32)
    stream = torch.cuda.Stream()
    model.capture(stream, compose=True)

    def one_step(ev=None):
        if ev:
            ev[0].record(stream)
        model.prefill(prompt, stream)
        if ev:
            ev[1].record(stream)
        for _ in range(DECODE_STEPS):
            model.decode_step(stream)
        if ev:
            ev[2].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one_step()
    stream.synchronize()

    if args.profile_step:
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("profile_step")
        with torch.cuda.stream(stream):
            model.prefill(prompt, stream)
            model.decode_step(stream)
            model.decode_step(stream)
        stream.synchronize()
        torch.cuda.nvtx.range_pop()
        per_step = model.step_kernels()
        model.release_graphs()
        print(json.dumps({"profile_step": "done", "launches_per_decode_step": per_step}))
        return 0

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = fs.launch_count()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_wall = time.perf_counter()
    torch.cuda.nvtx.range_push("timed_steps")
    with torch.cuda.stream(stream):
        for k in range(args.steps):
            one_step(events[k])
    stream.synchronize()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    if world > 1:
        dist.barrier()
    launches = fs.launch_count() - launches0
    clk = clocks.stop()

    pre_ms = sum(e[0].elapsed_time(e[1]) for e in events)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in events)
    tot_ms = sum(e[0].elapsed_time(e[2]) for e in events)
    pre_ms, dec_ms, tot_ms = max_over_ranks([pre_ms, dec_ms, tot_ms], world, "cuda")
    value = whole_job_rate(B * DECODE_STEPS * args.steps, world, dec_ms)
    prefill_tok_s = whole_job_rate(B * PROMPT * args.steps, world, pre_ms)
    peaks = measured_peaks()

    # Decode-step roofline: algorithmic bytes of the 128 steps / decode time.
    step_bytes = sum(model.decode_step_bytes(PROMPT + i) for i in range(DECODE_STEPS))
    dec_gbs = step_bytes * args.steps / (dec_ms / 1e3) / 1e9 if world == 1 else \
        step_bytes * args.steps / (dec_ms / 1e3) / 1e9

    # Dominant decode kernel: per-launch CUDA-event timings of one eager
    # decode step (the profiler brackets each library launch on the stream).
    # Steps at contexts PROMPT .. PROMPT + 2 (the timed region covers
    # PROMPT .. PROMPT + 127).
    model.seqlens.fill_(PROMPT)
    fs.profile_enable(True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            model.decode_step_eager(stream)
    prof = fs.profile_report(reset=True)
    fs.profile_enable(False)
    prof = {k: v for k, v in prof.items() if v["launches"] > 0}
    top = max(prof, key=lambda k: prof[k]["ms"])
    tp = prof[top]
    if top == "decode_layers_fused":
        # one launch = every decoder layer of a step: its algorithmic bytes
        # at the mean profiled context
        alg_per_launch = model.layers_decode_bytes(PROMPT + 1)
    else:
        alg_per_launch = tp["bytes"] / tp["launches"]
    achieved = alg_per_launch / (tp["ms"] / tp["launches"] / 1e3) / 1e9

    # Prefill roofline (tensor-core bound): algorithmic FLOPs of the timed
    # prefills / their time, and the dominant prefill kernel from one eager
    # prefill with every launch bracketed by CUDA events on its stream.
    pf_flops = model.prefill_flops(PROMPT)
    pf_tfs = pf_flops * args.steps / (pre_ms / 1e3) / 1e12
    fs.profile_enable(True)
    with torch.cuda.stream(stream):
        model.prefill(prompt, stream)
    pprof = fs.profile_report(reset=True)
    fs.profile_enable(False)
    pprof = {k: v for k, v in pprof.items() if v["launches"] > 0}
    ptop = max(pprof, key=lambda k: pprof[k]["ms"])
    pk = pprof[ptop]
    pk_tfs = pk["flops"] / (pk["ms"] / 1e3) / 1e12
    pf_total_ms = sum(v["ms"] for v in pprof.values())

    # End to end through the public call: pinned host prompt in, generated
    # tokens out, on the same stream, timed with events around everything.
    prompt_host = torch.empty((B, PROMPT), dtype=torch.int32, pin_memory=True)
    prompt_host.copy_(prompt.cpu())
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        out = model.generate(prompt_host, DECODE_STEPS, stream)
        e1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks([e0.elapsed_time(e1)], world, "cuda")[0]
    e2e_value = whole_job_rate(B * DECODE_STEPS, world, e2e_ms)
    assert out.shape == (B, DECODE_STEPS)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = oracle_decode_sample()
        cpu = {"value": v, "unit": "tok/s", "cores": cores, "kind": "oracle", "sample": sample}

    model.release_graphs()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": tot_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"llama2-7b-shaped low-rank decoder (rho=0.6, r=1216/1792), "
                                   f"B={B}, prefill {PROMPT} + {DECODE_STEPS} greedy decode steps, "
                                   + ("decode step = embedding + one fused launch of all 32 layers "
                                      "+ head, replayed as one CUDA graph" if model.plan is not None
                                      else "per-layer CUDA graphs"),
                       "batch": B, "prompt": PROMPT, "decode_steps": DECODE_STEPS,
                       "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (7.75 GB of factors streamed per step)"},
            "prefill": {
                "value": prefill_tok_s, "unit": "tok/s", "ms_per_step": pre_ms / args.steps,
                "roofline": {"bound": "tensor", "achieved": pf_tfs, "unit": "TFLOP/s",
                             "peak": peaks["bf16_tflops"], "frac": pf_tfs / peaks["bf16_tflops"],
                             "frac_of_sustained": pf_tfs / peaks["bf16_tflops_sustained"],
                             "flops_per_step": pf_flops,
                             "peak_source": peaks["source"] + " (dense bf16 GEMM, burst)"},
                "top_kernel": {"kernel": ptop, "launches": pk["launches"],
                               "share": pk["ms"] / pf_total_ms, "achieved": pk_tfs,
                               "unit": "TFLOP/s", "frac": pk_tfs / peaks["bf16_tflops"]},
                "kernel_times_ms": {k: round(v["ms"], 4) for k, v in sorted(pprof.items())}},
            "decode_hbm": {"achieved_gbs": dec_gbs, "peak_gbs": peaks["hbm_gbs"],
                           "frac": dec_gbs / peaks["hbm_gbs"],
                           "bytes_per_step": step_bytes / DECODE_STEPS},
            "roofline": {"bound": "hbm", "kernel": top, "achieved": achieved,
                         "algorithmic_bytes_per_launch": alg_per_launch,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"],
                         "traffic": ncu_traffic(top, cfg.layers),
                         "traffic_source": "ncu dram__bytes_read+write of a 2-layer launch of "
                                           "the same kernel source, scaled per layer",
                         "launches_timed": tp["launches"],
                         "peak_source": peaks["source"] + " (burst copy)"},
            "kernel_times_ms": {k: round(v["ms"], 4) for k, v in sorted(prof.items())},
            "e2e": {"value": e2e_value, "unit": "tok/s (prefill+decode wall, generated tokens)",
                    "h2d_bytes_per_step": 4 * B * PROMPT, "d2h_bytes_per_step": 4 * B * DECODE_STEPS,
                    "ms": e2e_ms},
            "gpu_launches": launches,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------- other workloads --

def _event_ms(fn, reps, stream):
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(reps):
        fn(i)
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps


def run_linear_sweep(args):
    """Isolated factorized linears, Llama-7B shapes: square 4096x4096 and the
    packed gate|up 4096 -> 2x11008 (+SwiGLU), r in {512, 1024, 2048}, M in
    {1, 8, 32} (HBM-bound GEMV path) and {512, 2048} (tcgen05 path).  Random
    factors of the SVD shapes; the calls rotate over enough factor copies
    that the factors come from HBM (2x L2 worth)."""
    import torch
    sys.path.insert(0, ROOT)
    from rank_transformer_b200 import flashsvd as fs
    torch.cuda.set_device(0)
    fs.init(0, max_tokens=2048, max_rank=4096, max_hidden=4096, max_ffn=11008)
    peaks = measured_peaks()
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    stream = torch.cuda.Stream()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    d, f = 4096, 11008

    def mat(r_, c_):
        return (torch.randn(r_, c_, device="cuda", generator=gen) * r_ ** -0.5).to(torch.bfloat16)

    for shape in ("square", "gateup"):
        for r in (512, 1024, 2048):
            if shape == "square":
                fp_bytes = 2 * (d * r + r * d)
            else:
                fp_bytes = 2 * (d * 2 * r + 2 * r * f)
            copies = max(1, min(64, math.ceil(2 * l2 / fp_bytes)))
            facs = [(mat(d, r), mat(r, d)) if shape == "square" else (mat(d, 2 * r), mat(2 * r, f))
                    for _ in range(copies)]
            for M in (1, 8, 32, 512, 2048):
                x = torch.randn(M, d, device="cuda", generator=gen).to(torch.bfloat16)
                n = d if shape == "square" else f
                y = torch.empty(M, n, device="cuda", dtype=torch.bfloat16)
                if shape == "square":
                    call = lambda i: fs.lowrank_linear(x, facs[i % copies][0], facs[i % copies][1], None,
                                                       y, M, d, r, d, stream)
                    flops = 2 * M * r * (d + d)
                    bytes_ = 2 * (d * r + r * d + M * d + M * d)
                else:
                    call = lambda i: fs.gateup_swiglu(x, facs[i % copies][0], facs[i % copies][1], y, M, d,
                                                      r, f, stream)
                    flops = 2 * M * (d * 2 * r + 2 * r * f)
                    bytes_ = 2 * (d * 2 * r + 2 * r * f + M * d + M * f)
                with torch.cuda.stream(stream):
                    for i in range(10):
                        call(i)
                    ms = _event_ms(call, 50, stream)
                fs.check_device_status(stream)
                gbs, tfs = bytes_ / (ms / 1e3) / 1e9, flops / (ms / 1e3) / 1e12
                hbm_bound = M <= 32
                print(json.dumps({
                    "workload": "linear-sweep", "shape": "4096x4096" if shape == "square" else
                    "gate|up 4096->2x11008 +SwiGLU", "r": r, "M": M, "us": round(ms * 1e3, 2),
                    "path": "split-K GEMV" if M <= 32 else "tcgen05 GEMM",
                    "bound": "hbm" if hbm_bound else "tensor",
                    "achieved": round(gbs if hbm_bound else tfs, 1),
                    "unit": "GB/s" if hbm_bound else "TFLOP/s",
                    "frac": round(gbs / peaks["hbm_gbs"] if hbm_bound else tfs / peaks["bf16_tflops"], 3),
                    "algorithmic_bytes": bytes_, "flops": flops, "factor_copies": copies}), flush=True)
            del facs
            torch.cuda.empty_cache()
    return 0


def _unfused_encoder_layer(x, w, B, S, H, eps):
    """One post-LN encoder layer in plain PyTorch eager, the unfused
    execution the streamed path is compared with: every factorized linear
    as two torch.matmul calls (the rank activation z materialised), torch's
    erf GELU, LayerNorm and scaled_dot_product_attention (no score matrix)."""
    import torch.nn.functional as F
    import torch
    M, d = x.shape
    D = d // H

    def lin(t, n):
        return torch.matmul(torch.matmul(t, w["U_" + n]), w["V_" + n]) + w["b_" + n]

    def heads(t):
        return t.view(B, S, H, D).transpose(1, 2)
    a = F.scaled_dot_product_attention(heads(lin(x, "q")), heads(lin(x, "k")), heads(lin(x, "v")))
    a = a.transpose(1, 2).reshape(M, d)
    h = F.layer_norm(x + lin(a, "o"), (d,), w["ln1_g"], w["ln1_b"], eps)
    u = F.gelu(lin(h, "up"))
    return F.layer_norm(h + lin(u, "dn"), (d,), w["ln2_g"], w["ln2_b"], eps)


def run_bert(args):
    """BERT-Base-shaped low-rank encoder: 12 layers, hidden 768, 12 heads,
    FFN 3072 (GELU), every linear at rank 192 with bias, batch 32 x 512,
    bf16, N(0,1) inputs (GLUE is not here; same shapes).  Throughput, the
    streamed FFN kernel's share, and memory against unfused execution:
    peak activation = device memory the forward holds beyond weights and
    input; transient = the largest intra-layer temporaries.  Unfused (torch
    eager, two matmuls per linear): torch allocator peaks.  Ours: the
    library workspace measured with cudaMemGetInfo around creating it (the
    part that grows with the token count: a workspace for these tokens
    minus one for 32 tokens) plus the caller's K/V buffers; no [M x f]
    buffer is allocated (max_ffn = 8), since the FFN is streamed."""
    import torch
    sys.path.insert(0, ROOT)
    from rank_transformer_b200 import flashsvd as fs
    from rank_transformer_b200.model import EncoderModel
    torch.cuda.set_device(0)
    B, S, d, H, f, r, nl = 32, 512, 768, 12, 3072, 192, 12
    M = B * S
    peaks = measured_peaks()

    def ws_bytes(tokens):
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        ctx = fs.Context(0, max_tokens=tokens, max_rank=r, max_hidden=d, max_ffn=8)
        free1 = torch.cuda.mem_get_info()[0]
        ctx.destroy()
        return free0 - free1
    ws_full, ws_small = ws_bytes(M), ws_bytes(32)
    fs.init(0, max_tokens=M, max_rank=r, max_hidden=d, max_ffn=8)
    if args.no_l2_discard:
        fs.set_l2_discard(False)
    before = torch.cuda.memory_allocated()
    m = EncoderModel(layers=nl, B=B, S=S, seed=3)
    model_bytes = torch.cuda.memory_allocated() - before   # weights + K/V buffers
    kv_bytes = m.k_buf.numel() * 2 + m.v_buf.numel() * 2
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4)
    x0 = torch.randn(M, d, device="cuda", generator=gen).to(torch.bfloat16)
    x = x0.clone()
    stream = torch.cuda.Stream()
    if args.profile_step:
        with torch.cuda.stream(stream):
            for _ in range(2):
                m.forward(x, stream)
            stream.synchronize()
            torch.cuda.nvtx.range_push("profile_step")
            m.forward(x, stream)
            stream.synchronize()
            torch.cuda.nvtx.range_pop()
        print(json.dumps({"profile_step": "done", "workload": "bert"}))
        return 0
    with torch.cuda.stream(stream):
        for _ in range(3):
            x.copy_(x0)
            m.forward(x, stream)
        ms = _event_ms(lambda i: m.forward(x, stream), 10, stream)
    fs.check_device_status(stream)
    fs.profile_enable(True)
    with torch.cuda.stream(stream):
        m.forward(x, stream)
    prof = fs.profile_report(reset=True)
    fs.profile_enable(False)
    tf = m.flops() / (ms / 1e3) / 1e12
    ours_act = (ws_full - ws_small) + kv_bytes

    # unfused torch eager over the same weights and input
    with torch.cuda.stream(stream):
        torch.cuda.synchronize()
        xu = x0.clone()
        base = torch.cuda.memory_allocated()
        torch.cuda.reset_peak_memory_stats()
        t = xu
        transient = 0
        for w in m.layers:
            live = torch.cuda.memory_allocated()
            torch.cuda.reset_peak_memory_stats()
            t = _unfused_encoder_layer(t, w, B, S, H, m.eps)
            transient = max(transient, torch.cuda.max_memory_allocated() - live)
        torch.cuda.synchronize()
        del t
        torch.cuda.reset_peak_memory_stats()
        base = torch.cuda.memory_allocated()
        t = xu
        for w in m.layers:
            t = _unfused_encoder_layer(t, w, B, S, H, m.eps)
        torch.cuda.synchronize()
        unfused_act = torch.cuda.max_memory_allocated() - base
        del t

        def unfused_fwd(i):
            t = xu
            for w in m.layers:
                t = _unfused_encoder_layer(t, w, B, S, H, m.eps)
        for _ in range(2):
            unfused_fwd(0)
        ms_unfused = _event_ms(unfused_fwd, 3, stream)
    ffn = prof.get("ffn_stream")
    line = {
        "workload": "bert", "config": {"layers": nl, "hidden": d, "heads": H, "ffn": f, "rank": r,
                                       "batch": B, "seq": S},
        "ms_per_forward": round(ms, 3), "sequences_per_s": round(B / (ms / 1e3), 1),
        "tokens_per_s": round(M / (ms / 1e3)), "tflops": round(tf, 1),
        "frac_of_bf16_peak": round(tf / peaks["bf16_tflops"], 3),
        "memory": {
            "ours_peak_activation_bytes": ours_act,
            "ours_workspace_bytes": ws_full, "ours_fixed_workspace_bytes": ws_small,
            "kv_buffer_bytes": kv_bytes, "model_allocation_bytes": model_bytes,
            "unfused_peak_activation_bytes": unfused_act,
            "unfused_peak_transient_bytes": transient,
            "ours_transient_bytes": ours_act,
            "peak_activation_reduction": round(1 - ours_act / unfused_act, 3),
            "transient_reduction": round(1 - ours_act / transient, 3),
            "how": "unfused: torch allocator peak during the forward minus the memory live "
                   "before it (transient: per layer, minus the live hidden state); ours: "
                   "cudaMemGetInfo delta of a workspace for these tokens minus one for 32 tokens, "
                   "plus the caller's K/V buffers (the forward allocates nothing)"},
        "unfused_ms_per_forward": round(ms_unfused, 3),
        "kernel_times_ms": {k: round(v["ms"], 4) for k, v in sorted(prof.items())},
    }
    if ffn:
        ffn_tf = ffn["flops"] / (ffn["ms"] / 1e3) / 1e12
        line["ffn_stream"] = {"launches": ffn["launches"], "ms": round(ffn["ms"], 4),
                              "tflops": round(ffn_tf, 1),
                              "frac_of_bf16_peak": round(ffn_tf / peaks["bf16_tflops"], 3)}
    print(json.dumps(line), flush=True)
    return 0


def run_prefill_attn(args):
    """Where forming the query inside the attention kernel pays: one
    Llama-2-7B-shaped decoder layer (hidden 4096, 32 heads of 128, SwiGLU
    11008 at rank 1792) over a 2048-token prompt, with the attention ranks
    (q, k, v, o) swept, prefilled with the dense q projection (mode 0) and
    with the query formed in the attention kernel (mode 1).  Times are CUDA
    events over 10 layer prefills; the attention and q/k/v second-stage
    kernels' shares come from the profiler (events around each launch)."""
    import torch
    sys.path.insert(0, ROOT)
    from rank_transformer_b200 import flashsvd as fs
    from rank_transformer_b200.model import _bf16_normal
    torch.cuda.set_device(0)
    d, H, D, f, r_f, S = 4096, 32, 128, 11008, 1792, 2048
    fs.init(0, max_tokens=S, max_rank=4096, max_hidden=d, max_ffn=f)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    stream = torch.cuda.Stream()
    cos_t = torch.empty((S, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S, D, 10000.0)
    x0 = _bf16_normal((S, d), 1.0, gen, "cuda")
    kc = torch.zeros((1, S, H, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    for r in ((1216,) if args.profile_step else (128, 256, 512, 832, 1216)):
        w = {}
        for n in ("q", "k", "v", "o"):
            w["U_" + n] = _bf16_normal((d, r), d ** -0.5, gen, "cuda")
            w["V_" + n] = _bf16_normal((r, d), r ** -0.5, gen, "cuda")
        w["U_gu"] = _bf16_normal((d, 2 * r_f), d ** -0.5, gen, "cuda")
        w["V_gu"] = _bf16_normal((2 * r_f, f), r_f ** -0.5, gen, "cuda")
        w["U_dn"] = _bf16_normal((f, r_f), f ** -0.5, gen, "cuda")
        w["V_dn"] = _bf16_normal((r_f, d), r_f ** -0.5, gen, "cuda")
        w["g1"] = torch.ones(d, dtype=torch.bfloat16, device="cuda")
        w["g2"] = torch.ones(d, dtype=torch.bfloat16, device="cuda")
        L = fs.Layer()
        L.kind, L.d, L.H, L.D, L.f, L.norm_eps = fs.DECODER, d, H, D, f, 1e-5
        L.norm1_g, L.norm2_g = w["g1"].data_ptr(), w["g2"].data_ptr()
        for n in ("q", "k", "v", "o"):
            F = getattr(L, n)
            F.U, F.V, F.bias, F.r = w["U_" + n].data_ptr(), w["V_" + n].data_ptr(), None, r
        L.U_gu, L.V_gu, L.r_f = w["U_gu"].data_ptr(), w["V_gu"].data_ptr(), r_f
        L.down.U, L.down.V, L.down.bias, L.down.r = w["U_dn"].data_ptr(), w["V_dn"].data_ptr(), None, r_f
        L.rope_cos, L.rope_sin = cos_t.data_ptr(), sin_t.data_ptr()
        out = {"workload": "prefill-attn", "layer": "7b-shaped decoder", "S": S, "rank_qkvo": r}
        if args.profile_step:
            fs.set_prefill_attention(1)
            x = x0.clone()
            with torch.cuda.stream(stream):
                fs.layer_forward(L, x, kc, vc, None, 1, S, S, fs.PREFILL_CAUSAL, stream)
                stream.synchronize()
                torch.cuda.nvtx.range_push("profile_step")
                fs.layer_forward(L, x, kc, vc, None, 1, S, S, fs.PREFILL_CAUSAL, stream)
                stream.synchronize()
                torch.cuda.nvtx.range_pop()
            fs.set_prefill_attention(0)
            print(json.dumps({"profile_step": "done", "workload": "prefill-attn", "rank_qkvo": r}))
            return 0
        for mode in (0, 1):
            fs.set_prefill_attention(mode)
            x = x0.clone()

            def one(i):
                fs.layer_forward(L, x, kc, vc, None, 1, S, S, fs.PREFILL_CAUSAL, stream)
            with torch.cuda.stream(stream):
                for i in range(3):
                    one(i)
                ms = _event_ms(one, 10, stream)
                fs.profile_enable(True)
                one(0)
                prof = fs.profile_report(reset=True)
                fs.profile_enable(False)
            fs.check_device_status(stream)
            key = "factorized_q" if mode else "dense_q"
            out[key] = {"layer_ms": round(ms, 4),
                        "attention_ms": round(sum(v["ms"] for k, v in prof.items()
                                                  if k.startswith("attn_prefill")), 4),
                        "qkv_stage2_ms": round(sum(prof.get(k, {}).get("ms", 0.0)
                                                   for k in ("tc_stage2_qkv_grouped", "tc_stage2_qkv_rope")), 4)}
        fs.set_prefill_attention(0)
        out["factorized_faster"] = out["factorized_q"]["layer_ms"] < out["dense_q"]["layer_ms"]
        print(json.dumps(out), flush=True)
        del w
    return 0


def _dense_decode_step(B, ctx, device, gen):
    """A dense Llama-2-7B-shaped decode step in plain PyTorch (the reference
    point of the retention curve): 32 pre-norm layers with dense bf16
    q/k/v/o [4096 x 4096], gate/up [4096 x 11008] and down [11008 x 4096]
    (cuBLAS), RoPE-free attention by scaled_dot_product_attention over a
    fixed 'ctx'-key bf16 cache, the 4096 x 32000 head and an argmax; the
    whole step captured as one CUDA graph.  Returns (graph, weight bytes,
    cache bytes read per step)."""
    import torch
    import torch.nn.functional as F
    d, H, D, f, V, nl = 4096, 32, 128, 11008, 32000, 32

    def w(*shape):
        return (torch.randn(*shape, device=device, generator=gen) * shape[0] ** -0.5).to(torch.bfloat16)
    layers = [dict(qkv=w(d, 3 * d), o=w(d, d), gu=w(d, 2 * f), dn=w(f, d)) for _ in range(nl)]
    kc = [torch.randn(B, H, ctx, D, device=device, generator=gen).to(torch.bfloat16) for _ in range(nl)]
    vc = [torch.randn(B, H, ctx, D, device=device, generator=gen).to(torch.bfloat16) for _ in range(nl)]
    W_lm = w(d, V)
    x = torch.randn(B, d, device=device, generator=gen).to(torch.bfloat16)
    tok = torch.zeros(B, dtype=torch.int64, device=device)

    def step():
        h = x
        for L, k_, v_ in zip(layers, kc, vc):
            n = F.rms_norm(h, (d,))
            q, _, _ = (n @ L["qkv"]).split(d, dim=1)
            a = F.scaled_dot_product_attention(q.view(B, H, 1, D), k_, v_).reshape(B, d)
            h = h + a @ L["o"]
            g, u = (F.rms_norm(h, (d,)) @ L["gu"]).split(f, dim=1)
            h = h + (F.silu(g) * u) @ L["dn"]
        tok.copy_(torch.argmax(F.rms_norm(h, (d,)) @ W_lm, dim=1))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(2):
            step()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    wbytes = 2 * (nl * (3 * d * d + d * d + 2 * d * f + f * d) + d * V)
    return g, wbytes, 2 * 2 * nl * B * ctx * d


def run_retention(args):
    """Decode speed against retention (FlashSVD v1.5 explainer, Results,
    Robustness: speedups shrink as the model approaches dense): the
    Llama-2-7B-shaped low-rank decoder at retention 0.2 / 0.4 / 0.6 / 0.8
    (ranks by parameter retention), B = 1, contexts 2048 and 8192 (caches of
    random history), 64 graph-replayed decode steps per point, beside a
    dense decode step of the same shapes in plain PyTorch (cuBLAS GEMVs,
    scaled_dot_product_attention, CUDA graph) at the same context.  Each
    point also gives its fraction of the HBM roofline (algorithmic bytes:
    factors or dense weights, head, K/V history)."""
    import dataclasses
    import torch
    sys.path.insert(0, ROOT)
    from rank_transformer_b200 import flashsvd as fs
    from rank_transformer_b200.model import LLAMA7B, DecoderModel
    torch.cuda.set_device(0)
    peaks = measured_peaks()
    fs.init(0, max_tokens=256, max_rank=4096, max_hidden=4096, max_ffn=11008)
    stream = torch.cuda.Stream()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(51)
    steps = 64
    for ctx in (2048, 8192):
        g, wb, kvb = _dense_decode_step(1, ctx, "cuda", gen)
        for _ in range(3):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            g.replay()
        e1.record()
        e1.synchronize()
        dense_ms = e0.elapsed_time(e1) / steps
        dense_gbs = (wb + kvb) / (dense_ms / 1e3) / 1e9
        del g
        torch.cuda.empty_cache()
        print(json.dumps({"workload": "retention", "model": "dense (torch, cuBLAS, CUDA graph)",
                          "context": ctx, "ms_per_step": round(dense_ms, 4),
                          "tok_s": round(1e3 / dense_ms, 1), "weight_bytes": wb,
                          "frac_of_hbm": round(dense_gbs / peaks["hbm_gbs"], 3)}), flush=True)
        for rho in (0.2, 0.4, 0.6, 0.8):
            cfg = dataclasses.replace(LLAMA7B, rho=(rho,))
            m = DecoderModel(cfg, 1, ctx + steps + 8, seed=61)
            with torch.cuda.stream(stream):
                for kc_, vc_ in zip(m.k_cache, m.v_cache):
                    kc_.normal_(generator=gen)
                    vc_.normal_(generator=gen)
            m.capture(stream)
            with torch.cuda.stream(stream):
                m.seqlens.fill_(ctx)
                for _ in range(3):
                    m.decode_step(stream)
                m.seqlens.fill_(ctx)
                ms = _event_ms(lambda i: m.decode_step(stream), steps, stream)
            fs.check_device_status(stream)
            byts = m.decode_step_bytes(ctx + steps // 2)
            r_a, r_f = cfg.ranks(0)
            print(json.dumps({
                "workload": "retention", "rho": rho, "ranks": [r_a, r_f], "context": ctx,
                "ms_per_step": round(ms, 4), "tok_s": round(1e3 / ms, 1),
                "speedup_vs_dense": round(dense_ms / ms, 3),
                "frac_of_hbm": round(byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 3),
                "decode_path": "decode plan" if m.plan is not None else "per-stage"}), flush=True)
            m.release_graphs()
            del m
            torch.cuda.empty_cache()
    return 0


def run_shared_basis(args):
    """Shared bases (FlashSVD v1.5 explainer, Methodology 1, Basis Sharing:
    one physical copy of a basis used by several layers): the
    Llama-2-7B-shaped low-rank decoder (retention 0.6) whose input-side
    factors U_q, U_k, U_v, U_o, U_gu, U_dn are shared by groups of 1 (no
    sharing), 4 and 32 consecutive layers.  The decode plan reads a shared
    factor from one pack with an L2 evict-last hint, so after the group's
    first layer it comes from L2.  B = 1, context 2048, 64 graph-replayed
    steps; algorithmic bytes count a shared factor once per step."""
    import dataclasses
    import torch
    sys.path.insert(0, ROOT)
    from rank_transformer_b200 import flashsvd as fs
    from rank_transformer_b200.model import LLAMA7B, DecoderModel, _bf16_normal
    torch.cuda.set_device(0)
    peaks = measured_peaks()
    cfg = LLAMA7B
    fs.init(0, max_tokens=256, max_rank=2368, max_hidden=cfg.d, max_ffn=cfg.f)
    stream = torch.cuda.Stream()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(71)
    ctx, steps = 2048, 64
    d, f = cfg.d, cfg.f
    r_a, r_f = cfg.ranks(0)
    shapes = {"U_q": (d, r_a), "U_k": (d, r_a), "U_v": (d, r_a), "U_o": (d, r_a),
              "U_gu": (d, 2 * r_f), "U_dn": (f, r_f)}
    for group in (1, 4, 32):
        layers, base = [], None
        for i in range(cfg.layers):
            w = {}
            if i % group == 0:
                base = {k: _bf16_normal(sh, sh[0] ** -0.5, gen, "cuda") for k, sh in shapes.items()}
            w.update(base)
            for n in ("q", "k", "v", "o"):
                w["V_" + n] = _bf16_normal((r_a, d), r_a ** -0.5, gen, "cuda")
            w["V_gu"] = _bf16_normal((2 * r_f, f), r_f ** -0.5, gen, "cuda")
            w["V_dn"] = _bf16_normal((r_f, d), r_f ** -0.5, gen, "cuda")
            w["g1"] = torch.ones(d, dtype=torch.bfloat16, device="cuda")
            w["g2"] = torch.ones(d, dtype=torch.bfloat16, device="cuda")
            layers.append(w)
        m = DecoderModel(cfg, 1, ctx + steps + 8, seed=72, weights=layers)
        with torch.cuda.stream(stream):
            for kc_, vc_ in zip(m.k_cache, m.v_cache):
                kc_.normal_(generator=gen)
                vc_.normal_(generator=gen)
        m.capture(stream)
        with torch.cuda.stream(stream):
            m.seqlens.fill_(ctx)
            for _ in range(3):
                m.decode_step(stream)
            m.seqlens.fill_(ctx)
            ms = _event_ms(lambda i: m.decode_step(stream), steps, stream)
        fs.check_device_status(stream)
        byts = m.decode_step_bytes(ctx + steps // 2)
        print(json.dumps({
            "workload": "shared-basis", "layers_per_shared_basis": group, "context": ctx,
            "ms_per_step": round(ms, 4), "tok_s": round(1e3 / ms, 1),
            "algorithmic_bytes_per_step": int(byts),
            "frac_of_hbm": round(byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 3),
            "decode_path": "decode plan" if m.plan is not None else "per-stage"}), flush=True)
        m.release_graphs()
        del m, layers, base
        torch.cuda.empty_cache()
    return 0


def run_mixed(args):
    """Same 7B-shaped model with one retention ratio per layer drawn from
    {0.4, 0.6, 0.8}: prefill B=4 x 2048 (tcgen05 path), then 256 greedy
    decode steps (B=4, decode plan)."""
    import dataclasses
    import torch
    sys.path.insert(0, ROOT)
    from rank_transformer_b200 import flashsvd as fs
    from rank_transformer_b200 import synth
    from rank_transformer_b200.model import LLAMA7B, DecoderModel
    torch.cuda.set_device(0)
    B, S, steps = 4, PROMPT, 256
    cfg = dataclasses.replace(LLAMA7B, rho=synth.mixed_rho(11, LLAMA7B.layers))
    fs.init(0, max_tokens=B * S, max_rank=2368, max_hidden=cfg.d, max_ffn=cfg.f)
    peaks = measured_peaks()
    model = DecoderModel(cfg, B, S + steps, seed=21)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(22)
    prompt = torch.randint(0, cfg.vocab, (B, S), generator=gen, device="cuda", dtype=torch.int32)
    stream = torch.cuda.Stream()
    model.capture(stream)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    with torch.cuda.stream(stream):
        for rep_ in range(2):
            ev[0].record(stream)
            model.prefill(prompt, stream)
            ev[1].record(stream)
            for _ in range(steps):
                model.decode_step(stream)
            ev[2].record(stream)
    stream.synchronize()
    fs.check_device_status(stream)
    pre_ms, dec_ms = ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2])
    lin = 2 * B * S * sum(cfg.layer_params(i) for i in range(cfg.layers))
    head = 2 * B * cfg.d * cfg.vocab
    attn = cfg.layers * 4 * B * S * S * cfg.d / 2
    pf_flops = lin + head + attn
    model.release_graphs()
    print(json.dumps({
        "workload": "mixed-rank", "rho_per_layer": list(cfg.rho),
        "ranks_per_layer": [list(cfg.ranks(i)) for i in range(cfg.layers)],
        "batch": B, "prompt": S, "decode_steps": steps,
        "prefill_tok_s": round(B * S / (pre_ms / 1e3)), "prefill_ms": round(pre_ms, 2),
        "prefill_tflops": round(pf_flops / (pre_ms / 1e3) / 1e12, 1),
        "prefill_frac_of_bf16_peak": round(pf_flops / (pre_ms / 1e3) / 1e12 / peaks["bf16_tflops"], 3),
        "decode_tok_s": round(B * steps / (dec_ms / 1e3), 1), "decode_ms": round(dec_ms, 2),
        "e2e_latency_ms": round(pre_ms + dec_ms, 2),
        "decode_path": "decode plan" if model.plan is not None else "per-stage"}), flush=True)
    return 0


def run_long_decode(args):
    """Decode over long histories: the 7B-shaped model with every layer's
    cache filled with a random history (N(0, 1) bf16) and the lengths set
    directly, at contexts 2048 / 4096 / 8192 / 16320 for B = 1 and B = 4,
    plus one B = 4 batch of very different lengths; each point times 64
    graph-replayed steps (embedding, one decode-plan launch of all 32
    layers, head) after 3 warm-up steps.  Algorithmic bytes per step: every
    factor, norm gain and the head once, each row's K/V history of every
    layer once, the new K/V rows and the activations.  The caches
    (8.6 GB per row at 16384 positions) exceed L2."""
    import torch
    sys.path.insert(0, ROOT)
    from rank_transformer_b200 import flashsvd as fs
    from rank_transformer_b200.model import LLAMA7B, DecoderModel
    torch.cuda.set_device(0)
    cfg, S_max, steps, warm = LLAMA7B, 16384, 64, 3
    contexts = (2048, 4096, 8192, S_max - steps)
    fs.init(0, max_tokens=256, max_rank=2368, max_hidden=cfg.d, max_ffn=cfg.f)
    peaks = measured_peaks()
    stream = torch.cuda.Stream()
    gen = torch.Generator(device="cuda")
    gen.manual_seed(31)
    for B in (1, 4):
        model = DecoderModel(cfg, B, S_max, seed=41 + B)
        with torch.cuda.stream(stream):
            for kc, vc in zip(model.k_cache, model.v_cache):
                kc.normal_(generator=gen)
                vc.normal_(generator=gen)
            model.tokens.copy_(torch.randint(0, cfg.vocab, (B,), generator=gen, device="cuda",
                                             dtype=torch.int32))
        model.capture(stream)
        points = [[c] * B for c in contexts]
        if B == 4:
            points.append([S_max - steps, 4096, 1024, 64])
        for lens in points:
            start = torch.tensor(lens, dtype=torch.int32, device="cuda")
            with torch.cuda.stream(stream):
                model.seqlens.copy_(start)
                for _ in range(warm):
                    model.decode_step(stream)
                model.seqlens.copy_(start)
                ms = _event_ms(lambda i: model.decode_step(stream), steps, stream)
            fs.check_device_status(stream)
            # mean history per step: the lengths grow by one each step
            hist = sum(c + (steps - 1) / 2 + 1 for c in lens)
            kv = 2 * cfg.layers * hist * cfg.d * 2
            act = B * cfg.d * 2 * 2 * cfg.layers
            byts = model.weight_bytes() + kv + act
            gbs = byts / (ms / 1e3) / 1e9
            print(json.dumps({
                "workload": "long-decode", "batch": B, "context": lens,
                "decode_steps": steps, "tok_s": round(B / (ms / 1e3), 1),
                "ms_per_step": round(ms, 3), "bytes_per_step": int(byts),
                "achieved_gbs": round(gbs, 1), "peak_gbs": peaks["hbm_gbs"],
                "frac": round(gbs / peaks["hbm_gbs"], 3),
                "decode_path": "decode plan" if model.plan is not None else "per-stage",
                "data": "synthetic (random weights and histories)"}), flush=True)
        model.release_graphs()
        del model
        torch.cuda.empty_cache()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "linear-sweep":
        return run_linear_sweep(args)
    if args.workload == "bert":
        return run_bert(args)
    if args.workload == "mixed-rank":
        return run_mixed(args)
    if args.workload == "long-decode":
        return run_long_decode(args)
    if args.workload == "prefill-attn":
        return run_prefill_attn(args)
    if args.workload == "retention":
        return run_retention(args)
    if args.workload == "shared-basis":
        return run_shared_basis(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
