#!/usr/bin/env python
"""Throughput of the GPT-2 training step on B200 (tokens/s and MFU).

Workload: GPT-2 124M (12 layers, 12 heads, width 768, vocabulary padded to
50304, block 1024), one full bf16 training step at B=16, T=1024: forward,
cross-entropy (ignore_index=-1), backward, global-norm clip at 1.0 and AdamW
(0.9, 0.95, wd 0.1 on 2-D tensors), fp32 master weights and moments. Tokens
are synthetic: Zipf(1.1) over the 50257 real GPT-2 ids, targets the same rows
shifted by one (the pages' FineWeb-Edu / Shakespeare corpora are not
available). Weights: the pages' random init (std 0.02, residual projections
0.02/sqrt(24)).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs one process per GPU (torchrun) as data parallelism: each rank runs the
forward and backward of its own B=16 sequences, the ranks sum their gradients
with a bucketed NCCL all-reduce that overlaps the backward, and every rank applies
the same update (decoder_only_transformer_sm_b200.ddp; weak scaling: the global
batch is 16 N sequences). The step time is the max over ranks. `--impl reference`
times the CPU oracle (float64 numpy) on a bounded sample of the same workload, on
rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

MODELS = {
    "124m": dict(name="GPT-2 124M", n_layer=12, n_head=12, n_embd=768, vocab_size=50304, vocab_real=50257,
                 block_size=1024, B=16, T=1024),
    "medium": dict(name="GPT-2 medium", n_layer=24, n_head=16, n_embd=1024, vocab_size=50304, vocab_real=50257,
                   block_size=1024, B=8, T=1024),
    "large": dict(name="GPT-2 large", n_layer=36, n_head=20, n_embd=1280, vocab_size=50304, vocab_real=50257,
                  block_size=1024, B=8, T=1024),
    "xl": dict(name="GPT-2 XL", n_layer=48, n_head=25, n_embd=1600, vocab_size=50304, vocab_real=50257,
               block_size=1024, B=4, T=1024),
}
WORKLOAD = MODELS["124m"]   # the benchmark workload
METRIC = "training tokens/sec and MFU at GPT-2 124M (B=16,T=1024, bf16), 1×B200"


def metric_for(w, B: int, T: int) -> str:
    if w is WORKLOAD and B == w["B"] and T == w["T"]:
        return METRIC
    return f"training tokens/sec and MFU at {w['name']} (B={B},T={T}, bf16)"
LR = 6e-4
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def n_params_padded(w) -> int:
    C, L, V, Tm = w["n_embd"], w["n_layer"], w["vocab_size"], w["block_size"]
    per_block = 2 * C + (3 * C * C + 3 * C) + (C * C + C) + 2 * C + (4 * C * C + 4 * C) + (4 * C * C + C)
    return V * C + Tm * C + L * per_block + 2 * C


def flops_per_token(w) -> float:
    """6N + 12 L C T (N with the tied wte counted once, padded vocabulary)."""
    return 6.0 * n_params_padded(w) + 12.0 * w["n_layer"] * w["n_embd"] * w["T"]


def exact_step_flops(w, B: int, T: int) -> float:
    """FLOPs one training step performs, with attention counted over the causal
    triangle only: every Linear layer's forward, input-gradient and weight-gradient
    GEMMs (3 x 2 M N K), attention forward 2 B H T (T+1) hd (QK^T and PV) and
    backward 5 B H T (T+1) hd (S recomputed, dV, dP, dQ, dK) per layer."""
    C, L, V, H = w["n_embd"], w["n_layer"], w["vocab_size"], w["n_head"]
    BT, hd = B * T, C // H
    gemm_fwd = L * 2.0 * BT * (3 * C * C + C * C + 4 * C * C + 4 * C * C) + 2.0 * BT * C * V
    attn = L * 7.0 * B * H * T * (T + 1) * hd
    return 3.0 * gemm_fwd + attn


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK), "fallback"


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                     hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        pmax = max(r["power"] for r in rows)
        loaded = [r for r in rows if r["power"] >= 0.5 * pmax] or rows
        reasons = []
        for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                          ("pcap", "sw_power_cap")):
            if any(r[key].lower().startswith("active") for r in loaded):
                reasons.append(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": reasons, "samples": len(loaded), "power_w_max": pmax}


# ----------------------------------------------------------------------------
# reference arm: the CPU oracle, as it stands
# ----------------------------------------------------------------------------
def oracle_step_time(T_sample: int, warm: int, steps: int):
    import numpy as np
    from threadpoolctl import threadpool_info
    from oracle import gpt2_oracle as O
    from decoder_only_transformer_sm_b200 import synthetic as S
    w = WORKLOAD
    s = O.Shape(w["n_layer"], w["n_head"], w["n_embd"], w["vocab_size"], w["block_size"])
    P = O.unflatten(s, S.init_params(S.GPT2_124M, seed=0))
    M, V = O.zeros_like(s), O.zeros_like(s)
    idx, tgt = S.zipf_tokens(1, T_sample, w["vocab_real"], seed=1001)
    for i in range(warm):
        wi, wt = S.zipf_tokens(1, 16, w["vocab_real"], seed=7 + i)
        O.forward(s, P, wi, wt)
    times = []
    t = 0
    for _ in range(steps):
        t += 1
        t0 = time.perf_counter()
        O.train_step(s, P, M, V, t, idx, tgt, lr=LR)
        times.append(time.perf_counter() - t0)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    del np
    return times, threads


def workload_config(B: int, T: int, world: int, w=None) -> dict:
    w = w or WORKLOAD
    return {"workload": f"{w['name']} train step (fwd+CE+bwd+clip+AdamW), B={B} T={T} V={w['vocab_size']} bf16",
            "B": B, "T": T, "tokens_per_step_per_gpu": B * T,
            "parallelism": f"dp{world}: bucketed gradient all-reduce overlapped with the backward" if world > 1
                           else "single-gpu",
            "l2": "working set (6+ GB of activations per step) larger than the 126 MB L2; no flush"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    T_sample = 512
    times, threads = oracle_step_time(T_sample, args.warmup, args.steps)
    sec = sum(times) / len(times)
    value = T_sample / sec
    sample = (f"each timed step is a bounded sample of the workload: one float64 oracle step (forward, loss, "
              f"backward, clip, AdamW on all 124.5M parameters) on B=1 x T={T_sample} Zipf tokens; warm-up "
              f"steps are forward passes on 16 tokens; value = sampled tokens / oracle seconds")
    line = {
        "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * sec, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic Zipf(1.1) tokens", "impl": "reference",
        "config": workload_config(16, 1024, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample,
                         "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
def kernel_source_sha(name: str) -> str:
    p = os.path.join(ROOT, "decoder_only_transformer_sm_b200", "csrc", name)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16] if os.path.exists(p) else ""


SITE_SOURCES = [("decode attention", "k_decode.cu"), ("sample", "k_decode.cu"), ("gemm", "k_gemm_tc.cu"), ("attention", "k_attention_tc.cu"), ("layernorm", "k_rowwise.cu"),
                ("classifier", "k_rowwise.cu"), ("adamw", "k_optim.cu"), ("grad norm", "k_optim.cu"),
                ("embed", "k_rowwise.cu"), ("bias colsum", "k_rowwise.cu")]


def source_of(site: str) -> str:
    for prefix, f in SITE_SOURCES:
        if prefix in site:
            return f
    return ""


def traffic_for(site: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(site)
    if not e or e.get("kernel_source_sha") != kernel_source_sha(source_of(site)):
        return None
    return e.get("bytes_per_launch")


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The largest of every rank's x (the job's time is that of its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_tokens(rank: int, B: int, T: int, vocab_real: int, nb: int = 2):
    """The nb synthetic batches of one replica: each rank draws its own seeded Zipf stream."""
    from decoder_only_transformer_sm_b200 import synthetic as S
    return [S.zipf_tokens(B, T, vocab_real, seed=1001 + 97 * rank + i) for i in range(nb)]


def step_stats(times_ms, world: int) -> dict:
    """Median, p10, p90 and mean of the per-step device times (each step bracketed
    by its own CUDA events on the launching stream); for N > 1 each statistic is
    the max over ranks."""
    xs = sorted(times_ms)

    def q(f):
        i = f * (len(xs) - 1)
        lo, hi = int(math.floor(i)), int(math.ceil(i))
        return xs[lo] + (xs[hi] - xs[lo]) * (i - lo)

    out = {"median": q(0.5), "p10": q(0.1), "p90": q(0.9), "mean": sum(xs) / len(xs)}
    return {k: max_over_ranks(v, world) for k, v in out.items()}


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def job_throughput(ms_per_step_max: float, B: int, T: int, world: int) -> float:
    """Whole-job tokens/s: every replica's tokens over the slowest rank's step time."""
    return B * T * world / (ms_per_step_max / 1000.0)


def run_eval(args):
    """Forward-only throughput on the benchmark's shapes: held-out loss (forward +
    cross-entropy, no gradients) and the last-position forward that feeds
    next-token sampling. Device-resident inputs, CUDA events, one GPU."""
    import torch

    from decoder_only_transformer_sm_b200 import native

    w = WORKLOAD
    B, T = args.batch or w["B"], w["T"]
    stream = torch.cuda.current_stream()
    m = native.GPT2(w["n_layer"], w["n_head"], w["n_embd"], w["vocab_size"], w["block_size"], B, T,
                    precision="bf16", seed=1234, stream=stream.cuda_stream)
    idx, tgt = (torch.from_numpy(a).cuda() for a in replica_tokens(0, B, T, w["vocab_real"], 1)[0])
    last = torch.empty((B, w["vocab_size"]), dtype=torch.bfloat16, device="cuda")

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    losses = []
    ms_loss = timed(lambda: losses.append(m.forward(idx, tgt)))
    ms_last = timed(lambda: m.forward_last(idx, last))
    m.close()
    line = {
        "metric": "eval tokens/sec (GPT-2 124M, B=16, T=1024, bf16 forward + loss)",
        "value": B * T / (ms_loss / 1000.0), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_loss, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic Zipf(1.1) tokens, random-init weights",
        "workload": "eval",
        "config": dict(workload_config(B, T, 1),
                       workload="gpt2-124m eval: forward + CE loss, no gradients; B=16 T=1024 V=50304 bf16"),
        "forward_last": {"ms_per_call": ms_last, "tokens_per_s": B * T / (ms_last / 1000.0),
                         "note": "blocks + ln_f on all B*T positions, lm_head on the B last rows"},
        "loss": losses[-1],
    }
    print(json.dumps(line), flush=True)


def run_generate(args):
    """Generation throughput ("GPT-2 from Scratch", "A generation loop"): the
    pages' sampling call (a short prompt, 40 new tokens, temperature 0.8,
    top-k 40) through gpt2_generate on GPT-2 124M bf16: one prefill that fills
    the key/value cache, then per token one decode step and one draw.
    Device-resident prompt and uniforms; CUDA events around whole calls (each
    call ends with one synchronisation). The bf16 weights (250 MB) exceed the
    L2, so every decode step streams them from HBM."""
    import torch

    from decoder_only_transformer_sm_b200 import native
    from decoder_only_transformer_sm_b200 import synthetic as S

    w = WORKLOAD
    B, T0, n_new, temperature, top_k = args.batch or 1, 4, 40, 0.8, 40
    stream = torch.cuda.current_stream()
    m = native.GPT2(w["n_layer"], w["n_head"], w["n_embd"], w["vocab_size"], w["block_size"], B, w["T"],
                    precision="bf16", seed=1234, stream=stream.cuda_stream)
    prompt = torch.from_numpy(S.zipf_tokens(B, T0, w["vocab_real"], seed=1001)[0]).cuda()
    u = torch.from_numpy(S.uniforms(n_new, B, seed=1002)).cuda()
    out = torch.empty((B, T0 + n_new), dtype=torch.int32, device="cuda")

    def call():
        m.generate(prompt, n_new, temperature, top_k, u, out)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            call()
            launches += m.last_launch_count()
        e1.record(stream)
        torch.cuda.synchronize()
    clocks = clk.summary()
    ms = e0.elapsed_time(e1) / args.steps
    m.profile(True)
    call()
    stats = m.profile_read()
    m.profile(False)
    m.close()

    peaks, peak_src = load_peaks()
    total_ms = sum(s["total_ms"] for s in stats)
    sites = sorted(stats, key=lambda s: -s["total_ms"])
    dom = sites[0]
    per_launch_ms = dom["total_ms"] / dom["launches"]
    achieved = dom["bytes"] / dom["launches"] / (per_launch_ms / 1e3) / 1e9
    peak = peaks.get("hbm_gbs")
    breakdown = [{"site": s["name"], "ms_per_call": round(s["total_ms"], 4), "share": round(s["total_ms"] / total_ms, 4),
                  "launches_per_call": s["launches"],
                  "gbs": round(s["bytes"] / (s["total_ms"] / 1e3) / 1e9, 1) if s["bytes"] > 0 else None}
                 for s in sites]
    line = {
        "metric": "generated tokens/sec (GPT-2 124M bf16; prompt 4, 40 new tokens, temperature 0.8, top-k 40)",
        "value": B * n_new / (ms / 1000.0), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic Zipf(1.1) prompt, seeded uniforms for the draws, random-init weights",
        "workload": "generate",
        "config": {"workload": f"gpt2-124m generation: gpt2_generate, B={B}, prompt {T0}, {n_new} new tokens, "
                               f"temperature {temperature}, top-k {top_k}; key/value cache; bf16 weights "
                               "(250 MB) larger than L2", "global_batch": B, "seq_len": T0 + n_new,
                   "parallelism": "single GPU"},
        "roofline": {"kernel": dom["name"], "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak if peak else None, "traffic": None, "per_launch_ms": per_launch_ms,
                     "peak_note": f"hbm_gbs of {peak_src}"},
        "kernels": breakdown,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def run_accum(args):
    """Gradient accumulation on the benchmark's micro-batch: zero_grad, 32 x
    accumulate (loss scale 1/32; the second half of the micro-batches with
    SFT-style masked target prefixes), one clip + AdamW update. A step here is one
    update (32 x B x T tokens). Device-resident inputs, CUDA events, one GPU."""
    import torch

    from decoder_only_transformer_sm_b200 import native, synthetic as S

    w = WORKLOAD
    B, T, n_micro = args.batch or w["B"], w["T"], 32
    stream = torch.cuda.current_stream()
    m = native.GPT2(w["n_layer"], w["n_head"], w["n_embd"], w["vocab_size"], w["block_size"], B, T,
                    precision="bf16", seed=1234, stream=stream.cuda_stream)
    dev = [(torch.from_numpy(i).cuda(), torch.from_numpy(t).cuda())
           for i, t in S.accumulation_batches(n_micro, B, T, w["vocab_real"], seed=1002)]
    out = []

    def update():
        m.zero_grad()
        for i, t in dev:
            m.accumulate(i, t, 1.0 / n_micro)
        out.append(m.update(LR))

    for _ in range(args.warmup):
        update()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            update()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    m.close()
    fpt = flops_per_token(w)
    tokens = n_micro * B * T
    line = {
        "metric": f"training tokens/sec and MFU at GPT-2 124M ({n_micro} x B={B},T={T} accumulation, bf16)",
        "value": tokens / (ms / 1000.0), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic Zipf(1.1) tokens, random-init weights",
        "workload": "accum",
        "config": dict(workload_config(B, T, 1), tokens_per_step_per_gpu=tokens,
                       workload=f"GPT-2 124M: zero_grad + {n_micro} x accumulate(1/{n_micro}) + update; "
                                f"micro-batches {n_micro // 2}-{n_micro - 1} with masked target prefixes"),
        "mfu": {"flops_per_token": fpt, "vs_nominal_2250": tokens / (ms / 1000.0) * fpt / (NOMINAL_BF16_TFLOPS * 1e12)},
        "clocks": clk.summary(),
        "loss_norm_last": list(out[-1]),
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# --workload kernel: one kernel of the step in isolation, through the kernel-level
# C ABI (gpt2_kernels.h), timed with CUDA events; the target of ncu captures
# ----------------------------------------------------------------------------
def _events(torch, fn, reps: int):
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    return times


def kernel_gemm(args):
    import torch
    from decoder_only_transformer_sm_b200 import native
    M, N, K = args.M, args.N, args.K
    g = torch.Generator().manual_seed(0)
    if args.layout == "NT":
        A, B = torch.randn((M, K), generator=g), torch.randn((N, K), generator=g)
    elif args.layout == "NN":
        A, B = torch.randn((M, K), generator=g), torch.randn((K, N), generator=g)
    else:
        A, B = torch.randn((K, M), generator=g), torch.randn((K, N), generator=g)
    A, B = A.to(torch.bfloat16).cuda(), B.to(torch.bfloat16).cuda()
    ep = args.epilogue
    f32_out = ep in ("bias_resid", "accum_f32")
    out = torch.zeros((M, N), dtype=torch.float32 if f32_out else torch.bfloat16, device="cuda")
    out2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda") if ep == "bias_gelu" else None
    bias = torch.randn(N, device="cuda") if ep.startswith("bias") else None
    resid = torch.randn((M, N), device="cuda") if ep == "bias_resid" else None
    aux = torch.randn((M, N), device="cuda").to(torch.bfloat16) if ep == "mul" else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn = lambda: native.matmul_bf16(args.layout, A, B, M, N, K, ep, out, out2=out2, bias=bias,  # noqa: E731
                                    resid=resid, aux=aux, beta=1.0, engine="tc" if args.engine else "simt",
                                    status=st)
    fn()
    torch.cuda.synchronize()
    t = _events(torch, fn, args.reps)
    best = min(t)
    print(json.dumps({"case": "gemm", "layout": args.layout, "M": M, "N": N, "K": K, "epilogue": ep,
                      "ms": t, "tflops_best": 2.0 * M * N * K / best / 1e9, "status": int(st.item())}))


def kernel_attention(args):
    import torch
    from decoder_only_transformer_sm_b200 import native
    B, T, H, hd = args.B, args.T, args.H, args.hd
    C = H * hd
    g = torch.Generator().manual_seed(0)
    qkv = torch.randn((B, T, 3 * C), generator=g).to(torch.bfloat16).cuda()
    dout = torch.randn((B, T, C), generator=g).to(torch.bfloat16).cuda()
    out = torch.empty((B, T, C), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    dqkv = torch.empty_like(qkv)
    ws = torch.empty(native.attention_bwd_workspace(B, T, H, hd, args.engine), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fwd = lambda: native.attention_fwd(qkv, out, lse, B, T, H, hd, engine=args.engine, status=st)  # noqa: E731
    bwd = lambda: native.attention_bwd(qkv, out, dout, lse, dqkv, B, T, H, hd, ws,  # noqa: E731
                                       engine=args.engine, status=st)
    fwd()
    bwd()
    torch.cuda.synchronize()
    tf = _events(torch, fwd, args.reps)
    tb = _events(torch, bwd, args.reps)
    flops = 2.0 * B * H * T * (T + 1) * hd
    print(json.dumps({"case": "attention", "B": B, "T": T, "H": H, "hd": hd, "fwd_ms": tf, "bwd_ms": tb,
                      "fwd_tflops_best": flops / min(tf) / 1e9, "bwd_tflops_best": 2.5 * flops / min(tb) / 1e9,
                      "status": int(st.item())}))


def run_kernel(args):
    {"gemm": kernel_gemm, "attention": kernel_attention}[args.kernel](args)


def run_ours(args):
    import torch
    import torch.distributed as dist

    from decoder_only_transformer_sm_b200 import native

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    w = MODELS[args.model]
    B, T = args.batch or w["B"], w["T"]
    stream = torch.cuda.current_stream()
    m = native.GPT2(w["n_layer"], w["n_head"], w["n_embd"], w["vocab_size"], w["block_size"], B, T,
                    precision="bf16", seed=1234 + rank, stream=stream.cuda_stream)
    nb = 2
    host = replica_tokens(rank, B, T, w["vocab_real"], nb)
    pin = [(torch.from_numpy(i).pin_memory(), torch.from_numpy(t).pin_memory()) for i, t in host]
    dev = [(i.cuda(), t.cuda()) for i, t in pin]
    torch.cuda.synchronize()
    # N > 1: data parallelism (one bucketed gradient all-reduce per step); N = 1: the
    # library's own step (its forward and backward replayed as one CUDA graph)
    dp = None
    if world > 1:
        from decoder_only_transformer_sm_b200.ddp import DataParallel
        dp = DataParallel(m)
        dp.broadcast_params()

    def step_dev(k):
        if dp is None:
            out = m.step(*dev[k % nb], LR)
            return out, m.last_launch_count()
        out = dp.step([dev[k % nb]], LR)
        return out, dp.last_launches

    def step_host(k):
        if dp is None:
            return m.step_host(pin[k % nb][0], pin[k % nb][1], LR)
        i, t = pin[k % nb]
        return dp.step([(i.cuda(non_blocking=True), t.cuda(non_blocking=True))], LR)

    def barrier():
        if world > 1:
            dist.barrier()

    for k in range(args.warmup):
        step_dev(k)
    torch.cuda.synchronize()

    # ---- timed region: device-resident inputs ----
    losses = []
    barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    launches = 0
    with ClockSampler(local) as clk:
        ev[0].record(stream)
        for k in range(args.steps):
            (loss, norm), n_launch = step_dev(k)
            launches += n_launch
            losses.append(loss)
            ev[k + 1].record(stream)
        torch.cuda.synchronize()
    barrier()
    clocks = clk.summary()
    ms = max_over_ranks(ev[0].elapsed_time(ev[-1]) / args.steps, world)
    per_step = step_stats([ev[k].elapsed_time(ev[k + 1]) for k in range(args.steps)], world)

    # ---- end to end: host (pinned) token buffers through gpt2_step_host ----
    barrier()
    torch.cuda.synchronize()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for k in range(args.steps):
        step_host(k)
    e3.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = max_over_ranks(e2.elapsed_time(e3) / args.steps, world)

    # ---- per-launch-site device times (CUDA events on the launching stream) ----
    m.profile(True)
    for k in range(args.steps):
        m.step(*dev[k % nb], LR)
    stats = m.profile_read()
    m.profile(False)
    m.close()

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    value = job_throughput(ms, B, T, world)
    fpt = flops_per_token(w)
    total_ms = sum(s["total_ms"] for s in stats) / args.steps
    sites = sorted(stats, key=lambda s: -s["total_ms"])
    dom = sites[0]
    per_launch_ms = dom["total_ms"] / dom["launches"]
    if dom["name"].startswith("gemm") or dom["name"].startswith("attention"):
        bound, unit = "tensor", "TFLOP/s"
        achieved = dom["flops"] / dom["launches"] / (per_launch_ms / 1e3) / 1e12
        peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
        peak_note = f"bf16_tflops_sustained of {peak_src} (kernel timed inside a long step)"
    else:
        bound, unit = "hbm", "GB/s"
        achieved = dom["bytes"] / dom["launches"] / (per_launch_ms / 1e3) / 1e9
        peak = peaks.get("hbm_gbs")
        peak_note = f"hbm_gbs of {peak_src}"
    breakdown = []
    for s in sites:
        t = s["total_ms"] / args.steps
        row = {"site": s["name"], "ms_per_step": round(t, 4), "share": round(t / total_ms, 4),
               "launches_per_step": s["launches"] // args.steps}
        if s["flops"] > 0:
            row["tflops"] = round(s["flops"] / (s["total_ms"] / 1e3) / 1e12, 1)
        if s["bytes"] > 0:
            row["gbs"] = round(s["bytes"] / (s["total_ms"] / 1e3) / 1e9, 1)
        breakdown.append(row)
    cpu = None
    if world == 1 and not args.no_cpu_baseline and w is WORKLOAD:
        times, threads = oracle_step_time(1024, 0, 1)
        cpu = {"value": 1024 / times[0], "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "cpu_model": cpu_model(),
               "sample": "one float64 oracle step (forward, loss, backward, clip, AdamW on all 124.5M "
                         "parameters) on B=1 x T=1024 Zipf tokens, timed on this host"}
    line = {
        "metric": metric_for(w, B, T),
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic Zipf(1.1) tokens, random-init weights",
        "config": workload_config(B, T, world, w),
        "mfu": {"flops_per_token": fpt, "vs_nominal_2250": value * fpt / world / (NOMINAL_BF16_TFLOPS * 1e12),
                "vs_measured_sustained": value * fpt / world / (peaks.get("bf16_tflops_sustained", 1400.0) * 1e12),
                "peak_source": peak_src,
                "exact_causal_flops_per_step": exact_step_flops(w, B, T),
                "exact_causal_tflops_per_gpu": exact_step_flops(w, B, T) / (ms / 1e3) / 1e12},
        "roofline": {"kernel": dom["name"], "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak if peak else None, "traffic": traffic_for(dom["name"]),
                     "per_launch_ms": per_launch_ms, "peak_note": peak_note},
        "kernels": breakdown,
        "cpu_baseline": cpu,
        "e2e": {"value": job_throughput(ms_e2e, B, T, world), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * B * T * 4, "d2h_bytes_per_step": 40},
        "gpu_launches": launches,
        "clocks": clocks,
        "step_ms": per_step,
        "loss_first_last": [losses[0], losses[-1]],
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["train", "eval", "accum", "generate", "kernel"], default="train",
                    help="train: the training step (the benchmark line); eval: forward + loss and the "
                         "last-position forward of generation; accum: one update over 32 accumulated "
                         "micro-batches (524,288 tokens); generate: the pages' sampling call with a "
                         "key/value cache (--batch sets B, default 1); kernel: one GEMM or attention "
                         "call in isolation (--kernel and the shape options below; prints its CUDA-event "
                         "times); eval, accum, generate and kernel on one GPU")
    kg = ap.add_argument_group("--workload kernel")
    kg.add_argument("--kernel", choices=["gemm", "attention"], default="gemm")
    kg.add_argument("--layout", default="NT", choices=["NT", "NN", "TN"])
    kg.add_argument("--M", type=int, default=16384)
    kg.add_argument("--N", type=int, default=3072)
    kg.add_argument("--K", type=int, default=768)
    kg.add_argument("--epilogue", default="store")
    kg.add_argument("--engine", type=int, default=1,
                    help="gemm: 1 tcgen05, 0 SIMT; attention: 2 tcgen05, 1 mma.sync, 0 SIMT")
    kg.add_argument("--B", type=int, default=16)
    kg.add_argument("--T", type=int, default=1024)
    kg.add_argument("--H", type=int, default=12)
    kg.add_argument("--hd", type=int, default=64)
    kg.add_argument("--reps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--model", choices=sorted(MODELS), default="124m",
                    help="124m is the benchmark workload; the others are the same step at GPT-2 medium, "
                         "large and XL sizes (B = 8, 8, 4)")
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per step (default: the model's B, 16 for the 124m benchmark workload); "
                         "other values are for small-footprint profiler captures and do not produce the "
                         "benchmark number")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "eval":
        run_eval(args)
    elif args.workload == "accum":
        run_accum(args)
    elif args.workload == "generate":
        run_generate(args)
    elif args.workload == "kernel":
        run_kernel(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
