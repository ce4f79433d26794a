#!/usr/bin/env python
"""Benchmark of the KV-cache Transformer engine on B200.

Metric: d20 bf16 prefill tok/s and decode tok/s (B=32), with the fraction of
the tensor-core / HBM roofline.

  python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

One timed step = one nc_prefill of the d20 prefill workload (8 prompts x 2048
Zipf tokens, N(0,0.02) bf16 weights): embedding + norm, 20 blocks (QKV, RoPE +
QK norm + KV append, causal MQA, O-proj, relu^2 MLP), final norm, lm_head with
softcap and the argmax token pick, all on the device. The decode workload (32
sequences prefilled to 2048 tokens, then 128 greedy decode steps at
positions 2048..2175) is timed as a whole loop and reported under "decode".
Inputs are synthetic; weights stream from HBM every step (1.0 GB > 126 MB L2).

With --gpus N > 1 (under torchrun) every rank runs the same workload on its own
GPU as an independent replica (the engine has no cross-GPU step); the timed
region is bracketed by barriers and the time is the max over ranks.

--impl reference times the CPU oracle (plain C, double precision) on a
bounded sample of the same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "d20 bf16 prefill tok/s & decode tok/s (B=32); % of HBM / tensor-core roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16, the vendor's figure
NOMINAL_HBM_GBS = 8000.0


def finite(v):
    """v with every non-finite float replaced by None (strict JSON)."""
    if isinstance(v, float):
        return v if math.isfinite(v) else None
    if isinstance(v, dict):
        return {k: finite(x) for k, x in v.items()}
    if isinstance(v, (list, tuple)):
        return [finite(x) for x in v]
    return v


def emit(line: dict):
    print(json.dumps(finite(line), allow_nan=False), flush=True)


# ------------------------------------------------------------ accounting
def linear_params(cfg) -> int:
    """Weights of the per-layer linears (QKV, O, fc, proj), all layers."""
    d, hd, H, Hkv, F = cfg.d_model, cfg.head_dim, cfg.n_head, cfg.n_kv_head, cfg.mlp_hidden
    return cfg.depth * (d * (H + 2 * Hkv) * hd + H * hd * d + 2 * d * F)


def prefill_flops(cfg, B: int, T: int) -> dict:
    """Algorithmic FLOPs of one prefill with last-position logits."""
    lin = 2 * B * T * linear_params(cfg)
    attn = cfg.depth * B * 4 * cfg.n_head * cfg.head_dim * T * (T + 1) // 2
    head = 2 * B * cfg.d_model * cfg.vocab
    return {"gemm": lin, "attn": attn, "head": head, "total": lin + attn + head}


def decode_bytes(cfg, B: int, ctx_avg: float, shared_rows: int = 0) -> dict:
    """Algorithmic HBM bytes of one decode step (bf16 weights and cache, fp32
    logits). shared_rows: key/value rows every sequence reads from one shared
    prefix (nc_kv_fork_shared), counted once."""
    kd = cfg.n_kv_head * cfg.head_dim
    w_lin = 2 * linear_params(cfg)
    w_head = 2 * cfg.vocab * cfg.d_model
    kv_read = cfg.depth * (shared_rows + B * (ctx_avg - shared_rows)) * kd * 2 * 2
    kv_write = cfg.depth * B * kd * 2 * 2
    logits = 4 * B * cfg.vocab
    total = w_lin + w_head + kv_read + kv_write + logits
    return {"weights_linear": w_lin, "weights_head": w_head, "kv_read": kv_read, "kv_write": kv_write,
            "logits": logits, "total": total}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d["bf16_tflops_sustained"])}, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


# ----------------------------------------------------------------- clocks
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# prefill GEMMs, the mean over the QKV, O-proj, MLP fc and MLP proj launches of
# one layer (one of each per layer, so also the mean over a step's 80 launches),
# from an ncu capture (cold L2; writes still in L2 at kernel end not counted)
# of `python bench.py --steps 1 --warmup 3 --no-decode --no-workloads
# --no-cpu-baseline` with -k regex:gemm_tc -s 240 -c 4. To be re-taken
# whenever nc_gemm_tc.cu changes.
GEMM_DRAM_BYTES_PER_LAUNCH = (56_577_792 + 196_133_632 + 169_057_280 + 400_016_384) / 4


# DRAM bytes of one whole-step decode launch (d20, 32 sequences at context
# 2051): dram__bytes_read.sum + dram__bytes_write.sum (1.550685 GB + 8.508 MB)
# from an ncu capture of `python bench.py --only decode --decode-steps 8
# --warmup 3` with -k regex:decode_step_kernel -s 6 -c 1. To be re-taken
# whenever nc_step.cu changes.
DECODE_STEP_DRAM_BYTES = 1_550_685_000 + 8_507_648


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            # nvidia-smi takes a moment to start: wait (up to 5 s) for its
            # first sample, so the samples cover the timed region
            t_end = time.time() + 5.0
            while time.time() < t_end and os.path.getsize(self.path) == 0 and self.proc.poll() is None:
                time.sleep(0.02)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, power, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                smax.append(float(parts[2].split()[0]))
                power.append(float(parts[3].split()[0]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


# ----------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank scalar (the timed region) over all ranks."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(units_per_rank: float, t_ms_max: float, world: int) -> float:
    """Whole-job throughput of independent replicas: every rank processed
    units_per_rank in at most t_ms_max milliseconds."""
    return world * units_per_rank / (t_ms_max / 1e3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------ CPU oracle
def oracle_prefill_sample(cfg, blob, prompts, n_tokens: int, threads: int | None = None):
    """Time the oracle's prefill of the first n_tokens of prompt 0 on `threads`
    host threads (all by default); -> (tok/s, seconds, threads used)."""
    import oracle as orc
    full = orc.num_threads()
    if threads:
        orc.set_threads(threads)
    try:
        om = orc.OracleModel(cfg, blob)
        used = orc.num_threads()
        t0 = time.perf_counter()
        om.forward_full(prompts[0, :n_tokens], all_positions=False)
        dt = time.perf_counter() - t0
    finally:
        orc.set_threads(full)
    return n_tokens / dt, dt, used


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import nc_synth as syn
    import oracle as orc
    w = syn.WORKLOADS["d20_prefill"]
    cfg = w.model
    blob = syn.make_blob(cfg, w.weight_seed)
    prompts = syn.prompt_tokens(w)
    om = orc.OracleModel(cfg, blob)
    n_tok = args.ref_tokens
    for _ in range(args.warmup):
        om.forward_full(prompts[0, :n_tok], all_positions=False)
    times = []
    for s in range(args.steps):
        seq = prompts[s % w.batch, :n_tok]
        t0 = time.perf_counter()
        om.forward_full(seq, all_positions=False)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = args.steps * n_tok / total
    sample = (f"oracle prefill of the first {n_tok} tokens of one d20 prompt per step "
              f"(the workload is 8 x 2048 tokens)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "d20_prefill: 8 x 2048 Zipf(1.1) tokens, d20 bf16 N(0,0.02) weights",
                   "batch": w.batch, "seq_len": w.prompt_len, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": orc.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit(line)


# --------------------------------------------------------------- our arm
def run_ours(args):
    import numpy as np
    import torch

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)

    import kv_cache_transformer_b200 as nc
    import nc_synth as syn
    from kv_cache_transformer_b200 import build as ncbuild
    if rank == 0:
        ncbuild.build()
    barrier(world)

    peaks, peaks_src = load_peaks()
    wp, wd = syn.WORKLOADS["d20_prefill"], syn.WORKLOADS["d20_decode"]
    cfg = wp.model
    blob = syn.make_blob(cfg, wp.weight_seed)
    model = nc.Model(cfg, blob)
    max_seq = wd.prompt_len + wd.decode_steps
    kv = model.kv(max(wp.batch, wd.batch), max_seq)
    stream = torch.cuda.current_stream()
    B, T, V = wp.batch, wp.prompt_len, cfg.vocab

    prompts_np = syn.prompt_tokens(wp)
    tokens = torch.from_numpy(prompts_np).cuda()
    logits = torch.empty((B, V), dtype=torch.float32, device="cuda")
    nxt = torch.empty((B,), dtype=torch.int32, device="cuda")

    if args.only == "decode":
        dec = run_decode(args, model, kv, wd, cfg, peaks, peaks_src, world, local)
        if rank == 0:
            emit({"metric": METRIC, "only": "decode", "decode": dec})
        kv.close()
        model.close()
        return

    # ---------------- prefill: device-resident inputs
    for _ in range(args.warmup):
        model.prefill(kv, tokens, 0, logits, nxt)
    torch.cuda.synchronize()
    assert model.status() == 0
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    n0 = nc.nc_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        model.prefill(kv, tokens, 0, logits, nxt)
    e1.record(stream)
    torch.cuda.synchronize()
    launches = nc.nc_launch_count() - n0
    clk = clocks.stop()
    barrier(world)
    t_ms = max_over_ranks(e0.elapsed_time(e1), world)
    ms_step = t_ms / args.steps
    value = replica_throughput(args.steps * B * T, t_ms, world)

    # per-kernel times: the same steps again with an event pair around every
    # launch. The events serialise the launches (no programmatic overlap of
    # one kernel's set-up with the previous one's tail), so this pass is
    # kept out of the headline timing above.
    model.profile(True)
    model.profile_read()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for _ in range(args.steps):
        model.prefill(kv, tokens, 0, logits, nxt)
    p1.record(stream)
    torch.cuda.synchronize()
    kms, kn = model.profile_read()
    model.profile(False)
    ms_step_profiled = p0.elapsed_time(p1) / args.steps

    fl = prefill_flops(cfg, B, T)
    gemm_ms = kms[nc.NC_K_GEMM] / args.steps  # GEMM time per step
    gemm_launch_per_step = kn[nc.NC_K_GEMM] / args.steps
    gemm_tflops = fl["gemm"] / (gemm_ms / 1e3) / 1e12
    # the burst peak (cuBLAS bf16 at full clock) is the denominator; the
    # sustained figure was measured over seconds at a lower, power-capped
    # clock than a prefill step runs at, so it is only reported beside it
    peak_tc = peaks["bf16_tflops"]
    roofline = {
        "bound": "tensor", "kernel": "prefill linear-layer GEMMs (QKV, O, fc relu^2, proj)",
        "achieved": gemm_tflops, "peak": peak_tc, "unit": "TFLOP/s", "frac": gemm_tflops / peak_tc,
        "traffic": GEMM_DRAM_BYTES_PER_LAUNCH, "peak_source": f"{peaks_src} bf16_tflops (burst)",
        "frac_of_sustained": gemm_tflops / peaks["bf16_tflops_sustained"],
        "flops_per_launch": fl["gemm"] / max(gemm_launch_per_step, 1),
        "ms_per_launch": gemm_ms / max(gemm_launch_per_step, 1),
        "launches_per_step": gemm_launch_per_step,
        "ms_per_step_profiled": ms_step_profiled,
    }
    step_tflops = fl["total"] / (ms_step / 1e3) / 1e12
    kernel_share = {nc.K_CLASS_NAMES[i]: round(float(kms[i] / max(kms.sum(), 1e-9)), 4) for i in range(nc.NC_K_COUNT)}

    # ---------------- prefill end to end: pinned host tokens in, logits + tokens out
    tok_host = torch.from_numpy(prompts_np).pin_memory()
    logits_host = torch.empty((B, V), dtype=torch.float32).pin_memory()
    nxt_host = torch.empty((B,), dtype=torch.int32).pin_memory()
    tok_dev = torch.empty_like(tokens)
    for _ in range(args.warmup):
        tok_dev.copy_(tok_host, non_blocking=True)
        model.prefill(kv, tok_dev, 0, logits, nxt)
        logits_host.copy_(logits, non_blocking=True)
        nxt_host.copy_(nxt, non_blocking=True)
    torch.cuda.synchronize()
    barrier(world)
    e0.record(stream)
    for _ in range(args.steps):
        tok_dev.copy_(tok_host, non_blocking=True)
        model.prefill(kv, tok_dev, 0, logits, nxt)
        logits_host.copy_(logits, non_blocking=True)
        nxt_host.copy_(nxt, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    te_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e = {"value": world * args.steps * B * T / (te_ms / 1e3), "unit": "tok/s",
           "h2d_bytes_per_step": tok_host.numel() * 4,
           "d2h_bytes_per_step": logits_host.numel() * 4 + nxt_host.numel() * 4}

    # ---------------- decode: 32 sequences at 2048 tokens, 128 greedy steps
    decode = None
    if not args.no_decode:
        decode = run_decode(args, model, kv, wd, cfg, peaks, peaks_src, world, local)

    # ---------------- the other decode workloads (d26 latency, d30 rollout)
    workloads = None
    if not args.no_workloads:
        workloads = {name: decode_workload(name, args, world, local, peaks, peaks_src)
                     for name in ("d26_latency", "d30_rollout")}
        workloads["d30_rollout_shared_prefix"] = decode_workload("d30_rollout", args, world, local, peaks, peaks_src,
                                                                 shared=True)
        workloads["d20_extend"] = extend_workload(args, world, local, peaks, peaks_src)
        workloads["sample_topk"] = sample_kernel_us(args)
        workloads["d20_mha"] = mha_workload(args, world, local, peaks, peaks_src)

    # ---------------- CPU oracle on a bounded sample (rank 0, N = 1)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, secs, thr = oracle_prefill_sample(cfg, blob, prompts_np, args.ref_tokens)
        n1 = max(8, args.ref_tokens // 8)
        tps1, secs1, _ = oracle_prefill_sample(cfg, blob, prompts_np, n1, threads=1)
        cpu = {"value": tps, "unit": "tok/s", "cores": thr, "kind": "oracle",
               "sample": f"oracle prefill of the first {args.ref_tokens} tokens of prompt 0 "
                         f"({secs:.1f} s on {thr} threads)",
               "single_core": {"value": tps1, "unit": "tok/s", "cores": 1,
                               "sample": f"first {n1} tokens of prompt 0 ({secs1:.1f} s on 1 thread)"}}

    line = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "d20_prefill: 8 x 2048 Zipf(1.1) tokens, d20 bf16 N(0,0.02) weights, "
                               "last-position logits + argmax", "batch": B, "seq_len": T,
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (1.0 GB of weights streamed per step)"},
        "roofline": roofline,
        "step_tflops": step_tflops, "step_frac_of_peak": step_tflops / peak_tc,
        "step_frac_of_nominal": step_tflops / NOMINAL_BF16_TFLOPS,
        "kernel_time_share": kernel_share,
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches), "clocks": clk,
        "decode": decode, "workloads": workloads,
    }
    if rank == 0:
        emit(line)
    kv.close()
    model.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_decode(args, model, kv, wd, cfg, peaks, peaks_src, world, local, traffic="d20", desc=None):
    import torch
    import kv_cache_transformer_b200 as nc
    import nc_synth as syn
    B, T, S, V = wd.batch, wd.prompt_len, args.decode_steps, cfg.vocab
    prompts = torch.from_numpy(syn.prompt_tokens(wd)).cuda()
    logits = torch.empty((B, V), dtype=torch.float32, device="cuda")
    tok = torch.empty((B,), dtype=torch.int32, device="cuda")  # fed tokens, overwritten by the next ones
    stream = torch.cuda.current_stream()

    def prefill():
        model.prefill(kv, prompts, 0, logits, tok)

    def step():
        # positions default to the current lengths (2048 + s); same pointers every
        # step, so the library replays one captured CUDA graph
        model.decode_step(kv, tok, None, None, logits, tok)

    prefill()
    for _ in range(min(args.warmup, S)):
        step()
    prefill()
    torch.cuda.synchronize()
    assert model.status() == 0
    clocks = ClockSampler(local)
    barrier(world)
    clocks.start()
    n0 = nc.nc_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(S):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = nc.nc_launch_count() - n0
    clk = clocks.stop()
    assert model.status() == 0
    assert int(kv.lengths(B).min()) == T + S
    barrier(world)
    t_ms = max_over_ranks(e0.elapsed_time(e1), world)
    ms_step = t_ms / S

    by = decode_bytes(cfg, B, T + (S + 1) / 2.0)
    gbs = by["total"] / (ms_step / 1e3) / 1e9

    # per-phase breakdown of one step of the whole-step kernel from its
    # timestamp trace (nc_decode_trace), at context ~2050, outside the timed loop
    prefill()
    for _ in range(2):
        step()
    trace = decode_phase_trace(kv, step, cfg.depth)

    return {
        "value": world * B * S / (t_ms / 1e3), "unit": "tok/s", "ms_per_step": ms_step, "steps": S,
        "config": {"workload": desc or ("d20_decode: 32 sequences prefilled to 2048 Zipf tokens, 128 greedy steps "
                                        "(positions 2048..2175), CUDA-graph replay"), "batch": B, "ctx": [T, T + S]},
        "roofline": {"bound": "hbm", "kernel": "whole decode step (one persistent kernel per step)",
                     "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "frac_of_nominal": gbs / NOMINAL_HBM_GBS,
                     "traffic": DECODE_STEP_DRAM_BYTES if traffic == "d20" else traffic,
                     "bytes_per_step": by["total"], "bytes": by, "peak_source": f"{peaks_src} hbm_gbs"},
        "phase_trace": trace,
        "gpu_launches": int(launches), "clocks": clk,
    }


def mha_workload(args, world: int, local: int, peaks, peaks_src) -> dict:
    """The d20 shapes with multi-head attention (n_kv_head = 10, the 560M
    model): prefill 8 x 2048 (tensor-core roofline of the GEMMs and of the
    whole step) and decode at batch 32, context 2048..2175 (HBM roofline;
    the KV cache is 10x the MQA model's, 6.9 of the 8.1 GB a step reads)."""
    import torch
    import kv_cache_transformer_b200 as nc
    import nc_synth as syn
    wp, wd = syn.WORKLOADS["d20_mha_prefill"], syn.WORKLOADS["d20_mha_decode"]
    cfg = wp.model
    model = nc.Model(cfg, syn.make_blob(cfg, wp.weight_seed))
    kv = model.kv(max(wp.batch, wd.batch), wd.prompt_len + args.decode_steps)
    B, T = wp.batch, wp.prompt_len
    tokens = torch.from_numpy(syn.prompt_tokens(wp)).cuda()
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    nxt = torch.empty((B,), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        model.prefill(kv, tokens, 0, logits, nxt)
    torch.cuda.synchronize()
    assert model.status() == 0
    steps = max(1, min(args.steps, 10))
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        model.prefill(kv, tokens, 0, logits, nxt)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    t_ms = max_over_ranks(e0.elapsed_time(e1), world)
    # per-kernel times in a second, event-bracketed pass (the events serialise
    # the launches, so it stays out of the step timing)
    model.profile(True)
    model.profile_read()
    for _ in range(steps):
        model.prefill(kv, tokens, 0, logits, nxt)
    torch.cuda.synchronize()
    kms, kn = model.profile_read()
    model.profile(False)
    fl = prefill_flops(cfg, B, T)
    ms_step = t_ms / steps
    gemm_ms = kms[nc.NC_K_GEMM] / steps
    attn_ms = kms[nc.NC_K_ATTN] / steps
    peak = peaks["bf16_tflops"]
    prefill = {
        "value": replica_throughput(steps * B * T, t_ms, world), "unit": "tok/s", "ms_per_step": ms_step,
        "steps": steps, "config": {"workload": "d20_mha_prefill: 8 x 2048 Zipf(1.1) tokens, d20 MHA bf16",
                                   "batch": B, "seq_len": T},
        "gemm_tflops": fl["gemm"] / (gemm_ms / 1e3) / 1e12,
        "gemm_frac": fl["gemm"] / (gemm_ms / 1e3) / 1e12 / peak,
        "attn_tflops": fl["attn"] / (attn_ms / 1e3) / 1e12 if attn_ms > 0 else None,
        "step_tflops": fl["total"] / (ms_step / 1e3) / 1e12,
        "step_frac_of_peak": fl["total"] / (ms_step / 1e3) / 1e12 / peak,
        "peak_source": f"{peaks_src} bf16_tflops (burst)",
    }
    decode = run_decode(args, model, kv, wd, cfg, peaks, peaks_src, world, local, traffic=None,
                        desc="d20_mha_decode: d20 MHA, 32 sequences prefilled to 2048 Zipf tokens, greedy steps "
                             "from position 2048, CUDA-graph replay")
    kv.close()
    model.close()
    return {"prefill": prefill, "decode": decode}


def decode_phase_trace(kv, step, depth: int):
    """Run step() once with the step kernel's phase timestamps on and reduce
    them to microseconds per phase type (summed over the layers): the median
    over CTAs of each phase's span and of its parts. None when the cache has
    no whole-step kernel."""
    import numpy as np
    import torch
    grid, P = kv.trace(None)
    if grid == 0:
        return None
    buf = torch.zeros(grid * P * 8, dtype=torch.int64, device="cuda")
    kv.trace(buf)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    step()
    e1.record()
    torch.cuda.synchronize()
    kv.trace(None)
    event_us = 1e3 * e0.elapsed_time(e1)
    tr = buf.cpu().numpy().reshape(grid, P, 8).astype(np.float64)
    tr[tr == 0] = np.nan
    t0 = np.nanmin(tr[:, 0, 0])
    tr = (tr - t0) / 1e3  # us from the first phase start
    kinds = ["embed"] + [k for _ in range(depth) for k in ("qkv", "attn", "oproj", "fc", "proj")] + ["head", "merge"]
    start = tr[:, :, 0]
    parts = ("stage", "first_acc", "reduce", "epilogue")
    out = {}
    for p, kind in enumerate(kinds):
        rec = out.setdefault(kind, {"phases": 0, "span": 0.0, "barrier": 0.0, **{k: 0.0 for k in parts}})
        rec["phases"] += 1
        end = start[:, p + 1] if p + 1 < P else tr[:, p, 4]
        rec["span"] += float(np.nanmedian(end - start[:, p]))
        if p + 1 < P:
            rec["barrier"] += float(np.nanmedian(start[:, p + 1] - tr[:, p, 4]))
        for j, k in enumerate(parts):
            d = tr[:, p, j + 1] - tr[:, p, j]
            if np.any(np.isfinite(d)):
                rec[k] += float(np.nanmedian(d))
    for rec in out.values():
        for k in list(rec):
            if isinstance(rec[k], float):
                rec[k] = round(rec[k], 2)
    span = float(np.nanmax(tr[:, P - 1, 4]))
    return {"note": "us per step by phase type, summed over layers; span = median over CTAs of a phase's "
                    "start-to-next-start, barrier = work done to next start; parts are medians over the CTAs "
                    "that reached them", "grid": grid, "kernel_span_us": round(span, 1),
            "event_us": round(event_us, 1), "by_phase": out}


def decode_workload(name: str, args, world: int, local: int, peaks, peaks_src, shared: bool = False) -> dict:
    """d26 latency decode (B=1, 1024-token prompt, 512 greedy steps) or d30
    rollout (256-token prompt prefilled once, forked to 16 samples, 256 steps
    of argmax over logits + Gumbel noise): decode tok/s over all ranks and the
    HBM roofline of a decode step."""
    import numpy as np
    import torch
    import kv_cache_transformer_b200 as nc
    import nc_synth as syn
    w = syn.WORKLOADS[name]
    cfg = w.model
    model = nc.Model(cfg, syn.make_blob(cfg, w.weight_seed))
    V, T, S = cfg.vocab, w.prompt_len, w.decode_steps
    max_seq = T + S
    prompts = torch.from_numpy(syn.prompt_tokens(w)).cuda()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    extra = {}
    caches = []
    if w.fork:
        n = w.fork
        src = model.kv(1, max_seq)
        dst = model.kv(n, max_seq)
        caches = [src, dst]
        tok1 = torch.empty((1,), dtype=torch.int32, device="cuda")
        logits = torch.empty((n, V), dtype=torch.float32, device="cuda")
        tok = torch.empty((n,), dtype=torch.int32, device="cuda")
        # seeded Gumbel noise per step and sample, generated up front (an input)
        noise = torch.from_numpy(np.stack([syn.gumbel(w.noise_seed, (n, V), stream=s_) for s_ in range(S)])).cuda()

        fork = src.fork_shared_to if shared else src.fork_to

        prefilled = []

        def start():
            # a source whose rows samples read cannot be replaced while they do:
            # with shared forks it is prefilled once, and each later fork into
            # dst replaces the samples (and their links)
            if not (shared and prefilled):
                model.prefill(src, prompts, 0, None, tok1)
                prefilled.append(True)
            fork(0, dst, 0, n)
            tok.copy_(tok1.expand(n))

        def step(s_):
            model.decode_step(dst, tok, None, noise[s_], logits, tok)

        B = n
        for _ in range(max(1, args.warmup // 3)):
            start()
            for s_ in range(S):
                step(s_)
        torch.cuda.synchronize()
        e0.record(stream)
        if not shared:
            model.prefill(src, prompts, 0, None, tok1)
        e1.record(stream)
        ef = torch.cuda.Event(enable_timing=True)
        fork(0, dst, 0, n)
        ef.record(stream)
        tok.copy_(tok1.expand(n))
        torch.cuda.synchronize()
        shared_rows = T // 64 * 64 if shared else 0
        extra = {"prefill_ms": None if shared else e0.elapsed_time(e1), "fork_ms": e1.elapsed_time(ef),
                 "fork_bytes": cfg.depth * 2 * (T - shared_rows) * cfg.head_dim * 2 * n,
                 "fork_kind": "nc_kv_fork_shared (prefix rows read from the source)" if shared
                 else "nc_kv_fork (copy)"}
    else:
        shared_rows = 0
        kv = model.kv(w.batch, max_seq)
        caches = [kv]
        B = w.batch
        logits = torch.empty((B, V), dtype=torch.float32, device="cuda")
        tok = torch.empty((B,), dtype=torch.int32, device="cuda")

        def start():
            model.prefill(kv, prompts, 0, logits, tok)

        def step(s_):
            model.decode_step(kv, tok, None, None, logits, tok)

        for _ in range(max(1, args.warmup // 3)):
            start()
            for s_ in range(min(S, 16)):
                step(s_)
        start()
    clocks = ClockSampler(local)
    torch.cuda.synchronize()
    barrier(world)
    clocks.start()
    n0 = nc.nc_launch_count()
    d0.record(stream)
    for s_ in range(S):
        step(s_)
    d1.record(stream)
    torch.cuda.synchronize()
    launches = nc.nc_launch_count() - n0
    clk = clocks.stop()
    assert model.status() == 0
    barrier(world)
    t_ms = max_over_ranks(d0.elapsed_time(d1), world)
    ctx_avg = T + (S + 1) / 2.0
    by = decode_bytes(cfg, B, ctx_avg, shared_rows)
    ms_step = t_ms / S
    gbs = by["total"] / (ms_step / 1e3) / 1e9
    for c in caches:
        c.close()
    model.close()
    return {
        "metric": f"{name} bf16 decode tok/s; % of HBM roofline", "value": world * B * S / (t_ms / 1e3),
        "unit": "tok/s", "n_gpus": world, "steps": S, "ms_per_step": ms_step, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": name, "batch": B, "prompt": T, "decode_steps": S, "fork": w.fork,
                   "gumbel_noise": bool(w.fork)},
        "roofline": {"bound": "hbm", "kernel": "whole decode step", "achieved": gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "bytes_per_step": by["total"], "peak_source": f"{peaks_src} hbm_gbs"},
        "gpu_launches": int(launches), "clocks": clk, **extra,
    }


def extend_workload(args, world: int, local: int, peaks, peaks_src) -> dict:
    """d20 chunked prefill: 8 sequences holding 2048-token prompts each take a
    256-token chunk at their current length (nc_prefill_extend). tok/s of the
    chunk tokens over all ranks; the chunk's FLOPs against the tensor peak."""
    import torch
    import kv_cache_transformer_b200 as nc
    import nc_synth as syn
    w = syn.WORKLOADS["d20_prefill"]
    cfg = w.model
    model = nc.Model(cfg, syn.make_blob(cfg, w.weight_seed))
    B, T0, T1 = w.batch, w.prompt_len, 256
    kv = model.kv(B, T0 + T1)
    prompts = torch.from_numpy(syn.prompt_tokens(w)).cuda()
    chunk = torch.from_numpy(syn.tokens_zipf(9, (B, T1), cfg.vocab)).cuda()
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    nxt = torch.empty((B,), dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for it in range(args.warmup + max(2, args.steps // 5)):
        model.prefill(kv, prompts, 0, logits, nxt)
        e0.record(stream)
        model.extend(kv, chunk, 0, logits, nxt)
        e1.record(stream)
        torch.cuda.synchronize()
        if it >= args.warmup:
            times.append(e0.elapsed_time(e1))
    assert model.status() == 0
    barrier(world)
    t_ms = max_over_ranks(sum(times) / len(times), world)
    lin = 2 * B * T1 * linear_params(cfg)
    ctx_avg = T0 + (T1 + 1) / 2.0
    attn = cfg.depth * B * T1 * 4 * cfg.n_head * cfg.head_dim * ctx_avg
    flops = lin + attn + 2 * B * cfg.d_model * cfg.vocab
    tf = flops / (t_ms / 1e3) / 1e12
    kv.close()
    model.close()
    return {"metric": "d20 chunked prefill tok/s (256-token chunk after 2048)", "value": world * B * T1 / (t_ms / 1e3),
            "unit": "tok/s", "n_gpus": world, "ms_per_chunk": t_ms, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "d20_extend", "batch": B, "prompt": T0, "chunk": T1},
            "roofline": {"bound": "tensor", "kernel": "whole chunk", "achieved": tf, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": tf / peaks["bf16_tflops"], "flops": flops,
                         "peak_source": f"{peaks_src} bf16_tflops (burst)"}}


def sample_kernel_us(args) -> dict:
    """Device time of one nc_sample_topk over 32 rows of 65536 fp32 logits
    (temperature 0.8, top_k 50) with Gumbel noise."""
    import numpy as np
    import torch
    import kv_cache_transformer_b200 as nc
    import nc_synth as syn
    B, V = 32, 65536
    lg = torch.from_numpy((np.random.default_rng(0).standard_normal((B, V)) * 3).astype(np.float32)).cuda()
    nz = torch.from_numpy(syn.gumbel(5, (B, V), stream=0)).cuda()
    nx = torch.empty((B,), dtype=torch.int32, device="cuda")
    for _ in range(3):
        nc.nc_sample_topk(lg, nx, nz, 0.8, 50)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 20
    e0.record()
    for _ in range(n):
        nc.nc_sample_topk(lg, nx, nz, 0.8, 50)
    e1.record()
    torch.cuda.synchronize()
    us = 1e3 * e0.elapsed_time(e1) / n
    return {"us_per_call": us, "rows": B, "vocab": V, "temperature": 0.8, "top_k": 50,
            "bytes_per_call": 4 * B * V * 2, "GB/s": 4 * B * V * 2 / (us / 1e6) / 1e9,
            "note": "each row is read twice (top-digit histogram, candidate compaction); the remaining radix "
                    "digits and the pick run on the compacted candidates and read only their noise"}


def run_decode_workload(args):
    """One JSON line for --workload d26_latency | d30_rollout | d20_mha | d20_extend | sample_topk."""
    import torch
    from kv_cache_transformer_b200 import build as ncbuild
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    ncbuild.build()
    peaks, peaks_src = load_peaks()
    if args.workload == "d20_mha":
        line = mha_workload(args, 1, local, peaks, peaks_src)
    elif args.workload == "sample_topk":
        line = sample_kernel_us(args)
    elif args.workload == "d20_extend":
        line = extend_workload(args, 1, local, peaks, peaks_src)
    else:
        line = decode_workload(args.workload, args, 1, local, peaks, peaks_src)
    line["warmup"] = args.warmup
    if rank == 0:
        emit(line)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--decode-steps", type=int, default=128)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--only", choices=("all", "decode"), default="all",
                    help="decode: skip the prefill timing (for profiling the decode kernels)")
    ap.add_argument("--workload", choices=("d20", "d26_latency", "d30_rollout", "d20_mha", "d20_extend", "sample_topk"), default="d20",
                    help="d20: the headline prefill + decode line; d26_latency / d30_rollout: the other "
                         "decode workloads, d20_mha: prefill and decode of the multi-head d20, one JSON line each")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="skip the d26 latency and d30 rollout lines")
    ap.add_argument("--ref-tokens", type=int, default=128,
                    help="tokens of one prompt the CPU oracle runs per sample")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    elif args.workload != "d20":
        run_decode_workload(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
