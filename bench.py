#!/usr/bin/env python
"""Benchmark of the block-sparse video attention path on B200.

One step = one pass of the whole path over one synthetic layer: pooling ->
pooled scoring + selection -> Macro block-sparse attention -> Micro selection
-> Micro attention with the fused exact LSE merge.  Default workload: the
HunyuanVideo-like 720p layer (B1 H24 N=118,800 padded to 118,912, d128,
128x128 blocks, 20% kept per row, Micro repair above the 99th percentile in 6
of 24 heads, heavy-tailed Q/K), bf16 inputs resident in HBM.

Metric: effective TFLOP/s over the kept tiles (4*Bq*Bk*d per kept Macro tile
plus 4*64*16*d per Micro tile, whole job over all ranks) with ms per step,
the fraction of the measured bf16 tensor peak, and the speedup over the same
attention kernel run with every block kept (dense).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

Multi-GPU (torchrun, one process per GPU): every rank runs its own full layer
(independent problems, no data-path collective; weak scaling); the step time
is the max over ranks.  --impl reference times the fp64 CPU oracle on a
bounded sample of the same workload on the host cores.
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

import numpy as np  # noqa: E402
import torch  # noqa: E402

from video_inputs import WORKLOADS, make_qkv, micro_heads, sweep_points  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
METRIC = "block-sparse attn ms & effective TFLOP/s (% bf16 peak), speedup vs dense, 1xB200"

# DRAM bytes (read + write) of the Macro pass per hunyuan step, from a
# one-pass ncu capture of its two launches (the summary sits under profiles/),
# valid only while the kernel sources hash to the value it was taken with.
MACRO_TRAFFIC = {
    "sources": ["csrc/attn_fwd_dual.cuh", "csrc/attn_fwd.cuh", "csrc/common.cuh"],
    "sha256_16": "85e1fb747ab1ff4a",
    "workload": "hunyuan",
    "bytes_per_step": (2218757376 + 545910016) + (786019584 + 343035136),
}


def macro_traffic(workload: str):
    """The captured Macro-pass DRAM bytes per step, or None when the workload
    differs or the kernel sources changed since the capture."""
    import hashlib
    if workload != MACRO_TRAFFIC["workload"]:
        return None
    h = hashlib.sha256()
    pkg = os.path.join(os.path.dirname(os.path.abspath(__file__)), "block_sparse_attention_pool_b200")
    for rel in MACRO_TRAFFIC["sources"]:
        with open(os.path.join(pkg, rel), "rb") as f:
            h.update(f.read())
    return MACRO_TRAFFIC["bytes_per_step"] if h.hexdigest()[:16] == MACRO_TRAFFIC["sha256_16"] else None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def workload_label(w):
    T, Y, X = w.grid
    s = (f"{w.name}: B{w.B} H{w.H} d{w.d} grid {T}x{Y}x{X} N={w.n_valid} (pad {w.n_pad}) "
         f"blocks {w.bq}x{w.bk}")
    if w.fixed_k:
        s += f" keep k={w.fixed_k}/{w.n_pad // w.bk}"
    if w.cum_mass > 0:
        s += f" cum-mass {w.cum_mass} k_min {w.k_min}"
    if w.n_anchor:
        s += f" + {w.n_anchor} anchors"
    if w.micro_mode == 2:
        s += f" + Micro 64x16 tiles > p{int(w.micro_percentile * 100)} in {int(micro_heads(w).sum())}/{w.H} heads"
    elif w.micro_mode == 1:
        s += f" + Micro top-{w.micro_topk} 64x16 tiles"
    return s


# ---------------------------------------------------------------------------
# clocks sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# multi-rank reductions (every rank runs its own layer; no data-path collective)
# ---------------------------------------------------------------------------

def max_over_ranks(values, device, world):
    """Element-wise maximum over ranks (step times: the job is as slow as its
    slowest rank)."""
    t = torch.tensor(values, device=device, dtype=torch.float64)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(values, device, world):
    """Element-wise sum over ranks (work done by the whole job)."""
    t = torch.tensor(values, device=device, dtype=torch.float64)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return t.tolist()


# ---------------------------------------------------------------------------
# FLOP accounting (algorithmic, over kept tiles)
# ---------------------------------------------------------------------------

def macro_flops(counts: torch.Tensor, w) -> float:
    """4 * Bq * Bk * d per kept (query block, key block) pair."""
    return 4.0 * w.bq * w.bk * w.d * float(counts.sum().item())


def micro_flops(m_counts: torch.Tensor, w) -> float:
    return 4.0 * 64 * 16 * w.d * float(m_counts.sum().item())


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_gpu(args, rank, world, local_rank):
    import block_sparse_attention_pool_b200 as vsa
    from block_sparse_attention_pool_b200 import build as vsa_build

    if rank == 0 or not os.path.exists(vsa_build.LIB):
        vsa_build.build()
    if world > 1:
        torch.distributed.barrier()
    vsa.lib()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    heads = micro_heads(w)
    q, k, v = make_qkv(w)
    to_dev = lambda x: torch.from_numpy(x).to(dev).to(torch.bfloat16).contiguous()
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    pin = lambda x: torch.from_numpy(x).to(torch.bfloat16).pin_memory()
    hq, hk, hv = pin(q), pin(k), pin(v)
    del q, k, v
    cfg = vsa.PathConfig.from_workload(w, heads if w.micro_mode else None)
    run = vsa.SparseVideoAttention(cfg)
    stream = torch.cuda.current_stream(dev)

    # the dominant kernel (Macro attention) is timed by events around its own
    # launch inside every step, on the launching stream
    macro_ev = []

    stage_ev = []  # per step: events bracketing pool, select, Macro, Micro select, Micro pass

    def run_with_events(qq, kk, vv):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        b = run(qq, kk, vv, stream=stream, on_stage=lambda i: ev[i].record(stream))
        macro_ev.append((ev[2], ev[3]))
        stage_ev.append(ev)
        return b

    # kernels launched per step by this path: pooling, selection, the Macro
    # pass (one launch for the heads without the Micro repair, one for those
    # with it), Micro selection (percentile: bitmap, score, 3 rank searches,
    # 2 histograms, compaction; top-k: bitmap, top-k) and the Micro pass
    n_rep = (sum(1 for f in heads if f) if heads is not None else w.H) if w.micro_mode else 0
    n_macro = 1 if not w.micro_mode else int(n_rep > 0) + int(n_rep < w.H)
    n_micro = 0 if not w.micro_mode else (8 if w.micro_mode == 2 else 2) + int(n_rep > 0)
    launches_per_step = 2 + n_macro + n_micro

    for _ in range(args.warmup):
        run_with_events(dq, dk, dv)
    torch.cuda.synchronize(dev)
    st = vsa.read_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {vsa.status_string(st)}")
    macro_ev.clear()
    stage_ev.clear()
    fl_macro = macro_flops(run.buf["counts"], w)
    fl_micro = micro_flops(run.buf["m_counts"], w) if w.micro_mode else 0.0

    clocks = ClockSampler(local_rank)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        run_with_events(dq, dk, dv)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    macro_ms = [a.elapsed_time(b) for a, b in macro_ev]
    names = ["pool", "select", "macro_attention", "micro_select", "micro_attention_merge"]
    stages = {n: round(statistics.mean(e[i].elapsed_time(e[i + 1]) for e in stage_ev), 4) for i, n in enumerate(names)}
    st = vsa.read_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status after timed steps: {vsa.status_string(st)}")

    # end to end through the public API with host buffers: every step is one
    # C-ABI call (vsa_path_fwd_host, through forward_host) that copies Q/K/V
    # from pinned host memory and O/LSE back, pipelining the copies of one
    # chunk of heads with the path on the previous chunk
    ho = torch.empty(run.buf["o"].shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(run.buf["lse"].shape, dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.steps, 5))
    run.forward_host(hq, hk, hv, ho, hl, chunk_heads=args.chunk_heads)  # warm-up (buffers, streams)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(e2e_steps):
        run.forward_host(hq, hk, hv, ho, hl, chunk_heads=args.chunk_heads)
    s1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = s0.elapsed_time(s1) / e2e_steps
    h2d = 3 * hq.numel() * 2
    d2h = ho.numel() * 2 + hl.numel() * 4

    # dense reference: the same attention kernel with every key block kept
    n_k = w.n_pad // w.bk
    dense_cfg = vsa.PathConfig(n_valid=w.n_valid, bq=w.bq, bk=w.bk, scale=w.scale, fixed_k=n_k)
    dense = vsa.SparseVideoAttention(dense_cfg)
    dense(dq, dk, dv)
    torch.cuda.synchronize(dev)
    dense_ms_list = []
    for _ in range(2):
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b = dense.buf
        shape = vsa.Shape(w.B, w.H, w.n_valid, w.n_pad, w.d)
        d0.record(stream)
        vsa.block_sparse_fwd(dq, dk, dv, shape, w.bq, w.bk, b["counts"], b["idx"], n_k, w.scale, b["o"], b["lse"])
        d1.record(stream)
        torch.cuda.synchronize(dev)
        dense_ms_list.append(d0.elapsed_time(d1))
    dense_ms = min(dense_ms_list)
    dense_flops = 4.0 * w.bq * w.bk * w.d * float(dense.buf["counts"].sum().item())
    del dense

    # the sweep's 85%-sparsity points on the same tensors (selection, then the
    # attention pass alone, CUDA events), so that both block shapes' efficiency
    # at high sparsity sits in the default line
    sweep85 = {}
    if args.workload == "hunyuan":
        for frac, sw in sweep_points():
            if frac != 0.15:
                continue
            scfg = vsa.PathConfig(n_valid=sw.n_valid, bq=sw.bq, bk=sw.bk, scale=sw.scale, fixed_k=sw.fixed_k)
            srun = vsa.SparseVideoAttention(scfg)
            srun(dq, dk, dv)
            sb = srun.buf
            sshape = vsa.Shape(sw.B, sw.H, sw.n_valid, sw.n_pad, sw.d)
            sfwd = lambda: vsa.block_sparse_fwd(dq, dk, dv, sshape, sw.bq, sw.bk, sb["counts"], sb["idx"],
                                                sw.n_pad // sw.bk, sw.scale, sb["o"], sb["lse"])
            sfwd()
            torch.cuda.synchronize(dev)
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            for _ in range(3):
                sfwd()
            s1.record(stream)
            torch.cuda.synchronize(dev)
            sms = s0.elapsed_time(s1) / 3
            stf = macro_flops(sb["counts"], sw) / (sms * 1e-3) / 1e12
            sweep85[f"{sw.bq}x{sw.bk}"] = {"kept_fraction": frac, "k": sw.fixed_k, "attn_ms": round(sms, 3),
                                           "effective_tflops": round(stf, 2)}
            del srun
        st = vsa.read_device_status(stream)
        if st != 0:
            raise RuntimeError(f"device status after the sweep points: {vsa.status_string(st)}")

    # job time = slowest rank; job work = all ranks' kept-tile FLOPs
    ms_total, e2e_ms = max_over_ranks([ms_total, e2e_ms], dev, world)
    (job_flops,) = sum_over_ranks([fl_macro + fl_micro], dev, world)
    ms_step = ms_total / args.steps
    flops_step = fl_macro + fl_micro
    value = job_flops / (ms_step * 1e-3) / 1e12
    e2e_value = job_flops / (e2e_ms * 1e-3) / 1e12
    pk = peaks()
    macro_avg_ms = statistics.mean(macro_ms)
    achieved = fl_macro / (macro_avg_ms * 1e-3) / 1e12
    # the burst figure: the step runs the Macro pass at clocks near the burst
    # measurement's (the sustained figure was taken power-capped at ~1.34 GHz);
    # the sustained fraction is reported beside it
    peak = pk["bf16"]
    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded video-shaped Q/K/V, no model weights)",
        "config": {
            "workload": workload_label(w),
            "global_batch": w.B * world,
            "seq_len": w.n_valid,
            "parallelism": f"independent layer per GPU x{world}",
            "l2": f"inputs {3 * w.B * w.H * w.n_pad * w.d * 2 / 1e9:.2f} GB > 126 MB L2 (no flush needed)",
            "kept_fraction_macro": round(float(run.buf["counts"].sum().item()) /
                                         (w.B * w.H * ((w.n_valid + w.bq - 1) // w.bq) * n_k), 4),
            "micro_tiles": int(run.buf["m_counts"].sum().item()) if w.micro_mode else 0,
        },
        "pct_of_bf16_peak": round(100.0 * flops_step / (ms_step * 1e-3) / 1e12 / peak, 2),
        "peak_tflops": peak,
        "peak_source": f"{pk['source']} bf16 burst",
        "dense_ms": round(dense_ms, 3),
        "dense_tflops": round(dense_flops / (dense_ms * 1e-3) / 1e12, 2),
        "speedup_vs_dense": round(dense_ms / ms_step, 3),
        "macro_kernel_ms": round(macro_avg_ms, 4),
        "stages_ms": stages,
        "sweep_85pct_sparsity": {key: dict(val, frac_of_bf16_peak=round(val["effective_tflops"] / pk["bf16"], 4))
                                 for key, val in sweep85.items()},
        "roofline": {
            "kernel": ("attn_fwd_dual_kernel<%d> (Macro pass" if (w.bq == 128 and w.bk == 128) else
                       "attn_fwd_kernel<%d> (Macro pass") % w.d + f", {n_macro} launch(es) per step timed together)",
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": peak,
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "traffic": macro_traffic(args.workload),
            "peak_source": f"{pk['source']} bf16 burst (cuBLAS 8192^3)",
            "frac_of_sustained": round(achieved / pk["bf16_sustained"], 4),
        },
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 3),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": f"vsa_path_fwd_host (one C-ABI call on pinned host buffers), {args.chunk_heads}-head chunks"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    return line


# ---------------------------------------------------------------------------
# CPU oracle (the baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(w, budget_blocks: int):
    """Time the fp64 oracle on a bounded sample of the workload: pooling and
    selection of one head, then Macro attention (and Micro, if any) of
    ``budget_blocks`` query blocks of that head.  Returns (flops, seconds,
    description)."""
    import oracle as orc
    q, k, v = make_qkv(w, heads=(0, 1))
    heads = micro_heads(w)[:1]
    t0 = time.perf_counter()
    qbar = orc.pool_block_means(q, w.bq, w.n_valid)
    kbar = orc.pool_block_means(k, w.bk, w.n_valid)
    kept = orc.select_blocks(qbar, kbar, w.n_valid, w.bq, w.bk, w.scale, w.k_min, w.cum_mass, w.fixed_k,
                             w.n_anchor, w.anchor_rot)
    n_q = w.n_pad // w.bq
    blocks = [(0, 0, int(i)) for i in np.linspace(0, (w.n_valid - 1) // w.bq, budget_blocks).astype(int)]
    orc.block_sparse_attention(q, k, v, kept, w.bq, w.bk, w.n_valid, w.scale, rows=blocks)
    flops = sum(4.0 * w.bq * w.bk * w.d * len(kept[0][0][i]) for _, _, i in blocks)
    desc = f"1 of {w.H} heads pooled+selected, Macro attention of {len(blocks)} of {n_q} query blocks"
    if w.micro_mode == 2 and heads[0]:
        q64 = orc.pool_block_means(q, 64, w.n_valid)
        k16 = orc.pool_block_means(k, 16, w.n_valid)
        tiles = orc.select_micro_percentile(q64, k16, kept, w.bq, w.bk, w.n_valid, w.scale, w.micro_percentile,
                                            heads)
        mrows = [(0, 0, r) for _, _, i in blocks for r in range(i * w.bq // 64, (i + 1) * w.bq // 64)]
        orc.micro_attention(q, k, v, tiles, w.n_valid, w.scale, rows=mrows)
        flops += sum(4.0 * 64 * 16 * w.d * len(tiles[0][0][r]) for _, _, r in mrows)
        desc += " + Micro selection of the head and Micro attention of their rows"
    dt = time.perf_counter() - t0
    return flops, dt, desc


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = WORKLOADS[args.workload]
    for _ in range(args.warmup):
        pass  # the oracle has no warm state worth priming; warm-up steps are no-ops
    tot_f, tot_s, desc = 0.0, 0.0, ""
    for _ in range(args.steps):
        f, s, desc = oracle_sample(w, budget_blocks=args.ref_blocks)
        tot_f += f
        tot_s += s
    val = tot_f / tot_s / 1e12
    return {
        "metric": METRIC, "impl": "reference", "value": val, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded video-shaped Q/K/V)",
        "config": {"workload": workload_label(w)},
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle", "sample": desc},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_sweep(args):
    """Sparsity sweep on the hunyuan tensors: kept fraction in {100, 50, 25,
    15, 8}% x blocks {128x128, 64x128}; selection + attention (no Micro),
    timed with CUDA events; one JSON line per point."""
    import block_sparse_attention_pool_b200 as vsa
    from block_sparse_attention_pool_b200 import build as vsa_build
    vsa_build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    base = WORKLOADS["hunyuan"]
    q, k, v = make_qkv(base)
    to_dev = lambda x: torch.from_numpy(x).to(dev).to(torch.bfloat16).contiguous()
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    del q, k, v
    stream = torch.cuda.current_stream(dev)
    pk = peaks()
    dense_ms = {}
    for frac, w in sweep_points():
        cfg = vsa.PathConfig(n_valid=w.n_valid, bq=w.bq, bk=w.bk, scale=w.scale, fixed_k=w.fixed_k)
        run = vsa.SparseVideoAttention(cfg)
        shape = vsa.Shape(w.B, w.H, w.n_valid, w.n_pad, w.d)
        run(dq, dk, dv)
        b = run.buf
        for _ in range(args.warmup):
            vsa.block_sparse_fwd(dq, dk, dv, shape, w.bq, w.bk, b["counts"], b["idx"], w.n_pad // w.bk, w.scale,
                                 b["o"], b["lse"])
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            vsa.block_sparse_fwd(dq, dk, dv, shape, w.bq, w.bk, b["counts"], b["idx"], w.n_pad // w.bk, w.scale,
                                 b["o"], b["lse"])
        e1.record(stream)
        torch.cuda.synchronize(dev)
        st = vsa.read_device_status(stream)
        if st != 0:
            raise RuntimeError(vsa.status_string(st))
        ms = e0.elapsed_time(e1) / args.steps
        flops = macro_flops(b["counts"], w)
        if frac == 1.0:
            dense_ms[(w.bq, w.bk)] = ms
        tf = flops / (ms * 1e-3) / 1e12
        print(json.dumps({"sweep_point": w.name, "blocks": f"{w.bq}x{w.bk}", "kept_fraction": frac,
                          "k": w.fixed_k, "attn_ms": round(ms, 3), "effective_tflops": round(tf, 2),
                          "frac_of_bf16_peak": round(tf / pk["bf16"], 4),
                          "peak": f"{pk['bf16']} TFLOP/s ({pk['source']} bf16 burst)",
                          "frac_of_sustained": round(tf / pk["bf16_sustained"], 4),
                          "speedup_vs_dense_same_blocks": round(dense_ms[(w.bq, w.bk)] / ms, 3)}), flush=True)
        del run


def run_cluster(args):
    """The cluster-permuted layout on the chosen workload (HyperVAttention
    Eq. (1), (4), (5)): 3D local-window clustering of Q and K, row
    permutation, the path on the permuted rows, and the output put back in
    token order.  One JSON line with the per-stage times (CUDA events), the
    step's effective TFLOP/s over kept tiles, and the relative L2 error of
    the final output against dense attention (the same kernel with every
    block kept) for the token-order and the cluster-permuted layouts."""
    import dataclasses
    import block_sparse_attention_pool_b200 as vsa
    from block_sparse_attention_pool_b200 import build as vsa_build
    vsa_build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    q, k, v = make_qkv(w)
    to_dev = lambda x: torch.from_numpy(x).to(dev).to(torch.bfloat16).contiguous()
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    del q, k, v
    stream = torch.cuda.current_stream(dev)
    heads = micro_heads(w) if w.micro_mode else None
    cfg = vsa.PathConfig.from_workload(w, heads)
    cfg.cluster_lattice = w.grid
    cfg.cluster_cell, cfg.cluster_window, cfg.cluster_iters = args.cluster_cell, args.cluster_window, args.cluster_iters
    run = vsa.SparseVideoAttention(cfg)
    B, H, n_pad, d = dq.shape
    shape = vsa.Shape(B, H, w.n_valid, n_pad, d)
    params = cfg.cluster_params()

    def step(ev):
        b = run.buf
        ev[0].record(stream)
        for name, x in (("q", dq), ("k", dk)):
            vsa.cluster_tokens(x, shape, params, b["assign_" + name], b["centroids_" + name], b["sizes_" + name],
                               b["perm_" + name], stream)
        ev[1].record(stream)
        vsa.permute_rows(dq, b["perm_q"], b["qp"], stream=stream)
        vsa.permute_rows(dk, b["perm_k"], b["kp"], stream=stream)
        vsa.permute_rows(dv, b["perm_k"], b["vp"], stream=stream)
        ev[2].record(stream)
        run._run(b["qp"], b["kp"], b["vp"], stream, b["op"], b["lp"])
        ev[3].record(stream)
        vsa.permute_rows(b["op"], b["perm_q"], b["o"], inverse=True, stream=stream)
        vsa.permute_rows(b["lp"], b["perm_q"], b["lse"], inverse=True, stream=stream)
        ev[4].record(stream)

    run(dq, dk, dv)  # buffers
    evs = []
    for i in range(args.warmup + args.steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        step(ev)
        if i >= args.warmup:
            evs.append(ev)
    torch.cuda.synchronize(dev)
    st = vsa.read_device_status(stream)
    if st != 0:
        raise RuntimeError(vsa.status_string(st))
    names = ["cluster_qk", "permute_in", "path", "permute_out"]
    stages = {n: round(statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs), 4) for i, n in enumerate(names)}
    ms = statistics.mean(e[0].elapsed_time(e[4]) for e in evs)
    flops = macro_flops(run.buf["counts"], w) + (micro_flops(run.buf["m_counts"], w) if w.micro_mode else 0.0)
    o_clu = run.buf["o"].float().clone()
    # the same path in token order, and dense attention of the same kernel
    plain = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, heads))
    o_tok = plain(dq, dk, dv)["o"].float().clone()
    del plain
    dense = vsa.SparseVideoAttention(vsa.PathConfig(n_valid=w.n_valid, bq=w.bq, bk=w.bk, scale=w.scale,
                                                    fixed_k=n_pad // w.bk))
    o_ref = dense(dq, dk, dv)["o"].float()
    nv = w.n_valid
    rel = lambda o: float(torch.linalg.vector_norm(o[:, :, :nv] - o_ref[:, :, :nv]) /
                          torch.linalg.vector_norm(o_ref[:, :, :nv]))
    sizes = run.buf["sizes_q"].float()
    line = {
        "metric": METRIC + " (cluster-permuted layout)",
        "value": round(flops / (ms * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s",
        "ms_per_step": round(ms, 4),
        "stages_ms": stages,
        "config": {"workload": workload_label(w), "lattice": list(w.grid), "cell": list(args.cluster_cell),
                   "window": list(args.cluster_window), "iters": args.cluster_iters,
                   "clusters_per_head": int(sizes.shape[-1]),
                   "cluster_size_mean_max": [round(float(sizes.mean()), 1), int(sizes.max())],
                   "kept_fraction_macro": round(float(run.buf["counts"].sum().item()) /
                                                (w.B * w.H * ((w.n_valid + w.bq - 1) // w.bq) * (n_pad // w.bk)), 4)},
        "rel_l2_error_vs_dense": {"token_order": round(rel(o_tok), 5), "cluster_permuted": round(rel(o_clu), 5)},
        "data": "synthetic (seeded video-shaped Q/K/V, no model weights)",
    }
    print(json.dumps(line), flush=True)


def run_cluster_blocks(args):
    """Cluster-aligned blocks on the chosen workload (HyperVAttention Eq. (1)-
    (5), (7)-(10), Algorithm 1): clustering, cluster-level selection, merging
    of query clusters, the group layout, attention per group tile, and the
    output back in token order, all on the device.  One JSON line: per-stage
    times (CUDA events), the attention kernel's tensor throughput over the
    tiles it executes, the cost model's CTA density and token density with
    and without merging, and the relative L2 error against dense attention."""
    import block_sparse_attention_pool_b200 as vsa
    from block_sparse_attention_pool_b200 import build as vsa_build
    from video_inputs import merge_sides
    vsa_build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    q, k, v = make_qkv(w)
    to_dev = lambda x: torch.from_numpy(x).to(dev).to(torch.bfloat16).contiguous()
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    del q, k, v
    stream = torch.cuda.current_stream(dev)
    B, H, n_pad, d = dq.shape
    rule = dict(k_min=w.k_min, cum_mass=w.cum_mass, fixed_k=0)
    if w.fixed_k:
        rule = dict(k_min=0, cum_mass=0.0, fixed_k=w.fixed_k)
    if args.cluster_cum_mass > 0:
        rule = dict(k_min=1, cum_mass=args.cluster_cum_mass, fixed_k=0)
    cfg = vsa.ClusterBlockConfig(n_valid=w.n_valid, lattice=w.grid, cell=args.cluster_cell,
                                 window=args.cluster_window, iters=args.cluster_iters, scale=w.scale,
                                 rounds=args.merge_rounds, **rule)
    G = vsa.cluster_count(cfg.cluster_params())
    if rule["fixed_k"]:
        cfg.fixed_k = max(1, min(G, int(round(rule["fixed_k"] * G / (n_pad // w.bk)))))
    sides = torch.from_numpy(merge_sides(w, args.merge_rounds, G)).to(dev) if args.merge_rounds else None
    run = vsa.ClusterBlockAttention(cfg)
    n_st = len(run.STAGES)

    def step(ev):
        run(dq, dk, dv, sides=sides, stream=stream, on_stage=lambda i: ev[i].record(stream))

    evs = []
    for i in range(args.warmup + args.steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_st + 1)]
        step(ev)
        if i >= args.warmup:
            evs.append(ev)
    torch.cuda.synchronize(dev)
    st = vsa.read_device_status(stream)
    if st != 0:
        raise RuntimeError(vsa.status_string(st))
    stages = {n: round(statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs), 4) for i, n in enumerate(run.STAGES)}
    ms = statistics.mean(e[0].elapsed_time(e[n_st]) for e in evs)
    b = run.buf

    def densities(buf):
        """Per head: groups' query tokens s_q(S), key tokens w_k(S), executed
        128 x 128 tiles (16-key segments packed per group) -> token density,
        CTA density of the cost model (Eq. (7)/(8)), executed tiles."""
        sq = buf["sizes_q"].long()
        sk = buf["sizes_k"].long()
        gof = buf["group_of"].long()
        cnt = buf["g_counts"].long()
        Gn = sq.shape[-1]
        valid = torch.arange(Gn, device=dev)[None, None, None, :] < cnt[..., None]
        # only the first g_counts entries of a row are written: index 0 elsewhere
        idx = torch.where(valid, buf["g_idx"].long(), 0).clamp(0, Gn - 1)
        wk = (torch.gather(sk[:, :, None, :].expand(-1, -1, Gn, -1), 3, idx) * valid).sum(-1)
        segs = (torch.gather(((sk + 15) // 16)[:, :, None, :].expand(-1, -1, Gn, -1), 3, idx) * valid).sum(-1)
        gsq = torch.zeros_like(sq).scatter_add_(2, gof, sq)
        lead = gof == torch.arange(Gn, device=dev)[None, None, :]
        gsq, wk, segs = gsq * lead, wk * lead, segs * lead
        nn = float(w.n_valid) ** 2 * B * H
        tok = float((gsq * wk).sum()) / nn
        cta = float((((gsq + 127) // 128) * ((wk + 127) // 128)).sum()) * 128 * 128 / nn
        tiles = int((((gsq + 127) // 128) * ((segs * 16 + 127) // 128)).sum())
        return tok, cta, tiles, int(lead.sum())

    tok_m, cta_m, tiles_m, n_groups = densities(b)
    o_merged = b["o"].float().clone()
    # the same path without merging (every query cluster its own group)
    run0 = vsa.ClusterBlockAttention(cfg)
    run0(dq, dk, dv, sides=None, stream=stream)
    torch.cuda.synchronize(dev)
    tok_0, cta_0, tiles_0, _ = densities(run0.buf)
    o_single = run0.buf["o"].float().clone()
    del run0
    dense = vsa.SparseVideoAttention(vsa.PathConfig(n_valid=w.n_valid, bq=w.bq, bk=w.bk, scale=w.scale,
                                                    fixed_k=n_pad // w.bk))
    o_ref = dense(dq, dk, dv)["o"].float()
    nv = w.n_valid
    rel = lambda o: float(torch.linalg.vector_norm(o[:, :, :nv] - o_ref[:, :, :nv]) /
                          torch.linalg.vector_norm(o_ref[:, :, :nv]))
    attn_ms = stages["attention"]
    tile_flops = 4.0 * d * 128 * 128 * tiles_m
    sizes = b["sizes_q"].float()
    line = {
        "metric": METRIC + " (cluster-aligned blocks)",
        "value": round(tile_flops / (attn_ms * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s (attention kernel, executed 128x128 tiles)",
        "ms_per_step": round(ms, 4),
        "stages_ms": stages,
        "config": {"workload": workload_label(w), "lattice": list(w.grid), "cell": list(args.cluster_cell),
                   "window": list(args.cluster_window), "iters": args.cluster_iters, "rounds": args.merge_rounds,
                   "tau": [cfg.tau_q, cfg.tau_k], "rule": {"k_min": cfg.k_min, "cum_mass": cfg.cum_mass,
                                                           "fixed_k": cfg.fixed_k},
                   "clusters_per_head": G, "groups_per_head_mean": round(n_groups / (B * H), 1),
                   "cluster_size_mean_max": [round(float(sizes.mean()), 1), int(sizes.max())]},
        "density": {"merged": {"token": round(tok_m, 4), "cta_cost_model": round(cta_m, 4), "tiles": tiles_m},
                    "unmerged": {"token": round(tok_0, 4), "cta_cost_model": round(cta_0, 4), "tiles": tiles_0}},
        "rel_l2_error_vs_dense": {"merged": round(rel(o_merged), 5), "unmerged": round(rel(o_single), 5)},
        "data": "synthetic (seeded video-shaped Q/K/V, no model weights)",
    }
    print(json.dumps(line), flush=True)


def run_rectify(args):
    """Pooled rectification of the omitted blocks on the chosen workload
    (Rectified SpaAttn): the path with rectification instead of the Micro
    repair.  One JSON line: per-stage times (CUDA events), the pooled pass's
    tensor throughput over the 128 x 128 tiles it executes, and the relative L2
    error of O against dense attention for plain block-sparse, Macro + Micro
    (the workload's repair) and rectified attention."""
    import dataclasses
    import block_sparse_attention_pool_b200 as vsa
    from block_sparse_attention_pool_b200 import build as vsa_build
    vsa_build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    q, k, v = make_qkv(w)
    to_dev = lambda x: torch.from_numpy(x).to(dev).to(torch.bfloat16).contiguous()
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    del q, k, v
    stream = torch.cuda.current_stream(dev)
    B, H, n_pad, d = dq.shape
    cfg = vsa.PathConfig.from_workload(w)
    cfg.micro_mode = 0
    cfg.rectify = True
    run = vsa.SparseVideoAttention(cfg)
    names = ["pool", "select", "macro", "pool_kv", "rectify"]
    evs = []
    for i in range(args.warmup + args.steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        run(dq, dk, dv, stream=stream, on_stage=lambda j: ev[j].record(stream))
        if i >= args.warmup:
            evs.append(ev)
    torch.cuda.synchronize(dev)
    st = vsa.read_device_status(stream)
    if st != 0:
        raise RuntimeError(vsa.status_string(st))
    stages = {n: round(statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs), 4) for i, n in enumerate(names)}
    ms = statistics.mean(e[0].elapsed_time(e[5]) for e in evs)
    o_rect = run.buf["o"].float().clone()
    n_k = n_pad // w.bk
    pooled_flops = 4.0 * d * 128 * (128 * -(-n_k // 128)) * (n_pad // 128) * B * H
    macro = macro_flops(run.buf["counts"], w)
    del run
    plain_cfg = vsa.PathConfig.from_workload(w)
    plain_cfg.micro_mode = 0
    o_plain = vsa.SparseVideoAttention(plain_cfg)(dq, dk, dv)["o"].float().clone()
    o_micro = None
    if w.micro_mode:
        o_micro = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, micro_heads(w)))(dq, dk, dv)["o"].float().clone()
    dense = vsa.SparseVideoAttention(vsa.PathConfig(n_valid=w.n_valid, bq=w.bq, bk=w.bk, scale=w.scale,
                                                    fixed_k=n_pad // w.bk))
    o_ref = dense(dq, dk, dv)["o"].float()
    nv = w.n_valid
    rel = lambda o: float(torch.linalg.vector_norm(o[:, :, :nv] - o_ref[:, :, :nv]) /
                          torch.linalg.vector_norm(o_ref[:, :, :nv]))
    errors = {"block_sparse": round(rel(o_plain), 5), "rectified": round(rel(o_rect), 5)}
    if o_micro is not None:
        errors["macro_plus_micro"] = round(rel(o_micro), 5)
    line = {
        "metric": METRIC + " (pooled rectification of omitted blocks)",
        "value": round(pooled_flops / (stages["rectify"] * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s (pooled pass, executed 128x128 tiles)",
        "ms_per_step": round(ms, 4),
        "stages_ms": stages,
        "macro_effective_tflops": round(macro / (stages["macro"] * 1e-3) / 1e12, 3),
        "config": {"workload": workload_label(w), "rectified_heads": H, "pooled_keys_per_tile": n_k},
        "rel_l2_error_vs_dense": errors,
        "data": "synthetic (seeded video-shaped Q/K/V, no model weights)",
    }
    print(json.dumps(line), flush=True)


def run_reuse(args):
    """Cross-step mask reuse over simulated denoising steps (MOD-DiT pattern
    refresh every delta-t steps; HyperVAttention section 3 temporal
    stability).  Step t's inputs are the workload's tensors plus a seeded drift,
    x_t = x_0 + drift * t * eps with eps ~ N(0, 1) per element (drawn on the
    device from a fixed seed).  SelectionSchedule(0, refresh) decides per step
    whether the path selects or reuses the last lists.  One JSON line: per
    step the mode, the path time (CUDA events), the relative L2 error against
    dense attention of that step with the scheduled lists and with a fresh
    selection, and the overlap (Jaccard) of the kept blocks."""
    import block_sparse_attention_pool_b200 as vsa
    from block_sparse_attention_pool_b200 import build as vsa_build
    vsa_build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    q, k, v = make_qkv(w)
    to_dev = lambda x: torch.from_numpy(x).to(dev).to(torch.bfloat16).contiguous()
    x0 = [to_dev(x) for x in (q, k, v)]
    del q, k, v
    gen = torch.Generator(device=dev).manual_seed(1000 + w.seed)
    eps = [torch.randn(x.shape, generator=gen, device=dev, dtype=torch.float32) for x in x0]
    stream = torch.cuda.current_stream(dev)
    heads = micro_heads(w) if w.micro_mode else None
    run = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, heads))
    fresh = vsa.SparseVideoAttention(vsa.PathConfig.from_workload(w, heads))
    n_pad = x0[0].shape[2]
    dense = vsa.SparseVideoAttention(vsa.PathConfig(n_valid=w.n_valid, bq=w.bq, bk=w.bk, scale=w.scale,
                                                    fixed_k=n_pad // w.bk))
    sched = vsa.SelectionSchedule(0, args.reuse_refresh)
    nv = w.n_valid
    rel = lambda o, ref: float(torch.linalg.vector_norm(o[:, :, :nv] - ref[:, :, :nv]) /
                               torch.linalg.vector_norm(ref[:, :, :nv]))

    def kept_mask(buf):
        n_k = buf["idx"].shape[-1]
        valid = torch.arange(n_k, device=dev)[None, None, None, :] < buf["counts"][..., None]
        # unused list slots scatter into a spare column n_k
        m = torch.zeros(buf["idx"].shape[:-1] + (n_k + 1,), dtype=torch.bool, device=dev)
        m.scatter_(3, torch.where(valid, buf["idx"].long(), n_k), True)
        return m[..., :n_k]

    steps = []
    for t in range(args.reuse_steps):
        xt = [(x.float() + args.reuse_drift * t * e).to(torch.bfloat16) for x, e in zip(x0, eps)]
        mode = sched.mode(t)
        for _ in range(args.warmup if t == 0 else 0):
            run(*xt)
        ms = []
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run(*xt, reuse_selection=(mode == "reuse"))
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ms.append(e0.elapsed_time(e1))
        o_sched = run.buf["o"].float().clone()
        fresh(*xt)
        ref = dense(*xt)["o"].float()
        a, b = kept_mask(run.buf), kept_mask(fresh.buf)
        jac = float((a & b).sum()) / max(1.0, float((a | b).sum()))
        steps.append({"t": t, "mode": mode, "ms": round(statistics.mean(ms), 4),
                      "rel_l2_error_vs_dense": round(rel(o_sched, ref), 5),
                      "rel_l2_error_fresh_selection": round(rel(fresh.buf["o"].float(), ref), 5),
                      "kept_jaccard_vs_fresh": round(jac, 4)})
        del xt, ref
    st = vsa.read_device_status(stream)
    if st != 0:
        raise RuntimeError(vsa.status_string(st))
    sel = [x["ms"] for x in steps if x["mode"] == "select"]
    reu = [x["ms"] for x in steps if x["mode"] == "reuse"]
    line = {
        "metric": METRIC + " (cross-step mask reuse)",
        "value": round(statistics.mean(sel) - statistics.mean(reu), 4) if reu else 0.0,
        "unit": "ms saved per reuse step",
        "config": {"workload": workload_label(w), "refresh": args.reuse_refresh, "drift_per_step": args.reuse_drift,
                   "steps": args.reuse_steps},
        "ms_select_step": round(statistics.mean(sel), 4),
        "ms_reuse_step": round(statistics.mean(reu), 4) if reu else None,
        "per_step": steps,
        "data": "synthetic (seeded video-shaped Q/K/V plus seeded per-step drift, no model weights)",
    }
    print(json.dumps(line), flush=True)


def run_cluster_hybrid(args):
    """Hybrid clustering across simulated denoising steps (HyperVAttention
    section 4.2; App. A.1: full clustering every two steps, 15% of the tokens
    cached).  Step t's inputs are the workload's tensors plus a seeded drift,
    x_t = x_0 + drift * t * eps (eps ~ N(0, 1), drawn on the device from a fixed
    seed).  The cluster-aligned path runs with an anchor step every
    --hybrid-every steps and refine steps in between, and, for comparison,
    with full clustering at every step.  One JSON line: per step the mode, the
    clustering time and the whole path time (CUDA events), and the relative L2
    error of O against dense attention for the hybrid and the full-clustering
    runs."""
    import block_sparse_attention_pool_b200 as vsa
    from block_sparse_attention_pool_b200 import build as vsa_build
    from video_inputs import merge_sides
    vsa_build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    q, k, v = make_qkv(w)
    to_dev = lambda x: torch.from_numpy(x).to(dev).to(torch.bfloat16).contiguous()
    x0 = [to_dev(x) for x in (q, k, v)]
    del q, k, v
    gen = torch.Generator(device=dev).manual_seed(2000 + w.seed)
    eps = [torch.randn(x.shape, generator=gen, device=dev, dtype=torch.float32) for x in x0]
    stream = torch.cuda.current_stream(dev)
    n_pad = x0[0].shape[2]
    rule = dict(k_min=1, cum_mass=args.cluster_cum_mass, fixed_k=0) if args.cluster_cum_mass > 0 else \
        (dict(k_min=0, cum_mass=0.0, fixed_k=w.fixed_k) if w.fixed_k else
         dict(k_min=w.k_min, cum_mass=w.cum_mass, fixed_k=0))
    cfg = vsa.ClusterBlockConfig(n_valid=w.n_valid, lattice=w.grid, cell=args.cluster_cell,
                                 window=args.cluster_window, iters=args.cluster_iters, scale=w.scale,
                                 rounds=args.merge_rounds, **rule)
    G = vsa.cluster_count(cfg.cluster_params())
    if rule["fixed_k"]:
        cfg.fixed_k = max(1, min(G, int(round(rule["fixed_k"] * G / (n_pad // w.bk)))))
    sides = torch.from_numpy(merge_sides(w, args.merge_rounds, G)).to(dev) if args.merge_rounds else None
    hyb = vsa.ClusterBlockAttention(cfg)
    full = vsa.ClusterBlockAttention(cfg)
    dense = vsa.SparseVideoAttention(vsa.PathConfig(n_valid=w.n_valid, bq=w.bq, bk=w.bk, scale=w.scale,
                                                    fixed_k=n_pad // w.bk))
    nv = w.n_valid
    rel = lambda o, ref: float(torch.linalg.vector_norm(o[:, :, :nv] - ref[:, :, :nv]) /
                               torch.linalg.vector_norm(ref[:, :, :nv]))
    n_st = len(hyb.STAGES)

    def timed(run, xt, mode):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_st + 1)]
        run(*xt, sides=sides, stream=stream, on_stage=lambda i: ev[i].record(stream), cluster_step=mode)
        torch.cuda.synchronize(dev)
        return ev[0].elapsed_time(ev[1]), ev[0].elapsed_time(ev[n_st])

    # warm-up of both modes on step 0's inputs
    for _ in range(args.warmup):
        hyb(*x0, sides=sides, cluster_step="anchor")
        hyb(*x0, sides=sides, cluster_step="refine")
        full(*x0, sides=sides, cluster_step="full")
    steps = []
    for t in range(args.reuse_steps):
        xt = [(x.float() + args.reuse_drift * t * e).to(torch.bfloat16) for x, e in zip(x0, eps)]
        mode = "anchor" if t % args.hybrid_every == 0 else "refine"
        c_ms, p_ms = timed(hyb, xt, mode)
        o_h = hyb.buf["o"].float().clone()
        cf_ms, pf_ms = timed(full, xt, "full")
        ref = dense(*xt)["o"].float()
        steps.append({"t": t, "mode": mode, "cluster_ms": round(c_ms, 4), "path_ms": round(p_ms, 4),
                      "cluster_ms_full": round(cf_ms, 4), "path_ms_full": round(pf_ms, 4),
                      "rel_l2_error_vs_dense": round(rel(o_h, ref), 5),
                      "rel_l2_error_full_clustering": round(rel(full.buf["o"].float(), ref), 5)})
        del xt, ref
    st = vsa.read_device_status(stream)
    if st != 0:
        raise RuntimeError(vsa.status_string(st))
    anc = [x["cluster_ms"] for x in steps if x["mode"] == "anchor"]
    ref_ms = [x["cluster_ms"] for x in steps if x["mode"] == "refine"]
    line = {
        "metric": METRIC + " (hybrid clustering across steps)",
        "value": round(statistics.mean(ref_ms), 4) if ref_ms else None,
        "unit": "ms clustering Q+K per refine step",
        "ms_cluster_anchor_step": round(statistics.mean(anc), 4),
        "ms_cluster_full_step": round(statistics.mean(x["cluster_ms_full"] for x in steps), 4),
        "config": {"workload": workload_label(w), "cell": list(args.cluster_cell), "window": list(args.cluster_window),
                   "iters": args.cluster_iters, "anchor_every": args.hybrid_every, "cached_fraction": cfg.hybrid_frac,
                   "drift_per_step": args.reuse_drift, "rounds": args.merge_rounds},
        "per_step": steps,
        "data": "synthetic (seeded video-shaped Q/K/V plus seeded per-step drift, no model weights)",
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="vsa", choices=["vsa", "reference"])
    ap.add_argument("--workload", default="hunyuan", choices=sorted(WORKLOADS))
    ap.add_argument("--ref-blocks", type=int, default=60, help="query blocks per oracle sample (reference arm)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--chunk-heads", type=int, default=2, help="heads per pipelined chunk of the e2e leg")
    ap.add_argument("--sweep", action="store_true", help="print the sparsity-sweep lines instead of the bench line")
    ap.add_argument("--cluster", action="store_true",
                    help="print the cluster-permuted-layout line (3D local-window clustering) instead of the bench line")
    ap.add_argument("--cluster-cell", type=int, nargs=3, default=(3, 5, 8))
    ap.add_argument("--cluster-window", type=int, nargs=3, default=(3, 5, 5))
    ap.add_argument("--cluster-iters", type=int, default=3)
    ap.add_argument("--cluster-blocks", action="store_true",
                    help="print the cluster-aligned-blocks line (selection on clusters, merging, group tiles)")
    ap.add_argument("--merge-rounds", type=int, default=3)
    ap.add_argument("--reuse", action="store_true",
                    help="print the cross-step mask reuse line (simulated denoising steps) instead of the bench line")
    ap.add_argument("--reuse-refresh", type=int, default=2)
    ap.add_argument("--cluster-hybrid", action="store_true",
                    help="print the hybrid-clustering line (anchor and refine steps over simulated steps)")
    ap.add_argument("--hybrid-every", type=int, default=2)
    ap.add_argument("--reuse-steps", type=int, default=6)
    ap.add_argument("--reuse-drift", type=float, default=0.05)
    ap.add_argument("--rectify", action="store_true",
                    help="print the pooled-rectification line (omitted blocks as pooled keys) instead of the bench line")
    ap.add_argument("--cluster-cum-mass", type=float, default=0.0,
                    help="cluster selection by cumulative mass instead of the workload's rule")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.sweep:
        run_sweep(args)
        return
    if args.cluster:
        run_cluster(args)
        return
    if args.cluster_blocks:
        run_cluster_blocks(args)
        return
    if args.rectify:
        run_rectify(args)
        return
    if args.reuse:
        run_reuse(args)
        return
    if args.cluster_hybrid:
        run_cluster_hybrid(args)
        return
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    line = run_gpu(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # size the sample to about 12 s of CPU work: a short calibration run, then the reported one
        w = WORKLOADS[args.workload]
        _, s2, _ = oracle_sample(w, budget_blocks=2)
        _, s6, _ = oracle_sample(w, budget_blocks=6)
        per_block = max((s6 - s2) / 4, 1e-4)
        fixed = max(0.0, s2 - 2 * per_block)
        n_blocks = int(max(6, min(w.n_pad // w.bq, round((args.cpu_seconds - fixed) / per_block))))
        f, s, desc = oracle_sample(w, budget_blocks=n_blocks)
        line["cpu_baseline"] = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                                "sample": desc, "seconds": round(s, 2)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
