#!/usr/bin/env python
"""Benchmark of the MoBA causal prefill forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

A step is one moba_forward over the whole workload (gate, scheduler,
past-block attention, own-block attention, merge) with inputs resident in
HBM.  Default workload: one 1,048,576-token sequence, 32 query heads over 8
KV heads, head dim 128, block 4096, top-k 12 (bf16, seeded synthetic N(0,1)).
Inputs of the default workload (8.6 GB of q alone) are far larger than the
126 MB L2; a workload whose inputs fit in L2 is flushed from it before every
timed step.

Timing: W untimed warm-up steps, then K steps between CUDA events on the
launching stream, bracketed by a barrier and a device synchronise; the max
over ranks is reported.  With N > 1 (torchrun) every rank runs an
independent replica of the workload: the forward has no exchange step.

Rank 0 prints one JSON line.  `value` is the whole-job effective TFLOP/s:
algorithmic flops 4 * d * (attended keys per query per head), summed, over
the step time.  `roofline` covers the dominant kernel (the tcgen05 block
attention: past blocks and own block), timed by stage events recorded
inside the library call.
`cpu_baseline` times the CPU oracle on a bounded sample of rows.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoBA prefill fwd ms and effective TFLOP/s (% bf16 peak) at 1M tokens, 1 B200"
DEFAULT_WORKLOAD = "long_1m_gqa32x8_b4096"
L2_BYTES = 126 * 1000 * 1000


def metric_for(w):
    """The headline metric for the 1M-token workload; the same measurement on
    any other workload is named by that workload."""
    if w.name == DEFAULT_WORKLOAD:
        return METRIC
    return (f"MoBA prefill fwd ms and effective TFLOP/s (% bf16 peak) on {w.name} "
            f"({w.total_tokens} tokens), 1 B200")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------------------
# algorithmic work (closed forms of the attended-key count)
# ------------------------------------------------------------------------------------
def work(seqlens, Hq, d, B, topk):
    """Flops of the whole forward, of the past-block part and of the own-block part.

    A query in block j attends t - jB + 1 keys of its own block and
    min(topk - 1, j) full past blocks of B keys; each attended key costs 4 d
    flops (one multiply-add in QK^T, one in PV).
    """
    past_keys = own_keys = 0
    for L in seqlens:
        nb = (L + B - 1) // B
        for j in range(nb):
            n = min(B, L - j * B)
            own_keys += n * (n + 1) // 2
            past_keys += n * min(topk - 1, j) * B
    f = 4 * d * Hq
    return f * (past_keys + own_keys), f * past_keys, f * own_keys


def max_over_ranks(ms: float, world: int, device) -> float:
    """Slowest rank's time: every rank's number goes through one MAX all-reduce."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, flops_per_replica: int, ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs a full replica of the workload."""
    return world * flops_per_replica / (ms * 1e-3) / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
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
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------
# CPU oracle on a bounded sample (test infrastructure, timed as a baseline)
# ------------------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, x, n_rows, seed, pooled=None):
    """Run the CPU oracle on n_rows sampled rows of workload w.

    Returns (flops of the rows, seconds for the rows, seconds of the one-time
    block pooling, pooled means cache).  Pooling serves every row of the
    sequence; callers amortise it over all T * Hq rows.
    """
    import numpy as np
    import torch
    import synth
    from oracle import moba_ref as R

    def bits(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    cu = w.cu_seqlens()
    rows = synth.sample_rows(w, n_rows, seed)
    pooled = {} if pooled is None else pooled
    t_pool = 0.0
    t_rows = 0.0
    flops = 0
    B, topk, d = w.block_size, w.topk, w.head_dim
    seq_of = np.searchsorted(np.asarray(cu), [r[0] for r in rows], side="right") - 1
    for s in sorted(set(seq_of.tolist())):
        a, b = cu[s], cu[s + 1]
        if s not in pooled:
            ks, vs = bits(x["k"][a:b]), bits(x["v"][a:b])
            t = time.perf_counter()
            kbar = R.block_means(ks, B)
            t_pool += time.perf_counter() - t
            pooled[s] = (ks, vs, kbar)
        ks, vs, kbar = pooled[s]
        sel = [i for i in range(len(rows)) if seq_of[i] == s]
        tl = [rows[i][0] - a for i in sel]
        hh = [rows[i][1] for i in sel]
        tq = torch.tensor([rows[i][0] for i in sel], device=x["q"].device)
        th = torch.tensor(hh, device=x["q"].device)
        qr = bits(x["q"][tq, th])
        t = time.perf_counter()
        R.forward_rows(qr, tl, hh, ks, vs, w.n_heads, w.n_kv_heads, B, topk, kbar=kbar)
        t_rows += time.perf_counter() - t
        flops += sum(4 * d * R.attended_keys(u, B, topk) for u in tl)
    return flops, t_rows, t_pool, pooled


def cpu_baseline(w, x, n_rows, seed):
    flops, t_rows, t_pool, _ = oracle_sample(w, x, n_rows, seed)
    total_rows = w.total_tokens * w.n_heads
    t = t_rows + t_pool * n_rows / total_rows
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": (f"{n_rows} seeded (token, head) rows of the workload through the fp64 "
                       f"NumPy oracle (gate + masked attention): {t_rows:.1f} s; the one-time "
                       f"block pooling of the sequence ({t_pool:.1f} s) amortised over all "
                       f"{total_rows} rows")}


# ------------------------------------------------------------------------------------
# reference arm: the oracle, on the machine's host cores
# ------------------------------------------------------------------------------------
def run_reference(args, w):
    import torch
    import synth

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = synth.make_inputs(w, dev)
    total_rows = w.total_tokens * w.n_heads
    rows_per_step = args.ref_rows
    pooled = {}
    t0 = time.perf_counter()
    _, _, t_pool, pooled = oracle_sample(w, x, rows_per_step, 1000, pooled)
    for i in range(args.warmup):
        oracle_sample(w, x, rows_per_step, 2000 + i, pooled)
    flops = 0
    t_rows = 0.0
    for i in range(args.steps):
        f, tr, _, _ = oracle_sample(w, x, rows_per_step, 3000 + i, pooled)
        flops += f
        t_rows += tr
    n = args.steps * rows_per_step
    t = t_rows + t_pool * n / total_rows
    value = flops / t / 1e12
    ms_per_step = 1e3 * t / args.steps
    line = {
        "impl": "reference", "metric": metric_for(w), "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "tokens": w.total_tokens, "n_heads": w.n_heads,
                   "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
                   "block_size": w.block_size, "topk": w.topk,
                   "sample_rows_per_step": rows_per_step},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": (f"{rows_per_step} seeded rows per step through the fp64 "
                                    f"NumPy oracle; block pooling ({t_pool:.1f} s, once) "
                                    f"amortised over all {total_rows} rows")},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": time.perf_counter() - t0,
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------
# the other side of the full <-> sparse switch: dense causal attention
# ------------------------------------------------------------------------------------
def run_full(args, w, x, dev, world, rank, local, barrier):
    import torch
    import block_sparse_long_11_b200 as mb
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    T, Hq, d = q.shape
    flops = 4 * d * Hq * sum(L * (L + 1) // 2 for L in w.seqlens)
    ws = mb.Workspace()
    out = torch.empty_like(q)
    lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        mb.moba_forward_full(q, k, v, cu, workspace=ws, out=out, lse=lse)
    mb.moba_check(ws)
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        mb.moba_forward_full(q, k, v, cu, workspace=ws, out=out, lse=lse)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    mb.moba_check(ws)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    value = job_value(world, flops, ms)
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    per_gpu = flops / (ms * 1e-3) / 1e12
    if rank == 0:
        print(json.dumps({
            "metric": "dense causal attention fwd (moba_forward_full), effective TFLOP/s",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "tokens": T, "n_seqs": len(w.seqlens), "n_heads": Hq,
                       "n_kv_heads": w.n_kv_heads, "head_dim": d, "mode": "full causal",
                       "l2": "inputs larger than L2", "parallelism": "single" if world == 1
                       else f"replicas{world}"},
            "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel (full mode)",
                         "achieved": per_gpu, "peak": peak, "unit": "TFLOP/s",
                         "frac": per_gpu / peak, "traffic": None,
                         "peak_source": peak_src + " bf16_tflops_sustained",
                         "flops_per_step": flops},
            "gpu_launches": args.steps * 2,
            "clocks": clk,
        }))
        sys.stdout.flush()


# ------------------------------------------------------------------------------------
# decode: one new token per sequence against a cache of the workload's length
# ------------------------------------------------------------------------------------
def run_decode(args, w, dev, world, rank, local, barrier):
    import numpy as np
    import torch
    import block_sparse_long_11_b200 as mb
    import synth
    n, B, topk = args.decode, w.block_size, w.topk
    Hq, Hkv, d = w.n_heads, w.n_kv_heads, w.head_dim
    max_len = w.seqlens[0]
    L = max_len - 7 if max_len % B == 0 else max_len  # no block completes during the timed steps
    x = synth.make_decode(n, max_len, Hq, Hkv, d, w.seed, dev)
    sl = torch.full((n,), L, dtype=torch.int32, device=dev)
    ws = mb.Workspace()
    kbar = mb.moba_decode_init(x["k_cache"], sl, B, workspace=ws)
    out = torch.empty_like(x["q"])
    lse = torch.empty((n, Hq), dtype=torch.float32, device=dev)
    idx = torch.empty((n, Hq, topk), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        mb.moba_decode(x["q"], x["k_cache"], x["v_cache"], sl, kbar, B, topk, workspace=ws,
                       out=out, lse=lse, idx=idx)

    for _ in range(args.warmup):
        step()
    mb.moba_check(ws)
    # algorithmic bytes of one step: K and V of every distinct selected
    # (sequence, kv head, block) -- the heads of a group share a block's reads
    # -- plus the block means the gate reads, q, and the outputs
    sel = idx.cpu().numpy()
    G = Hq // Hkv
    t = L - 1
    nbytes = 0
    for s_ in range(n):
        for g in range(Hkv):
            blocks = set(int(b) for b in sel[s_, g * G:(g + 1) * G].ravel() if b >= 0)
            for b in blocks:
                nbytes += 2 * d * 2 * (min(B, t + 1 - b * B))
    nbytes += n * Hkv * (t // B) * d * 4 + n * Hq * d * 2 * 2 + n * Hq * 4
    # enough steps for about a second of timed work (clock samples every 200 ms)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(10):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    est = max(e0.elapsed_time(e1) / 10, 1e-3)
    steps = max(args.steps, int(1000.0 / est))
    if world > 1:  # every rank runs the same number of steps
        t_ = torch.tensor([steps], device=dev)
        torch.distributed.all_reduce(t_, op=torch.distributed.ReduceOp.MAX)
        steps = int(t_.item())
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    mb.moba_check(ws)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    peaks, peak_src = load_peaks()
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    gbs = nbytes / (ms * 1e-3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "MoBA decode step (one new token per sequence) ms and HBM GB/s",
            "value": gbs * world, "unit": "GB/s", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"decode_{n}x{L}_gqa{Hq}x{Hkv}_b{B}", "n_seqs": n,
                       "context": L, "n_heads": Hq, "n_kv_heads": Hkv, "head_dim": d,
                       "block_size": B, "topk": topk,
                       "l2": "selected K/V far larger than L2", "parallelism": "single"
                       if world == 1 else f"replicas{world}"},
            "roofline": {"bound": "hbm", "kernel": "decode (gate + attention + merge)",
                         "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": None, "peak_source": peak_src + " hbm_gbs",
                         "bytes_per_step": nbytes},
            "gpu_launches": steps * 3,
            "clocks": clk,
        }))
        sys.stdout.flush()


# ------------------------------------------------------------------------------------
# backward (selection of the forward held fixed), on the tensor cores
# ------------------------------------------------------------------------------------
def run_backward(args, w, dev, world, rank, local, barrier):
    import torch
    import block_sparse_long_11_b200 as mb
    import synth
    L = args.backward
    wb, x = synth.make_custom([L], w.n_heads, w.n_kv_heads, w.head_dim, w.block_size, w.topk,
                              seed=w.seed, device=dev)
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    T, Hq, d = q.shape
    dout = synth.normal_bf16((T, Hq, d), w.seed, 50, dev)
    out, lse, idx = mb.moba_forward(q, k, v, cu, w.block_size, w.topk, return_idx=True)
    fwd_flops, _, _ = work([L], Hq, d, w.block_size, w.topk)
    # the five products of the definition (q.k again, dout.v, dv, dk, dq): 10 d per attended key
    flops = fwd_flops * 10 // 4
    ws = mb.Workspace()
    stream = torch.cuda.current_stream(dev)

    def step():
        return mb.moba_backward(q, k, v, out, lse, dout, cu, idx, w.block_size, w.topk,
                                workspace=ws)

    for _ in range(args.warmup):
        step()
    mb.moba_check(ws)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    mb.moba_check(ws)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    per_gpu = flops / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    if rank == 0:
        print(json.dumps({
            "metric": "MoBA backward (selection fixed) ms and effective TFLOP/s",
            "value": per_gpu * world, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 (fp32 gradients)",
            "data": "synthetic",
            "config": {"workload": f"backward_1x{L}_gqa{Hq}x{w.n_kv_heads}_b{w.block_size}",
                       "tokens": L, "n_heads": Hq, "n_kv_heads": w.n_kv_heads, "head_dim": d,
                       "block_size": w.block_size, "topk": w.topk, "parallelism": "single"
                       if world == 1 else f"replicas{world}"},
            "roofline": {"bound": "tensor",
                         "kernel": "dkv_tc_kernel + dq_tc_kernel (tcgen05) and the row passes",
                         "achieved": per_gpu, "peak": peak, "unit": "TFLOP/s",
                         "frac": per_gpu / peak, "traffic": None,
                         "peak_source": peak_src + " bf16_tflops_sustained",
                         "flops_per_step": flops},
            "gpu_launches": args.steps * backward_launches(L, Hq, d, w.topk),
            "clocks": clk,
        }))
        sys.stdout.flush()


def backward_launches(T, Hq, d, topk):
    """Kernels one moba_backward launches: plan, the prep pass, the stable
    scheduler (5), a pack + dK/dV pair per chunk of packed entries (every
    entry when the packed rows fit in 8 GiB), and per dQ chunk (the binding's
    choice) the scheduler (4), dQ and the slot sum."""
    entries = T * Hq * (topk - 1)
    cap = max(64, min(entries, (8 << 30) // (4 * d + 8)))
    n_dkv = max(1, -(-entries // cap))
    from block_sparse_long_11_b200 import _lib
    per_token = Hq * topk * d * 4
    n_dq = max(1, -(-T * per_token // _lib.BWD_PARTIAL_BUDGET_BYTES))
    return 2 + 5 + 2 * n_dkv + 6 * n_dq


# ------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=48)
    ap.add_argument("--ref-rows", type=int, default=16)
    ap.add_argument("--full", action="store_true",
                    help="time dense causal attention (moba_forward_full) on the workload instead")
    ap.add_argument("--backward", type=int, default=0, metavar="TOKENS",
                    help="time the backward on one sequence of TOKENS tokens with the "
                         "workload's heads, block and top-k instead")
    ap.add_argument("--decode", type=int, default=0, metavar="N",
                    help="time decode steps of N sequences whose context is the workload's "
                         "first sequence length instead")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)

    import synth
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
        return

    import torch
    import torch.distributed as dist
    import block_sparse_long_11_b200 as mb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    if args.decode:
        run_decode(args, w, dev, world, rank, local, barrier)
        return
    if args.backward:
        run_backward(args, w, dev, world, rank, local, barrier)
        return
    x = synth.make_inputs(w, dev)
    if args.full:
        run_full(args, w, x, dev, world, rank, local, barrier)
        return
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    T, Hq, d = q.shape
    flops, past_flops, own_flops = work(w.seqlens, Hq, d, w.block_size, w.topk)
    chunk = mb.default_chunk_tokens(T, Hq, d, w.topk)
    n_chunks = 1 if chunk == 0 else -(-T // chunk)
    n_ev = 2 + 3 * n_chunks
    ws = mb.Workspace()
    out = torch.empty_like(q)
    lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def make_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record(stream)
        return evs

    def step(evs=None):
        mb.moba_forward(q, k, v, cu, w.block_size, w.topk, chunk_tokens=chunk, workspace=ws,
                        out=out, lse=lse, stage_events=evs)

    # inputs that fit in L2 are flushed from it before every timed step (a
    # write of twice its size, outside the step's events)
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    flush = (torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
             if in_bytes < 2 * L2_BYTES else None)
    l2_note = (f"inputs larger than L2 (q + k + v {in_bytes / 1e9:.2f} GB vs 126 MB)"
               if flush is None else
               f"L2 flushed before every step (q + k + v {in_bytes / 1e6:.1f} MB fit in L2)")
    for _ in range(args.warmup):
        step()
    mb.moba_check(ws)
    step_events = [make_events(n_ev) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if flush is None:
        t_start.record(stream)
        for i in range(args.steps):
            step(step_events[i])
        t_end.record(stream)
    else:
        for i in range(args.steps):
            flush.zero_()
            step(step_events[i])
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    mb.moba_check(ws)
    if flush is None:
        ms = t_start.elapsed_time(t_end) / args.steps
    else:  # first to last stage event of each step
        ms = sum(ev[0].elapsed_time(ev[-1]) for ev in step_events) / args.steps
    # per-stage times (ms per step, averaged over the timed steps)
    stage = {"gate_prefix": 0.0, "sched": 0.0, "attn": 0.0, "merge": 0.0}
    for evs in step_events:
        stage["gate_prefix"] += evs[0].elapsed_time(evs[1])
        prev = evs[1]
        for c in range(n_chunks):
            e = evs[2 + 3 * c:5 + 3 * c]
            stage["sched"] += prev.elapsed_time(e[0])
            stage["attn"] += e[0].elapsed_time(e[1])
            stage["merge"] += e[1].elapsed_time(e[2])
            prev = e[2]
    stage = {kk: vv / args.steps for kk, vv in stage.items()}
    ms = max_over_ranks(ms, world, dev)
    value = job_value(world, flops, ms)

    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    achieved = flops / (stage["attn"] * 1e-3) / 1e12 if stage["attn"] > 0 else 0.0
    traffic = measured_traffic(w.name)

    # ---- end to end: pinned host buffers, copies inside the timed region -----------
    # Every step copies its inputs host -> device and its result device -> host.
    # The steps are pipelined over three streams with two device buffer sets:
    # step i's input copy runs while step i - 1 computes, and step i - 1's
    # result copy runs while step i computes (PCIe is full duplex).  The timed
    # region spans every copy of every timed step, fill and drain included.
    e2e = None
    if not args.no_e2e:
        hq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
        hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
        hcu = torch.empty(cu.shape, dtype=cu.dtype, pin_memory=True)
        ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        hq.copy_(q)
        hk.copy_(k)
        hv.copy_(v)
        hcu.copy_(cu)
        # buffer set 0 reuses the benchmark's own device tensors (the copies
        # write the same values back); set 1 is allocated here
        dins = [(q, k, v, cu), (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                                torch.empty_like(cu))]
        douts = [(out, lse), (torch.empty_like(out), torch.empty_like(lse))]
        s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        in_free = [torch.cuda.Event() for _ in range(2)]    # compute done with the inputs
        in_ready = [torch.cuda.Event() for _ in range(2)]   # inputs copied
        out_free = [torch.cuda.Event() for _ in range(2)]   # result copied out
        for e in in_free + out_free:
            e.record(stream)

        def e2e_steps(n):
            for i in range(n):
                b = i % 2
                dq_, dk_, dv_, dcu_ = dins[b]
                do_, dl_ = douts[b]
                with torch.cuda.stream(s_in):
                    s_in.wait_event(in_free[b])
                    dq_.copy_(hq, non_blocking=True)
                    dk_.copy_(hk, non_blocking=True)
                    dv_.copy_(hv, non_blocking=True)
                    dcu_.copy_(hcu, non_blocking=True)
                    in_ready[b].record(s_in)
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(in_ready[b])
                    s_comp.wait_event(out_free[b])
                    mb.moba_forward(dq_, dk_, dv_, dcu_, w.block_size, w.topk, chunk_tokens=chunk,
                                    workspace=ws, out=do_, lse=dl_)
                    in_free[b].record(s_comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(in_free[b])
                    ho.copy_(do_, non_blocking=True)
                    hl.copy_(dl_, non_blocking=True)
                    out_free[b].record(s_out)

        e2e_steps(2)
        torch.cuda.synchronize(dev)
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b_ = torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, args.steps)  # the device-timed step count (at least 3)
        a.record(s_in)
        s_comp.wait_event(a)
        s_out.wait_event(a)
        e2e_steps(n_e2e)
        s_out.wait_event(in_free[(n_e2e - 1) % 2])
        b_.record(s_out)
        torch.cuda.synchronize(dev)
        barrier()
        mb.moba_check(ws)
        ms_e2e = a.elapsed_time(b_) / n_e2e
        ms_e2e = max_over_ranks(ms_e2e, world, dev)
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hcu))
        d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
        e2e = {"value": job_value(world, flops, ms_e2e), "unit": "TFLOP/s",
               "ms_per_step": ms_e2e, "steps": n_e2e, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "pipelined": "two device buffer sets, copies in and out overlap the "
                            "neighbouring steps' compute"}
        del hq, hk, hv, ho, hl, dins, douts

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, x, args.cpu_rows, 4242)

    if rank == 0:
        line = {
            "metric": metric_for(w), "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": w.name, "tokens": T, "n_seqs": w.n_seqs, "n_heads": Hq,
                       "n_kv_heads": w.n_kv_heads, "head_dim": d, "block_size": w.block_size,
                       "topk": w.topk, "query_chunks": n_chunks,
                       "l2": l2_note,
                       "parallelism": "replicas" if world > 1 else "single"},
            "pct_bf16_peak": {"burst": 100 * value / world / peaks.get("bf16_tflops", 1633.5),
                              "sustained": 100 * value / world / peak},
            "stages_ms": stage,
            "roofline": {"bound": "tensor", "kernel": "block attention (tcgen05, past + own blocks)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16_tflops_sustained",
                         "flops_per_step": flops, "past_block_flops": past_flops,
                         "own_block_flops": own_flops, "launches_per_step": n_chunks},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * (4 + 6 * n_chunks),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# DRAM bytes per attention launch from the committed ncu summary, valid only
# while the kernel source is the one that summary was taken with.
TRAFFIC_SUMMARY = "attn_tc_kernel_65k_gqa32x8_b4096.md"
TRAFFIC_KERNEL_HASH = "a88005b282e1f8b2"  # csrc the summary was captured with


def measured_traffic(workload):
    p = os.path.join(ROOT, "profiles", TRAFFIC_SUMMARY)
    if not os.path.exists(p) or TRAFFIC_KERNEL_HASH != _kernel_hash():
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if ":" in line and line.split(":")[0].startswith("traffic_"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    if vals.get("traffic_workload") != workload:
        return None
    return int(vals["traffic_bytes_per_launch"])


def _kernel_hash():
    """Hash of the sources the block attention kernel is built from."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_long_11_b200", "csrc")
    for n in ("attn_tc.cu", "tc_ptx.cuh", "common.cuh"):
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    main()
