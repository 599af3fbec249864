#!/usr/bin/env python
"""Throughput of the MSA hot path on B200: one JSON line per run.

A step is one pass of the whole prefill hot path over one 131072-token sequence (32 query / 4 KV
heads, head dim 128, 64-token blocks, top-k 64 + sink + local, index dim 64): block keys, index
scores, per-group top-k, block-sparse attention and its split-softmax combine, in row chunks.
Inputs are synthetic (seeded normal bf16, the shapes the pages' long-context GQA workloads use)
and larger than L2 (Q alone is 1.07 GB), so no flush is needed between prefill steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (one independent sequence per rank)

Besides the headline line items, the line carries:
  roofline      the dominant kernel (sparse prefill attention, tensor-bound): selected-block FLOPs
                per launch / its launch time from CUDA events recorded around it in the timed region
  cpu_baseline  the fp64 CPU oracle on a bounded sample of rows of the same workload (rank 0, N=1)
  e2e           the same step from pinned host buffers to pinned host buffers (Q/K/V/W in, O/lse
                out), chunk copies overlapping other chunks' compute
  secondary     decode at 128K and 1M (whole step, and the attention kernel against the HBM roofline
                on selected-block bytes), prefill at 1M, the ragged prefill and decode workloads, and
                the dense causal GQA baselines at 128K and 1M with the sparse path's speed-up over
                them; with its own clock record (--quick skips the 1M and ragged workloads)
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MSA prefill & decode tokens/s at 128K/1M ctx; % of HBM/tensor roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_128k")
    ap.add_argument("--chunk-rows", type=int, default=16384)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU oracle sample budget")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--quick", action="store_true", help="skip the 1M-token and ragged workloads")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense GQA baselines")
    ap.add_argument("--seq-len", type=int, default=0, help="scaled-down sequence (profiling captures)")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


# ------------------------------------------------------------------------------ environment


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_for(kernel: str, source: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this exact source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    with open(os.path.join(ROOT, source), "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()[:16]
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 3 and not line.startswith("#") and parts[0] == kernel:
                return float(parts[2]) if parts[1] == digest else None
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.gpu_id, self.proc, self.file = gpu_id, None, None

    def start(self):
        if not shutil.which("nvidia-smi"):
            return
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu_id}", "--query-gpu=" + ",".join(self.FIELDS),
                                      "--format=csv,noheader,nounits", "-lms", "100"],
                                     stdout=self.file, stderr=subprocess.DEVNULL)

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.file.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.file.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------ helpers


class Dist:
    """One process per GPU (torchrun); NCCL on GPUs, gloo for the CPU tests of this logic."""

    def __init__(self, n_gpus: int, backend: str | None = None):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.on = self.world > 1
        self.backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        self.device = torch.device("cuda", self.local) if self.backend == "nccl" else torch.device("cpu")
        if self.backend == "nccl":
            torch.cuda.set_device(self.local)
        if self.on:
            kw = {"device_id": self.device} if self.backend == "nccl" else {}
            torch.distributed.init_process_group(self.backend, timeout=datetime.timedelta(seconds=300), **kw)

    def barrier(self):
        if self.on:
            torch.distributed.barrier()

    def max(self, v: float) -> float:
        """Largest value over ranks (device times are reported as the slowest rank's)."""
        if not self.on:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.on:
            torch.distributed.destroy_process_group()


def throughput(world: int, rows_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank's rows over the slowest rank's time (weak scaling)."""
    return world * rows_per_rank * steps / (ms_max / 1000.0)


def gpu_id(dist: Dist) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if dist.local < len(ids):
            return ids[dist.local]
    return str(dist.local)


L2_NOTE = "256 MB written, then another 256 MB read, between steps (L2 holds none of the step's data)"


def l2_flusher():
    """Flush L2 between timed steps: write a 256 MB buffer (2x L2), then read another one so the
    written lines are evicted before the step starts."""
    a = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    b = torch.zeros(32 << 20, dtype=torch.int64, device="cuda")

    def flush():
        a.fill_(1)
        b.sum()
    return flush


def graph_of(fn):
    """fn captured once in a CUDA graph (after one eager call)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def timed(fn, steps: int, warmup: int, dist: Dist, between=None) -> float:
    """Device milliseconds for `steps` calls of fn (CUDA events on the current stream), max over
    ranks.  `between`, if given, runs before every step outside the events (an L2 flush)."""
    for _ in range(warmup):
        if between:
            between()
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    total = 0.0
    if between is None:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        total = a.elapsed_time(b)
    else:
        for _ in range(steps):
            between()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            total += a.elapsed_time(b)
    dist.barrier()
    torch.cuda.synchronize()
    return dist.max(total)


def selected_flops(pf) -> float:
    """Selected-block attention FLOPs of a prefill (4 * D per query head and visible key): full
    blocks count B keys, each row's local block only its causal part."""
    w = pf.w
    bi = pf.block_idx
    valid = int((bi >= 0).sum().item())
    T = pf.shape.total_rows
    cu = pf.cu_seqlens.to(torch.int64)
    rows = torch.arange(T, device=bi.device)
    seq = torch.searchsorted(cu[1:], rows, right=True)
    pos = rows - cu[seq]
    local_keys = int(((pos % w.B) + 1).sum().item()) * w.Hkv
    full = valid - T * w.Hkv
    keys = full * w.B + local_keys
    return 4.0 * w.D * w.G * keys


def dense_flops(w) -> float:
    total = 0
    for L in w.seqlens:
        total += L * (L + 1) // 2
    return 4.0 * w.D * w.Hq * total


def decode_selected_bytes(dc) -> float:
    """K+V bytes of the selected blocks of one decode step (partial local blocks count their valid rows)."""
    w = dc.w
    bi = dc.block_idx
    sl = dc.seqlens.to(torch.int64).view(-1, 1, 1)
    j = bi.to(torch.int64)
    rows = torch.clamp(sl - j * w.B, 0, w.B)
    rows = torch.where(j >= 0, rows, torch.zeros_like(rows))
    return float(rows.sum().item()) * w.D * 2 * 2


# ------------------------------------------------------------------------------ CPU oracle


def oracle_sample(w, x_cpu, seconds: float, seed: int = 0):
    """Run the fp64 oracle's whole path on randomly sampled rows for about `seconds`; returns
    (tokens per second, rows, threads)."""
    import numpy as np
    from oracle import oracle as orc

    threads = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(threads))
    sh = orc.prefill_shape(x_cpu["cu_seqlens"].numpy(), w.Hq, w.Hkv, w.D, w.B, w.d, w.n_topk, w.use_sink)
    T = sh.T
    t0 = time.perf_counter()
    kidx, _ = orc.block_keys(sh, x_cpu["k"], x_cpu["wk"])
    t_keys = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    ncols = (w.max_blocks + 3) // 4 * 4
    done, spent = 0, 0.0
    batch = 8
    while spent < seconds:
        rows = np.sort(rng.integers(0, T, size=batch))
        t0 = time.perf_counter()
        q_idx, _ = orc.index_query(sh, x_cpu["q"], x_cpu["wq"], rows)
        S = orc.index_scores(sh, q_idx, kidx, rows, ncols)
        sel = orc.select_topk_f64(sh, S, rows)
        orc.sparse_attn(sh, x_cpu["q"], x_cpu["k"], x_cpu["v"], sel, rows)
        spent += time.perf_counter() - t0
        done += batch
        batch = min(batch * 2, 256)
    per_row = spent / done + t_keys / T
    return 1.0 / per_row, done, threads


def reference_arm(args, dist: Dist):
    """The oracle as the reference implementation, timed on the host cores (rank 0 only)."""
    from block_sparse_long_scores_b200.workloads import WORKLOADS, make_inputs

    if dist.rank != 0:
        dist.close()
        return
    w = WORKLOADS[args.workload]
    x = make_inputs(w, device="cpu")
    per_step = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, x, per_step / 4)
    vals, rows_total = [], 0
    t0 = time.perf_counter()
    for s in range(args.steps):
        v, n, threads = oracle_sample(w, x, per_step, seed=s + 1)
        vals.append(v)
        rows_total += n
    wall = time.perf_counter() - t0
    value = statistics.median(vals)
    sample = f"{rows_total} random rows of {w.name} over {args.steps} steps (~{per_step:.0f} s each), block keys of all blocks"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall * 1000 / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, w.total_rows, min(args.chunk_rows, w.total_rows), dist.world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    dist.close()


# ------------------------------------------------------------------------------ our arm


def main():
    args = parse_args()
    dist = Dist(args.gpus)
    if args.impl == "reference":
        return reference_arm(args, dist)

    from block_sparse_long_scores_b200 import msa
    from block_sparse_long_scores_b200.pipeline import Decode, Prefill
    from block_sparse_long_scores_b200.workloads import WORKLOADS, make_inputs, scaled_down

    pk, pk_kind = peaks()
    w = WORKLOADS[args.workload]
    if args.seq_len:
        w = scaled_down(w, (args.seq_len,))
    x = make_inputs(w, device="cuda", seed=dist.rank)
    pf = Prefill(w, x, chunk_rows=args.chunk_rows)
    T = pf.shape.total_rows
    clocks = ClockSampler(gpu_id(dist))

    # --- headline: inputs resident in HBM.  Inside the timed region only the dominant kernel is
    # bracketed by CUDA events (for the roofline); the per-family split comes from a separate pass.
    clocks.start()
    for _ in range(args.warmup):
        pf.run()
    torch.cuda.synchronize()
    msa.profile_reset()
    msa.profile_only("prefill_attn")
    msa.profile_enable(True)
    n0 = msa.launch_count()
    ms = timed(pf.run, args.steps, 0, dist)
    launches = msa.launch_count() - n0
    msa.profile_enable(False)
    msa.profile_only(None)
    attn_ms, attn_n = msa.profile_read("prefill_attn")
    msa.profile_reset()
    fam = family_split(msa, pf)
    flops = selected_flops(pf)
    ms_step = ms / args.steps
    value = throughput(dist.world, T, args.steps, ms)
    attn_launch_ms = attn_ms / max(1, attn_n)
    flops_per_launch = flops / max(1, attn_n // args.steps)
    achieved = flops_per_launch / (attn_launch_ms / 1000.0) / 1e12
    peak = float(pk["bf16_tflops_sustained"])
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                # the committed figure is per launch of the default workload's 16384-row chunks
                "traffic": (traffic_for("prefill_attn_128k", "block_sparse_long_scores_b200/csrc/attn_prefill.cu")
                            if (w.name == "prefill_128k" and pf.chunk == 16384) else None),
                "kernel": "sparse_prefill_attn_kernel", "launches_per_step": attn_n // args.steps,
                "peak_kind": f"{pk_kind} bf16 sustained", "flops_per_step": flops}
    step_tflops = flops / (ms_step / 1000.0) / 1e12

    # --- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(args, dist, pf, x, T)
    clk = clocks.stop()

    chunk = pf.chunk
    # --- CPU oracle baseline (rank 0, N=1 only)
    cpu_baseline = None
    if dist.world == 1 and args.cpu_seconds > 0:
        xc = {k: v.cpu() for k, v in x.items()}
        v, n, threads = oracle_sample(w, xc, args.cpu_seconds)
        cpu_baseline = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                        "sample": f"{n} random rows of {w.name} (whole path per row: index query, scores, "
                                  f"top-k, attention) plus block keys of all {pf.shape.total_blocks} blocks "
                                  f"amortised per row, fp64, ~{args.cpu_seconds:.0f} s"}
        del xc

    # --- secondary: decode 128K, 1M, ragged and the dense baselines (rank 0 reports, every rank
    # runs), with their own clock record
    secondary = {}
    if not args.no_secondary:
        sec_clocks = ClockSampler(gpu_id(dist))
        sec_clocks.start()
        secondary = secondary_measurements(args, dist, pf, x, ms_step, pk)
        del pf, x
        torch.cuda.empty_cache()
        if not args.quick:
            secondary.update(one_million(args, dist, pk))
            secondary.update(ragged(args, dist, pk))
        secondary["clocks"] = sec_clocks.stop()

    emit(args, dist, w, T, chunk, value, ms_step, roofline, cpu_baseline, e2e, launches, clk, step_tflops, fam,
         secondary)
    dist.close()


def family_split(msa, job) -> dict:
    """Milliseconds per kernel family of one untimed eager pass of a prefill or decode step (every
    launch bracketed by events)."""
    torch.cuda.synchronize()
    msa.profile_reset()
    msa.profile_enable(True)
    job.run()
    torch.cuda.synchronize()
    msa.profile_enable(False)
    fam = {}
    for f in ("block_keys", "index_scores", "select_topk", "index_topk", "prefill_lists", "prefill_attn",
              "prefill_combine", "decode_attn", "prefill_bwd"):
        t, n = msa.profile_read(f)
        if n:
            fam[f] = round(t, 3)
    msa.profile_reset()
    return fam


def end_to_end(args, dist, pf, x, T):
    """The same step from pinned host buffers to pinned host buffers (Prefill.run_from_host: chunk
    copies overlap the computation of other chunks)."""
    host = {k: v.cpu().pin_memory() for k, v in x.items() if k in ("q", "k", "v", "wq", "wk")}
    o_host = torch.empty(pf.o.shape, dtype=pf.o.dtype, pin_memory=True)
    lse_host = torch.empty(pf.lse.shape, dtype=pf.lse.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_host.numel() * o_host.element_size() + lse_host.numel() * lse_host.element_size()

    def e2e_step():
        pf.run_from_host(host, o_host, lse_host)

    ms_e2e = timed(e2e_step, args.steps, 1, dist)
    return {"value": throughput(dist.world, T, args.steps, ms_e2e), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e / args.steps,
            "overlap": "per-chunk query copies and output copies overlap other chunks' compute"}


def workload_config(w, T: int, chunk: int, world: int) -> dict:
    """The `config` object of both arms' JSON lines."""
    return {"workload": f"{w.name}: {len(w.seqlens)} x {T // len(w.seqlens)} tokens"
                        f"{' (ragged)' if len(set(w.seqlens)) > 1 else ''}, {w.Hq} q / {w.Hkv} kv heads, "
                        f"D {w.D}, block {w.B}, top-k {w.n_topk}{' + sink' if w.use_sink else ''} + local, "
                        f"index dim {w.d}",
            "global_batch": world, "seq_len": T, "chunk_rows": chunk,
            "l2": f"inputs exceed L2 (Q {T * w.Hq * w.D * 2 / 1e9:.2f} GB read per step); no flush",
            "parallelism": f"dp{world} (one independent sequence per rank)"}


def emit(args, dist, w, T, chunk, value, ms_step, roofline, cpu_baseline, e2e, launches, clk, step_tflops, fam,
         secondary):
    if dist.rank != 0:
        return
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": dist.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, T, chunk, dist.world),
            "roofline": roofline, "cpu_baseline": cpu_baseline, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk, "step_tflops_selected": step_tflops, "kernel_ms_one_step": fam,
            "secondary": secondary}
    print(json.dumps(line), flush=True)


def secondary_measurements(args, dist, pf, x, sparse_ms, pk):
    from block_sparse_long_scores_b200 import msa
    from block_sparse_long_scores_b200.pipeline import Decode
    from block_sparse_long_scores_b200.workloads import WORKLOADS, make_inputs

    out = {}
    # dense causal GQA prefill over the same 128K sequence
    if not args.no_dense:
        od = torch.empty_like(pf.o)
        ld = torch.empty_like(pf.lse)
        T = pf.shape.total_rows
        ms_dense = timed(lambda: msa.msa_dense_attn_prefill(pf.cfg, pf.shape, x["q"], x["k"], x["v"], 0, T, od, ld),
                         1, 1, dist)
        out["dense_prefill_128k"] = {"ms": ms_dense, "tflops": dense_flops(pf.w) / (ms_dense / 1000) / 1e12,
                                     "speedup_of_sparse_step": ms_dense / sparse_ms}
        del od, ld
    out["backward_128k"] = backward(dist, pf, x, pk)
    # decode at 128K: batch 32, each step replayed from a CUDA graph, L2 flushed between steps
    wd = WORKLOADS["decode_128k"]
    xd = make_inputs(wd, device="cuda", seed=100 + dist.rank)
    dc = Decode(wd, xd)
    dc.prepare_keys()
    between = l2_flusher()
    step = dc.graph()
    ms = timed(step, 20, 3, dist, between=between)
    attn = graph_of(lambda: msa.msa_sparse_attn_decode(dc.cfg, dc.shape, xd["q"], xd["k"], xd["v"], dc.block_idx,
                                                       dc.o, dc.lse, dc.workspace, dc.err))
    a_ms_launch = timed(attn.replay, 20, 3, dist, between=between) / 20
    sel_bytes = decode_selected_bytes(dc)
    gbs = sel_bytes / (a_ms_launch / 1000) / 1e9
    between()
    out["decode_128k"] = {"tokens_per_s": dist.world * wd.batch * 20 / (ms / 1000), "ms_per_step": ms / 20,
                          "attn_ms": a_ms_launch, "selected_bytes": sel_bytes, "attn_gbs": gbs,
                          "hbm_frac": gbs / float(pk["hbm_gbs"]), "graph": True, "l2": L2_NOTE,
                          "kernel_ms_one_eager_step": family_split(msa, dc)}
    del attn
    if not args.no_dense:
        ws = msa.msa_dense_attn_decode(dc.cfg, dc.shape, None, None, None, None, None, None)
        wsb = torch.empty(ws, dtype=torch.uint8, device="cuda")
        msd = timed(lambda: msa.msa_dense_attn_decode(dc.cfg, dc.shape, xd["q"], xd["k"], xd["v"], dc.o, dc.lse,
                                                      wsb), 5, 2, dist, between=between)
        dense_bytes = sum(wd.seqlens) * wd.Hkv * wd.D * 4
        out["dense_decode_128k"] = {"ms": msd / 5, "gbs": dense_bytes / (msd / 5 / 1000) / 1e9,
                                    "speedup_of_sparse_attn": (msd / 5) / a_ms_launch}
        del wsb
    del xd, dc
    torch.cuda.empty_cache()
    return out


def backward(dist, pf, x, pk):
    """Gradients of the prefill attention (dQ, dK, dV over the selected blocks, selection fixed) for
    the forward just run: a step zeroes the fp32 gradients and runs msa_sparse_attn_prefill_bwd over
    all rows; dO is seeded N(0, 0.05^2) bf16.  Work = 10 D FLOPs per (query head, visible key): S
    recomputed, dP, dV, dK, dQ (2.5 x the forward's 4 D)."""
    from block_sparse_long_scores_b200 import msa
    w = pf.w
    T = pf.shape.total_rows
    gen = torch.Generator(device="cuda").manual_seed(600 + dist.rank)
    d_o = (torch.randn(pf.o.shape, generator=gen, device="cuda") * 0.05).to(torch.bfloat16)
    dq = torch.zeros(T, w.Hq, w.D, dtype=torch.float32, device="cuda")
    dk = torch.zeros(T, w.Hkv, w.D, dtype=torch.float32, device="cuda")
    dv = torch.zeros_like(dk)
    n = msa.msa_sparse_attn_prefill_bwd(pf.cfg, pf.shape, None, None, None, None, None, None, None, 0, T,
                                        None, None, None, None)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")

    def step():
        dq.zero_()
        dk.zero_()
        dv.zero_()
        msa.msa_sparse_attn_prefill_bwd(pf.cfg, pf.shape, x["q"], x["k"], x["v"], pf.o, pf.lse, d_o, pf.block_idx,
                                        0, T, dq, dk, dv, ws, pf.err)
    ms = timed(step, 3, 1, dist) / 3
    torch.cuda.synchronize()
    msa.profile_reset()
    msa.profile_enable(True)
    step()
    torch.cuda.synchronize()
    msa.profile_enable(False)
    fam = {f: round(msa.profile_read(f)[0], 3) for f in ("prefill_lists", "prefill_bwd")}
    msa.profile_reset()
    flops = 2.5 * selected_flops(pf)
    kern_ms = fam["prefill_bwd"]
    peak = float(pk["bf16_tflops_sustained"])
    out = {"ms": ms, "tokens_per_s": dist.world * T / (ms / 1000), "flops": flops,
           "tflops_step": flops / (ms / 1000) / 1e12, "kernel_ms_one_step": fam,
           "roofline": {"bound": "tensor", "kernel": "sparse_prefill_bwd_kernel (mma.sync)",
                        "achieved": flops / (kern_ms / 1000) / 1e12, "peak": peak, "unit": "TFLOP/s",
                        "frac": flops / (kern_ms / 1000) / 1e12 / peak, "peak_kind": "bf16 sustained"},
           "err": int(pf.err.item()), "finite": bool(torch.isfinite(dq).all().item())}
    del d_o, dq, dk, dv, ws
    torch.cuda.empty_cache()
    return out


def one_million(args, dist, pk):
    from block_sparse_long_scores_b200 import msa
    from block_sparse_long_scores_b200.pipeline import Decode, Prefill
    from block_sparse_long_scores_b200.workloads import WORKLOADS, make_inputs

    out = {}
    w = WORKLOADS["prefill_1m"]
    x = make_inputs(w, device="cuda", seed=200 + dist.rank)
    pf = Prefill(w, x, chunk_rows=args.chunk_rows)
    ms = timed(pf.run, 1, 1, dist)
    flops = selected_flops(pf)
    out["prefill_1m"] = {"ms": ms, "tokens_per_s": dist.world * w.total_rows / (ms / 1000),
                         "tflops_selected": flops / (ms / 1000) / 1e12,
                         "kernel_ms_one_step": family_split(msa, pf)}
    if not args.no_dense:
        od = torch.empty_like(pf.o)
        ld = torch.empty_like(pf.lse)
        T = pf.shape.total_rows
        msd = timed(lambda: msa.msa_dense_attn_prefill(pf.cfg, pf.shape, x["q"], x["k"], x["v"], 0, T, od, ld), 1, 0,
                    dist)
        out["dense_prefill_1m"] = {"ms": msd, "tflops": dense_flops(w) / (msd / 1000) / 1e12,
                                   "speedup_of_sparse": msd / ms}
        del od, ld
    del x, pf
    torch.cuda.empty_cache()
    wd = WORKLOADS["decode_1m"]
    xd = make_inputs(wd, device="cuda", seed=300 + dist.rank)
    dc = Decode(wd, xd)
    dc.prepare_keys()
    between = l2_flusher()
    ms = timed(dc.graph(), 20, 3, dist, between=between)
    attn = graph_of(lambda: msa.msa_sparse_attn_decode(dc.cfg, dc.shape, xd["q"], xd["k"], xd["v"], dc.block_idx,
                                                       dc.o, dc.lse, dc.workspace, dc.err))
    a_ms = timed(attn.replay, 20, 3, dist, between=between) / 20
    sel = decode_selected_bytes(dc)
    between()
    out["decode_1m"] = {"ms_per_step": ms / 20, "tokens_per_s": dist.world * wd.batch * 20 / (ms / 1000),
                        "attn_ms": a_ms, "selected_bytes": sel, "attn_gbs": sel / (a_ms / 1000) / 1e9,
                        "hbm_frac": sel / (a_ms / 1000) / 1e9 / float(pk["hbm_gbs"]), "graph": True, "l2": L2_NOTE,
                        "kernel_ms_one_eager_step": family_split(msa, dc)}
    del attn
    if not args.no_dense:
        ws = msa.msa_dense_attn_decode(dc.cfg, dc.shape, None, None, None, None, None, None)
        wsb = torch.empty(ws, dtype=torch.uint8, device="cuda")
        msd = timed(lambda: msa.msa_dense_attn_decode(dc.cfg, dc.shape, xd["q"], xd["k"], xd["v"], dc.o, dc.lse,
                                                      wsb), 3, 1, dist, between=between)
        out["dense_decode_1m"] = {"ms": msd / 3, "speedup_of_sparse_step": (msd / 3) / (ms / 20)}
    return out


def ragged(args, dist, pk):
    """The ragged workloads: 16 sequences of 1K-256K tokens, 64 q / 8 kv heads, D 64, block 128,
    top-k 32 + local, index keys from 8 discrete vectors (exact score ties)."""
    from block_sparse_long_scores_b200 import msa
    from block_sparse_long_scores_b200.pipeline import Decode, Prefill
    from block_sparse_long_scores_b200.workloads import WORKLOADS, make_inputs

    out = {}
    w = WORKLOADS["ragged_prefill"]
    x = make_inputs(w, device="cuda", seed=400 + dist.rank)
    pf = Prefill(w, x, chunk_rows=args.chunk_rows)
    ms = timed(pf.run, 1, 1, dist)
    flops = selected_flops(pf)
    out["ragged_prefill"] = {"ms": ms, "tokens": pf.shape.total_rows,
                             "tokens_per_s": dist.world * pf.shape.total_rows / (ms / 1000),
                             "tflops_selected": flops / (ms / 1000) / 1e12}
    del x, pf
    torch.cuda.empty_cache()
    wd = WORKLOADS["ragged_decode"]
    xd = make_inputs(wd, device="cuda", seed=500 + dist.rank)
    dc = Decode(wd, xd)   # its block keys are the workload's discrete ones (given, not recomputed)
    between = l2_flusher()
    ms = timed(dc.graph(), 20, 3, dist, between=between)
    attn = graph_of(lambda: msa.msa_sparse_attn_decode(dc.cfg, dc.shape, xd["q"], xd["k"], xd["v"], dc.block_idx,
                                                       dc.o, dc.lse, dc.workspace, dc.err))
    a_ms = timed(attn.replay, 20, 3, dist, between=between) / 20
    sel = decode_selected_bytes(dc)
    out["ragged_decode"] = {"ms_per_step": ms / 20, "tokens_per_s": dist.world * wd.batch * 20 / (ms / 1000),
                            "attn_ms": a_ms, "selected_bytes": sel, "attn_gbs": sel / (a_ms / 1000) / 1e9,
                            "hbm_frac": sel / (a_ms / 1000) / 1e9 / float(pk["hbm_gbs"]), "graph": True,
                            "l2": L2_NOTE}
    del attn, xd, dc
    torch.cuda.empty_cache()
    return out


if __name__ == "__main__":
    main()
