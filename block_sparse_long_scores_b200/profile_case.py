"""Run one named workload a few times with no timing, as the target of a profiler.

    python -m block_sparse_long_scores_b200.profile_case decode_128k --seq-len 16384 --steps 2
    python -m block_sparse_long_scores_b200.profile_case prefill_128k --seq-len 32768 --chunk-rows 4096
    python -m block_sparse_long_scores_b200.profile_case prefill_128k --seq-len 32768 --dense --steps 1
    python -m block_sparse_long_scores_b200.profile_case prefill_128k --seq-len 32768 --backward --steps 1

A prefill workload runs whole prefill steps (index -> selection -> attention -> combine in
chunks); a decode workload prepares the cache's block keys once and then runs decode steps;
`--dense` runs the dense causal GQA baseline on the same inputs instead; `--backward` runs one
prefill step and then the attention backward (dQ, dK, dV for a seeded dO) `--steps` times.
`--seq-len` shortens every sequence (the decode work per step -- batch x kv heads x selected
blocks -- does not depend on it, so a short cache keeps a capture's device memory small);
`--batch` changes the number of decode sequences.  Inputs are the workload's seeded synthetic
tensors.  The process exits non-zero if a kernel reported a device-side error flag.
"""
from __future__ import annotations

import argparse
import sys

import torch

from .pipeline import Decode, Prefill
from .workloads import WORKLOADS, make_inputs, scaled_down


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("workload", choices=sorted(WORKLOADS))
    ap.add_argument("--seq-len", type=int, default=0)
    ap.add_argument("--batch", type=int, default=0)
    ap.add_argument("--chunk-rows", type=int, default=16384)
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--unfused", action="store_true", help="prefill: index scores + top-k as two calls")
    ap.add_argument("--dense", action="store_true", help="the dense causal GQA baseline instead of MSA")
    ap.add_argument("--backward", action="store_true", help="prefill: the attention backward after one step")
    ap.add_argument("--subchunk-rows", type=int, default=0,
                    help="prefill attention sub-chunk rows (smaller: a smaller workspace)")
    a = ap.parse_args(argv)
    w = WORKLOADS[a.workload]
    if w.mode == "decode" and (a.seq_len or a.batch):
        n = a.batch or w.batch
        w = w.with_(seqlens=(a.seq_len or w.max_seqlen,) * n)
    elif a.seq_len:
        w = scaled_down(w, (a.seq_len,))
    if a.subchunk_rows:
        from . import msa
        msa.prefill_set_subchunk_rows(a.subchunk_rows)
    x = make_inputs(w, device="cuda")
    if w.mode == "prefill":
        job = Prefill(w, x, chunk_rows=a.chunk_rows, fused=not a.unfused)
    else:
        job = Decode(w, x)
        job.prepare_keys()
    if a.dense:
        from . import msa
        job.workspace = None           # the sparse path's workspace is not needed
        torch.cuda.empty_cache()
        o, lse = torch.empty_like(job.o), torch.empty_like(job.lse)
        if w.mode == "prefill":
            run = lambda: msa.msa_dense_attn_prefill(job.cfg, job.shape, x["q"], x["k"], x["v"], 0,
                                                     job.shape.total_rows, o, lse, job.err)
        else:
            n = msa.msa_dense_attn_decode(job.cfg, job.shape, None, None, None, None, None, None)
            ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
            run = lambda: msa.msa_dense_attn_decode(job.cfg, job.shape, x["q"], x["k"], x["v"], o, lse, ws, job.err)
    elif a.backward and w.mode == "prefill":
        from . import msa
        job.run()
        job.workspace = None           # the forward's workspace is not needed
        torch.cuda.empty_cache()
        T = job.shape.total_rows
        gen = torch.Generator(device="cuda").manual_seed(7)
        d_o = (torch.randn(job.o.shape, generator=gen, device="cuda") * 0.05).to(torch.bfloat16)
        dq = torch.zeros(T, w.Hq, w.D, dtype=torch.float32, device="cuda")
        dk = torch.zeros(T, w.Hkv, w.D, dtype=torch.float32, device="cuda")
        dv = torch.zeros_like(dk)
        n = msa.msa_sparse_attn_prefill_bwd(job.cfg, job.shape, None, None, None, None, None, None, None, 0, T,
                                            None, None, None, None)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
        run = lambda: msa.msa_sparse_attn_prefill_bwd(job.cfg, job.shape, x["q"], x["k"], x["v"], job.o, job.lse,
                                                      d_o, job.block_idx, 0, T, dq, dk, dv, ws, job.err)
    else:
        run = job.run
    for _ in range(a.steps):
        run()
    torch.cuda.synchronize()
    err = int(job.err.item())
    print(f"{w.name}: {a.steps} steps, rows {job.shape.total_rows}, device error flag {err}")
    return 1 if err else 0


if __name__ == "__main__":
    sys.exit(main())
