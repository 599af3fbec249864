"""Run one named workload a few times with no timing, as the target of a profiler.

    python -m block_sparse_long_scores_b200.profile_case decode_128k --seq-len 16384 --steps 2
    python -m block_sparse_long_scores_b200.profile_case prefill_128k --seq-len 32768 --chunk-rows 4096

A prefill workload runs whole prefill steps (index -> selection -> attention -> combine in
chunks); a decode workload prepares the cache's block keys once and then runs decode steps.
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
    a = ap.parse_args(argv)
    w = WORKLOADS[a.workload]
    if w.mode == "decode" and (a.seq_len or a.batch):
        n = a.batch or w.batch
        w = w.with_(seqlens=(a.seq_len or w.max_seqlen,) * n)
    elif a.seq_len:
        w = scaled_down(w, (a.seq_len,))
    x = make_inputs(w, device="cuda")
    if w.mode == "prefill":
        job = Prefill(w, x, chunk_rows=a.chunk_rows, fused=not a.unfused)
    else:
        job = Decode(w, x)
        job.prepare_keys()
    for _ in range(a.steps):
        job.run()
    torch.cuda.synchronize()
    err = int(job.err.item())
    print(f"{w.name}: {a.steps} steps, rows {job.shape.total_rows}, device error flag {err}")
    return 1 if err else 0


if __name__ == "__main__":
    sys.exit(main())
