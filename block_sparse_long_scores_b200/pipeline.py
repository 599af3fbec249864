"""The MSA hot path end to end on device tensors: index scores -> top-k -> sparse attention.

This module only allocates buffers (torch) and calls the four C-ABI entry points in order,
chunking prefill rows so that the score buffer and the attention workspace stay bounded.
Every arithmetic step runs in the library's kernels.
"""
from __future__ import annotations

import torch

from . import msa
from .workloads import Workload


def _ceil4(x: int) -> int:
    return (x + 3) // 4 * 4


class Prefill:
    """Packed prefill of workload `w` on inputs `x` (device tensors from workloads.make_inputs).

    With `fused` (the default) the index branch is one call per row chunk (msa_index_topk: scores
    and selection without a score buffer); otherwise msa_index_scores writes the chunk's scores and
    msa_select_topk selects from them."""

    def __init__(self, w: Workload, x: dict, chunk_rows: int | None = None, with_lse: bool = True,
                 fused: bool = True):
        assert w.mode == "prefill"
        self.w, self.x = w, x
        dev = x["q"].device
        self.cfg = msa.make_config(w.Hq, w.Hkv, w.D, w.B, w.d, w.n_topk, w.use_sink)
        self.cu_seqlens = x["cu_seqlens"].to(dev, torch.int32).contiguous()
        self.cu_blocks = x["cu_blocks"].to(dev, torch.int32).contiguous()
        self.shape = msa.prefill_shape(self.cu_seqlens, self.cu_blocks, list(w.seqlens), w.B)
        T, nblk = self.shape.total_rows, self.shape.total_blocks
        self.stride = _ceil4(self.shape.max_blocks)
        self.chunk = T if chunk_rows is None else max(1, min(chunk_rows, T))
        self.given_kidx = "k_idx" in x
        self.k_idx = x["k_idx"] if self.given_kidx else torch.empty(nblk, w.Hkv, w.d, dtype=torch.bfloat16, device=dev)
        self.fused = fused
        self._scores = None
        self.block_idx = torch.empty(T, w.Hkv, w.k_tot, dtype=torch.int32, device=dev)
        self.o = torch.empty(T, w.Hq, w.D, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(T, w.Hq, dtype=torch.float32, device=dev) if with_lse else None
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        # one attention call may cover every row: the library works in sub-chunks and needs at most
        # two sub-chunks' workspace (enough for any smaller call as well)
        ws = msa.msa_sparse_attn_prefill(self.cfg, self.shape, None, None, None, None, 0, T, None, None, None)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)

    @property
    def scores(self) -> torch.Tensor:
        """Score buffer of one row chunk (allocated on first use: the fused path needs none)."""
        if self._scores is None:
            self._scores = torch.empty(self.chunk, self.w.Hkv, self.stride, dtype=torch.float32,
                                       device=self.x["q"].device)
        return self._scores

    def chunks(self):
        T = self.shape.total_rows
        for r0 in range(0, T, self.chunk):
            yield r0, min(T, r0 + self.chunk)

    def index(self, r0: int, r1: int, compute_keys: bool, q_idx_out=None):
        x = self.x
        k = None if (self.given_kidx or not compute_keys) else x["k"]
        msa.msa_index_scores(self.cfg, self.shape, x["q"], k, x["wq"], x["wk"], self.k_idx, 0, r0, r1,
                             self.scores, self.stride, q_idx_out)

    def select(self, r0: int, r1: int):
        msa.msa_select_topk(self.cfg, self.shape, self.scores, self.stride, r0, r1, self.block_idx[r0:r1], self.err)

    def index_select(self, r0: int, r1: int, compute_keys: bool, block_idx=None, q_idx_out=None):
        """Fused index branch for rows [r0, r1) into block_idx (default: this pass's own)."""
        x = self.x
        k = None if (self.given_kidx or not compute_keys) else x["k"]
        out = self.block_idx[r0:r1] if block_idx is None else block_idx
        msa.msa_index_topk(self.cfg, self.shape, x["q"], k, x["wq"], x["wk"], self.k_idx, 0, r0, r1, out,
                           q_idx_out, self.err)

    def _index_branch(self, r0: int, r1: int, first: bool):
        if self.fused:
            self.index_select(r0, r1, compute_keys=first)
        else:
            self.index(r0, r1, compute_keys=first)
            self.select(r0, r1)

    def attend(self, r0: int, r1: int):
        x = self.x
        msa.msa_sparse_attn_prefill(self.cfg, self.shape, x["q"], x["k"], x["v"], self.block_idx[r0:r1], r0, r1,
                                    self.o, self.lse, self.workspace, self.err)

    def run(self):
        """One pass of the whole hot path over every row.  The fused index branch needs no score
        buffer and the attention call works through its rows in sub-chunks (overlapping each
        sub-chunk's combine with the next one's attention), so both are one call over all rows."""
        if self.fused:
            T = self.shape.total_rows
            self.index_select(0, T, compute_keys=True)
            self.attend(0, T)
            return self.o, self.lse
        first = True
        for r0, r1 in self.chunks():
            self._index_branch(r0, r1, first)
            first = False
            self.attend(r0, r1)
        return self.o, self.lse

    def run_from_host(self, host: dict, o_host: torch.Tensor, lse_host: torch.Tensor | None = None):
        """One pass of the hot path whose inputs start in (pinned) host memory and whose outputs end
        there.  K, V, W_q and W_k are copied first; then each row chunk's queries are copied on a
        copy stream while the previous chunk computes, and each chunk's O (and lse) rows go back on
        a second copy stream as soon as the chunk is done.  Returns once everything is enqueued; the
        caller's current stream waits for the last copy back."""
        cur = torch.cuda.current_stream()
        if not hasattr(self, "_h2d"):
            self._h2d, self._d2h = torch.cuda.Stream(), torch.cuda.Stream()
        h2d, d2h = self._h2d, self._d2h
        x = self.x
        h2d.wait_stream(cur)        # the previous pass may still read the device inputs
        d2h.wait_stream(cur)
        ready = []
        with torch.cuda.stream(h2d):
            for name in ("k", "v", "wq", "wk"):
                x[name].copy_(host[name], non_blocking=True)
            for r0, r1 in self.chunks():
                x["q"][r0:r1].copy_(host["q"][r0:r1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(h2d)
                ready.append(ev)
        first = True
        for c, (r0, r1) in enumerate(self.chunks()):
            cur.wait_event(ready[c])
            self._index_branch(r0, r1, first)
            first = False
            self.attend(r0, r1)
            done = torch.cuda.Event()
            done.record(cur)
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                o_host[r0:r1].copy_(self.o[r0:r1], non_blocking=True)
                if lse_host is not None and self.lse is not None:
                    lse_host[r0:r1].copy_(self.lse[r0:r1], non_blocking=True)
        cur.wait_stream(d2h)
        return o_host, lse_host


class Decode:
    """One decode step of workload `w`: the new token of every sequence against its cache."""

    def __init__(self, w: Workload, x: dict, with_lse: bool = True):
        assert w.mode == "decode"
        self.w, self.x = w, x
        dev = x["q"].device
        self.cfg = msa.make_config(w.Hq, w.Hkv, w.D, w.B, w.d, w.n_topk, w.use_sink)
        self.seqlens = x["seqlens"].to(dev, torch.int32).contiguous()
        Lmax = x["k"].shape[2]
        self.shape = msa.decode_shape(self.seqlens, w.batch, Lmax, w.B)
        self.stride = _ceil4(self.shape.max_blocks)
        self.given_kidx = "k_idx" in x
        self.k_idx = (x["k_idx"] if self.given_kidx else
                      torch.empty(w.batch, w.Hkv, self.shape.max_blocks, w.d, dtype=torch.bfloat16, device=dev))
        self.scores = torch.empty(w.batch, w.Hkv, self.stride, dtype=torch.float32, device=dev)
        self.block_idx = torch.empty(w.batch, w.Hkv, w.k_tot, dtype=torch.int32, device=dev)
        self.o = torch.empty(w.batch, w.Hq, w.D, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(w.batch, w.Hq, dtype=torch.float32, device=dev) if with_lse else None
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        ws = msa.msa_sparse_attn_decode(self.cfg, self.shape, None, None, None, None, None, None, None)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
        self.keys_ready = self.given_kidx

    def prepare_keys(self):
        """Block keys of the whole cache (kept by the caller between steps)."""
        x = self.x
        msa.msa_index_scores(self.cfg, self.shape, x["q"], x["k"], x["wq"], x["wk"], self.k_idx, 0, 0, 0,
                             self.scores, self.stride)
        self.keys_ready = True

    def graph(self, q_idx_out=None):
        """Capture one decode step (newest block key -> index scores -> selection -> attention) in
        a CUDA graph and return its replay function.  Every replay reads the same input tensors
        (refresh them in place between steps: new queries, the new tokens' K/V in the cache, the
        advanced seqlens) and writes the same outputs; the kernels inside are chained with
        programmatic dependent launch."""
        if not self.keys_ready:
            self.prepare_keys()
        self.run(q_idx_out)        # first call: per-kernel attributes set outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run(q_idx_out)
        self._graph = g
        return g.replay

    def run(self, q_idx_out=None):
        """One decode step.  Unless the block keys were given, the step first refreshes the key of
        each sequence's newest block (the block the new token belongs to), so a loop that appends
        one token per sequence per step -- writing its K/V into the cache and advancing `seqlens` in
        place -- keeps the key cache current, also under CUDA graph replay."""
        x = self.x
        if not self.keys_ready:
            self.prepare_keys()
        if self.given_kidx:
            msa.msa_index_scores(self.cfg, self.shape, x["q"], None, x["wq"], None, self.k_idx, 0, 0,
                                 self.w.batch, self.scores, self.stride, q_idx_out)
        else:
            msa.msa_index_scores(self.cfg, self.shape, x["q"], x["k"], x["wq"], x["wk"], self.k_idx,
                                 msa.MSA_KIDX_NEWEST_BLOCK, 0, self.w.batch, self.scores, self.stride, q_idx_out)
        msa.msa_select_topk(self.cfg, self.shape, self.scores, self.stride, 0, self.w.batch, self.block_idx, self.err)
        msa.msa_sparse_attn_decode(self.cfg, self.shape, x["q"], x["k"], x["v"], self.block_idx, self.o, self.lse,
                                   self.workspace, self.err)
        return self.o, self.lse
