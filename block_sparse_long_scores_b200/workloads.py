"""Named MSA workloads and their seeded synthetic inputs.

This module only describes shapes and draws random numbers; it holds none of MSA's arithmetic,
so both the CUDA path and the fp64 oracle can be fed from it without sharing any computation.

Inputs are drawn with a torch Generator seeded per workload, in the fixed order
Q, K, V, W_q, W_k (then the discrete index keys, when a workload asks for them), as
``randn(float32) * std`` rounded to bf16.  The pages use no dataset for this path; every
input is synthetic, shaped like the long-context GQA workloads the pages discuss (128K-1M tokens,
GQA groups of 4-8 heads).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str                      # "prefill" or "decode"
    Hq: int
    Hkv: int
    D: int
    B: int                         # KV block size (tokens)
    d: int                         # index dimension
    n_topk: int                    # scored picks per (row, group); local (and sink) come on top
    use_sink: int                  # 1: block 0 is always kept
    seqlens: tuple                 # prefill: sequence lengths; decode: cache lengths (incl. new token)
    std_q: float
    std_kv: float
    std_w: float
    discrete_kidx: int = 0         # >0: k_idx rows drawn from this many fixed vectors per KV head
    seed: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def k_tot(self) -> int:
        return self.n_topk + 1 + self.use_sink

    @property
    def batch(self) -> int:
        return len(self.seqlens)

    @property
    def total_rows(self) -> int:
        return sum(self.seqlens) if self.mode == "prefill" else len(self.seqlens)

    @property
    def max_seqlen(self) -> int:
        return max(self.seqlens)

    @property
    def max_blocks(self) -> int:
        return (self.max_seqlen + self.B - 1) // self.B

    def cu_seqlens(self) -> torch.Tensor:
        return torch.tensor([0] + list(_cumsum(self.seqlens)), dtype=torch.int32)

    def cu_blocks(self) -> torch.Tensor:
        nb = [(l + self.B - 1) // self.B for l in self.seqlens]
        return torch.tensor([0] + list(_cumsum(nb)), dtype=torch.int32)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _cumsum(xs):
    acc = 0
    for x in xs:
        acc += x
        yield acc


def ragged_lengths(n: int, lo: int, hi: int, seed: int) -> tuple:
    g = torch.Generator().manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g))


_S128 = 1.0 / math.sqrt(128)

WORKLOADS = {
    # Tiny MSA prefill: 1 x 2048, 8/2 heads, D 128, B 64, top-k 8 incl. local -> 7 scored picks.
    "tiny_prefill": Workload("tiny_prefill", "prefill", 8, 2, 128, 64, 64, 7, 0, (2048,),
                             _S128, _S128, _S128),
    # MSA prefill 128K: 32/4 heads, D 128, B 64, 64 picks + sink + local.
    "prefill_128k": Workload("prefill_128k", "prefill", 32, 4, 128, 64, 64, 64, 1, (131072,),
                             _S128, _S128, _S128),
    # MSA decode at 128K: batch 32, cache 131072 each, cache and q ~N(0,1).
    "decode_128k": Workload("decode_128k", "decode", 32, 4, 128, 64, 64, 64, 1, (131072,) * 32,
                            1.0, 1.0, _S128),
    # MSA at 1M: prefill of one 1,048,576-token sequence, 128 picks + sink + local ...
    "prefill_1m": Workload("prefill_1m", "prefill", 32, 4, 128, 64, 64, 128, 1, (1 << 20,),
                           _S128, _S128, _S128),
    # ... and decode batch 8 over a 1M-token cache.
    "decode_1m": Workload("decode_1m", "decode", 32, 4, 128, 64, 64, 128, 1, (1 << 20,) * 8,
                          1.0, 1.0, _S128),
    # Ragged stress: 16 sequences, lengths uniform in [1K, 256K], 64/8 heads, D 64, B 128,
    # 32 picks, index keys from 8 discrete vectors (forces score ties).
    "ragged_prefill": Workload("ragged_prefill", "prefill", 64, 8, 64, 128, 64, 32, 0,
                               ragged_lengths(16, 1024, 262144, 0), 0.125, 0.125, 0.125,
                               discrete_kidx=8),
    "ragged_decode": Workload("ragged_decode", "decode", 64, 8, 64, 128, 64, 32, 0,
                              ragged_lengths(16, 1024, 262144, 0), 1.0, 1.0, 0.125,
                              discrete_kidx=8),
}


def scaled_down(w: Workload, seqlens: tuple, name: str | None = None) -> Workload:
    """Same heads/blocks/selection as `w`, other lengths (for parity sizes the oracle finishes)."""
    return replace(w, seqlens=tuple(seqlens), name=name or f"{w.name}@{sum(seqlens)}")


def _randn(shape, std, g, device):
    x = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    return (x * std).to(torch.bfloat16)


def make_inputs(w: Workload, device="cpu", seed: int | None = None, logit_gain: float = 1.0) -> dict:
    """Seeded inputs for workload `w` on `device`.

    prefill: q [T,Hq,D], k/v [T,Hkv,D] (packed over cu_seqlens)
    decode:  q [batch,Hq,D], k/v cache [batch,Hkv,Lmax,D] (Lmax = max cache length)
    both:    wq, wk [D,d]; optional k_idx (discrete workloads) in the library's k_idx layout.
    `logit_gain` multiplies the std of q and k (sharp-logit variants).
    """
    seed = w.seed if seed is None else seed
    g = torch.Generator(device=device).manual_seed(seed)
    sq, skv = w.std_q * logit_gain, w.std_kv * logit_gain
    out = {}
    if w.mode == "prefill":
        T = w.total_rows
        out["q"] = _randn((T, w.Hq, w.D), sq, g, device)
        out["k"] = _randn((T, w.Hkv, w.D), skv, g, device)
        out["v"] = _randn((T, w.Hkv, w.D), w.std_kv, g, device)
    else:
        Lmax = w.max_seqlen
        out["q"] = _randn((w.batch, w.Hq, w.D), sq, g, device)
        out["k"] = _randn((w.batch, w.Hkv, Lmax, w.D), skv, g, device)
        out["v"] = _randn((w.batch, w.Hkv, Lmax, w.D), w.std_kv, g, device)
    out["wq"] = _randn((w.D, w.d), w.std_w, g, device)
    out["wk"] = _randn((w.D, w.d), w.std_w, g, device)
    if w.discrete_kidx:
        # one of `discrete_kidx` fixed bf16 vectors per KV head for every block row
        vecs = _randn((w.Hkv, w.discrete_kidx, w.d), 1.0 / math.sqrt(w.d), g, device)
        if w.mode == "prefill":
            nblk = int(w.cu_blocks()[-1])
            pick = torch.randint(0, w.discrete_kidx, (nblk, w.Hkv), generator=g, device=device)
            heads = torch.arange(w.Hkv, device=device).expand(nblk, w.Hkv)
            out["k_idx"] = vecs[heads, pick].contiguous()                 # [nblk, Hkv, d]
        else:
            mb = w.max_blocks
            pick = torch.randint(0, w.discrete_kidx, (w.batch, w.Hkv, mb), generator=g, device=device)
            heads = torch.arange(w.Hkv, device=device).view(1, w.Hkv, 1).expand(w.batch, w.Hkv, mb)
            out["k_idx"] = vecs[heads, pick].contiguous()                 # [batch, Hkv, mb, d]
    if w.mode == "prefill":
        out["cu_seqlens"] = w.cu_seqlens().to(device)
        out["cu_blocks"] = w.cu_blocks().to(device)
    else:
        out["seqlens"] = torch.tensor(w.seqlens, dtype=torch.int32, device=device)
    return out
