"""Shared helpers of the GPU parity tests: run the oracle on the same seeded inputs and compare.

Tolerances (fixed for the MSA hot path):
* block selection: bit-exact, given the GPU's own fp32 index scores;
* index scores: row-relative 1e-3 -- max_j |S_gpu - S_ref| <= 1e-3 * max_j |S_ref| over each
  (row, group)'s candidates;
* attention output (bf16, fp32 accumulation): max-abs 1e-2 and relative L2 5e-3 against fp64;
* log-sum-exp: 1e-3 absolute (derived: fp32 accumulation over <= 10^4 terms plus bf16 inputs
  keeps the error near 1e-5; 1e-3 leaves margin for the exp2/log2 approximations).
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as orc

ATOL_O = 1e-2
RL2_O = 5e-3
ATOL_LSE = 1e-3
RTOL_SCORES = 1e-3


def oracle_shape(w, x):
    if w.mode == "prefill":
        return orc.prefill_shape(x["cu_seqlens"].cpu().numpy(), w.Hq, w.Hkv, w.D, w.B, w.d, w.n_topk, w.use_sink)
    Lmax = x["k"].shape[2]
    return orc.decode_shape(x["seqlens"].cpu().numpy(), Lmax, (Lmax + w.B - 1) // w.B, w.Hq, w.Hkv, w.D, w.B,
                            w.d, w.n_topk, w.use_sink)


def cpu(x: dict) -> dict:
    return {k: v.cpu() for k, v in x.items()}


def row_geometry(w, x, rows):
    """(in-sequence position, local block) of each row."""
    if w.mode == "prefill":
        cu = x["cu_seqlens"].cpu().numpy()
        b = np.searchsorted(cu, rows, side="right") - 1
        pos = np.asarray(rows) - cu[b]
    else:
        pos = x["seqlens"].cpu().numpy()[np.asarray(rows)] - 1
    return pos, pos // w.B


def check_scores(w, x, rows, S_gpu, S_ref):
    """Row-relative comparison over each row's candidate range [use_sink, i)."""
    _, i = row_geometry(w, x, rows)
    worst = 0.0
    for a in range(len(rows)):
        lo, hi = w.use_sink, int(i[a])
        if hi <= lo:
            continue
        ref = S_ref[a, :, lo:hi]
        got = S_gpu[a, :, lo:hi].astype(np.float64)
        scale = np.abs(ref).max(axis=1, keepdims=True)
        scale[scale == 0] = 1.0
        worst = max(worst, float((np.abs(got - ref) / scale).max()))
    assert worst <= RTOL_SCORES, f"index scores off by {worst:.3e} (row-relative)"
    return worst


def check_attention(O_gpu, O_ref, L_gpu=None, L_ref=None):
    O_gpu = O_gpu.astype(np.float64)
    err = np.abs(O_gpu - O_ref)
    max_abs = float(err.max()) if err.size else 0.0
    rl2 = float(np.linalg.norm(O_gpu - O_ref) / max(np.linalg.norm(O_ref), 1e-300))
    assert max_abs <= ATOL_O, f"O max-abs error {max_abs:.3e} > {ATOL_O}"
    assert rl2 <= RL2_O, f"O relative L2 error {rl2:.3e} > {RL2_O}"
    lse_err = 0.0
    if L_gpu is not None:
        lse_err = float(np.abs(L_gpu.astype(np.float64) - L_ref).max())
        assert lse_err <= ATOL_LSE, f"lse error {lse_err:.3e} > {ATOL_LSE}"
    return max_abs, rl2, lse_err


def check_bf16_near(gpu_bits: np.ndarray, ref_f64: np.ndarray, what: str):
    """GPU bf16 value is the bf16 nearest to the fp64 value, or its neighbour (fp32 vs fp64
    accumulation can move a value across a rounding boundary).  A value that cancels to near zero
    carries the fp32 accumulation error in absolute terms, hence the small absolute floor
    (1e-6 of the largest value)."""
    g = orc.bf16_bits_to_f64(gpu_bits)
    mag = np.maximum(np.abs(ref_f64), 1e-30)
    ulp = np.exp2(np.floor(np.log2(mag)) - 7)
    floor = 1e-6 * float(np.abs(ref_f64).max()) if ref_f64.size else 0.0
    bad = np.abs(g - ref_f64) > 1.5 * ulp + floor
    assert not bad.any(), f"{what}: {int(bad.sum())} values more than one bf16 step away"
    near = orc.round_bf16(ref_f64)
    return float(np.mean(near != gpu_bits))


def sample_rows(w, n: int, seed: int = 0):
    """First and last 64 rows of every sequence plus random rows (for full-size parity)."""
    rng = np.random.default_rng(seed)
    if w.mode == "decode":
        return np.arange(w.batch)
    cu = np.concatenate([[0], np.cumsum(w.seqlens)])
    rows = set()
    for b in range(len(w.seqlens)):
        s0, s1 = cu[b], cu[b + 1]
        rows.update(range(s0, min(s1, s0 + 64)))
        rows.update(range(max(s0, s1 - 64), s1))
    extra = rng.integers(0, cu[-1], size=max(0, n - len(rows)))
    rows.update(int(r) for r in extra)
    return np.array(sorted(rows), dtype=np.int64)


class Guards:
    """Guard bands after device buffers: a guarded tensor is a view of a larger allocation whose
    tail holds a byte pattern; check() asserts that no call wrote past the tensor (or past the
    workspace size the library reported)."""

    PATTERN = 0xA5

    def __init__(self, tail_bytes: int = 4096):
        self.tail = tail_bytes
        self.items = []

    def wrap(self, t: torch.Tensor, name: str = "") -> torch.Tensor:
        nb = t.numel() * t.element_size()
        raw = torch.empty(nb + self.tail, dtype=torch.uint8, device=t.device)
        raw[nb:] = self.PATTERN
        if nb:
            raw[:nb].copy_(t.contiguous().view(-1).view(torch.uint8))
        self.items.append((name, raw, nb))
        return raw[:nb].view(t.dtype).view(t.shape)

    def guard(self, obj, *names: str):
        """Replace the listed tensor attributes of obj with guarded copies."""
        for n in names:
            t = getattr(obj, n)
            if t is not None:
                setattr(obj, n, self.wrap(t, n))

    def check(self):
        torch.cuda.synchronize()
        for name, raw, nb in self.items:
            bad = int((raw[nb:] != self.PATTERN).sum().item())
            assert bad == 0, f"{bad} guard bytes after '{name}' were overwritten"
