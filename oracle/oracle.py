"""Python face of the fp64 CPU oracle for the MSA hot path (``msa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's CPU-baseline leg
are the only callers.  This module imports nothing from the CUDA package and the CUDA package
imports nothing from here; the two meet only in the tests, on inputs from the seeded generators.

Every function takes torch CPU tensors (bf16 inputs are passed to C as their raw 16-bit
patterns, so widening to double happens exactly, inside the oracle) and returns numpy arrays.
Shapes follow the library's layouts:

* prefill: Q [T, Hq, D], K/V [T, Hkv, D] packed over ``cu_seqlens``; k_idx [nblk, Hkv, d]
  packed over ``cu_blocks``;
* decode: Q [batch, Hq, D], K/V cache [batch, Hkv, Lmax, D]; k_idx [batch, Hkv, max_blocks, d];
* W_q, W_k: [D, d].

Outputs of the row-wise functions are compact over the requested ``rows`` list.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libmsa_oracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, IEEE arithmetic, OpenMP); returns the .so path."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Shape(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("batch", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32), ("B", ctypes.c_int32),
                ("d", ctypes.c_int32), ("n_topk", ctypes.c_int32), ("use_sink", ctypes.c_int32),
                ("_pad", ctypes.c_int32), ("T", ctypes.c_int64), ("Lmax", ctypes.c_int64),
                ("max_blocks", ctypes.c_int64), ("cu_seqlens", ctypes.c_void_p),
                ("cu_blocks", ctypes.c_void_p), ("seqlens", ctypes.c_void_p)]


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
    return _lib


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _bits(t) -> np.ndarray:
    """Raw bf16 bit patterns of a torch bf16 tensor (or pass-through for uint16 numpy)."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    assert t.dtype == torch.bfloat16, t.dtype
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@dataclass
class Shape:
    """Problem shape handed to the oracle (kept alive while the C side holds its pointers)."""
    mode: int                 # 0 prefill, 1 decode
    batch: int
    Hq: int
    Hkv: int
    D: int
    B: int
    d: int
    n_topk: int
    use_sink: int
    T: int = 0
    Lmax: int = 0
    max_blocks: int = 0
    cu_seqlens: np.ndarray | None = None
    cu_blocks: np.ndarray | None = None
    seqlens: np.ndarray | None = None

    @property
    def k_tot(self) -> int:
        return self.n_topk + 1 + self.use_sink

    def c(self) -> _Shape:
        for name in ("cu_seqlens", "cu_blocks", "seqlens"):
            v = getattr(self, name)
            if v is not None:
                setattr(self, name, np.ascontiguousarray(np.asarray(v, dtype=np.int32)))
        s = _Shape(self.mode, self.batch, self.Hq, self.Hkv, self.D, self.B, self.d, self.n_topk,
                   self.use_sink, 0, self.T, self.Lmax, self.max_blocks,
                   _p(self.cu_seqlens) if self.cu_seqlens is not None else None,
                   _p(self.cu_blocks) if self.cu_blocks is not None else None,
                   _p(self.seqlens) if self.seqlens is not None else None)
        return s


def prefill_shape(cu_seqlens, Hq, Hkv, D, B, d, n_topk, use_sink) -> Shape:
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lens = np.diff(cu)
    cu_blocks = np.concatenate([[0], np.cumsum((lens + B - 1) // B)])
    return Shape(0, len(lens), Hq, Hkv, D, B, d, n_topk, use_sink, T=int(cu[-1]),
                 cu_seqlens=cu.astype(np.int32), cu_blocks=cu_blocks.astype(np.int32))


def decode_shape(seqlens, Lmax, max_blocks, Hq, Hkv, D, B, d, n_topk, use_sink) -> Shape:
    sl = np.asarray(seqlens, dtype=np.int32)
    return Shape(1, len(sl), Hq, Hkv, D, B, d, n_topk, use_sink, Lmax=int(Lmax),
                 max_blocks=int(max_blocks), seqlens=sl)


def _rows(rows) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round doubles to bf16 bit patterns (nearest, ties to even, straight from double)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty(x.shape, dtype=np.uint16)
    _check(_L().orc_round_bf16(_p(x), ctypes.c_int64(x.size), _p(out)), "round_bf16")
    return out


def block_keys(shape: Shape, K, Wk, from_block: int = 0, n_blocks_total: int | None = None,
               k_idx_init: np.ndarray | None = None):
    """k_idx (bf16 bits) and khat (fp64, pre-rounding) for every block >= from_block."""
    s = shape.c()
    Kb, Wb = _bits(K), _bits(Wk)
    if shape.mode == 0:
        nblk = int(shape.cu_blocks[-1]) if n_blocks_total is None else n_blocks_total
        out_shape = (nblk, shape.Hkv, shape.d)
    else:
        out_shape = (shape.batch, shape.Hkv, shape.max_blocks, shape.d)
    kidx = np.zeros(out_shape, np.uint16) if k_idx_init is None else np.ascontiguousarray(k_idx_init.copy())
    khat = np.full(out_shape, np.nan)
    _check(_L().orc_block_keys(ctypes.byref(s), _p(Kb), _p(Wb), ctypes.c_int64(from_block),
                               _p(khat), _p(kidx)), "block_keys")
    return kidx, khat


def index_query(shape: Shape, Q, Wq, rows):
    """q_idx (bf16 bits) and qhat (fp64) for the listed rows: [n_rows, Hkv, d]."""
    s = shape.c()
    rows = _rows(rows)
    Qb, Wb = _bits(Q), _bits(Wq)
    q_idx = np.zeros((len(rows), shape.Hkv, shape.d), np.uint16)
    qhat = np.zeros((len(rows), shape.Hkv, shape.d), np.float64)
    _check(_L().orc_index_query(ctypes.byref(s), _p(Qb), _p(Wb), _p(rows), ctypes.c_int64(len(rows)),
                                _p(qhat), _p(q_idx)), "index_query")
    return q_idx, qhat


def index_scores(shape: Shape, q_idx: np.ndarray, k_idx: np.ndarray, rows, ncols: int) -> np.ndarray:
    """fp64 scores [n_rows, Hkv, ncols]; NaN outside each row's candidate range."""
    s = shape.c()
    rows = _rows(rows)
    q_idx = np.ascontiguousarray(q_idx, dtype=np.uint16)
    k_idx = np.ascontiguousarray(k_idx, dtype=np.uint16)
    S = np.empty((len(rows), shape.Hkv, ncols), np.float64)
    _check(_L().orc_index_scores(ctypes.byref(s), _p(q_idx), _p(k_idx), _p(rows),
                                 ctypes.c_int64(len(rows)), ctypes.c_int64(ncols), _p(S)), "index_scores")
    return S


def select_topk_f64(shape: Shape, S: np.ndarray, rows) -> np.ndarray:
    s = shape.c()
    rows = _rows(rows)
    S = np.ascontiguousarray(S, dtype=np.float64)
    out = np.empty((len(rows), shape.Hkv, shape.k_tot), np.int32)
    _check(_L().orc_select_topk_f64(ctypes.byref(s), _p(S), ctypes.c_int64(S.shape[-1]), _p(rows),
                                    ctypes.c_int64(len(rows)), _p(out)), "select_topk_f64")
    return out


def select_topk_f32(shape: Shape, S32: np.ndarray, rows) -> np.ndarray:
    """Selection on fp32 scores (e.g. the GPU's own), compared as floats."""
    s = shape.c()
    rows = _rows(rows)
    S32 = np.ascontiguousarray(S32, dtype=np.float32)
    out = np.empty((len(rows), shape.Hkv, shape.k_tot), np.int32)
    _check(_L().orc_select_topk_f32(ctypes.byref(s), _p(S32), ctypes.c_int64(S32.shape[-1]), _p(rows),
                                    ctypes.c_int64(len(rows)), _p(out)), "select_topk_f32")
    return out


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


def sparse_attn(shape: Shape, Q, K, V, block_idx: np.ndarray, rows, scale: float | None = None):
    """Exact attention over the selected blocks: O [n_rows, Hq, D], LSE [n_rows, Hq] (fp64)."""
    s = shape.c()
    rows = _rows(rows)
    Qb, Kb, Vb = _bits(Q), _bits(K), _bits(V)
    bi = np.ascontiguousarray(block_idx, dtype=np.int32)
    k_tot = bi.shape[-1]
    O = np.empty((len(rows), shape.Hq, shape.D), np.float64)
    LSE = np.empty((len(rows), shape.Hq), np.float64)
    sc = default_scale(shape.D) if scale is None else scale
    _check(_L().orc_sparse_attn(ctypes.byref(s), _p(Qb), _p(Kb), _p(Vb), _p(bi), ctypes.c_int(k_tot),
                                _p(rows), ctypes.c_int64(len(rows)), ctypes.c_double(sc), _p(O), _p(LSE)),
           "sparse_attn")
    return O, LSE


def dense_attn(shape: Shape, Q, K, V, rows, scale: float | None = None):
    """Dense causal GQA attention: O [n_rows, Hq, D], LSE [n_rows, Hq] (fp64)."""
    s = shape.c()
    rows = _rows(rows)
    Qb, Kb, Vb = _bits(Q), _bits(K), _bits(V)
    O = np.empty((len(rows), shape.Hq, shape.D), np.float64)
    LSE = np.empty((len(rows), shape.Hq), np.float64)
    sc = default_scale(shape.D) if scale is None else scale
    _check(_L().orc_dense_attn(ctypes.byref(s), _p(Qb), _p(Kb), _p(Vb), _p(rows), ctypes.c_int64(len(rows)),
                               ctypes.c_double(sc), _p(O), _p(LSE)), "dense_attn")
    return O, LSE


def sparse_attn_bwd(shape: Shape, Q, K, V, dO, block_idx: np.ndarray, scale: float | None = None):
    """Gradients of the selected-block attention for upstream dO (prefill, all rows):
    dQ [T, Hq, D], dK [T, Hkv, D], dV [T, Hkv, D] (fp64)."""
    s = shape.c()
    Qb, Kb, Vb, dOb = _bits(Q), _bits(K), _bits(V), _bits(dO)
    bi = np.ascontiguousarray(block_idx, dtype=np.int32)
    k_tot = bi.shape[-1]
    dQ = np.empty((shape.T, shape.Hq, shape.D), np.float64)
    dK = np.empty((shape.T, shape.Hkv, shape.D), np.float64)
    dV = np.empty((shape.T, shape.Hkv, shape.D), np.float64)
    sc = default_scale(shape.D) if scale is None else scale
    _check(_L().orc_sparse_attn_bwd(ctypes.byref(s), _p(Qb), _p(Kb), _p(Vb), _p(dOb), _p(bi), ctypes.c_int(k_tot),
                                    ctypes.c_double(sc), _p(dQ), _p(dK), _p(dV)), "sparse_attn_bwd")
    return dQ, dK, dV
