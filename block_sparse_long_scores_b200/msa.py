"""ctypes binding of the MSA C ABI (include/msa.h).

Argument marshalling only: every function here forwards device pointers and sizes to the
library and raises :class:`MSAError` on a non-OK status.  There is no CPU fallback: if the
library is missing the first call raises.

Tensors are torch tensors on the current CUDA device; ``stream`` defaults to torch's current
stream.  Layouts and semantics are those of the header (summarised in each docstring).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa_b200.so")

MSA_PREFILL = 0
MSA_DECODE = 1
MSA_KIDX_NEWEST_BLOCK = -1    # kidx_from_block: only each decode sequence's newest block

STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED", 3: "MSA_ERR_WORKSPACE",
          4: "MSA_ERR_CUDA"}
DERR = {1: "BLOCK_RANGE", 2: "DUPLICATE", 4: "NAN_SCORE", 8: "TIMEOUT", 16: "SHAPE"}

EXPORTED = ("msa_index_scores", "msa_select_topk", "msa_sparse_attn_prefill", "msa_sparse_attn_decode",
            "msa_dense_attn_prefill", "msa_dense_attn_decode", "msa_status_string", "msa_version",
            "msa_launch_count", "msa_profile_enable", "msa_profile_reset", "msa_profile_read",
            "msa_sparse_attn_decode_noalloc", "msa_profile_only", "msa_index_topk",
            "msa_prefill_set_subchunk_rows", "msa_prefill_subchunk_rows", "msa_diag_wait_timeout",
            "msa_sparse_attn_prefill_bwd")


class MSAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("index_dim", ctypes.c_int32), ("n_topk", ctypes.c_int32),
                ("use_sink", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]

    @property
    def k_tot(self) -> int:
        return self.n_topk + 1 + self.use_sink


class Shape(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("cu_seqlens", ctypes.c_void_p), ("cu_blocks", ctypes.c_void_p),
                ("seqlens", ctypes.c_void_p), ("total_rows", ctypes.c_int64),
                ("total_blocks", ctypes.c_int64), ("max_seqlen", ctypes.c_int64),
                ("max_blocks", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the library (raises if it has not been built: there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"MSA CUDA library not built: {LIB_PATH} missing "
                              "(run python -m block_sparse_long_scores_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)
        CP, SP = ctypes.POINTER(Config), ctypes.POINTER(Shape)
        sig = {
            "msa_index_scores": [CP, SP, P, P, P, P, P, I64, I64, I64, P, I64, P, P],
            "msa_select_topk": [CP, SP, P, I64, I64, I64, P, P, P],
            "msa_index_topk": [CP, SP, P, P, P, P, P, I64, I64, I64, P, P, P, P],
            "msa_sparse_attn_prefill": [CP, SP, P, P, P, P, I64, I64, P, P, P, SZ, P, P],
            "msa_sparse_attn_decode": [CP, SP, P, P, P, P, P, P, P, SZ, P, P],
            "msa_sparse_attn_prefill_bwd": [CP, SP, P, P, P, P, P, P, P, I64, I64, P, P, P, P, SZ, P, P],
            "msa_dense_attn_prefill": [CP, SP, P, P, P, I64, I64, P, P, P, P],
            "msa_dense_attn_decode": [CP, SP, P, P, P, P, P, P, SZ, P, P],
            "msa_sparse_attn_decode_noalloc": [CP, SP, P, P, P, P, P, P, P, P],
            "msa_diag_wait_timeout": [P, I64, P],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.msa_status_string.argtypes = [ctypes.c_int]
        L.msa_status_string.restype = ctypes.c_char_p
        L.msa_version.restype = I32
        L.msa_launch_count.restype = I64
        L.msa_profile_enable.argtypes = [ctypes.c_int]
        L.msa_profile_enable.restype = None
        L.msa_prefill_set_subchunk_rows.argtypes = [I64]
        L.msa_prefill_set_subchunk_rows.restype = None
        L.msa_prefill_subchunk_rows.argtypes = []
        L.msa_prefill_subchunk_rows.restype = I64
        L.msa_profile_only.argtypes = [ctypes.c_char_p]
        L.msa_profile_only.restype = None
        L.msa_profile_reset.argtypes = []
        L.msa_profile_reset.restype = None
        L.msa_profile_read.argtypes = [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(I64)]
        L.msa_profile_read.restype = I32
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, rc: int):
    if rc != 0:
        raise MSAError(fn, rc)


# ------------------------------------------------------------------------------ descriptors


def make_config(Hq: int, Hkv: int, D: int, B: int, d: int, n_topk: int, use_sink: int,
                softmax_scale: float = 0.0) -> Config:
    return Config(Hq, Hkv, D, B, d, n_topk, use_sink, softmax_scale)


def prefill_shape(cu_seqlens: torch.Tensor, cu_blocks: torch.Tensor, seqlens: list, B: int) -> Shape:
    """Shape of a packed prefill; cu_seqlens/cu_blocks are device int32 tensors (kept alive by
    the caller), `seqlens` the host list of sequence lengths."""
    max_len = max(seqlens)
    total_blocks = sum((l + B - 1) // B for l in seqlens)
    return Shape(MSA_PREFILL, len(seqlens), cu_seqlens.data_ptr(), cu_blocks.data_ptr(), None,
                 sum(seqlens), total_blocks, max_len, (max_len + B - 1) // B)


def decode_shape(seqlens_dev: torch.Tensor, batch: int, Lmax: int, B: int, max_blocks: int | None = None) -> Shape:
    mb = (Lmax + B - 1) // B if max_blocks is None else max_blocks
    return Shape(MSA_DECODE, batch, None, None, seqlens_dev.data_ptr(), batch, 0, Lmax, mb)


# ------------------------------------------------------------------------------ the 4 calls


def msa_index_scores(cfg: Config, shape: Shape, q, k, wq, wk, k_idx, kidx_from_block: int,
                     row_begin: int, row_end: int, scores, scores_row_stride: int,
                     q_idx_out=None, stream=None):
    """Index branch scoring: (optionally) block keys, index queries and raw-logit scores for
    rows [row_begin, row_end) into scores [rows, Hkv, scores_row_stride] (fp32)."""
    rc = lib().msa_index_scores(ctypes.byref(cfg), ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(wq), _ptr(wk),
                                _ptr(k_idx), kidx_from_block, row_begin, row_end, _ptr(scores),
                                scores_row_stride, _ptr(q_idx_out), _stream(stream))
    _check("msa_index_scores", rc)


def msa_select_topk(cfg: Config, shape: Shape, scores, scores_row_stride: int, row_begin: int, row_end: int,
                    block_idx, err_flag=None, stream=None):
    """Per-group exp-free top-k -> block_idx [rows, Hkv, k_tot] (ascending, -1 padded)."""
    rc = lib().msa_select_topk(ctypes.byref(cfg), ctypes.byref(shape), _ptr(scores), scores_row_stride,
                               row_begin, row_end, _ptr(block_idx), _ptr(err_flag), _stream(stream))
    _check("msa_select_topk", rc)


def msa_index_topk(cfg: Config, shape: Shape, q, k, wq, wk, k_idx, kidx_from_block: int, row_begin: int,
                   row_end: int, block_idx, q_idx_out=None, err_flag=None, stream=None):
    """Index scores and per-group top-k in one call (prefill): block_idx [rows, Hkv, k_tot] as
    msa_index_scores + msa_select_topk would give, without a score buffer."""
    rc = lib().msa_index_topk(ctypes.byref(cfg), ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(wq), _ptr(wk),
                              _ptr(k_idx), kidx_from_block, row_begin, row_end, _ptr(block_idx), _ptr(q_idx_out),
                              _ptr(err_flag), _stream(stream))
    _check("msa_index_topk", rc)


def msa_sparse_attn_prefill(cfg: Config, shape: Shape, q, k, v, block_idx, row_begin: int, row_end: int,
                            o, lse, workspace, err_flag=None, stream=None) -> int:
    """Exact attention over the selected blocks for rows [row_begin, row_end).  With
    workspace=None returns the workspace size in bytes (nothing launched)."""
    nbytes = ctypes.c_size_t(0 if workspace is None else workspace.numel() * workspace.element_size())
    rc = lib().msa_sparse_attn_prefill(ctypes.byref(cfg), ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(block_idx), row_begin, row_end, _ptr(o), _ptr(lse),
                                       _ptr(workspace), ctypes.byref(nbytes), _ptr(err_flag), _stream(stream))
    _check("msa_sparse_attn_prefill", rc)
    return nbytes.value


def msa_sparse_attn_prefill_bwd(cfg: Config, shape: Shape, q, k, v, o, lse, d_o, block_idx, row_begin: int,
                                row_end: int, dq, dk, dv, workspace, err_flag=None, stream=None) -> int:
    """Gradients of the prefill attention for rows [row_begin, row_end), accumulated into the fp32
    dq [T, Hq, D], dk and dv [T, Hkv, D].  With workspace=None returns the workspace size."""
    nbytes = ctypes.c_size_t(0 if workspace is None else workspace.numel() * workspace.element_size())
    rc = lib().msa_sparse_attn_prefill_bwd(ctypes.byref(cfg), ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(o), _ptr(lse), _ptr(d_o), _ptr(block_idx), row_begin, row_end,
                                           _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ctypes.byref(nbytes),
                                           _ptr(err_flag), _stream(stream))
    _check("msa_sparse_attn_prefill_bwd", rc)
    return nbytes.value


def msa_sparse_attn_decode(cfg: Config, shape: Shape, q, k_cache, v_cache, block_idx, o, lse, workspace,
                           err_flag=None, stream=None) -> int:
    """Exact attention of each sequence's new token over its selected cache blocks."""
    nbytes = ctypes.c_size_t(0 if workspace is None else workspace.numel() * workspace.element_size())
    rc = lib().msa_sparse_attn_decode(ctypes.byref(cfg), ctypes.byref(shape), _ptr(q), _ptr(k_cache),
                                      _ptr(v_cache), _ptr(block_idx), _ptr(o), _ptr(lse), _ptr(workspace),
                                      ctypes.byref(nbytes), _ptr(err_flag), _stream(stream))
    _check("msa_sparse_attn_decode", rc)
    return nbytes.value


def msa_sparse_attn_decode_noalloc(cfg: Config, shape: Shape, q, k_cache, v_cache, block_idx, o, lse,
                                   err_flag=None, stream=None):
    """msa_sparse_attn_decode without a workspace argument, for callers that cannot allocate:
    scratch comes from the library's fixed 40 MiB device array (include/msa.h gives the limit,
    the first-call set-up and why overlapping calls must be serialised)."""
    rc = lib().msa_sparse_attn_decode_noalloc(ctypes.byref(cfg), ctypes.byref(shape), _ptr(q), _ptr(k_cache),
                                              _ptr(v_cache), _ptr(block_idx), _ptr(o), _ptr(lse), _ptr(err_flag),
                                              _stream(stream))
    _check("msa_sparse_attn_decode_noalloc", rc)


def msa_dense_attn_prefill(cfg: Config, shape: Shape, q, k, v, row_begin: int, row_end: int, o, lse,
                           err_flag=None, stream=None):
    rc = lib().msa_dense_attn_prefill(ctypes.byref(cfg), ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                      row_begin, row_end, _ptr(o), _ptr(lse), _ptr(err_flag), _stream(stream))
    _check("msa_dense_attn_prefill", rc)


def msa_dense_attn_decode(cfg: Config, shape: Shape, q, k_cache, v_cache, o, lse, workspace,
                          err_flag=None, stream=None) -> int:
    nbytes = ctypes.c_size_t(0 if workspace is None else workspace.numel() * workspace.element_size())
    rc = lib().msa_dense_attn_decode(ctypes.byref(cfg), ctypes.byref(shape), _ptr(q), _ptr(k_cache),
                                     _ptr(v_cache), _ptr(o), _ptr(lse), _ptr(workspace), ctypes.byref(nbytes),
                                     _ptr(err_flag), _stream(stream))
    _check("msa_dense_attn_decode", rc)
    return nbytes.value


def diag_wait_timeout(err_flag, limit_ns: int, stream=None):
    """Launch a wait that nothing completes, bounded by limit_ns; it sets MSA_DERR_TIMEOUT."""
    _check("msa_diag_wait_timeout", lib().msa_diag_wait_timeout(_ptr(err_flag), int(limit_ns), _stream(stream)))


def prefill_set_subchunk_rows(rows: int):
    """Rows per internal prefill sub-chunk (<= 0: the default, 16384)."""
    lib().msa_prefill_set_subchunk_rows(int(rows))


def prefill_subchunk_rows() -> int:
    return int(lib().msa_prefill_subchunk_rows())


def launch_count() -> int:
    return int(lib().msa_launch_count())


def profile_enable(on: bool = True):
    lib().msa_profile_enable(1 if on else 0)


def profile_only(family: str | None = None):
    """Bracket only this kernel family while profiling is enabled (None: every family)."""
    lib().msa_profile_only(family.encode() if family else None)


def profile_reset():
    lib().msa_profile_reset()


def profile_read(family: str | None = None):
    """(total milliseconds, launches) of one kernel family since the last reset."""
    ms, n = ctypes.c_double(0.0), ctypes.c_int64(0)
    rc = lib().msa_profile_read(family.encode() if family else None, ctypes.byref(ms), ctypes.byref(n))
    _check("msa_profile_read", rc)
    return ms.value, n.value


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
