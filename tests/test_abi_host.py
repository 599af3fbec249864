"""Host-side checks of the C ABI that need no GPU: the library loads, exports every function the
header declares, rejects bad arguments before launching anything, and sizes workspaces."""
import ctypes
import os
import re

import pytest

from block_sparse_long_scores_b200 import msa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(msa.LIB_PATH):
        from block_sparse_long_scores_b200 import build
        build.build()
    return msa.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("msa_index_scores", "msa_select_topk", "msa_sparse_attn_prefill", "msa_sparse_attn_decode"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), f"{name} declared in msa.h but not exported"
    assert set(msa.EXPORTED) <= set(declared_functions())


def test_status_strings(L):
    assert L.msa_status_string(0) == b"ok"
    assert L.msa_status_string(3) == b"workspace too small"


def _cfg(**kw):
    base = dict(Hq=32, Hkv=4, D=128, B=64, d=64, n_topk=64, use_sink=1)
    base.update(kw)
    return msa.make_config(base["Hq"], base["Hkv"], base["D"], base["B"], base["d"], base["n_topk"], base["use_sink"])


def _prefill_shape(T=131072, B=64, fake_ptr=0x10000):
    nb = (T + B - 1) // B
    return msa.Shape(msa.MSA_PREFILL, 1, fake_ptr, fake_ptr, None, T, nb, T, nb)


def _ws(L, cfg, shape, r0, r1):
    n = ctypes.c_size_t(0)
    rc = L.msa_sparse_attn_prefill(ctypes.byref(cfg), ctypes.byref(shape), None, None, None, None, r0, r1, None,
                                   None, None, ctypes.byref(n), None, None)
    return rc, n.value


def test_prefill_workspace_query_is_host_only_and_grows_with_rows(L):
    cfg, shape = _cfg(), _prefill_shape()
    rc, small = _ws(L, cfg, shape, 0, 1024)
    assert rc == 0 and small > 0
    rc, big = _ws(L, cfg, shape, 0, 16384)
    assert rc == 0 and big > small
    # partial outputs dominate: rows x Hkv x k_tot x G x D bf16
    assert big >= 16384 * 4 * 66 * 8 * 128 * 2


def test_prefill_workspace_stops_growing_past_two_subchunks(L):
    # past one sub-chunk the call alternates two sub-chunk workspaces, whatever the row count
    cfg, shape = _cfg(), _prefill_shape()
    assert L.msa_prefill_subchunk_rows() == 16384
    _, one = _ws(L, cfg, shape, 0, 16384)
    _, two = _ws(L, cfg, shape, 0, 16385)
    _, all_rows = _ws(L, cfg, shape, 0, 131072)
    assert two == all_rows and one < two <= 2 * one + 256
    L.msa_prefill_set_subchunk_rows(1000)
    try:
        assert L.msa_prefill_subchunk_rows() == 1000
        _, small = _ws(L, cfg, shape, 0, 131072)
        assert small < one
    finally:
        L.msa_prefill_set_subchunk_rows(0)
    assert L.msa_prefill_subchunk_rows() == 16384


def test_decode_workspace_query(L):
    cfg = _cfg()
    shape = msa.Shape(msa.MSA_DECODE, 32, None, None, 0x10000, 32, 0, 131072, 2048)
    n = ctypes.c_size_t(0)
    rc = L.msa_sparse_attn_decode(ctypes.byref(cfg), ctypes.byref(shape), None, None, None, None, None, None, None,
                                  ctypes.byref(n), None, None)
    assert rc == 0 and n.value > 0


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), 2), (dict(B=32), 2), (dict(d=32), 2), (dict(Hq=24, Hkv=8), 2),
    (dict(Hq=30, Hkv=4), 1), (dict(n_topk=-1), 1), (dict(use_sink=2), 1), (dict(n_topk=300), 2),
])
def test_bad_config_is_rejected_before_launch(L, kw, code):
    cfg, shape = _cfg(**kw), _prefill_shape()
    rc, _ = _ws(L, cfg, shape, 0, 128)
    assert rc == code


def test_bad_shape_and_ranges_are_rejected(L):
    cfg = _cfg()
    assert _ws(L, cfg, _prefill_shape(), 10, 5)[0] == 1          # row_end < row_begin
    assert _ws(L, cfg, _prefill_shape(), 0, 131073)[0] == 1      # past the rows
    bad = _prefill_shape()
    bad.max_blocks = 7
    assert _ws(L, cfg, bad, 0, 10)[0] == 1                       # inconsistent block count
    bad = _prefill_shape()
    bad.cu_seqlens = None
    assert _ws(L, cfg, bad, 0, 10)[0] == 1                       # missing device array
    n = ctypes.c_size_t(1)
    rc = L.msa_sparse_attn_prefill(None, ctypes.byref(_prefill_shape()), None, None, None, None, 0, 1, None, None,
                                   None, ctypes.byref(n), None, None)
    assert rc == 1                                               # null config


def test_workspace_too_small_and_misaligned(L):
    cfg, shape = _cfg(), _prefill_shape()
    _, need = _ws(L, cfg, shape, 0, 256)
    small = ctypes.c_size_t(need - 1)
    fake = ctypes.c_void_p(0x100000)
    rc = L.msa_sparse_attn_prefill(ctypes.byref(cfg), ctypes.byref(shape), fake, fake, fake, fake, 0, 256, fake, None,
                                   fake, ctypes.byref(small), None, None)
    assert rc == 3
    ok = ctypes.c_size_t(need)
    mis = ctypes.c_void_p(0x100008)
    rc = L.msa_sparse_attn_prefill(ctypes.byref(cfg), ctypes.byref(shape), mis, fake, fake, fake, 0, 256, fake, None,
                                   fake, ctypes.byref(ok), None, None)
    assert rc == 1


def test_index_scores_rejects_bad_stride(L):
    cfg, shape = _cfg(), _prefill_shape()
    fake = ctypes.c_void_p(0x100000)
    for stride in (2047, 2050):   # below max_blocks / not a multiple of 4
        rc = L.msa_index_scores(ctypes.byref(cfg), ctypes.byref(shape), fake, fake, fake, fake, fake, 0, 0, 10, fake,
                                stride, None, None)
        assert rc == 1


def test_newest_block_key_mode_is_decode_only(L):
    # kidx_from_block = MSA_KIDX_NEWEST_BLOCK (-1) needs decode mode and K; other negatives are errors
    cfg = _cfg()
    fake = ctypes.c_void_p(0x100000)
    pre = _prefill_shape()
    rc = L.msa_index_scores(ctypes.byref(cfg), ctypes.byref(pre), fake, fake, fake, fake, fake,
                            msa.MSA_KIDX_NEWEST_BLOCK, 0, 10, fake, 2048, None, None)
    assert rc == 1
    dec = _decode_shape(4, 4096)
    rc = L.msa_index_scores(ctypes.byref(cfg), ctypes.byref(dec), fake, None, fake, None, fake,
                            msa.MSA_KIDX_NEWEST_BLOCK, 0, 4, fake, 64, None, None)
    assert rc == 1                                                # no K to compute keys from
    rc = L.msa_index_scores(ctypes.byref(cfg), ctypes.byref(dec), fake, fake, fake, fake, fake, -2, 0, 4, fake, 64,
                            None, None)
    assert rc == 1


def test_wait_timeout_diagnostic_checks_its_arguments(L):
    fake = ctypes.c_void_p(0x100000)
    assert L.msa_diag_wait_timeout(None, 1000, None) == 1              # no flag to report into
    assert L.msa_diag_wait_timeout(ctypes.c_void_p(0x100002), 1000, None) == 1   # misaligned
    assert L.msa_diag_wait_timeout(fake, 0, None) == 1                 # no bound
    assert L.msa_diag_wait_timeout(fake, 2_000_000_000, None) == 1     # beyond the kernels' 1 s bound


def test_select_topk_rejects_misaligned_scores_and_bad_stride(L):
    # long score rows are copied 16 bytes at a time: the base must be 16-byte aligned and the row
    # stride a multiple of 4 floats (at least max_blocks), as for msa_index_scores
    cfg, shape = _cfg(), _prefill_shape()
    fake = ctypes.c_void_p(0x100000)
    cases = [(ctypes.c_void_p(0x100004), 2048),   # 4-byte aligned only
             (fake, 2047),                        # below max_blocks
             (fake, 2050)]                        # not a multiple of 4
    for scores, stride in cases:
        rc = L.msa_select_topk(ctypes.byref(cfg), ctypes.byref(shape), scores, stride, 0, 10, fake, None, None)
        assert rc == 1
    # a valid call on an empty row range launches nothing and succeeds
    rc = L.msa_select_topk(ctypes.byref(cfg), ctypes.byref(shape), fake, 2048, 5, 5, fake, None, None)
    assert rc == 0


def _decode_shape(batch, Lmax, B=64):
    return msa.Shape(msa.MSA_DECODE, batch, None, None, 0x10000, batch, 0, Lmax, (Lmax + B - 1) // B)


def _decode_ws(L, cfg, shape):
    n = ctypes.c_size_t(0)
    rc = L.msa_sparse_attn_decode(ctypes.byref(cfg), ctypes.byref(shape), None, None, None, None, None, None, None,
                                  ctypes.byref(n), None, None)
    return rc, n.value


def test_decode_workspace_follows_the_split_geometry(L):
    # Without a GPU the library sizes for 148 SMs; (head_dim 128, 64-token blocks) runs 2 CTAs per
    # SM.  Items = batch x Hkv x k_tot split into equal runs; one (m, l, O) partial slot of 16 rows
    # per CTA and segment it touches (a separate kernel merges them, so there are no counters).
    def expected(batch, Hkv, k_tot, D):
        items = batch * Hkv * k_tot
        slots = min(148 * 2, items)
        per = -(-items // slots)
        n_ctas = -(-items // per)
        max_seg = -(-per // k_tot) + 1
        rows = n_ctas * max_seg * 16
        a = lambda x: (x + 255) & ~255
        return 2 * a(4 * rows) + a(4 * rows * D)

    rc, n = _decode_ws(L, _cfg(), _decode_shape(32, 131072))                    # decode 128K
    assert rc == 0 and n == expected(32, 4, 66, 128)
    assert 4.5 * 2**20 < n < 4.9 * 2**20                                        # "4.7 MiB" in the header
    rc, n = _decode_ws(L, _cfg(n_topk=128), _decode_shape(8, 1 << 20))         # decode 1M
    assert rc == 0 and n == expected(8, 4, 130, 128)


def test_noalloc_decode_refuses_problems_beyond_its_scratch_on_the_host(L):
    cfg = _cfg()
    args = [None] * 6 + [None, None]   # q, k, v, block_idx, o, lse, err_flag, stream
    # 4096 sequences x 4 kv heads x 66 slots: ~140 MiB of partials > the 40 MiB array
    rc = L.msa_sparse_attn_decode_noalloc(ctypes.byref(cfg), ctypes.byref(_decode_shape(4096, 64)), *args)
    assert rc == 3
    # the 128K decode workload fits: it passes the size check and stops at the null pointers
    rc = L.msa_sparse_attn_decode_noalloc(ctypes.byref(cfg), ctypes.byref(_decode_shape(32, 131072)), *args)
    assert rc == 1


def test_decode_refuses_problems_beyond_32_bit_indexing(L):
    # batch x Hkv x Lmax = 8192 x 4 x 65536 = 2^31 cache rows: refused on the size query as well
    rc, _ = _decode_ws(L, _cfg(), _decode_shape(8192, 65536))
    assert rc == 2
    rc, _ = _decode_ws(L, _cfg(), _decode_shape(4096, 65536))                  # 2^30 rows: accepted
    assert rc == 0


def _bwd(L, cfg, shape, r0, r1, ptrs=None, ws=None, nbytes=0, dq=None):
    """msa_sparse_attn_prefill_bwd with fake (never dereferenced) device pointers."""
    p = ptrs if ptrs is not None else ctypes.c_void_p(0x100000)
    n = ctypes.c_size_t(nbytes)
    rc = L.msa_sparse_attn_prefill_bwd(ctypes.byref(cfg), ctypes.byref(shape), p, p, p, p, p, p, p, r0, r1,
                                       dq if dq is not None else p, p, p, ws, ctypes.byref(n), None, None)
    return rc, n.value


def test_backward_workspace_query_and_validation(L):
    # the size query launches nothing and needs no device; every bad argument is refused first
    cfg, shape = _cfg(), _prefill_shape()
    rc, need = _bwd(L, cfg, shape, 0, 4096, ptrs=None, ws=None)
    assert rc == 0 and need > 4096 * 32 * 4                       # at least D = dO . O for the rows
    rc, need_all = _bwd(L, cfg, shape, 0, 131072, ptrs=None, ws=None)
    assert rc == 0 and need_all >= need
    assert _bwd(L, cfg, shape, 10, 5)[0] == 1                     # row_end < row_begin
    assert _bwd(L, cfg, shape, 0, 131073)[0] == 1                 # past the rows
    dec = _decode_shape(4, 4096)
    assert _bwd(L, cfg, dec, 0, 1)[0] == 1                        # prefill only
    assert _bwd(L, _cfg(B=128), _prefill_shape(B=128), 0, 10)[0] == 2   # head_dim 128 x 128-token blocks
    ws = ctypes.c_void_p(0x200000)
    assert _bwd(L, cfg, shape, 0, 4096, ws=ws, nbytes=need - 1)[0] == 3                     # too small
    assert _bwd(L, cfg, shape, 0, 4096, ws=ws, nbytes=need, dq=ctypes.c_void_p(0x100004))[0] == 1   # dq not 16-B
    assert _bwd(L, cfg, shape, 0, 4096, ws=ctypes.c_void_p(0x200010), nbytes=need)[0] == 1  # workspace not 256-B
    n = ctypes.c_size_t(need)
    fake = ctypes.c_void_p(0x100000)
    rc = L.msa_sparse_attn_prefill_bwd(ctypes.byref(cfg), ctypes.byref(shape), fake, fake, fake, fake, None, fake,
                                       fake, 0, 4096, fake, fake, fake, ws, ctypes.byref(n), None, None)
    assert rc == 1                                                # missing lse
    # an empty row range with valid arguments is a no-op (nothing launched, no device needed)
    assert _bwd(L, cfg, shape, 7, 7, ws=ws, nbytes=need)[0] == 0


def test_fused_index_topk_validation(L):
    # msa_index_topk is prefill-only and checks pointers, alignment and ranges before any launch
    cfg, shape = _cfg(), _prefill_shape()
    f = ctypes.c_void_p(0x100000)

    def call(q=f, k=None, wq=f, wk=None, kidx=f, frm=0, r0=0, r1=16, bi=f, shp=shape):
        return L.msa_index_topk(ctypes.byref(cfg), ctypes.byref(shp), q, k, wq, wk, kidx, frm, r0, r1, bi, None,
                                None, None)
    assert call(shp=_decode_shape(4, 4096)) == 2                   # decode: use msa_index_scores + select
    assert call(q=None) == 1
    assert call(k=f, wk=None) == 1                                 # keys to pool but no W_k
    assert call(bi=ctypes.c_void_p(0x100002)) == 1                 # block_idx not 4-byte aligned
    assert call(q=ctypes.c_void_p(0x100008)) == 1                  # q not 16-byte aligned
    assert call(r0=5, r1=4) == 1
    assert call(r1=131073) == 1
    assert call(frm=-1) == 1                                       # the newest-block mode is decode-only
    assert call(r0=9, r1=9) == 0                                   # empty range, keys precomputed: no launch


def test_dense_prefill_validation(L):
    cfg, shape = _cfg(), _prefill_shape()
    f = ctypes.c_void_p(0x100000)

    def call(q=f, o=f, lse=None, r0=0, r1=16, shp=shape):
        return L.msa_dense_attn_prefill(ctypes.byref(cfg), ctypes.byref(shp), q, f, f, r0, r1, o, lse, None, None)
    assert call(shp=_decode_shape(4, 4096)) == 1
    assert call(q=None) == 1
    assert call(o=ctypes.c_void_p(0x100008)) == 1                  # o not 16-byte aligned
    assert call(lse=ctypes.c_void_p(0x100002)) == 1                # lse not 4-byte aligned
    assert call(r0=3, r1=2) == 1
    assert call(r0=4, r1=4) == 0                                   # empty range: nothing launched


def test_prefill_accepts_head_dim_128_with_128_token_blocks(L):
    rc, n = _ws(L, _cfg(B=128), _prefill_shape(B=128), 0, 4096)
    assert rc == 0 and n > 0
