"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

Covers every step of the hot path -- block keys, index queries, index scores, per-group top-k,
sparse prefill and decode attention with their split-softmax combine -- and the dense GQA
baseline, at sizes spanning many tiles with ragged tails, the degenerate cases (empty ranges,
rows with no candidates, k >= candidates, forced score ties) and sharp-logit variants.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_scores_b200 import msa
from block_sparse_long_scores_b200.pipeline import Decode, Prefill
from block_sparse_long_scores_b200.workloads import WORKLOADS, make_inputs, scaled_down
from oracle import oracle as orc
from tests.parity_helpers import (Guards, check_attention, check_bf16_near, check_scores, cpu, oracle_shape,
                                  row_geometry, sample_rows)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _prefill_full_check(w, x, chunk_rows=None, rows=None, check_keys=True):
    """Run the prefill path on the GPU and compare each step with the oracle on `rows`; every
    output, the score buffer and the workspace carry guard bands that must stay untouched."""
    pf = Prefill(w, x, chunk_rows=chunk_rows)
    guards = Guards()
    pf.scores  # allocate the score buffer before guarding it
    guards.guard(pf, "o", "lse", "block_idx", "workspace", "_scores", "k_idx")
    T = pf.shape.total_rows
    rows = np.arange(T) if rows is None else rows
    xc = cpu(x)
    sh = oracle_shape(w, xc)
    # GPU: keys + scores per chunk, keeping the scores of the checked rows
    S_gpu = np.zeros((len(rows), w.Hkv, pf.stride), np.float32)
    qidx_gpu = torch.empty(pf.chunk, w.Hkv, w.d, dtype=torch.bfloat16, device=DEV)
    qidx_rows = np.zeros((len(rows), w.Hkv, w.d), np.uint16)
    first = True
    fused_idx = torch.full_like(pf.block_idx, -2)
    for r0, r1 in pf.chunks():
        pf.index(r0, r1, compute_keys=first, q_idx_out=qidx_gpu)
        first = False
        pf.select(r0, r1)
        pf.index_select(r0, r1, compute_keys=False, block_idx=fused_idx[r0:r1])
        pf.attend(r0, r1)
        sel = (rows >= r0) & (rows < r1)
        if sel.any():
            S_gpu[sel] = pf.scores[torch.as_tensor(rows[sel] - r0, device=DEV)].cpu().numpy()
            qidx_rows[sel] = _bits(qidx_gpu[torch.as_tensor(rows[sel] - r0, device=DEV)])
    torch.cuda.synchronize()
    assert int(pf.err.item()) == 0, f"device error flag {int(pf.err.item())}"
    # the fused index branch selects exactly what scores + selection do, on every row
    assert torch.equal(fused_idx, pf.block_idx), "fused index-topk differs from index scores + top-k"
    # index branch
    if "k_idx" in xc:
        kidx_ref = _bits(xc["k_idx"])
        assert np.array_equal(_bits(pf.k_idx), kidx_ref)
    else:
        kidx_ref, khat = orc.block_keys(sh, xc["k"], xc["wk"])
        if check_keys:
            check_bf16_near(_bits(pf.k_idx), khat, "k_idx")
        kidx_ref = _bits(pf.k_idx)          # score the GPU's keys to isolate the GEMM
    qref, qhat = orc.index_query(sh, xc["q"], xc["wq"], rows)
    check_bf16_near(qidx_rows, qhat, "q_idx")
    S_ref = orc.index_scores(sh, qidx_rows, kidx_ref, rows, pf.stride)
    check_scores(w, xc, rows, S_gpu, S_ref)
    # selection: bit-exact given the GPU's own scores
    sel_gpu = pf.block_idx.cpu().numpy()[rows]
    sel_ref = orc.select_topk_f32(sh, S_gpu, rows)
    assert np.array_equal(sel_gpu, sel_ref), "block selection differs from the oracle on the GPU's scores"
    # main branch on the GPU's selection
    O_ref, L_ref = orc.sparse_attn(sh, xc["q"], xc["k"], xc["v"], sel_gpu, rows)
    O_gpu = pf.o.float().cpu().numpy()[rows]
    L_gpu = pf.lse.cpu().numpy()[rows]
    guards.check()
    return check_attention(O_gpu, O_ref, L_gpu, L_ref)


def test_library_loads_and_reports_version():
    assert msa.lib().msa_version() >= 100


def test_tiny_prefill_parity():
    w = WORKLOADS["tiny_prefill"]
    x = make_inputs(w, device=DEV)
    _prefill_full_check(w, x)


@pytest.mark.parametrize("gain", [11.3137, 45.2548])
def test_tiny_prefill_sharp_logits(gain):
    # q, k ~ N(0,1) (gain sqrt(128)) and 4x that: exercises the max-subtraction and rescaling
    w = WORKLOADS["tiny_prefill"]
    x = make_inputs(w, device=DEV, logit_gain=gain, seed=1)
    _prefill_full_check(w, x)


def test_prefill_128k_shape_small_multichunk():
    # the 128K workload's heads/blocks/selection at 6000 rows (ragged tail), three chunks
    w = scaled_down(WORKLOADS["prefill_128k"], (6000,))
    x = make_inputs(w, device=DEV, seed=2)
    _prefill_full_check(w, x, chunk_rows=2048)


@pytest.mark.parametrize("gain", [11.3137, 45.2548])
def test_prefill_128k_shape_sharp_logits(gain):
    # the headline kernel instantiation (G 8, D 128, B 64) with q, k ~ N(0,1) and 4x that: the
    # logits reach several units, so the running max and the partials' rescaling are exercised
    w = scaled_down(WORKLOADS["prefill_128k"], (6000,))
    x = make_inputs(w, device=DEV, seed=31, logit_gain=gain)
    _prefill_full_check(w, x, chunk_rows=2048)


@pytest.mark.parametrize("gain", [8.0, 32.0])
def test_ragged_shape_sharp_logits(gain):
    # the ragged instantiation (G 8, D 64, B 128) with q, k ~ N(0,1) and 4x that
    w = scaled_down(WORKLOADS["ragged_prefill"], (130, 3000, 64, 2100))
    x = make_inputs(w, device=DEV, seed=32, logit_gain=gain)
    _prefill_full_check(w, x, chunk_rows=1500)


@pytest.mark.parametrize("gain", [1.0, 11.3137])
def test_prefill_head_dim_128_with_128_token_blocks(gain):
    # (head_dim 128, 128-token blocks): one S buffer in tensor memory and a two-stage query ring;
    # two sequences with ragged tails, 8 scored blocks + local + sink, three chunks
    w = scaled_down(WORKLOADS["prefill_128k"], (3000, 1777)).with_(B=128, n_topk=8)
    x = make_inputs(w, device=DEV, seed=44, logit_gain=gain)
    _prefill_full_check(w, x, chunk_rows=2048)


def test_prefill_in_subchunks():
    # one attention call over 6000 rows in sub-chunks of 1000 rows: two alternating workspace halves
    w = scaled_down(WORKLOADS["prefill_128k"], (6000,))
    x = make_inputs(w, device=DEV, seed=33, logit_gain=11.3137)
    msa.prefill_set_subchunk_rows(1000)
    try:
        pf = Prefill(w, x)
        pf.run()
        o1 = pf.o.clone()
        pf.o.zero_()
        pf.run()                                   # again: the halves are reused, results repeat
        torch.cuda.synchronize()
        assert int(pf.err.item()) == 0
        assert torch.equal(o1, pf.o)
    finally:
        msa.prefill_set_subchunk_rows(0)
    xc = cpu(x)
    sh = oracle_shape(w, xc)
    rows = np.arange(w.total_rows)
    O_ref, L_ref = orc.sparse_attn(sh, xc["q"], xc["k"], xc["v"], pf.block_idx.cpu().numpy(), rows)
    check_attention(pf.o.float().cpu().numpy(), O_ref, pf.lse.cpu().numpy(), L_ref)


def test_ragged_prefill_small_with_ties():
    # ragged workload shape (64/8 heads, D 64, B 128, k 32, discrete index keys -> exact ties)
    w = scaled_down(WORKLOADS["ragged_prefill"], (1, 130, 1000, 64, 2900, 129, 700))
    x = make_inputs(w, device=DEV, seed=3)
    _prefill_full_check(w, x, chunk_rows=1500)


def test_prefill_k_covers_all_candidates_equals_dense():
    # n_topk >= every candidate: the sparse path must reproduce dense causal attention
    w = scaled_down(WORKLOADS["tiny_prefill"], (700, 1100)).with_(n_topk=40)
    x = make_inputs(w, device=DEV, seed=4)
    pf = Prefill(w, x)
    pf.run()
    od = torch.empty_like(pf.o)
    ld = torch.empty_like(pf.lse)
    msa.msa_dense_attn_prefill(pf.cfg, pf.shape, x["q"], x["k"], x["v"], 0, pf.shape.total_rows, od, ld)
    torch.cuda.synchronize()
    xc = cpu(x)
    sh = oracle_shape(w, xc)
    rows = np.arange(pf.shape.total_rows)
    O_ref, L_ref = orc.dense_attn(sh, xc["q"], xc["k"], xc["v"], rows)
    check_attention(pf.o.float().cpu().numpy(), O_ref, pf.lse.cpu().numpy(), L_ref)
    check_attention(od.float().cpu().numpy(), O_ref, ld.cpu().numpy(), L_ref)


def _dense_check(w, x, r0=None, r1=None):
    """Dense causal GQA prefill over rows [r0, r1) against the fp64 oracle; rows outside the range
    must keep their previous contents."""
    cfg = msa.make_config(w.Hq, w.Hkv, w.D, w.B, w.d, w.n_topk, w.use_sink)
    shape = msa.prefill_shape(x["cu_seqlens"].to(DEV, torch.int32).contiguous(),
                              x["cu_blocks"].to(DEV, torch.int32).contiguous(), list(w.seqlens), w.B)
    T = shape.total_rows
    r0, r1 = (0, T) if r0 is None else (r0, r1)
    od = torch.full((T, w.Hq, w.D), float("nan"), dtype=torch.bfloat16, device=DEV)
    ld = torch.full((T, w.Hq), float("nan"), dtype=torch.float32, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.msa_dense_attn_prefill(cfg, shape, x["q"], x["k"], x["v"], r0, r1, od, ld, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    xc = cpu(x)
    rows = np.arange(r0, r1)
    O_ref, L_ref = orc.dense_attn(oracle_shape(w, xc), xc["q"], xc["k"], xc["v"], rows)
    check_attention(od[r0:r1].float().cpu().numpy(), O_ref, ld[r0:r1].cpu().numpy(), L_ref)
    assert torch.isnan(od[:r0]).all() and torch.isnan(od[r1:]).all()
    assert torch.isnan(ld[:r0]).all() and torch.isnan(ld[r1:]).all()


@pytest.mark.parametrize("gain", [1.0, 11.3137, 45.2548])
def test_dense_prefill_128k_shape(gain):
    # the dense baseline as the benchmarks run it (G 8, D 128, 64-token key steps): two sequences
    # with ragged tails; with sharp logits the rows' running max outgrows the rescale slack
    w = scaled_down(WORKLOADS["prefill_128k"], (1000, 1437))
    x = make_inputs(w, device=DEV, seed=41, logit_gain=gain)
    _dense_check(w, x)


def test_dense_prefill_head_dim_64_and_row_range():
    # D 64 with 64-token blocks (G 8), sharp logits, only rows [300, 1700) of three sequences
    w = scaled_down(WORKLOADS["ragged_prefill"], (500, 77, 1300)).with_(B=64)
    x = make_inputs(w, device=DEV, seed=42, logit_gain=8.0)
    _dense_check(w, x, 300, 1700)


@pytest.mark.parametrize("D_and_workload", [("128", "prefill_128k"), ("64", "ragged_prefill")])
def test_dense_prefill_128_token_blocks(D_and_workload):
    # 128-token blocks take the single-warpgroup dense kernel (the flash-attention kernel steps 64
    # keys): head_dim 128 (a shape the sparse prefill refuses, the dense call accepts) and 64, two
    # sequences with ragged tails, sharp logits
    _, name = D_and_workload
    w = scaled_down(WORKLOADS[name], (900, 1333)).with_(B=128)
    x = make_inputs(w, device=DEV, seed=43, logit_gain=8.0)
    _dense_check(w, x)


def test_prefill_sink_and_zero_topk():
    for k, sink in [(0, 0), (0, 1), (3, 1)]:
        w = scaled_down(WORKLOADS["tiny_prefill"], (300, 5, 64)).with_(n_topk=k, use_sink=sink)
        x = make_inputs(w, device=DEV, seed=5 + k + sink)
        _prefill_full_check(w, x)


def test_empty_row_range_is_a_no_op():
    w = WORKLOADS["tiny_prefill"]
    x = make_inputs(w, device=DEV)
    pf = Prefill(w, x)
    pf.o.zero_()
    before = pf.o.clone()
    msa.msa_sparse_attn_prefill(pf.cfg, pf.shape, x["q"], x["k"], x["v"], pf.block_idx, 5, 5, pf.o, pf.lse,
                                pf.workspace)
    msa.msa_select_topk(pf.cfg, pf.shape, pf.scores, pf.stride, 7, 7, pf.block_idx)
    torch.cuda.synchronize()
    assert torch.equal(before, pf.o)


def test_bad_block_ids_are_flagged_and_skipped():
    w = scaled_down(WORKLOADS["tiny_prefill"], (512,))
    x = make_inputs(w, device=DEV, seed=6)
    pf = Prefill(w, x)
    T = pf.shape.total_rows
    rows = np.arange(T)
    _, i = row_geometry(w, cpu(x), rows)
    rng = np.random.default_rng(0)
    bi = np.full((T, w.Hkv, w.k_tot), -1, np.int32)
    for r in range(T):
        for g in range(w.Hkv):
            pick = sorted(set(rng.integers(0, i[r] + 1, size=3).tolist()) | {int(i[r])})
            bi[r, g, :len(pick)] = pick
    clean = bi.copy()
    bad = bi.copy()
    bad[10, 0, -1] = 9999            # beyond the local block -> skipped, flagged
    bad[300, 1, -1] = bad[300, 1, 0]  # repeated block -> skipped, flagged
    bad[400, 0, 5] = -7              # negative other than -1 -> skipped, flagged
    dev_bi = torch.as_tensor(bad, device=DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    msa.msa_sparse_attn_prefill(pf.cfg, pf.shape, x["q"], x["k"], x["v"], dev_bi, 0, T, pf.o, pf.lse, pf.workspace, err)
    torch.cuda.synchronize()
    flags = int(err.item())
    assert flags & 1 and flags & 2, flags
    xc = cpu(x)
    sh = oracle_shape(w, xc)
    clean[400, 0, 5] = -1
    O_ref, L_ref = orc.sparse_attn(sh, xc["q"], xc["k"], xc["v"], clean, rows)
    check_attention(pf.o.float().cpu().numpy(), O_ref, pf.lse.cpu().numpy(), L_ref)


def test_block_order_does_not_matter():
    w = scaled_down(WORKLOADS["tiny_prefill"], (900,))
    x = make_inputs(w, device=DEV, seed=7)
    pf = Prefill(w, x)
    pf.run()
    o1 = pf.o.clone()
    shuffled = pf.block_idx.flip(-1).contiguous()
    msa.msa_sparse_attn_prefill(pf.cfg, pf.shape, x["q"], x["k"], x["v"], shuffled, 0, pf.shape.total_rows, pf.o,
                                pf.lse, pf.workspace, pf.err)
    torch.cuda.synchronize()
    # the combine sums partials in slot order, so fp32 rounding may differ: same tolerance as parity
    from tests.parity_helpers import check_attention
    check_attention(pf.o.float().cpu().numpy(), o1.double().cpu().numpy())
    assert int(pf.err.item()) == 0


# --------------------------------------------------------------------------------- decode


def _decode_check(w, x):
    dc = Decode(w, x)
    guards = Guards()
    guards.guard(dc, "o", "lse", "block_idx", "workspace", "scores", "k_idx")
    qidx = guards.wrap(torch.empty(w.batch, w.Hkv, w.d, dtype=torch.bfloat16, device=DEV), "q_idx")
    dc.run(q_idx_out=qidx)
    torch.cuda.synchronize()
    guards.check()
    return _decode_compare(w, x, dc, qidx)


def _decode_compare(w, x, dc, qidx):
    """One decode step's outputs (key cache, q_idx, scores, selection, O, lse) against the oracle."""
    assert int(dc.err.item()) == 0
    xc = cpu(x)
    sh = oracle_shape(w, xc)
    rows = np.arange(w.batch)
    if "k_idx" in xc:
        kidx = _bits(xc["k_idx"])
    else:
        kidx_ref, khat = orc.block_keys(sh, xc["k"], xc["wk"])
        _, i = row_geometry(w, xc, rows)
        # complete blocks only are ever scored; compare those
        mask = np.zeros(khat.shape[:3], bool)
        for b in range(w.batch):
            mask[b, :, : i[b]] = True
        check_bf16_near(_bits(dc.k_idx)[mask], khat[mask], "k_idx (cache)")
        kidx = _bits(dc.k_idx)
    check_bf16_near(_bits(qidx), orc.index_query(sh, xc["q"], xc["wq"], rows)[1], "q_idx")
    S_gpu = dc.scores.cpu().numpy()
    S_ref = orc.index_scores(sh, _bits(qidx), kidx, rows, dc.stride)
    check_scores(w, xc, rows, S_gpu, S_ref)
    sel = dc.block_idx.cpu().numpy()
    assert np.array_equal(sel, orc.select_topk_f32(sh, S_gpu, rows))
    O_ref, L_ref = orc.sparse_attn(sh, xc["q"], xc["k"], xc["v"], sel, rows)
    check_attention(dc.o.float().cpu().numpy(), O_ref, dc.lse.cpu().numpy(), L_ref)
    return dc


def test_decode_small_ragged():
    w = scaled_down(WORKLOADS["decode_128k"], (1, 63, 64, 65, 1000, 4096, 2000, 3333))
    x = make_inputs(w, device=DEV, seed=8)
    _decode_check(w, x)


def test_decode_many_short_sequences():
    # 300 sequences: every CTA of the streaming grid covers several (sequence, kv head) segments,
    # so in-CTA flushes and cross-CTA merges both run many times
    lens = tuple(int(v) for v in np.random.default_rng(21).integers(1, 2049, size=300))
    w = scaled_down(WORKLOADS["decode_128k"], lens)
    x = make_inputs(w, device=DEV, seed=21)
    _decode_check(w, x)


def test_decode_single_sequence():
    # one sequence: every CTA holds one or two selected blocks, so a segment's merge spans more
    # partials than one merge chunk
    w = scaled_down(WORKLOADS["decode_128k"], (5000,))
    x = make_inputs(w, device=DEV, seed=22)
    _decode_check(w, x)


def test_decode_workspace_needs_no_clearing_and_repeats_bitwise():
    # the merge counters carry a per-call generation: a workspace full of 0xFF bytes is as good as
    # a fresh one, and the partials are combined in a fixed order, so a repeat is bit-identical
    w = scaled_down(WORKLOADS["decode_128k"], (1, 70, 4096, 2500))
    x = make_inputs(w, device=DEV, seed=23)
    dc = _decode_check(w, x)
    o1, l1 = dc.o.clone(), dc.lse.clone()
    for _ in range(2):
        dc.workspace.fill_(0xFF)
        dc.o.fill_(0)
        msa.msa_sparse_attn_decode(dc.cfg, dc.shape, x["q"], x["k"], x["v"], dc.block_idx, dc.o, dc.lse,
                                   dc.workspace, dc.err)
        torch.cuda.synchronize()
        assert int(dc.err.item()) == 0
        assert torch.equal(dc.o, o1) and torch.equal(dc.lse, l1)


def test_decode_graph_replay_recomputes():
    # a CUDA graph replays one set of kernel arguments: every replay must still recompute and
    # merge (the kernel leaves its counters clear); 24 sequences make a pool of batches as well
    lens = tuple(int(v) for v in np.random.default_rng(24).integers(2000, 6000, size=24))
    w = scaled_down(WORKLOADS["decode_128k"], lens)
    x = make_inputs(w, device=DEV, seed=24)
    dc = Decode(w, x)
    step = dc.graph()
    g = torch.Generator(device="cpu").manual_seed(25)
    for _ in range(3):
        x["q"].copy_(torch.randn(x["q"].shape, generator=g).to(x["q"].dtype))
        step()
        torch.cuda.synchronize()
        o_graph, lse_graph = dc.o.clone(), dc.lse.clone()
        dc.o.fill_(0)
        dc.run()
        torch.cuda.synchronize()
        assert int(dc.err.item()) == 0
        assert torch.equal(o_graph, dc.o) and torch.equal(lse_graph, dc.lse)


def test_decode_graph_appends_tokens_across_block_boundaries():
    # a decode loop on one captured step: before each replay every sequence gains a token (its K/V
    # are already in the cache tensor; seqlens advances in place) and new queries arrive.  The step
    # refreshes the key of each sequence's newest block, so blocks that completed in earlier steps
    # (at lengths 64, 128, 192) are scored with the mean of all their tokens
    Lmax = 320
    lens0 = np.array([62, 126, 190, 1, 255], np.int32)
    w = scaled_down(WORKLOADS["decode_128k"], (Lmax,) * len(lens0)).with_(n_topk=2)
    x = make_inputs(w, device=DEV, seed=27)
    x["seqlens"].copy_(torch.as_tensor(lens0))
    w = w.with_(seqlens=tuple(int(v) for v in lens0))   # host view of the starting lengths
    dc = Decode(w, x)
    qidx = torch.empty(w.batch, w.Hkv, w.d, dtype=torch.bfloat16, device=DEV)
    step = dc.graph(q_idx_out=qidx)
    g = torch.Generator(device="cpu").manual_seed(28)
    for t in range(5):
        if t:
            x["seqlens"].add_(1)
            x["q"].copy_(torch.randn(x["q"].shape, generator=g).to(x["q"].dtype))
        step()
        torch.cuda.synchronize()
        lens = lens0 + t
        assert np.array_equal(x["seqlens"].cpu().numpy(), lens)
        _decode_compare(w.with_(seqlens=tuple(int(v) for v in lens)), x, dc, qidx)


def test_wait_timeout_is_reported_and_the_context_stays_usable():
    # a bounded wait that nothing completes (the path every kernel's internal waits take on a hang):
    # MSA_DERR_TIMEOUT comes back after the short limit, and the GPU keeps working afterwards
    import time
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    t0 = time.perf_counter()
    msa.diag_wait_timeout(err, 2_000_000)          # 2 ms
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert int(err.item()) & 8
    w = scaled_down(WORKLOADS["decode_128k"], (70, 1000))
    x = make_inputs(w, device=DEV, seed=34)
    _decode_check(w, x)


def test_decode_lengths_beyond_the_cache_are_clamped_and_flagged():
    # a seqlens entry above the cache capacity (or below 1) is a shape error: flagged, clamped
    w = scaled_down(WORKLOADS["decode_128k"], (300, 200))
    x = make_inputs(w, device=DEV, seed=29)
    dc = Decode(w, x)
    dc.run()
    torch.cuda.synchronize()
    assert int(dc.err.item()) == 0
    x["seqlens"][1] = 100000
    dc.run()
    torch.cuda.synchronize()
    assert int(dc.err.item()) & 16
    o_clamped = dc.o[1].clone()
    x["seqlens"][1] = 300
    dc.err.zero_()
    dc.run()
    torch.cuda.synchronize()
    assert int(dc.err.item()) == 0
    assert torch.equal(o_clamped, dc.o[1])


def test_decode_bad_and_unordered_block_ids_are_flagged_and_skipped():
    # the decode kernel sanitises each block list once per CTA: out-of-range ids and repeats are
    # skipped and flagged, any order is accepted (the selection is a set)
    w = scaled_down(WORKLOADS["decode_128k"], (300, 5000, 4096, 2))
    x = make_inputs(w, device=DEV, seed=26)
    dc = Decode(w, x)
    dc.run()
    torch.cuda.synchronize()
    assert int(dc.err.item()) == 0
    sel = dc.block_idx.cpu().numpy()
    bad, clean = sel.copy(), sel.copy()
    bad[1, 0] = sel[1, 0][::-1]                        # valid, descending, padding first
    v = np.flatnonzero(sel[1, 1] >= 0)
    bad[1, 1, v[-1]] = sel[1, 1, v[0]]                  # a repeat of the first block replaces the last
    clean[1, 1, v[-1]] = -1
    v = np.flatnonzero(sel[2, 2] >= 0)
    bad[2, 2, v[1]] = 99999                            # beyond the local block
    clean[2, 2, v[1]] = -1
    bad[0, 3, 1] = -7                                   # negative other than -1
    clean[0, 3, 1] = -1
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = torch.empty_like(dc.o), torch.empty_like(dc.lse)
    msa.msa_sparse_attn_decode(dc.cfg, dc.shape, x["q"], x["k"], x["v"], torch.as_tensor(bad, device=DEV), o, lse,
                               dc.workspace, err)
    torch.cuda.synchronize()
    flags = int(err.item())
    assert flags & 1 and flags & 2, flags
    xc = cpu(x)
    O_ref, L_ref = orc.sparse_attn(oracle_shape(w, xc), xc["q"], xc["k"], xc["v"], clean, np.arange(w.batch))
    check_attention(o.float().cpu().numpy(), O_ref, lse.cpu().numpy(), L_ref)


def test_decode_ragged_shape_with_ties():
    w = scaled_down(WORKLOADS["ragged_decode"], (129, 5000, 1, 3000))
    x = make_inputs(w, device=DEV, seed=9)
    _decode_check(w, x)


def test_dense_decode_matches_oracle():
    w = scaled_down(WORKLOADS["decode_128k"], (1, 100, 4096, 2500))
    x = make_inputs(w, device=DEV, seed=10)
    dc = Decode(w, x)
    ws = msa.msa_dense_attn_decode(dc.cfg, dc.shape, None, None, None, None, None, None)
    wsb = torch.empty(max(ws, 256), dtype=torch.uint8, device=DEV)
    msa.msa_dense_attn_decode(dc.cfg, dc.shape, x["q"], x["k"], x["v"], dc.o, dc.lse, wsb)
    torch.cuda.synchronize()
    xc = cpu(x)
    sh = oracle_shape(w, xc)
    O_ref, L_ref = orc.dense_attn(sh, xc["q"], xc["k"], xc["v"], np.arange(w.batch))
    check_attention(dc.o.float().cpu().numpy(), O_ref, dc.lse.cpu().numpy(), L_ref)


# ----------------------------------------------------------------- full-size, sampled rows


@pytest.mark.slow
def test_prefill_128k_full_size_sampled():
    w = WORKLOADS["prefill_128k"]
    x = make_inputs(w, device=DEV)
    rows = sample_rows(w, 4096)
    _prefill_full_check(w, x, chunk_rows=16384, rows=rows, check_keys=True)


@pytest.mark.slow
def test_decode_128k_full_size():
    w = WORKLOADS["decode_128k"]
    x = make_inputs(w, device=DEV)
    _decode_check(w, x)


# ------------------------------------------------- full-size 1M and ragged, sampled rows
# Host copies hold only what the oracle reads: Q rows of the sampled tokens (and, for decode, the
# cache blocks the GPU selected); the rest of each host tensor is never touched.


def _sparse_rows_cpu(t, rows):
    out = torch.empty(t.shape, dtype=t.dtype)
    idx = torch.as_tensor(rows, device=t.device)
    out[torch.as_tensor(rows)] = t[idx].cpu()
    return out


def _prefill_sampled_check(w, x, rows, chunk_rows):
    pf = Prefill(w, x, chunk_rows=chunk_rows)
    S_gpu = np.zeros((len(rows), w.Hkv, pf.stride), np.float32)
    qidx_gpu = torch.empty(pf.chunk, w.Hkv, w.d, dtype=torch.bfloat16, device=DEV)
    qidx_rows = np.zeros((len(rows), w.Hkv, w.d), np.uint16)
    first = True
    fused_idx = torch.full_like(pf.block_idx, -2)
    for r0, r1 in pf.chunks():
        pf.index(r0, r1, compute_keys=first, q_idx_out=qidx_gpu)
        first = False
        pf.select(r0, r1)
        pf.index_select(r0, r1, compute_keys=False, block_idx=fused_idx[r0:r1])
        pf.attend(r0, r1)
        sel = (rows >= r0) & (rows < r1)
        if sel.any():
            loc = torch.as_tensor(rows[sel] - r0, device=DEV)
            S_gpu[sel] = pf.scores[loc].cpu().numpy()
            qidx_rows[sel] = _bits(qidx_gpu[loc])
    torch.cuda.synchronize()
    assert int(pf.err.item()) == 0
    assert torch.equal(fused_idx, pf.block_idx), "fused index-topk differs from index scores + top-k"
    xc = {"q": _sparse_rows_cpu(x["q"], rows), "k": x["k"].cpu(), "v": x["v"].cpu(), "wq": x["wq"].cpu(),
          "wk": x["wk"].cpu(), "cu_seqlens": x["cu_seqlens"].cpu(), "cu_blocks": x["cu_blocks"].cpu()}
    sh = oracle_shape(w, xc)
    kidx = _bits(pf.k_idx)
    if "k_idx" in x:
        assert np.array_equal(kidx, _bits(x["k_idx"]))
    else:
        _, khat = orc.block_keys(sh, xc["k"], xc["wk"])
        check_bf16_near(kidx, khat, "k_idx")
    check_bf16_near(qidx_rows, orc.index_query(sh, xc["q"], xc["wq"], rows)[1], "q_idx")
    check_scores(w, xc, rows, S_gpu, orc.index_scores(sh, qidx_rows, kidx, rows, pf.stride))
    sel_gpu = pf.block_idx[torch.as_tensor(rows, device=DEV)].cpu().numpy()
    assert np.array_equal(sel_gpu, orc.select_topk_f32(sh, S_gpu, rows))
    O_ref, L_ref = orc.sparse_attn(sh, xc["q"], xc["k"], xc["v"], sel_gpu, rows)
    idx = torch.as_tensor(rows, device=DEV)
    check_attention(pf.o[idx].float().cpu().numpy(), O_ref, pf.lse[idx].cpu().numpy(), L_ref)


@pytest.mark.slow
def test_prefill_1m_full_size_sampled():
    w = WORKLOADS["prefill_1m"]
    x = make_inputs(w, device=DEV)
    # 4096 sampled rows, including the first and last 64 of the sequence
    _prefill_sampled_check(w, x, sample_rows(w, 4096, seed=1), chunk_rows=16384)


@pytest.mark.slow
def test_ragged_prefill_full_size_sampled():
    w = WORKLOADS["ragged_prefill"]
    x = make_inputs(w, device=DEV)
    # 4096 sampled rows, including the first and last 64 of every sequence
    _prefill_sampled_check(w, x, sample_rows(w, 4096, seed=2), chunk_rows=16384)


def _check_decode_key_cache(w, x, dc, n_blocks, seed):
    """The GPU's block-key cache against the oracle on sampled blocks: their K rows are gathered
    into a compact host cache (a block key depends only on its own rows), so the oracle reads only
    the sampled blocks.  Every sampled block is complete."""
    rng = np.random.default_rng(seed)
    lens = x["seqlens"].cpu().numpy()
    full = [int(l) // w.B for l in lens]
    ns = min(n_blocks, min(full))
    picks = [np.sort(rng.choice(full[b], size=ns, replace=False)) for b in range(w.batch)]
    kc = torch.empty((w.batch, w.Hkv, ns * w.B, w.D), dtype=x["k"].dtype)
    for b in range(w.batch):
        rows = (torch.as_tensor(picks[b], device=x["k"].device).view(-1, 1) * w.B +
                torch.arange(w.B, device=x["k"].device).view(1, -1)).reshape(-1)
        kc[b] = x["k"][b][:, rows].cpu()
    sh = orc.decode_shape(np.full(w.batch, ns * w.B, np.int32), ns * w.B, ns, w.Hq, w.Hkv, w.D, w.B, w.d,
                          w.n_topk, w.use_sink)
    _, khat = orc.block_keys(sh, kc, x["wk"].cpu())
    gpu = _bits(dc.k_idx)
    got = np.stack([gpu[b][:, picks[b]] for b in range(w.batch)])
    check_bf16_near(got, khat[:, :, :ns], "k_idx (sampled cache blocks)")


def _decode_sampled_check(w, x, key_blocks=0):
    dc = Decode(w, x)
    qidx = torch.empty(w.batch, w.Hkv, w.d, dtype=torch.bfloat16, device=DEV)
    dc.run(q_idx_out=qidx)
    torch.cuda.synchronize()
    assert int(dc.err.item()) == 0
    rows = np.arange(w.batch)
    sel = dc.block_idx.cpu().numpy()
    # host cache with only the selected blocks copied
    kc = torch.empty(x["k"].shape, dtype=x["k"].dtype)
    vc = torch.empty(x["v"].shape, dtype=x["v"].dtype)
    for b in range(w.batch):
        for g in range(w.Hkv):
            for j in sel[b, g]:
                if j >= 0:
                    kc[b, g, j * w.B:(j + 1) * w.B] = x["k"][b, g, j * w.B:(j + 1) * w.B].cpu()
                    vc[b, g, j * w.B:(j + 1) * w.B] = x["v"][b, g, j * w.B:(j + 1) * w.B].cpu()
    xc = {"q": x["q"].cpu(), "k": kc, "v": vc, "wq": x["wq"].cpu(), "seqlens": x["seqlens"].cpu()}
    sh = oracle_shape(w, xc)
    kidx = _bits(dc.k_idx)
    check_bf16_near(_bits(qidx), orc.index_query(sh, xc["q"], xc["wq"], rows)[1], "q_idx")
    S_gpu = dc.scores.cpu().numpy()
    check_scores(w, xc, rows, S_gpu, orc.index_scores(sh, _bits(qidx), kidx, rows, dc.stride))
    assert np.array_equal(sel, orc.select_topk_f32(sh, S_gpu, rows))
    O_ref, L_ref = orc.sparse_attn(sh, xc["q"], xc["k"], xc["v"], sel, rows)
    check_attention(dc.o.float().cpu().numpy(), O_ref, dc.lse.cpu().numpy(), L_ref)
    if key_blocks:
        _check_decode_key_cache(w, x, dc, key_blocks, seed=7)


@pytest.mark.slow
def test_decode_1m_full_size():
    # the 1M decode workload as benchmarked: 8 sequences of 2^20 tokens, 128 picks + sink + local;
    # the host copies hold only the selected blocks (the rest of each host tensor is never touched)
    w = WORKLOADS["decode_1m"]
    x = make_inputs(w, device=DEV, seed=3)
    _decode_sampled_check(w, x, key_blocks=512)


@pytest.mark.slow
def test_decode_1m_length_with_partial_last_block():
    # a 1M-long cache whose last block is partial (its local block holds 27 of 64 keys)
    w = WORKLOADS["decode_1m"].with_(seqlens=(1 << 20, (1 << 20) - 37))
    x = make_inputs(w, device=DEV, seed=5)
    _decode_sampled_check(w, x, key_blocks=256)


@pytest.mark.slow
def test_ragged_decode_full_size():
    w = WORKLOADS["ragged_decode"]
    x = make_inputs(w, device=DEV, seed=4)
    _decode_sampled_check(w, x)
