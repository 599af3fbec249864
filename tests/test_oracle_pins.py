"""Pins for the fp64 CPU oracle: checks against things other than the oracle itself.

Each check is chosen so that a plausible mistake in the oracle (a dropped term, a wrong sign or
index, a transposed operand, a wrong tie rule) fails at least one of them:
hand-worked golden values, closed forms, brute force on tiny inputs, independent library
routines (torch fp64 softmax, numpy matmul) and invariants the pages fix:

* exact attention over the selected blocks ("深度解析 MiniMax-M3", section "架构核心：MoE 与 MSA
  的深度融合", item 2) -> with every causal block selected it is dense causal GQA attention;
* masked-dense restatement ("MiniMax M3 开源 ... 完全指南", section 3.1 stage 3): attention over a
  subset equals dense attention with the other logits at -inf;
* per-group selection (same page as the first, item 1) -> groups are independent;
* exp-free top-k on raw logits (wiki.500nian.com digest, flowchart "exp-free Top-k") -> the
  selection depends only on the order of the scores.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def bf(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


def f64(t):
    return t.to(torch.float64).numpy()


def rand_bf16(shape, std, g):
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


# ------------------------------------------------------------------ bf16 rounding


def test_round_bf16_matches_torch_on_fp32_values():
    g = torch.Generator().manual_seed(1)
    x32 = torch.randn(20000, generator=g) * torch.exp(torch.randn(20000, generator=g) * 8)
    ours = orc.round_bf16(x32.double().numpy())
    ref = x32.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_round_bf16_ties_to_even_and_no_double_rounding():
    one = 1.0
    cases = {
        one + 2.0 ** -8: one,                                   # tie -> even mantissa (0)
        one + 3 * 2.0 ** -8: one + 2.0 ** -6,                   # tie -> even mantissa (2)
        one + 2.0 ** -8 + 2.0 ** -30: one + 2.0 ** -7,          # just above the tie: up
        -(one + 2.0 ** -8 + 2.0 ** -30): -(one + 2.0 ** -7),
        0.0: 0.0,
    }
    got = orc.bf16_bits_to_f64(orc.round_bf16(np.array(list(cases.keys()))))
    assert np.array_equal(got, np.array(list(cases.values())))


# ------------------------------------------------------------------ golden, hand-worked


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_golden_index_branch():
    gd = _golden()["index"]
    shape = orc.prefill_shape([0, 3], gd["Hq"], gd["Hkv"], gd["D"], gd["B"], gd["d"], gd["n_topk"],
                              gd["use_sink"])
    K = bf(gd["K"])
    Wk, Wq = bf(gd["W_k"]), bf(gd["W_q"])
    Q = torch.zeros(3, 2, 2, dtype=torch.bfloat16)
    Q[2] = bf(gd["Q_row2"])
    kidx, khat = orc.block_keys(shape, K, Wk)
    assert np.array_equal(orc.bf16_bits_to_f64(kidx), np.array(gd["expected_k_idx"]))
    assert np.array_equal(khat, np.array(gd["expected_k_idx"]))
    qidx, _ = orc.index_query(shape, Q, Wq, [2])
    assert np.array_equal(orc.bf16_bits_to_f64(qidx)[0], np.array(gd["expected_q_idx_row2"]))
    S = orc.index_scores(shape, qidx, kidx, [2], ncols=2)
    assert S[0, 0, 0] == gd["expected_score_row2_block0"]
    assert np.isnan(S[0, 0, 1])                     # the local block is never scored
    sel = orc.select_topk_f64(shape, S, [2])
    assert sel[0, 0].tolist() == gd["expected_block_idx_row2"]


def test_golden_attention_closed_form():
    gd = _golden()["attention"]
    shape = orc.prefill_shape([0, 3], 1, 1, 1, 1, 1, 3, 0)
    K = bf(gd["K"]).view(3, 1, 1)
    V = bf(gd["V"]).view(3, 1, 1)
    Q = bf([gd["q_row0"], 0, gd["q_row2"]]).view(3, 1, 1)
    e = math.e
    O, L = orc.sparse_attn(shape, Q, K, V, np.array([[[0, 1, 2, -1]]]), [2], scale=1.0)
    assert O[0, 0, 0] == pytest.approx((1 + 2 * e + 4 * e * e) / (1 + e + e * e), rel=1e-15)
    assert L[0, 0] == pytest.approx(math.log(1 + e + e * e), rel=1e-15)
    O, L = orc.sparse_attn(shape, Q, K, V, np.array([[[1, 2, -1, -1]]]), [2], scale=1.0)
    assert O[0, 0, 0] == pytest.approx((2 + 4 * e) / (1 + e), rel=1e-15)
    assert L[0, 0] == pytest.approx(math.log(e + e * e), rel=1e-15)
    O, L = orc.sparse_attn(shape, Q, K, V, np.array([[[0, -1, -1, -1]]]), [0], scale=1.0)
    assert O[0, 0, 0] == 1.0 and L[0, 0] == 0.0
    Od, Ld = orc.dense_attn(shape, Q, K, V, [2], scale=1.0)
    assert Od[0, 0, 0] == pytest.approx((1 + 2 * e + 4 * e * e) / (1 + e + e * e), rel=1e-15)
    assert Ld[0, 0] == pytest.approx(math.log(1 + e + e * e), rel=1e-15)


# ------------------------------------------------------------------ index branch vs brute force


def _small_prefill(seed=0, lens=(37, 130, 64), Hq=8, Hkv=2, D=16, B=8, d=8, k=3, sink=0):
    g = torch.Generator().manual_seed(seed)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    shape = orc.prefill_shape(cu, Hq, Hkv, D, B, d, k, sink)
    Q = rand_bf16((T, Hq, D), 1.0, g)
    K = rand_bf16((T, Hkv, D), 1.0, g)
    V = rand_bf16((T, Hkv, D), 1.0, g)
    Wq = rand_bf16((D, d), D ** -0.5, g)
    Wk = rand_bf16((D, d), D ** -0.5, g)
    return shape, cu, Q, K, V, Wq, Wk


def test_block_keys_pool_then_project_equals_project_then_mean():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill()
    kidx, khat = orc.block_keys(shape, K, Wk)
    Kf, Wf = f64(K), f64(Wk)
    B = shape.B
    ref = []
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        for t0 in range(s0, s1, B):
            t1 = min(t0 + B, s1)
            proj = np.einsum("tge,ec->tgc", Kf[t0:t1], Wf)       # project each token, then mean
            ref.append(proj.mean(axis=0))
    ref = np.stack(ref)
    np.testing.assert_allclose(khat, ref, rtol=0, atol=1e-12)
    # the bf16 value is the nearest bf16 to khat
    back = orc.bf16_bits_to_f64(kidx)
    ulp = np.exp2(np.floor(np.log2(np.abs(khat))) - 7)
    assert np.all(np.abs(back - khat) <= ulp / 2 + 1e-300)


def test_block_keys_from_block_and_decode_layout():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(lens=(70,))
    kidx, _ = orc.block_keys(shape, K, Wk)
    # the same keys as a decode cache [1, Hkv, Lmax, D]
    cache = K.permute(1, 0, 2).unsqueeze(0).contiguous()
    dshape = orc.decode_shape([70], 70, 9, shape.Hq, shape.Hkv, shape.D, shape.B, shape.d, 3, 0)
    init = np.full((1, shape.Hkv, 9, shape.d), 0x7777, np.uint16)
    dk, _ = orc.block_keys(dshape, cache, Wk, from_block=4, k_idx_init=init)
    assert np.all(dk[0, :, :4] == 0x7777)                        # blocks below from_block untouched
    assert np.array_equal(dk[0, :, 4:9], kidx[4:9].transpose(1, 0, 2))


def test_index_query_head_mean_then_project():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill()
    rows = [0, 5, 36, 37, 200, 230]
    qidx, qhat = orc.index_query(shape, Q, Wq, rows)
    G = shape.Hq // shape.Hkv
    Qf = f64(Q)[rows].reshape(len(rows), shape.Hkv, G, shape.D)
    ref = np.einsum("rge,ec->rgc", Qf.mean(axis=2), f64(Wq))
    np.testing.assert_allclose(qhat, ref, rtol=0, atol=1e-12)
    # the head mean is over the group's own heads: the other group's mean gives another answer
    other = np.einsum("rge,ec->rgc", Qf[:, ::-1].mean(axis=2), f64(Wq))
    assert not np.allclose(other, ref, atol=1e-6)


def test_index_scores_brute_force_and_candidate_range():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(sink=1)
    rows = list(range(shape.T))
    kidx, _ = orc.block_keys(shape, K, Wk)
    qidx, _ = orc.index_query(shape, Q, Wq, rows)
    ncols = 17
    S = orc.index_scores(shape, qidx, kidx, rows, ncols)
    qf, kf = orc.bf16_bits_to_f64(qidx), orc.bf16_bits_to_f64(kidx)
    for r in rows:
        b = np.searchsorted(cu, r, side="right") - 1
        pos = r - cu[b]
        i = pos // shape.B
        for g in range(shape.Hkv):
            for j in range(ncols):
                if 1 <= j < i:
                    ref = float(np.dot(qf[r, g], kf[shape.cu_blocks[b] + j, g]))
                    assert S[r, g, j] == pytest.approx(ref, rel=1e-15, abs=1e-300)
                else:
                    assert math.isnan(S[r, g, j])


# ------------------------------------------------------------------ exp-free per-group top-k


def _brute_select(scores_row, i, k, sink):
    cands = [(scores_row[j], j) for j in range(sink, i)]
    cands.sort(key=lambda t: (-t[0], t[1]))
    sel = {j for _, j in cands[:k]} | {i}
    if sink and i > 0:
        sel.add(0)
    return sorted(sel)


@pytest.mark.parametrize("k,sink", [(1, 0), (3, 0), (3, 1), (40, 1)])
def test_select_topk_brute_force_with_ties(k, sink):
    rng = np.random.default_rng(7 + k + sink)
    shape = orc.prefill_shape([0, 400], 2, 2, 4, 8, 4, k, sink)
    rows = list(range(0, 400, 3))
    ncols = 50
    S = rng.integers(-3, 4, size=(len(rows), 2, ncols)).astype(np.float64)  # many exact ties
    S[rng.random(S.shape) < 0.1] = -0.0
    sel = orc.select_topk_f64(shape, S, rows)
    for a, r in enumerate(rows):
        i = r // 8
        for g in range(2):
            ref = _brute_select(S[a, g], i, k, sink)
            got = [x for x in sel[a, g] if x >= 0]
            assert got == ref
            assert all(x == -1 for x in sel[a, g][len(ref):])
            # count invariant
            assert len(got) == min(k, max(0, i - sink)) + 1 + (1 if sink and i > 0 else 0)


def test_select_topk_order_only_invariance_and_zero_signs():
    rng = np.random.default_rng(3)
    shape = orc.prefill_shape([0, 1024], 1, 1, 4, 16, 4, 5, 1)
    rows = list(range(1024))
    S = rng.standard_normal((1024, 1, 64)).astype(np.float32).astype(np.float64)
    base = orc.select_topk_f64(shape, S, rows)
    for e in (-40, -3, 5, 60):
        assert np.array_equal(orc.select_topk_f64(shape, S * 2.0 ** e, rows), base)
    # strictly increasing map keeps the order (no new ties here): exp-free means order-only
    assert np.array_equal(orc.select_topk_f64(shape, np.arctan(S) * 7 + 3, rows), base)
    # fp32 path on the same (fp32-representable) values agrees
    assert np.array_equal(orc.select_topk_f32(shape, S.astype(np.float32), rows), base)
    # -0 and +0 tie; the lower block wins
    S2 = np.full((1, 1, 64), -1.0)
    S2[0, 0, 9] = 0.0
    S2[0, 0, 4] = -0.0
    shape1 = orc.prefill_shape([0, 1024], 1, 1, 4, 16, 4, 1, 1)
    got = orc.select_topk_f32(shape1, S2.astype(np.float32), [1023])
    assert got[0, 0].tolist() == [0, 4, 63]


def test_select_structure_sorted_unique_within_causal():
    rng = np.random.default_rng(11)
    shape = orc.prefill_shape([0, 700, 1500], 4, 2, 4, 16, 4, 6, 1)
    rows = list(range(1500))
    S = rng.standard_normal((1500, 2, 64))
    sel = orc.select_topk_f64(shape, S, rows)
    cu = [0, 700, 1500]
    for a, r in enumerate(rows):
        b = 0 if r < 700 else 1
        i = (r - cu[b]) // 16
        for g in range(2):
            got = [x for x in sel[a, g] if x >= 0]
            assert got == sorted(set(got))
            assert got[-1] == i and max(got) <= i
            if i > 0:
                assert got[0] == 0


# ------------------------------------------------------------------ main branch


def _masked_dense_torch(Q, K, V, cu, B, rows, sel, scale):
    """Dense scores with every unselected logit at -inf, torch fp64 softmax (independent path)."""
    G = Q.shape[1] // K.shape[1]
    out, lses = [], []
    for a, r in enumerate(rows):
        b = int(np.searchsorted(cu, r, side="right") - 1)
        s0 = int(cu[b])
        pos = r - s0
        keys = torch.arange(s0, r + 1)
        O_r, L_r = [], []
        for h in range(Q.shape[1]):
            g = h // G
            z = (Q[r, h].double() @ K[keys, g].double().T) * scale
            allowed = torch.zeros(len(keys), dtype=torch.bool)
            for j in sel[a, g]:
                if j >= 0:
                    allowed[j * B: (j + 1) * B] = True
            z = z.masked_fill(~allowed[: len(keys)], float("-inf"))
            w = torch.softmax(z, dim=0)
            O_r.append((w @ V[keys, g].double()).numpy())
            L_r.append(torch.logsumexp(z, 0).item())
        out.append(O_r)
        lses.append(L_r)
    return np.array(out), np.array(lses)


def _all_blocks(shape, cu, rows):
    kt = shape.k_tot
    out = np.full((len(rows), shape.Hkv, kt), -1, np.int32)
    for a, r in enumerate(rows):
        b = np.searchsorted(cu, r, side="right") - 1
        i = (r - cu[b]) // shape.B
        for g in range(shape.Hkv):
            out[a, g, : i + 1] = np.arange(i + 1)
    return out


def test_all_causal_blocks_equals_dense():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(k=17)            # k_tot=18 >= 17 blocks
    rows = list(range(shape.T))
    sel = _all_blocks(shape, cu, rows)
    O, L = orc.sparse_attn(shape, Q, K, V, sel, rows)
    Od, Ld = orc.dense_attn(shape, Q, K, V, rows)
    np.testing.assert_allclose(O, Od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Ld, rtol=0, atol=1e-12)


def test_dense_matches_torch_softmax():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(lens=(40, 25))
    rows = [0, 1, 39, 40, 41, 64]
    Od, Ld = orc.dense_attn(shape, Q, K, V, rows)
    sel = _all_blocks(orc.prefill_shape(cu, shape.Hq, shape.Hkv, shape.D, shape.B, shape.d, 10, 0), cu, rows)
    Ot, Lt = _masked_dense_torch(Q, K, V, cu, shape.B, rows, sel, 1 / math.sqrt(shape.D))
    np.testing.assert_allclose(Od, Ot, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Ld, Lt, rtol=0, atol=1e-12)


def test_sparse_equals_masked_dense_formulation():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(sink=1, k=2)
    rows = [3, 20, 36, 37, 80, 150, 230]
    kidx, _ = orc.block_keys(shape, K, Wk)
    qidx, _ = orc.index_query(shape, Q, Wq, rows)
    S = orc.index_scores(shape, qidx, kidx, rows, 17)
    sel = orc.select_topk_f64(shape, S, rows)
    O, L = orc.sparse_attn(shape, Q, K, V, sel, rows)
    Ot, Lt = _masked_dense_torch(Q, K, V, cu, shape.B, rows, sel, 1 / math.sqrt(shape.D))
    np.testing.assert_allclose(O, Ot, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lt, rtol=0, atol=1e-12)


def test_sparse_order_duplicates_and_padding_do_not_matter():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(k=4)
    rows = [120, 150, 230]
    sel = np.array([[[0, 5, 9, 14, -1], [2, 3, 10, 14, -1]],
                    [[1, 2, 8, 14, -1], [0, 1, 2, 14, -1]],
                    [[0, 4, 6, 11, -1], [0, 3, 7, 11, -1]]], np.int32)
    # rows 120/150 are in sequence 1 (start 37): local blocks (120-37)//8=10 and 14; row 230 -> 11
    O, L = orc.sparse_attn(shape, Q, K, V, sel, rows)
    perm = sel[:, :, ::-1].copy()
    O2, L2 = orc.sparse_attn(shape, Q, K, V, perm, rows)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-13)
    dup = sel.copy()
    dup[:, :, 4] = dup[:, :, 0]
    O3, _ = orc.sparse_attn(shape, Q, K, V, dup, rows)
    np.testing.assert_allclose(O3, O, rtol=0, atol=1e-13)


def test_weights_sum_to_one_constant_v_and_zero_q():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(k=3)
    rows = [10, 50, 100, 200]
    rng = np.random.default_rng(0)
    sel = np.full((len(rows), shape.Hkv, shape.k_tot), -1, np.int32)
    for a, r in enumerate(rows):
        b = np.searchsorted(cu, r, side="right") - 1
        i = (r - cu[b]) // shape.B
        for g in range(shape.Hkv):
            pick = sorted(set(rng.choice(i + 1, size=min(3, i + 1), replace=False).tolist()) | {i})
            sel[a, g, : len(pick)] = pick
    Vc = torch.full_like(V, 0.375)                               # sum w = 1  <=>  O = c for V = c
    O, _ = orc.sparse_attn(shape, Q, K, Vc, sel, rows)
    np.testing.assert_allclose(O, 0.375, rtol=0, atol=1e-14)
    Qz = torch.zeros_like(Q)                                     # uniform weights: mean of visible V
    O, L = orc.sparse_attn(shape, Qz, K, V, sel, rows)
    Vf = f64(V)
    for a, r in enumerate(rows):
        b = np.searchsorted(cu, r, side="right") - 1
        s0 = cu[b]
        for g in range(shape.Hkv):
            keys = [s0 + t for j in sel[a, g] if j >= 0 for t in range(j * 8, j * 8 + 8) if s0 + t <= r]
            ref = Vf[keys, g].mean(axis=0)
            G = shape.Hq // shape.Hkv
            for h in range(g * G, (g + 1) * G):
                np.testing.assert_allclose(O[a, h], ref, rtol=0, atol=1e-14)
                assert L[a, h] == pytest.approx(math.log(len(keys)), rel=1e-14)


def test_groups_are_independent():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(k=3)
    rows = list(range(0, shape.T, 7))
    rng = np.random.default_rng(5)
    sel = np.full((len(rows), shape.Hkv, shape.k_tot), -1, np.int32)
    for a, r in enumerate(rows):
        b = np.searchsorted(cu, r, side="right") - 1
        i = (r - cu[b]) // shape.B
        for g in range(shape.Hkv):
            pick = sorted(set(rng.choice(i + 1, size=min(2, i + 1), replace=False).tolist()) | {i})
            sel[a, g, : len(pick)] = pick
    O, L = orc.sparse_attn(shape, Q, K, V, sel, rows)
    G = shape.Hq // shape.Hkv
    # swap the two kv heads together with their query-head groups and block sets
    Qs = torch.cat([Q[:, G:], Q[:, :G]], dim=1)
    Ks, Vs = K.flip(1).contiguous(), V.flip(1).contiguous()
    O2, L2 = orc.sparse_attn(shape, Qs, Ks, Vs, sel[:, ::-1].copy(), rows)
    np.testing.assert_allclose(np.concatenate([O2[:, G:], O2[:, :G]], axis=1), O, rtol=0, atol=1e-14)
    np.testing.assert_allclose(np.concatenate([L2[:, G:], L2[:, :G]], axis=1), L, rtol=0, atol=1e-14)


def test_decode_equals_prefill_last_row():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(lens=(77, 50), k=3, sink=1)
    cache_k = torch.zeros(2, shape.Hkv, 80, shape.D, dtype=torch.bfloat16)
    cache_v = torch.zeros_like(cache_k)
    cache_k[0, :, :77] = K[:77].permute(1, 0, 2)
    cache_k[1, :, :50] = K[77:].permute(1, 0, 2)
    cache_v[0, :, :77] = V[:77].permute(1, 0, 2)
    cache_v[1, :, :50] = V[77:].permute(1, 0, 2)
    qd = torch.stack([Q[76], Q[126]])
    ds = orc.decode_shape([77, 50], 80, 10, shape.Hq, shape.Hkv, shape.D, shape.B, shape.d, 3, 1)
    # index branch
    kp, _ = orc.block_keys(shape, K, Wk)
    kd, _ = orc.block_keys(ds, cache_k, Wk)
    qp, _ = orc.index_query(shape, Q, Wq, [76, 126])
    qdd, _ = orc.index_query(ds, qd, Wq, [0, 1])
    assert np.array_equal(qp, qdd)
    Sp = orc.index_scores(shape, qp, kp, [76, 126], 10)
    Sd = orc.index_scores(ds, qdd, kd, [0, 1], 10)
    np.testing.assert_array_equal(Sp, Sd)
    selp = orc.select_topk_f64(shape, Sp, [76, 126])
    seld = orc.select_topk_f64(ds, Sd, [0, 1])
    assert np.array_equal(selp, seld)
    Op, Lp = orc.sparse_attn(shape, Q, K, V, selp, [76, 126])
    Od, Ld = orc.sparse_attn(ds, qd, cache_k, cache_v, seld, [0, 1])
    np.testing.assert_array_equal(Op, Od)
    np.testing.assert_array_equal(Lp, Ld)


def test_planted_mistakes_are_caught():
    """Mutations planted on the CPU side show that the pins above can see such mistakes."""
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(k=2, sink=1)
    rows = [100, 200]
    kidx, _ = orc.block_keys(shape, K, Wk)
    qidx, _ = orc.index_query(shape, Q, Wq, rows)
    S = orc.index_scores(shape, qidx, kidx, rows, 17)
    sel = orc.select_topk_f64(shape, S, rows)
    O, _ = orc.sparse_attn(shape, Q, K, V, sel, rows)
    Ot, _ = _masked_dense_torch(Q, K, V, cu, shape.B, rows, sel, 1 / math.sqrt(shape.D))
    # a wrong softmax scale (sqrt(D) missing) would be caught by the masked-dense comparison
    Obad, _ = orc.sparse_attn(shape, Q, K, V, sel, rows, scale=1.0)
    assert not np.allclose(Obad, Ot, atol=1e-6)
    np.testing.assert_allclose(O, Ot, atol=1e-12)
    # a reversed tie rule (higher block first) would be caught by the brute-force sort
    Sties = np.zeros_like(S)
    Sties[np.isnan(S)] = np.nan
    got = orc.select_topk_f64(shape, Sties, rows)
    for a, r in enumerate(rows):
        b = np.searchsorted(cu, r, side="right") - 1
        i = (r - cu[b]) // 8
        assert [x for x in got[a, 0] if x >= 0] == sorted({0, 1, 2, i})
