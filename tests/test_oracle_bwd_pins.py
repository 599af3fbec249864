"""Pins of the oracle's main-branch backward (orc_sparse_attn_bwd) against things other than itself.

* torch fp64 autograd of the masked-dense formulation (every unselected or future logit at -inf,
  the chenxutan.com page, section 3.1 stage 3), an independent library path, on selections the
  oracle's own index branch makes (sink, local, partial blocks, several sequences, GQA groups);
* with every causal block selected, torch autograd of plain dense causal GQA attention;
* closed forms: a row that sees a single key passes no gradient to Q; constant keys give dQ = 0
  and constant values give dQ = dK = 0 (the softmax weights' gradients sum to zero).
"""
import math

import numpy as np
import torch

from oracle import oracle as orc
from tests.test_oracle_pins import _all_blocks, _small_prefill, rand_bf16


def _torch_masked_grads(Q, K, V, dO, cu, B, sel, scale, causal_only=False):
    """dQ, dK, dV of sum(O * dO) for the masked formulation, by torch autograd in fp64."""
    Qd = Q.double().clone().requires_grad_(True)
    Kd = K.double().clone().requires_grad_(True)
    Vd = V.double().clone().requires_grad_(True)
    G = Q.shape[1] // K.shape[1]
    loss = 0.0
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        L = s1 - s0
        pos = torch.arange(L)
        causal = pos.view(-1, 1) >= pos.view(1, -1)
        for h in range(Q.shape[1]):
            g = h // G
            allowed = causal.clone()
            if not causal_only:
                blk = torch.zeros(L, L, dtype=torch.bool)
                for r in range(L):
                    for j in sel[s0 + r, g]:
                        if j >= 0:
                            blk[r, j * B: (j + 1) * B] = True
                allowed &= blk
            z = (Qd[s0:s1, h] @ Kd[s0:s1, g].T) * scale
            z = z.masked_fill(~allowed, float("-inf"))
            w = torch.softmax(z, dim=1)
            O = w @ Vd[s0:s1, g]
            loss = loss + (O * dO[s0:s1, h].double()).sum()
    loss.backward()
    return Qd.grad.numpy(), Kd.grad.numpy(), Vd.grad.numpy()


def _selection(shape, Q, K, Wq, Wk):
    rows = np.arange(shape.T)
    kidx, _ = orc.block_keys(shape, K, Wk)
    qidx, _ = orc.index_query(shape, Q, Wq, rows)
    S = orc.index_scores(shape, qidx, kidx, rows, 17)
    return orc.select_topk_f64(shape, S, rows)


def test_bwd_matches_autograd_of_the_masked_formulation():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(seed=11, sink=1, k=2)
    sel = _selection(shape, Q, K, Wq, Wk)
    dO = rand_bf16(Q.shape, 1.0, torch.Generator().manual_seed(12))
    scale = 1 / math.sqrt(shape.D)
    dQ, dK, dV = orc.sparse_attn_bwd(shape, Q, K, V, dO, sel)
    tQ, tK, tV = _torch_masked_grads(Q, K, V, dO, cu, shape.B, sel, scale)
    np.testing.assert_allclose(dQ, tQ, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dK, tK, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dV, tV, rtol=0, atol=1e-11)
    assert np.abs(dQ).max() > 1e-3 and np.abs(dK).max() > 1e-3   # non-trivial gradients


def test_bwd_all_blocks_equals_dense_autograd():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(seed=13, k=17)       # k_tot 18 >= every causal block
    sel = _all_blocks(shape, cu, list(range(shape.T)))
    dO = rand_bf16(Q.shape, 1.0, torch.Generator().manual_seed(14))
    dQ, dK, dV = orc.sparse_attn_bwd(shape, Q, K, V, dO, sel)
    tQ, tK, tV = _torch_masked_grads(Q, K, V, dO, cu, shape.B, None, 1 / math.sqrt(shape.D), causal_only=True)
    np.testing.assert_allclose(dQ, tQ, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dK, tK, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dV, tV, rtol=0, atol=1e-11)


def test_bwd_closed_forms():
    shape, cu, Q, K, V, Wq, Wk = _small_prefill(seed=15, k=3)
    sel = _selection(shape, Q, K, Wq, Wk)
    dO = rand_bf16(Q.shape, 1.0, torch.Generator().manual_seed(16))
    dQ, dK, dV = orc.sparse_attn_bwd(shape, Q, K, V, dO, sel)
    # the first token of every sequence sees only itself: no gradient reaches its query
    for b in range(len(cu) - 1):
        assert np.abs(dQ[cu[b]]).max() < 1e-12
    # constant keys: every weight is equal and dQ = scale * c * sum(dS) = 0
    Kc = torch.ones_like(K) * 0.5
    dQc, _, _ = orc.sparse_attn_bwd(shape, Q, Kc, V, dO, sel)
    assert np.abs(dQc).max() < 1e-12
    # constant values: O = c and dO . v = D for every key, so dS = 0
    Vc = torch.ones_like(V) * 0.25
    dQv, dKv, dVv = orc.sparse_attn_bwd(shape, Q, K, Vc, dO, sel)
    assert np.abs(dQv).max() < 1e-12 and np.abs(dKv).max() < 1e-12
    # dV sums the weights times dO: over all keys of a head it equals the sum of dO of its rows' heads
    G = shape.Hq // shape.Hkv
    for g in range(shape.Hkv):
        np.testing.assert_allclose(dV[:, g].sum(0), dO[:, g * G:(g + 1) * G].double().numpy().sum((0, 1)),
                                   rtol=0, atol=1e-10)
