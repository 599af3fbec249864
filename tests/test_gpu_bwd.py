"""GPU parity of the main-branch backward (msa_sparse_attn_prefill_bwd) against the fp64 oracle.

The forward runs on the GPU (its block selection, bf16 O and fp32 LSE feed the backward, as in a
training step); the oracle recomputes the forward in double on the same selection and forms dQ,
dK, dV from the gradient of softmax attention.  Tolerance (per gradient tensor): relative L2
error <= 1e-2 and max-abs error <= 2e-2 of the tensor's largest magnitude -- the GPU rounds the
weights p and dS to bf16 before its tensor-core products and takes D = dO . O from the bf16 O,
each a relative error near 2^-9 per term.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_scores_b200 import msa
from block_sparse_long_scores_b200.pipeline import Prefill
from block_sparse_long_scores_b200.workloads import WORKLOADS, make_inputs, scaled_down
from oracle import oracle as orc
from tests.parity_helpers import Guards, cpu, oracle_shape

pytestmark = pytest.mark.gpu
DEV = "cuda"
RL2_GRAD = 1e-2
MAXREL_GRAD = 2e-2


def check_grad(got: np.ndarray, ref: np.ndarray, what: str):
    got = got.astype(np.float64)
    scale = float(np.abs(ref).max())
    rl2 = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    mx = float(np.abs(got - ref).max()) / max(scale, 1e-300)
    assert rl2 <= RL2_GRAD, f"{what}: relative L2 {rl2:.3e}"
    assert mx <= MAXREL_GRAD, f"{what}: max-abs {mx:.3e} of the largest magnitude"
    return rl2, mx


def _run(w, x, seed, row_split=None):
    pf = Prefill(w, x)
    pf.run()
    T = pf.shape.total_rows
    g = torch.Generator(device="cpu").manual_seed(seed)
    d_o = torch.randn(x["q"].shape, generator=g).to(torch.bfloat16).to(DEV)
    guards = Guards()
    dq = guards.wrap(torch.zeros(x["q"].shape, dtype=torch.float32, device=DEV), "dq")
    dk = guards.wrap(torch.zeros(x["k"].shape, dtype=torch.float32, device=DEV), "dk")
    dv = guards.wrap(torch.zeros(x["v"].shape, dtype=torch.float32, device=DEV), "dv")
    n = msa.msa_sparse_attn_prefill_bwd(pf.cfg, pf.shape, None, None, None, None, None, None, None, 0, T,
                                        None, None, None, None)
    ws = guards.wrap(torch.empty(max(n, 256), dtype=torch.uint8, device=DEV), "workspace")
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    bounds = [0, T] if row_split is None else [0, row_split, T]
    for r0, r1 in zip(bounds[:-1], bounds[1:]):   # row ranges accumulate into the same outputs
        msa.msa_sparse_attn_prefill_bwd(pf.cfg, pf.shape, x["q"], x["k"], x["v"], pf.o, pf.lse, d_o,
                                        pf.block_idx[r0:r1], r0, r1, dq, dk, dv, ws, err)
    torch.cuda.synchronize()
    guards.check()
    assert int(err.item()) == 0 and int(pf.err.item()) == 0
    xc = cpu(x)
    sh = oracle_shape(w, xc)
    dQ, dK, dV = orc.sparse_attn_bwd(sh, xc["q"], xc["k"], xc["v"], d_o.cpu(), pf.block_idx.cpu().numpy())
    return [check_grad(dq.cpu().numpy(), dQ, "dQ"), check_grad(dk.cpu().numpy(), dK, "dK"),
            check_grad(dv.cpu().numpy(), dV, "dV")]


def test_bwd_tiny_prefill():
    w = WORKLOADS["tiny_prefill"]
    _run(w, make_inputs(w, device=DEV, seed=40), seed=41)


@pytest.mark.parametrize("gain", [1.0, 11.3137])
def test_bwd_128k_shape(gain):
    # the 128K workload's heads and selection (G 8, D 128, B 64, sink) at 3000 rows; N(0,1) q, k too
    w = scaled_down(WORKLOADS["prefill_128k"], (3000,))
    _run(w, make_inputs(w, device=DEV, seed=42, logit_gain=gain), seed=43)


def test_bwd_ragged_shape_with_ties_in_row_ranges():
    # ragged workload shape (D 64, B 128, G 8, discrete index keys), the rows in two calls
    w = scaled_down(WORKLOADS["ragged_prefill"], (130, 2100, 64, 900))
    _run(w, make_inputs(w, device=DEV, seed=44), seed=45, row_split=1500)


def test_bwd_in_subchunks_and_small_k():
    # sub-chunks of 700 rows inside one call; k = 3 with sink over several sequences
    w = scaled_down(WORKLOADS["tiny_prefill"], (1200, 5, 900)).with_(n_topk=3, use_sink=1)
    msa.prefill_set_subchunk_rows(700)
    try:
        _run(w, make_inputs(w, device=DEV, seed=46), seed=47)
    finally:
        msa.prefill_set_subchunk_rows(0)
