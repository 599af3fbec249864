"""The allocation-free decode entry point (msa_sparse_attn_decode_noalloc).

Some callers cannot pass the library a workspace -- their device memory belongs to another
allocator, or their decode step must not call the CUDA allocator -- so the library offers a
decode call whose scratch is a fixed device array it declares itself.  This file checks, through
the C ABI, that the call gives the same output as the workspace-taking msa_sparse_attn_decode
(within the parity tolerances) on two calls in a row, since every call reuses the same scratch,
and that both match the fp64 oracle on the same selection.
It is named to be collected last, and works in a fresh process (where the first call performs
the one-time address look-up) as well as after the other tests.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_scores_b200 import msa
from block_sparse_long_scores_b200.pipeline import Decode
from block_sparse_long_scores_b200.workloads import WORKLOADS, make_inputs, scaled_down
from oracle import oracle as orc
from tests.parity_helpers import check_attention, cpu, oracle_shape

pytestmark = pytest.mark.gpu


def _decode_inputs(seed):
    w = scaled_down(WORKLOADS["decode_128k"], (1, 70, 4096, 2500, 64, 3001))
    x = make_inputs(w, device="cuda", seed=seed)
    dc = Decode(w, x)
    dc.run()                      # index branch + selection + reference attention with a workspace
    torch.cuda.synchronize()
    return w, x, dc


def test_noalloc_decode_matches_workspace_decode_twice():
    w, x, dc = _decode_inputs(11)
    ref_o = dc.o.double().cpu().numpy()
    ref_lse = dc.lse.double().cpu().numpy()
    xc = cpu(x)
    O_orc, L_orc = orc.sparse_attn(oracle_shape(w, xc), xc["q"], xc["k"], xc["v"], dc.block_idx.cpu().numpy(),
                                   np.arange(w.batch))
    check_attention(ref_o, O_orc, ref_lse, L_orc)
    for _ in range(2):
        o = torch.full_like(dc.o, float("nan"))
        lse = torch.full_like(dc.lse, float("nan"))
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        msa.msa_sparse_attn_decode_noalloc(dc.cfg, dc.shape, x["q"], x["k"], x["v"], dc.block_idx, o, lse, err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        check_attention(o.float().cpu().numpy(), ref_o, lse.cpu().numpy(), ref_lse)
        check_attention(o.float().cpu().numpy(), O_orc, lse.cpu().numpy(), L_orc)


def test_noalloc_decode_second_problem_after_first():
    # a different problem right after: nothing left in the shared scratch may leak into it
    _, _, dc1 = _decode_inputs(12)
    w, x, dc2 = _decode_inputs(13)
    o = torch.empty_like(dc2.o)
    lse = torch.empty_like(dc2.lse)
    msa.msa_sparse_attn_decode_noalloc(dc1.cfg, dc1.shape, dc1.x["q"], dc1.x["k"], dc1.x["v"], dc1.block_idx,
                                       torch.empty_like(dc1.o), None)
    msa.msa_sparse_attn_decode_noalloc(dc2.cfg, dc2.shape, x["q"], x["k"], x["v"], dc2.block_idx, o, lse)
    torch.cuda.synchronize()
    check_attention(o.float().cpu().numpy(), dc2.o.double().cpu().numpy(), lse.cpu().numpy(),
                    dc2.lse.double().cpu().numpy())


def test_noalloc_decode_rejects_problems_beyond_its_scratch():
    # 4096 short sequences x 4 kv heads x 66 slots make ~140 MiB of split partials: refused before
    # any pointer is used, nothing launched
    nseq = 4096
    w = WORKLOADS["decode_128k"].with_(seqlens=(64,) * nseq)
    cfg = msa.make_config(w.Hq, w.Hkv, w.D, w.B, w.d, w.n_topk, w.use_sink)
    seqlens = torch.full((nseq,), 64, dtype=torch.int32, device="cuda")
    shape = msa.decode_shape(seqlens, nseq, 64, w.B)
    fake = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(msa.MSAError) as ei:
        msa.msa_sparse_attn_decode_noalloc(cfg, shape, fake, fake, fake, fake, fake, None)
    assert ei.value.code == 3
