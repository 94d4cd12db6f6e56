"""MoBA decode: the CUDA path (moba_block_means + moba_decode_attn through the C ABI)
against the oracle's MoBA at the last position (oracle.moba.decode_step)."""
import numpy as np
import pytest
import torch

import query_aware_selective_b200 as qas
from oracle import moba as omoba
from query_aware_selective_b200 import pipeline, synthetic
from tests.parity import ATOL_BF16, max_abs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _check(q, k, v, block, topk, seqs=None):
    """Run one decode step on the GPU and compare sequences `seqs` with the oracle:
    kept blocks exactly (a differing block only inside the 1e-3 score band), outputs
    within the bf16 bar against the oracle's where the kept blocks agree, and for every
    head against the oracle's attention over the GPU's own blocks."""
    b, s, h, d = k.shape
    dec = pipeline.MobaDecode(b, s, h, d, block, topk, device=DEV)
    dec.fill(k)
    o = dec.step(q, k, v).clone()
    blocks = dec.blocks.cpu().numpy().astype(np.int64)
    qas.device_status()
    for bi in (range(b) if seqs is None else seqs):
        kb = k[bi:bi + 1].float().cpu().numpy()
        ref = omoba.decode_step(q[bi:bi + 1].float().cpu().numpy(), kb, v[bi:bi + 1].float().cpu().numpy(),
                                block, topk)
        cur = (s - 1) // block
        kbar = omoba.block_means(kb, block)[0]                   # [H, nb, D]
        agree = np.ones(h, dtype=bool)
        for hh in range(h):
            got, want = blocks[bi, hh], ref["blocks"][0, 0, hh]
            if np.array_equal(got, want):
                continue
            agree[hh] = False
            sc = kbar[hh, :cur] @ q[bi, 0, hh].float().cpu().numpy().astype(np.float64)
            kth = np.sort(sc)[::-1][min(topk, cur) - 1]
            for blk in set(got.tolist()) ^ set(want.tolist()):
                assert abs(sc[blk] - kth) <= 1e-3 * abs(kth) + 1e-6, (bi, hh, got, want)
        got_o = o[bi, 0].float().cpu().numpy()                     # [H, D]
        if agree.any():
            assert max_abs(got_o[agree], ref["o"][0, 0][agree]) <= ATOL_BF16
        # every head, swapped gates included: attention over the GPU's own blocks
        # the oracle reads the query at position s - 1 only; a broadcast view stands in
        # for the rest of the rows
        q_at = np.broadcast_to(q[bi:bi + 1].float().cpu().numpy().astype(np.float64), (1, s, h, d))
        own_o, _ = omoba.attend(q_at, kb, v[bi:bi + 1].float().cpu().numpy(), blocks[bi][None, None], block,
                                positions=[s - 1])
        assert max_abs(got_o, own_o[0, 0]) <= ATOL_BF16


@pytest.mark.parametrize("batch,seq,heads,block,topk", [
    (2, 8192, 8, 1024, 3),      # 7 past blocks, top-3
    (3, 5000, 4, 256, 5),       # ragged last block, top-5 of 19
    (2, 700, 2, 1024, 3),       # no past block: the current block only
    (1, 2048, 4, 512, 5),       # fewer past blocks (3) than topk: all kept
])
def test_moba_decode_parity(batch, seq, heads, block, topk):
    w = synthetic.MOBA_DECODE_64K
    inp = synthetic.make_moba_decode_inputs(w, device=DEV, seq=seq, batch=batch)
    q, k, v = inp["q"][:, :, :heads].contiguous(), inp["k"][:, :, :heads].contiguous(), \
        inp["v"][:, :, :heads].contiguous()
    _check(q, k, v, block, topk)


def test_moba_decode_64k_batch16_sampled():
    w = synthetic.MOBA_DECODE_64K
    inp = synthetic.make_moba_decode_inputs(w, device=DEV)
    _check(inp["q"], inp["k"], inp["v"], w.block, w.topk, seqs=(0, 15))
    del inp
    torch.cuda.empty_cache()
