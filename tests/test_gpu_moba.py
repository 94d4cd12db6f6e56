"""MoBA parity: the CUDA path through the C ABI against the CPU oracle."""
import numpy as np
import pytest
import torch

import query_aware_selective_b200 as qas
from oracle import moba as omoba
from query_aware_selective_b200 import synthetic
from tests.parity import ATOL_BF16, max_abs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def _np(t):
    return t.detach().cpu().double().numpy()


def _gate_check(q, k, block, topk, got_blocks):
    """Gate choices per (query, head): same count and order rules as the oracle,
    and any difference only among blocks whose score ties the k-th within 1e-3."""
    kbar = omoba.block_means(_np(k), block)
    ref = omoba.gate(_np(q), kbar, block, topk)
    got = got_blocks.cpu().numpy().astype(np.int64)
    assert got.shape == ref.shape
    qn = _np(q)
    b_, s_, h_ = ref.shape[:3]
    same = np.all(got == ref, axis=-1)
    swaps = 0
    for b, p, h in zip(*np.nonzero(~same)):
        cur = p // block
        g_list = [x for x in got[b, p, h] if x >= 0]
        r_list = [x for x in ref[b, p, h] if x >= 0]
        assert g_list[-1] == cur and len(g_list) == len(r_list)
        assert g_list == sorted(g_list)
        sc = kbar[b, h, :cur] @ qn[b, p, h]
        kth = np.sort(sc)[::-1][len(r_list) - 2]
        for blk in set(g_list) ^ set(r_list):
            assert abs(sc[blk] - kth) <= 1e-3 * abs(kth) + 1e-6, (p, h, blk, sc[blk], kth)
        swaps += 1
    return same


@pytest.mark.parametrize("s,h,block,topk", [
    (2048, 4, 128, 3),
    (1000, 2, 64, 2),      # ragged last block, block smaller than a 128-row tile
    (1536, 2, 256, 15),
])
def test_gate_parity(s, h, block, topk):
    q, k = _rand((1, s, h, 128), 1), _rand((1, s, h, 128), 2)
    blocks = qas.moba_block_gate(q.to(DEV), k.to(DEV), block, topk)
    same = _gate_check(q, k, block, topk, blocks)
    assert same.mean() > 0.99


@pytest.mark.parametrize("b,s,h,block,topk", [
    (1, 1024, 2, 128, 3),
    (2, 700, 2, 128, 2),     # ragged
    (1, 512, 3, 64, 4),      # block < 128 rows
    (1, 1024, 1, 256, 1),
])
def test_block_attn_parity(b, s, h, block, topk):
    q, k, v = _rand((b, s, h, 128), 3), _rand((b, s, h, 128), 4), _rand((b, s, h, 128), 5)
    blocks = synthetic.random_block_lists(b, s, h, block, topk, seed=6)
    o, lse = qas.moba_block_attn(q.to(DEV), k.to(DEV), v.to(DEV), block, topk, blocks.to(DEV), want_lse=True)
    ref_o, ref_lse = omoba.attend(_np(q), _np(k), _np(v), blocks.numpy().astype(np.int64), block)
    assert max_abs(_np(o), ref_o) <= ATOL_BF16
    assert max_abs(lse.cpu().numpy(), ref_lse) <= 2e-2


def test_no_past_block_is_block_local():
    s, h, block = 512, 2, 128
    q, k, v = _rand((1, s, h, 128), 7), _rand((1, s, h, 128), 8), _rand((1, s, h, 128), 9)
    o, _, blocks = qas.moba_block_gate_attn(q.to(DEV), k.to(DEV), v.to(DEV), block, 0, want_blocks=True)
    assert torch.all(blocks[..., 0].cpu() == (torch.arange(s) // block).to(torch.int16).view(1, s, 1))
    pos = torch.arange(s)
    mask = ((pos.view(s, 1) // block) == (pos.view(1, s) // block)) & (pos.view(1, s) <= pos.view(s, 1))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().permute(0, 2, 1, 3), k.double().permute(0, 2, 1, 3), v.double().permute(0, 2, 1, 3),
        attn_mask=mask).permute(0, 2, 1, 3)
    assert max_abs(_np(o), ref.numpy()) <= ATOL_BF16


def test_all_blocks_is_full_attention():
    s, h, block = 640, 2, 128
    q, k, v = _rand((1, s, h, 128), 10), _rand((1, s, h, 128), 11), _rand((1, s, h, 128), 12)
    o, _, _ = qas.moba_block_gate_attn(q.to(DEV), k.to(DEV), v.to(DEV), block, 15)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().permute(0, 2, 1, 3), k.double().permute(0, 2, 1, 3), v.double().permute(0, 2, 1, 3),
        is_causal=True).permute(0, 2, 1, 3)
    assert max_abs(_np(o), ref.numpy()) <= ATOL_BF16


def test_gate_attn_end_to_end():
    s, h, block, topk = 2048, 2, 256, 3
    q, k, v = _rand((1, s, h, 128), 13), _rand((1, s, h, 128), 14), _rand((1, s, h, 128), 15)
    o, lse, blocks = qas.moba_block_gate_attn(q.to(DEV), k.to(DEV), v.to(DEV), block, topk, want_blocks=True,
                                              want_lse=True)
    same = _gate_check(q, k, block, topk, blocks)
    ref = omoba.moba(_np(q), _np(k), _np(v), block, topk)
    got, got_lse = _np(o), lse.cpu().numpy()
    assert same.mean() > 0.99
    # rows whose gate agrees with the oracle's: the oracle's end-to-end output
    assert max_abs(got[same], ref["o"][same]) <= ATOL_BF16
    assert max_abs(got_lse[same], ref["lse"][same]) <= 2e-2
    # every row, those whose gate swapped a block inside the tie band included: the
    # oracle's attention over the GPU's own block lists (the article's
    # Softmax(q K[I]^T) V[I] over the set the gate chose)
    own_o, own_lse = omoba.attend(_np(q), _np(k), _np(v), blocks.cpu().numpy().astype(np.int64), block)
    assert max_abs(got, own_o) <= ATOL_BF16
    assert max_abs(got_lse, own_lse) <= 2e-2
    qas.device_status()
