"""Per-head selection variant: the CUDA path through the C ABI against the oracle
(oracle/esa_heads.py). Selection per group of compressed columns, attention with
one key list per KV head, and the whole per-head decode and prefill paths."""
import math

import numpy as np
import pytest
import torch

import query_aware_selective_b200 as qas
from oracle import esa as oesa
from oracle import esa_heads as oh
from query_aware_selective_b200 import pipeline, synthetic
from tests.parity import ATOL_BF16, ATOL_F32, check_selection, max_abs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _rand(shape, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype)


@pytest.mark.parametrize("batch,lq,n_cap,dc,ng,n_init,window,topk,eps,clamp", [
    (3, 1, 6000, 128, 8, 128, 512, 300, 2, 45.25),     # decode shape: 8 groups of 16 columns
    (1, 1, 2048, 16, 4, 16, 256, 128, 2, 16.0),        # tiny decode: 4 groups of 4 columns
    (2, 3, 3000, 64, 4, 8, 100, 77, 1, 10.0),          # a few queries (register path)
    (2, 1, 4000, 128, 2, 32, 300, 500, 3, math.inf),   # 2 groups, no clamp
    (1, 64, 4096, 128, 8, 128, 512, 1024, 2, 45.25),   # a chunk (tiled path per group)
    (2, 130, 3000, 128, 8, 16, 300, 200, 2, 8.0),      # ragged chunk
    (5, 1, 5000, 128, 8, 32, 300, 400, 2, 45.25),      # 40 selections in flight
    (10, 1, 3000, 128, 8, 32, 300, 200, 2, 45.25),     # 80 selections
    (40, 1, 2000, 128, 8, 32, 200, 100, 2, 45.25),     # 320 selections (more clusters than fit at once)
])
def test_score_select_heads_parity(batch, lq, n_cap, dc, ng, n_init, window, topk, eps, clamp):
    p = qas.params(n_init, window, topk, eps, clamp)
    c0 = n_cap - lq
    q_c = _rand((batch, lq, dc), 51 + lq)
    k_c = _rand((batch, n_cap, dc), 52 + lq)
    idx, cnt, sp = qas.score_select_heads(q_c.to(DEV), k_c.to(DEV), c0, ng, p, want_scores=True)
    ref_idx, ref_cnt, ref_sp = oh.score_select_heads(q_c.double().numpy(), k_c.double().numpy(), c0, ng, n_init,
                                                     window, topk, eps, clamp)
    _, (m0, m1), _ = oesa.regions(c0, c0 + lq, n_init, window)
    idx, cnt, sp = idx.cpu().numpy(), cnt.cpu().numpy(), sp.cpu().double().numpy()
    for b in range(batch):
        for g in range(ng):
            check_selection(idx[b, g], cnt[b, g], ref_idx[b, g], ref_cnt[b, g], ref_sp[b][g], m0, topk)
            if m1 > m0:
                scale = max(1.0, float(np.abs(ref_sp[b][g]).max()))
                assert float(np.abs(sp[b, g] - ref_sp[b][g]).max()) <= 1e-4 * scale


def _per_head_lists(batch, hkv, m0, m1, topk, seed, shrink=17):
    """Valid per-head selections with counts that differ between heads."""
    idx = torch.full((batch, hkv, topk), -1, dtype=torch.int32)
    cnt = torch.zeros((batch, hkv), dtype=torch.int32)
    gen = torch.Generator().manual_seed(seed)
    n = max(0, m1 - m0)
    for b in range(batch):
        for g in range(hkv):
            c = max(0, min(topk, n) - shrink * ((b + g) % 4))
            sel = torch.randperm(n, generator=gen)[:c].sort().values + m0
            idx[b, g, :c] = sel.to(torch.int32)
            cnt[b, g] = c
    return idx, cnt


@pytest.mark.parametrize("batch,lq,n_cap,hq,hkv,d,dtype,n_init,window,topk", [
    (4, 1, 5000, 32, 8, 128, torch.bfloat16, 128, 1024, 700),   # decode, bulk-copy kernel per (sequence, head)
    (2, 1, 3000, 16, 4, 128, torch.bfloat16, 32, 256, 333),     # G = 4 with 4 KV heads
    (1, 1, 2048, 4, 4, 64, torch.float32, 16, 256, 128),        # fp32, head dim 64 (SIMT)
    (2, 2, 3000, 16, 2, 64, torch.bfloat16, 32, 256, 300),      # GQA 8 (SIMT)
    (1, 128, 2048, 8, 2, 128, torch.bfloat16, 16, 256, 256),    # a chunk (tensor cores, staged rows)
])
def test_sparse_attn_heads_parity(batch, lq, n_cap, hq, hkv, d, dtype, n_init, window, topk):
    p = qas.params(n_init, window, topk, 2, 10.0)
    c0 = n_cap - lq
    q = _rand((batch, lq, hq, d), 61, dtype)
    k = _rand((batch, n_cap, hkv, d), 62, dtype)
    v = _rand((batch, n_cap, hkv, d), 63, dtype)
    _, (m0, m1), _ = oesa.regions(c0, c0 + lq, n_init, window)
    idx, cnt = _per_head_lists(batch, hkv, m0, m1, topk, seed=64)
    o, lse = qas.sparse_attn_heads(q.to(DEV), k.to(DEV), v.to(DEV), c0, idx.to(DEV), cnt.to(DEV), p, want_lse=True)
    ref_o, ref_lse = oh.sparse_attn_heads(q.float().numpy(), k.float().numpy(), v.float().numpy(), c0,
                                          idx.numpy(), cnt.numpy(), n_init, window)
    atol = ATOL_F32 if dtype == torch.float32 else ATOL_BF16
    assert max_abs(o.cpu().double().numpy(), ref_o) <= atol
    assert max_abs(lse.cpu().numpy(), ref_lse) <= 1e-3


def test_equal_per_head_lists_match_the_merged_call():
    # the same list for every KV head: esa_sparse_attn_heads == esa_sparse_attn
    b, n, hq, hkv = 3, 4000, 32, 8
    p = qas.params(64, 512, 300, 2, 10.0)
    c0 = n - 1
    q = _rand((b, 1, hq, 128), 71, torch.bfloat16).to(DEV)
    k = _rand((b, n, hkv, 128), 72, torch.bfloat16).to(DEV)
    v = _rand((b, n, hkv, 128), 73, torch.bfloat16).to(DEV)
    _, (m0, m1), _ = oesa.regions(c0, c0 + 1, 64, 512)
    idx, cnt = synthetic.random_index_list(b, m0, m1, 300, seed=74)
    o1, _ = qas.sparse_attn(q, k, v, c0, idx.to(DEV), cnt.to(DEV), p)
    o2, _ = qas.sparse_attn_heads(q, k, v, c0, idx[:, None].repeat(1, hkv, 1).contiguous().to(DEV),
                                  cnt[:, None].repeat(1, hkv).contiguous().to(DEV), p)
    assert max_abs(o1.cpu().double().numpy(), o2.cpu().double().numpy()) <= 2e-3


def _decode_heads(w, n_ctx, batch, seqs):
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    inp = synthetic.make_esa_inputs(w, device=DEV, n_ctx=n_ctx, batch=batch)
    wq_g, wk_g = synthetic.make_group_maps(w, device=DEV)
    wq, wk = pipeline.block_diagonal(wq_g), pipeline.block_diagonal(wk_g)
    n = inp["k"].shape[1]
    dec = pipeline.EsaDecode(batch, n, w.hq, w.hkv, w.head_dim, w.d_c, p, dtype=w.torch_dtype, device=DEV,
                             per_head=True)
    dec.fill_cache(inp["k"], wk)
    o = dec.step(inp["q"], inp["k"], inp["v"], wq, wk).clone()
    idx, cnt = dec.idx.cpu().numpy(), dec.count.cpu().numpy()
    qas.device_status()
    _, (m0, _), _ = oesa.regions(n - 1, n, w.n_init, w.window)
    for b in seqs:
        ref = oh.decode_step_heads(inp["q"][b:b + 1].float().cpu().numpy(), inp["k"][b:b + 1].float().cpu().numpy(),
                                   inp["v"][b:b + 1].float().cpu().numpy(), wq_g.cpu().numpy(),
                                   wk_g.cpu().numpy(), w.n_init, w.window, w.topk, w.eps, w.clamp_c)
        for g in range(w.hkv):
            check_selection(idx[b, g], cnt[b, g], ref["idx"][0, g], ref["count"][0, g], ref["s_prime"][0][g], m0,
                            w.topk)
        atol = ATOL_F32 if w.dtype == "f32" else ATOL_BF16
        assert max_abs(o[b:b + 1].cpu().double().numpy(), ref["o"]) <= atol
    return dec


def test_per_head_decode_tiny():
    _decode_heads(synthetic.TINY_DECODE, None, 1, seqs=(0,))


def test_per_head_decode_llama_shape():
    _decode_heads(synthetic.DECODE_128K, 12000, 3, seqs=(0, 2))


def test_per_head_prefill_chunks():
    # chunked prefill with per-head selection; chunks past the window compared
    w = synthetic.PREFILL_32K
    n, chunk = 6144, 512
    p = qas.params(w.n_init, 1024, 512, w.eps, w.clamp_c)
    inp = synthetic.make_esa_inputs(w, device=DEV, n_ctx=n)
    wq_g, wk_g = synthetic.make_group_maps(w, device=DEV)
    wq, wk = pipeline.block_diagonal(wq_g), pipeline.block_diagonal(wk_g)
    pf = pipeline.EsaPrefill(1, n, chunk, w.hq, w.hkv, w.head_dim, w.d_c, p, device=DEV, per_head=True)
    out = pf.run(inp["q"], inp["k"], inp["v"], wq, wk).clone()
    qas.device_status()
    q, k, v = (inp[x].float().cpu().numpy() for x in ("q", "k", "v"))
    k_c = np.stack([oh.compress_heads(k[0], wk_g.cpu().numpy(), w.hq)])
    for c0 in (4096, n - chunk):
        qc = oh.compress_heads(q[0, c0:c0 + chunk], wq_g.cpu().numpy(), w.hq)[None]
        idx, cnt, _ = oh.score_select_heads(qc, k_c, c0, w.hkv, w.n_init, 1024, 512, w.eps, w.clamp_c)
        rows = [(0, i) for i in (0, 1, 255, chunk - 1)]
        ref_o, _ = oh.sparse_attn_heads(q[:, c0:c0 + chunk], k, v, c0, idx, cnt, w.n_init, 1024, rows=rows)
        got = out[:, c0:c0 + chunk].float().cpu().numpy()
        for _, i in rows:
            assert max_abs(got[0, i], ref_o[0, i]) <= ATOL_BF16
