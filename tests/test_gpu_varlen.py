"""Variable-length decode batches: the CUDA path through the C ABI against the oracle
(oracle/esa_varlen.py). Each sequence holds its own number of cached tokens and its
query sits at its last position; lengths live on the device."""
import numpy as np
import pytest
import torch

import query_aware_selective_b200 as qas
from oracle import esa as oesa
from oracle import esa_varlen as ov
from query_aware_selective_b200 import pipeline, synthetic
from tests.parity import ATOL_BF16, ATOL_F32, check_selection, max_abs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _rand(shape, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype)


def _mid(n, n_init, window):
    c0 = n - 1
    lo = synthetic.local_start(c0, n_init, window)
    return n_init, max(n_init, lo)


@pytest.mark.parametrize("n_cap,dc,ng,lens,n_init,window,topk,eps,clamp", [
    # full length, ragged, shorter middle than topk, no middle, a single token
    (6000, 128, 1, [6000, 4321, 900, 350, 1], 128, 512, 300, 2, 45.25),
    (3000, 64, 1, [3000, 2999, 2048, 700], 16, 256, 77, 1, 10.0),
    (5000, 128, 8, [5000, 2600, 1200, 40], 32, 300, 400, 2, 45.25),        # per-head groups
    (20000, 128, 1, [20000, 19000, 5000, 16500, 300, 12000, 8000, 20000], 64, 1024, 2048, 2, 45.25),
    (2048, 16, 4, [2048, 1111, 300], 16, 256, 128, 2, 16.0),
])
def test_score_select_varlen_parity(n_cap, dc, ng, lens, n_init, window, topk, eps, clamp):
    p = qas.params(n_init, window, topk, eps, clamp)
    b = len(lens)
    q_c = _rand((b, 1, dc), 81)
    k_c = _rand((b, n_cap, dc), 82)
    seq_len = torch.tensor(lens, dtype=torch.int64)
    idx, cnt, sp = qas.score_select_varlen(q_c.to(DEV), k_c.to(DEV), seq_len.to(DEV), p, n_groups=ng,
                                           want_scores=True)
    qas.device_status()
    ref_idx, ref_cnt, ref_sp = ov.score_select_varlen(q_c.double().numpy(), k_c.double().numpy(), lens, n_init,
                                                      window, topk, eps, clamp, n_groups=ng)
    idx, cnt, sp = idx.cpu().numpy(), cnt.cpu().numpy(), sp.cpu().double().numpy()
    for bi, n in enumerate(lens):
        m0, m1 = _mid(n, n_init, window)
        for g in range(ng):
            check_selection(idx[bi, g], cnt[bi, g], ref_idx[bi, g], ref_cnt[bi, g], ref_sp[bi][g], m0, topk)
            if m1 > m0:
                want = ref_sp[bi][g]
                scale = max(1.0, float(np.abs(want).max()))
                assert float(np.abs(sp[bi, g, :m1 - m0] - want).max()) <= 1e-4 * scale


def _lists(lens, lists, n_init, window, topk, seed):
    """Valid selections per sequence (and per KV head), drawn from each sequence's
    own middle, with counts that differ between lists."""
    gen = torch.Generator().manual_seed(seed)
    b = len(lens)
    idx = torch.full((b, lists, topk), -1, dtype=torch.int32)
    cnt = torch.zeros((b, lists), dtype=torch.int32)
    for bi, n in enumerate(lens):
        m0, m1 = _mid(n, n_init, window)
        for g in range(lists):
            c = max(0, min(topk, m1 - m0) - 13 * ((bi + g) % 3))
            sel = torch.randperm(m1 - m0, generator=gen)[:c].sort().values + m0
            idx[bi, g, :c] = sel.to(torch.int32)
            cnt[bi, g] = c
    return idx, cnt


@pytest.mark.parametrize("n_cap,hq,hkv,d,dtype,lists,lens,n_init,window,topk", [
    (6000, 32, 8, 128, torch.bfloat16, 1, [6000, 3500, 800, 1], 128, 1024, 700),      # bulk-copy decode kernel
    (5000, 32, 8, 128, torch.bfloat16, 8, [5000, 2222, 90], 64, 512, 500),            # per KV head lists (rows)
    (3000, 16, 4, 128, torch.bfloat16, 1, [3000, 1000, 2999], 32, 256, 333),          # G = 4, 4 KV heads
    (2048, 4, 4, 64, torch.float32, 1, [2048, 700, 300, 64], 16, 256, 128),           # fp32, head dim 64 (SIMT)
    (3000, 16, 2, 64, torch.bfloat16, 2, [3000, 1500], 32, 256, 300),                 # GQA 8, per head (SIMT)
])
def test_sparse_attn_varlen_parity(n_cap, hq, hkv, d, dtype, lists, lens, n_init, window, topk):
    p = qas.params(n_init, window, topk, 2, 10.0)
    b = len(lens)
    q = _rand((b, 1, hq, d), 91, dtype)
    k = _rand((b, n_cap, hkv, d), 92, dtype)
    v = _rand((b, n_cap, hkv, d), 93, dtype)
    idx, cnt = _lists(lens, lists, n_init, window, topk, seed=94)
    seq_len = torch.tensor(lens, dtype=torch.int64)
    o, lse = qas.sparse_attn_varlen(q.to(DEV), k.to(DEV), v.to(DEV), seq_len.to(DEV), idx.to(DEV), cnt.to(DEV), p,
                                    want_lse=True)
    qas.device_status()
    ref_o, ref_lse = ov.sparse_attn_varlen(q.float().numpy(), k.float().numpy(), v.float().numpy(), lens,
                                           idx.numpy(), cnt.numpy(), n_init, window)
    atol = ATOL_F32 if dtype == torch.float32 else ATOL_BF16
    assert max_abs(o.cpu().double().numpy(), ref_o) <= atol
    assert max_abs(lse.cpu().numpy(), ref_lse) <= 1e-3


def test_equal_lengths_match_the_batch_calls():
    # every length = n_cap: the variable-length calls give the equal-length results
    b, n = 3, 4000
    p = qas.params(64, 512, 300, 2, 45.25)
    q_c = _rand((b, 1, 128), 101).to(DEV)
    k_c = _rand((b, n, 128), 102).to(DEV)
    seq_len = torch.full((b,), n, dtype=torch.int64, device=DEV)
    i1, c1, _ = qas.score_select_varlen(q_c, k_c, seq_len, p)
    i2, c2, _ = qas.score_select(q_c, k_c, n - 1, p)
    assert torch.equal(i1[:, 0].cpu(), i2.cpu()) and torch.equal(c1[:, 0].cpu(), c2.cpu())
    q = _rand((b, 1, 32, 128), 103, torch.bfloat16).to(DEV)
    k = _rand((b, n, 8, 128), 104, torch.bfloat16).to(DEV)
    v = _rand((b, n, 8, 128), 105, torch.bfloat16).to(DEV)
    o1, _ = qas.sparse_attn_varlen(q, k, v, seq_len, i1, c1, p)
    o2, _ = qas.sparse_attn(q, k, v, n - 1, i2, c2, p)
    assert torch.equal(o1.cpu(), o2.cpu())


def _decode(per_head, n_cap, lens, seqs):
    w = synthetic.DECODE_128K
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    b = len(lens)
    inp = synthetic.make_esa_inputs(w, device=DEV, n_ctx=n_cap, batch=b)
    if per_head:
        wq_g, wk_g = synthetic.make_group_maps(w, device=DEV)
        wq, wk = pipeline.block_diagonal(wq_g), pipeline.block_diagonal(wk_g)
    else:
        wq, wk = inp["wq"], inp["wk"]
    seq_len = torch.tensor(lens, dtype=torch.int64)
    dec = pipeline.EsaDecodeVarlen(b, n_cap, w.hq, w.hkv, w.head_dim, w.d_c, p, device=DEV, per_head=per_head)
    dec.fill_cache(inp["k"], wk, lens)
    pos = (seq_len - 1).to(DEV)
    k_new = inp["k"][torch.arange(b, device=DEV), pos].contiguous()           # [B, Hkv, D]
    o = dec.step(inp["q"], k_new, inp["k"], inp["v"], wq, wk, seq_len.to(DEV)).clone()
    idx, cnt = dec.idx.cpu().numpy(), dec.count.cpu().numpy()
    kc_last = dec.k_c[torch.arange(b, device=DEV), pos].cpu().double().numpy()
    qas.device_status()
    q, k, v = (inp[x].float().cpu().numpy() for x in ("q", "k", "v"))
    for bi in seqs:
        n = lens[bi]
        m0, _ = _mid(n, w.n_init, w.window)
        if per_head:
            from oracle import esa_heads as oh
            ref = oh.decode_step_heads(q[bi:bi + 1], k[bi:bi + 1, :n], v[bi:bi + 1, :n], wq_g.cpu().numpy(),
                                       wk_g.cpu().numpy(), w.n_init, w.window, w.topk, w.eps, w.clamp_c)
            for g in range(w.hkv):
                check_selection(idx[bi, g], cnt[bi, g], ref["idx"][0, g], ref["count"][0, g], ref["s_prime"][0][g],
                                m0, w.topk)
        else:
            ref = oesa.decode_step(q[bi:bi + 1], k[bi:bi + 1, :n], v[bi:bi + 1, :n], wq.cpu().numpy(),
                                   wk.cpu().numpy(), w.n_init, w.window, w.topk, w.eps, w.clamp_c)
            check_selection(idx[bi, 0], cnt[bi, 0], ref["idx"][0], ref["count"][0], ref["s_prime"][0], m0, w.topk)
            # the new key's compressed row landed at the sequence's last token
            assert float(np.abs(kc_last[bi] - ref["k_c"][0, n - 1]).max()) <= 1e-3
        assert max_abs(o[bi:bi + 1].cpu().double().numpy(), ref["o"]) <= ATOL_BF16


def test_decode_varlen_llama_shape():
    _decode(False, 12000, [12000, 6100, 3000, 9001], seqs=(0, 1, 2, 3))


def test_decode_varlen_per_head():
    _decode(True, 9000, [9000, 4000, 7777], seqs=(0, 1))


def test_graph_replays_with_new_lengths():
    # a captured step reads the lengths from the device: new lengths, same graph
    w = synthetic.DECODE_128K
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    b, n_cap = 4, 10000
    inp = synthetic.make_esa_inputs(w, device=DEV, n_ctx=n_cap, batch=b)
    dec = pipeline.EsaDecodeVarlen(b, n_cap, w.hq, w.hkv, w.head_dim, w.d_c, p, device=DEV)
    dec.fill_cache(inp["k"], inp["wk"], [n_cap] * b)
    seq_len = torch.full((b,), n_cap, dtype=torch.int64, device=DEV)
    k_new = inp["k"][:, -1].contiguous()
    dec.step(inp["q"], k_new, inp["k"], inp["v"], inp["wq"], inp["wk"], seq_len)     # pack, warm up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dec.step(inp["q"], k_new, inp["k"], inp["v"], inp["wq"], inp["wk"], seq_len)
    new = torch.tensor([10000, 5000, 2500, 7000], dtype=torch.int64)
    seq_len.copy_(new.to(DEV))
    g.replay()
    torch.cuda.synchronize()
    got_o, got_idx = dec.out.clone(), dec.idx.clone()
    # eager step with the same lengths (k_new rows as the graph wrote them: the cache
    # rows past each length are untouched by either)
    dec.step(inp["q"], k_new, inp["k"], inp["v"], inp["wq"], inp["wk"], seq_len)
    torch.cuda.synchronize()
    assert torch.equal(got_idx.cpu(), dec.idx.cpu())
    assert torch.equal(got_o.cpu(), dec.out.cpu())
    qas.device_status()
    del g


def test_length_outside_the_cache_is_reported():
    # lengths 0 and n_cap + 5 are clamped on the device (no access outside the cache)
    # and reported by the next device_status
    p = qas.params(16, 64, 32, 2, 10.0)
    q_c = _rand((2, 1, 64), 111).to(DEV)
    k_c = _rand((2, 1000, 64), 112).to(DEV)
    seq_len = torch.tensor([0, 1005], dtype=torch.int64, device=DEV)
    _, cnt, _ = qas.score_select_varlen(q_c, k_c, seq_len, p)
    with pytest.raises(qas.EsaError):
        qas.device_status()
    qas.device_status()                       # cleared by the read
    assert cnt.cpu().tolist() == [[0], [min(32, 999 - 64 - 16)]]
