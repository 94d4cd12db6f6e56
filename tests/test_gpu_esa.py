"""ESA parity: the CUDA path through the C ABI against the CPU oracle.

Small and medium sizes that still span several tiles and ragged tails; the
full workloads are in test_gpu_fullsize.py. Inputs are seeded and synthetic;
the oracle receives the same tensors bit for bit (copied to the host).
"""
import math

import numpy as np
import pytest
import torch

import query_aware_selective_b200 as qas
from oracle import esa as oesa
from query_aware_selective_b200 import synthetic
from tests.parity import ATOL_BF16, ATOL_F32, check_selection, max_abs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _np(t):
    return t.detach().cpu().double().numpy() if t.dtype in (torch.bfloat16, torch.float32) else t.cpu().numpy()


def _rand(shape, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype)


# ----------------------------------------------------------------------------- compress

@pytest.mark.parametrize("rows,hin,hout,d,dc,dtype", [
    (37, 8, 32, 128, 128, torch.bfloat16),    # GQA keys, ragged rows
    (512, 32, 32, 128, 128, torch.bfloat16),  # one prefill chunk of queries
    (5, 4, 4, 64, 16, torch.float32),         # the tiny fp32 layer, d' = 16
    (1, 2, 8, 64, 48, torch.float32),         # one row, d' = 48
    (300, 4, 16, 64, 128, torch.bfloat16),    # tensor-core path, head_dim 64, 3 row tiles
    (1, 8, 32, 128, 128, torch.bfloat16),     # a single row
])
def test_compress_parity(rows, hin, hout, d, dc, dtype):
    x = _rand((rows, hin, d), 1, dtype)
    w = _rand((hout * d, dc), 2, torch.float32) / math.sqrt(hout * d)
    y = qas.compress(x.to(DEV), w.to(DEV), hout)
    ref = oesa.compress(_np(x), _np(w), hout)
    assert max_abs(_np(y), ref) <= ATOL_F32


def test_compress_strided_rows_of_a_batched_cache():
    """One call compresses the new key of every sequence (rows n_ctx apart) and writes
    each into that sequence's row of the compressed cache."""
    b, n, hkv, hq, d, dc, pos = 5, 40, 8, 32, 128, 128, 37
    k = _rand((b, n, hkv, d), 5, torch.bfloat16).to(DEV)
    w = (_rand((hq * d, dc), 6, torch.float32) / math.sqrt(hq * d)).to(DEV)
    cache = torch.zeros((b, n, dc), device=DEV)
    qas.compress(k[:, pos], w, hq, out=cache[:, pos], out_row_stride=n * dc)
    ref = oesa.compress(_np(k[:, pos].cpu()), _np(w.cpu()), hq)
    got = cache.cpu().numpy()
    assert max_abs(got[:, pos], ref) <= ATOL_F32
    assert np.all(np.delete(got, pos, axis=1) == 0.0)


def test_compress_writes_into_a_cache_slice():
    x = _rand((20, 2, 128), 3, torch.bfloat16)
    w = _rand((8 * 128, 32), 4, torch.float32) / 32.0
    cache = torch.full((64, 40), 7.0, device=DEV)
    qas.compress(x.to(DEV), w.to(DEV), 8, out=cache[10:], out_row_stride=40)
    ref = oesa.compress(_np(x), _np(w), 8)
    got = cache.cpu().numpy()
    assert max_abs(got[10:30, :32], ref) <= ATOL_F32
    assert np.all(got[:10] == 7.0) and np.all(got[30:] == 7.0) and np.all(got[10:30, 32:] == 7.0)


@pytest.mark.parametrize("rows,hin,hout", [
    (512, 32, 32),     # one chunk of queries: K = 4096, 4 row tiles
    (300, 8, 32),      # keys under GQA (G = 4, K = 1024), ragged last row tile
    (1, 4, 4),         # K = 512: the smallest reduction the packed path takes
    (129, 16, 32),     # G = 2, one full tile + one row
])
def test_compress_packed_parity(rows, hin, hout):
    """Packed weight (fold + bf16 hi/lo split, once) then the TMA/tcgen05 map: the
    oracle's fp64 map within the fp32 bar."""
    d, dc = 128, 128
    x = _rand((rows, hin, d), 11, torch.bfloat16)
    w = _rand((hout * d, dc), 12, torch.float32) / math.sqrt(hout * d)
    packed = qas.compress_pack(w.to(DEV), hin, hout, d)
    y = qas.compress_packed(x.to(DEV), packed, dc)
    ref = oesa.compress(_np(x), _np(w), hout)
    assert max_abs(_np(y), ref) <= ATOL_F32
    y2 = qas.compress(x.to(DEV), w.to(DEV), hout)      # the unpacked path: same split, other sum order
    assert max_abs(_np(y), _np(y2)) <= ATOL_F32


def test_compress_packed_strided_rows_of_a_batched_cache():
    """Decode form: the new key of every sequence (rows n_ctx apart) into that
    sequence's row of the compressed cache; nothing else is written."""
    b, n, hkv, hq, d, dc, pos = 5, 40, 8, 32, 128, 128, 37
    k = _rand((b, n, hkv, d), 15, torch.bfloat16).to(DEV)
    w = (_rand((hq * d, dc), 16, torch.float32) / math.sqrt(hq * d)).to(DEV)
    cache = torch.zeros((b, n, dc), device=DEV)
    packed = qas.compress_pack(w, hkv, hq, d)
    qas.compress_packed(k[:, pos], packed, dc, out=cache[:, pos], out_row_stride=n * dc)
    ref = oesa.compress(_np(k[:, pos].cpu()), _np(w.cpu()), hq)
    got = cache.cpu().numpy()
    assert max_abs(got[:, pos], ref) <= ATOL_F32
    assert np.all(np.delete(got, pos, axis=1) == 0.0)


def test_compress_packed_is_deterministic():
    x = _rand((640, 32, 128), 17, torch.bfloat16).to(DEV)
    w = (_rand((32 * 128, 128), 18, torch.float32) / 64.0).to(DEV)
    packed = qas.compress_pack(w, 32, 32, 128)
    a = qas.compress_packed(x, packed)
    b = qas.compress_packed(x, packed)
    assert torch.equal(a, b)


# ----------------------------------------------------------------------------- selection

def _selection_case(batch, lq, n_cap, c0, dc, p, seed, planted=False):
    g = torch.Generator().manual_seed(seed)
    q_c = torch.randn((batch, lq, dc), generator=g)
    k_c = torch.randn((batch, n_cap, dc), generator=g)
    if planted:
        # integer-valued keys: exact ties everywhere, so the tie order decides
        k_c = torch.round(k_c * 2) / 2
        q_c = torch.round(q_c * 2) / 2
    idx, cnt, sp = qas.score_select(q_c.to(DEV), k_c.to(DEV), c0, p, want_scores=True)
    ref_idx, ref_cnt, ref_sp = oesa.score_select(q_c.double().numpy(), k_c.double().numpy(), c0, p.n_init,
                                                 p.window, p.topk, p.eps, p.clamp_c)
    _, (m0, m1), _ = oesa.regions(c0, c0 + lq, p.n_init, p.window)
    swaps = 0
    for b in range(batch):
        swaps += check_selection(idx[b].cpu().numpy(), cnt[b].item(), ref_idx[b], ref_cnt[b], ref_sp[b], m0, p.topk)
        if m1 > m0:
            ref_v = ref_sp[b]
            got_v = sp[b].cpu().double().numpy()
            scale = max(1.0, float(np.abs(ref_v).max()))
            # fp32 scoring (few queries) is held to 1e-4 of the scale; the tensor-core
            # path reads the compressed operands as tf32 (10-bit mantissa), so it is held
            # to the selection band's own 1e-3
            rel = 1e-3 if (lq >= 16 and dc in (32, 64, 128)) else 1e-4
            assert float(np.abs(got_v - ref_v).max()) <= rel * scale
    return swaps


@pytest.mark.parametrize("batch,lq,n_cap,c0,dc,n_init,window,topk,eps,clamp", [
    (1, 1, 2048, 2047, 16, 16, 256, 128, 2, 16.0),         # tiny decode shape
    (3, 1, 5000, 4999, 128, 128, 512, 300, 2, 45.25),      # decode, batch, ragged tiles
    (2, 3, 3000, 2997, 64, 8, 100, 77, 1, 10.0),           # few queries (register path)
    (1, 8, 2600, 2592, 128, 64, 128, 512, 0, math.inf),    # no clamp, eps 0
    (1, 64, 4096, 4032, 128, 128, 512, 1024, 2, 45.25),    # prefill-like chunk (tiled path)
    (2, 130, 3000, 2870, 48, 16, 300, 200, 3, 8.0),        # ragged chunk, d' = 48
    (1, 512, 9000, 8488, 128, 128, 1024, 2048, 2, 45.25),  # a full 512-query chunk
    (1, 1, 300000, 299999, 16, 16, 256, 2048, 2, 16.0),    # > 16K positions per cluster CTA: keys in scratch
    (2, 1, 40, 39, 16, 4, 28, 3, 2, 4.0),                  # 7-token middle: most cluster CTAs own nothing
])
def test_score_select_parity(batch, lq, n_cap, c0, dc, n_init, window, topk, eps, clamp):
    p = qas.params(n_init, window, topk, eps, clamp)
    _selection_case(batch, lq, n_cap, c0, dc, p, seed=batch * 1000 + lq)


def test_score_select_ties_follow_position_order():
    p = qas.params(8, 40, 50, 2, 3.0)
    _selection_case(2, 2, 800, 798, 16, p, seed=9, planted=True)


@pytest.mark.parametrize("topk,c0,window", [
    (500, 520, 8),     # |mid| = 504 > topk by 4
    (503, 520, 8),     # |mid| = topk + 1: one position dropped
    (504, 520, 8),     # |mid| == topk: everything
    (600, 520, 8),     # |mid| < topk: everything, -1 padding
    (10, 300, 292),    # empty middle
    (1, 520, 8),       # k = 1
])
def test_score_select_edges(topk, c0, window):
    p = qas.params(8, window, topk, 2, 5.0)
    _selection_case(2, 1, c0 + 1, c0, 32, p, seed=topk + c0)


def test_zero_clamp_keeps_the_first_k_on_gpu():
    p = qas.params(8, 30, 10, 2, 0.0)
    g = torch.Generator().manual_seed(4)
    q_c = torch.randn((2, 3, 16), generator=g).to(DEV)
    k_c = torch.randn((2, 100, 16), generator=g).to(DEV)
    idx, cnt, _ = qas.score_select(q_c, k_c, 97, p)
    assert idx.cpu().tolist() == [list(range(8, 18))] * 2


# ----------------------------------------------------------------------------- attention

@pytest.mark.parametrize("batch,lq,n_cap,c0,hq,hkv,d,dtype,n_init,window,topk", [
    (1, 1, 2048, 2047, 4, 4, 64, torch.float32, 16, 256, 128),       # tiny decode (fp32)
    (2, 1, 6000, 5999, 32, 8, 128, torch.bfloat16, 128, 1024, 700),  # decode, GQA 4
    (3, 1, 3000, 2999, 16, 2, 64, torch.bfloat16, 32, 256, 333),     # GQA 8, head_dim 64
    (1, 5, 3000, 2995, 8, 8, 128, torch.float32, 16, 128, 256),      # few queries, fp32
    (1, 4, 1000, 996, 8, 2, 128, torch.bfloat16, 16, 128, 100),      # few queries bf16 (SIMT)
])
def test_sparse_attn_simt_parity(batch, lq, n_cap, c0, hq, hkv, d, dtype, n_init, window, topk):
    p = qas.params(n_init, window, topk, 2, 10.0)
    q = _rand((batch, lq, hq, d), 11, dtype)
    k = _rand((batch, n_cap, hkv, d), 12, dtype)
    v = _rand((batch, n_cap, hkv, d), 13, dtype)
    _, (m0, m1), _ = oesa.regions(c0, c0 + lq, n_init, window)
    idx, cnt = synthetic.random_index_list(batch, m0, m1, topk, seed=14)
    o, lse = qas.sparse_attn(q.to(DEV), k.to(DEV), v.to(DEV), c0, idx.to(DEV), cnt.to(DEV), p, want_lse=True)
    ref_o, ref_lse = oesa.sparse_attn(_np(q), _np(k), _np(v), c0, idx.numpy(), cnt.numpy(), n_init, window)
    atol = ATOL_F32 if dtype == torch.float32 else ATOL_BF16
    assert max_abs(_np(o), ref_o) <= atol
    assert max_abs(lse.cpu().numpy(), ref_lse) <= 1e-3


@pytest.mark.parametrize("batch,n_cap,hq,hkv,n_init,window,topk", [
    (16, 4000, 32, 8, 128, 1024, 2048),   # 9 key splits per sequence, ragged last stage
    (150, 200, 8, 2, 16, 64, 50),         # more sequences than SMs: one CTA each, direct output
    (3, 5000, 8, 4, 32, 512, 777),        # G = 2, two warps per KV head
    (2, 4000, 8, 2, 16, 300, 500),        # G = 4, four warps per KV head
    (2, 3000, 1, 1, 8, 200, 300),         # a single head: 128 keys per stage
    (4, 2500, 8, 8, 0, 100, 1000),        # no initial tokens
    (2, 300, 32, 8, 128, 4096, 2048),     # the window covers the middle: nothing selected
])
def test_sparse_attn_decode_parity(batch, n_cap, hq, hkv, n_init, window, topk):
    """The bulk-copy decode kernel (bf16, head_dim 128, one query per sequence), with
    per-sequence selection counts that differ (ragged key lists and splits)."""
    p = qas.params(n_init, window, topk, 2, 10.0)
    c0 = n_cap - 1
    q = _rand((batch, 1, hq, 128), 41, torch.bfloat16)
    k = _rand((batch, n_cap, hkv, 128), 42, torch.bfloat16)
    v = _rand((batch, n_cap, hkv, 128), 43, torch.bfloat16)
    _, (m0, m1), _ = oesa.regions(c0, c0 + 1, n_init, window)
    idx, cnt = synthetic.random_index_list(batch, m0, m1, topk, seed=44)
    for b in range(batch):
        c = max(0, int(cnt[b]) - 37 * b)
        idx[b, c:] = -1
        cnt[b] = c
    o, lse = qas.sparse_attn(q.to(DEV), k.to(DEV), v.to(DEV), c0, idx.to(DEV), cnt.to(DEV), p, want_lse=True)
    o2, _ = qas.sparse_attn(q.to(DEV), k.to(DEV), v.to(DEV), c0, idx.to(DEV), cnt.to(DEV), p)
    assert torch.equal(o, o2)                    # no state carried between calls
    ref_o, ref_lse = oesa.sparse_attn(q.float().numpy(), k.float().numpy(), v.float().numpy(), c0, idx.numpy(),
                                      cnt.numpy(), n_init, window)
    assert max_abs(_np(o), ref_o) <= ATOL_BF16
    assert max_abs(lse.cpu().numpy(), ref_lse) <= 1e-3


@pytest.mark.parametrize("batch,lq,n_cap,c0,hq,hkv,n_init,window,topk", [
    (1, 128, 1024, 640, 8, 2, 16, 256, 128),      # 4 row tiles, selection active
    (1, 200, 3000, 2800, 32, 8, 128, 1024, 700),  # ragged chunk (800 rows), 7 row tiles
    (2, 64, 700, 0, 4, 4, 16, 256, 64),           # first chunk: causal only
    (1, 512, 5000, 4488, 32, 8, 128, 2048, 1024), # a full chunk, several key tiles
    (1, 96, 4000, 333, 16, 4, 128, 512, 2048),    # short middle: full causal attention
    (10, 64, 1500, 1000, 32, 8, 16, 256, 256),    # 80 tile pairs: no key split
    (5, 64, 2500, 2000, 32, 8, 64, 512, 512),     # 40 tile pairs: two key parts per pair
])
def test_sparse_attn_tensor_core_parity(batch, lq, n_cap, c0, hq, hkv, n_init, window, topk):
    p = qas.params(n_init, window, topk, 2, 10.0)
    q = _rand((batch, lq, hq, 128), 21, torch.bfloat16)
    k = _rand((batch, n_cap, hkv, 128), 22, torch.bfloat16)
    v = _rand((batch, n_cap, hkv, 128), 23, torch.bfloat16)
    _, (m0, m1), _ = oesa.regions(c0, c0 + lq, n_init, window)
    idx, cnt = synthetic.random_index_list(batch, m0, m1, topk, seed=24)
    o, lse = qas.sparse_attn(q.to(DEV), k.to(DEV), v.to(DEV), c0, idx.to(DEV), cnt.to(DEV), p, want_lse=True)
    o2, lse2 = qas.sparse_attn(q.to(DEV), k.to(DEV), v.to(DEV), c0, idx.to(DEV), cnt.to(DEV), p, want_lse=True)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)     # the key-split merge is deterministic
    ref_o, ref_lse = oesa.sparse_attn(_np(q), _np(k), _np(v), c0, idx.numpy(), cnt.numpy(), n_init, window)
    assert max_abs(_np(o), ref_o) <= ATOL_BF16
    assert max_abs(lse.cpu().numpy(), ref_lse) <= 2e-2


def test_tensor_core_path_equals_full_causal_attention():
    """k >= |mid|: the chunk attends every earlier token; compare with torch SDPA on
    the GPU's own inputs in float64 (library routine) as well as with the oracle."""
    b, lq, n, hq, hkv, d = 1, 256, 1280, 8, 2, 128
    c0 = n - lq
    p = qas.params(16, 128, 4096, 2, 10.0)
    q = _rand((b, lq, hq, d), 31, torch.bfloat16)
    k = _rand((b, n, hkv, d), 32, torch.bfloat16)
    v = _rand((b, n, hkv, d), 33, torch.bfloat16)
    _, (m0, m1), _ = oesa.regions(c0, n, 16, 128)
    idx = torch.full((b, 4096), -1, dtype=torch.int32)
    idx[0, :m1 - m0] = torch.arange(m0, m1, dtype=torch.int32)
    cnt = torch.tensor([m1 - m0], dtype=torch.int32)
    o, _ = qas.sparse_attn(q.to(DEV), k.to(DEV), v.to(DEV), c0, idx.to(DEV), cnt.to(DEV), p)
    mask = torch.arange(n).view(1, n) <= torch.arange(c0, n).view(lq, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().permute(0, 2, 1, 3), k.double().permute(0, 2, 1, 3), v.double().permute(0, 2, 1, 3),
        attn_mask=mask, enable_gqa=True).permute(0, 2, 1, 3)
    assert max_abs(_np(o), ref.numpy()) <= ATOL_BF16


# ----------------------------------------------------------------------------- end to end

def test_tiny_decode_end_to_end():
    w = synthetic.TINY_DECODE
    inp = synthetic.make_esa_inputs(w)
    q, k, v = (inp[x].to(DEV) for x in ("q", "k", "v"))
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    n = w.n_ctx
    q_c = qas.compress(q[:, 0], inp["wq"].to(DEV), w.hq).view(1, 1, -1)
    k_c = qas.compress(k[0], inp["wk"].to(DEV), w.hq).view(1, n, -1)
    idx, cnt, sp = qas.score_select(q_c, k_c, n - 1, p, want_scores=True)
    o, lse = qas.sparse_attn(q, k, v, n - 1, idx, cnt, p, want_lse=True)
    ref = oesa.decode_step(*(inp[x].numpy() for x in ("q", "k", "v", "wq", "wk")), w.n_init, w.window, w.topk,
                           w.eps, w.clamp_c)
    _, (m0, _), _ = oesa.regions(n - 1, n, w.n_init, w.window)
    check_selection(idx[0].cpu().numpy(), cnt[0].item(), ref["idx"][0], ref["count"][0], ref["s_prime"][0], m0,
                    w.topk)
    assert max_abs(_np(o), ref["o"]) <= ATOL_F32
    assert max_abs(lse.cpu().numpy(), ref["lse"]) <= ATOL_F32
    chosen = set(idx[0, :cnt[0]].tolist())
    for pos in inp["needles"][0].tolist():
        assert all(j in chosen for j in range(pos - w.eps, pos + w.eps + 1))
    qas.device_status()


def test_small_chunked_prefill_end_to_end():
    """Four chunks of 256 over a 1024-token GQA layer: compress, select, attend,
    each chunk against the oracle (selection band rule, outputs within 2e-2)."""
    hq, hkv, d, n, chunk, dc = 8, 2, 128, 1024, 256, 128
    p = qas.params(32, 128, 128, 2, 4 * math.sqrt(dc))
    q = _rand((1, n, hq, d), 41, torch.bfloat16)
    k = _rand((1, n, hkv, d), 42, torch.bfloat16)
    v = _rand((1, n, hkv, d), 43, torch.bfloat16)
    wq = _rand((hq * d, dc), 44, torch.float32) / math.sqrt(hq * d)
    wk = _rand((hq * d, dc), 45, torch.float32) / math.sqrt(hq * d)
    qd, kd, vd, wqd, wkd = (t.to(DEV) for t in (q, k, v, wq, wk))
    k_c = torch.zeros((1, n, dc), device=DEV)
    ref_kc = oesa.compress(_np(k[0]), _np(wk), hq)[None]
    for c0 in range(0, n, chunk):
        qas.compress(kd[0, c0:c0 + chunk], wkd, hq, out=k_c[0, c0:c0 + chunk])
        q_c = qas.compress(qd[0, c0:c0 + chunk], wqd, hq).view(1, chunk, dc)
        idx, cnt, _ = qas.score_select(q_c, k_c, c0, p)
        o, _ = qas.sparse_attn(qd[:, c0:c0 + chunk], kd, vd, c0, idx, cnt, p)
        ref = oesa.prefill_chunk(_np(q[:, c0:c0 + chunk]), _np(k), _np(v), ref_kc, _np(wq), c0, p.n_init, p.window,
                                 p.topk, p.eps, p.clamp_c)
        _, (m0, _), _ = oesa.regions(c0, c0 + chunk, p.n_init, p.window)
        check_selection(idx[0].cpu().numpy(), cnt[0].item(), ref["idx"][0], ref["count"][0], ref["s_prime"][0], m0,
                        p.topk)
        # the output over the GPU's own selection, always (a band swap changes the key
        # set but not the rule), and against the oracle's end-to-end output when the
        # two selections agree
        own_o, _ = oesa.sparse_attn(_np(q[:, c0:c0 + chunk]), _np(k), _np(v), c0, idx.cpu().numpy(),
                                    cnt.cpu().numpy(), p.n_init, p.window)
        assert max_abs(_np(o), own_o) <= ATOL_BF16
        if set(idx[0, :cnt[0]].tolist()) == set(ref["idx"][0, :ref["count"][0]].tolist()):
            assert max_abs(_np(o), ref["o"]) <= ATOL_BF16
    qas.device_status()
