"""Parity at the full benchmark sizes, in the launch configuration bench.py times
(the same pipeline drivers), on outputs the oracle computes one by one: whole
sequences for decode, sampled chunks and rows for prefill, sampled positions for
MoBA."""
import numpy as np
import pytest
import torch

import query_aware_selective_b200 as qas
from oracle import esa as oesa
from oracle import moba as omoba
from query_aware_selective_b200 import pipeline, synthetic
from tests.parity import ATOL_BF16, check_selection, max_abs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _f64(t):
    return t.detach().cpu().double().numpy()


def _decode_full(w, seqs):
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    inp = synthetic.make_esa_inputs(w, device=DEV)
    dec = pipeline.EsaDecode(w.batch, w.n_ctx, w.hq, w.hkv, w.head_dim, w.d_c, p, device=DEV)
    dec.fill_cache(inp["k"], inp["wk"])
    o = dec.step(inp["q"], inp["k"], inp["v"], inp["wq"], inp["wk"]).clone()
    idx, cnt = dec.idx.cpu().numpy(), dec.count.cpu().numpy()
    qas.device_status()
    _, (m0, _), _ = oesa.regions(w.n_ctx - 1, w.n_ctx, w.n_init, w.window)
    wq, wk = inp["wq"].cpu().numpy(), inp["wk"].cpu().numpy()
    for b in seqs:
        qb = inp["q"][b:b + 1].float().cpu().numpy()
        kb = inp["k"][b:b + 1].float().cpu().numpy()
        vb = inp["v"][b:b + 1].float().cpu().numpy()
        ref = oesa.decode_step(qb, kb, vb, wq, wk, w.n_init, w.window, w.topk, w.eps, w.clamp_c)
        check_selection(idx[b], cnt[b], ref["idx"][0], ref["count"][0], ref["s_prime"][0], m0, w.topk)
        chosen = set(idx[b, :cnt[b]].tolist())
        for pos in inp["needles"][b].tolist():
            assert all(j in chosen for j in range(pos - w.eps, pos + w.eps + 1)), pos
        assert max_abs(_f64(o[b:b + 1]), ref["o"]) <= ATOL_BF16
        own_o, _ = oesa.sparse_attn(qb, kb, vb, w.n_ctx - 1, idx[b:b + 1], cnt[b:b + 1], w.n_init, w.window)
        assert max_abs(_f64(o[b:b + 1]), own_o) <= ATOL_BF16      # over the GPU's own selection
    del inp, dec
    torch.cuda.empty_cache()


def test_decode_128k_batch16():
    _decode_full(synthetic.DECODE_128K, seqs=(0, 15))


def test_decode_1m_batch4():
    _decode_full(synthetic.DECODE_1M, seqs=(0,))


def test_decode_per_head_128k_batch16():
    # the per-head selection variant on the decode workload bench.py times
    from tests.test_gpu_heads import _decode_heads
    _decode_heads(synthetic.DECODE_128K, None, synthetic.DECODE_128K.batch, seqs=(0, 15))
    torch.cuda.empty_cache()


def test_decode_varlen_128k_batch16():
    # the variable-length decode workload bench.py times (the 128K inputs, the same
    # seeded length mix); the longest and the shortest sequence against the oracle
    from tests.test_gpu_varlen import _decode
    w = synthetic.DECODE_128K
    lens = synthetic.varlen_lengths(w.batch, w.n_ctx, 8192, seed=w.seed + 2000).tolist()
    shortest = min(range(len(lens)), key=lambda i: lens[i])
    _decode(False, w.n_ctx, lens, seqs=(0, shortest))
    torch.cuda.empty_cache()


def test_prefill_32k_sampled_chunks():
    w = synthetic.PREFILL_32K
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    inp = synthetic.make_esa_inputs(w, device=DEV)
    pf = pipeline.EsaPrefill(w.batch, w.n_ctx, w.chunk, w.hq, w.hkv, w.head_dim, w.d_c, p, device=DEV)
    # the two-stream pipelined run bench.py times; every chunk's selection stays readable
    out = pf.run(inp["q"], inp["k"], inp["v"], inp["wq"], inp["wk"])
    sampled = {ci: (pf.idx_all[ci].cpu().numpy(), pf.count_all[ci].cpu().numpy()) for ci in (0, 13, 40, 63)}
    qas.device_status()
    qn = inp["q"].float().cpu().numpy()
    kn = inp["k"].float().cpu().numpy()
    vn = inp["v"].float().cpu().numpy()
    wq, wk = inp["wq"].cpu().numpy(), inp["wk"].cpu().numpy()
    k_c = oesa.compress(kn[0], wk, w.hq)[None]
    rng = np.random.default_rng(0)
    for ci, (idx, cnt) in sampled.items():
        c0 = ci * w.chunk
        rows = sorted(set(rng.integers(0, w.chunk, 6).tolist()) | {0, w.chunk - 1})
        ref = oesa.prefill_chunk(qn[:, c0:c0 + w.chunk], kn, vn, k_c, wq, c0, w.n_init, w.window, w.topk, w.eps,
                                 w.clamp_c, rows=[(0, i) for i in rows])
        _, (m0, _), _ = oesa.regions(c0, c0 + w.chunk, w.n_init, w.window)
        check_selection(idx[0], cnt[0], ref["idx"][0], ref["count"][0], ref["s_prime"][0], m0, w.topk)
        got = _f64(out[:, c0:c0 + w.chunk])
        assert max_abs(got[:, rows], ref["o"][:, rows]) <= ATOL_BF16
        # the same rows over the GPU's own selection (equal to the above unless a band
        # swap changed a key)
        own_o, _ = oesa.sparse_attn(qn[:, c0:c0 + w.chunk], kn, vn, c0, idx, cnt, w.n_init, w.window,
                                    rows=[(0, i) for i in rows])
        assert max_abs(got[:, rows], own_o[:, rows]) <= ATOL_BF16


def test_moba_64k_sampled_positions():
    w = synthetic.MOBA_64K
    inp = synthetic.make_moba_inputs(w, device=DEV)
    mb = pipeline.MobaPrefill(w.batch, w.seq, w.heads, w.head_dim, w.block, w.topk, device=DEV)
    out = mb.run(inp["q"], inp["k"], inp["v"])
    blocks = mb.blocks.cpu().numpy().astype(np.int64)
    qas.device_status()
    kn = inp["k"].float().cpu().numpy()
    kbar = omoba.block_means(kn, w.block)
    qn = inp["q"].float().cpu().numpy()
    vn = inp["v"].float().cpu().numpy()
    rng = np.random.default_rng(1)
    pos = sorted(set(rng.integers(0, w.seq, 20).tolist()) | {0, w.block - 1, w.block, 3 * w.block + 5, w.seq - 1})
    ref_blocks = omoba.gate(qn, kbar, w.block, w.topk, positions=pos)
    got_blocks = blocks[:, pos]
    same = np.all(got_blocks == ref_blocks, axis=-1)
    for b, r, h in zip(*np.nonzero(~same)):
        p_ = pos[r]
        cur = p_ // w.block
        sc = kbar[b, h, :cur] @ qn[b, p_, h]
        kth = np.sort(sc)[::-1][min(w.topk, cur) - 1]
        for blk in set(got_blocks[b, r, h].tolist()) ^ set(ref_blocks[b, r, h].tolist()):
            assert abs(sc[blk] - kth) <= 1e-3 * abs(kth) + 1e-6
    assert same.mean() > 0.97
    ref_o, _ = omoba.attend(qn, kn, vn, ref_blocks, w.block, positions=pos)
    got = _f64(out[:, pos])
    assert max_abs(got[same], ref_o[same]) <= ATOL_BF16
    # every sampled row, swapped gates included: attention over the GPU's own blocks
    own_o, _ = omoba.attend(qn, kn, vn, got_blocks, w.block, positions=pos)
    assert max_abs(got, own_o) <= ATOL_BF16
