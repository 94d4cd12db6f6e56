"""Pins of the variable-length decode oracle (oracle/esa_varlen.py) against what the
equal-length batch calls, closed forms and constructed inputs fix."""
import math

import numpy as np
import torch

from oracle import esa, esa_varlen


def _rng(seed):
    return np.random.default_rng(seed)


def _sdpa_causal_last(q, k, v):
    """softmax(q K^T / sqrt(D)) V for one query over every row given (float64 SDPA)."""
    hq, hkv = q.shape[1], k.shape[1]
    g = hq // hkv
    qt = torch.from_numpy(q[None]).permute(0, 2, 1, 3)                          # [1, Hq, 1, D]
    kt = torch.from_numpy(np.repeat(k, g, axis=1)[None]).permute(0, 2, 1, 3)    # [1, Hq, n, D]
    vt = torch.from_numpy(np.repeat(v, g, axis=1)[None]).permute(0, 2, 1, 3)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).permute(0, 2, 1, 3)[0].numpy()


def check_equal_lengths_are_the_batch_call():
    # every sequence at the full length: the equal-length batch calls, row for row
    r = _rng(0)
    bsz, n, dc = 3, 400, 16
    q_c = r.standard_normal((bsz, 1, dc))
    k_c = r.standard_normal((bsz, n, dc))
    lens = np.full(bsz, n)
    idx, count, _ = esa_varlen.score_select_varlen(q_c, k_c, lens, 8, 32, 40, 2, 6.0)
    ref_idx, ref_count, _ = esa.score_select(q_c, k_c, n - 1, 8, 32, 40, 2, 6.0)
    np.testing.assert_array_equal(idx[:, 0], ref_idx)
    np.testing.assert_array_equal(count[:, 0], ref_count)
    hq, hkv, d = 4, 2, 8
    q = r.standard_normal((bsz, 1, hq, d))
    k = r.standard_normal((bsz, n, hkv, d))
    v = r.standard_normal((bsz, n, hkv, d))
    o, lse = esa_varlen.sparse_attn_varlen(q, k, v, lens, idx, count, 8, 32)
    ref_o, ref_lse = esa.sparse_attn(q, k, v, n - 1, ref_idx, ref_count, 8, 32)
    np.testing.assert_allclose(o, ref_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def check_rows_past_the_length_take_no_part():
    # replacing every row past seq_len[b] (keys, values, compressed keys) changes nothing
    r = _rng(1)
    bsz, n, hq, hkv, d = 3, 300, 4, 2, 8
    lens = np.array([300, 170, 95])
    q = r.standard_normal((bsz, 1, hq, d))
    k = r.standard_normal((bsz, n, hkv, d))
    v = r.standard_normal((bsz, n, hkv, d))
    wq = r.standard_normal((hq * d, 8)) / math.sqrt(hq * d)
    wk = r.standard_normal((hq * d, 8)) / math.sqrt(hq * d)
    a = esa_varlen.decode_step_varlen(q, k, v, wq, wk, lens, 4, 20, 16, 1, 5.0)
    k2, v2 = k.copy(), v.copy()
    for b in range(bsz):
        k2[b, lens[b]:] = 50.0 * r.standard_normal(k2[b, lens[b]:].shape)
        v2[b, lens[b]:] = 50.0 * r.standard_normal(v2[b, lens[b]:].shape)
    b2 = esa_varlen.decode_step_varlen(q, k2, v2, wq, wk, lens, 4, 20, 16, 1, 5.0)
    np.testing.assert_array_equal(a["idx"], b2["idx"])
    np.testing.assert_allclose(a["o"], b2["o"], rtol=1e-12, atol=1e-12)
    # and each sequence equals a batch of one at its own length
    for b in range(bsz):
        one = esa.decode_step(q[b:b + 1], k[b:b + 1, :lens[b]], v[b:b + 1, :lens[b]], wq, wk, 4, 20, 16, 1, 5.0)
        np.testing.assert_array_equal(a["idx"][b, 0], one["idx"][0])
        np.testing.assert_allclose(a["o"][b], one["o"][0], rtol=1e-12, atol=1e-12)


def check_short_sequences_attend_everything():
    # a sequence with no middle (len <= n_init + window + 1) or with topk >= its middle
    # attends all its rows: full causal softmax of its one query (SDPA in float64)
    r = _rng(2)
    bsz, n, hq, hkv, d = 3, 200, 4, 2, 8
    n_init, window, topk = 4, 30, 64
    lens = np.array([20, n_init + window + 1, 90])      # no middle, an empty middle, middle 55 <= topk
    q = r.standard_normal((bsz, 1, hq, d))
    k = r.standard_normal((bsz, n, hkv, d))
    v = r.standard_normal((bsz, n, hkv, d))
    wq = r.standard_normal((hq * d, 8))
    wk = r.standard_normal((hq * d, 8))
    out = esa_varlen.decode_step_varlen(q, k, v, wq, wk, lens, n_init, window, topk, 2, 3.0)
    np.testing.assert_array_equal(out["count"][:, 0], [0, 0, lens[2] - 1 - window - n_init])
    for b in range(bsz):
        ref = _sdpa_causal_last(q[b], k[b, :lens[b]], v[b, :lens[b]])
        np.testing.assert_allclose(out["o"][b], ref, rtol=1e-10, atol=1e-10)


def check_needle_belongs_to_its_own_sequence():
    # a compressed key aligned with the query is selected in the sequence whose middle
    # holds it; placed past another sequence's length it plays no part there
    r = _rng(3)
    bsz, n, dc = 2, 500, 8
    q_c = r.standard_normal((bsz, 1, dc))
    k_c = 0.1 * r.standard_normal((bsz, n, dc))
    lens = np.array([500, 200])
    k_c[0, 100] = 20.0 * q_c[0, 0]         # in sequence 0's middle [4, 500 - 1 - 16)
    k_c[1, 300] = 20.0 * q_c[1, 0]         # past sequence 1's length
    idx, count, sp = esa_varlen.score_select_varlen(q_c, k_c, lens, 4, 16, 5, 0, math.inf)
    assert 100 in idx[0, 0, :count[0, 0]]
    assert 300 not in idx[1, 0]
    assert len(sp[1][0]) == lens[1] - 1 - 16 - 4


def check_per_head_lists_per_sequence():
    # n_groups > 1 and lists = Hkv run the per-head calls per sequence
    from oracle import esa_heads
    r = _rng(4)
    bsz, n, hq, hkv, d, dc = 2, 260, 8, 4, 8, 16
    lens = np.array([260, 140])
    q_c = r.standard_normal((bsz, 1, dc))
    k_c = r.standard_normal((bsz, n, dc))
    idx, count, _ = esa_varlen.score_select_varlen(q_c, k_c, lens, 4, 20, 12, 1, 4.0, n_groups=hkv)
    q = r.standard_normal((bsz, 1, hq, d))
    k = r.standard_normal((bsz, n, hkv, d))
    v = r.standard_normal((bsz, n, hkv, d))
    o, _ = esa_varlen.sparse_attn_varlen(q, k, v, lens, idx, count, 4, 20)
    for b in range(bsz):
        i1, c1, _ = esa_heads.score_select_heads(q_c[b:b + 1], k_c[b:b + 1, :lens[b]], lens[b] - 1, hkv, 4, 20, 12,
                                                 1, 4.0)
        np.testing.assert_array_equal(idx[b], i1[0])
        o1, _ = esa_heads.sparse_attn_heads(q[b:b + 1], k[b:b + 1, :lens[b]], v[b:b + 1, :lens[b]], lens[b] - 1,
                                            i1, c1, 4, 20)
        np.testing.assert_allclose(o[b], o1[0], rtol=1e-12, atol=1e-12)


def test_equal_lengths_are_the_batch_call():
    check_equal_lengths_are_the_batch_call()


def test_rows_past_the_length_take_no_part():
    check_rows_past_the_length_take_no_part()


def test_short_sequences_attend_everything():
    check_short_sequences_attend_everything()


def test_needle_belongs_to_its_own_sequence():
    check_needle_belongs_to_its_own_sequence()


def test_per_head_lists_per_sequence():
    check_per_head_lists_per_sequence()
