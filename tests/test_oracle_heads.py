"""Pins of the per-head selection oracle (oracle/esa_heads.py) against what the
merged form, textbook per-head scores and constructed inputs fix."""
import math

import numpy as np
import pytest
import torch

from oracle import esa, esa_heads


def _rng(seed):
    return np.random.default_rng(seed)


def test_group_maps_equal_the_block_diagonal_merged_map():
    # stacking the groups' maps block-diagonally gives the merged form's map, whose
    # compress() is pinned to torch.matmul on the expanded input
    r = _rng(0)
    hq, hkv, d, dg = 8, 2, 16, 4
    wq = r.standard_normal((hkv, (hq // hkv) * d, dg))
    wk = r.standard_normal((hkv, (hq // hkv) * d, dg))
    q = r.standard_normal((5, hq, d))
    k = r.standard_normal((7, hkv, d))
    np.testing.assert_allclose(esa_heads.compress_heads(q, wq, hq),
                               esa.compress(q, esa_heads.block_diagonal(wq), hq), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(esa_heads.compress_heads(k, wk, hq),
                               esa.compress(k, esa_heads.block_diagonal(wk), hq), rtol=1e-12, atol=1e-12)
    # and the merged map's output for group g depends on group g's inputs only
    k2 = k.copy()
    k2[:, 1] += 1.0
    a, b = esa_heads.compress_heads(k, wk, hq), esa_heads.compress_heads(k2, wk, hq)
    np.testing.assert_array_equal(a[:, :dg], b[:, :dg])
    assert np.abs(a[:, dg:] - b[:, dg:]).max() > 0


def test_identity_maps_give_textbook_per_head_top_k():
    # one query head per KV head, identity maps: group g's score is the textbook
    # per-head dot product q^g . k^g_j; with one query, eps 0 and no clamp the
    # selection is torch.topk of those products per head
    r = _rng(1)
    h, d, n = 3, 4, 300
    eye = np.stack([np.eye(d)] * h)
    q = r.standard_normal((1, 1, h, d))
    k = r.standard_normal((1, n, h, d))
    q_c = esa_heads.compress_heads(q[0], eye, h)[None]
    k_c = esa_heads.compress_heads(k[0], eye, h)[None]
    c0, n_init, window, topk = n - 1, 4, 20, 25
    idx, count, _ = esa_heads.score_select_heads(q_c, k_c, c0, h, n_init, window, topk, 0, math.inf)
    _, (m0, m1), _ = esa.regions(c0, c0 + 1, n_init, window)
    for g in range(h):
        scores = torch.from_numpy(np.einsum("d,nd->n", q[0, 0, g], k[0, m0:m1, g]))
        want = np.sort(torch.topk(scores, topk).indices.numpy() + m0)
        assert count[0, g] == topk
        np.testing.assert_array_equal(idx[0, g], want)


def test_a_needle_seen_by_one_head_is_selected_by_that_head_only():
    r = _rng(2)
    h, d, n = 4, 8, 400
    eye = np.stack([np.eye(d)] * h)
    q = r.standard_normal((1, 1, h, d))
    k = 0.1 * r.standard_normal((1, n, h, d))
    pos = 150
    k[0, pos, 2] = 10.0 * q[0, 0, 2]           # aligned with head 2's query
    for g in (0, 1, 3):
        k[0, pos, g] = -10.0 * q[0, 0, g]      # opposed to every other head's query
    q_c = esa_heads.compress_heads(q[0], eye, h)[None]
    k_c = esa_heads.compress_heads(k[0], eye, h)[None]
    idx, count, _ = esa_heads.score_select_heads(q_c, k_c, n - 1, h, 8, 32, 10, 1, 5.0)
    for g in range(h):
        chosen = set(idx[0, g, :count[0, g]].tolist())
        assert (pos in chosen) == (g == 2), g


def test_one_group_is_the_merged_selection():
    r = _rng(3)
    q_c = r.standard_normal((2, 3, 16))
    k_c = r.standard_normal((2, 500, 16))
    a = esa_heads.score_select_heads(q_c, k_c, 497, 1, 8, 64, 40, 2, 6.0)
    b = esa.score_select(q_c, k_c, 497, 8, 64, 40, 2, 6.0)
    np.testing.assert_array_equal(a[0][:, 0], b[0])
    np.testing.assert_array_equal(a[1][:, 0], b[1])


def test_groups_select_on_their_own_slices():
    # the selection of group g equals the merged selection run on group g's columns
    # alone, and changing another group's columns leaves it unchanged
    r = _rng(4)
    ng, dg = 4, 8
    q_c = r.standard_normal((1, 2, ng * dg))
    k_c = r.standard_normal((1, 700, ng * dg))
    idx, count, sp = esa_heads.score_select_heads(q_c, k_c, 698, ng, 16, 100, 50, 2, 10.0)
    for g in range(ng):
        cols = slice(g * dg, (g + 1) * dg)
        ref = esa.score_select(q_c[:, :, cols], k_c[:, :, cols], 698, 16, 100, 50, 2, 10.0)
        np.testing.assert_array_equal(idx[:, g], ref[0])
    k2 = k_c.copy()
    k2[:, :, dg:] = r.standard_normal(k2[:, :, dg:].shape)
    idx2, _, _ = esa_heads.score_select_heads(q_c, k2, 698, ng, 16, 100, 50, 2, 10.0)
    np.testing.assert_array_equal(idx2[:, 0], idx[:, 0])
    assert not np.array_equal(idx2[:, 1:], idx[:, 1:])


def test_equal_lists_give_the_merged_attention():
    r = _rng(5)
    b, lq, hq, hkv, d, n = 2, 3, 8, 2, 16, 300
    c0 = n - lq
    q = r.standard_normal((b, lq, hq, d))
    k = r.standard_normal((b, n, hkv, d))
    v = r.standard_normal((b, n, hkv, d))
    _, (m0, m1), _ = esa.regions(c0, c0 + lq, 8, 50)
    sel = np.sort(r.choice(np.arange(m0, m1), 40, replace=False))
    idx = np.full((b, 64), -1)
    idx[:, :40] = sel
    count = np.full(b, 40)
    o_m, l_m = esa.sparse_attn(q, k, v, c0, idx, count, 8, 50)
    o_h, l_h = esa_heads.sparse_attn_heads(q, k, v, c0, np.repeat(idx[:, None], hkv, axis=1),
                                           np.repeat(count[:, None], hkv, axis=1), 8, 50)
    np.testing.assert_allclose(o_h, o_m, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l_h, l_m, rtol=1e-12, atol=1e-12)


def test_each_group_attends_its_own_list():
    # heads of group g with per-head lists equal the merged attention run with
    # group g's list, restricted to group g's heads
    r = _rng(6)
    b, lq, hq, hkv, d, n = 1, 2, 8, 4, 8, 260
    c0 = n - lq
    q = r.standard_normal((b, lq, hq, d))
    k = r.standard_normal((b, n, hkv, d))
    v = r.standard_normal((b, n, hkv, d))
    _, (m0, m1), _ = esa.regions(c0, c0 + lq, 4, 30)
    idx = np.full((b, hkv, 32), -1)
    count = np.zeros((b, hkv), dtype=np.int64)
    for g in range(hkv):
        c = 10 + 5 * g
        idx[0, g, :c] = np.sort(r.choice(np.arange(m0, m1), c, replace=False))
        count[0, g] = c
    o_h, _ = esa_heads.sparse_attn_heads(q, k, v, c0, idx, count, 4, 30)
    gs = hq // hkv
    for g in range(hkv):
        o_m, _ = esa.sparse_attn(q, k, v, c0, idx[:, g], count[:, g], 4, 30)
        np.testing.assert_allclose(o_h[:, :, g * gs:(g + 1) * gs], o_m[:, :, g * gs:(g + 1) * gs],
                                   rtol=1e-12, atol=1e-12)


def test_full_lists_give_full_causal_attention():
    # k >= |middle| for every head: exactly full causal attention (SDPA in float64)
    r = _rng(7)
    b, hq, hkv, d, n = 1, 4, 2, 8, 90
    q = r.standard_normal((b, 1, hq, d))
    k = r.standard_normal((b, n, hkv, d))
    v = r.standard_normal((b, n, hkv, d))
    wq = r.standard_normal((hkv, 2 * d, 4))
    wk = r.standard_normal((hkv, 2 * d, 4))
    out = esa_heads.decode_step_heads(q, k, v, wq, wk, 4, 10, n, 2, 3.0)
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.repeat(k, 2, axis=2)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.repeat(v, 2, axis=2)).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(out["o"], ref, rtol=1e-10, atol=1e-10)
