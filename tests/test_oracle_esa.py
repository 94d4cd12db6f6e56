"""Pins for the ESA oracle against things other than itself.

Each check is a plain function so that tests/test_oracle_mutations.py can plant
a mistake in the oracle and show that some check fails. Pins used:
  * torch's scaled_dot_product_attention (float64, CPU) when every middle token
    is selected: ESA then is exactly full causal attention;
  * a probe key that reads the log-sum-exp back out of the library attention;
  * identity compression, which turns the compressed score into the textbook
    multi-head dot product;
  * a hand-derived worked example (tests/golden/esa_selection_worked.json);
  * brute-force subset enumeration for the top-k order;
  * algebraic identities of the max filter and of the unclamped correction;
  * planted needles found together with their +-eps neighbours.
"""
import itertools
import json
import math

import numpy as np
import pytest
import torch

from oracle import esa
from query_aware_selective_b200 import synthetic
from tests.conftest import golden_path


def _rand(shape, seed, dtype=np.float64):
    return np.random.default_rng(seed).standard_normal(shape).astype(dtype)


# --------------------------------------------------------------------------- attention

def _sdpa_reference(q, k, v, c0, extra_probe=False):
    """Full causal attention for queries at c0.. from torch SDPA (float64)."""
    bsz, lq, hq, d = q.shape
    hkv = k.shape[2]
    n = c0 + lq
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)                  # [B, Hq, Lq, D]
    kt = torch.from_numpy(np.ascontiguousarray(k[:, :n])).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.ascontiguousarray(v[:, :n])).permute(0, 2, 1, 3)
    qpos = torch.arange(c0, c0 + lq).view(lq, 1)
    kpos = torch.arange(n).view(1, n)
    mask = kpos <= qpos
    if extra_probe:
        # a zero key (logit 0 for every query) whose value is a unit vector in a new
        # dimension; the output's last component is 1 / (1 + exp(lse)).
        kt = torch.cat([kt, torch.zeros(bsz, hkv, 1, d, dtype=kt.dtype)], dim=2)
        vt = torch.cat([vt, torch.zeros(bsz, hkv, n, 1, dtype=vt.dtype)], dim=3)
        probe_v = torch.zeros(bsz, hkv, 1, d + 1, dtype=vt.dtype)
        probe_v[..., -1] = 1.0
        vt = torch.cat([vt, probe_v], dim=2)
        mask = torch.cat([mask, torch.ones(lq, 1, dtype=torch.bool)], dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask,
                                                           enable_gqa=True)
    return out.permute(0, 2, 1, 3).numpy()


def check_full_selection_is_causal_attention():
    bsz, hq, hkv, d, n_init, window = 2, 4, 2, 16, 4, 16
    for c0, lq in [(64, 32), (95, 1), (40, 8), (0, 24), (3, 5)]:
        n = c0 + lq
        q = _rand((bsz, lq, hq, d), 1 + c0)
        k = _rand((bsz, n, hkv, d), 2 + c0)
        v = _rand((bsz, n, hkv, d), 3 + c0)
        _, (m0, m1), _ = esa.regions(c0, c0 + lq, n_init, window)
        topk = max(1, m1 - m0) + 3
        idx = np.full((bsz, topk), -1)
        idx[:, :m1 - m0] = np.arange(m0, m1)
        count = np.full(bsz, m1 - m0)
        o, lse = esa.sparse_attn(q, k, v, c0, idx, count, n_init, window)
        ref = _sdpa_reference(q, k, v, c0)
        np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)
        probe = _sdpa_reference(q, k, v, c0, extra_probe=True)[..., -1]
        lse_ref = np.log(1.0 / probe - 1.0)
        np.testing.assert_allclose(lse, lse_ref, atol=1e-9, rtol=0)


def test_full_selection_is_causal_attention():
    check_full_selection_is_causal_attention()


def check_attended_count():
    """Every query attends initial + min(k, |mid|) + its causal share of local."""
    bsz, hq, hkv, d = 1, 2, 1, 4
    for (c0, lq, n_init, window, topk) in [(200, 8, 16, 32, 20), (60, 1, 8, 16, 100),
                                           (5, 4, 8, 16, 3), (1000, 3, 0, 64, 50)]:
        n = c0 + lq
        (i0, i1), (m0, m1), (l0, l1) = esa.regions(c0, c0 + lq, n_init, window)
        assert i0 == 0 and i1 <= m0 or m1 == m0
        assert l1 == n and (m1 - m0 == 0 or m1 == l0)
        # parts are disjoint and cover [0, n)
        cover = np.concatenate([np.arange(i0, i1), np.arange(m0, m1), np.arange(l0, l1)])
        assert np.array_equal(np.sort(cover), np.arange(n))
        cnt = min(topk, m1 - m0)
        idx = np.full((bsz, topk), -1)
        idx[0, :cnt] = np.arange(m0, m0 + cnt)
        keys = esa.attended_keys(c0, lq, n_init, window, idx[0], cnt)
        for i in range(lq):
            seen = int((keys <= c0 + i).sum())
            assert seen == (i1 - i0) + cnt + (c0 + i - l0 + 1)
        # the local part holds `window` cached tokens before the chunk once the
        # chunk is past the initial tokens and the window
        if c0 >= n_init + window:
            assert c0 - l0 == window


def test_attended_count():
    check_attended_count()


def test_decode_128k_attends_about_6k_tokens():
    """ESA write-up, experiments: the attention window is about 6k tokens."""
    pages = json.load(open(golden_path("pages_numbers.json")))
    w = synthetic.DECODE_128K
    c0 = w.n_ctx - 1
    (i0, i1), (m0, m1), (l0, l1) = esa.regions(c0, c0 + 1, w.n_init, w.window)
    total = (i1 - i0) + min(w.topk, m1 - m0) + (l1 - l0)
    assert total == 128 + 2048 + 4097
    assert abs(total - pages["esa_window_tokens"]["value"]) <= \
        pages["esa_window_tokens"]["tol_rel"] * pages["esa_window_tokens"]["value"]


# --------------------------------------------------------------------------- compression

def check_identity_compression_is_multihead_dot():
    """With W = I the compressed vectors are the merged heads, and q~.k~ is the
    sum over query heads h of q_h . k_{h // G} (textbook GQA dot product)."""
    hq, hkv, d = 4, 2, 3
    g = hq // hkv
    rng = np.random.default_rng(7)
    xq = rng.standard_normal((5, hq, d))
    xk = rng.standard_normal((6, hkv, d))
    eye = np.eye(hq * d)
    qc = esa.compress(xq, eye, hq)
    kc = esa.compress(xk, eye, hq)
    for r in range(5):
        assert np.array_equal(qc[r], np.concatenate([xq[r, h] for h in range(hq)]))
    for r in range(6):
        expect = np.concatenate([xk[r, h // g] for h in range(hq)])
        assert np.array_equal(kc[r], expect)
    for a in range(5):
        for b in range(6):
            dot = sum(float(np.dot(xq[a, h], xk[b, h // g])) for h in range(hq))
            assert abs(float(qc[a] @ kc[b]) - dot) < 1e-12


def test_identity_compression_is_multihead_dot():
    check_identity_compression_is_multihead_dot()


def test_compress_is_linear_and_matches_a_plain_matmul():
    """Against torch.matmul on the explicitly expanded input (library routine)."""
    hq, hkv, d, dc = 8, 2, 16, 5
    rng = np.random.default_rng(3)
    x = rng.standard_normal((9, hkv, d))
    w = rng.standard_normal((hq * d, dc))
    got = esa.compress(x, w, hq)
    xt = torch.from_numpy(x).repeat_interleave(hq // hkv, dim=1).reshape(9, hq * d)
    ref = (xt @ torch.from_numpy(w)).numpy()
    np.testing.assert_allclose(got, ref, atol=1e-12)
    np.testing.assert_allclose(esa.compress(2 * x, w, hq), 2 * got, atol=1e-12)


# --------------------------------------------------------------------------- selection

def check_worked_example():
    ex = json.load(open(golden_path("esa_selection_worked.json")))
    qc = np.array(ex["q_c"])
    kc = np.array(ex["k_c"])
    for case in ex["cases"]:
        c = math.inf if case["clamp_c"] == "inf" else float(case["clamp_c"])
        s = esa.importance(qc, kc, c)
        np.testing.assert_array_equal(s, np.array(case["s"], dtype=float))
        sp = esa.neighbour_max(s, case["eps"])
        np.testing.assert_array_equal(sp, np.array(case["s_prime"], dtype=float))
        got = esa.topk_ascending(sp, case["topk"])
        assert got.tolist() == case["idx"], (case, got)
        # the same through the batched call (middle starts at n_init=0, window 0)
        n = kc.shape[0]
        kcache = np.concatenate([kc, np.zeros((qc.shape[0], 2))])[None]
        idx, count, _ = esa.score_select(qc[None], kcache, n, 0, 0, case["topk"], case["eps"], c)
        assert idx[0, :count[0]].tolist() == case["idx"]


def test_worked_example():
    check_worked_example()


def _dominates(a, b, v):
    """(value desc, index asc) order: a ranks above b."""
    return v[a] > v[b] or (v[a] == v[b] and a < b)


def check_topk_brute_force():
    """The kept set is the unique size-k subset whose every member ranks above
    every non-member; found here by enumerating all subsets."""
    rng = np.random.default_rng(11)
    for trial in range(60):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, 10))
        vals = np.round(rng.standard_normal(n) * 2) / 2      # coarse values: many ties
        keep = min(k, n)
        winners = [set(c) for c in itertools.combinations(range(n), keep)
                   if all(_dominates(a, b, vals) for a in c for b in range(n) if b not in c)]
        assert len(winners) == 1
        got = esa.topk_ascending(vals, k)
        assert set(got.tolist()) == winners[0]
        assert list(got) == sorted(got)


def test_topk_brute_force():
    check_topk_brute_force()


def check_neighbour_max_properties():
    rng = np.random.default_rng(5)
    for n in [1, 2, 5, 17, 64]:
        s = rng.standard_normal(n)
        for eps in [0, 1, 2, 3]:
            sp = esa.neighbour_max(s, eps)
            assert np.all(sp >= s)
            if eps == 0:
                assert np.array_equal(sp, s)
            # symmetric window: reversing the input reverses the output
            assert np.array_equal(esa.neighbour_max(s[::-1], eps), sp[::-1])
            # max filters compose: radius a then radius b is radius a + b
            for e2 in [1, 2]:
                assert np.array_equal(esa.neighbour_max(sp, e2), esa.neighbour_max(s, eps + e2))
        # a single spike becomes a plateau of width 2*eps+1, cut at the edges
        for eps in [1, 2]:
            for j0 in [0, n // 2, n - 1]:
                spike = np.full(n, -1.0)
                spike[j0] = 5.0
                sp = esa.neighbour_max(spike, eps)
                expect = [5.0 if abs(j - j0) <= eps else -1.0 for j in range(n)]
                assert sp.tolist() == expect


def test_neighbour_max_properties():
    check_neighbour_max_properties()


def check_single_query_no_clamp_is_plain_topk():
    """eps = 0, C = inf, one query: the selection is the plain top-k of q~.k~
    (checked with torch.topk on tie-free values)."""
    rng = np.random.default_rng(21)
    for trial in range(5):
        n_mid, dc, k = 300, 8, 17
        qc = rng.standard_normal((1, 1, dc))
        kc = rng.standard_normal((1, 10 + n_mid + 20, dc))
        c0 = kc.shape[1] - 1
        n_init, window = 10, c0 - 10 - n_mid
        idx, count, _ = esa.score_select(qc, kc, c0, n_init, window, k, 0, math.inf)
        scores = torch.from_numpy(kc[0, n_init:n_init + n_mid] @ qc[0, 0])
        ref = torch.topk(scores, k).indices.sort().values.numpy() + n_init
        assert count[0] == k and np.array_equal(idx[0], ref)


def test_single_query_no_clamp_is_plain_topk():
    check_single_query_no_clamp_is_plain_topk()


def check_unclamped_chunk_is_summed_query():
    """C = inf: sum_i (S_ij - m_i) = (sum_i q~_i).k~_j - const, so the selection
    equals the one made by the single summed query."""
    rng = np.random.default_rng(22)
    n_mid, dc, lq, k, eps = 400, 8, 6, 25, 2
    qc = rng.standard_normal((1, lq, dc))
    kc = rng.standard_normal((1, 5 + n_mid + 40, dc))
    c0 = kc.shape[1] - lq
    window = c0 - 5 - n_mid
    a, ca, _ = esa.score_select(qc, kc, c0, 5, window, k, eps, math.inf)
    b, cb, _ = esa.score_select(qc.sum(axis=1, keepdims=True), kc, c0, 5, window, k, eps, math.inf)
    assert np.array_equal(a, b) and np.array_equal(ca, cb)


def test_unclamped_chunk_is_summed_query():
    check_unclamped_chunk_is_summed_query()


def test_zero_clamp_keeps_the_first_k():
    """C = 0: every corrected score is 0, and the tie order keeps the first k."""
    rng = np.random.default_rng(23)
    qc = rng.standard_normal((2, 3, 4))
    kc = rng.standard_normal((2, 100, 4))
    idx, count, _ = esa.score_select(qc, kc, 97, 8, 30, 10, 2, 0.0)
    for b in range(2):
        assert idx[b].tolist() == list(range(8, 18))


def test_short_middle_selects_everything():
    rng = np.random.default_rng(24)
    qc = rng.standard_normal((1, 1, 4))
    kc = rng.standard_normal((1, 50, 4))
    idx, count, _ = esa.score_select(qc, kc, 49, 8, 30, 64, 2, 16.0)
    assert count[0] == 11 and idx[0, :11].tolist() == list(range(8, 19))
    assert (idx[0, 11:] == -1).all()
    idx, count, _ = esa.score_select(qc, kc, 49, 8, 41, 64, 2, 16.0)   # empty middle
    assert count[0] == 0 and (idx == -1).all()


def check_needles_selected_with_neighbours():
    """Planted needle keys aimed at the query are selected, each together with
    its +-eps neighbours (consequence of the max-pool reading)."""
    w = synthetic.TINY_DECODE
    inp = synthetic.make_esa_inputs(w)
    r = esa.decode_step(inp["q"].numpy(), inp["k"].numpy(), inp["v"].numpy(),
                        inp["wq"].numpy(), inp["wk"].numpy(), w.n_init, w.window,
                        w.topk, w.eps, w.clamp_c)
    chosen = set(r["idx"][0, :r["count"][0]].tolist())
    assert r["count"][0] == w.topk
    for p in inp["needles"][0].tolist():
        for j in range(p - w.eps, p + w.eps + 1):
            assert j in chosen, (p, j)


def test_needles_selected_with_neighbours():
    check_needles_selected_with_neighbours()


def test_tiny_decode_output_is_finite_and_normalised():
    w = synthetic.TINY_DECODE
    inp = synthetic.make_esa_inputs(w)
    r = esa.decode_step(inp["q"].numpy(), inp["k"].numpy(), inp["v"].numpy(),
                        inp["wq"].numpy(), inp["wk"].numpy(), w.n_init, w.window,
                        w.topk, w.eps, w.clamp_c)
    assert np.isfinite(r["o"]).all() and np.isfinite(r["lse"]).all()
    # attention output is a convex combination of the attended values
    assert np.abs(r["o"]).max() <= np.abs(inp["v"].numpy()).max() + 1e-12
