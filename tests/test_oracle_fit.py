"""Pins of the offline compression-map fit (oracle/esa_fit.py) against what the
mathematics fixes: exact reconstruction at full rank, recovery of planted low-rank
scores, agreement with an independent alternating least-squares solver, local
optimality, the GQA folding of the key map, scale equivariance, and better top-k
recall than random maps on held-out tokens."""
import math

import numpy as np

from oracle import esa, esa_fit
from query_aware_selective_b200 import synthetic


def _rng(seed):
    return np.random.default_rng(seed)


def _calibration(hq, hkv, d, n, rank, seed, noise=0.1):
    q, k = synthetic.make_calibration(hq, hkv, d, n, rank, seed, noise)
    return q.double().numpy(), k.double().numpy()


def check_full_rank_fit_is_exact():
    # d' = Hkv * D: the maps can carry every merged score exactly
    r = _rng(0)
    q = r.standard_normal((64, 4, 4))
    k = r.standard_normal((48, 2, 4))
    w_q, w_k = esa_fit.fit_maps(q, k, 8)
    s = esa_fit.scores_full(q, k)
    q_c, k_c = esa.compress(q, w_q, 4), esa.compress(k, w_k, 4)
    np.testing.assert_allclose(q_c @ k_c.T, s, rtol=1e-9, atol=1e-9 * np.abs(s).max())


def check_planted_rank_is_recovered():
    # scores of exact rank 3 (noise-free latents) are fitted exactly with d' = 3 < Hkv * D
    q, k = _calibration(8, 2, 16, 300, 3, seed=6, noise=0.0)
    w_q, w_k = esa_fit.fit_maps(q, k, 3, ridge=1e-12)
    s = esa_fit.scores_full(q, k)
    assert esa_fit.fit_loss(q, k, w_q, w_k) <= 1e-16 * float((s ** 2).sum())


def _als(q, k, d_c, iters, seed):
    """Alternating least squares on the same loss, written independently: with the
    compressed keys fixed, W_q solves a linear least-squares problem, and back."""
    hq, hkv, d = q.shape[1], k.shape[1], q.shape[2]
    x = q.reshape(len(q), hq * d)
    y = np.repeat(k, hq // hkv, axis=1).reshape(len(k), hq * d)
    s = x @ y.T
    r = _rng(seed)
    w_k = r.standard_normal((hq * d, d_c))
    for _ in range(iters):
        kc = y @ w_k                                                   # [n_k, d']
        # s ~ x W_q kc^T: vec(W_q) by least squares on kron(kc, x)
        a = np.kron(kc, x)
        w_q = np.linalg.lstsq(a, s.T.reshape(-1), rcond=None)[0].reshape(d_c, hq * d).T
        qc = x @ w_q
        a = np.kron(qc, y)
        w_k = np.linalg.lstsq(a, s.reshape(-1), rcond=None)[0].reshape(d_c, hq * d).T
    return w_q, w_k


def check_matches_alternating_least_squares():
    # the closed form is the global minimum: ALS converges to the same loss, never below
    q, k = _calibration(2, 1, 3, 40, 3, seed=8, noise=0.3)
    w_q, w_k = esa_fit.fit_maps(q, k, 2)
    best = esa_fit.fit_loss(q, k, w_q, w_k)
    for seed in (0, 1):
        a_q, a_k = _als(q, k, 2, iters=300, seed=seed)
        als = esa_fit.fit_loss(q, k, a_q, a_k)
        assert als >= best * (1 - 1e-9)
        assert als <= best * (1 + 1e-4), (als, best)


def check_local_optimality():
    q, k = _calibration(4, 2, 8, 200, 4, seed=9)
    w_q, w_k = esa_fit.fit_maps(q, k, 4)
    base = esa_fit.fit_loss(q, k, w_q, w_k)
    r = _rng(10)
    for _ in range(10):
        dq = 1e-4 * r.standard_normal(w_q.shape) * np.abs(w_q).max()
        dk = 1e-4 * r.standard_normal(w_k.shape) * np.abs(w_k).max()
        assert esa_fit.fit_loss(q, k, w_q + dq, w_k + dk) >= base * (1 - 1e-12)


def check_key_map_folds_per_group():
    # the key map's G row blocks per KV head are equal, so the expanded key map equals
    # the folded one (the sum over the group) applied to the unexpanded key
    hq, hkv, d = 8, 2, 4
    q, k = _calibration(hq, hkv, d, 120, 4, seed=11)
    _, w_k = esa_fit.fit_maps(q, k, 4)
    g = hq // hkv
    blocks = w_k.reshape(hq, d, 4)
    for kv in range(hkv):
        for j in range(1, g):
            np.testing.assert_allclose(blocks[kv * g + j], blocks[kv * g], rtol=0, atol=0)
    folded = blocks.reshape(hkv, g, d, 4).sum(axis=1).reshape(hkv * d, 4)
    np.testing.assert_allclose(esa.compress(k, w_k, hq), k.reshape(len(k), -1) @ folded, rtol=1e-12, atol=1e-12)


def check_scale_equivariance():
    # queries scaled by c: the fitted compressed scores scale by c
    q, k = _calibration(4, 2, 8, 150, 4, seed=12)
    w_q, w_k = esa_fit.fit_maps(q, k, 4)
    v_q, v_k = esa_fit.fit_maps(3.0 * q, k, 4)
    a = esa.compress(q, w_q, 4) @ esa.compress(k, w_k, 4).T
    b = esa.compress(3.0 * q, v_q, 4) @ esa.compress(k, v_k, 4).T
    np.testing.assert_allclose(b, 3.0 * a, rtol=1e-8, atol=1e-8 * np.abs(a).max())


def check_fit_improves_held_out_selection():
    # fitted on half of the tokens, the maps keep most of the other half's top-50 by full
    # score; random maps of the same size keep few
    hq, hkv, d, d_c, topk = 8, 2, 16, 8, 50
    q, k = _calibration(hq, hkv, d, 2000, 8, seed=7)
    w_q, w_k = esa_fit.fit_maps(q[:1000], k[:1000], d_c)
    r = _rng(1)
    r_q = r.standard_normal((hq * d, d_c)) / math.sqrt(hq * d)
    r_k = r.standard_normal((hq * d, d_c)) / math.sqrt(hq * d)
    qh, kh = q[1000:1020], k[1000:]
    full = esa_fit.scores_full(qh, kh)

    def recall(a, b):
        comp = esa.compress(qh, a, hq) @ esa.compress(kh, b, hq).T
        return np.mean([len(set(np.argsort(-full[i])[:topk]) & set(np.argsort(-comp[i])[:topk])) / topk
                        for i in range(len(qh))])
    fitted, random = recall(w_q, w_k), recall(r_q, r_k)
    assert fitted >= 0.9 and random <= 0.5, (fitted, random)


def test_full_rank_fit_is_exact():
    check_full_rank_fit_is_exact()


def test_planted_rank_is_recovered():
    check_planted_rank_is_recovered()


def test_matches_alternating_least_squares():
    check_matches_alternating_least_squares()


def test_local_optimality():
    check_local_optimality()


def test_key_map_folds_per_group():
    check_key_map_folds_per_group()


def test_scale_equivariance():
    check_scale_equivariance()


def test_fit_improves_held_out_selection():
    check_fit_improves_held_out_selection()
