"""Offline fit of ESA's two compression maps: plain float64 restatement.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: the ESA write-up, compression paragraph (the one-layer maps of query and
key are learned offline: the model runs once over a small calibration set, its
queries and keys are kept, and the maps are trained on them without touching the
model; what matters is the relative size of the scores) and experiments paragraph
(4096 -> 128, two long calibration samples). The loss is not on the pages. The
reading taken here is the plain one: least squares of the compressed scores against
the full merged-head scores over every (calibration query, calibration key) pair,

    minimise  sum_ij ( compress(q_i, W_q) . compress(k_j, W_k) - s_ij )^2,
    s_ij = sum_h q_i^h . k_j^{h / G}   (the merged score of ``oracle.esa``),

with no bias and no activation (the maps of ``oracle.esa.compress``).

Solution. Write X [n_q, Hq*D] for the queries, Y [n_k, Hkv*D] for the keys and E
[Hq*D, Hkv*D] for the GQA expansion (E[h*D+e, g*D+e] = 1 when g = h / G). The
compressed key is Y B with B = E^T W_k, and the loss is ||X (W_q B^T - E) Y^T||_F^2.
With Cholesky factors X^T X = Rq^T Rq and Y^T Y = Rk^T Rk this equals
||Rq (W_q B^T - E) Rk^T||_F^2, so Rq W_q B^T Rk^T is the best rank-d' approximation
of C = Rq E Rk^T (Eckart-Young): with C's leading singular triples (U, S, V),
W_q = Rq^-1 U S^1/2 and B = Rk^-1 V S^1/2. Of the key maps with E^T W_k = B the
fit returns the smallest, W_k = E B / G (each of a group's G row blocks is B / G,
so the folded map used by the kernels, the sum over the group, is B). A ridge term
r * trace(G) / dim added to each Gram matrix keeps the factors defined when the
calibration set has fewer tokens than dimensions (r = 0: none).

Functions:
  expansion     - the GQA expansion matrix E
  fit_maps      - the least-squares maps (W_q, W_k), [Hq*D, d'] each
  scores_full   - s_ij for every calibration pair
  fit_loss      - the loss above for given maps
"""
from __future__ import annotations

import numpy as np


def expansion(hq, hkv, d):
    """E [hq*d, hkv*d]: query head h reads KV head h // (hq // hkv)."""
    g = hq // hkv
    e = np.zeros((hq * d, hkv * d))
    for h in range(hq):
        kv = h // g
        e[h * d:(h + 1) * d, kv * d:(kv + 1) * d] = np.eye(d)
    return e


def scores_full(q, k):
    """s [n_q, n_k]: merged-head scores of calibration queries q [n_q, Hq, D] and keys
    k [n_k, Hkv, D]."""
    hq, hkv = q.shape[1], k.shape[1]
    g = hq // hkv
    k_exp = np.repeat(k, g, axis=1)                                  # head h -> KV head h // g
    return q.reshape(q.shape[0], -1) @ k_exp.reshape(k.shape[0], -1).T


def _upper_cholesky(gram, ridge):
    dim = gram.shape[0]
    if ridge > 0.0:
        gram = gram + ridge * np.trace(gram) / dim * np.eye(dim)
    return np.linalg.cholesky(gram).T                                # gram = R^T R, R upper


def fit_maps(q, k, d_c, ridge=0.0):
    """Least-squares compression maps from calibration queries q [n_q, Hq, D] and keys
    k [n_k, Hkv, D] (float64). Returns (w_q, w_k), each [Hq*D, d_c], in the layout of
    ``oracle.esa.compress`` (keys are expanded to Hq heads before w_k)."""
    n_q, hq, d = q.shape
    hkv = k.shape[1]
    g = hq // hkv
    x = q.reshape(n_q, hq * d)
    y = k.reshape(k.shape[0], hkv * d)
    e = expansion(hq, hkv, d)
    r_q = _upper_cholesky(x.T @ x, ridge)
    r_k = _upper_cholesky(y.T @ y, ridge)
    c = r_q @ e @ r_k.T
    u, s, vt = np.linalg.svd(c, full_matrices=False)
    root = np.sqrt(s[:d_c])
    w_q = np.linalg.solve(r_q, u[:, :d_c] * root)
    b = np.linalg.solve(r_k, vt[:d_c].T * root)                      # [Hkv*D, d_c]
    w_k = e @ b / g
    return w_q, w_k


def fit_loss(q, k, w_q, w_k):
    """sum_ij (q~_i . k~_j - s_ij)^2 for the maps (w_q, w_k)."""
    from oracle import esa
    hq = q.shape[1]
    q_c = esa.compress(q, w_q, hq)
    k_c = esa.compress(k, w_k, hq)
    return float(((q_c @ k_c.T - scores_full(q, k)) ** 2).sum())
