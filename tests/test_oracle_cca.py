"""Pins of the CCA-style oracle (oracle/cca.py): reductions to full causal attention
(groups of one token, a window over everything), closed forms of the pooling (equal
keys, one dominant key), exact key counts and tiling of the past (through the
log-sum-exp and a position ramp), and causality."""
import math

import numpy as np
import torch

from oracle import cca


def _rng(seed):
    return np.random.default_rng(seed)


def _sdpa_causal(q, k, v):
    """float64 causal SDPA with GQA; q [B, S, Hq, D], k, v [B, S, Hkv, D]."""
    g = q.shape[2] // k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.repeat(k, g, axis=2)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.repeat(v, g, axis=2)).permute(0, 2, 1, 3)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True).permute(0, 2, 1, 3).numpy()


def _inputs(seed, b=1, s=40, hq=4, hkv=2, d=8):
    r = _rng(seed)
    return (r.standard_normal((b, s, hq, d)), r.standard_normal((b, s, hkv, d)), r.standard_normal((b, s, hkv, d)))


def check_groups_of_one_are_full_attention():
    # g = 1: each core token is its own token, and core + window cover [0, i]
    q, k, v = _inputs(0)
    o, _ = cca.attend(q, k, v, 1, 6)
    np.testing.assert_allclose(o, _sdpa_causal(q, k, v), rtol=1e-10, atol=1e-10)


def check_window_over_everything_is_full_attention():
    q, k, v = _inputs(1, s=37)
    o, _ = cca.attend(q, k, v, 4, 40)
    np.testing.assert_allclose(o, _sdpa_causal(q, k, v), rtol=1e-10, atol=1e-10)


def check_equal_keys_pool_to_the_mean():
    # equal keys in a group: uniform weights, so the core key is that key and the core
    # value the plain mean of the group's values
    q, k, v = _inputs(2, s=24)
    g = 6
    for j in range(24 // g):
        k[:, j * g:(j + 1) * g] = k[:, j * g:j * g + 1]
    kc, vc = cca.core_tokens(q, k, v, g)
    for j in range(24 // g):
        for h in range(4):
            np.testing.assert_allclose(kc[0, j, h], k[0, j * g, h // 2], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(vc[0, j, h], v[0, j * g:(j + 1) * g, h // 2].mean(axis=0), rtol=1e-12,
                                       atol=1e-12)


def check_dominant_key_is_the_core_token():
    # a key far along the group's LAST query takes all the weight of that query head;
    # the group's other queries point the opposite way, so pooling with any of them
    # would give that key almost none
    q, k, v = _inputs(3, s=16, hq=2, hkv=2)
    g, j, t = 8, 1, 11                                  # group 1 = tokens 8..15, last query at 15
    h = 0
    last = q[0, (j + 1) * g - 1, h]
    q[0, j * g:(j + 1) * g - 1, h] = -last
    k[0, t, h] = 60.0 * last / np.linalg.norm(last)
    kc, vc = cca.core_tokens(q, k, v, g)
    np.testing.assert_allclose(vc[0, j, h], v[0, t, h], rtol=0, atol=1e-9)
    np.testing.assert_allclose(kc[0, j, h], k[0, t, h], rtol=0, atol=1e-7)


def check_counts_and_tiling():
    # zero keys: every attended key gets the same weight, so lse = log(#keys) and, with
    # values = the position ramp, o = the mean over the attended keys of their values:
    # a core token contributes its group's mean position. This fixes the number of core
    # tokens and the window of every query, and that they tile [0, i] exactly.
    b, s, hq, hkv, d, g, w = 1, 50, 2, 1, 4, 5, 10
    q = _rng(4).standard_normal((b, s, hq, d))
    k = np.zeros((b, s, hkv, d))
    v = np.repeat(np.arange(s, dtype=np.float64)[None, :, None, None], d, axis=3)
    o, lse = cca.attend(q, k, v, g, w)
    for i in range(s):
        lo = max(0, g * (i // g) - w)
        cores = [j * g + (g - 1) / 2 for j in range(lo // g)]
        vals = cores + list(range(lo, i + 1))
        assert lo % g == 0 and i - lo + 1 >= min(i + 1, w)
        np.testing.assert_allclose(lse[0, i], math.log(len(vals)), rtol=0, atol=1e-12)
        np.testing.assert_allclose(o[0, i, :, 0], np.mean(vals), rtol=0, atol=1e-9)
    # and the reading itself: the groups behind the core tokens and the window cover
    # every position of [0, i] exactly once
    for i in range(s):
        lo = max(0, g * (i // g) - w)
        covered = [t for j in range(lo // g) for t in range(j * g, (j + 1) * g)] + list(range(lo, i + 1))
        assert sorted(covered) == list(range(i + 1))


def check_causal():
    q, k, v = _inputs(5, s=30)
    g, w = 3, 6
    o, _ = cca.attend(q, k, v, g, w)
    for i in (0, 7, 14, 22):
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        q2[:, i + 1:] += 5.0
        k2[:, i + 1:] -= 3.0
        v2[:, i + 1:] *= -2.0
        o2, _ = cca.attend(q2, k2, v2, g, w, rows=[(0, i)])
        np.testing.assert_allclose(o2[0, i], o[0, i], rtol=0, atol=0)


def test_groups_of_one_are_full_attention():
    check_groups_of_one_are_full_attention()


def test_window_over_everything_is_full_attention():
    check_window_over_everything_is_full_attention()


def test_equal_keys_pool_to_the_mean():
    check_equal_keys_pool_to_the_mean()


def test_dominant_key_is_the_core_token():
    check_dominant_key_is_the_core_token()


def test_counts_and_tiling():
    check_counts_and_tiling()


def test_causal():
    check_causal()
