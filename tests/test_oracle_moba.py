"""Pins for the MoBA oracle against things other than itself.

  * every past block selected  -> full causal attention (torch SDPA, float64);
  * no past block selected      -> block-local causal attention (torch SDPA with
    a block-diagonal causal mask): the sliding-window special case the MoBA
    article names in section 4;
  * a ramp key makes each block mean a closed form, pinning block boundaries;
  * gate choices checked by brute-force subset enumeration;
  * causality: perturbing tokens at or after p leaves every output before p;
  * the article's 95.31% sparsity at 64 blocks with 3 attended blocks.
"""
import itertools
import json

import numpy as np
import torch

from oracle import moba
from tests.conftest import golden_path


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, mask):
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    out = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    return out.permute(0, 2, 1, 3).numpy()


def check_all_blocks_is_full_attention():
    for s, block in [(40, 8), (37, 8), (16, 16)]:
        q, k, v = _rand((2, s, 3, 8), 1), _rand((2, s, 3, 8), 2), _rand((2, s, 3, 8), 3)
        r = moba.moba(q, k, v, block, topk=64)
        mask = torch.tril(torch.ones(s, s, dtype=torch.bool))
        np.testing.assert_allclose(r["o"], _sdpa(q, k, v, mask), atol=1e-12, rtol=0)


def test_all_blocks_is_full_attention():
    check_all_blocks_is_full_attention()


def check_no_past_block_is_block_local():
    s, block = 36, 8
    q, k, v = _rand((1, s, 2, 4), 4), _rand((1, s, 2, 4), 5), _rand((1, s, 2, 4), 6)
    r = moba.moba(q, k, v, block, topk=0)
    pos = torch.arange(s)
    same_block = (pos.view(s, 1) // block) == (pos.view(1, s) // block)
    mask = same_block & (pos.view(1, s) <= pos.view(s, 1))
    np.testing.assert_allclose(r["o"], _sdpa(q, k, v, mask), atol=1e-12, rtol=0)


def test_no_past_block_is_block_local():
    check_no_past_block_is_block_local()


def check_block_means_of_a_ramp():
    s, block = 29, 8
    k = np.broadcast_to(np.arange(s, dtype=np.float64).reshape(1, s, 1, 1), (1, s, 2, 3)).copy()
    kbar = moba.block_means(k, block)
    for b in range(4):
        lo, hi = b * block, min((b + 1) * block, s) - 1
        assert np.all(kbar[0, :, b, :] == (lo + hi) / 2.0)


def test_block_means_of_a_ramp():
    check_block_means_of_a_ramp()


def check_gate_brute_force():
    s, block, h, d = 48, 4, 2, 3
    rng = np.random.default_rng(9)
    q = np.round(rng.standard_normal((1, s, h, d)))
    k = np.round(rng.standard_normal((1, s, h, d)) * 2)       # integer-ish: ties happen
    kbar = moba.block_means(k, block)
    for topk in [0, 1, 3]:
        blocks = moba.gate(q, kbar, block, topk)
        for p in range(s):
            cur = p // block
            for hh in range(h):
                lst = [b for b in blocks[0, p, hh].tolist() if b >= 0]
                assert lst[-1] == cur and lst == sorted(lst)
                past = lst[:-1]
                assert len(past) == min(topk, cur)
                sc = [float(q[0, p, hh] @ kbar[0, hh, b]) for b in range(cur)]
                ok = [set(c) for c in itertools.combinations(range(cur), len(past))
                      if all(sc[a] > sc[b] or (sc[a] == sc[b] and a < b)
                             for a in c for b in range(cur) if b not in c)]
                assert len(ok) == 1 and set(past) == ok[0]


def test_gate_brute_force():
    check_gate_brute_force()


def check_causality():
    s, block = 40, 8
    q, k, v = _rand((1, s, 2, 4), 7), _rand((1, s, 2, 4), 8), _rand((1, s, 2, 4), 9)
    base = moba.moba(q, k, v, block, topk=2)
    for p0 in [9, 16, 33]:
        k2, v2 = k.copy(), v.copy()
        k2[:, p0:] += 3.0
        v2[:, p0:] -= 2.0
        r = moba.moba(q, k2, v2, block, topk=2)
        np.testing.assert_array_equal(r["o"][:, :p0], base["o"][:, :p0])
        np.testing.assert_array_equal(r["blocks"][:, :p0], base["blocks"][:, :p0])


def test_causality():
    check_causality()


def test_sparsity_matches_the_article():
    """MoBA article, experiments: 95.31% sparsity with 64 blocks and top-k = 3.
    Under this build's reading the article's 3 attended blocks are 2 gated past
    blocks plus the current one (topk = 2 here); a query in the last block then
    attends 3 of 64 blocks."""
    pages = json.load(open(golden_path("pages_numbers.json")))["moba_sparsity_pct"]
    s, block = 128, 2
    q, k = _rand((1, s, 1, 4), 10), _rand((1, s, 1, 4), 11)
    kbar = moba.block_means(k, block)
    blocks = moba.gate(q, kbar, block, topk=2, positions=[s - 1])
    attended = int((blocks[0, 0, 0] >= 0).sum())
    assert attended == pages["attended"]
    sparsity = 100.0 * (1.0 - attended / pages["blocks"])
    assert abs(sparsity - pages["value"]) <= pages["tol"]


def test_decode_step_pins():
    # all past blocks kept: the last row of full causal attention; none kept (topk 0):
    # attention over the current block only; otherwise the prefill's last row
    s, block, h, d = 43, 8, 3, 8
    q1, k, v = _rand((2, 1, h, d), 11), _rand((2, s, h, d), 12), _rand((2, s, h, d), 13)
    qfull = np.concatenate([np.zeros((2, s - 1, h, d)), q1], axis=1)
    full = _sdpa(qfull, k, v, torch.tril(torch.ones(s, s, dtype=torch.bool)))[:, -1:]
    np.testing.assert_allclose(moba.decode_step(q1, k, v, block, 64)["o"], full, atol=1e-12, rtol=0)
    cur0 = (s - 1) // block * block
    local = _sdpa(q1, k[:, cur0:], v[:, cur0:], None)
    np.testing.assert_allclose(moba.decode_step(q1, k, v, block, 0)["o"], local, atol=1e-12, rtol=0)
    r = moba.decode_step(q1, k, v, block, 2)
    assert (r["blocks"][:, 0, :, -1] == (s - 1) // block).all()
