"""MoBA oracle: plain float64 restatement of Mixture of Block Attention.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: the MoBA article (arXiv 2502.13189), "MoBA architecture": section 1
(standard attention), section 2 (dynamic block selection,
MoBA(q, K, V) = Softmax(q K[I]^T) V[I]), section 3 (block partition
I_i = [(i-1)B + 1, iB], gate s_i = <q, mean_pool(K[I_i])>, top-k gate, and
causality: s_i = -inf for blocks after the query, the current block always
attended with a causal mask).

Positions here are 0-based: block b covers [b*Bs, min((b+1)*Bs, S)).

Readings:
  * Gate candidates are the blocks strictly before the query's block. With the
    article's 1-based positions the last token of block i has pos = i*B and is
    not masked by "pos(q) < i*B", which would make its own block a gate
    candidate too; since the current block is added anyway, the gate is read as
    choosing among past blocks only, then adding the current block.
  * `topk` counts past blocks; the current block is extra (at most topk + 1
    blocks attended). A query in block c < topk attends every past block.
  * Ties in the gate go to the lower block index.
  * Every (query, head) gates on its own; block means are per head.
  * The softmax takes the scale 1/sqrt(D) of standard attention (the article's
    formulas print none); the gate uses the raw <q, mean> (the scale would not
    change its ranking).
"""
from __future__ import annotations

import math

import numpy as np


def block_means(k, block):
    """Mean of the keys of each block, per head: [B, S, H, D] -> [B, H, nb, D]."""
    k = np.asarray(k, dtype=np.float64)
    bsz, s, h, d = k.shape
    nb = (s + block - 1) // block
    out = np.empty((bsz, h, nb, d))
    for b in range(nb):
        out[:, :, b, :] = k[:, b * block:min((b + 1) * block, s)].mean(axis=1)
    return out


def gate(q, kbar, block, topk, positions=None):
    """Block choice per (query, head): top-k past blocks by <q, mean>, then the
    current block. Returns [B, S', H, topk+1] int64 lists, ascending, -1 padded.

    q: [B, S, H, D]; kbar: [B, H, nb, D]; positions: optional subset of query
    positions (default all). Output rows follow ``positions``.
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, s, h, _ = q.shape
    if positions is None:
        positions = np.arange(s)
    out = np.full((bsz, len(positions), h, topk + 1), -1, dtype=np.int64)
    for r, p in enumerate(positions):
        cur = p // block
        for b in range(bsz):
            if cur > 0:
                sc = np.einsum("hd,hnd->hn", q[b, p], kbar[b, :, :cur, :])   # [H, cur]
            for hh in range(h):
                if cur > 0:
                    vals = sc[hh]
                    order = np.lexsort((np.arange(cur), -vals))               # value desc, index asc
                    chosen = np.sort(order[:min(topk, cur)])
                else:
                    chosen = np.zeros(0, dtype=np.int64)
                lst = np.concatenate([chosen, [cur]])
                out[b, r, hh, :len(lst)] = lst
    return out


def attend(q, k, v, blocks, block, scale=None, positions=None):
    """Attention of each (query, head) over its blocks; the current block is
    cut causally at the query. blocks: [B, S', H, topk+1] as ``gate`` returns
    (rows follow ``positions``). Returns (o [B, S', H, D], lse [B, S', H])."""
    bsz, s, h, d = q.shape
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    if positions is None:
        positions = np.arange(s)
    o = np.empty((bsz, len(positions), h, d))
    lse = np.empty((bsz, len(positions), h))
    for r, p in enumerate(positions):
        cur = p // block
        for b in range(bsz):
            for hh in range(h):
                keys = []
                for blk in blocks[b, r, hh]:
                    if blk < 0:
                        continue
                    end = min((blk + 1) * block, s)
                    if blk == cur:
                        end = p + 1
                    keys.append(np.arange(blk * block, end))
                keys = np.concatenate(keys)
                kk = np.asarray(k[b, keys, hh], dtype=np.float64)
                vv = np.asarray(v[b, keys, hh], dtype=np.float64)
                logits = kk @ np.asarray(q[b, p, hh], dtype=np.float64) * scale
                mx = logits.max()
                e = np.exp(logits - mx)
                o[b, r, hh] = e @ vv / e.sum()
                lse[b, r, hh] = mx + math.log(e.sum())
    return o, lse


def moba(q, k, v, block, topk, scale=None, positions=None):
    """The whole MoBA causal prefill for the given query positions."""
    kbar = block_means(k, block)
    blocks = gate(q, kbar, block, topk, positions)
    o, lse = attend(q, k, v, blocks, block, scale, positions)
    return dict(kbar=kbar, blocks=blocks, o=o, lse=lse)


def decode_step(q1, k, v, block, topk, scale=None):
    """MoBA for one query per sequence at the last cached position (decode): the same
    gate and attention as the prefill, evaluated at position S - 1 only.
    q1: [B, 1, H, D]; k, v: [B, S, H, D]. Returns dict(blocks [B, 1, H, topk+1],
    o [B, 1, H, D], lse [B, 1, H])."""
    bsz, s, h, d = np.shape(k)
    q = np.zeros((bsz, s, h, d))
    q[:, s - 1] = np.asarray(q1, dtype=np.float64)[:, 0]
    out = moba(q, k, v, block, topk, scale, positions=[s - 1])
    return dict(blocks=out["blocks"], o=out["o"], lse=out["lse"])

