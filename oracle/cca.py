"""CCA-style attention (core-token pooling + locality-preserving attention): plain
float64 restatement.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: the CCA-Attention article ("Core Context Aware Transformers for Long Context
Language Modeling"): global-aware pooling, locality-preserving module, and the
differentiable fusion of the two. The extracted text lost every formula; the
readings taken here:

  C1 pooling. The sequence is cut into groups of g consecutive tokens. Group j's core
     token is the average of the group's tokens weighted by the softmax of the scores
     of the group's last query against the group's keys (scale 1 / sqrt(D)). The
     article pools the hidden states and then applies the key and value projections;
     both are linear, so pooling the projected keys and values with the same weights
     is the same thing, and that is what is done here. The weights come from a query
     head, so core keys and values are per query head (head h pools KV head h / G).
     Only complete groups have a core token.
  C2 locality. Query i sees the original tokens of its window [lo_i, i] with
     lo_i = max(0, g * floor(i / g) - w), w a multiple of g: at least the previous w
     tokens, the window starting on a group boundary so that windows and groups tile
     the past without gap or overlap.
  C3 fusion. Query i attends, in one softmax (scale 1 / sqrt(D)), the core tokens of
     the groups that end before lo_i and the window's tokens. Causal by construction:
     a core token only summarises a group that ended before the window.

Functions:
  core_tokens  - core keys and values of every complete group
  window_start - lo_i of C2
  attend       - the fused attention of C3 (all rows, or sampled rows)
"""
from __future__ import annotations

import math

import numpy as np


def core_tokens(q, k, v, g, scale=None):
    """q [B, S, Hq, D], k, v [B, S, Hkv, D] -> (kc, vc) [B, S // g, Hq, D] (C1)."""
    bsz, s, hq, d = q.shape
    hkv = k.shape[2]
    gq = hq // hkv
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    m = s // g
    kc = np.zeros((bsz, m, hq, d))
    vc = np.zeros((bsz, m, hq, d))
    for b in range(bsz):
        for j in range(m):
            t0, t1 = j * g, (j + 1) * g
            for h in range(hq):
                kv = h // gq
                x = scale * (k[b, t0:t1, kv] @ q[b, t1 - 1, h])          # [g]
                a = np.exp(x - x.max())
                a /= a.sum()
                kc[b, j, h] = a @ k[b, t0:t1, kv]
                vc[b, j, h] = a @ v[b, t0:t1, kv]
    return kc, vc


def window_start(i, g, w):
    """lo_i = max(0, g * floor(i / g) - w) (C2)."""
    return max(0, g * (i // g) - w)


def attend(q, k, v, g, w, scale=None, rows=None):
    """The fused attention (C3). q [B, S, Hq, D], k, v [B, S, Hkv, D]; w a multiple of g.
    rows: None for every (b, i), or a list of (b, i). Returns (o [B, S, Hq, D],
    lse [B, S, Hq]); rows not computed are zero."""
    if w % g:
        raise ValueError("the window must be a multiple of the group size")
    bsz, s, hq, d = q.shape
    hkv = k.shape[2]
    gq = hq // hkv
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    kc, vc = core_tokens(q, k, v, g, scale)
    o = np.zeros((bsz, s, hq, d))
    lse = np.zeros((bsz, s, hq))
    todo = [(b, i) for b in range(bsz) for i in range(s)] if rows is None else rows
    for b, i in todo:
        lo = window_start(i, g, w)
        n_core = lo // g                                                  # groups ending before lo
        for h in range(hq):
            kv = h // gq
            keys = np.concatenate([kc[b, :n_core, h], k[b, lo:i + 1, kv]])
            vals = np.concatenate([vc[b, :n_core, h], v[b, lo:i + 1, kv]])
            x = scale * (keys @ q[b, i, h])
            mx = x.max()
            e = np.exp(x - mx)
            den = e.sum()
            o[b, i, h] = (e @ vals) / den
            lse[b, i, h] = mx + math.log(den)
    return o, lse
