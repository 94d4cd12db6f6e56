"""ESA decode over a batch of sequences of different lengths: plain float64 restatement.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: the ESA write-up ("Efficient Selective Attention"), problem statement
(decode of one query against its sequence's KV cache) and core steps. The pages
treat one sequence at a time and never batch sequences of different lengths, so
this module takes the plain reading: sequence b of a batch, holding seq_len[b]
cached tokens, runs the one-sequence decode step of ``oracle.esa`` (or of
``oracle.esa_heads`` for per-head selection) on rows [0, seq_len[b]) of its
caches, with its query at position seq_len[b] - 1. Rows past seq_len[b] take no
part. Outputs are padded to the batch shape: idx with -1, count with 0.

Functions:
  score_select_varlen - a3..a7 for each sequence at its own position
  sparse_attn_varlen  - a8 for each sequence at its own position
  decode_step_varlen  - a1..a8 for each sequence at its own position
"""
from __future__ import annotations

import numpy as np

from oracle import esa, esa_heads


def score_select_varlen(q_c, k_c, seq_len, n_init, window, topk, eps, clamp_c, n_groups=1):
    """Selection of one query per sequence at position seq_len[b] - 1.

    q_c: [B, 1, d'] and k_c: [B, n_cap, d'] compressed query and key cache.
    n_groups 1: the merged selection (esa.score_select); n_groups > 1: one selection
    per group of d' / n_groups columns (esa_heads.score_select_heads).
    Returns idx [B, n_groups, topk] (-1 padded), count [B, n_groups] and, per
    sequence, the list of per-group s' arrays over that sequence's own middle.
    """
    bsz = q_c.shape[0]
    idx = np.full((bsz, n_groups, topk), -1, dtype=np.int64)
    count = np.zeros((bsz, n_groups), dtype=np.int64)
    s_prime = []
    for b in range(bsz):
        n = int(seq_len[b])
        c0 = n - 1
        qb, kb = q_c[b:b + 1], k_c[b:b + 1, :n]
        if n_groups == 1:
            i1, c1, sp = esa.score_select(qb, kb, c0, n_init, window, topk, eps, clamp_c)
            idx[b, 0], count[b, 0] = i1[0], c1[0]
            s_prime.append([sp[0]])
        else:
            i1, c1, sp = esa_heads.score_select_heads(qb, kb, c0, n_groups, n_init, window, topk, eps, clamp_c)
            idx[b], count[b] = i1[0], c1[0]
            s_prime.append(list(sp[0]))
    return idx, count, s_prime


def sparse_attn_varlen(q, k, v, seq_len, idx, count, n_init, window, scale=None):
    """Attention of one query per sequence at position seq_len[b] - 1 over initial +
    idx[:count] + local tokens of its own sequence.

    q: [B, 1, Hq, D]; k, v: [B, n_cap, Hkv, D]; idx [B, L, >= topk], count [B, L] with
    L = 1 (one list for every head) or L = Hkv (one list per KV head).
    Returns o [B, 1, Hq, D] and lse [B, 1, Hq].
    """
    bsz, _, hq, d = q.shape
    lists = count.shape[1]
    o = np.zeros((bsz, 1, hq, d))
    lse = np.zeros((bsz, 1, hq))
    for b in range(bsz):
        n = int(seq_len[b])
        c0 = n - 1
        qb, kb, vb = q[b:b + 1], k[b:b + 1, :n], v[b:b + 1, :n]
        if lists == 1:
            ob, lb = esa.sparse_attn(qb, kb, vb, c0, idx[b:b + 1, 0], count[b:b + 1, 0], n_init, window, scale)
        else:
            ob, lb = esa_heads.sparse_attn_heads(qb, kb, vb, c0, idx[b:b + 1], count[b:b + 1], n_init, window,
                                                 scale)
        o[b], lse[b] = ob[0], lb[0]
    return o, lse


def decode_step_varlen(q, k, v, wq, wk, seq_len, n_init, window, topk, eps, clamp_c, scale=None):
    """The whole merged-selection decode step for a variable-length batch (a1..a8).

    q: [B, 1, Hq, D], the query of sequence b at position seq_len[b] - 1;
    k, v: [B, n_cap, Hkv, D]; wq, wk: [Hq*D, d'].
    Returns dict(idx, count, s_prime, o, lse) in the layouts of the functions above.
    """
    bsz, _, hq, _ = q.shape
    q_c = np.stack([esa.compress(q[b], wq, hq) for b in range(bsz)])                     # [B, 1, d']
    k_c = np.zeros((bsz, k.shape[1], wk.shape[1]))
    for b in range(bsz):
        n = int(seq_len[b])
        k_c[b, :n] = esa.compress(k[b, :n], wk, hq)
    idx, count, sp = score_select_varlen(q_c, k_c, seq_len, n_init, window, topk, eps, clamp_c)
    o, lse = sparse_attn_varlen(q, k, v, seq_len, idx, count, n_init, window, scale)
    return dict(idx=idx, count=count, s_prime=sp, o=o, lse=lse)
