"""ESA per-head selection variant: plain float64 restatement.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: the ESA write-up (Huawei Noah's Ark, "Efficient Selective Attention";
arXiv 2502.14477), ablation paragraph after "experiments": ESA does not choose
tokens for every head on its own but merges all heads into one importance score,
and the authors compare that with a per-head choice (the difference is small).
The per-head form is not written out. Reading taken here (one index set per KV
head, because the K/V rows the attention reads are per KV head):

  * group g = the query heads h with h // G == g and KV head g;
  * group g's queries and keys go through the group's own one-layer map,
    G*D -> d_g with d_g = d' / Hkv (512 -> 16 at the Llama-3-8B shape: the same
    ~3.1% as the merged 4096 -> 128); keys are expanded to the G query heads of
    the group first, exactly as the merged form expands them to all Hq heads;
  * S^g_ij = q~^g_i . k~^g_j, then the merged form's correction, clamp, chunk sum,
    neighbour max and top-k, separately for every (sequence, group);
  * query head h attends initial + I_{h // G} + local.

Stacked block-diagonally, the groups' maps form one Hq*D -> Hkv*d_g map whose
output is the concatenation of the groups' compressed vectors; the kernels use
that form, this file the per-group one.

Functions:
  compress_heads        - the groups' maps (a1, a2 per group)
  score_select_heads    - a3..a7 per (sequence, group)
  sparse_attn_heads     - a8 with one key list per KV head
  decode_step_heads     - the whole per-head decode path
"""
from __future__ import annotations

import math

import numpy as np

from oracle import esa


def compress_heads(x, w_groups, n_heads_out):
    """The groups' one-layer maps.

    x: [rows, n_heads_in, D] (n_heads_in = Hq for queries, Hkv for keys);
    w_groups: [n_groups, (n_heads_out / n_groups) * D, d_g]. Keys are expanded to
    the n_heads_out query heads (head h <- input head h // (n_heads_out / n_heads_in))
    before the group of head h takes them. Returns [rows, n_groups * d_g]: group g's
    compressed vector in columns [g * d_g, (g + 1) * d_g).
    """
    w_groups = np.asarray(w_groups, dtype=np.float64)
    n_groups, gin, dg = w_groups.shape
    rows, n_in, d = x.shape
    assert n_heads_out % n_in == 0 and n_heads_out % n_groups == 0
    hpg = n_heads_out // n_groups                      # query heads per group
    assert gin == hpg * d
    xe = np.repeat(np.asarray(x, dtype=np.float64), n_heads_out // n_in, axis=1)   # [rows, Hq, D]
    out = np.empty((rows, n_groups * dg), dtype=np.float64)
    for g in range(n_groups):
        xg = xe[:, g * hpg:(g + 1) * hpg, :].reshape(rows, hpg * d)
        out[:, g * dg:(g + 1) * dg] = xg @ w_groups[g]
    return out


def score_select_heads(q_c, k_c, c0, n_groups, n_init, window, topk, eps, clamp_c):
    """Per-group selection for one chunk of every sequence (a3..a7 per group).

    q_c: [B, Lq, n_groups * d_g]; k_c: [B, >= c0 + Lq, n_groups * d_g].
    Returns (idx [B, n_groups, topk] int64, ascending, -1 padded;
             count [B, n_groups]; s_prime[b][g] arrays of the middle).
    """
    q_c = np.asarray(q_c, dtype=np.float64)
    bsz, lq, dc = q_c.shape
    assert dc % n_groups == 0
    dg = dc // n_groups
    idx = np.full((bsz, n_groups, topk), -1, dtype=np.int64)
    count = np.zeros((bsz, n_groups), dtype=np.int64)
    s_primes = [[None] * n_groups for _ in range(bsz)]
    for g in range(n_groups):
        cols = slice(g * dg, (g + 1) * dg)
        ig, cg, sg = esa.score_select(q_c[:, :, cols], np.asarray(k_c)[:, :, cols], c0, n_init, window, topk, eps,
                                      clamp_c)
        idx[:, g] = ig
        count[:, g] = cg
        for b in range(bsz):
            s_primes[b][g] = sg[b]
    return idx, count, s_primes


def sparse_attn_heads(q, k, v, c0, idx, count, n_init, window, scale=None, rows=None):
    """Exact attention with one key list per KV head (a8 per group).

    q: [B, Lq, Hq, D]; k, v: [B, >= c0 + Lq, Hkv, D]; idx [B, Hkv, >= count],
    count [B, Hkv]. Query head h uses the list of KV head h // G. rows: optional
    list of (b, i) pairs. Returns (o [B, Lq, Hq, D], lse [B, Lq, Hq]) float64.
    """
    bsz, lq, hq, d = q.shape
    hkv = k.shape[2]
    g_sz = hq // hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    o = np.full((bsz, lq, hq, d), np.nan)
    lse = np.full((bsz, lq, hq), np.nan)
    if rows is None:
        rows = [(b, i) for b in range(bsz) for i in range(lq)]
    by_seq = {}
    for b, i in rows:
        by_seq.setdefault(b, []).append(i)
    for b, items in by_seq.items():
        for g in range(hkv):
            keys = esa.attended_keys(c0, lq, n_init, window, idx[b, g], int(count[b, g]))
            kg = np.asarray(k[b, keys, g], dtype=np.float64)      # [L, D]
            vg = np.asarray(v[b, keys, g], dtype=np.float64)
            for i in items:
                vis = keys <= c0 + i
                qi = np.asarray(q[b, i, g * g_sz:(g + 1) * g_sz], dtype=np.float64)   # [G, D]
                logits = (qi @ kg[vis].T) * scale                # [G, L']
                mx = logits.max(axis=1, keepdims=True)
                e = np.exp(logits - mx)
                den = e.sum(axis=1, keepdims=True)
                o[b, i, g * g_sz:(g + 1) * g_sz] = (e / den) @ vg[vis]
                lse[b, i, g * g_sz:(g + 1) * g_sz] = (mx + np.log(den))[:, 0]
    return o, lse


def decode_step_heads(q, k, v, wq_groups, wk_groups, n_init, window, topk, eps, clamp_c, scale=None):
    """The per-head decode path for a batch: the groups' maps, per-group selection,
    attention with per-head lists. q: [B, 1, Hq, D] at position N-1; k, v: [B, N,
    Hkv, D]; wq_groups, wk_groups: [Hkv, G*D, d_g]. Returns dict(q_c, k_c, idx,
    count, s_prime, o, lse)."""
    bsz, _, hq, _ = q.shape
    n, hkv = k.shape[1], k.shape[2]
    c0 = n - 1
    q_c = np.stack([compress_heads(q[b], wq_groups, hq) for b in range(bsz)])
    k_c = np.stack([compress_heads(k[b], wk_groups, hq) for b in range(bsz)])
    idx, count, sp = score_select_heads(q_c, k_c, c0, hkv, n_init, window, topk, eps, clamp_c)
    o, lse = sparse_attn_heads(q, k, v, c0, idx, count, n_init, window, scale)
    return dict(q_c=q_c, k_c=k_c, idx=idx, count=count, s_prime=sp, o=o, lse=lse)


def block_diagonal(w_groups):
    """The groups' maps [n_groups, gin, d_g] stacked into one [n_groups * gin,
    n_groups * d_g] map (zero off the diagonal blocks)."""
    w_groups = np.asarray(w_groups)
    n_groups, gin, dg = w_groups.shape
    out = np.zeros((n_groups * gin, n_groups * dg), dtype=w_groups.dtype)
    for g in range(n_groups):
        out[g * gin:(g + 1) * gin, g * dg:(g + 1) * dg] = w_groups[g]
    return out
