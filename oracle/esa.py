"""ESA oracle: plain float64 restatement of Efficient Selective Attention.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source: the ESA write-up ("Efficient Selective Attention", Huawei Noah's Ark;
arXiv 2502.14477), paragraphs "core steps", "implementation", "score
correction", "neighbour influence", "final attention" and "experiments". The
extracted text lost every ESA formula; each step below states the reading it
takes where the words alone leave a choice.

Notation: B sequences, Hq query heads, Hkv KV heads, G = Hq / Hkv, D head dim,
d' compressed dim. A chunk is the query positions [c0, c1); the caches hold
tokens [0, c1). Decode is a chunk of one (c0 = N - 1).

Functions, in the pages' order:
  compress        - one-layer linear map of the merged-head vector (a1, a2)
  regions         - initial / middle / local split of the sequence
  importance      - per-query dot product, per-query max correction with clamp,
                    sum over the chunk's queries (a3, a4, a5)
  neighbour_max   - neighbour influence as a max over +-eps (a6)
  topk_ascending  - fixed-count top-k with (value desc, index asc) order (a7)
  score_select    - a3..a7 for a batch, as the C-ABI call does it
  sparse_attn     - exact attention over initial + selected + local (a8)
"""
from __future__ import annotations

import math

import numpy as np


def compress(x, w, n_heads_out):
    """One-layer linear map to the compressed space (a1, a2).

    ESA write-up, "implementation": query and key are each passed through a
    one-layer MLP that shrinks the 4096-wide vector to 128 (about 3.2%).
    Reading: a linear map with no bias and no activation. The input is the
    concatenation over the Hq query heads; for keys under GQA each query head h
    takes KV head h // G, so the key vector is expanded to Hq heads first
    (the literal expansion is done here; no weight folding).

    x: [rows, n_heads_in, D]; w: [n_heads_out * D, d']. Returns [rows, d'].
    """
    w = np.asarray(w, dtype=np.float64)
    rows, n_in, d = x.shape
    assert n_heads_out % n_in == 0
    g = n_heads_out // n_in
    out = np.empty((rows, w.shape[1]), dtype=np.float64)
    step = 4096                                              # row blocks bound the host memory used
    for r0 in range(0, rows, step):
        xb = np.asarray(x[r0:r0 + step], dtype=np.float64)
        xe = np.repeat(xb, g, axis=1)                        # [r, Hq, D]: head h <- x[:, h // g]
        out[r0:r0 + step] = xe.reshape(xe.shape[0], n_heads_out * d) @ w
    return out


def regions(c0, c1, n_init, window):
    """Split [0, c1) into initial, middle and local parts for the chunk [c0, c1).

    ESA write-up, "implementation": the sequence is cut into four parts -
    initial tokens, middle tokens (the selection candidates), local tokens, and
    the current chunk/token. Reading (positions are not on the page): the local
    part is the `window` cached tokens right before the chunk plus the chunk
    itself (causal), so the same rule covers prefill and decode:
      lo      = min(c0, max(n_init, c0 - window))
      initial = [0, min(n_init, lo))
      middle  = [n_init, lo)            (empty when lo <= n_init)
      local   = [lo, c1)                (query at p sees local keys <= p)
    Returns ((i0, i1), (m0, m1), (l0, l1)).
    """
    lo = min(c0, max(n_init, c0 - window))
    init_end = min(n_init, lo)
    mid = (n_init, max(n_init, lo))
    return (0, init_end), mid, (lo, c1)


def importance(q_c, k_c_mid, clamp_c):
    """Per-token importance summed over the chunk's queries (a3, a4, a5).

    ESA write-up, "implementation": the importance of one middle token against
    one query is the q.k dot product with all heads merged (here the compressed
    q~ . k~), and a middle token's importance counts every query of the current
    chunk (a single query in decode).
    ESA write-up, "score correction" (formula stripped): scores are corrected so
    that relative sizes are kept and no single score dominates. Reading: each
    query's scores are shifted by that query's maximum over the middle tokens
    and clamped from below at -C:
        S_ij   = q~_i . k~_j
        m_i    = max_j S_ij
        Shat_ij = max(S_ij - m_i, -C)
        s_j    = sum_i Shat_ij
    C = +inf turns the clamp off.

    q_c: [Lq, d']; k_c_mid: [n_mid, d']. Returns s: [n_mid] float64.
    """
    q_c = np.asarray(q_c, dtype=np.float64)
    k_c_mid = np.asarray(k_c_mid, dtype=np.float64)
    s_full = q_c @ k_c_mid.T                       # [Lq, n_mid]
    m = s_full.max(axis=1, keepdims=True)          # per-query maximum
    corrected = s_full - m
    if math.isfinite(clamp_c):
        corrected = np.maximum(corrected, -float(clamp_c))
    return corrected.sum(axis=0)


def neighbour_max(s, eps):
    """Neighbour influence (a6).

    ESA write-up, "neighbour influence" (formula stripped): a middle token's
    score is not only its own but is lifted by the tokens around it, so that a
    selected token brings its surroundings. Reading: a max over the window of
    radius eps, cut at the edges of the middle (no padding values enter):
        s'_j = max_{m in middle, |m - j| <= eps} s_m
    """
    s = np.asarray(s, dtype=np.float64)
    n = s.shape[0]
    out = s.copy()
    for off in range(1, eps + 1):
        if off >= n:
            break
        out[:-off] = np.maximum(out[:-off], s[off:])    # neighbour on the right
        out[off:] = np.maximum(out[off:], s[:-off])     # neighbour on the left
    return out


def topk_ascending(values, k):
    """Fixed-count top-k (a7).

    ESA write-up, "core steps": the top-k tokens by importance are kept, and the
    key length stays fixed. Reading of the unstated details: order by value
    descending, then by index ascending; keep min(k, n); return the kept indices
    in ascending order.
    """
    values = np.asarray(values, dtype=np.float64)
    n = values.shape[0]
    keep = min(k, n)
    order = np.lexsort((np.arange(n), -values))    # primary: value desc; ties: index asc
    return np.sort(order[:keep])


def score_select(q_c, k_c, c0, n_init, window, topk, eps, clamp_c):
    """Selection for one chunk of every sequence in a batch (a3..a7).

    q_c: [B, Lq, d'] compressed queries of the chunk at positions [c0, c0+Lq).
    k_c: [B, >= c0+Lq, d'] compressed key cache.
    Returns (idx [B, topk] int64 of absolute positions, ascending, -1 padded;
             count [B]; s_prime: list of [n_mid] arrays, one per sequence).
    """
    q_c = np.asarray(q_c, dtype=np.float64)
    bsz, lq, _ = q_c.shape
    _, (m0, m1), _ = regions(c0, c0 + lq, n_init, window)
    n_mid = m1 - m0
    idx = np.full((bsz, topk), -1, dtype=np.int64)
    count = np.zeros(bsz, dtype=np.int64)
    s_primes = []
    for b in range(bsz):
        if n_mid == 0:
            s_primes.append(np.zeros(0))
            continue
        s = importance(q_c[b], np.asarray(k_c[b, m0:m1], dtype=np.float64), clamp_c)
        sp = neighbour_max(s, eps)
        chosen = topk_ascending(sp, topk)
        idx[b, :len(chosen)] = chosen + m0
        count[b] = len(chosen)
        s_primes.append(sp)
    return idx, count, s_primes


def attended_keys(c0, lq, n_init, window, idx_row, count):
    """Key positions one chunk attends, before the causal cut, ascending:
    initial, then the selected middle tokens, then local [lo, c1)."""
    (i0, i1), _, (l0, l1) = regions(c0, c0 + lq, n_init, window)
    sel = np.asarray(idx_row[:count], dtype=np.int64)
    return np.concatenate([np.arange(i0, i1), sel, np.arange(l0, l1)])


def sparse_attn(q, k, v, c0, idx, count, n_init, window, scale=None, rows=None):
    """Exact attention over initial + selected + local tokens (a8).

    ESA write-up, "implementation" and "final attention" (formula stripped): the
    initial tokens and the selected middle tokens form the global part, the local
    tokens the window part, and the two attentions are fused into one output,
    computed with the full (uncompressed) queries, keys and values. Reading: one
    softmax over the disjoint union of the parts (the same as merging the two
    partial softmaxes by their log-sum-exp), scale 1/sqrt(D), causal inside the
    local part, standard GQA (query head h reads KV head h // G).

    q: [B, Lq, Hq, D]; k, v: [B, >= c0+Lq, Hkv, D]; idx [B, >= count], count [B].
    rows: optional list of (b, i) pairs to compute (others stay NaN).
    Returns (o [B, Lq, Hq, D], lse [B, Lq, Hq]) in float64; lse is the natural
    log of the softmax denominator of the scaled logits.
    """
    bsz, lq, hq, d = q.shape
    hkv = k.shape[2]
    g = hq // hkv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    o = np.full((bsz, lq, hq, d), np.nan)
    lse = np.full((bsz, lq, hq), np.nan)
    if rows is None:
        rows = [(b, i) for b in range(bsz) for i in range(lq)]
    head_map = np.arange(hq) // g
    by_seq = {}
    for b, i in rows:
        by_seq.setdefault(b, []).append(i)
    for b, items in by_seq.items():
        keys = attended_keys(c0, lq, n_init, window, idx[b], int(count[b]))
        kk = np.asarray(k[b, keys], dtype=np.float64)     # [L, Hkv, D]
        vv = np.asarray(v[b, keys], dtype=np.float64)
        kh = np.ascontiguousarray(kk[:, head_map, :].transpose(1, 0, 2))   # [Hq, L, D]
        vh = np.ascontiguousarray(vv[:, head_map, :].transpose(1, 0, 2))
        for i in items:
            p = c0 + i
            vis = keys <= p
            qi = np.asarray(q[b, i], dtype=np.float64)    # [Hq, D]
            logits = np.matmul(kh[:, vis, :], qi[:, :, None])[:, :, 0] * scale   # [Hq, L']
            mx = logits.max(axis=1, keepdims=True)
            e = np.exp(logits - mx)
            den = e.sum(axis=1, keepdims=True)
            o[b, i] = np.matmul((e / den)[:, None, :], vh[:, vis, :])[:, 0, :]
            lse[b, i] = (mx + np.log(den))[:, 0]
    return o, lse


def decode_step(q, k, v, wq, wk, n_init, window, topk, eps, clamp_c, scale=None):
    """The whole decode path for a batch: compress, select, attend (a1..a8).

    q: [B, 1, Hq, D] at position N-1; k, v: [B, N, Hkv, D]; wq, wk: [Hq*D, d'].
    Returns dict(q_c, k_c, idx, count, s_prime, o, lse).
    """
    bsz, _, hq, d = q.shape
    n = k.shape[1]
    c0 = n - 1
    q_c = np.stack([compress(q[b], wq, hq) for b in range(bsz)])          # [B, 1, d']
    k_c = np.stack([compress(k[b], wk, hq) for b in range(bsz)])          # [B, N, d']
    idx, count, sp = score_select(q_c, k_c, c0, n_init, window, topk, eps, clamp_c)
    o, lse = sparse_attn(q, k, v, c0, idx, count, n_init, window, scale)
    return dict(q_c=q_c, k_c=k_c, idx=idx, count=count, s_prime=sp, o=o, lse=lse)


def prefill_chunk(q_chunk, k, v, k_c, wq, c0, n_init, window, topk, eps, clamp_c,
                  scale=None, rows=None):
    """One chunk of chunked prefill: compress the chunk's queries, select against
    the compressed key cache, attend. k_c must already hold compressed keys for
    [0, c0 + Lq). Returns dict(q_c, idx, count, s_prime, o, lse)."""
    bsz, lq, hq, _ = q_chunk.shape
    q_c = np.stack([compress(q_chunk[b], wq, hq) for b in range(bsz)])
    idx, count, sp = score_select(q_c, k_c, c0, n_init, window, topk, eps, clamp_c)
    o, lse = sparse_attn(q_chunk, k, v, c0, idx, count, n_init, window, scale, rows)
    return dict(q_c=q_c, idx=idx, count=count, s_prime=sp, o=o, lse=lse)
