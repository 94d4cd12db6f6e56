"""Algorithmic work of the hot path: bytes and flops that any implementation must
move or compute, used as roofline numerators.

Flops count 2 per multiply-add. Bytes count compulsory reads and writes only
(each input read once, each output written once), never a re-read.

Pins (tests/test_cost.py): the KV-cache example of the attention-optimisation blog
(section 2.2: 1000 tokens x 32 heads x 128 x 2 x 4 bytes, about 32 MB), ESA's
compression ratio (ESA write-up, experiments: 4096 -> 128, about 3.2%) and its
asymptotic per-step compute ratio (ESA write-up, complexity paragraph: about 1.6%).
"""
from __future__ import annotations


def region_lo(c0: int, n_init: int, window: int) -> int:
    return min(c0, max(n_init, c0 - window))


def n_middle(c0: int, n_init: int, window: int) -> int:
    return max(0, region_lo(c0, n_init, window) - n_init)


def attended(c0: int, i: int, n_init: int, window: int, topk: int) -> int:
    """Keys query c0 + i attends: initial + min(k, |mid|) + local up to itself."""
    lo = region_lo(c0, n_init, window)
    return min(n_init, lo) + min(topk, n_middle(c0, n_init, window)) + (c0 + i - lo + 1)


def kv_cache_bytes(tokens: int, heads: int, head_dim: int, bytes_per_value: int) -> int:
    """K and V for `tokens` tokens."""
    return tokens * heads * head_dim * 2 * bytes_per_value


# ----------------------------------------------------------------------------- ESA prefill

def prefill_chunk_attn_flops(c0: int, lq: int, hq: int, d: int, n_init: int, window: int, topk: int) -> int:
    """QK^T and PV of one chunk: 4 * D flops per (query, head, attended key)."""
    lo = region_lo(c0, n_init, window)
    base = min(n_init, lo) + min(topk, n_middle(c0, n_init, window)) + (c0 - lo)
    keys = lq * base + lq * (lq + 1) // 2
    return 4 * d * hq * keys


def prefill_chunk_select_flops(c0: int, lq: int, d_c: int, n_init: int, window: int, topk: int) -> int:
    """Compressed scores S = Q~ K~^T over the middle (computed once), when selection runs."""
    n = n_middle(c0, n_init, window)
    return 2 * lq * n * d_c if n > topk else 0


def compress_flops(rows: int, hq: int, d: int, d_c: int) -> int:
    return 2 * rows * hq * d * d_c


def prefill_flops(n_ctx: int, chunk: int, hq: int, d: int, d_c: int, n_init: int, window: int, topk: int) -> dict:
    att = sel = cmp = 0
    for c0 in range(0, n_ctx, chunk):
        lq = min(chunk, n_ctx - c0)
        att += prefill_chunk_attn_flops(c0, lq, hq, d, n_init, window, topk)
        sel += prefill_chunk_select_flops(c0, lq, d_c, n_init, window, topk)
        cmp += 2 * compress_flops(lq, hq, d, d_c)          # queries and keys
    return dict(attention=att, selection=sel, compression=cmp, total=att + sel + cmp)


def full_causal_attn_flops(n_ctx: int, hq: int, d: int) -> int:
    return 4 * d * hq * n_ctx * (n_ctx + 1) // 2


# ----------------------------------------------------------------------------- ESA decode

def decode_bytes(batch: int, n_ctx: int, hq: int, hkv: int, d: int, d_c: int, n_init: int, window: int,
                 topk: int, kv_bytes: int = 2) -> dict:
    """One decode step (query at n_ctx - 1) for a batch."""
    c0 = n_ctx - 1
    n_mid = n_middle(c0, n_init, window)
    n_att = attended(c0, 0, n_init, window, topk)
    kc = batch * n_mid * d_c * 4                    # compressed middle keys, fp32
    kv = batch * n_att * hkv * d * kv_bytes * 2     # gathered K and V rows
    weights = 2 * hq * d * d_c * 4                  # W_q and W_k
    io = batch * (hq * d * kv_bytes * 2 + hkv * d * kv_bytes + d_c * 4 * 2)   # q, o, new key, q~, k~
    return dict(compressed_keys=kc, kv_rows=kv, weights=weights, io=io, total=kc + kv + weights + io,
                n_mid=n_mid, attended=n_att)


def decode_varlen_bytes(lengths, hq: int, hkv: int, d: int, d_c: int, n_init: int, window: int, topk: int,
                        kv_bytes: int = 2) -> dict:
    """One decode step of a batch whose sequence b holds lengths[b] tokens (its query at
    lengths[b] - 1): the per-sequence bytes summed, the weights read once."""
    parts = [decode_bytes(1, int(n), hq, hkv, d, d_c, n_init, window, topk, kv_bytes) for n in lengths]
    kc = sum(x["compressed_keys"] for x in parts)
    kv = sum(x["kv_rows"] for x in parts)
    io = sum(x["io"] for x in parts)
    weights = parts[0]["weights"]
    return dict(compressed_keys=kc, kv_rows=kv, weights=weights, io=io, total=kc + kv + weights + io)


def full_decode_bytes(batch: int, n_ctx: int, hkv: int, d: int, kv_bytes: int = 2) -> int:
    return batch * n_ctx * hkv * d * kv_bytes * 2


def esa_step_compute_ratio(n_ctx: int, hq: int, d: int, d_c: int, n_init: int, window: int, topk: int) -> float:
    """Multiply-adds of one ESA decode step (scores over the middle + attention over the
    kept keys) over those of full attention, per query: tends to d' / (2 * Hq * D)."""
    c0 = n_ctx - 1
    esa = n_middle(c0, n_init, window) * d_c + attended(c0, 0, n_init, window, topk) * 2 * hq * d
    full = n_ctx * 2 * hq * d
    return esa / full


# ----------------------------------------------------------------------------- MoBA

def moba_flops(seq: int, heads: int, d: int, block: int, topk: int) -> dict:
    """Block attention (past blocks kept + causal current block) and the gate."""
    nb = (seq + block - 1) // block
    keys = 0
    gate = 0
    for c in range(nb):
        n_q = min(seq, (c + 1) * block) - c * block
        keys += n_q * min(topk, c) * block          # kept past blocks are full blocks
        keys += n_q * (n_q + 1) // 2                # causal current block
        gate += n_q * c * d * 2                     # <q, mean> against every past block
    att = 4 * d * heads * keys
    return dict(attention=att, gate=gate * heads, total=att + gate * heads)


def moba_decode_bytes(batch: int, n_ctx: int, heads: int, d: int, block: int, topk: int,
                      kv_bytes: int = 2) -> dict:
    """Compulsory HBM bytes of one MoBA decode step (query at n_ctx - 1): the past
    blocks' means (fp32, read by the gate) and the K and V rows of the kept blocks and
    of the current block up to the query, for every (sequence, head)."""
    cur = (n_ctx - 1) // block
    means = batch * heads * cur * d * 4
    keys = min(topk, cur) * block + (n_ctx - cur * block)
    rows = batch * heads * keys * d * kv_bytes * 2
    return dict(block_means=means, kv_rows=rows, total=means + rows)


# ----------------------------------------------------------------------------- CCA-style attention

def cca_keys(i: int, g: int, w: int) -> int:
    """Keys query i attends: the core tokens of the groups that end before its window
    [max(0, g * (i // g) - w), i], then the window's tokens."""
    lo = max(0, g * (i // g) - w)
    return lo // g + (i - lo + 1)


def cca_flops(seq: int, hq: int, d: int, g: int, w: int) -> dict:
    """Causal prefill of one layer: pooling (per complete group and query head: the
    last query's g scores and the weighted sums of g keys and g values) and the fused
    attention (4 * D flops per (query, head, attended key))."""
    keys = sum(cca_keys(i, g, w) for i in range(seq))
    att = 4 * d * hq * keys
    pool = (seq // g) * hq * g * 6 * d
    return dict(attention=att, pooling=pool, total=att + pool)


# ----------------------------------------------------------------------------- offline fit

def fit_flops(n_q: int, n_k: int, hq: int, hkv: int, d: int, d_c: int) -> dict:
    """The least-squares fit of the two maps: the Gram matrices of the calibration
    queries (n_q x Hq*D) and keys (n_k x Hkv*D), their Cholesky factorisations, the
    coupled matrix Rq E Rk^T and its leading d' singular triples (counted as one dense
    SVD of that matrix), and the two triangular solves."""
    dq, dk = hq * d, hkv * d
    gram = 2 * n_q * dq * dq + 2 * n_k * dk * dk
    chol = (dq ** 3 + dk ** 3) // 3
    couple = 2 * dq * dk * dk
    svd = 4 * dq * dk * dk + 8 * dk ** 3
    solve = dq * dq * d_c + dk * dk * d_c
    return dict(gram=gram, cholesky=chol, couple=couple, svd=svd, solve=solve,
                total=gram + chol + couple + svd + solve)
