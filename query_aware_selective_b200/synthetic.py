"""Seeded synthetic inputs for query-aware selective attention.

This module only draws random tensors and fixes the workload shapes. It is
imported by the tests, the benchmark and the smoke check, and it is the one
module that both the CUDA path and the CPU oracle receive their inputs from.
It computes none of the method's steps: no compression of stored tensors, no
scoring, no selection and no attention. The single piece of linear algebra in
here aims the planted needle keys (see ``plant_needles``), which is part of how
the input is built, not something any output is checked against.

Shapes follow the attention layers the ESA write-up evaluates on
(Llama-3-8B-Instruct / Mistral-7B-Instruct-v0.2: 32 query heads, 8 KV heads,
head dim 128, hidden 4096; "Efficient Selective Attention" article, experiment
section) and the MoBA article's 64-block setting (MoBA article, "experiments",
the fixed-sparsity scaling figure). The benchmarks those pages use (LongBench,
InfiniteBench, NeedleBench) are not available; these tensors stand in for them.

Recipe, for every workload: one ``torch.Generator`` seeded with the workload's
seed draws, in this order, Q, K, V (standard normal, in the workload dtype),
then W_q and W_k (normal with variance 1/in_dim, fp32), then the needle
positions. Needle keys overwrite K at those positions.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class EsaWorkload:
    """Shape and parameters of one ESA workload (decode or chunked prefill)."""

    name: str
    batch: int
    hq: int
    hkv: int
    head_dim: int
    n_ctx: int          # tokens in the KV cache when the step runs
    chunk: int          # prefill chunk length; 1 for decode
    d_c: int            # compressed dimension d'
    n_init: int
    window: int
    topk: int
    eps: int
    clamp_c: float      # +inf disables the clamp
    n_needles: int
    dtype: str          # "f32" or "bf16"
    seed: int
    mode: str           # "decode" or "prefill"

    @property
    def hidden(self) -> int:
        return self.hq * self.head_dim

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


@dataclasses.dataclass(frozen=True)
class MobaWorkload:
    """Shape and parameters of one MoBA causal prefill workload."""

    name: str
    batch: int
    heads: int
    head_dim: int
    seq: int
    block: int
    topk: int           # past blocks selected per (query, head); the current block is extra
    dtype: str
    seed: int

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


def default_clamp(d_c: int) -> float:
    """Default clamp bound C of the score correction: 4 * sqrt(d')."""
    return 4.0 * math.sqrt(d_c)


TINY_DECODE = EsaWorkload("esa_tiny_decode_n2048_f32", 1, 4, 4, 64, 2048, 1, 16,
                          16, 256, 128, 2, default_clamp(16), 3, "f32", 0, "decode")
PREFILL_32K = EsaWorkload("esa_prefill_llama3_8b_ctx32768_chunk512", 1, 32, 8, 128, 32768, 512,
                          128, 128, 4096, 2048, 2, default_clamp(128), 0, "bf16", 1, "prefill")
DECODE_128K = EsaWorkload("esa_decode_llama3_8b_b16_ctx131072", 16, 32, 8, 128, 131072, 1,
                          128, 128, 4096, 2048, 2, default_clamp(128), 8, "bf16", 2, "decode")
MOBA_64K = MobaWorkload("moba_prefill_h32_seq65536_block1024_top3", 1, 32, 128, 65536, 1024, 3,
                        "bf16", 3)
DECODE_1M = EsaWorkload("esa_decode_mistral_7b_b4_ctx1048576", 4, 32, 8, 128, 1048576, 1,
                        128, 128, 4096, 2048, 2, default_clamp(128), 16, "bf16", 4, "decode")

# MoBA decode (a next row past the five configurations): batch 16 of the MoBA layer,
# one query at position 65535 of a 65536-token cache, top-3 past blocks + current
MOBA_DECODE_64K = MobaWorkload("moba_decode_h32_b16_ctx65536_block1024_top3", 16, 32, 128, 65536, 1024, 3,
                               "bf16", 5)

WORKLOADS = {w.name: w for w in (TINY_DECODE, PREFILL_32K, DECODE_128K, MOBA_64K, DECODE_1M, MOBA_DECODE_64K)}


def local_start(c0: int, n_init: int, window: int) -> int:
    """First position of the local part for a chunk starting at c0 (region rule).

    Initial = [0, min(n_init, lo)), middle = [n_init, lo), local = [lo, c1),
    lo = min(c0, max(n_init, c0 - window)). This is a shape rule shared by the
    generator (needle placement) and callers; it involves no data.
    """
    return min(c0, max(n_init, c0 - window))


def _randn(shape, dtype, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(dtype) \
        if dtype == torch.float32 else torch.randn(shape, generator=gen, device=device, dtype=dtype)


def make_esa_inputs(w: EsaWorkload, device="cpu", n_ctx: Optional[int] = None,
                    batch: Optional[int] = None) -> dict:
    """Draw Q, K, V, W_q, W_k (and plant needles) for an ESA workload.

    Decode: q is [B, 1, Hq, D] for position N-1; k, v are [B, N, Hkv, D].
    Prefill: q is [B, N, Hq, D] for every position; k, v as above.
    ``n_ctx``/``batch`` shrink the workload for small tests (same recipe).
    """
    n = n_ctx or w.n_ctx
    b = batch or w.batch
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.torch_dtype
    lq = 1 if w.mode == "decode" else n
    q = _randn((b, lq, w.hq, w.head_dim), dt, gen, device)
    k = _randn((b, n, w.hkv, w.head_dim), dt, gen, device)
    v = _randn((b, n, w.hkv, w.head_dim), dt, gen, device)
    std = 1.0 / math.sqrt(w.hidden)
    wq = torch.randn((w.hidden, w.d_c), generator=gen, device=device, dtype=torch.float32) * std
    wk = torch.randn((w.hidden, w.d_c), generator=gen, device=device, dtype=torch.float32) * std
    out = dict(q=q, k=k, v=v, wq=wq, wk=wk, needles=None)
    if w.n_needles and w.mode == "decode":
        out["needles"] = plant_needles(w, q, k, wq, wk, gen)
    return out


def make_group_maps(w: EsaWorkload, device="cpu") -> tuple:
    """Per-head selection: the groups' one-layer maps for queries and keys, each
    [Hkv, G * D, d' / Hkv] ~ N(0, 1 / (G * D)), from their own generator (seed
    w.seed + 1000) so that the workload's Q, K, V stay those of the merged form.
    Returns (wq_groups, wk_groups), fp32."""
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed + 1000)
    g = w.hq // w.hkv
    gin, dg = g * w.head_dim, w.d_c // w.hkv
    std = 1.0 / math.sqrt(gin)
    wq = torch.randn((w.hkv, gin, dg), generator=gen, device=device, dtype=torch.float32) * std
    wk = torch.randn((w.hkv, gin, dg), generator=gen, device=device, dtype=torch.float32) * std
    return wq, wk


def needle_positions(w: EsaWorkload, n_ctx: int, gen: torch.Generator) -> torch.Tensor:
    """Needle positions per sequence: one per equal segment of the middle,
    at least eps from either edge of the segment (hence >= 2*eps+1 apart)."""
    c0 = n_ctx - 1
    lo = local_start(c0, w.n_init, w.window)
    mid0, mid1 = w.n_init, lo
    seg = (mid1 - mid0) // w.n_needles
    assert seg >= 2 * w.eps + 2, "middle too short for the needles"
    r = torch.randint(0, seg - 2 * w.eps, (w.n_needles,), generator=gen,
                      device=gen.device).cpu()
    base = torch.arange(w.n_needles) * seg + mid0 + w.eps
    return base + r


def plant_needles(w: EsaWorkload, q, k, wq, wk, gen) -> torch.Tensor:
    """Overwrite K at the needle positions with keys aimed at the query.

    A needle key (the same vector for every KV head's slot of its group layout)
    is beta * u / |u| with u the direction in raw key space along which the
    compressed score of the decode query grows fastest: u = d(score)/d(key).
    beta = 3 * sqrt(Hkv * D). Returns the positions, [B, n_needles] int64.
    """
    b, n = k.shape[0], k.shape[1]
    g = w.hq // w.hkv
    pos = torch.empty((b, w.n_needles), dtype=torch.int64)
    beta = 3.0 * math.sqrt(w.hkv * w.head_dim)
    for s in range(b):
        p = needle_positions(w, n, gen)
        pos[s] = p
        qf = q[s, 0].reshape(-1).float()                          # [Hq*D]
        qc = qf @ wq                                              # aim point in compressed space
        grad_expanded = (wk @ qc).reshape(w.hq, w.head_dim)       # d score / d expanded key
        u = grad_expanded.reshape(w.hkv, g, w.head_dim).sum(1)    # fold the GQA copies
        key = (beta * u / u.norm()).to(k.dtype)
        k[s, p.to(k.device)] = key.unsqueeze(0).expand(len(p), -1, -1)
    return pos


@dataclasses.dataclass(frozen=True)
class CcaWorkload:
    """Shape and parameters of one CCA-style causal prefill workload (random inputs;
    the article's group size and window are not on the pages: g = 128, w = 1024)."""

    name: str
    batch: int
    hq: int
    hkv: int
    head_dim: int
    seq: int
    group: int
    window: int
    seed: int


CCA_64K = CcaWorkload("cca_prefill_llama3_8b_seq65536_group128_window1024", 1, 32, 8, 128, 65536, 128, 1024, 6)


def make_cca_inputs(w: CcaWorkload, device="cpu", seq: Optional[int] = None, batch: Optional[int] = None) -> dict:
    """Draw Q [B, S, Hq, D] and K, V [B, S, Hkv, D] ~ N(0, 1), bf16, for a CCA workload."""
    s = seq or w.seq
    b = batch or w.batch
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    q = _randn((b, s, w.hq, w.head_dim), torch.bfloat16, gen, device)
    k = _randn((b, s, w.hkv, w.head_dim), torch.bfloat16, gen, device)
    v = _randn((b, s, w.hkv, w.head_dim), torch.bfloat16, gen, device)
    return dict(q=q, k=k, v=v)


def make_moba_inputs(w: MobaWorkload, device="cpu", seq: Optional[int] = None,
                     heads: Optional[int] = None, batch: Optional[int] = None) -> dict:
    """Draw Q, K, V ([B, S, H, D]) for a MoBA workload."""
    s = seq or w.seq
    h = heads or w.heads
    b = batch or w.batch
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.torch_dtype
    q = _randn((b, s, h, w.head_dim), dt, gen, device)
    k = _randn((b, s, h, w.head_dim), dt, gen, device)
    v = _randn((b, s, h, w.head_dim), dt, gen, device)
    return dict(q=q, k=k, v=v)


def make_moba_decode_inputs(w: MobaWorkload, device="cpu", seq: Optional[int] = None,
                            batch: Optional[int] = None) -> dict:
    """Draw the decode query q [B, 1, H, D] (position seq - 1), then K, V [B, S, H, D],
    standard normal in the workload dtype, from the workload's seed."""
    s = seq or w.seq
    b = batch or w.batch
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.torch_dtype
    q = _randn((b, 1, w.heads, w.head_dim), dt, gen, device)
    k = _randn((b, s, w.heads, w.head_dim), dt, gen, device)
    v = _randn((b, s, w.heads, w.head_dim), dt, gen, device)
    return dict(q=q, k=k, v=v)


def make_calibration(hq: int, hkv: int, d: int, n_tokens: int, rank: int, seed: int, noise: float = 0.1) -> tuple:
    """Calibration queries and keys for the offline fit of the compression maps (they
    stand in for the model's own queries and keys on a calibration text, which are not
    available here). Each token's query is a rank-`rank` latent times fixed loadings
    plus N(0, noise^2) noise, and so is each key, with their own latents and loadings:
    the merged scores then have a dominant low-rank part, as attention scores do.
    Returns (q [n, hq, d], k [n, hkv, d]) float32 on the host."""
    gen = torch.Generator()
    gen.manual_seed(seed)
    a_q = torch.randn((rank, hq * d), generator=gen) / math.sqrt(rank)
    a_k = torch.randn((rank, hkv * d), generator=gen) / math.sqrt(rank)
    z_q = torch.randn((n_tokens, rank), generator=gen)
    z_k = torch.randn((n_tokens, rank), generator=gen)
    q = z_q @ a_q + noise * torch.randn((n_tokens, hq * d), generator=gen)
    k = z_k @ a_k + noise * torch.randn((n_tokens, hkv * d), generator=gen)
    return q.reshape(n_tokens, hq, d), k.reshape(n_tokens, hkv, d)


@dataclasses.dataclass(frozen=True)
class FitWorkload:
    """Offline fit of the compression maps: calibration tokens of one attention layer
    (make_calibration: rank-`rank` latents plus noise), the compressed width d_c and the
    fit's knobs (ridge, power iterations of the range finder)."""

    name: str
    hq: int
    hkv: int
    head_dim: int
    n_tokens: int
    rank: int
    d_c: int
    oversample: int
    noise: float
    ridge: float
    power_iters: int
    seed: int


FIT_64K = FitWorkload("esa_fit_llama3_8b_calib65536_dc128", 32, 8, 128, 65536, 128, 128, 32, 0.1, 0.0, 8, 7)


def make_fit_inputs(w: FitWorkload, device="cpu", n_tokens: Optional[int] = None) -> dict:
    """Calibration queries q [n, hq, d] and keys k [n, hkv, d] in bf16 (make_calibration,
    rounded), and the subspace iteration's Gaussian start omega [hkv * d, d_c +
    oversample] (float64, its own generator, seed + 1)."""
    n = n_tokens or w.n_tokens
    q, k = make_calibration(w.hq, w.hkv, w.head_dim, n, w.rank, w.seed, w.noise)
    gen = torch.Generator()
    gen.manual_seed(w.seed + 1)
    omega = torch.randn((w.hkv * w.head_dim, w.d_c + w.oversample), generator=gen, dtype=torch.float64)
    return dict(q=q.to(torch.bfloat16).to(device), k=k.to(torch.bfloat16).to(device), omega=omega.to(device))


def varlen_lengths(batch: int, n_max: int, n_min: int, seed: int) -> torch.Tensor:
    """Lengths of a variable-length decode batch: sequence 0 holds n_max tokens, the
    others a seeded uniform draw from [n_min, n_max]. Returns int64 [batch] (host)."""
    gen = torch.Generator()
    gen.manual_seed(seed)
    lens = torch.randint(n_min, n_max + 1, (batch,), generator=gen, dtype=torch.int64)
    lens[0] = n_max
    return lens


def random_index_list(batch: int, mid0: int, mid1: int, topk: int, seed: int) -> tuple:
    """A valid selection result drawn at random: per sequence, min(topk, |mid|)
    distinct middle positions, ascending, padded with -1. Used to test the
    attention call on its own. Returns (idx [B, topk] int32, count [B] int32)."""
    gen = torch.Generator()
    gen.manual_seed(seed)
    n = max(0, mid1 - mid0)
    cnt = min(topk, n)
    idx = torch.full((batch, topk), -1, dtype=torch.int32)
    for b in range(batch):
        sel = torch.randperm(n, generator=gen)[:cnt].sort().values + mid0
        idx[b, :cnt] = sel.to(torch.int32)
    return idx, torch.full((batch,), cnt, dtype=torch.int32)


def random_block_lists(batch: int, seq: int, heads: int, block: int, topk: int,
                       seed: int) -> torch.Tensor:
    """Valid MoBA block lists drawn at random: for a query in block c, min(topk, c)
    distinct past blocks, ascending, then c, then -1 padding.
    Returns [B, S, H, topk+1] int16."""
    gen = torch.Generator()
    gen.manual_seed(seed)
    out = torch.full((batch, seq, heads, topk + 1), -1, dtype=torch.int16)
    cur = torch.arange(seq) // block
    keys = torch.rand((batch, seq, heads, max(1, (seq + block - 1) // block)), generator=gen)
    nb = keys.shape[-1]
    blk = torch.arange(nb)
    # past blocks only: push current and future blocks to the end
    keys = keys.masked_fill(blk.view(1, 1, 1, nb) >= cur.view(1, seq, 1, 1), 2.0)
    order = keys.argsort(dim=-1)[..., :topk]
    cnt = torch.clamp(cur, max=topk)
    valid = torch.arange(topk).view(1, 1, 1, topk) < cnt.view(1, seq, 1, 1)
    order = torch.where(valid, order, torch.full_like(order, 1 << 14))
    order = order.sort(dim=-1).values
    order = torch.where(order == (1 << 14), torch.full_like(order, -1), order)
    out[..., :topk] = order.to(torch.int16)
    # the current block goes right after the last valid past block
    for c in range(topk + 1):
        mask = cnt == c
        out[:, mask, :, c] = cur[mask].to(torch.int16).view(1, -1, 1)
    return out
