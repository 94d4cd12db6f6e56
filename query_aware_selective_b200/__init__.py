"""Query-aware top-k selective attention (ESA and MoBA forms) on B200 (sm_100a).

The compute path is libesa.so (C ABI in include/esa.h, CUDA kernels in csrc/);
this package only marshals torch tensors into it. ``synthetic`` draws the seeded
benchmark inputs; ``cost`` holds the algorithmic byte and flop counts used for
rooflines.
"""
from ._abi import (EsaError, EsaParams, cca_attn, compress, compress_pack, compress_pack_size, compress_packed,
                   compress_packed_varlen, device_status, fit_maps, gram, load, moba_block_attn, moba_block_gate,
                   moba_block_gate_attn, moba_block_means, moba_decode_attn, params, score_select,
                   score_select_heads, score_select_varlen, sparse_attn, sparse_attn_heads, sparse_attn_varlen)

__all__ = ["EsaError", "EsaParams", "cca_attn", "compress", "compress_pack", "compress_pack_size", "compress_packed",
           "compress_packed_varlen", "device_status", "fit_maps", "gram", "load", "moba_block_attn",
           "moba_block_gate", "moba_block_gate_attn", "moba_block_means", "moba_decode_attn", "params",
           "score_select", "score_select_heads", "score_select_varlen", "sparse_attn", "sparse_attn_heads",
           "sparse_attn_varlen"]
