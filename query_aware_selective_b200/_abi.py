"""Thin ctypes binding of libesa (include/esa.h).

Argument marshalling only: every step of the path runs in libesa's CUDA kernels.
Outputs and workspaces are torch tensors (the caller's device memory); a function
allocates them when the caller passes none. There is no CPU fallback: without the
built library, or without a CUDA device, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libesa.so")

ESA_OK, ESA_ERR_INVALID_ARG, ESA_ERR_UNSUPPORTED, ESA_ERR_CUDA, ESA_ERR_TIMEOUT, ESA_ERR_WORKSPACE = range(6)
ESA_F32, ESA_BF16 = 0, 1

# Every exported function of include/esa.h: name -> (restype, argtypes)
_vp, _i32, _i64, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


class EsaParams(ctypes.Structure):
    """esa_params_t: n_init, window, topk, eps, clamp_c (+inf = no clamp)."""

    _fields_ = [("n_init", ctypes.c_int32), ("window", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("eps", ctypes.c_int32), ("clamp_c", ctypes.c_float)]


SIGNATURES = {
    "esa_compress": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _i32, _i32, _i32, _vp, _i32, _vp, _i64, _vp]),
    "esa_compress_pack_size": (_sz, [_i32, _i32, _i32]),
    "esa_compress_pack": (ctypes.c_int, [_vp, _i32, _i32, _i32, _i32, _vp, _sz, _vp]),
    "esa_compress_packed": (ctypes.c_int, [_vp, _i64, _i64, _i32, _i32, _vp, _i32, _vp, _i64, _vp]),
    "esa_score_select": (ctypes.c_int, [_vp, _vp, _i32, _i32, _i64, _i64, _i32, EsaParams, _vp, _vp, _vp,
                                        _vp, _sz, _vp]),
    "esa_score_select_workspace_size": (_sz, [_i32, _i32, _i64, _i64, _i32, EsaParams]),
    "esa_sparse_attn": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i32, _i64, _i64, _i32, _i32, _i32,
                                       _vp, _vp, EsaParams, _f32, _vp, _vp, _vp, _sz, _vp]),
    "esa_sparse_attn_workspace_size": (_sz, [_i32, _i32, _i64, _i32, _i32, _i32, ctypes.c_int, EsaParams]),
    "moba_block_gate": (ctypes.c_int, [_vp, _vp, ctypes.c_int, _i32, _i64, _i32, _i32, _i32, _i32, _vp, _vp,
                                       _sz, _vp]),
    "moba_block_attn": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i64, _i32, _i32, _i32, _i32, _vp,
                                       _f32, _vp, _vp, _vp, _sz, _vp]),
    "moba_block_gate_attn": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i64, _i32, _i32, _i32, _i32,
                                            _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moba_workspace_size": (_sz, [_i32, _i32, _i64, _i32, _i32, _i32, _i32]),
    "esa_last_error": (ctypes.c_char_p, []),
    "esa_device_status": (ctypes.c_int, [_vp]),
    "esa_version": (ctypes.c_char_p, []),
    "esa_launch_count": (ctypes.c_uint64, []),
    "esa_score_select_noalloc": (ctypes.c_int, [_vp, _vp, _i32, _i32, _i64, _i64, _i32, EsaParams, _vp, _vp, _vp,
                                                _vp]),
    "esa_score_select_noalloc_capacity": (_sz, []),
    "moba_block_means": (ctypes.c_int, [_vp, ctypes.c_int, _i32, _i64, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "moba_decode_attn": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i64, _i64, _i32, _i32, _i32, _i32, _vp,
                                        _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moba_decode_workspace_size": (_sz, [_i32, _i64, _i64, _i32, _i32, _i32, _i32]),
    "esa_score_select_heads": (ctypes.c_int, [_vp, _vp, _i32, _i32, _i64, _i64, _i32, _i32, EsaParams, _vp, _vp,
                                              _vp, _vp, _sz, _vp]),
    "esa_score_select_heads_workspace_size": (_sz, [_i32, _i32, _i64, _i64, _i32, _i32, EsaParams]),
    "esa_sparse_attn_heads": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i32, _i64, _i64, _i32, _i32,
                                             _i32, _vp, _vp, EsaParams, _f32, _vp, _vp, _vp, _sz, _vp]),
    "esa_sparse_attn_heads_workspace_size": (_sz, [_i32, _i32, _i64, _i32, _i32, _i32, ctypes.c_int, EsaParams]),
    "esa_wait_selftest": (ctypes.c_int, [ctypes.c_uint64, _vp]),
    "cca_attn": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i64, _i32, _i32, _i32, _i32, _i32, _f32, _vp,
                                _vp, _vp, _sz, _vp]),
    "cca_workspace_size": (_sz, [_i32, _i64, _i32, _i32, _i32]),
    "esa_gram": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i32, _vp, _vp, _sz, _vp]),
    "esa_gram_workspace_size": (_sz, [_i64, _i32]),
    "esa_fit_maps": (ctypes.c_int, [_vp, _i64, _vp, _i64, ctypes.c_int, _i32, _i32, _i32, _i32, _i32,
                                    ctypes.c_double, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "esa_fit_workspace_size": (_sz, [_i64, _i64, _i32, _i32, _i32, _i32, _i32]),
    "esa_compress_packed_varlen": (ctypes.c_int, [_vp, _i32, _i64, _i32, _i32, _vp, _i32, _vp, _i64, _vp, _vp]),
    "esa_score_select_varlen": (ctypes.c_int, [_vp, _vp, _i32, _i64, _vp, _i32, _i32, EsaParams, _vp, _vp, _vp,
                                               _vp, _sz, _vp]),
    "esa_score_select_varlen_workspace_size": (_sz, [_i32, _i64, _i32, _i32, EsaParams]),
    "esa_sparse_attn_varlen": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _i32, _i64, _vp, _i32, _i32, _i32, _vp,
                                              _vp, _i32, EsaParams, _f32, _vp, _vp, _vp, _sz, _vp]),
    "esa_sparse_attn_varlen_workspace_size": (_sz, [_i32, _i64, _i32, _i32, _i32, ctypes.c_int, _i32, EsaParams]),
}

_lib = None


class EsaError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: status {status}: {message}")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libesa and declare every signature. Raises if the library is missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libesa is not built ({path} missing); run __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(status: int, where: str):
    if status != ESA_OK:
        raise EsaError(status, where, load().esa_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return ESA_F32
    if t.dtype == torch.bfloat16:
        return ESA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("libesa takes CUDA tensors (no CPU path)")
            if not t.is_contiguous():
                raise ValueError("libesa takes contiguous tensors")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _workspace(nbytes: int, device, ws: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return ws
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws
    return torch.empty(nbytes + 256, dtype=torch.uint8, device=device)


def _ws_ptr(ws: Optional[torch.Tensor]) -> tuple:
    if ws is None:
        return None, 0
    p = ws.data_ptr()
    pad = (-p) % 256
    return p + pad, ws.numel() * ws.element_size() - pad


def params(n_init: int, window: int, topk: int, eps: int, clamp_c: float = math.inf) -> EsaParams:
    return EsaParams(n_init, window, topk, eps, clamp_c)


def compress(x: torch.Tensor, w: torch.Tensor, n_heads_out: int, out: Optional[torch.Tensor] = None,
             out_row_stride: Optional[int] = None) -> torch.Tensor:
    """esa_compress. x: [rows, Hin, D] (f32 or bf16; each row contiguous, rows may be
    strided); w: [Hout*D, d'] f32 -> [rows, d'] f32. With `out` given, rows are written
    at out + r * out_row_stride (default d')."""
    if not x.is_cuda or not w.is_cuda or not w.is_contiguous():
        raise ValueError("libesa takes CUDA tensors (no CPU path); w must be contiguous")
    rows, hin, d = x.shape
    if x.stride(2) != 1 or x.stride(1) != d:
        raise ValueError("each row of x must be contiguous [Hin, D]")
    dout = w.shape[1]
    if out is None:
        out = torch.empty((rows, dout), dtype=torch.float32, device=x.device)
        stride = dout
    else:
        stride = out_row_stride or dout
    _check(load().esa_compress(_ptr(x), _dtype_code(x), rows, x.stride(0) if rows > 1 else hin * d, hin,
                               n_heads_out, d, _ptr(w), dout, _ptr(out), stride, _stream()), "esa_compress")
    return out


def compress_pack_size(n_heads_in: int, head_dim: int, d_out: int) -> int:
    """esa_compress_pack_size: bytes of the packed weight, 0 if the packed path does
    not take the shape."""
    return load().esa_compress_pack_size(n_heads_in, head_dim, d_out)


def compress_pack(w: torch.Tensor, n_heads_in: int, n_heads_out: int, head_dim: int,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """esa_compress_pack: w [Hout*D, d'] f32 -> packed weight (uint8 device tensor)."""
    if not w.is_cuda or not w.is_contiguous():
        raise ValueError("libesa takes contiguous CUDA tensors (no CPU path)")
    dout = w.shape[1]
    n = compress_pack_size(n_heads_in, head_dim, dout)
    if n == 0:
        raise EsaError(ESA_ERR_UNSUPPORTED, "esa_compress_pack", "shape not supported by the packed path")
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=w.device)
    _check(load().esa_compress_pack(_ptr(w), n_heads_in, n_heads_out, head_dim, dout, _ptr(out),
                                    out.numel() * out.element_size(), _stream()), "esa_compress_pack")
    return out


def compress_packed(x: torch.Tensor, packed: torch.Tensor, d_out: int = 128, out: Optional[torch.Tensor] = None,
                    out_row_stride: Optional[int] = None) -> torch.Tensor:
    """esa_compress_packed. x: [rows, Hin, D] bf16 (each row contiguous, rows may be
    strided); packed from compress_pack -> [rows, d_out] f32 (or written into `out`
    with row stride out_row_stride)."""
    if not x.is_cuda or not packed.is_cuda:
        raise ValueError("libesa takes CUDA tensors (no CPU path)")
    rows, hin, d = x.shape
    if x.stride(2) != 1 or x.stride(1) != d:
        raise ValueError("each row of x must be contiguous [Hin, D]")
    if out is None:
        out = torch.empty((rows, d_out), dtype=torch.float32, device=x.device)
        stride = d_out
    else:
        stride = out_row_stride or d_out
    _check(load().esa_compress_packed(_ptr(x), rows, x.stride(0) if rows > 1 else hin * d, hin, d, _ptr(packed),
                                      d_out, _ptr(out), stride, _stream()), "esa_compress_packed")
    return out


def score_select_workspace_size(batch, lq, n_cap, c0, d_c, p: EsaParams) -> int:
    return load().esa_score_select_workspace_size(batch, lq, n_cap, c0, d_c, p)


def score_select(q_c: torch.Tensor, k_c: torch.Tensor, c0: int, p: EsaParams, want_scores: bool = False,
                 idx: Optional[torch.Tensor] = None, count: Optional[torch.Tensor] = None,
                 scores: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """esa_score_select. q_c [B, Lq, d'] f32, k_c [B, n_cap, d'] f32.
    Returns (idx [B, topk] int32, count [B] int32, s' [B, n_mid] f32 or None)."""
    _dev(q_c, k_c)
    b, lq, dc = q_c.shape
    n_cap = k_c.shape[1]
    dev = q_c.device
    if idx is None:
        idx = torch.empty((b, p.topk), dtype=torch.int32, device=dev)
    if count is None:
        count = torch.empty((b,), dtype=torch.int32, device=dev)
    if want_scores and scores is None:
        lo = min(c0, max(p.n_init, c0 - p.window))
        scores = torch.empty((b, max(0, lo - p.n_init)), dtype=torch.float32, device=dev)
    ws = _workspace(score_select_workspace_size(b, lq, n_cap, c0, dc, p), dev, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().esa_score_select(_ptr(q_c), _ptr(k_c), b, lq, n_cap, c0, dc, p, _ptr(idx), _ptr(count),
                                   _ptr(scores) if want_scores else None, wp, wn, _stream()), "esa_score_select")
    return idx, count, (scores if want_scores else None)


def score_select_noalloc(q_c: torch.Tensor, k_c: torch.Tensor, c0: int, p: EsaParams, want_scores: bool = False,
                         idx: Optional[torch.Tensor] = None, count: Optional[torch.Tensor] = None,
                         scores: Optional[torch.Tensor] = None):
    """esa_score_select_noalloc: the same selection, with the library's fixed scratch
    instead of a workspace (for callers that cannot allocate device memory)."""
    _dev(q_c, k_c)
    b, lq, dc = q_c.shape
    dev = q_c.device
    if idx is None:
        idx = torch.empty((b, p.topk), dtype=torch.int32, device=dev)
    if count is None:
        count = torch.empty((b,), dtype=torch.int32, device=dev)
    if want_scores and scores is None:
        lo = min(c0, max(p.n_init, c0 - p.window))
        scores = torch.empty((b, max(0, lo - p.n_init)), dtype=torch.float32, device=dev)
    _check(load().esa_score_select_noalloc(_ptr(q_c), _ptr(k_c), b, lq, k_c.shape[1], c0, dc, p, _ptr(idx),
                                           _ptr(count), _ptr(scores) if want_scores else None, _stream()),
           "esa_score_select_noalloc")
    return idx, count, (scores if want_scores else None)


def score_select_heads_workspace_size(batch, lq, n_cap, c0, d_c, n_groups, p: EsaParams) -> int:
    return load().esa_score_select_heads_workspace_size(batch, lq, n_cap, c0, d_c, n_groups, p)


def score_select_heads(q_c: torch.Tensor, k_c: torch.Tensor, c0: int, n_groups: int, p: EsaParams,
                       want_scores: bool = False, idx: Optional[torch.Tensor] = None,
                       count: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None):
    """esa_score_select_heads (per-head selection: one per group of compressed columns).
    Returns (idx [B, G, topk] int32, count [B, G] int32, s' [B, G, n_mid] f32 or None)."""
    _dev(q_c, k_c)
    b, lq, dc = q_c.shape
    n_cap = k_c.shape[1]
    dev = q_c.device
    if idx is None:
        idx = torch.empty((b, n_groups, p.topk), dtype=torch.int32, device=dev)
    if count is None:
        count = torch.empty((b, n_groups), dtype=torch.int32, device=dev)
    if want_scores and scores is None:
        lo = min(c0, max(p.n_init, c0 - p.window))
        scores = torch.empty((b, n_groups, max(0, lo - p.n_init)), dtype=torch.float32, device=dev)
    ws = _workspace(score_select_heads_workspace_size(b, lq, n_cap, c0, dc, n_groups, p), dev, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().esa_score_select_heads(_ptr(q_c), _ptr(k_c), b, lq, n_cap, c0, dc, n_groups, p, _ptr(idx),
                                         _ptr(count), _ptr(scores) if want_scores else None, wp, wn, _stream()),
           "esa_score_select_heads")
    return idx, count, (scores if want_scores else None)


def sparse_attn_heads_workspace_size(batch, lq, c0, hq, hkv, d, dtype_code, p: EsaParams) -> int:
    return load().esa_sparse_attn_heads_workspace_size(batch, lq, c0, hq, hkv, d, dtype_code, p)


def sparse_attn_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, c0: int, idx: torch.Tensor,
                      count: torch.Tensor, p: EsaParams, scale: float = 0.0, want_lse: bool = False,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None):
    """esa_sparse_attn_heads: idx [B, Hkv, >=topk], count [B, Hkv] (one list per KV head).
    Returns (o [B, Lq, Hq, D], lse [B, Lq, Hq] f32 or None)."""
    _dev(q, k, v, idx, count)
    b, lq, hq, d = q.shape
    n_cap, hkv = k.shape[1], k.shape[2]
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((b, lq, hq), dtype=torch.float32, device=q.device)
    ws = _workspace(sparse_attn_heads_workspace_size(b, lq, c0, hq, hkv, d, dt, p), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().esa_sparse_attn_heads(_ptr(q), _ptr(k), _ptr(v), dt, b, lq, n_cap, c0, hq, hkv, d, _ptr(idx),
                                        _ptr(count), p, scale, _ptr(out), _ptr(lse) if want_lse else None, wp, wn,
                                        _stream()), "esa_sparse_attn_heads")
    return out, (lse if want_lse else None)


def sparse_attn_workspace_size(batch, lq, c0, hq, hkv, d, dtype_code, p: EsaParams) -> int:
    return load().esa_sparse_attn_workspace_size(batch, lq, c0, hq, hkv, d, dtype_code, p)


def sparse_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, c0: int, idx: torch.Tensor,
                count: torch.Tensor, p: EsaParams, scale: float = 0.0, want_lse: bool = False,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None):
    """esa_sparse_attn. q [B, Lq, Hq, D]; k, v [B, n_cap, Hkv, D]; idx [B, >=topk] int32.
    Returns (o [B, Lq, Hq, D], lse [B, Lq, Hq] f32 or None)."""
    _dev(q, k, v, idx, count)
    b, lq, hq, d = q.shape
    n_cap, hkv = k.shape[1], k.shape[2]
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((b, lq, hq), dtype=torch.float32, device=q.device)
    ws = _workspace(sparse_attn_workspace_size(b, lq, c0, hq, hkv, d, dt, p), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().esa_sparse_attn(_ptr(q), _ptr(k), _ptr(v), dt, b, lq, n_cap, c0, hq, hkv, d, _ptr(idx),
                                  _ptr(count), p, scale, _ptr(out), _ptr(lse) if want_lse else None, wp, wn,
                                  _stream()), "esa_sparse_attn")
    return out, (lse if want_lse else None)


def _seq_len(seq_len: torch.Tensor, batch: int) -> torch.Tensor:
    if not seq_len.is_cuda or seq_len.dtype != torch.int64 or seq_len.shape != (batch,) or not seq_len.is_contiguous():
        raise ValueError("seq_len must be a contiguous CUDA int64 tensor of shape [batch]")
    return seq_len


def compress_packed_varlen(x: torch.Tensor, packed: torch.Tensor, k_c: torch.Tensor, seq_len: torch.Tensor) -> None:
    """esa_compress_packed_varlen: x [B, Hin, D] bf16 (one new key row per sequence, each
    row contiguous) -> k_c[b, seq_len[b] - 1] of k_c [B, n_cap, d_out] f32."""
    if not x.is_cuda or not packed.is_cuda or not k_c.is_cuda:
        raise ValueError("libesa takes CUDA tensors (no CPU path)")
    b, hin, d = x.shape
    if x.stride(2) != 1 or x.stride(1) != d:
        raise ValueError("each row of x must be contiguous [Hin, D]")
    if not k_c.is_contiguous():
        raise ValueError("k_c must be contiguous")
    _check(load().esa_compress_packed_varlen(_ptr(x), b, x.stride(0) if b > 1 else hin * d, hin, d, _ptr(packed),
                                             k_c.shape[2], _ptr(k_c), k_c.shape[1], _ptr(_seq_len(seq_len, b)),
                                             _stream()), "esa_compress_packed_varlen")


def score_select_varlen_workspace_size(batch, n_cap, d_c, n_groups, p: EsaParams) -> int:
    return load().esa_score_select_varlen_workspace_size(batch, n_cap, d_c, n_groups, p)


def score_select_varlen(q_c: torch.Tensor, k_c: torch.Tensor, seq_len: torch.Tensor, p: EsaParams, n_groups: int = 1,
                        want_scores: bool = False, idx: Optional[torch.Tensor] = None,
                        count: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None):
    """esa_score_select_varlen: one query per sequence at position seq_len[b] - 1.
    q_c [B, 1, d_c], k_c [B, n_cap, d_c] f32. Returns (idx [B, G, topk] int32,
    count [B, G] int32, s' [B, G, n_mid_max] f32 or None); G = n_groups."""
    _dev(q_c, k_c)
    b, lq, dc = q_c.shape
    if lq != 1:
        raise ValueError("one query per sequence")
    n_cap = k_c.shape[1]
    dev = q_c.device
    if idx is None:
        idx = torch.empty((b, n_groups, p.topk), dtype=torch.int32, device=dev)
    if count is None:
        count = torch.empty((b, n_groups), dtype=torch.int32, device=dev)
    if want_scores and scores is None:
        c0 = n_cap - 1
        lo = min(c0, max(p.n_init, c0 - p.window))
        scores = torch.full((b, n_groups, max(0, lo - p.n_init)), float("nan"), dtype=torch.float32, device=dev)
    ws = _workspace(score_select_varlen_workspace_size(b, n_cap, dc, n_groups, p), dev, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().esa_score_select_varlen(_ptr(q_c), _ptr(k_c), b, n_cap, _ptr(_seq_len(seq_len, b)), dc, n_groups,
                                          p, _ptr(idx), _ptr(count), _ptr(scores) if want_scores else None, wp, wn,
                                          _stream()), "esa_score_select_varlen")
    return idx, count, (scores if want_scores else None)


def sparse_attn_varlen_workspace_size(batch, n_cap, hq, hkv, d, dtype_code, lists, p: EsaParams) -> int:
    return load().esa_sparse_attn_varlen_workspace_size(batch, n_cap, hq, hkv, d, dtype_code, lists, p)


def sparse_attn_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, seq_len: torch.Tensor, idx: torch.Tensor,
                       count: torch.Tensor, p: EsaParams, scale: float = 0.0, want_lse: bool = False,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None):
    """esa_sparse_attn_varlen: q [B, 1, Hq, D]; k, v [B, n_cap, Hkv, D]; idx [B, L, >=topk],
    count [B, L] with L = 1 (shared list) or Hkv (one per KV head), or idx [B, topk] and
    count [B]. Returns (o [B, 1, Hq, D], lse [B, 1, Hq] f32 or None)."""
    _dev(q, k, v, idx, count)
    b, lq, hq, d = q.shape
    if lq != 1:
        raise ValueError("one query per sequence")
    n_cap, hkv = k.shape[1], k.shape[2]
    lists = count.shape[1] if count.dim() == 2 else 1
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((b, lq, hq), dtype=torch.float32, device=q.device)
    ws = _workspace(sparse_attn_varlen_workspace_size(b, n_cap, hq, hkv, d, dt, lists, p), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().esa_sparse_attn_varlen(_ptr(q), _ptr(k), _ptr(v), dt, b, n_cap, _ptr(_seq_len(seq_len, b)), hq,
                                         hkv, d, _ptr(idx), _ptr(count), lists, p, scale, _ptr(out),
                                         _ptr(lse) if want_lse else None, wp, wn, _stream()),
           "esa_sparse_attn_varlen")
    return out, (lse if want_lse else None)


def gram(x: torch.Tensor, workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """esa_gram: G = X^T X (fp64 [dim, dim]) of bf16 rows x [n, dim] (any leading shape
    flattened to rows)."""
    _dev(x)
    dim = x.shape[-1]
    n = x.numel() // dim
    if out is None:
        out = torch.empty((dim, dim), dtype=torch.float64, device=x.device)
    ws = _workspace(load().esa_gram_workspace_size(n, dim), x.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().esa_gram(_ptr(x), _dtype_code(x), n, dim, _ptr(out), wp, wn, _stream()), "esa_gram")
    return out


def fit_workspace_size(n_q, n_k, hq, hkv, d, d_c, oversample) -> int:
    return load().esa_fit_workspace_size(n_q, n_k, hq, hkv, d, d_c, oversample)


def fit_maps(q: torch.Tensor, k: torch.Tensor, d_c: int, omega: torch.Tensor, ridge: float = 0.0,
             power_iters: int = 8, workspace: Optional[torch.Tensor] = None):
    """esa_fit_maps: compression maps fitted to calibration queries q [n_q, hq, d] and keys
    k [n_k, hkv, d] (bf16). omega: [hkv * d, d_c + oversample] float64 standard normal
    start (its width sets the oversampling). Returns (w_q, w_k), fp32 [hq * d, d_c] each,
    in the layout esa_compress takes."""
    _dev(q, k, omega)
    n_q, hq, d = q.shape
    n_k, hkv = k.shape[0], k.shape[1]
    if omega.dtype != torch.float64 or omega.dim() != 2 or omega.shape[0] != hkv * d or omega.shape[1] < d_c:
        raise ValueError("omega must be a contiguous float64 [hkv * d, d_c + oversample] tensor")
    oversample = omega.shape[1] - d_c
    w_q = torch.empty((hq * d, d_c), dtype=torch.float32, device=q.device)
    w_k = torch.empty((hq * d, d_c), dtype=torch.float32, device=q.device)
    ws = _workspace(fit_workspace_size(n_q, n_k, hq, hkv, d, d_c, oversample), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().esa_fit_maps(_ptr(q), n_q, _ptr(k), n_k, _dtype_code(q), hq, hkv, d, d_c, oversample,
                               float(ridge), int(power_iters), _ptr(omega), _ptr(w_q), _ptr(w_k), wp, wn,
                               _stream()), "esa_fit_maps")
    return w_q, w_k


def cca_workspace_size(batch, seq, hq, d, group) -> int:
    return load().cca_workspace_size(batch, seq, hq, d, group)


def cca_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, group: int, window: int, scale: float = 0.0,
             want_lse: bool = False, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None):
    """cca_attn: CCA-style causal attention. q [B, S, Hq, D], k, v [B, S, Hkv, D] bf16.
    Returns (o [B, S, Hq, D], lse [B, S, Hq] f32 or None)."""
    _dev(q, k, v)
    b, s, hq, d = q.shape
    hkv = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((b, s, hq), dtype=torch.float32, device=q.device)
    ws = _workspace(cca_workspace_size(b, s, hq, d, group), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().cca_attn(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), b, s, hq, hkv, d, group, window, scale,
                           _ptr(out), _ptr(lse) if want_lse else None, wp, wn, _stream()), "cca_attn")
    return out, (lse if want_lse else None)


def moba_block_means(k: torch.Tensor, block: int, blk_begin: int = 0, blk_end: Optional[int] = None,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """moba_block_means: means of blocks [blk_begin, blk_end) of k [B, n_cap, H, D] bf16
    into kbar [B, H, ceil(n_cap / block), D] fp32 (allocated when out is None)."""
    _dev(k)
    b, n_cap, h, d = k.shape
    nb = (n_cap + block - 1) // block
    if out is None:
        out = torch.zeros((b, h, nb, d), dtype=torch.float32, device=k.device)
    end = nb if blk_end is None else blk_end
    _check(load().moba_block_means(_ptr(k), _dtype_code(k), b, n_cap, h, d, block, blk_begin, end, _ptr(out),
                                   _stream()), "moba_block_means")
    return out


def moba_decode_workspace_size(batch, n_cap, pos, heads, d, block, topk) -> int:
    return load().moba_decode_workspace_size(batch, n_cap, pos, heads, d, block, topk)


def moba_decode_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, pos: int, kbar: torch.Tensor, block: int,
                     topk: int, scale: float = 0.0, want_lse: bool = False, want_blocks: bool = False,
                     out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                     blocks: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """moba_decode_attn: one decode step for the query q [B, 1, H, D] at position pos.
    Returns (o [B, 1, H, D], lse [B, 1, H] or None, blocks [B, H, topk+1] int16 or None)."""
    _dev(q, k, v, kbar)
    b, _, h, d = q.shape
    n_cap = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((b, 1, h), dtype=torch.float32, device=q.device)
    if want_blocks and blocks is None:
        blocks = torch.empty((b, h, topk + 1), dtype=torch.int16, device=q.device)
    ws = _workspace(moba_decode_workspace_size(b, n_cap, pos, h, d, block, topk), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().moba_decode_attn(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), b, n_cap, pos, h, d, block, topk,
                                   _ptr(kbar), scale, _ptr(out), _ptr(lse) if want_lse else None,
                                   _ptr(blocks) if want_blocks else None, wp, wn, _stream()), "moba_decode_attn")
    return out, (lse if want_lse else None), (blocks if want_blocks else None)


def moba_workspace_size(which, batch, seq, heads, d, block, topk) -> int:
    return load().moba_workspace_size(which, batch, seq, heads, d, block, topk)


def moba_block_gate(q, k, block: int, topk: int, out=None, workspace=None) -> torch.Tensor:
    """moba_block_gate -> blocks [B, S, H, topk+1] int16."""
    _dev(q, k)
    b, s, h, d = q.shape
    if out is None:
        out = torch.empty((b, s, h, topk + 1), dtype=torch.int16, device=q.device)
    ws = _workspace(moba_workspace_size(0, b, s, h, d, block, topk), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().moba_block_gate(_ptr(q), _ptr(k), _dtype_code(q), b, s, h, d, block, topk, _ptr(out), wp, wn,
                                  _stream()), "moba_block_gate")
    return out


def moba_block_attn(q, k, v, block: int, topk: int, blocks: torch.Tensor, scale: float = 0.0,
                    want_lse: bool = False, out=None, lse=None, workspace=None):
    """moba_block_attn -> (o [B, S, H, D], lse [B, S, H] or None)."""
    _dev(q, k, v, blocks)
    b, s, h, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((b, s, h), dtype=torch.float32, device=q.device)
    ws = _workspace(moba_workspace_size(1, b, s, h, d, block, topk), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().moba_block_attn(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), b, s, h, d, block, topk, _ptr(blocks),
                                  scale, _ptr(out), _ptr(lse) if want_lse else None, wp, wn, _stream()),
           "moba_block_attn")
    return out, (lse if want_lse else None)


def moba_block_gate_attn(q, k, v, block: int, topk: int, scale: float = 0.0, want_blocks: bool = False,
                         want_lse: bool = False, out=None, lse=None, blocks=None, workspace=None):
    """moba_block_gate_attn -> (o, lse or None, blocks or None)."""
    _dev(q, k, v)
    b, s, h, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((b, s, h), dtype=torch.float32, device=q.device)
    if want_blocks and blocks is None:
        blocks = torch.empty((b, s, h, topk + 1), dtype=torch.int16, device=q.device)
    ws = _workspace(moba_workspace_size(2, b, s, h, d, block, topk), q.device, workspace)
    wp, wn = _ws_ptr(ws)
    _check(load().moba_block_gate_attn(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), b, s, h, d, block, topk, scale,
                                       _ptr(out), _ptr(lse) if want_lse else None,
                                       _ptr(blocks) if want_blocks else None, wp, wn, _stream()),
           "moba_block_gate_attn")
    return out, (lse if want_lse else None), (blocks if want_blocks else None)


def launch_count() -> int:
    """Kernels libesa has launched in this process."""
    return int(load().esa_launch_count())


def wait_selftest(limit_ns: int) -> None:
    """esa_wait_selftest: a kernel whose bounded wait runs out after limit_ns and
    records a timeout (read back by device_status)."""
    _check(load().esa_wait_selftest(int(limit_ns), _stream()), "esa_wait_selftest")


def device_status() -> None:
    """Raise EsaError if a kernel's bounded wait ran out since the last check."""
    _check(load().esa_device_status(_stream()), "esa_device_status")
