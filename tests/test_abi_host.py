"""Host-side checks of the C ABI that need no GPU.

The library must load, export every function include/esa.h declares, and reject
bad arguments on the host before anything is launched (no CUDA call happens on
these paths). The Python binding must refuse CPU tensors: there is no CPU path.
"""
import ctypes
import math
import os
import re

import pytest
import torch

import query_aware_selective_b200 as qas
from query_aware_selective_b200 import _abi
from query_aware_selective_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "esa.h")


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return _abi.load()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:esa_status_t|size_t|uint64_t|const char\*)\s+(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = set(header_functions())
    for required in ["esa_compress", "esa_score_select", "esa_sparse_attn", "moba_block_gate_attn",
                     "esa_last_error", "esa_device_status"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
        assert name in _abi.SIGNATURES, f"binding does not declare {name}"


def test_params_struct_layout():
    assert ctypes.sizeof(_abi.EsaParams) == 20
    assert [f[0] for f in _abi.EsaParams._fields_] == ["n_init", "window", "topk", "eps", "clamp_c"]


FAKE = 0x10000  # a 256-byte aligned non-null value: never dereferenced on the rejected paths


def _err(lib):
    return lib.esa_last_error().decode()


def test_compress_rejects_bad_arguments(lib):
    f = lib.esa_compress
    xs = 8 * 128
    assert f(FAKE, 1, -1, xs, 8, 32, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG
    assert "rows" in _err(lib)
    assert f(None, 1, 4, xs, 8, 32, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG
    assert f(FAKE, 7, 4, xs, 8, 32, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG
    assert f(FAKE, 1, 4, xs, 8, 30, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG
    assert f(FAKE, 1, 4, xs, 8, 32, 96, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_UNSUPPORTED
    assert f(FAKE, 1, 4, xs, 8, 32, 128, FAKE, 24, FAKE, 24, None) == _abi.ESA_ERR_UNSUPPORTED
    assert f(FAKE, 1, 4, xs, 8, 32, 128, FAKE, 128, FAKE, 64, None) == _abi.ESA_ERR_INVALID_ARG
    assert f(FAKE, 1, 4, xs - 8, 8, 32, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG
    assert f(FAKE, 1, 4, xs + 4, 8, 32, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG
    # zero rows is a no-op that launches nothing
    assert f(FAKE, 1, 0, xs, 8, 32, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_OK


def test_compress_pack_size_and_rejections(lib):
    # K = n_heads_in * head_dim must be a multiple of 512 and d_out 128
    assert lib.esa_compress_pack_size(32, 128, 128) == 2 * 128 * 4096 * 2
    assert lib.esa_compress_pack_size(8, 128, 128) == 2 * 128 * 1024 * 2
    assert lib.esa_compress_pack_size(4, 64, 128) == 0          # K = 256
    assert lib.esa_compress_pack_size(32, 128, 64) == 0         # d_out 64
    assert lib.esa_compress_pack_size(0, 128, 128) == 0
    f = lib.esa_compress_pack
    n = lib.esa_compress_pack_size(8, 128, 128)
    assert f(None, 8, 32, 128, 128, FAKE, n, None) == _abi.ESA_ERR_INVALID_ARG
    assert f(FAKE, 8, 30, 128, 128, FAKE, n, None) == _abi.ESA_ERR_INVALID_ARG
    assert f(FAKE, 4, 4, 64, 128, FAKE, n, None) == _abi.ESA_ERR_UNSUPPORTED
    assert f(FAKE, 8, 32, 128, 128, FAKE, n - 16, None) == _abi.ESA_ERR_INVALID_ARG
    assert f(FAKE, 8, 32, 128, 128, FAKE + 8, n, None) == _abi.ESA_ERR_INVALID_ARG
    g = lib.esa_compress_packed
    assert g(FAKE, -1, 1024, 8, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG
    assert g(FAKE, 0, 1024, 8, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_OK
    assert g(None, 4, 1024, 8, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG
    assert g(FAKE, 4, 1024, 8, 128, FAKE, 64, FAKE, 128, None) == _abi.ESA_ERR_UNSUPPORTED
    assert g(FAKE, 4, 1000, 8, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG
    assert g(FAKE, 4, 1028, 8, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG
    assert g(FAKE, 4, 1024, 8, 128, FAKE, 128, FAKE, 96, None) == _abi.ESA_ERR_INVALID_ARG
    assert g(FAKE + 2, 4, 1024, 8, 128, FAKE, 128, FAKE, 128, None) == _abi.ESA_ERR_INVALID_ARG


def test_score_select_rejects_bad_arguments(lib):
    f = lib.esa_score_select
    good = _abi.params(128, 4096, 2048, 2, 45.25)
    args = lambda p, lq=1, n_cap=131072, c0=131071, dc=128, ws=FAKE, wsn=1 << 40: (
        FAKE, FAKE, 16, lq, n_cap, c0, dc, p, FAKE, FAKE, None, ws, wsn, None)
    assert f(*args(_abi.params(128, 4096, 0, 2, 1.0))) == _abi.ESA_ERR_INVALID_ARG      # topk 0
    assert f(*args(_abi.params(128, 4096, 16, 65, 1.0))) == _abi.ESA_ERR_INVALID_ARG    # eps too large
    assert f(*args(_abi.params(128, 4096, 16, 2, -1.0))) == _abi.ESA_ERR_INVALID_ARG    # negative clamp
    assert f(*args(_abi.params(128, 4096, 16, 2, math.nan))) == _abi.ESA_ERR_INVALID_ARG
    assert f(*args(good, c0=131072)) == _abi.ESA_ERR_INVALID_ARG                          # c0 + lq > n_cap
    assert f(*args(good, lq=0)) == _abi.ESA_ERR_INVALID_ARG
    assert f(*args(good, dc=24)) == _abi.ESA_ERR_UNSUPPORTED
    assert f(*args(good, ws=None)) == _abi.ESA_ERR_WORKSPACE
    assert f(*args(good, wsn=16)) == _abi.ESA_ERR_WORKSPACE
    assert f(*args(good, ws=FAKE + 8)) == _abi.ESA_ERR_WORKSPACE                          # misaligned
    assert "workspace" in _err(lib)


def test_sparse_attn_rejects_bad_arguments(lib):
    f = lib.esa_sparse_attn
    p = _abi.params(128, 4096, 2048, 2, 45.25)
    a = lambda hq=32, hkv=8, d=128, dt=1, q=FAKE, o=FAKE: (
        q, FAKE, FAKE, dt, 16, 1, 131072, 131071, hq, hkv, d, FAKE, FAKE, p, 0.0, o, None, FAKE, 1 << 40, None)
    assert f(*a(hq=12, hkv=4)) == _abi.ESA_ERR_UNSUPPORTED        # group of 3
    assert f(*a(hq=30, hkv=8)) == _abi.ESA_ERR_INVALID_ARG
    assert f(*a(d=80)) == _abi.ESA_ERR_UNSUPPORTED
    assert f(*a(dt=5)) == _abi.ESA_ERR_INVALID_ARG
    assert f(*a(q=FAKE + 2)) == _abi.ESA_ERR_INVALID_ARG           # misaligned
    assert f(*a(o=None)) == _abi.ESA_ERR_INVALID_ARG


def test_moba_rejects_bad_arguments(lib):
    f = lib.moba_block_gate_attn
    a = lambda dt=1, block=1024, topk=3, d=128: (FAKE, FAKE, FAKE, dt, 1, 65536, 32, d, block, topk, 0.0, FAKE,
                                                 None, None, FAKE, 1 << 40, None)
    assert f(*a(dt=0)) == _abi.ESA_ERR_UNSUPPORTED
    assert f(*a(block=100)) == _abi.ESA_ERR_INVALID_ARG
    assert f(*a(topk=16)) == _abi.ESA_ERR_INVALID_ARG
    assert f(*a(d=64)) == _abi.ESA_ERR_UNSUPPORTED
    assert f(*a(block=16)) == _abi.ESA_ERR_UNSUPPORTED              # 4096 blocks > 1024


def test_workspace_sizes(lib):
    p = _abi.params(128, 4096, 2048, 2, 45.25)
    small = _abi.score_select_workspace_size(1, 1, 32768, 16384, 128, p)
    big = _abi.score_select_workspace_size(16, 1, 131072, 131071, 128, p)
    assert 0 < small < big
    assert _abi.score_select_workspace_size(0, 1, 10, 5, 128, p) == 0
    assert _abi.moba_workspace_size(0, 1, 65536, 32, 128, 1024, 3) < _abi.moba_workspace_size(2, 1, 65536, 32, 128,
                                                                                              1024, 3)
    assert _abi.moba_workspace_size(7, 1, 65536, 32, 128, 1024, 3) == 0


def test_binding_refuses_cpu_tensors():
    x = torch.zeros(4, 8, 128, dtype=torch.bfloat16)
    w = torch.zeros(4096, 128)
    with pytest.raises(ValueError, match="CUDA"):
        qas.compress(x, w, 32)


def test_rejected_calls_launch_nothing(lib):
    before = lib.esa_launch_count()
    lib.esa_compress(None, 1, 4, 1024, 8, 32, 128, FAKE, 128, FAKE, 128, None)
    lib.esa_compress(FAKE, 1, 0, 1024, 8, 32, 128, FAKE, 128, FAKE, 128, None)
    assert lib.esa_launch_count() == before


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        _abi.load(str(tmp_path / "libesa.so"))


def test_varlen_calls_reject_bad_arguments(lib):
    p = _abi.params(128, 4096, 2048, 2, 45.25)
    sel = lambda seq_len=FAKE, n_cap=131072, dc=128, ng=1, ws=FAKE, wsn=1 << 40: lib.esa_score_select_varlen(
        FAKE, FAKE, 16, n_cap, seq_len, dc, ng, p, FAKE, FAKE, None, ws, wsn, None)
    assert sel(seq_len=None) == _abi.ESA_ERR_INVALID_ARG
    assert sel(n_cap=0) == _abi.ESA_ERR_INVALID_ARG
    assert sel(ng=3) == _abi.ESA_ERR_UNSUPPORTED
    assert sel(dc=96) == _abi.ESA_ERR_UNSUPPORTED            # no one-query scoring path for d_c 96
    assert sel(wsn=16) == _abi.ESA_ERR_WORKSPACE
    att = lambda seq_len=FAKE, lists=1, n_cap=131072: lib.esa_sparse_attn_varlen(
        FAKE, FAKE, FAKE, 1, 16, n_cap, seq_len, 32, 8, 128, FAKE, FAKE, lists, p, 0.0, FAKE, None, FAKE, 1 << 40,
        None)
    assert att(seq_len=None) == _abi.ESA_ERR_INVALID_ARG
    assert att(lists=3) == _abi.ESA_ERR_INVALID_ARG           # 1 or hkv lists
    assert att(n_cap=0) == _abi.ESA_ERR_INVALID_ARG
    cmp = lambda seq_len=FAKE, n_cap=131072, d_out=128: lib.esa_compress_packed_varlen(
        FAKE, 16, 1024, 8, 128, FAKE, d_out, FAKE, n_cap, seq_len, None)
    assert cmp(seq_len=None) == _abi.ESA_ERR_INVALID_ARG
    assert cmp(n_cap=0) == _abi.ESA_ERR_INVALID_ARG
    assert cmp(d_out=64) == _abi.ESA_ERR_UNSUPPORTED


def test_varlen_workspaces_cover_the_longest_sequence(lib):
    # sized for a query at n_cap - 1: the equal-length call's workspace at that position
    p = _abi.params(128, 4096, 2048, 2, 45.25)
    assert _abi.score_select_varlen_workspace_size(16, 131072, 128, 1, p) == \
        _abi.score_select_workspace_size(16, 1, 131072, 131071, 128, p)
    assert _abi.score_select_varlen_workspace_size(16, 131072, 128, 8, p) == \
        _abi.score_select_heads_workspace_size(16, 1, 131072, 131071, 128, 8, p)
    assert _abi.sparse_attn_varlen_workspace_size(16, 131072, 32, 8, 128, 1, 1, p) == \
        _abi.sparse_attn_workspace_size(16, 1, 131071, 32, 8, 128, 1, p)
    assert _abi.sparse_attn_varlen_workspace_size(16, 131072, 32, 8, 128, 1, 8, p) == \
        _abi.sparse_attn_heads_workspace_size(16, 1, 131071, 32, 8, 128, 1, p)
    assert _abi.score_select_varlen_workspace_size(16, 0, 128, 1, p) == 0


def test_cca_rejects_bad_arguments(lib):
    a = lambda dt=1, hq=32, hkv=8, d=128, group=128, window=1024, q=FAKE: lib.cca_attn(
        q, FAKE, FAKE, dt, 1, 65536, hq, hkv, d, group, window, 0.0, FAKE, None, FAKE, 1 << 40, None)
    assert a(dt=0) == _abi.ESA_ERR_UNSUPPORTED                 # fp32
    assert a(hq=24) == _abi.ESA_ERR_UNSUPPORTED                # GQA group 3
    assert a(hq=30) == _abi.ESA_ERR_INVALID_ARG
    assert a(d=64) == _abi.ESA_ERR_UNSUPPORTED
    assert a(group=64) == _abi.ESA_ERR_UNSUPPORTED             # not a multiple of the 128-row tile
    assert a(window=1000) == _abi.ESA_ERR_INVALID_ARG          # not a multiple of the group
    assert a(q=None) == _abi.ESA_ERR_INVALID_ARG
    assert a(q=FAKE + 2) == _abi.ESA_ERR_INVALID_ARG
    f = lib.cca_attn
    assert f(FAKE, FAKE, FAKE, 1, 1, 65536, 32, 8, 128, 128, 1024, 0.0, FAKE, None, FAKE, 16, None) == \
        _abi.ESA_ERR_WORKSPACE
    assert _abi.cca_workspace_size(1, 65536, 32, 128, 128) > _abi.cca_workspace_size(1, 65536, 32, 128, 256) > 0


def test_wait_selftest_rejects_out_of_range_limits(lib):
    assert lib.esa_wait_selftest(10, None) == _abi.ESA_ERR_INVALID_ARG
    assert lib.esa_wait_selftest(10 ** 12, None) == _abi.ESA_ERR_INVALID_ARG


def test_fit_calls_reject_bad_arguments(lib):
    # every rejection happens on the host, before a launch
    before = lib.esa_launch_count()
    g = lambda dt=1, n=1000, dim=512, x=FAKE, out=FAKE, ws=FAKE, nb=1 << 40: lib.esa_gram(x, dt, n, dim, out, ws, nb,
                                                                                         None)
    assert g(dt=0) == _abi.ESA_ERR_UNSUPPORTED                 # fp32 rows
    assert g(dim=200) == _abi.ESA_ERR_UNSUPPORTED               # not a multiple of 128
    assert g(n=0) == _abi.ESA_ERR_INVALID_ARG
    assert g(x=None) == _abi.ESA_ERR_INVALID_ARG
    assert g(x=FAKE + 2) == _abi.ESA_ERR_INVALID_ARG            # misaligned
    assert g(out=None) == _abi.ESA_ERR_INVALID_ARG
    assert g(nb=16) == _abi.ESA_ERR_WORKSPACE
    f = lambda hq=32, hkv=8, d=128, dc=128, over=32, ridge=0.0, it=8, om=FAKE, nb=1 << 40, dt=1: lib.esa_fit_maps(
        FAKE, 65536, FAKE, 65536, dt, hq, hkv, d, dc, over, ridge, it, om, FAKE, FAKE, FAKE, nb, None)
    assert f(hq=30) == _abi.ESA_ERR_INVALID_ARG                 # not a multiple of hkv
    assert f(d=40) == _abi.ESA_ERR_UNSUPPORTED                  # 8 * 40 = 320 is not a multiple of 128
    assert f(dc=0) == _abi.ESA_ERR_UNSUPPORTED
    assert f(dc=129) == _abi.ESA_ERR_UNSUPPORTED                # 129 + 32 > 160
    assert f(dc=128, over=33) == _abi.ESA_ERR_UNSUPPORTED
    assert f(over=-1) == _abi.ESA_ERR_UNSUPPORTED
    assert f(ridge=-1.0) == _abi.ESA_ERR_INVALID_ARG
    assert f(ridge=math.nan) == _abi.ESA_ERR_INVALID_ARG
    assert f(it=65) == _abi.ESA_ERR_INVALID_ARG
    assert f(om=None) == _abi.ESA_ERR_INVALID_ARG
    assert f(nb=1024) == _abi.ESA_ERR_WORKSPACE
    assert f(dt=0) == _abi.ESA_ERR_UNSUPPORTED
    assert lib.esa_launch_count() == before


def test_fit_workspace_sizes(lib):
    # Gram partials: one fp64 [dim, dim] per slice of the rows (slices only when the
    # upper triangle has fewer than 148 tiles); the fit adds its fp64 matrices
    assert _abi.load().esa_gram_workspace_size(65536, 4096) == 4096 * 4096 * 8        # 528 tiles: one slice
    assert _abi.load().esa_gram_workspace_size(65536, 1024) == 4 * 1024 * 1024 * 8    # 36 tiles: 4 slices
    assert _abi.load().esa_gram_workspace_size(100, 1024) == 1 * 1024 * 1024 * 8      # one 128-row chunk
    assert _abi.load().esa_gram_workspace_size(100, 1000) == 0
    need = _abi.fit_workspace_size(65536, 65536, 32, 8, 128, 128, 32)
    dq, dk, dc, l = 4096, 1024, 128, 160
    fp64 = 8 * (dq * dq + 2 * dk * dk + 2 * dq * dk + 2 * dk * l + l * l + l * l + l * dc + dk * dc + dq * dc)
    assert need >= fp64 + dq * dq * 8 and need <= fp64 + dq * dq * 8 + 13 * 256
    assert _abi.fit_workspace_size(65536, 65536, 32, 8, 40, 128, 32) == 0
