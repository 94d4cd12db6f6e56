"""The allocation-free selection entry point, esa_score_select_noalloc.

Some callers cannot allocate device memory: a service that plans all of its memory
at start-up, a plugin inside another runtime that cannot reach that runtime's
allocator, a latency-critical loop that may not stall on an allocation. For them the
library keeps a fixed scratch array in device memory and offers this entry point,
which takes no workspace. These tests call it through the C ABI and compare it, on
two calls in a row (the array keeps the previous call's contents), with
esa_score_select, which takes a caller-allocated workspace, and with the oracle's
selection. This file runs last so
that a failure here cannot hide the rest of the suite.
"""
import math

import numpy as np
import pytest
import torch

from oracle import esa as oesa
from query_aware_selective_b200 import _abi
from tests.parity import check_selection

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _inputs(batch, lq, n_cap, dc, seed):
    g = torch.Generator().manual_seed(seed)
    q_c = torch.randn((batch, lq, dc), generator=g).to(DEV)
    k_c = torch.randn((batch, n_cap, dc), generator=g).to(DEV)
    return q_c, k_c


@pytest.mark.parametrize("batch,lq,n_cap,dc,n_init,window,topk,eps,clamp", [
    (2, 1, 6000, 128, 128, 512, 700, 2, 45.25),       # decode: register scoring path
    (1, 64, 5000, 128, 64, 1024, 512, 2, 45.25),      # prefill chunk: tensor-core scoring path
    (3, 5, 3000, 64, 16, 256, 300, 1, math.inf),      # a few queries, no clamp
])
def test_noalloc_matches_the_workspace_entry_point(batch, lq, n_cap, dc, n_init, window, topk, eps, clamp):
    p = _abi.params(n_init, window, topk, eps, clamp)
    c0 = n_cap - lq
    for call, seed in enumerate((11, 12)):           # two calls in a row, different inputs
        q_c, k_c = _inputs(batch, lq, n_cap, dc, seed + lq)
        ref_idx, ref_cnt, ref_s = _abi.score_select(q_c, k_c, c0, p, want_scores=True)
        idx, cnt, sc = _abi.score_select_noalloc(q_c, k_c, c0, p, want_scores=True)
        torch.cuda.synchronize()
        assert torch.equal(cnt.cpu(), ref_cnt.cpu()), call
        assert torch.equal(idx.cpu(), ref_idx.cpu()), call        # index work: bit-exact
        scale = max(1.0, float(ref_s.abs().max()))
        assert float((sc - ref_s).abs().max()) <= 1e-4 * scale, call
        # and against the oracle itself: the same selection rule as every other
        # selection test (exact outside the 1e-3 tie band around the k-th value)
        o_idx, o_cnt, o_sp = oesa.score_select(q_c.double().cpu().numpy(), k_c.double().cpu().numpy(), c0, n_init,
                                               window, topk, eps, clamp)
        _, (m0, _), _ = oesa.regions(c0, c0 + lq, n_init, window)
        for b in range(batch):
            check_selection(idx[b].cpu().numpy(), int(cnt[b]), o_idx[b], o_cnt[b], o_sp[b], m0, topk)
    _abi.device_status()


def test_noalloc_rejects_a_selection_larger_than_its_scratch():
    cap = _abi.load().esa_score_select_noalloc_capacity()
    assert cap == 8 << 20
    p = _abi.params(128, 4096, 2048, 2, 45.25)
    n_cap = 1 << 21                                   # 2M-token middle: far more scratch than 8 MiB
    need = _abi.score_select_workspace_size(4, 1, n_cap, n_cap - 1, 128, p)
    assert need > cap
    q_c = torch.zeros((4, 1, 128), device=DEV)
    k_c = torch.zeros((4, 8, 128), device=DEV)        # never read: the call is rejected first
    idx = torch.full((4, 2048), 7, dtype=torch.int32, device=DEV)
    cnt = torch.full((4,), 7, dtype=torch.int32, device=DEV)
    lib = _abi.load()
    before = lib.esa_launch_count()
    st = lib.esa_score_select_noalloc(q_c.data_ptr(), k_c.data_ptr(), 4, 1, n_cap, n_cap - 1, 128, p,
                                      idx.data_ptr(), cnt.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
    assert st == _abi.ESA_ERR_WORKSPACE
    assert "scratch" in lib.esa_last_error().decode()
    assert lib.esa_launch_count() == before
    assert int(cnt[0]) == 7 and int(idx[0, 0]) == 7   # outputs untouched
