"""CCA-style attention: the CUDA path (cca_attn through the C ABI) against the oracle
(oracle/cca.py), element by element at sizes that span several tiles and groups and a
ragged last tile, and on sampled rows at the full workload size."""
import numpy as np
import pytest
import torch

import query_aware_selective_b200 as qas
from oracle import cca as occa
from query_aware_selective_b200 import synthetic
from tests.parity import ATOL_BF16, max_abs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("batch,seq,hq,hkv,group,window", [
    (1, 1000, 8, 2, 128, 256),     # ragged last tile, an incomplete last group
    (2, 640, 4, 4, 128, 0),        # no window beyond the own group
    (1, 1536, 8, 1, 256, 512),     # GQA 8, groups of two tiles
    (1, 300, 4, 2, 128, 1024),     # the window covers everything: full causal attention
])
def test_cca_parity(batch, seq, hq, hkv, group, window):
    g = torch.Generator().manual_seed(seq + hq)
    q = torch.randn(batch, seq, hq, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(batch, seq, hkv, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(batch, seq, hkv, 128, generator=g).to(torch.bfloat16)
    o, lse = qas.cca_attn(q.to(DEV), k.to(DEV), v.to(DEV), group, window, want_lse=True)
    qas.device_status()
    ref_o, ref_lse = occa.attend(q.double().numpy(), k.double().numpy(), v.double().numpy(), group, window)
    assert max_abs(o.cpu().double().numpy(), ref_o) <= ATOL_BF16
    assert max_abs(lse.cpu().double().numpy(), ref_lse) <= 1e-2


def test_cca_64k_sampled_rows():
    w = synthetic.CCA_64K
    inp = synthetic.make_cca_inputs(w, device=DEV)
    o, _ = qas.cca_attn(inp["q"], inp["k"], inp["v"], w.group, w.window)
    qas.device_status()
    rows = [(0, i) for i in (0, 127, 128, 1151, 1152, 40000, w.seq - 1)]
    q, k, v = (inp[x].double().cpu().numpy() for x in ("q", "k", "v"))
    ref_o, _ = occa.attend(q, k, v, w.group, w.window, rows=rows)
    got = o.double().cpu().numpy()
    for b, i in rows:
        assert max_abs(got[b, i], ref_o[b, i]) <= ATOL_BF16, i
    del inp
    torch.cuda.empty_cache()
