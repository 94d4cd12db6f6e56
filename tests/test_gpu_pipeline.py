"""The prefill driver's host-buffer entry (EsaPrefill.run_from_host: inputs streamed in
chunk by chunk, outputs streamed back, overlapping the compute) gives the same output,
bit for bit, as the run on device-resident inputs, eagerly and as a replayed graph."""
import math

import pytest
import torch

import query_aware_selective_b200 as qas
from query_aware_selective_b200 import pipeline, synthetic

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_run_from_host_matches_the_device_run():
    w = synthetic.PREFILL_32K
    n = 6144                                      # 12 chunks: selection starts at chunk 9
    p = qas.params(w.n_init, w.window, w.topk, w.eps, w.clamp_c)
    inp = synthetic.make_esa_inputs(w, device=DEV, n_ctx=n)
    pf = pipeline.EsaPrefill(1, n, w.chunk, w.hq, w.hkv, w.head_dim, w.d_c, p, device=DEV)
    ref = pf.run(inp["q"], inp["k"], inp["v"], inp["wq"], inp["wk"]).clone()
    host = {x: inp[x].cpu().pin_memory() for x in ("q", "k", "v")}
    dev = {x: torch.zeros_like(inp[x]) for x in ("q", "k", "v")}
    out_host = torch.empty(ref.shape, dtype=ref.dtype).pin_memory()
    pf.run_from_host(host["q"], host["k"], host["v"], dev["q"], dev["k"], dev["v"], inp["wq"], inp["wk"],
                     out_host)
    torch.cuda.synchronize()
    qas.device_status()
    assert torch.equal(out_host, ref.cpu())
    # as a graph, replayed with new host inputs
    graph = pipeline.graph_of(lambda: pf.run_from_host(host["q"], host["k"], host["v"], dev["q"], dev["k"],
                                                       dev["v"], inp["wq"], inp["wk"], out_host))
    host["q"].mul_(-1.0)
    expect = pf.run(host["q"].to(DEV), inp["k"], inp["v"], inp["wq"], inp["wk"]).clone()
    out_host.zero_()
    graph.replay()
    torch.cuda.synchronize()
    qas.device_status()
    assert torch.equal(out_host, expect.cpu())
    del graph
