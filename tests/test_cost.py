"""Pins of the roofline numerators (query_aware_selective_b200.cost) against numbers
the pages print (tests/golden/pages_numbers.json) and closed forms."""
import json

from query_aware_selective_b200 import cost, synthetic
from tests.conftest import golden_path

PAGES = json.load(open(golden_path("pages_numbers.json")))


def test_kv_cache_example_of_the_blog():
    e = PAGES["kv_cache_example_bytes"]
    b = cost.kv_cache_bytes(e["tokens"], e["heads"], e["head_dim"], e["bytes_per_value"])
    assert b == 32_768_000
    assert abs(b / 1e6 - e["value_mb"]) / e["value_mb"] < 0.05


def test_esa_compression_ratio():
    r = 100.0 * PAGES["esa_compress_out"]["value"] / PAGES["esa_compress_in"]["value"]
    assert abs(r - PAGES["esa_compress_ratio_pct"]["value"]) <= PAGES["esa_compress_ratio_pct"]["tol"]
    w = synthetic.DECODE_128K
    assert w.hidden == PAGES["esa_compress_in"]["value"] and w.d_c == PAGES["esa_compress_out"]["value"]


def test_esa_step_ratio_tends_to_the_pages_figure():
    w = synthetic.DECODE_128K
    r = [cost.esa_step_compute_ratio(n, w.hq, w.head_dim, w.d_c, w.n_init, w.window, w.topk)
         for n in (1 << 20, 1 << 24, 1 << 30)]
    assert r[0] > r[1] > r[2]                                   # falls towards the limit
    limit = w.d_c / (2 * w.hq * w.head_dim)                     # d' / (2 Hq D) = 1.5625%
    assert abs(100 * r[2] - 100 * limit) < 0.01
    assert abs(100 * r[2] - PAGES["esa_step_compute_pct"]["value"]) <= PAGES["esa_step_compute_pct"]["tol"]


def test_attended_count_and_full_attention_limit():
    # with k >= |mid| the prefill attention flops are those of full causal attention
    n, chunk, hq, d = 4096, 512, 4, 64
    f = cost.prefill_flops(n, chunk, hq, d, 16, 16, 128, 10**9)
    assert f["attention"] == cost.full_causal_attn_flops(n, hq, d)
    assert cost.attended(131071, 0, 128, 4096, 2048) == 6273


def test_moba_flops_limits():
    # all blocks kept -> full causal attention; no past block -> block-diagonal causal
    s, h, d, blk = 4096, 2, 64, 256
    assert cost.moba_flops(s, h, d, blk, 10**6)["attention"] == cost.full_causal_attn_flops(s, h, d)
    assert cost.moba_flops(s, h, d, blk, 0)["attention"] == (s // blk) * cost.full_causal_attn_flops(blk, h, d)


def test_varlen_bytes_reduce_to_the_equal_length_batch():
    a = cost.decode_varlen_bytes([131072] * 16, 32, 8, 128, 128, 128, 4096, 2048)
    b = cost.decode_bytes(16, 131072, 32, 8, 128, 128, 128, 4096, 2048)
    assert a["total"] == b["total"]
    # a short sequence reads no compressed keys (empty middle) and only its own rows
    c = cost.decode_varlen_bytes([131072, 100], 32, 8, 128, 128, 128, 4096, 2048)
    d = cost.decode_bytes(1, 131072, 32, 8, 128, 128, 128, 4096, 2048)
    assert c["compressed_keys"] == d["compressed_keys"]
    assert c["kv_rows"] == d["kv_rows"] + 100 * 8 * 128 * 2 * 2


def test_cca_keys_match_the_oracle():
    # zero keys make every attended key equally likely: the oracle's lse is log(#keys)
    import math
    import numpy as np
    from oracle import cca
    s, g, w = 45, 5, 10
    q = np.random.default_rng(0).standard_normal((1, s, 2, 4))
    k = np.zeros((1, s, 1, 4))
    v = np.zeros((1, s, 1, 4))
    _, lse = cca.attend(q, k, v, g, w)
    for i in range(s):
        assert cost.cca_keys(i, g, w) == round(math.exp(lse[0, i, 0]))


def test_cca_flops_reduce_to_full_attention():
    # groups of one token or a window over everything: every earlier token once
    assert cost.cca_flops(300, 32, 128, 1, 7)["attention"] == cost.full_causal_attn_flops(300, 32, 128)
    assert cost.cca_flops(300, 32, 128, 4, 400)["attention"] == cost.full_causal_attn_flops(300, 32, 128)


def test_fit_flops_gram_dominates_for_long_calibration():
    f = cost.fit_flops(65536, 65536, 32, 8, 128, 128)
    assert f["gram"] == 2 * 65536 * 4096 ** 2 + 2 * 65536 * 1024 ** 2
    assert f["gram"] > 0.5 * f["total"]
