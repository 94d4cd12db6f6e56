"""Plant plausible mistakes in the oracle and check that a pin catches each.

Each mutation rewrites one snippet of one oracle function's source (the snippet
must occur exactly once), installs the rewritten function in place of the
original for the duration of the test, and runs the pin that should fail.
Mistakes are planted in the oracle, on the CPU, never in the CUDA path.
"""
import inspect
import textwrap

import pytest

from oracle import cca, esa, esa_fit, esa_heads, esa_varlen, moba
from tests import test_oracle_cca as tc
from tests import test_oracle_esa as pe
from tests import test_oracle_fit as tf
from tests import test_oracle_heads as th
from tests import test_oracle_moba as pm
from tests import test_oracle_varlen as tv

MUTATIONS = [
    # (module, function, snippet, replacement, pin)
    (esa, "compress", "np.repeat(xb, g, axis=1)", "np.tile(xb, (1, g, 1))",
     pe.check_identity_compression_is_multihead_dot),                      # GQA head order
    (esa, "importance", "corrected = np.maximum(corrected, -float(clamp_c))", "pass",
     pe.check_worked_example),                                             # clamp dropped
    (esa, "importance", "m = s_full.max(axis=1, keepdims=True)", "m = s_full.max(axis=0, keepdims=True)",
     pe.check_worked_example),                                             # max over the wrong axis
    (esa, "importance", "return corrected.sum(axis=0)", "return corrected.mean(axis=0)",
     pe.check_worked_example),                                             # mean instead of sum
    (esa, "importance", "corrected = s_full - m", "corrected = s_full + m",
     pe.check_worked_example),                                             # wrong sign
    (esa, "neighbour_max", "for off in range(1, eps + 1):", "for off in range(1, eps):",
     pe.check_neighbour_max_properties),                                   # radius off by one
    (esa, "neighbour_max", "out[off:] = np.maximum(out[off:], s[:-off])", "pass",
     pe.check_neighbour_max_properties),                                   # one-sided window
    (esa, "topk_ascending", "order = np.lexsort((np.arange(n), -values))",
     "order = np.lexsort((-np.arange(n), -values))", pe.check_topk_brute_force),   # tie order
    (esa, "topk_ascending", "return np.sort(order[:keep])", "return np.sort(order[:keep - 1])",
     pe.check_worked_example),                                             # one short
    (esa, "sparse_attn", "scale = 1.0 / math.sqrt(d)", "scale = 1.0",
     pe.check_full_selection_is_causal_attention),                         # missing scale
    (esa, "sparse_attn", "vis = keys <= p", "vis = keys < p",
     pe.check_full_selection_is_causal_attention),                         # causal off by one
    (esa, "sparse_attn", "head_map = np.arange(hq) // g", "head_map = np.arange(hq) % hkv",
     pe.check_full_selection_is_causal_attention),                         # GQA head order
    (esa, "sparse_attn", "lse[b, i] = (mx + np.log(den))[:, 0]", "lse[b, i] = np.log(den)[:, 0]",
     pe.check_full_selection_is_causal_attention),                         # lse without max
    (esa, "regions", "lo = min(c0, max(n_init, c0 - window))", "lo = min(c0, max(n_init, c0 - window + 1))",
     pe.check_attended_count),                                             # window off by one
    (esa, "attended_keys", "np.arange(l0, l1)", "np.arange(l0, l1 - 1)",
     pe.check_full_selection_is_causal_attention),                         # chunk cut short
    (esa_heads, "compress_heads", "xg = xe[:, g * hpg:(g + 1) * hpg, :].reshape(rows, hpg * d)",
     "xg = xe[:, :hpg, :].reshape(rows, hpg * d)",
     th.test_group_maps_equal_the_block_diagonal_merged_map),              # every group reads group 0's heads
    (esa_heads, "score_select_heads", "cols = slice(g * dg, (g + 1) * dg)",
     "cols = slice(((g + 1) % n_groups) * dg, ((g + 1) % n_groups + 1) * dg)",
     th.test_a_needle_seen_by_one_head_is_selected_by_that_head_only),     # another group's slice
    (esa_heads, "sparse_attn_heads", "idx[b, g], int(count[b, g])", "idx[b, 0], int(count[b, 0])",
     th.test_each_group_attends_its_own_list),                             # one list for every head
    (moba, "block_means", "k[:, b * block:min((b + 1) * block, s)]", "k[:, b * block:min((b + 1) * block + 1, s)]",
     pm.check_block_means_of_a_ramp),                                      # block boundary
    (moba, "gate", "sc = np.einsum(\"hd,hnd->hn\", q[b, p], kbar[b, :, :cur, :])",
     "sc = -np.einsum(\"hd,hnd->hn\", q[b, p], kbar[b, :, :cur, :])", pm.check_gate_brute_force),  # sign
    (moba, "gate", "order = np.lexsort((np.arange(cur), -vals))", "order = np.lexsort((-np.arange(cur), -vals))",
     pm.check_gate_brute_force),                                           # tie order
    (moba, "attend", "end = p + 1", "end = min((blk + 1) * block, s)",
     pm.check_all_blocks_is_full_attention),                               # current block not causal
    (moba, "attend", "scale = 1.0 / math.sqrt(d)", "scale = 1.0",
     pm.check_no_past_block_is_block_local),                               # missing scale
    (esa_varlen, "score_select_varlen", "c0 = n - 1", "c0 = n - 2",
     tv.check_short_sequences_attend_everything),                          # query position off by one
    (esa_varlen, "sparse_attn_varlen", "c0 = n - 1", "c0 = n - 2",
     tv.check_short_sequences_attend_everything),                          # attention stops one row short
    (esa_varlen, "sparse_attn_varlen", "if lists == 1:", "if True:",
     tv.check_per_head_lists_per_sequence),                                # first list for every head
    (esa_fit, "expansion", "kv = h // g", "kv = h % hkv",
     tf.check_full_rank_fit_is_exact),                                     # GQA order in the fit
    (esa_fit, "fit_maps", "w_k = e @ b / g", "w_k = e @ b",
     tf.check_full_rank_fit_is_exact),                                     # expanded key map not divided
    (esa_fit, "fit_maps", "u[:, :d_c] * root", "u[:, -d_c:] * root",
     tf.check_matches_alternating_least_squares),                          # trailing singular vectors
    (esa_fit, "_upper_cholesky", "return np.linalg.cholesky(gram).T", "return np.linalg.cholesky(gram)",
     tf.check_matches_alternating_least_squares),                          # lower factor for the upper one
    (esa_fit, "scores_full", "np.repeat(k, g, axis=1)", "np.tile(k, (1, g, 1))",
     tf.check_full_rank_fit_is_exact),                                     # target scores with the wrong heads
    (cca, "window_start", "return max(0, g * (i // g) - w)", "return max(0, i - w)",
     tc.check_counts_and_tiling),                                          # window not on a group boundary
    (cca, "attend", "n_core = lo // g", "n_core = lo // g + 1",
     tc.check_counts_and_tiling),                                          # core of the window's first group too
    (cca, "core_tokens", "x = scale * (k[b, t0:t1, kv] @ q[b, t1 - 1, h])",
     "x = scale * (k[b, t0:t1, kv] @ q[b, t0, h])", tc.check_dominant_key_is_the_core_token),  # first query pools
    (cca, "attend", "kv = h // gq", "kv = h % hkv",
     tc.check_groups_of_one_are_full_attention),                           # GQA order
    (cca, "attend", "x = scale * (keys @ q[b, i, h])", "x = keys @ q[b, i, h]",
     tc.check_window_over_everything_is_full_attention),                   # missing scale
]


def _mutated(module, name, old, new):
    src = textwrap.dedent(inspect.getsource(getattr(module, name)))
    assert src.count(old) == 1, f"snippet not found exactly once in {name}: {old}"
    ns = dict(module.__dict__)
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    return ns[name]


@pytest.mark.parametrize("mut", MUTATIONS, ids=lambda m: f"{m[0].__name__.split('.')[-1]}.{m[1]}:{m[3][:28]}")
def test_pin_catches_planted_mistake(mut, monkeypatch):
    module, name, old, new, pin = mut
    monkeypatch.setattr(module, name, _mutated(module, name, old, new))
    with pytest.raises(AssertionError):
        pin()


def test_unmutated_pins_pass():
    for mut in MUTATIONS:
        mut[4]()
