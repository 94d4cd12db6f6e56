"""Host logic of the prefill pipeline that needs no GPU: the key-compression batch a
chunk's selection waits for covers every middle position it reads, against the
oracle's region rule."""
import pytest

from oracle import esa as oesa
from query_aware_selective_b200 import pipeline


@pytest.mark.parametrize("n_ctx,chunk,n_init,window,kbatch", [
    (32768, 512, 128, 4096, 2),      # the prefill workload
    (32768, 512, 128, 4096, 1),
    (16384, 512, 128, 4096, 3),
    (5000, 300, 16, 700, 2),         # ragged last chunk, window not a multiple of the chunk
    (2048, 256, 0, 0, 4),            # no initial tokens, no window
])
def test_selection_waits_for_every_key_it_reads(n_ctx, chunk, n_init, window, kbatch):
    prev = -1
    for c0 in range(0, n_ctx, chunk):
        lq = min(chunk, n_ctx - c0)
        _, (m0, m1), _ = oesa.regions(c0, c0 + lq, n_init, window)
        batch = pipeline.key_batch_needed(c0, chunk, n_init, window, kbatch)
        if m1 <= m0:
            assert batch == -1                                   # empty middle: nothing to wait for
            continue
        covered_end = min(n_ctx, (batch + 1) * kbatch * chunk)   # keys compressed by batches 0..batch
        assert covered_end >= m1                                 # every middle row is there
        assert batch * kbatch * chunk < m1                       # and the batch is the last one needed
        assert batch >= prev                                     # batches are issued in order
        prev = batch


def test_region_rule_matches_the_oracle():
    for c0 in (0, 1, 100, 128, 129, 4224, 4225, 20000):
        lo = pipeline._region_lo(c0, 128, 4096)
        _, (m0, m1), (l0, _) = oesa.regions(c0, c0 + 1, 128, 4096)
        assert l0 == lo and (m1 == lo or m1 <= m0)
