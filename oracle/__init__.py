"""CPU oracle for query-aware top-k selective attention (ESA and MoBA forms).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA library never
calls it, and it never calls the CUDA library: the two share no code, headers,
helpers or constants. Both receive their inputs from
``query_aware_selective_b200.synthetic``.

Everything here is plain numpy in float64: slow, literal, and written so that it
can be checked against the pages by eye.

* ``oracle.esa``  - Efficient Selective Attention ("Efficient Selective Attention"
  article, implementation section): compression, importance score, score
  correction, chunk sum, neighbour influence, top-k, attention over
  initial + selected + local tokens.
* ``oracle.esa_heads`` - the per-head selection variant of ESA (the article's
  ablation of merged versus per-head importance): one index set per KV head.
* ``oracle.esa_varlen`` - ESA decode over a batch of sequences of different
  lengths: each sequence runs the one-sequence step at its own position.
* ``oracle.esa_fit`` - the offline least-squares fit of ESA's two compression maps
  from calibration queries and keys.
* ``oracle.cca`` - CCA-style attention: core tokens pooled per group of g tokens by
  the group's last query, plus a group-aligned local window, in one softmax.
* ``oracle.moba`` - Mixture of Block Attention (MoBA article, sections 1-3):
  block mean pooling, gate, causal top-k, block attention.

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
closed forms, library routines (torch SDPA in float64), brute force on tiny
inputs, hand-worked examples and invariants. Parity that the pages cannot fix
(the clamp constant C, the region boundary, MoBA's off-by-one) is stated as a
reading in the docstrings of the functions concerned.
"""
