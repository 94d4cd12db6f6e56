"""Host drivers of the hot path: ESA chunked prefill, ESA decode, MoBA prefill.

ESA write-up, implementation paragraph: key and value are cached chunk by chunk;
each chunk's queries select the important middle tokens (all queries of the chunk
count), and in decoding the single current query does. These classes hold the
caller-side state (compressed key cache, index buffers, workspaces, outputs) and
issue the C-ABI calls in order on the current stream. They allocate everything up
front, so a step launches kernels only and can be captured in a CUDA graph
(``graph_of``), which replays the whole step with one launch.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import _abi


def graph_of(fn):
    """Capture fn() into a CUDA graph. fn runs once eagerly first, on a side stream,
    so that every one-time host setting (kernel attributes, cluster sizes) is made
    outside the capture. The graph holds the kernels with the pointers fn used; replay
    it only while those buffers stay alive and in place."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    # captured on a high-priority stream: the work fn issues on the current stream (the
    # attention of a pipelined prefill) goes ahead of what it forks to low-priority
    # side streams (see _side_stream) when both wait for free SMs
    with torch.cuda.graph(g, stream=torch.cuda.Stream(priority=torch.cuda.Stream.priority_range()[1])):
        fn()
    return g


def _side_stream(device) -> torch.cuda.Stream:
    """A lowest-priority stream for work that runs beside the main stream's."""
    return torch.cuda.Stream(device=device, priority=torch.cuda.Stream.priority_range()[0])


def _timing_event(external: bool):
    # external: a record node when captured in a graph (readable after each replay)
    return torch.cuda.Event(enable_timing=True, external=external) if external else \
        torch.cuda.Event(enable_timing=True)


def _region_lo(c0: int, n_init: int, window: int) -> int:
    return min(c0, max(n_init, c0 - window))


def key_batch_needed(c0: int, chunk: int, n_init: int, window: int, kbatch: int) -> int:
    """The last batch of kbatch consecutive chunks whose compressed keys the selection of
    the chunk starting at c0 reads (its middle is [n_init, lo), lo <= c0), or -1 when
    its middle is empty."""
    lo = _region_lo(c0, n_init, window)
    if lo <= n_init:
        return -1
    return ((lo - 1) // chunk) // kbatch


def block_diagonal(w_groups: torch.Tensor) -> torch.Tensor:
    """Per-head selection: the groups' maps [G, gin, d_g] stacked into the one
    [G * gin, G * d_g] map the compression calls take (zero off the diagonal
    blocks), so that group g's compressed columns see group g's heads only."""
    return torch.block_diag(*w_groups.unbind(0)).contiguous()


class _Compressor:
    """The two compression maps of a layer (queries: Hq heads in; keys: Hkv heads in,
    expanded to Hq). With bf16 inputs and a shape the packed path takes, the weights
    are packed once per pack() call (fold + bf16 high/low split, esa_compress_pack)
    and every map runs esa_compress_packed; otherwise esa_compress reads the fp32
    weights directly."""

    def __init__(self, hq: int, hkv: int, head_dim: int, d_c: int, dtype, device):
        self.hq, self.hkv, self.d, self.d_c = hq, hkv, head_dim, d_c
        nq = _abi.compress_pack_size(hq, head_dim, d_c) if dtype == torch.bfloat16 else 0
        nk = _abi.compress_pack_size(hkv, head_dim, d_c) if dtype == torch.bfloat16 else 0
        self.packed = bool(nq and nk)
        if self.packed:
            self.wq_p = torch.empty(nq, dtype=torch.uint8, device=device)
            self.wk_p = torch.empty(nk, dtype=torch.uint8, device=device)
        self.key = None
        self.wq = self.wk = None

    def pack(self, wq, wk):
        self.wq, self.wk = wq, wk
        if self.packed:
            _abi.compress_pack(wq, self.hq, self.hq, self.d, out=self.wq_p)
            _abi.compress_pack(wk, self.hkv, self.hq, self.d, out=self.wk_p)
        self.key = (wq.data_ptr(), wq._version, wk.data_ptr(), wk._version)

    def pack_keys(self, wk):
        """Key map only (filling a cache); the next pack_if_changed packs both."""
        self.wk = wk
        if self.packed:
            _abi.compress_pack(wk, self.hkv, self.hq, self.d, out=self.wk_p)
        self.key = None

    def pack_if_changed(self, wq, wk):
        if self.key != (wq.data_ptr(), wq._version, wk.data_ptr(), wk._version):
            self.pack(wq, wk)

    def queries(self, x, out, out_row_stride=None):
        if self.packed:
            return _abi.compress_packed(x, self.wq_p, self.d_c, out=out, out_row_stride=out_row_stride)
        return _abi.compress(x, self.wq, self.hq, out=out, out_row_stride=out_row_stride)

    def keys(self, x, out, out_row_stride=None):
        if self.packed:
            return _abi.compress_packed(x, self.wk_p, self.d_c, out=out, out_row_stride=out_row_stride)
        return _abi.compress(x, self.wk, self.hq, out=out, out_row_stride=out_row_stride)


class EsaPrefill:
    """Chunked prefill of one attention layer: for every chunk [c0, c0 + chunk),
    compress the chunk's keys into the compressed cache, compress its queries,
    select middle tokens, attend over initial + selected + local."""

    def __init__(self, batch: int, n_ctx: int, chunk: int, hq: int, hkv: int, head_dim: int, d_c: int,
                 p: _abi.EsaParams, dtype=torch.bfloat16, device="cuda", per_head: bool = False,
                 key_chunks: int = 2):
        self.batch, self.n_ctx, self.chunk = batch, n_ctx, chunk
        self.key_chunks = key_chunks      # chunks whose keys run() compresses in one launch
        self.hq, self.hkv, self.d, self.d_c, self.p = hq, hkv, head_dim, d_c, p
        self.per_head = per_head      # one selection per KV head (block-diagonal maps)
        lists = (batch, hkv) if per_head else (batch,)
        self.device = torch.device(device)
        self.k_c = torch.zeros((batch, n_ctx, d_c), dtype=torch.float32, device=device)
        self.q_c = torch.empty((batch, chunk, d_c), dtype=torch.float32, device=device)
        # one index list (set) per chunk: chunk j + 1's selection may run while chunk j
        # attends, and a chunk's selection stays readable after run()
        n_chunks = (n_ctx + chunk - 1) // chunk
        self.idx_all = torch.empty((n_chunks, *lists, p.topk), dtype=torch.int32, device=device)
        self.count_all = torch.empty((n_chunks, *lists), dtype=torch.int32, device=device)
        self.out = torch.empty((batch, n_ctx, hq, head_dim), dtype=dtype, device=device)
        code = _abi.ESA_BF16 if dtype == torch.bfloat16 else _abi.ESA_F32
        if per_head:
            ws_sel = max(_abi.score_select_heads_workspace_size(batch, min(chunk, n_ctx - c0), n_ctx, c0, d_c, hkv, p)
                         for c0 in range(0, n_ctx, chunk))
            ws_att = max(_abi.sparse_attn_heads_workspace_size(batch, min(chunk, n_ctx - c0), c0, hq, hkv, head_dim,
                                                               code, p)
                         for c0 in range(0, n_ctx, chunk))
        else:
            ws_sel = max(_abi.score_select_workspace_size(batch, min(chunk, n_ctx - c0), n_ctx, c0, d_c, p)
                         for c0 in range(0, n_ctx, chunk))
            ws_att = max(_abi.sparse_attn_workspace_size(batch, min(chunk, n_ctx - c0), c0, hq, hkv, head_dim, code,
                                                         p)
                         for c0 in range(0, n_ctx, chunk))
        self.ws_sel = torch.empty(ws_sel + 256, dtype=torch.uint8, device=device)
        self.ws_att = torch.empty(ws_att + 256, dtype=torch.uint8, device=device) if ws_att else None
        self.out_views = []
        self.cmp = _Compressor(hq, hkv, head_dim, d_c, dtype, device)
        self.side = _side_stream(device)
        self.kside = _side_stream(device)

    def chunks(self):
        return [(c0, min(self.chunk, self.n_ctx - c0)) for c0 in range(0, self.n_ctx, self.chunk)]

    def compress_keys(self, c0: int, lq: int, k):
        """Chunk [c0, c0 + lq)'s keys into the compressed cache. A chunk's scoring reads
        only positions before c0 (the middle ends at most at c0), so these rows are
        first needed by a later chunk."""
        for s in range(self.batch):
            self.cmp.keys(k[s, c0:c0 + lq], out=self.k_c[s, c0:c0 + lq])

    def front(self, ci: int, c0: int, lq: int, q, k=None):
        """Chunk ci's work before its attention, on the current stream: (its keys, if k
        is given,) its queries, and the selection into the chunk's index list."""
        b = self.batch
        if k is not None:
            self.compress_keys(c0, lq, k)
        for s in range(b):
            self.cmp.queries(q[s, c0:c0 + lq], out=self.q_c[s, :lq])
        q_c = self.q_c[:, :lq] if lq == self.chunk else self.q_c[:, :lq].contiguous()
        if self.per_head:
            _abi.score_select_heads(q_c, self.k_c, c0, self.hkv, self.p, idx=self.idx_all[ci],
                                    count=self.count_all[ci], workspace=self.ws_sel)
        else:
            _abi.score_select(q_c, self.k_c, c0, self.p, idx=self.idx_all[ci], count=self.count_all[ci],
                              workspace=self.ws_sel)

    def attend(self, ci: int, c0: int, lq: int, q, k, v, attn_events=None):
        """Chunk ci's attention over initial + its selected + local tokens."""
        qv = q[:, c0:c0 + lq]
        if not qv.is_contiguous():
            qv = qv.contiguous()
        ov = self.out[:, c0:c0 + lq]
        target = ov if ov.is_contiguous() else torch.empty_like(ov)
        if attn_events is not None:
            attn_events[0].record()
        attn = _abi.sparse_attn_heads if self.per_head else _abi.sparse_attn
        attn(qv, k, v, c0, self.idx_all[ci], self.count_all[ci], self.p, out=target, workspace=self.ws_att)
        if attn_events is not None:
            attn_events[1].record()
        if target is not ov:
            ov.copy_(target)

    def run_chunk(self, c0: int, lq: int, q, k, v, wq, wk, attn_events=None):
        """One chunk, in order on the current stream (the chunks must come in order)."""
        self.cmp.pack_if_changed(wq, wk)
        ci = c0 // self.chunk
        self.front(ci, c0, lq, q, k)
        self.attend(ci, c0, lq, q, k, v, attn_events)

    def run(self, q, k, v, wq, wk, attn_events=None, external_events=False, chunk_ready=None,
            on_attended=None):
        """q [B, N, Hq, D], k, v [B, N, Hkv, D] (device), wq, wk [Hq*D, d'].
        attn_events: optional list that receives one (start, end) CUDA event pair per
        attention launch (external_events: made to be captured in a graph). Returns
        the output [B, N, Hq, D]. The weights are packed for the tensor-core
        compression at the start of every run.
        chunk_ready: optional per-chunk CUDA events; work that reads chunk j's rows of
        q, k, v (and so every later chunk's) waits for event j, so the rows may still be
        arriving when run() is called. on_attended(ci, c0, lq): called after chunk ci's
        attention is issued (on the current stream), e.g. to copy its output out.

        Three streams: the chunks' key compressions run in order on one, their query
        compression and selection in order on another (chunk j's selection waiting for
        the keys of chunks < j only), and each chunk's attention on the current stream
        once its selection is done, so chunk j + 1's selection overlaps chunk j's
        attention and no chunk's selection waits for its own keys."""
        main = torch.cuda.current_stream()
        self.cmp.pack(wq, wk)
        self.side.wait_stream(main)
        self.kside.wait_stream(main)
        chunks = self.chunks()
        # keys are compressed in batches of up to kbatch chunks (fewer, larger launches
        # beside the attention); chunk j's selection waits for the batch holding the
        # last chunk its middle reads (positions < lo <= c0)
        kbatch = max(1, self.key_chunks)
        n_batches = (len(chunks) + kbatch - 1) // kbatch
        issued = 0                                  # batches issued so far, in order
        last_done = None                            # event after the last issued batch

        def issue_batches(upto):                    # batches [issued, upto] on the key stream
            nonlocal issued, last_done
            while issued <= upto:
                b0, b1 = issued * kbatch, min(len(chunks), (issued + 1) * kbatch)
                if chunk_ready is not None:
                    self.kside.wait_event(chunk_ready[b1 - 1])
                with torch.cuda.stream(self.kside):
                    self.compress_keys(chunks[b0][0], chunks[b1 - 1][0] + chunks[b1 - 1][1] - chunks[b0][0], k)
                    last_done = torch.cuda.Event()
                    last_done.record()
                issued += 1

        for ci, (c0, lq) in enumerate(chunks):
            needed = key_batch_needed(c0, self.chunk, self.p.n_init, self.p.window, kbatch)
            wait = None
            if needed >= 0:
                issue_batches(needed)
                wait = last_done
            done = torch.cuda.Event()
            with torch.cuda.stream(self.side):
                if wait is not None:
                    self.side.wait_event(wait)
                if chunk_ready is not None:
                    self.side.wait_event(chunk_ready[ci])
                self.front(ci, c0, lq, q)
                done.record()
            main.wait_event(done)                  # (after chunk_ready[ci]: the rows up to c1 are in)
            ev = None
            if attn_events is not None:
                ev = (_timing_event(external_events), _timing_event(external_events))
                attn_events.append(ev)
            self.attend(ci, c0, lq, q, k, v, ev)
            if on_attended is not None:
                on_attended(ci, c0, lq)
        issue_batches(n_batches - 1)               # the rest complete the compressed cache
        main.wait_stream(self.side)
        main.wait_stream(self.kside)
        return self.out


    def run_from_host(self, q_host, k_host, v_host, q, k, v, wq, wk, out_host):
        """The prefill with its inputs in pinned host memory and its output returned to
        pinned host memory, the copies overlapping the compute: chunk by chunk, the
        chunk's rows of q, k, v go up on one copy stream (one copy per tensor and chunk)
        and each chunk's output comes back on another as soon as its attention is done.
        q_host, k_host, v_host: pinned host tensors shaped like the device buffers q, k,
        v, which receive them; out_host: pinned host tensor like the output. Works for
        batch 1 (a chunk's rows are then contiguous). Returns out_host; the copies are
        complete once the current stream reaches this point."""
        if self.batch != 1:
            raise ValueError("run_from_host streams chunks of one sequence (batch 1)")
        main = torch.cuda.current_stream()
        cin, cout = self._copy_streams()
        cin.wait_stream(main)
        cout.wait_stream(main)
        ready = []
        with torch.cuda.stream(cin):
            for c0, lq in self.chunks():
                for dev, host in ((q, q_host), (k, k_host), (v, v_host)):
                    dev[:, c0:c0 + lq].copy_(host[:, c0:c0 + lq], non_blocking=True)
                e = torch.cuda.Event()
                e.record()
                ready.append(e)

        def copy_out(ci, c0, lq):
            e = torch.cuda.Event()
            e.record()
            cout.wait_event(e)
            with torch.cuda.stream(cout):
                out_host[:, c0:c0 + lq].copy_(self.out[:, c0:c0 + lq], non_blocking=True)

        self.run(q, k, v, wq, wk, chunk_ready=ready, on_attended=copy_out)
        main.wait_stream(cin)
        main.wait_stream(cout)
        return out_host

    def _copy_streams(self):
        if not hasattr(self, "_cin"):
            self._cin = torch.cuda.Stream(device=self.device)
            self._cout = torch.cuda.Stream(device=self.device)
        return self._cin, self._cout


class EsaDecode:
    """One decode step for a batch: compress the new query and the new key (written
    into the compressed cache), select over the middle, attend. The KV cache holds
    n_ctx tokens; the query sits at position n_ctx - 1."""

    def __init__(self, batch: int, n_ctx: int, hq: int, hkv: int, head_dim: int, d_c: int, p: _abi.EsaParams,
                 dtype=torch.bfloat16, device="cuda", per_head: bool = False):
        self.batch, self.n_ctx, self.hq, self.hkv, self.d, self.d_c, self.p = batch, n_ctx, hq, hkv, head_dim, d_c, p
        # per_head: one selection per KV head (the compression maps given to step() are
        # then block-diagonal, see block_diagonal)
        self.per_head = per_head
        lists = (batch, hkv) if per_head else (batch,)
        self.k_c = torch.zeros((batch, n_ctx, d_c), dtype=torch.float32, device=device)
        self.q_c = torch.empty((batch, 1, d_c), dtype=torch.float32, device=device)
        self.idx = torch.empty((*lists, p.topk), dtype=torch.int32, device=device)
        self.count = torch.empty(lists, dtype=torch.int32, device=device)
        self.out = torch.empty((batch, 1, hq, head_dim), dtype=dtype, device=device)
        code = _abi.ESA_BF16 if dtype == torch.bfloat16 else _abi.ESA_F32
        c0 = n_ctx - 1
        if per_head:
            n_sel = _abi.score_select_heads_workspace_size(batch, 1, n_ctx, c0, d_c, hkv, p)
            nb = _abi.sparse_attn_heads_workspace_size(batch, 1, c0, hq, hkv, head_dim, code, p)
        else:
            n_sel = _abi.score_select_workspace_size(batch, 1, n_ctx, c0, d_c, p)
            nb = _abi.sparse_attn_workspace_size(batch, 1, c0, hq, hkv, head_dim, code, p)
        self.ws_sel = torch.empty(n_sel + 256, dtype=torch.uint8, device=device)
        self.ws_att = torch.empty(nb + 256, dtype=torch.uint8, device=device) if nb else None
        self.cmp = _Compressor(hq, hkv, head_dim, d_c, dtype, device)
        self.side = _side_stream(device)

    def fill_cache(self, k, wk, upto: Optional[int] = None):
        """Compress cached keys [0, upto) of every sequence (prefill state)."""
        upto = self.n_ctx - 1 if upto is None else upto
        self.cmp.pack_keys(wk)
        step = 1 << 16
        for s in range(self.batch):
            for r0 in range(0, upto, step):
                r1 = min(upto, r0 + step)
                self.cmp.keys(k[s, r0:r1], out=self.k_c[s, r0:r1])

    def step(self, q, k, v, wq, wk, phase_events=None):
        """q [B, 1, Hq, D]; k, v [B, n_ctx, Hkv, D] with the new token at n_ctx - 1.
        The packed weights are reused across steps while wq and wk are the same tensors,
        unmodified (pointer and version counter); otherwise they are packed again."""
        pos = self.n_ctx - 1
        ev = phase_events
        cur = torch.cuda.current_stream()
        if ev is not None:
            ev[0].record()
        self.cmp.pack_if_changed(wq, wk)
        # The new token is in the local window, so this step's scoring never reads its
        # compressed key: that compression runs beside the query's on a second stream.
        self.side.wait_stream(cur)
        with torch.cuda.stream(self.side):
            self.cmp.keys(k[:, pos], out=self.k_c[:, pos], out_row_stride=self.n_ctx * self.d_c)
        self.cmp.queries(q[:, 0], out=self.q_c.view(self.batch, self.d_c))
        if ev is not None:
            ev[1].record()
        if self.per_head:
            _abi.score_select_heads(self.q_c, self.k_c, pos, self.hkv, self.p, idx=self.idx, count=self.count,
                                    workspace=self.ws_sel)
        else:
            _abi.score_select(self.q_c, self.k_c, pos, self.p, idx=self.idx, count=self.count,
                              workspace=self.ws_sel)
        if ev is not None:
            ev[2].record()
        attn = _abi.sparse_attn_heads if self.per_head else _abi.sparse_attn
        attn(q, k, v, pos, self.idx, self.count, self.p, out=self.out, workspace=self.ws_att)
        cur.wait_stream(self.side)
        if ev is not None:
            ev[3].record()
        return self.out


class EsaDecodeVarlen:
    """One decode step for a batch of sequences of different lengths. Sequence b holds
    seq_len[b] tokens (a device int64 tensor, so a captured step replays with new
    lengths) in caches of n_cap rows, its query at position seq_len[b] - 1; its new
    key row (already appended to the KV cache by the caller) is compressed into row
    seq_len[b] - 1 of the compressed cache. Needs the packed compression path (bf16,
    d_c 128)."""

    def __init__(self, batch: int, n_cap: int, hq: int, hkv: int, head_dim: int, d_c: int, p: _abi.EsaParams,
                 dtype=torch.bfloat16, device="cuda", per_head: bool = False):
        self.batch, self.n_cap, self.hq, self.hkv, self.d, self.d_c, self.p = batch, n_cap, hq, hkv, head_dim, d_c, p
        self.per_head = per_head
        self.ng = hkv if per_head else 1
        self.cmp = _Compressor(hq, hkv, head_dim, d_c, dtype, device)
        if not self.cmp.packed:
            raise ValueError("variable-length decode needs the packed compression path (bf16, d_c 128)")
        self.k_c = torch.zeros((batch, n_cap, d_c), dtype=torch.float32, device=device)
        self.q_c = torch.empty((batch, 1, d_c), dtype=torch.float32, device=device)
        self.idx = torch.empty((batch, self.ng, p.topk), dtype=torch.int32, device=device)
        self.count = torch.empty((batch, self.ng), dtype=torch.int32, device=device)
        self.out = torch.empty((batch, 1, hq, head_dim), dtype=dtype, device=device)
        code = _abi.ESA_BF16 if dtype == torch.bfloat16 else _abi.ESA_F32
        n_sel = _abi.score_select_varlen_workspace_size(batch, n_cap, d_c, self.ng, p)
        nb = _abi.sparse_attn_varlen_workspace_size(batch, n_cap, hq, hkv, head_dim, code, self.ng, p)
        self.ws_sel = torch.empty(n_sel + 256, dtype=torch.uint8, device=device)
        self.ws_att = torch.empty(nb + 256, dtype=torch.uint8, device=device) if nb else None
        self.side = _side_stream(device)

    def fill_cache(self, k, wk, lengths):
        """Compress cached keys [0, lengths[b] - 1) of every sequence (prefill state);
        lengths: host integers."""
        self.cmp.pack_keys(wk)
        step = 1 << 16
        for s in range(self.batch):
            upto = int(lengths[s]) - 1
            for r0 in range(0, upto, step):
                r1 = min(upto, r0 + step)
                self.cmp.keys(k[s, r0:r1], out=self.k_c[s, r0:r1])

    def step(self, q, k_new, k, v, wq, wk, seq_len):
        """q [B, 1, Hq, D]; k_new [B, Hkv, D] the new key rows (also at row seq_len[b] - 1
        of k); k, v [B, n_cap, Hkv, D]; seq_len [B] int64 on the device."""
        cur = torch.cuda.current_stream()
        self.cmp.pack_if_changed(wq, wk)
        # the new token is local to its own query: its compressed key is not read this step
        self.side.wait_stream(cur)
        with torch.cuda.stream(self.side):
            _abi.compress_packed_varlen(k_new, self.cmp.wk_p, self.k_c, seq_len)
        self.cmp.queries(q[:, 0], out=self.q_c.view(self.batch, self.d_c))
        _abi.score_select_varlen(self.q_c, self.k_c, seq_len, self.p, n_groups=self.ng, idx=self.idx,
                                 count=self.count, workspace=self.ws_sel)
        _abi.sparse_attn_varlen(q, k, v, seq_len, self.idx, self.count, self.p, out=self.out,
                                workspace=self.ws_att)
        cur.wait_stream(self.side)
        return self.out


class MobaPrefill:
    """MoBA causal prefill of one layer: gate, then block attention."""

    def __init__(self, batch: int, seq: int, heads: int, head_dim: int, block: int, topk: int,
                 dtype=torch.bfloat16, device="cuda"):
        self.batch, self.seq, self.heads, self.d, self.block, self.topk = batch, seq, heads, head_dim, block, topk
        self.out = torch.empty((batch, seq, heads, head_dim), dtype=dtype, device=device)
        self.blocks = torch.empty((batch, seq, heads, topk + 1), dtype=torch.int16, device=device)
        self.ws = torch.empty(_abi.moba_workspace_size(2, batch, seq, heads, head_dim, block, topk) + 256,
                              dtype=torch.uint8, device=device)

    def run(self, q, k, v):
        _abi.moba_block_gate_attn(q, k, v, self.block, self.topk, out=self.out, blocks=self.blocks,
                                  want_blocks=True, workspace=self.ws)
        return self.out


class MobaDecode:
    """MoBA decode for a batch at position n_ctx - 1: the block means of the cache's
    complete blocks are computed once by fill() (a decode loop adds one block's mean
    each time a block fills), every step gates over them and attends."""

    def __init__(self, batch: int, n_ctx: int, heads: int, head_dim: int, block: int, topk: int,
                 dtype=torch.bfloat16, device="cuda"):
        self.batch, self.n_ctx, self.heads, self.d, self.block, self.topk = batch, n_ctx, heads, head_dim, block, topk
        nb = (n_ctx + block - 1) // block
        self.kbar = torch.zeros((batch, heads, nb, head_dim), dtype=torch.float32, device=device)
        self.out = torch.empty((batch, 1, heads, head_dim), dtype=dtype, device=device)
        self.blocks = torch.empty((batch, heads, topk + 1), dtype=torch.int16, device=device)
        pos = n_ctx - 1
        self.ws = torch.empty(_abi.moba_decode_workspace_size(batch, n_ctx, pos, heads, head_dim, block, topk) + 256,
                              dtype=torch.uint8, device=device)

    def fill(self, k):
        """Means of the blocks before the query's block."""
        _abi.moba_block_means(k, self.block, 0, (self.n_ctx - 1) // self.block, out=self.kbar)

    def step(self, q, k, v):
        _abi.moba_decode_attn(q, k, v, self.n_ctx - 1, self.kbar, self.block, self.topk, out=self.out,
                              blocks=self.blocks, want_blocks=True, workspace=self.ws)
        return self.out

