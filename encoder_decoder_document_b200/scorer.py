"""One query against a ragged batch of documents: the four scoring steps chained.

``FBNLScorer`` owns the decoder weights (device, bf16) and reusable device
buffers, and runs, on one stream:

  kalm_ragged_offsets -> kalm_chunk_pool (document cache) -> kalm_cross_kv_proj
  (all layers at once) -> kalm_broadcast_rows (the query's decoder input for
  every document) -> per layer: kalm_linear (Q | K_self | V_self),
  kalm_merged_attention, kalm_linear (output projection + residual) ->
  kalm_yes_no_score.

Python only sequences the calls and owns the buffers; every step runs in the
CUDA kernels of libkalm.  ``capture()`` records the whole sequence in a CUDA
graph so a query costs one graph launch.  ``rerank()`` is the user-facing call:
host inputs in, the best-first list out ("KaLM-Reranker-V1-Nano - MLX",
"Usage": rerank returns {index, relevance_score} entries, highest first;
"KaLM-Reranker-V1-Small-Q4_K_M-GGUF", "Score a pair": larger margins rank first).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from . import (kalm_broadcast_rows, kalm_check_device_errors, kalm_chunk_pool, kalm_cross_kv_proj,
               kalm_device_check, kalm_linear, kalm_merged_attention_out_proj, kalm_attention_out_proj_sync_len,
               kalm_merged_attention, kalm_ragged_offsets, kalm_yes_no_score, kalm_attention_items,
               kalm_attention_schedule, kalm_linear_rope, kalm_rope_table, kalm_linear_chain,
               kalm_linear_chain_rope, kalm_linear_chain_sync_len)

HEAD_DIM = 256
# the pages' runtime limits ("Runtime boundaries"): passages of at most 1,024 encoder
# tokens, a query budget of 512 tokens
MAX_DOC_TOKENS = 1024
MAX_QUERY_TOKENS = 512


def bf16_from_bits(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns (host) -> bf16 device tensor (bit-exact)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


@dataclasses.dataclass
class DeviceWeights:
    w_qkv: torch.Tensor       # [L][(n_q + 2 n_kv) D][H]
    w_o: torch.Tensor         # [L][H][n_q D]
    w_kv_cross: torch.Tensor  # [L][2 n_kv D][H]
    w_yes: torch.Tensor       # [H]
    w_no: torch.Tensor        # [H]

    @classmethod
    def from_bits(cls, w, device="cuda") -> "DeviceWeights":
        return cls(bf16_from_bits(w.w_qkv, device), bf16_from_bits(w.w_o, device),
                   bf16_from_bits(w.w_kv_cross, device), bf16_from_bits(w.w_yes, device),
                   bf16_from_bits(w.w_no, device))


class FBNLScorer:
    """Scores one query's documents.  With ``prune`` (the default) work that
    cannot reach the score is skipped, exactly: the first layer's Q/K/V are
    computed once for the query's common decoder input (every document starts
    from it), and the last layer computes attention only for the query tile that
    holds each document's final row and the output projection only for that row
    (the readout reads nothing else)."""

    def __init__(self, weights: DeviceWeights, n_q: int, n_kv: int, chunk: int = 4, head_dim: int = HEAD_DIM,
                 prune: bool = True, rope_theta: Optional[float] = None, fused_out: bool = False,
                 chain: bool = True):
        kalm_device_check()
        self.w = weights
        self.L, qkv_rows, self.H = weights.w_qkv.shape
        self.n_q, self.n_kv, self.D, self.chunk = n_q, n_kv, head_dim, chunk
        assert qkv_rows == (n_q + 2 * n_kv) * head_dim
        self.scale = head_dim ** -0.5
        self.prune = prune
        self.rope_theta = rope_theta  # rotary base for the decoder's self Q/K, or None (no rotation)
        # attention and output projection of every layer but the pruned last one in one
        # launch (kalm_merged_attention_out_proj)
        self.fused_out = fused_out
        # each layer's output projection and the next layer's Q|K|V projection in one launch
        # (kalm_linear_chain, or kalm_linear_chain_rope with rotation), in the pruned stack
        # without the fused layer
        self.chain = chain and prune and not fused_out
        self._qkv_ready = -1  # layer whose Q|K|V the last chained launch produced
        # the rotary angles' (cos, sin), built once for this base
        self.rope_tab = kalm_rope_table(rope_theta, head_dim) if rope_theta is not None else None
        self._shape = None
        self.graph: Optional[torch.cuda.CUDAGraph] = None
        self.graphs = None
        self.graphs_decode = None
        # optional per-launch timing: (label, event) recorded after every entry-point call
        self.marks: Optional[list] = None
        self.launches = 0  # kernel launches issued by the last forward()
        self.side: Optional[torch.cuda.Stream] = None  # second stream for work beside the pooling
        self._side_pending = False  # the broadcast of X is on the second stream, not yet joined

    # ------------------------------------------------------------------ buffers
    def prepare(self, n_docs: int, total_tokens: int, total_pooled: int, lq: int, device="cuda") -> None:
        """Allocate the device buffers for one query shape (re-used across calls)."""
        shape = (n_docs, total_tokens, total_pooled, lq)
        if self._shape == shape:
            return
        self._shape = shape
        self.graph = None
        D, H, L = self.D, self.H, self.L
        rows = n_docs * lq
        kw = dict(device=device)
        self.n_docs, self.total_tokens, self.total_pooled, self.lq = shape
        # two input slots, so the next query's inputs can be copied while this one runs
        self.slots = [dict(enc=torch.empty(max(total_tokens, 1), H, dtype=torch.bfloat16, **kw),
                           doc_len=torch.empty(n_docs, dtype=torch.int32, **kw),
                           x0=torch.empty(lq, H, dtype=torch.bfloat16, **kw)) for _ in range(2)]
        self.use_slot(0)
        self.tok_off = torch.empty(n_docs + 1, dtype=torch.int64, **kw)
        self.pool_off = torch.empty(n_docs + 1, dtype=torch.int64, **kw)
        # every document of a query has the query's Lq decoder rows, so their offsets belong
        # to the shape and are fixed here once (document d's rows start at d * Lq)
        self.q_off = torch.arange(n_docs + 1, dtype=torch.int64, **kw) * lq
        self.zero_off = torch.zeros(n_docs, dtype=torch.int64, **kw)
        self.one_doc_off = torch.tensor([0, lq], dtype=torch.int64, **kw)  # the query's common rows
        self.pooled = torch.empty(max(total_pooled, 1), H, dtype=torch.bfloat16, **kw)
        self.kv_cross = torch.empty(max(total_pooled, 1), L * 2 * self.n_kv * D, dtype=torch.bfloat16, **kw)
        self.qkv = torch.empty(rows, (self.n_q + 2 * self.n_kv) * D, dtype=torch.bfloat16, **kw)
        self.o = torch.empty(rows, self.n_q * D, dtype=torch.bfloat16, **kw)
        self.x = torch.empty(rows, H, dtype=torch.bfloat16, **kw)
        # (yes, no, margin, score) rows of one buffer: one device->host copy per query
        self.result = torch.empty(4, n_docs, dtype=torch.float32, **kw)
        # work order of the full-layer attention launches (same costs in every layer)
        self.order = torch.empty(max(kalm_attention_items(n_docs, lq, self.n_q, self.n_kv), 1), dtype=torch.int32,
                                 **kw)
        self.yes, self.no, self.margin, self.score = self.result[0], self.result[1], self.result[2], self.result[3]
        # the fused layer's per-document counters (zero before a launch, left zero by it)
        self.sync = torch.zeros(max(kalm_attention_out_proj_sync_len(n_docs, lq, H), 1), dtype=torch.int32, **kw)
        # the chained projections' per-row-block counters (zero before a launch, left zero by it)
        self.chain_sync = torch.zeros(max(kalm_linear_chain_sync_len(rows), 1), dtype=torch.int32, **kw)
        self.graphs = None
        self.graphs_decode = None

    def use_slot(self, i: int) -> None:
        """Point the input buffers at slot i (for the next forward() or capture)."""
        self.slot = i
        self.enc, self.doc_len, self.x0 = (self.slots[i][k] for k in ("enc", "doc_len", "x0"))

    # ------------------------------------------------------------------ steps
    def _mark(self, label: str) -> None:
        self.launches += 1
        if self.marks is not None:
            ev = torch.cuda.Event(enable_timing=True, external=True)
            ev.record()
            self.marks.append((label, ev))

    def pool(self, side: Optional[torch.cuda.Stream] = None) -> None:
        """Offsets, attention work order, pooled document cache.  With a ``side`` stream
        the work order and the query input broadcast (both need only the offsets) run
        there, beside the pooling and the cross projection; the caller joins it."""
        kalm_ragged_offsets(self.doc_len, self.tok_off, self.pool_off, self.chunk)
        self._mark("offsets")
        if side is not None:
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                kalm_attention_schedule(self.q_off, self.pool_off, self.lq, self.n_q, self.n_kv, self.order)
                kalm_broadcast_rows(self.x0, self.q_off, self.x)
            self.launches += 2
        else:
            kalm_attention_schedule(self.q_off, self.pool_off, self.lq, self.n_q, self.n_kv, self.order)
            self._mark("schedule")
        kalm_chunk_pool(self.enc, self.tok_off, self.doc_len, self.pooled, self.pool_off, self.total_pooled,
                        self.chunk)
        self._mark("chunk_pool")

    def cross_kv(self) -> None:
        kalm_cross_kv_proj(self.pooled[: self.total_pooled], self.w.w_kv_cross, self.kv_cross[: self.total_pooled],
                           self.n_kv, self.D)
        self._mark("cross_kv_proj")

    def cross_views(self, l: int):
        w = self.n_kv * self.D
        kc = self.kv_cross[:, (2 * l) * w:(2 * l + 1) * w]
        vc = self.kv_cross[:, (2 * l + 1) * w:(2 * l + 2) * w]
        return kc, vc

    def qkv_views(self):
        D, nq, nkv = self.D, self.n_q, self.n_kv
        return (self.qkv[:, : nq * D], self.qkv[:, nq * D:(nq + nkv) * D], self.qkv[:, (nq + nkv) * D:])

    def qkv_proj(self, x: torch.Tensor, l: int, qkv: torch.Tensor, q_off: torch.Tensor) -> None:
        """Fused Q|K|V projection; with a rotary base the self Q and K heads are
        rotated in the projection's epilogue."""
        if self.rope_theta is None:
            kalm_linear(x, self.w.w_qkv[l], qkv)
        else:
            kalm_linear_rope(x, self.w.w_qkv[l], qkv, q_off, self.n_q + self.n_kv, self.rope_tab, self.D)
        self._mark("qkv_proj")

    def layer_qkv(self, l: int) -> None:
        self.qkv_proj(self.x, l, self.qkv, self.q_off)

    def layer_attention(self, l: int) -> None:
        q, ks, vs = self.qkv_views()
        kc, vc = self.cross_views(l)
        kalm_merged_attention(q, ks, vs, kc, vc, self.q_off, self.pool_off, self.lq, self.n_q, self.n_kv, self.o,
                              self.scale, order=self.order)
        self._mark("merged_attention")

    def _join_side(self) -> None:
        """The residual stream X is first read by an output projection: wait for the
        broadcast if it was issued on the second stream."""
        if self._side_pending:
            torch.cuda.current_stream().wait_stream(self.side)
            self._side_pending = False

    def layer_out(self, l: int) -> None:
        self._join_side()
        kalm_linear(self.o, self.w.w_o[l], self.x, residual=self.x)
        self._mark("o_proj")

    def attention_out(self, l: int, q, ks, vs, in_off=None) -> None:
        """Fused attention + output projection of layer l (X updated in place)."""
        kc, vc = self.cross_views(l)
        self._join_side()
        kalm_merged_attention_out_proj(q, ks, vs, kc, vc, self.q_off, self.pool_off, self.lq, self.n_q, self.n_kv,
                                       self.o, self.w.w_o[l], self.x, self.sync, self.scale, in_off=in_off,
                                       order=self.order)
        self._mark("attention_out_proj")

    def layer(self, l: int) -> None:
        self.layer_qkv(l)
        if self.fused_out:
            q, ks, vs = self.qkv_views()
            self.attention_out(l, q, ks, vs)
            return
        self.layer_attention(l)
        self.layer_out(l)

    def layer_pruned(self, l: int) -> None:
        """Layer l with the exact pruning described in the class docstring."""
        first, last = l == 0, l == self.L - 1
        Lq = self.lq
        kc, vc = self.cross_views(l)
        if first:
            # every document's decoder input is the query's common input: one Q|K|V for all
            self.qkv_proj(self.x0, l, self.qkv[:Lq], self.one_doc_off)
            q, ks, vs = (t[:Lq] for t in self.qkv_views())
            in_off = self.zero_off
        else:
            if not (self.chain and self._qkv_ready == l):  # else the previous launch projected them
                self.layer_qkv(l)
            q, ks, vs = self.qkv_views()
            in_off = None
        if self.fused_out and not last:
            self.attention_out(l, q, ks, vs, in_off)
            return
        kalm_merged_attention(q, ks, vs, kc, vc, self.q_off, self.pool_off, Lq, self.n_q, self.n_kv, self.o,
                              self.scale, in_off=in_off, last_tile_only=last, order=None if last else self.order)
        self._mark("merged_attention")
        if last:
            # only each document's final row reaches the readout
            x_last = self.x[Lq - 1::Lq]
            self._join_side()
            kalm_linear(self.o[Lq - 1::Lq], self.w.w_o[l], x_last, residual=x_last)
            self._mark("o_proj")
        elif self.chain:
            # X += O Wo, then the next layer's Q|K|V from the updated X, in one launch
            self._join_side()
            if self.rope_theta is None:
                kalm_linear_chain(self.o, self.w.w_o[l], self.x, self.w.w_qkv[l + 1], self.qkv, self.chain_sync)
            else:
                kalm_linear_chain_rope(self.o, self.w.w_o[l], self.x, self.w.w_qkv[l + 1], self.qkv, self.q_off,
                                       self.n_q + self.n_kv, self.rope_tab, self.chain_sync, self.D)
            self._mark("o_proj_qkv")
            self._qkv_ready = l + 1
        else:
            self.layer_out(l)

    def readout(self) -> None:
        kalm_yes_no_score(self.x, self.q_off, self.w.w_yes, self.w.w_no, self.yes, self.no, self.score,
                          self.margin)
        self._mark("yes_no_score")

    def documents(self) -> None:
        """The document side: offsets, the pooled document cache and every layer's cross K/V."""
        self.pool()
        self.cross_kv()

    def decode(self, broadcast: bool = True) -> None:
        """The query side: the decoder stack over the cached cross K/V, then the readout."""
        self._qkv_ready = -1
        if broadcast and self.marks is None and self.prune:
            # layer 0's Q|K|V and attention read only the query input: the broadcast of X
            # runs beside them and the first output projection waits for it
            if self.side is None:
                self.side = torch.cuda.Stream()
            self.side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(self.side):
                kalm_broadcast_rows(self.x0, self.q_off, self.x)
            self.launches += 1
            self._side_pending = True
        elif broadcast:
            kalm_broadcast_rows(self.x0, self.q_off, self.x)
            self._mark("broadcast")
        for l in range(self.L):
            if self.prune:
                self.layer_pruned(l)
            else:
                self.layer(l)
        self.readout()

    def forward(self, cached: bool = False) -> None:
        """All steps on the current stream, from the inputs in self.enc / doc_len / x0.

        With ``cached`` only decode() runs: the documents' offsets, work order and
        cross K/V from the last full forward over the same documents are reused
        (the persistent-cache regime: one document set, many queries)."""
        self.launches = 0
        if self.marks is not None:
            self._mark("start")
            self.launches = 0
        if cached:
            self.decode()
        elif self.marks is None:
            # the work order and the broadcast beside the pooling and cross projection
            if self.side is None:
                self.side = torch.cuda.Stream()
            self.pool(side=self.side)
            self.cross_kv()
            torch.cuda.current_stream().wait_stream(self.side)
            self.decode(broadcast=False)
        else:  # instrumented: one launch after another, so each gets its own interval
            self.documents()
            self.decode()

    def capture(self, instrument: bool = False) -> None:
        """Record forward() as a CUDA graph (buffers must stay allocated).

        With ``instrument`` a second graph is recorded with an external timing
        event after every launch (``graph_inst``), so each of its replays yields
        per-kernel durations (``kernel_times()``).  The events sit between the
        launches and keep them from overlapping, so the plain graph is the one to
        time a step with."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.forward()  # warm-up: one-time device set-up happens outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.marks = None
        slot = self.slot
        self.graphs = []
        for i in range(2):  # one graph per input slot
            self.use_slot(i)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.forward()
            self.graphs.append(g)
        self.graphs_decode = []
        for i in range(2):  # decode-only graphs (persistent-cache regime), one per input slot
            self.use_slot(i)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.forward(cached=True)
            self.graphs_decode.append(g)
        self.use_slot(slot)
        self.graph = self.graphs[slot]
        self.graph_inst = None
        if instrument:
            self.marks = []
            gi = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gi):
                self.forward()
            self.graph_inst = gi

    def kernel_times(self) -> dict:
        """{label: [ms per launch, ...]} of the last replay of the instrumented graph."""
        out: dict = {}
        if not self.marks:
            return out
        for (_, a), (label, b) in zip(self.marks[:-1], self.marks[1:]):
            out.setdefault(label, []).append(a.elapsed_time(b))
        return out

    def run(self) -> None:
        if self.graph is not None:
            self.graph.replay()
        else:
            self.forward()

    # ------------------------------------------------------------------ user API
    def load_inputs(self, enc_host: torch.Tensor, doc_len_host: torch.Tensor, x0_host: torch.Tensor) -> None:
        """Host -> device copies of one query's inputs (pinned host tensors copy asynchronously)."""
        self.enc[: enc_host.shape[0]].copy_(enc_host, non_blocking=True)
        self.doc_len.copy_(doc_len_host, non_blocking=True)
        self.x0.copy_(x0_host, non_blocking=True)

    def scores_to_host(self, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Device -> host copy of (yes, no, margin, score) as a [4][n_docs] fp32 tensor."""
        if out is None:
            return self.result.cpu()
        out.copy_(self.result, non_blocking=True)
        return out

    def score_stream(self, inputs, outs) -> None:
        """Score a stream of queries of this shape, overlapping transfers with compute.

        inputs[k] = (enc, doc_len, x0) pinned host tensors of query k; outs[k] a
        pinned [4][n_docs] fp32 host tensor that receives (yes, no, margin, score).
        Query k+1's inputs are copied on a side stream into the other input slot
        while query k runs (one captured graph per slot); every copy and every
        result read happen inside the call, which returns without synchronising.
        Device errors (an expired bounded wait, invalid device data) are only
        flagged on the device: call ``check_errors()`` before trusting ``outs``.
        Requires capture() first."""
        if self.graphs is None:
            raise RuntimeError("score_stream needs capture() first")
        comp = torch.cuda.current_stream()
        if getattr(self, "_copy_stream", None) is None:
            self._copy_stream = torch.cuda.Stream()
            self._ready = [torch.cuda.Event(), torch.cuda.Event()]
            self._free = [torch.cuda.Event(), torch.cuda.Event()]
        cs = self._copy_stream
        cs.wait_stream(comp)

        def h2d(k):
            i = k % 2
            slot = self.slots[i]
            with torch.cuda.stream(cs):
                if k >= 2:
                    cs.wait_event(self._free[i])  # the query that last used this slot is done with it
                enc, doc_len, x0 = inputs[k]
                slot["enc"][: enc.shape[0]].copy_(enc, non_blocking=True)
                slot["doc_len"].copy_(doc_len, non_blocking=True)
                slot["x0"].copy_(x0, non_blocking=True)
                self._ready[i].record(cs)

        if inputs:
            h2d(0)
        for k in range(len(inputs)):
            if k + 1 < len(inputs):
                h2d(k + 1)
            i = k % 2
            comp.wait_event(self._ready[i])
            self.graphs[i].replay()
            self._free[i].record(comp)
            outs[k].copy_(self.result, non_blocking=True)

    def cache_documents(self, enc_host: torch.Tensor, doc_len_host: torch.Tensor) -> None:
        """Build the document cache (pooled vectors and every layer's cross K/V) for a
        document set that many queries will be scored against; stream-ordered.  Both
        input slots share the cache, so score_cached_stream can use either."""
        for slot in self.slots:
            slot["enc"][: enc_host.shape[0]].copy_(enc_host, non_blocking=True)
            slot["doc_len"].copy_(doc_len_host, non_blocking=True)
        self.documents()

    def score_cached_stream(self, x0s, outs) -> None:
        """Score queries against the cached documents (decode-only graphs), overlapping
        each query's decoder-input copy with the previous query's compute.

        x0s[k]: pinned host bf16 [lq][H] decoder input of query k; outs[k]: pinned
        [4][n_docs] fp32 host tensor for (yes, no, margin, score).  Returns without
        synchronising; call ``check_errors()`` before trusting ``outs``.  Requires
        cache_documents() (or a full forward over the same documents) and capture()."""
        if not getattr(self, "graphs_decode", None):
            raise RuntimeError("score_cached_stream needs capture() first")
        comp = torch.cuda.current_stream()
        if getattr(self, "_copy_stream", None) is None:
            self._copy_stream = torch.cuda.Stream()
            self._ready = [torch.cuda.Event(), torch.cuda.Event()]
            self._free = [torch.cuda.Event(), torch.cuda.Event()]
        cs = self._copy_stream
        cs.wait_stream(comp)

        def h2d(k):
            i = k % 2
            with torch.cuda.stream(cs):
                if k >= 2:
                    cs.wait_event(self._free[i])
                self.slots[i]["x0"].copy_(x0s[k], non_blocking=True)
                self._ready[i].record(cs)

        if x0s:
            h2d(0)
        for k in range(len(x0s)):
            if k + 1 < len(x0s):
                h2d(k + 1)
            i = k % 2
            comp.wait_event(self._ready[i])
            self.graphs_decode[i].replay()
            self._free[i].record(comp)
            outs[k].copy_(self.result, non_blocking=True)

    def rerank(self, x0: np.ndarray, enc: np.ndarray, doc_len: np.ndarray, top_n: Optional[int] = None):
        """Score one query's documents and return [{index, relevance_score}] best first.

        x0: bf16 bits [lq][H] (decoder input of the query); enc: bf16 bits
        [sum(doc_len)][H] (packed encoder states); doc_len: int [n_docs]."""
        res = self.score_rows(x0, enc, doc_len)
        return rank(res[:, 2], res[:, 3], top_n)

    def rerank_sharded(self, x0: np.ndarray, enc: np.ndarray, doc_len: np.ndarray, top_n: Optional[int] = None,
                       group=None):
        """``rerank`` over the documents of one query split across the ranks of a
        process group (one process per GPU, each with its own scorer): every rank
        passes the whole query, scores its share of the documents (balanced by
        length) and receives the full ranking.  The only exchange is one gather of the
        per-document scores on the host."""
        from .sharding import sharded_rerank
        return sharded_rerank(self.score_rows, x0, enc, doc_len, top_n, group)

    def score_rows(self, x0: np.ndarray, enc: np.ndarray, doc_len: np.ndarray) -> np.ndarray:
        """Rows (yes, no, margin, score) of one query's documents, in input order
        (``[n_docs][4]`` float32 on the host); arguments as for ``rerank``."""
        doc_len = np.asarray(doc_len)
        if doc_len.ndim != 1:
            raise ValueError("rerank: doc_len must be one length per document")
        if doc_len.size and (doc_len.min() < 0 or doc_len.max() > MAX_DOC_TOKENS):
            raise ValueError(f"rerank: document lengths must lie in [0, {MAX_DOC_TOKENS}] "
                             f"(got {int(doc_len.min())}..{int(doc_len.max())})")
        lq = int(np.asarray(x0).shape[0])
        if not 1 <= lq <= MAX_QUERY_TOKENS:
            raise ValueError(f"rerank: the query input must have 1..{MAX_QUERY_TOKENS} rows (got {lq})")
        doc_len = doc_len.astype(np.int32)
        n = int(doc_len.shape[0])
        if n == 0:
            return np.zeros((0, 4), dtype=np.float32)
        total_tokens = int(doc_len.sum())
        if np.asarray(enc).shape[0] < total_tokens:
            raise ValueError(f"rerank: enc holds {np.asarray(enc).shape[0]} rows, doc_len sums to {total_tokens}")
        total_pooled = int(((doc_len.astype(np.int64) + self.chunk - 1) // self.chunk).sum())
        self.prepare(n, total_tokens, total_pooled, lq)
        self.load_inputs(torch.from_numpy(np.ascontiguousarray(enc).view(np.int16)).view(torch.bfloat16),
                         torch.from_numpy(doc_len), torch.from_numpy(np.ascontiguousarray(x0).view(np.int16))
                         .view(torch.bfloat16))
        self.run()
        res = self.scores_to_host().numpy()
        # a bounded wait that expired or invalid device data leaves only a flag on the
        # device: raise instead of returning scores computed past it
        self.check_errors()
        return np.ascontiguousarray(res.T)

    def check_errors(self) -> None:
        """Wait for this scorer's streams and raise ``KalmError`` if a kernel recorded a
        device error (a bounded wait that expired, or invalid device data) since the
        last check.  ``score_stream`` and ``score_cached_stream`` return without waiting;
        call this once their results are needed."""
        if self.side is not None:
            torch.cuda.current_stream().wait_stream(self.side)
        if getattr(self, "_copy_stream", None) is not None:
            torch.cuda.current_stream().wait_stream(self._copy_stream)
        kalm_check_device_errors()


def rank(margin: np.ndarray, score: np.ndarray, top_n: Optional[int] = None):
    """Best-first order: larger margin first, ties broken by the lower index."""
    order = sorted(range(len(margin)), key=lambda i: (-float(margin[i]), i))
    if top_n is not None:
        order = order[:top_n]
    return [{"index": i, "relevance_score": float(score[i])} for i in order]
