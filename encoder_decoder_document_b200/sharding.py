"""Splitting one query's documents across GPUs (one process per GPU).

Documents are independent on this path: a document's score depends only on the
query's decoder input, the weights and its own pooled vectors.  So a batch
shards by documents with no exchange on the data path; the only collective is
the final gather of the per-document scores, in input order ("KaLM-Reranker-V1-
Large-Q8_0-GGUF", "JSONL scoring": results preserve input order).

Assignment: longest-processing-time-first greedy on an estimated cost per
document, ``base + len`` (a fixed share for the decoder projections, which do
not depend on the document, plus a share that grows with its encoder length).
"""
from __future__ import annotations

import heapq
from typing import Callable, List, Optional, Sequence, Tuple

import numpy as np


def shard_documents(doc_len: Sequence[int], world: int, base: float = 512.0) -> List[np.ndarray]:
    """Return, for each rank, the sorted indices of the documents it scores."""
    if world < 1:
        raise ValueError("world must be >= 1")
    lens = np.asarray(doc_len, dtype=np.int64)
    order = sorted(range(len(lens)), key=lambda i: (-(base + lens[i]), i))
    heap = [(0.0, r) for r in range(world)]
    out: List[list] = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        out[r].append(i)
        heapq.heappush(heap, (load + base + float(lens[i]), r))
    return [np.array(sorted(s), dtype=np.int64) for s in out]


def merge_scores(shards: Sequence[np.ndarray], parts: Sequence[np.ndarray], n_docs: int) -> np.ndarray:
    """Put each rank's per-document rows (``parts[r][k]`` belongs to document
    ``shards[r][k]``) back into input order."""
    first = next((p for p in parts if len(p)), None)
    if first is None:  # no rows at all: keep the row shape the (empty) parts carry
        first = next((p for p in parts if np.asarray(p).ndim > 1), np.zeros(0))
    width = np.asarray(first).shape[1:]
    out = np.full((n_docs,) + tuple(width), np.nan)
    for idx, p in zip(shards, parts):
        out[np.asarray(idx, dtype=np.int64)] = p
    return out


def slice_documents(enc: np.ndarray, doc_len: Sequence[int], idx: Sequence[int]) -> Tuple[np.ndarray, np.ndarray]:
    """The packed encoder rows and the lengths of documents ``idx`` (in that order)
    of a batch packed row after row (``enc[sum(doc_len)][H]``)."""
    lens = np.asarray(doc_len, dtype=np.int64)
    off = np.zeros(len(lens) + 1, dtype=np.int64)
    np.cumsum(lens, out=off[1:])
    idx = np.asarray(idx, dtype=np.int64)
    rows = [enc[off[i]:off[i + 1]] for i in idx]
    local = np.concatenate(rows, axis=0) if rows else enc[:0]
    return np.ascontiguousarray(local), lens[idx].astype(np.int32)


def _rank_and_world(group) -> Tuple[int, int]:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def sharded_scores(score_fn: Callable[[np.ndarray, np.ndarray, np.ndarray], np.ndarray], x0: np.ndarray,
                   enc: np.ndarray, doc_len: Sequence[int], group=None, base: float = 512.0) -> np.ndarray:
    """Per-document rows of one query (``[n_docs][k]``, input order) from every rank
    of ``group`` (the default process group; without one, this process alone).

    Every rank passes the same query (``x0``, ``enc``, ``doc_len``); each scores the
    documents ``shard_documents`` gives it with ``score_fn(x0, enc_local, len_local)``
    (for instance ``FBNLScorer.score_rows`` on that rank's GPU), and one host gather of
    the small per-document rows brings them back together.  Every rank takes part
    in the gather even when its own scoring fails, and then every rank raises, so a
    failure on one rank never leaves the others waiting in a collective."""
    rank, world = _rank_and_world(group)
    lens = np.asarray(doc_len, dtype=np.int64)
    shards = shard_documents(lens, world, base)
    try:
        enc_l, len_l = slice_documents(enc, lens, shards[rank])
        rows = np.asarray(score_fn(x0, enc_l, len_l)) if len(len_l) else np.zeros((0, 4), dtype=np.float32)
        local = (True, rows)
        if local[1].shape[0] != len(len_l):
            local = (False, f"rank {rank}: score_fn returned {local[1].shape[0]} rows for {len(len_l)} documents")
    except Exception as e:  # reported on every rank after the gather
        local = (False, f"rank {rank}: {type(e).__name__}: {e}")
    if world == 1:
        parts = [local]
    else:
        import torch.distributed as dist
        parts = [None] * world
        dist.all_gather_object(parts, local, group=group)
    failed = [msg for ok, msg in parts if not ok]
    if failed:
        raise RuntimeError("sharded scoring failed: " + "; ".join(failed))
    return merge_scores(shards, [p for _, p in parts], len(lens))


def sharded_rerank(score_fn: Callable[[np.ndarray, np.ndarray, np.ndarray], np.ndarray], x0: np.ndarray,
                   enc: np.ndarray, doc_len: Sequence[int], top_n: Optional[int] = None, group=None):
    """``[{index, relevance_score}]`` best first over all ranks' documents (the same
    list on every rank); ``score_fn`` returns rows (yes, no, margin, score)."""
    from .scorer import rank as rank_order
    res = sharded_scores(score_fn, x0, enc, doc_len, group)
    return rank_order(res[:, 2], res[:, 3], top_n)
