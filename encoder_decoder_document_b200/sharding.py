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
from typing import List, Sequence

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
    width = () if first is None else np.asarray(first).shape[1:]
    out = np.full((n_docs,) + tuple(width), np.nan)
    for idx, p in zip(shards, parts):
        out[np.asarray(idx, dtype=np.int64)] = p
    return out
