"""Seeded synthetic inputs for the KaLM-Reranker-V1 FBNL scoring path.

This module is shared by the fp64 oracle tests and by the CUDA path.  It holds
none of the method's arithmetic: it only draws document lengths, encoder
states, decoder states and weights from seeded generators and stores them as
bf16 bit patterns (uint16), the storage type of the path.

Workload shapes follow the five published configurations of the scoring path
(Tiny, Nano, Small, Large, and the Nano-shaped throughput sweep):

* encoder states N(0, 1), one row of ``hidden`` values per encoder token, packed
  document after document (no padding rows);
* the decoder input ``x0`` N(0, 1), ``[lq][hidden]``, shared by all documents of a
  query (the decoder reads the same instruction + query for every passage);
* per layer, independent N(0, 0.02) weights in the ``[out][in]`` (K-contiguous)
  layout: ``w_qkv [(n_q + 2 n_kv) * D][hidden]`` (q heads, then the self K head(s),
  then the self V head(s)), ``w_o [hidden][n_q * D]``, and the cross projection
  ``w_kv_cross [2 * n_kv * D][hidden]`` (cross K head(s), then cross V head(s));
* two readout rows ``w_yes``, ``w_no`` N(0, 0.02) standing in for the LM-head rows
  of the "yes" and "no" tokens.

Every array comes from its own child stream of ``SeedSequence([seed, tag, ...])``
so that any single piece (one layer's weights, one document) can be regenerated
without drawing the rest.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

# Limits fixed by the pages' runtime contract: encoder input of at most 1,024
# tokens per passage and a query budget of 512 tokens (KaLM-Reranker-V1-Small
# Q4_K_M GGUF card, "Runtime boundaries").
MAX_DOC_TOKENS = 1024
MAX_QUERY_TOKENS = 512
HEAD_DIM = 256

# name -> shape description.  "len" is the document-length law, "lq" the
# decoder length law.
CONFIGS = {
    "tiny": dict(n_docs=4, hidden=640, len=("uniform", 1, 64), lq=("fixed", 32),
                 n_q=4, n_kv=1, layers=1, seed=0),
    "nano": dict(n_docs=100, hidden=640, len=("uniform", 64, 1024), lq=("fixed", 128),
                 n_q=4, n_kv=1, layers=18, seed=1),
    "small": dict(n_docs=100, hidden=1152, len=("uniform", 64, 1024), lq=("uniform", 128, 512),
                  n_q=4, n_kv=1, layers=26, seed=2),
    "large": dict(n_docs=100, hidden=2560, len=("lognormal", 300.0, 0.6, 16, 1024),
                  lq=("fixed", 256), n_q=8, n_kv=4, layers=34, seed=3),
    # Nano-shaped throughput sweep: one query per draw, docs-per-query chosen
    # from SWEEP_DOCS; the seed of query i is 4 + i.
    "sweep": dict(n_docs=100, hidden=640, len=("lognormal", 200.0, 0.6, 1, 1024),
                  lq=("uniform", 32, 512), n_q=4, n_kv=1, layers=18, seed=4),
}
SWEEP_DOCS = (1, 16, 100, 1024, 4096)

WEIGHT_STD = 0.02

_TAG_LEN, _TAG_LQ, _TAG_ENC, _TAG_X0, _TAG_QKV, _TAG_O, _TAG_KVC, _TAG_READ = range(8)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bits.

    Inputs here are finite by construction (draws from normal laws)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, *tags: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *tags])))


def _normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def draw_lengths(law, n: int, rng: np.random.Generator) -> np.ndarray:
    kind = law[0]
    if kind == "fixed":
        return np.full(n, law[1], dtype=np.int32)
    if kind == "uniform":
        return rng.integers(law[1], law[2], size=n, endpoint=True).astype(np.int32)
    if kind == "lognormal":
        median, sigma, lo, hi = law[1:]
        v = np.exp(rng.normal(np.log(median), sigma, size=n))
        return np.clip(np.rint(v), lo, hi).astype(np.int32)
    raise ValueError(f"unknown length law {law!r}")


@dataclasses.dataclass
class Weights:
    """Decoder weights of one query's synthetic stack (bf16 bits)."""
    w_qkv: np.ndarray       # [layers][(n_q + 2 n_kv) D][hidden]
    w_o: np.ndarray         # [layers][hidden][n_q D]
    w_kv_cross: np.ndarray  # [layers][2 n_kv D][hidden]
    w_yes: np.ndarray       # [hidden]
    w_no: np.ndarray        # [hidden]


@dataclasses.dataclass
class Query:
    """One query with its ragged document batch (bf16 bits, packed rows)."""
    name: str
    hidden: int
    n_q: int
    n_kv: int
    head_dim: int
    layers: int
    doc_len: np.ndarray     # int32 [n_docs], encoder tokens per document
    tok_off: np.ndarray     # int64 [n_docs + 1], first encoder row of each document
    enc: np.ndarray         # uint16 [sum(doc_len)][hidden]
    lq: int                 # decoder length (shared by every document of the query)
    x0: np.ndarray          # uint16 [lq][hidden]
    weights: Optional[Weights]

    @property
    def n_docs(self) -> int:
        return int(self.doc_len.shape[0])


def make_weights(seed: int, hidden: int, n_q: int, n_kv: int, layers: int,
                 head_dim: int = HEAD_DIM) -> Weights:
    D = head_dim
    w_qkv = np.empty((layers, (n_q + 2 * n_kv) * D, hidden), np.uint16)
    w_o = np.empty((layers, hidden, n_q * D), np.uint16)
    w_kv = np.empty((layers, 2 * n_kv * D, hidden), np.uint16)
    for l in range(layers):
        w_qkv[l] = _normal_bf16(_rng(seed, _TAG_QKV, l), w_qkv.shape[1:], WEIGHT_STD)
        w_o[l] = _normal_bf16(_rng(seed, _TAG_O, l), w_o.shape[1:], WEIGHT_STD)
        w_kv[l] = _normal_bf16(_rng(seed, _TAG_KVC, l), w_kv.shape[1:], WEIGHT_STD)
    rr = _rng(seed, _TAG_READ)
    w_yes = _normal_bf16(rr, (hidden,), WEIGHT_STD)
    w_no = _normal_bf16(rr, (hidden,), WEIGHT_STD)
    return Weights(w_qkv, w_o, w_kv, w_yes, w_no)


def make_query(name: str = "tiny", *, n_docs: Optional[int] = None, seed: Optional[int] = None,
               layers: Optional[int] = None, with_weights: bool = True,
               doc_len: Optional[np.ndarray] = None, lq: Optional[int] = None,
               hidden: Optional[int] = None, n_q: Optional[int] = None,
               n_kv: Optional[int] = None) -> Query:
    """Draw one query of configuration ``name``.

    Keyword overrides exist for tests (edge cases and reduced sizes); the
    published configurations use none of them, except ``n_docs`` and ``seed``
    for the throughput sweep."""
    cfg = dict(CONFIGS[name])
    seed = cfg["seed"] if seed is None else seed
    n = cfg["n_docs"] if n_docs is None else n_docs
    H = cfg["hidden"] if hidden is None else hidden
    L = cfg["layers"] if layers is None else layers
    nq = cfg["n_q"] if n_q is None else n_q
    nkv = cfg["n_kv"] if n_kv is None else n_kv
    if doc_len is None:
        doc_len = draw_lengths(cfg["len"], n, _rng(seed, _TAG_LEN))
    doc_len = np.asarray(doc_len, dtype=np.int32)
    if lq is None:
        lq = int(draw_lengths(cfg["lq"], 1, _rng(seed, _TAG_LQ))[0])
    tok_off = np.zeros(doc_len.shape[0] + 1, np.int64)
    np.cumsum(doc_len, out=tok_off[1:])
    enc = _normal_bf16(_rng(seed, _TAG_ENC), (int(tok_off[-1]), H), 1.0)
    x0 = _normal_bf16(_rng(seed, _TAG_X0), (lq, H), 1.0)
    w = make_weights(seed, H, nq, nkv, L) if with_weights else None
    return Query(name, H, nq, nkv, HEAD_DIM, L, doc_len, tok_off, enc, lq, x0, w)


def describe() -> str:
    """One-line recipe of the synthetic inputs, for logs and bench output."""
    return ("PCG64 child streams of SeedSequence([seed, tag, ...]); encoder states and x0 N(0,1), "
            "weights N(0,0.02), all rounded to bf16; lengths: uniform or log-normal(median, sigma=0.6) "
            "rounded and clipped, per configuration")
