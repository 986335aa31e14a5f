"""KaLM-Reranker-V1 FBNL scoring hot path on B200: thin PyTorch binding of libkalm.

Every function here marshals torch tensors (device memory owned by the caller)
into the C ABI of ``include/kalm.h``; all arithmetic runs in the CUDA kernels of
``libkalm.so``.  Functions keep the C names.  There is no CPU fallback: without
the built library or an sm_100 device they raise ``KalmError``.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from ._abi import KalmError, call, load, library_path  # noqa: F401

__all__ = [
    "KalmError", "load", "library_path", "kalm_version", "kalm_device_check", "kalm_check_device_errors",
    "kalm_ragged_offsets", "kalm_chunk_pool", "kalm_linear", "kalm_linear_chain", "kalm_linear_chain_sync_len",
    "kalm_linear_chain_rope",
    "kalm_cross_kv_proj", "kalm_merged_attention",
    "kalm_merged_attention_out_proj", "kalm_merged_attention_out_proj_static", "kalm_attention_out_proj_sync_len",
    "kalm_yes_no_score", "kalm_broadcast_rows", "kalm_selftest_wait_timeout", "kalm_attention_items",
    "kalm_attention_schedule", "kalm_rope", "kalm_rope_table", "kalm_linear_rope",
]

HEAD_DIM = 256
MAX_QUERY_TOKENS = 512  # KALM_MAX_QUERY_TOKENS


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _p(t: Optional[torch.Tensor], dtype: Optional[torch.dtype] = None) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise KalmError(1, "binding", "tensors must live on the CUDA device")
    if dtype is not None and t.dtype != dtype:
        raise KalmError(1, "binding", f"expected {dtype}, got {t.dtype}")
    return t.data_ptr()


def _ld(t: torch.Tensor) -> int:
    """Row stride (elements) of a 2-D view whose last dimension is contiguous."""
    if t.dim() != 2 or t.stride(1) != 1:
        raise KalmError(1, "binding", "expected a 2-D tensor with contiguous rows")
    return t.stride(0)


def kalm_version() -> int:
    return load().kalm_version()


def kalm_device_check() -> None:
    call("kalm_device_check")


def kalm_check_device_errors(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise the stream and raise if a kernel recorded a device error."""
    word = ctypes.c_uint32(0)
    call("kalm_check_device_errors", _stream(stream), ctypes.byref(word))
    return word.value


def kalm_ragged_offsets(length: torch.Tensor, tok_off: Optional[torch.Tensor], pool_off: Optional[torch.Tensor],
                        chunk: int = 4, stream=None) -> None:
    call("kalm_ragged_offsets", _p(length, torch.int32), length.numel(), chunk, _p(tok_off, torch.int64),
         _p(pool_off, torch.int64), _stream(stream))


def kalm_chunk_pool(enc: torch.Tensor, tok_off: torch.Tensor, length: torch.Tensor, pooled: torch.Tensor,
                    pool_off: torch.Tensor, total_pooled: int, chunk: int = 4, stream=None) -> None:
    call("kalm_chunk_pool", _p(enc, torch.bfloat16), _ld(enc), _p(tok_off, torch.int64), _p(length, torch.int32),
         length.numel(), enc.shape[1], chunk, _p(pooled, torch.bfloat16), _ld(pooled), _p(pool_off, torch.int64),
         int(total_pooled), _stream(stream))


def kalm_linear(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor, residual: Optional[torch.Tensor] = None,
                stream=None) -> None:
    """y = x . w^T (+ residual); w is [out][in]."""
    m, k = x.shape
    n = w.shape[0]
    if w.shape[1] != k or y.shape[0] != m or y.shape[1] != n:
        raise KalmError(1, "kalm_linear", f"shapes x{tuple(x.shape)} w{tuple(w.shape)} y{tuple(y.shape)}")
    call("kalm_linear", _p(x, torch.bfloat16), _ld(x), _p(w, torch.bfloat16), _ld(w),
         _p(residual, torch.bfloat16), _ld(residual) if residual is not None else 0,
         _p(y, torch.bfloat16), _ld(y), m, n, k, _stream(stream))


def kalm_linear_chain_sync_len(m: int) -> int:
    return int(load().kalm_linear_chain_sync_len(m))


def kalm_linear_chain(x1: torch.Tensor, w1: torch.Tensor, y1: torch.Tensor, w2: torch.Tensor, y2: torch.Tensor,
                      sync: Optional[torch.Tensor], stream=None) -> None:
    """y1 = x1 . w1^T + y1 (in place), then y2 = y1 . w2^T, in one launch; ``sync`` is an
    int32 tensor of ``kalm_linear_chain_sync_len(m)`` entries, zero before the first call
    (every call leaves it zero)."""
    m, k1 = x1.shape
    n1, n2 = w1.shape[0], w2.shape[0]
    if w1.shape[1] != k1 or y1.shape != (m, n1) or w2.shape[1] != n1 or y2.shape != (m, n2):
        raise KalmError(1, "kalm_linear_chain", f"shapes x1{tuple(x1.shape)} w1{tuple(w1.shape)} y1{tuple(y1.shape)} "
                                                f"w2{tuple(w2.shape)} y2{tuple(y2.shape)}")
    call("kalm_linear_chain", _p(x1, torch.bfloat16), _ld(x1), _p(w1, torch.bfloat16), _ld(w1),
         _p(y1, torch.bfloat16), _ld(y1), _p(w2, torch.bfloat16), _ld(w2), _p(y2, torch.bfloat16), _ld(y2), m, n1, k1,
         n2, _p(sync, torch.int32), sync.numel() if sync is not None else 0, _stream(stream))


def kalm_linear_chain_rope(x1: torch.Tensor, w1: torch.Tensor, y1: torch.Tensor, w2: torch.Tensor, y2: torch.Tensor,
                           q_off: torch.Tensor, rot_heads: int, table: torch.Tensor, sync: Optional[torch.Tensor],
                           head_dim: int = HEAD_DIM, stream=None) -> None:
    """kalm_linear_chain with the first rot_heads head vectors of every row of y2 rotated
    by the row's decoder position (angles from kalm_rope_table), as kalm_linear_rope."""
    m, k1 = x1.shape
    n1, n2 = w1.shape[0], w2.shape[0]
    if w1.shape[1] != k1 or y1.shape != (m, n1) or w2.shape[1] != n1 or y2.shape != (m, n2):
        raise KalmError(1, "kalm_linear_chain_rope", f"shapes x1{tuple(x1.shape)} w1{tuple(w1.shape)} "
                                                     f"y1{tuple(y1.shape)} w2{tuple(w2.shape)} y2{tuple(y2.shape)}")
    if table.numel() != MAX_QUERY_TOKENS * head_dim or not table.is_contiguous():
        raise KalmError(1, "kalm_linear_chain_rope", "table must be a contiguous kalm_rope_table output")
    call("kalm_linear_chain_rope", _p(x1, torch.bfloat16), _ld(x1), _p(w1, torch.bfloat16), _ld(w1),
         _p(y1, torch.bfloat16), _ld(y1), _p(w2, torch.bfloat16), _ld(w2), _p(y2, torch.bfloat16), _ld(y2), m, n1, k1,
         n2, rot_heads * head_dim, head_dim, _p(q_off, torch.int64), q_off.numel() - 1, _p(table, torch.float32),
         _p(sync, torch.int32), sync.numel() if sync is not None else 0, _stream(stream))


def kalm_cross_kv_proj(pooled: torch.Tensor, w_kv: torch.Tensor, kv_cross: torch.Tensor, n_kv: int,
                       head_dim: int = HEAD_DIM, stream=None) -> None:
    """w_kv: [n_layers][2*n_kv*D][hidden]; kv_cross: [rows][n_layers*2*n_kv*D]."""
    n_layers = w_kv.shape[0]
    if not w_kv.is_contiguous() or not kv_cross.is_contiguous():
        raise KalmError(1, "kalm_cross_kv_proj", "w_kv and kv_cross must be contiguous")
    call("kalm_cross_kv_proj", _p(pooled, torch.bfloat16), _ld(pooled), pooled.shape[0], pooled.shape[1],
         _p(w_kv, torch.bfloat16), n_layers, n_kv, head_dim, _p(kv_cross, torch.bfloat16), _stream(stream))


def kalm_merged_attention(q: torch.Tensor, k_self: torch.Tensor, v_self: torch.Tensor, k_cross: torch.Tensor,
                          v_cross: torch.Tensor, q_off: torch.Tensor, pool_off: torch.Tensor, max_q: int,
                          n_q: int, n_kv: int, out: torch.Tensor, scale: Optional[float] = None,
                          lse: Optional[torch.Tensor] = None, head_dim: int = HEAD_DIM,
                          in_off: Optional[torch.Tensor] = None, last_tile_only: bool = False,
                          total_q: Optional[int] = None, order: Optional[torch.Tensor] = None, stream=None) -> None:
    """2-D row views: q/k/v self [input rows][...], out [q_off[-1] rows][>= n_q*D],
    k/v cross [pooled rows][>= n_kv*D].  ``in_off`` (optional) gives each document's
    first input row; by default it is q_off.  ``order`` (optional) is a work order
    from ``kalm_attention_schedule`` for the same offsets and sizes."""
    if scale is None:
        scale = head_dim ** -0.5
    if _ld(k_self) != _ld(v_self) or _ld(k_cross) != _ld(v_cross):
        raise KalmError(1, "kalm_merged_attention", "K and V views must share a row stride")
    n_docs = q_off.numel() - 1
    total_q = out.shape[0] if total_q is None else total_q
    call("kalm_merged_attention", _p(q, torch.bfloat16), _ld(q), _p(k_self, torch.bfloat16),
         _p(v_self, torch.bfloat16), _ld(k_self), _p(k_cross, torch.bfloat16), _p(v_cross, torch.bfloat16),
         _ld(k_cross), _p(q_off, torch.int64), _p(in_off, torch.int64), q.shape[0], _p(pool_off, torch.int64),
         n_docs, int(max_q), int(total_q), k_cross.shape[0], n_q, n_kv, head_dim, float(scale),
         1 if last_tile_only else 0, _p(order, torch.int32), _p(out, torch.bfloat16), _ld(out), _p(lse, torch.float32),
         _stream(stream))


def kalm_merged_attention_out_proj(q: torch.Tensor, k_self: torch.Tensor, v_self: torch.Tensor,
                                   k_cross: torch.Tensor, v_cross: torch.Tensor, q_off: torch.Tensor,
                                   pool_off: torch.Tensor, max_q: int, n_q: int, n_kv: int, out: torch.Tensor,
                                   w_o: torch.Tensor, x: torch.Tensor, sync: torch.Tensor,
                                   scale: Optional[float] = None, head_dim: int = HEAD_DIM,
                                   in_off: Optional[torch.Tensor] = None, total_q: Optional[int] = None,
                                   order: Optional[torch.Tensor] = None, stream=None) -> None:
    """Merged attention into ``out`` and then ``x[rows of d] += out[rows of d] . w_o^T`` for
    every document, in one launch.  ``sync``: int32 device tensor of at least
    ``kalm_attention_out_proj_sync_len(n_docs, max_q, hidden)`` entries, zero before the first call
    (every call leaves it zero)."""
    if scale is None:
        scale = head_dim ** -0.5
    if _ld(k_self) != _ld(v_self) or _ld(k_cross) != _ld(v_cross):
        raise KalmError(1, "kalm_merged_attention_out_proj", "K and V views must share a row stride")
    n_docs = q_off.numel() - 1
    total_q = out.shape[0] if total_q is None else total_q
    call("kalm_merged_attention_out_proj", _p(q, torch.bfloat16), _ld(q), _p(k_self, torch.bfloat16),
         _p(v_self, torch.bfloat16), _ld(k_self), _p(k_cross, torch.bfloat16), _p(v_cross, torch.bfloat16),
         _ld(k_cross), _p(q_off, torch.int64), _p(in_off, torch.int64), q.shape[0], _p(pool_off, torch.int64),
         n_docs, int(max_q), int(total_q), k_cross.shape[0], n_q, n_kv, head_dim, float(scale),
         _p(order, torch.int32), _p(out, torch.bfloat16), _ld(out), _p(w_o, torch.bfloat16), _ld(w_o),
         _p(x, torch.bfloat16), _ld(x), x.shape[1], _p(sync, torch.int32), sync.numel(), _stream(stream))


def kalm_merged_attention_out_proj_static(q: torch.Tensor, k_self: torch.Tensor, v_self: torch.Tensor,
                                          k_cross: torch.Tensor, v_cross: torch.Tensor, q_off: torch.Tensor,
                                          pool_off: torch.Tensor, max_q: int, n_q: int, n_kv: int,
                                          out: torch.Tensor, w_o: torch.Tensor, x: torch.Tensor,
                                          scale: Optional[float] = None, head_dim: int = HEAD_DIM,
                                          in_off: Optional[torch.Tensor] = None, total_q: Optional[int] = None,
                                          order: Optional[torch.Tensor] = None, stream=None) -> None:
    """kalm_merged_attention_out_proj with the library's built-in counters (no counter
    array from the caller): for callers that cannot allocate device memory.  At most
    KALM_OUT_PROJ_STATIC_MAX_DOCS (4096) documents and KALM_OUT_PROJ_STATIC_MAX_TILES (49152)
    projection tiles; calls that overlap on the GPU race."""
    if scale is None:
        scale = head_dim ** -0.5
    if _ld(k_self) != _ld(v_self) or _ld(k_cross) != _ld(v_cross):
        raise KalmError(1, "kalm_merged_attention_out_proj_static", "K and V views must share a row stride")
    n_docs = q_off.numel() - 1
    total_q = out.shape[0] if total_q is None else total_q
    call("kalm_merged_attention_out_proj_static", _p(q, torch.bfloat16), _ld(q), _p(k_self, torch.bfloat16),
         _p(v_self, torch.bfloat16), _ld(k_self), _p(k_cross, torch.bfloat16), _p(v_cross, torch.bfloat16),
         _ld(k_cross), _p(q_off, torch.int64), _p(in_off, torch.int64), q.shape[0], _p(pool_off, torch.int64),
         n_docs, int(max_q), int(total_q), k_cross.shape[0], n_q, n_kv, head_dim, float(scale),
         _p(order, torch.int32), _p(out, torch.bfloat16), _ld(out), _p(w_o, torch.bfloat16), _ld(w_o),
         _p(x, torch.bfloat16), _ld(x), x.shape[1], _stream(stream))


def kalm_attention_out_proj_sync_len(n_docs: int, max_q: int, hidden: int) -> int:
    """Entries of the sync array kalm_merged_attention_out_proj needs (-1 for bad sizes)."""
    return int(load().kalm_attention_out_proj_sync_len(n_docs, max_q, hidden))


def kalm_attention_items(n_docs: int, max_q: int, n_q: int, n_kv: int, last_tile_only: bool = False) -> int:
    """Work items of one kalm_merged_attention call (-1 for rejected sizes)."""
    return int(load().kalm_attention_items(n_docs, max_q, n_q, n_kv, 1 if last_tile_only else 0))


def kalm_attention_schedule(q_off: torch.Tensor, pool_off: torch.Tensor, max_q: int, n_q: int, n_kv: int,
                            order: torch.Tensor, last_tile_only: bool = False, stream=None) -> None:
    """Write a balanced work order for kalm_merged_attention into ``order`` (int32)."""
    call("kalm_attention_schedule", _p(q_off, torch.int64), _p(pool_off, torch.int64), q_off.numel() - 1, int(max_q),
         n_q, n_kv, 1 if last_tile_only else 0, _p(order, torch.int32), order.numel(), _stream(stream))


def kalm_yes_no_score(hidden: torch.Tensor, q_off: torch.Tensor, w_yes: torch.Tensor, w_no: torch.Tensor,
                      yes: torch.Tensor, no: torch.Tensor, score: torch.Tensor,
                      margin: Optional[torch.Tensor] = None, stream=None) -> None:
    call("kalm_yes_no_score", _p(hidden, torch.bfloat16), _ld(hidden), _p(q_off, torch.int64), q_off.numel() - 1,
         hidden.shape[1], _p(w_yes, torch.bfloat16), _p(w_no, torch.bfloat16), _p(yes, torch.float32),
         _p(no, torch.float32), _p(margin, torch.float32), _p(score, torch.float32), _stream(stream))


def kalm_broadcast_rows(src: torch.Tensor, q_off: torch.Tensor, dst: torch.Tensor, stream=None) -> None:
    call("kalm_broadcast_rows", _p(src, torch.bfloat16), _ld(src), src.shape[0], src.shape[1],
         _p(q_off, torch.int64), q_off.numel() - 1, _p(dst, torch.bfloat16), _ld(dst), _stream(stream))


def kalm_rope(x: torch.Tensor, q_off: torch.Tensor, n_heads: int, theta: float, head_dim: int = HEAD_DIM,
              stream=None) -> None:
    """Rotate the first n_heads head vectors of every row of x in place by the row's
    decoder position (row - q_off[d] for the document d owning the row)."""
    call("kalm_rope", _p(x, torch.bfloat16), _ld(x), x.shape[0], n_heads, head_dim, _p(q_off, torch.int64),
         q_off.numel() - 1, float(theta), _stream(stream))


def kalm_rope_table(theta: float, head_dim: int = HEAD_DIM, stream=None) -> torch.Tensor:
    """(cos, sin) of every rotary angle: float32 [head_dim/4][KALM_MAX_QUERY_TOKENS][4],
    entry [q][pos] = (cos, sin) of pair 2q then of pair 2q + 1."""
    table = torch.empty(head_dim // 4, MAX_QUERY_TOKENS, 4, dtype=torch.float32, device="cuda")
    call("kalm_rope_table", float(theta), head_dim, _p(table, torch.float32), _stream(stream))
    return table


def kalm_linear_rope(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor, q_off: torch.Tensor, rot_heads: int,
                     table: torch.Tensor, head_dim: int = HEAD_DIM, stream=None) -> None:
    """y = x . w^T with the first rot_heads head vectors of every row rotated by the
    row's decoder position, in the projection's epilogue (angles from kalm_rope_table)."""
    m, k = x.shape
    n = w.shape[0]
    if w.shape[1] != k or y.shape[0] != m or y.shape[1] != n:
        raise KalmError(1, "kalm_linear_rope", f"shapes x{tuple(x.shape)} w{tuple(w.shape)} y{tuple(y.shape)}")
    if table.numel() != MAX_QUERY_TOKENS * head_dim or not table.is_contiguous():
        raise KalmError(1, "kalm_linear_rope", "table must be a contiguous kalm_rope_table output")
    call("kalm_linear_rope", _p(x, torch.bfloat16), _ld(x), _p(w, torch.bfloat16), _ld(w), _p(y, torch.bfloat16),
         _ld(y), m, n, k, rot_heads * head_dim, head_dim, _p(q_off, torch.int64), q_off.numel() - 1,
         _p(table, torch.float32), _stream(stream))


def kalm_selftest_wait_timeout(wait_ns: int, stream=None) -> None:
    call("kalm_selftest_wait_timeout", int(wait_ns), _stream(stream))
