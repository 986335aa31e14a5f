"""Plain fp64 definitions of the four scoring steps (test infrastructure only).

Every function works on float64 arrays whose values are bf16-representable
where the path stores bf16, and returns float64 arrays (rounded to bf16 where
the path stores bf16).  Nothing is tiled, fused or reordered.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

# ----------------------------------------------------------------------------
# bf16 storage rounding
# ----------------------------------------------------------------------------
# bf16 keeps 8 significant bits (1 implicit + 7 stored) with float32's
# exponent range: normal numbers down to 2^-126, subnormals spaced 2^-133,
# largest finite value (2 - 2^-7) * 2^127.
_BF16_MIN_NORMAL = 2.0 ** -126
_BF16_SUB_STEP = 2.0 ** -133
_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def bf16_round(x) -> np.ndarray:
    """Round fp64 values once to the nearest bf16 value (ties to even).

    Implemented from the definition: for |x| in the normal range the spacing of
    bf16 values around x is 2^(e-7) with e = floor(log2|x|); x / spacing is
    rounded to an integer with numpy's rint (ties to even) and scaled back.
    Below 2^-126 the spacing is the fixed subnormal step 2^-133.  A result
    above the largest finite bf16 becomes +-inf (what round-to-nearest gives
    once the rounded magnitude reaches 2^128).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    a = np.abs(x)
    fin = np.isfinite(x) & (a > 0)
    normal = fin & (a >= _BF16_MIN_NORMAL)
    sub = fin & (a < _BF16_MIN_NORMAL)
    if np.any(normal):
        _, e = np.frexp(a[normal])          # a = m * 2^e with m in [0.5, 1)
        step = np.ldexp(1.0, e - 8)         # 8 significant bits
        out[normal] = np.sign(x[normal]) * np.rint(a[normal] / step) * step
    if np.any(sub):
        out[sub] = np.sign(x[sub]) * np.rint(a[sub] / _BF16_SUB_STEP) * _BF16_SUB_STEP
    big = np.abs(out) > _BF16_MAX
    out[big] = np.sign(out[big]) * np.inf
    return out


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Decode bf16 bit patterns (uint16) to float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Encode values that are already bf16-representable as uint16 bits."""
    r = bf16_round(x)
    f = r.astype(np.float32)  # exact: r has at most 8 significant bits
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ----------------------------------------------------------------------------
# Step 1: chunk pooling into the document cache
# ----------------------------------------------------------------------------
def pooled_counts(doc_len, chunk: int = 4) -> np.ndarray:
    """Pooled vectors per document: ceil(len / chunk).

    Reading: the mask is a prefix of ``len`` valid tokens (right padding,
    "Frozen inference contract"); groups start at token 0; a group with no
    valid token is not emitted."""
    doc_len = np.asarray(doc_len, dtype=np.int64)
    return (doc_len + chunk - 1) // chunk


def chunk_pool(enc: np.ndarray, tok_off: Sequence[int], doc_len: Sequence[int],
               chunk: int = 4, round_out: bool = True):
    """Masked mean over consecutive groups of ``chunk`` valid tokens.

    "KaLM-Reranker-V1-Nano - MLX", "What this is" (chunk size 4, masked mean per
    chunk) and "KaLM-Reranker-V1-Large-Q8_0-GGUF", "Frozen inference contract"
    (masked mean pooling over consecutive groups of 4 tokens, right padding).

    ``enc`` holds one row per encoder token; document d owns rows
    ``tok_off[d] .. tok_off[d] + doc_len[d] - 1``.  Reading of the partial last
    group: it is averaged over its valid tokens only (a masked mean divides by
    the number of unmasked entries).

    Returns ``(pooled, pool_off)``: pooled rows of all documents packed in
    document order, and the exclusive prefix sum of the per-document counts.
    """
    enc = np.asarray(enc, dtype=np.float64)
    doc_len = np.asarray(doc_len, dtype=np.int64)
    counts = pooled_counts(doc_len, chunk)
    pool_off = np.zeros(len(doc_len) + 1, dtype=np.int64)
    np.cumsum(counts, out=pool_off[1:])
    H = enc.shape[1]
    pooled = np.zeros((int(pool_off[-1]), H), dtype=np.float64)
    for d in range(len(doc_len)):
        base = int(tok_off[d])
        n = int(doc_len[d])
        for c in range(int(counts[d])):
            lo = c * chunk
            hi = min(lo + chunk, n)
            pooled[pool_off[d] + c] = enc[base + lo: base + hi].sum(axis=0) / (hi - lo)
    if round_out:
        pooled = bf16_round(pooled)
    return pooled, pool_off


# ----------------------------------------------------------------------------
# Step 2 (and the decoder projections): dense products
# ----------------------------------------------------------------------------
def linear(x: np.ndarray, w: np.ndarray, residual: Optional[np.ndarray] = None,
           round_out: bool = True) -> np.ndarray:
    """y = x . w^T (+ residual), weights stored ``[out][in]``.

    Used for the cross K/V projection of the cached pooled vectors ("What this
    is": cross-attention KV computed over the cached passage encodings) and for
    the synthetic decoder's Q/K/V and output projections.  Reading: no bias, no
    norm and no rotary embedding on the cross K/V (the pages name none).
    The residual is added before the single rounding to bf16."""
    y = np.asarray(x, np.float64) @ np.asarray(w, np.float64).T
    if residual is not None:
        y = y + np.asarray(residual, np.float64)
    return bf16_round(y) if round_out else y


# ----------------------------------------------------------------------------
# Step 3: merged self + cross attention
# ----------------------------------------------------------------------------
def merged_attention_doc(q: np.ndarray, k_self: np.ndarray, v_self: np.ndarray,
                         k_cross: np.ndarray, v_cross: np.ndarray, scale: float,
                         round_out: bool = True):
    """One document's merged attention.

    "KaLM-Reranker-V1-Nano - MLX", "What this is": a single scaled-dot-product
    attention whose keys/values are the concatenation of the decoder's self
    K/V and the cross K/V of the document's cached vectors.

    Shapes: ``q [Lq][n_q][D]``, ``k_self, v_self [Lq][n_kv][D]``,
    ``k_cross, v_cross [Nc][n_kv][D]``.  Readings: the self part is causal with
    the diagonal included (row i sees self keys 0..i); cross keys carry no mask;
    the concatenation order is self then cross; query head h reads KV head
    h // (n_q / n_kv); one softmax covers both parts; logits are q.k * scale.

    The concatenated key and value lists are built explicitly, the logits of
    masked self keys are set to -inf, and each row takes a plain softmax.
    Returns ``(o [Lq][n_q][D], lse [Lq][n_q])`` where lse is the natural log of
    the softmax denominator (in logit units, after scaling).
    """
    q = np.asarray(q, np.float64)
    Lq, n_q, D = q.shape
    n_kv = k_self.shape[1]
    G = n_q // n_kv
    Nc = k_cross.shape[0]
    o = np.zeros((Lq, n_q, D))
    lse = np.zeros((Lq, n_q))
    causal = np.tril(np.ones((Lq, Lq), dtype=bool))
    mask = np.concatenate([causal, np.ones((Lq, Nc), dtype=bool)], axis=1)
    for h in range(n_q):
        g = h // G
        keys = np.concatenate([np.asarray(k_self, np.float64)[:, g, :],
                               np.asarray(k_cross, np.float64)[:, g, :]], axis=0)
        vals = np.concatenate([np.asarray(v_self, np.float64)[:, g, :],
                               np.asarray(v_cross, np.float64)[:, g, :]], axis=0)
        logits = (q[:, h, :] @ keys.T) * scale
        logits = np.where(mask, logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        s = e.sum(axis=1, keepdims=True)
        o[:, h, :] = (e / s) @ vals
        lse[:, h] = (m + np.log(s))[:, 0]
    if round_out:
        o = bf16_round(o)
    return o, lse


def merged_attention(q, k_self, v_self, k_cross, v_cross, q_off, pool_off, scale,
                     round_out: bool = True):
    """Batched form over documents with packed ragged rows.

    ``q [rows][n_q][D]``, ``k_self/v_self [rows][n_kv][D]`` with document d at
    rows ``q_off[d] .. q_off[d+1]-1``; ``k_cross/v_cross [pooled rows][n_kv][D]``
    with document d at ``pool_off[d] .. pool_off[d+1]-1``.  Each document is
    independent ("one big decode" batches documents; nothing crosses them)."""
    q = np.asarray(q, np.float64)
    o = np.zeros_like(q)
    lse = np.zeros(q.shape[:2])
    for d in range(len(q_off) - 1):
        a, b = int(q_off[d]), int(q_off[d + 1])
        c0, c1 = int(pool_off[d]), int(pool_off[d + 1])
        if b == a:
            continue
        o[a:b], lse[a:b] = merged_attention_doc(q[a:b], k_self[a:b], v_self[a:b],
                                                k_cross[c0:c1], v_cross[c0:c1], scale,
                                                round_out=round_out)
    return o, lse


# ----------------------------------------------------------------------------
# Step 4: yes/no readout
# ----------------------------------------------------------------------------
def sigmoid(m):
    """Logistic function evaluated without overflow: 1/(1+e^-m) for m >= 0,
    e^m/(1+e^m) for m < 0."""
    m = np.asarray(m, np.float64)
    out = np.empty_like(m)
    pos = m >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-m[pos]))
    e = np.exp(m[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def yes_no_score(x_last: np.ndarray, w_yes: np.ndarray, w_no: np.ndarray):
    """Readout at the decoder's final position.

    "What this is": score = softmax([logit_yes, logit_no])[yes];
    "Score a pair" / "Frozen inference contract": margin = yes - no and
    score = sigmoid(margin), which is the same number.  Reading: the two logits
    are dot products of the last hidden state with the two LM-head rows (no
    final norm and no soft-capping; the pages name none).

    ``x_last [n][H]``; returns ``(yes, no, margin, score)`` as fp64 arrays.
    The score is the softmax's first entry written as 1 / (1 + e^(no - yes)),
    evaluated through the overflow-free logistic above."""
    x = np.asarray(x_last, np.float64)
    yes = x @ np.asarray(w_yes, np.float64)
    no = x @ np.asarray(w_no, np.float64)
    margin = yes - no
    return yes, no, margin, sigmoid(margin)


# ----------------------------------------------------------------------------
# Rotary position embedding of the decoder's self Q and K
# ----------------------------------------------------------------------------
def rope_inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """Inverse frequencies theta^(-2i/head_dim), i = 0 .. head_dim/2 - 1: the table a
    model config's rope parameters define ("KaLM-Reranker-V1-Nano - MLX",
    "Derivation": the inverse-frequency tables are computed from the config)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return float(theta) ** (-2.0 * i / head_dim)


def apply_rope(x: np.ndarray, positions: Sequence[int], theta: float, round_out: bool = True) -> np.ndarray:
    """Rotate each head vector of row r by its decoder position ``positions[r]``.

    x: [rows][heads][D].  Element i (< D/2) pairs with element i + D/2 and the pair
    (a, b) turns by the angle pos * inv_freq[i]: (a cos - b sin, b cos + a sin).
    Rounded to bf16 (the rotated Q and K are stored)."""
    D = x.shape[-1]
    h = D // 2
    ang = np.asarray(positions, np.float64)[:, None] * rope_inv_freq(D, theta)[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a, b = x[..., :h], x[..., h:]
    out = np.concatenate([a * c - b * s, b * c + a * s], axis=-1)
    return bf16_round(out) if round_out else out


# ----------------------------------------------------------------------------
# End to end (oracle mode (ii): the oracle chains its own rounded outputs)
# ----------------------------------------------------------------------------
def decoder_layer(X: np.ndarray, pooled: np.ndarray, w_qkv_l, w_o_l, w_kv_l, n_q: int, n_kv: int,
                  head_dim: int, scale: float, trace: Optional[dict] = None,
                  rope_theta: Optional[float] = None) -> np.ndarray:
    """One layer of the synthetic attention-only decoder for one document.

    Reading of the synthetic stack (the pages name no MLP/norm on this path):
    ``X <- X + MergedAttn(X Wq, X Wk, X Wv, P Wk_c, P Wv_c) Wo`` with P the
    document's pooled vectors.  With ``rope_theta`` the self Q and K are rotated
    by decoder position 0 .. Lq-1 before the attention (the cross keys have no
    decoder position and are not rotated).  Returns the new X (bf16-rounded)."""
    D = head_dim
    Lq = X.shape[0]
    kv = linear(pooled, w_kv_l).reshape(-1, 2, n_kv, D)
    qkv = linear(X, w_qkv_l)
    if rope_theta is not None:
        qk = apply_rope(qkv[:, :(n_q + n_kv) * D].reshape(Lq, n_q + n_kv, D), np.arange(Lq), rope_theta)
        qkv = np.concatenate([qk.reshape(Lq, -1), qkv[:, (n_q + n_kv) * D:]], axis=1)
    q = qkv[:, : n_q * D].reshape(Lq, n_q, D)
    ks = qkv[:, n_q * D:(n_q + n_kv) * D].reshape(Lq, n_kv, D)
    vs = qkv[:, (n_q + n_kv) * D:].reshape(Lq, n_kv, D)
    o, lse = merged_attention_doc(q, ks, vs, kv[:, 0], kv[:, 1], scale)
    Xn = linear(o.reshape(Lq, n_q * D), w_o_l, residual=X)
    if trace is not None:
        trace.setdefault("layers", []).append(dict(x_in=X, qkv=qkv, kv_cross=kv, o=o, lse=lse, x_out=Xn))
    return Xn


def forward_doc(enc_doc: np.ndarray, x0: np.ndarray, w_qkv, w_o, w_kv_cross,
                w_yes, w_no, n_q: int, n_kv: int, head_dim: int, scale: float,
                chunk: int = 4, layers: Optional[Sequence[int]] = None,
                trace: Optional[dict] = None, rope_theta: Optional[float] = None):
    """Score one document with the synthetic attention-only decoder stack
    (``decoder_layer`` per layer, X0 = the query's decoder input).
    Returns ``(yes, no, margin, score)`` as floats.  ``trace`` (a dict), if
    given, receives the intermediate tensors of every layer."""
    Lq = x0.shape[0]
    pooled, _ = chunk_pool(enc_doc, [0], [enc_doc.shape[0]], chunk)
    X = np.asarray(x0, np.float64)
    lay = range(len(w_qkv)) if layers is None else layers
    for l in lay:
        X = decoder_layer(X, pooled, w_qkv[l], w_o[l], w_kv_cross[l], n_q, n_kv, head_dim, scale, trace,
                          rope_theta)
    if trace is not None:
        trace["pooled"] = pooled
        trace["x_final"] = X
    y, n, m, s = yes_no_score(X[Lq - 1:Lq], w_yes, w_no)
    return float(y[0]), float(n[0]), float(m[0]), float(s[0])


def forward_query(query, docs: Optional[Sequence[int]] = None, chunk: int = 4,
                  scale: Optional[float] = None, rope_theta: Optional[float] = None):
    """End-to-end oracle scores for documents ``docs`` (default: all) of a
    ``synthetic.Query``.  Returns fp64 arrays (yes, no, margin, score)."""
    D = query.head_dim
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    w = query.weights
    w_qkv = bf16_bits_to_f64(w.w_qkv)
    w_o = bf16_bits_to_f64(w.w_o)
    w_kv = bf16_bits_to_f64(w.w_kv_cross)
    w_yes = bf16_bits_to_f64(w.w_yes)
    w_no = bf16_bits_to_f64(w.w_no)
    x0 = bf16_bits_to_f64(query.x0)
    docs = range(query.n_docs) if docs is None else docs
    res = []
    for d in docs:
        a, b = int(query.tok_off[d]), int(query.tok_off[d + 1])
        enc = bf16_bits_to_f64(query.enc[a:b])
        res.append(forward_doc(enc, x0, w_qkv, w_o, w_kv, w_yes, w_no,
                               query.n_q, query.n_kv, D, scale, chunk, rope_theta=rope_theta))
    r = np.array(res, dtype=np.float64).reshape(-1, 4)
    return r[:, 0], r[:, 1], r[:, 2], r[:, 3]
