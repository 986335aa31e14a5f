/*
 * kalm.h - C ABI of the KaLM-Reranker-V1 "fast but not late interaction" (FBNL)
 * scoring hot path on NVIDIA B200 (sm_100a).
 *
 * The path has four steps, each an entry point below:
 *   1. kalm_chunk_pool        masked-mean chunk pooling of cached passage encoder
 *                             states into the document cache;
 *   2. kalm_cross_kv_proj     cross-attention K/V projection of the pooled vectors
 *                             (kalm_linear is the same GEMM for the decoder's
 *                             Q/K/V and output projections);
 *   3. kalm_merged_attention  one softmax over [causal self K/V ; cross K/V];
 *   4. kalm_yes_no_score      final-position yes/no readout, score = sigmoid(yes - no).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller; the library
 *   allocates no device memory on these calls.  Host-side arguments are sizes,
 *   strides, flags and the stream.
 * - bf16 tensors are raw IEEE bfloat16 bit patterns (kalm_bf16).  Strides ("ld",
 *   leading dimension) are in ELEMENTS between consecutive rows; every bf16
 *   pointer must be 16-byte aligned and every bf16 row stride a multiple of 8.
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *   default stream).  Argument errors are detected on the host and returned
 *   synchronously; nothing is launched in that case.
 * - Errors found on the device (a bounded wait that expired, an out-of-range
 *   length) are recorded in a per-device error word that
 *   kalm_check_device_errors() reads after synchronising the stream.  Kernels
 *   never trap.
 * - There is no CPU fallback: without an sm_100 device every call returns
 *   KALM_ERR_NO_DEVICE (the pages' "--require-gpu" rule: a missing GPU is an
 *   explicit error, never a silent fallback).
 *
 * Ragged layout.  Documents are packed one after another.  For n documents:
 *   tok_off[n+1]   exclusive prefix sum of the encoder lengths len[d];
 *   pool_off[n+1]  exclusive prefix sum of Nc[d] = ceil(len[d] / chunk);
 *   q_off[n+1]     exclusive prefix sum of the decoder lengths Lq[d].
 * These are int64 device arrays; kalm_ragged_offsets() computes the first two.
 */
#ifndef KALM_H_
#define KALM_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t kalm_bf16;   /* bfloat16 bit pattern */
typedef void* kalm_stream_t;  /* cudaStream_t */

typedef enum kalm_status {
  KALM_OK = 0,
  KALM_ERR_INVALID_ARG = 1,   /* null pointer, bad size/stride/alignment, limit exceeded */
  KALM_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim != 256) */
  KALM_ERR_NO_DEVICE = 3,     /* no sm_100 device current; never falls back to the CPU */
  KALM_ERR_CUDA = 4,          /* a CUDA runtime call failed (see kalm_last_error) */
  KALM_ERR_TIMEOUT = 5,       /* a device-side bounded wait expired (device error word) */
  KALM_ERR_DEVICE_ARG = 6     /* a kernel found an invalid value in device data */
} kalm_status;

/* Limits of the pages' runtime contract ("KaLM-Reranker-V1-Small-Q4_K_M-GGUF",
 * "Runtime boundaries"; "KaLM-Reranker-V1-Large-Q8_0-GGUF", "Frozen inference
 * contract"): at most 1,024 encoder tokens per passage, a query budget of 512
 * tokens, encoder chunk size 4. */
#define KALM_MAX_DOC_TOKENS 1024
#define KALM_MAX_QUERY_TOKENS 512
#define KALM_DEFAULT_CHUNK 4
#define KALM_HEAD_DIM 256

/* Version of this ABI (major * 100 + minor). */
int kalm_version(void);

/* Human-readable name of a status code (static string). */
const char* kalm_status_string(int status);

/* Detail of the last error returned on the calling host thread (static,
 * thread-local buffer; empty string if none). */
const char* kalm_last_error(void);

/* KALM_OK if the current CUDA device is an sm_100 part, else KALM_ERR_NO_DEVICE. */
kalm_status kalm_device_check(void);

/* Synchronise `stream`, read and clear the current device's error word.
 * The read and the clear are one atomic exchange, ordered on `stream` after the
 * work already queued there.  Kernels still running on other streams may set
 * bits after it; those bits are kept for the next call (to see them in this
 * one, let every stream that runs library kernels go idle first).
 * *word_out (nullable) receives the raw word: bit 0 = a bounded wait expired,
 * bit 1 = invalid device data (e.g. a length above its limit); bits 8..15 name
 * the kernel (1 pool, 2 linear, 3 attention, 4 readout, 5 offsets, 6 self-test).
 * Returns KALM_ERR_TIMEOUT, KALM_ERR_DEVICE_ARG or KALM_OK. */
kalm_status kalm_check_device_errors(kalm_stream_t stream, uint32_t* word_out);

/* Ragged offsets: tok_off[d] = sum_{e<d} len[e], pool_off[d] = sum_{e<d}
 * ceil(len[e] / chunk), for d = 0..n (both arrays hold n+1 int64 values).
 * "KaLM-Reranker-V1-Small-Q4_K_M-GGUF", "Runtime boundaries": passages of at
 * most 1,024 encoder tokens, pooled in groups of 4; "KaLM-Reranker-V1-Large-
 * Q8_0-GGUF", "Frozen inference contract": right padding, so a document's
 * valid tokens are its first len[d] rows and it yields ceil(len[d] / 4)
 * pooled vectors.  The documents of one query are packed one after another
 * ("KaLM-Reranker-V1-Nano - MLX", "Speed": all documents decoded in one batch).
 * len: int32 device array of n values in [0, KALM_MAX_DOC_TOKENS]; a value out
 * of range is clamped to the range and flagged in the device error word.
 * n >= 0, chunk >= 1.  Either output may be NULL. */
kalm_status kalm_ragged_offsets(const int32_t* len, int32_t n, int32_t chunk,
                                int64_t* tok_off, int64_t* pool_off,
                                kalm_stream_t stream);

/* Step 1 - chunk pooling into the document cache.
 * "KaLM-Reranker-V1-Nano - MLX (Apple Silicon)", "What this is": each passage is
 * encoded once and chunk-pooled (chunk size 4 tokens, masked mean per chunk)
 * into a small set of cached document vectors; "KaLM-Reranker-V1-Large-Q8_0-
 * GGUF", "Frozen inference contract": right padding, masked mean pooling over
 * consecutive groups of 4 tokens.
 *
 *   pooled[pool_off[d] + c][:] = mean of enc[tok_off[d] + t][:] over
 *       t = chunk*c .. min(chunk*c + chunk, len[d]) - 1
 * i.e. a partial last group is averaged over its valid tokens only; groups
 * start at token 0; no vector is emitted for a group with no valid token.
 * Accumulation in fp32, one rounding to bf16 (nearest even) per output.
 *
 * enc     [rows][enc_ld] bf16; document d starts at row tok_off[d] (packed or
 *         padded layouts both work; rows past len[d] are never read)
 * tok_off int64[n_docs] (entries beyond n_docs are not read)
 * len     int32[n_docs], each in [0, KALM_MAX_DOC_TOKENS]
 * pooled  [total_pooled][pooled_ld] bf16, written for rows pool_off[d] ..
 *         pool_off[d] + ceil(len[d]/chunk) - 1
 * pool_off int64[n_docs + 1], must equal the prefix sums of ceil(len/chunk);
 *         total_pooled = pool_off[n_docs] (host-known, sizes the launch)
 * hidden % 8 == 0; 1 <= chunk <= 64. */
kalm_status kalm_chunk_pool(const kalm_bf16* enc, int64_t enc_ld, const int64_t* tok_off,
                            const int32_t* len, int32_t n_docs, int32_t hidden,
                            int32_t chunk, kalm_bf16* pooled, int64_t pooled_ld,
                            const int64_t* pool_off, int64_t total_pooled,
                            kalm_stream_t stream);

/* Dense projection y = x . w^T (+ residual), bf16 in, fp32 accumulate, bf16 out.
 * The tcgen05 (5th-generation tensor core) GEMM behind steps 2 and the decoder
 * projections.  "KaLM-Reranker-V1-Nano - MLX", "What this is": the decoder
 * projects its hidden states to the self-attention Q/K/V, and the cross K/V
 * are projections of the cached passage encodings; the attention output goes
 * back through the output projection onto the residual stream (the synthetic
 * attention-only decoder: X <- X + Attn(X Wq, X Wk, X Wv, P Wk_c, P Wv_c) Wo).
 *
 * x        [m][ldx] bf16 (m rows of k values)
 * w        [n][ldw] bf16, the nn.Linear layout [out][in]
 * residual [m][ldr] bf16 or NULL; added before the single rounding to bf16.
 *          It may alias y (same pointer and stride): every output tile reads
 *          its residual tile before it writes that tile.
 * y        [m][ldy] bf16
 * Requirements: m >= 0, n % 32 == 0, k % 8 == 0, k >= 8. */
kalm_status kalm_linear(const kalm_bf16* x, int64_t ldx, const kalm_bf16* w, int64_t ldw,
                        const kalm_bf16* residual, int64_t ldr, kalm_bf16* y, int64_t ldy,
                        int64_t m, int32_t n, int32_t k, kalm_stream_t stream);

/* A decoder layer's output projection and the next layer's Q|K|V projection,
 * chained in one launch (same passage as kalm_linear: the residual update
 * X <- X + O Wo, then the next layer projects the updated X):
 *   y1 <- x1 . w1^T + y1            (in place: y1 is also the residual)
 *   y2 <- y1 . w2^T                  (reads the y1 just written)
 * Each output element is computed as kalm_linear computes it (same K order, one
 * rounding to bf16), so the results are bit for bit those of the two separate
 * calls.  A tile of the second product starts as soon as the first product's
 * tiles of its 256-row block are stored, instead of after the whole first product.
 *
 * x1 [m][ldx1], w1 [n1][ldw1] (k1 inputs), y1 [m][ldy1] (n1 columns, in/out),
 * w2 [n2][ldw2] (n1 inputs), y2 [m][ldy2] (n2 columns); bf16, 16-byte aligned,
 * strides multiples of 8.  y1 must not overlap x1 or w1, and y2 none of x1, w1, y1.
 * sync: int32[sync_len], sync_len >= kalm_linear_chain_sync_len(m), caller-owned
 *   device memory that must be zero at the call; every launch that ends without
 *   a device error leaves it zero again.  After a device error (see
 *   kalm_check_device_errors) zero it before the next call.  Calls that share
 *   one array must not overlap on the GPU.  Unused (may be NULL) when m < 256,
 *   where the two products run as two launches.
 * Requirements: m >= 0, n1 % 32 == 0, n2 % 32 == 0, k1 % 8 == 0. */
kalm_status kalm_linear_chain(const kalm_bf16* x1, int64_t ldx1, const kalm_bf16* w1, int64_t ldw1,
                              kalm_bf16* y1, int64_t ldy1, const kalm_bf16* w2, int64_t ldw2,
                              kalm_bf16* y2, int64_t ldy2, int64_t m, int32_t n1, int32_t k1,
                              int32_t n2, int32_t* sync, int64_t sync_len, kalm_stream_t stream);

/* Length in int32 of kalm_linear_chain's sync array for m rows (2 per 256-row
 * block), or -1 for m < 0. */
int64_t kalm_linear_chain_sync_len(int64_t m);

/* kalm_linear_chain with the rotary embedding of the second product's first
 * rot_cols columns applied in its epilogue, as kalm_linear_rope applies it (same
 * passages, pairing, angle table and position rule): the output projection of a
 * layer and the next layer's rotated Q|K|V projection in one launch.  Results
 * are bit for bit those of kalm_linear (residual in place) then kalm_linear_rope.
 * Arguments as kalm_linear_chain, and rot_cols, head_dim, q_off, n_docs, table
 * as kalm_linear_rope (head_dim 256, n2 % 256 == 0, rot_cols a positive multiple
 * of head_dim <= n2). */
kalm_status kalm_linear_chain_rope(const kalm_bf16* x1, int64_t ldx1, const kalm_bf16* w1, int64_t ldw1,
                                   kalm_bf16* y1, int64_t ldy1, const kalm_bf16* w2, int64_t ldw2,
                                   kalm_bf16* y2, int64_t ldy2, int64_t m, int32_t n1, int32_t k1,
                                   int32_t n2, int32_t rot_cols, int32_t head_dim, const int64_t* q_off,
                                   int32_t n_docs, const float* table, int32_t* sync, int64_t sync_len,
                                   kalm_stream_t stream);

/* Step 2 - cross-attention K/V projection of the cached pooled vectors for
 * n_layers decoder layers at once.
 * "KaLM-Reranker-V1-Nano - MLX", "What this is": the cross-attention KV is
 * computed over the cached passage encodings.  Reading: no bias, norm or
 * rotary embedding on the cross K/V (the pages name none).
 *
 * pooled   [total_pooled][pooled_ld] bf16 (the document cache)
 * w_kv     [n_layers][2][n_kv][head_dim][hidden] bf16 (per layer: cross K rows,
 *          then cross V rows, nn.Linear layout)
 * kv_cross [total_pooled][n_layers][2][n_kv][head_dim] bf16: for pooled row r,
 *          layer l, cross K of KV head g starts at element
 *          r*ld + (l*2 + 0)*n_kv*head_dim + g*head_dim and cross V at
 *          r*ld + (l*2 + 1)*n_kv*head_dim + g*head_dim, ld = n_layers*2*n_kv*head_dim. */
kalm_status kalm_cross_kv_proj(const kalm_bf16* pooled, int64_t pooled_ld, int64_t total_pooled,
                               int32_t hidden, const kalm_bf16* w_kv, int32_t n_layers,
                               int32_t n_kv, int32_t head_dim, kalm_bf16* kv_cross,
                               kalm_stream_t stream);

/* Step 3 - merged self + cross attention for a ragged batch of documents.
 * "KaLM-Reranker-V1-Nano - MLX", "What this is": a single scaled-dot-product
 * attention that concatenates the decoder's self-attention K/V with the
 * cross-attention K/V of the document's cached vectors.
 *
 * For document d, query head h (KV head g = h / (n_q / n_kv)) and decoder row i
 * (0 <= i < Lq[d]):
 *   out[i, h] = sum_j softmax_j(scale * q[i,h] . key_j) value_j over
 *   j in {self rows 0..i} U {cross rows 0..Nc[d]-1}
 * one softmax over both segments (causal self part, diagonal included; cross
 * part unmasked).  The concatenation is never materialised.
 *
 * q       [rows][ldq] bf16; row in(d)+i, head h at element h*head_dim
 * k_self, v_self  [rows][ld_self] bf16; KV head g at element g*head_dim
 * k_cross, v_cross [pool_off[n_docs]][ld_cross] bf16; KV head g at g*head_dim
 * q_off   int64[n_docs+1]: document d has Lq[d] = q_off[d+1]-q_off[d] decoder
 *         rows; its outputs go to rows q_off[d] .. q_off[d+1]-1 of `out`
 * in_off  int64[n_docs] or NULL: first row in(d) of document d's q / k_self /
 *         v_self rows (NULL: in(d) = q_off[d]).  Documents may share input rows
 *         (e.g. in_off all zero when every document's decoder input is the same,
 *         as in the first decoder layer, where all documents start from the
 *         query's common input).  total_in = number of input rows (ignored when
 *         in_off is NULL).
 * pool_off int64[n_docs+1] (cross rows of document d: pool_off[d] .. pool_off[d+1]-1)
 * max_q   host upper bound of Lq[d] (<= KALM_MAX_QUERY_TOKENS); sizes the grid
 * total_q = q_off[n_docs], total_pool = pool_off[n_docs] (host-known; bound the
 *         tensor views)
 * scale   logit scale (1/sqrt(head_dim) for the standard attention)
 * last_tile_only  nonzero: compute only the 128-row query tile (128/(n_q/n_kv)
 *         positions) that holds each document's last decoder row; the other
 *         rows of `out` are left untouched.  Enough when only the final
 *         position is read afterwards (the yes/no readout of the last layer).
 * order   int32[kalm_attention_items(...)] written by kalm_attention_schedule
 *         for the same offsets and sizes, or NULL.  The persistent CTA c takes
 *         entry k * grid + c in its k-th pass (grid = min(items, SMs)); without an
 *         order it takes item k * grid + c.  Only which CTA computes which item
 *         changes; the results are the same.  An entry outside the item range is
 *         skipped and flagged in the device error word.  The order must come
 *         from kalm_attention_schedule called with the same q_off, pool_off,
 *         n_docs, max_q, n_q, n_kv and last_tile_only: an order made for other
 *         sizes can repeat or leave out items while every entry is in range, and
 *         the items it leaves out are then not written (nothing detects that).
 * out     [total_q][ldo] bf16, head h at element h*head_dim
 * lse     fp32 [total_q][n_q] or NULL: natural log of each row's softmax
 *         denominator, in scaled-logit units.
 * Requirements: head_dim == 256; n_q % n_kv == 0; (n_q / n_kv) divides 128;
 * strides multiples of 8. */
kalm_status kalm_merged_attention(const kalm_bf16* q, int64_t ldq,
                                  const kalm_bf16* k_self, const kalm_bf16* v_self, int64_t ld_self,
                                  const kalm_bf16* k_cross, const kalm_bf16* v_cross, int64_t ld_cross,
                                  const int64_t* q_off, const int64_t* in_off, int64_t total_in,
                                  const int64_t* pool_off, int32_t n_docs, int32_t max_q,
                                  int64_t total_q, int64_t total_pool,
                                  int32_t n_q, int32_t n_kv, int32_t head_dim, float scale,
                                  int32_t last_tile_only, const int32_t* order,
                                  kalm_bf16* out, int64_t ldo, float* lse, kalm_stream_t stream);

/* Step 3 followed by the decoder's output projection in one launch (a fused decoder
 * layer).  "KaLM-Reranker-V1-Nano - MLX", "What this is": the decoder's merged
 * self + cross attention, whose output goes back through the output projection onto
 * the residual stream (the synthetic attention-only decoder: X <- X + Attn(...) . Wo).
 *
 * Computes exactly what kalm_merged_attention (last_tile_only = 0, lse = NULL) writes
 * to `out`, and then, for every document, X[rows of d] += out[rows of d] . w_o^T with
 * one bf16 rounding (as kalm_linear with residual = x, in place).  Inside the launch
 * each CTA first computes its attention work items; when a document's last item is
 * done, its projection tiles (document x 128 rows x 256 columns) are queued, and CTAs
 * that have finished their own items take tiles from the queue in that order, so the
 * projection fills the tail of the attention.
 *
 * Arguments up to `ldo`: as kalm_merged_attention (q_off, in_off, pool_off, order, out
 *          ... with the same requirements; `order` must come from kalm_attention_schedule
 *          for the same sizes, or be NULL).
 * w_o      [hidden][ldw] bf16, the output projection in the nn.Linear layout [out][in],
 *          in = n_q * head_dim
 * x        [total_q][ldx] bf16, the residual stream, updated in place
 * hidden   multiple of 64
 * sync     int32 device array of sync_len >= kalm_attention_out_proj_sync_len(n_docs,
 *          max_q, hidden) entries: the launch's per-document completion counters and a
 *          queue of projection tiles whose documents are complete.
 *          Caller-owned; must be zero before the first call (e.g. cudaMemset), and every
 *          call leaves it zero again.  Launches that share one array must not overlap on
 *          the GPU.  After a call that recorded a device error, zero it again.
 * Errors: as kalm_merged_attention; NULL w_o/x/sync, hidden not a multiple of 64, a
 *          short sync array, misaligned pointers or strides -> KALM_ERR_INVALID_ARG.  A
 *          wait on another CTA's items that runs out its bound is recorded in the device
 *          error word (timeout). */
kalm_status kalm_merged_attention_out_proj(const kalm_bf16* q, int64_t ldq,
                                           const kalm_bf16* k_self, const kalm_bf16* v_self, int64_t ld_self,
                                           const kalm_bf16* k_cross, const kalm_bf16* v_cross, int64_t ld_cross,
                                           const int64_t* q_off, const int64_t* in_off, int64_t total_in,
                                           const int64_t* pool_off, int32_t n_docs, int32_t max_q,
                                           int64_t total_q, int64_t total_pool,
                                           int32_t n_q, int32_t n_kv, int32_t head_dim, float scale,
                                           const int32_t* order, kalm_bf16* out, int64_t ldo,
                                           const kalm_bf16* w_o, int64_t ldw, kalm_bf16* x, int64_t ldx,
                                           int32_t hidden, int32_t* sync, int64_t sync_len,
                                           kalm_stream_t stream);

/* kalm_merged_attention_out_proj without the caller's counter array, for callers that
 * cannot allocate device memory: code that only receives tensors from a host program
 * that owns every allocation (an inference server with its own pooled allocator, or an
 * embedding that forbids allocation while it serves), and C callers with no allocator
 * of their own.  The pages have no counterpart; this is an interface convenience.
 *
 * Same arguments, results and errors as kalm_merged_attention_out_proj, minus sync and
 * sync_len.  The counters live in a fixed array inside the library's device memory,
 * sized for KALM_OUT_PROJ_STATIC_MAX_DOCS documents and KALM_OUT_PROJ_STATIC_MAX_TILES
 * projection tiles (n_docs * ceil(max_q / 128) * ceil(hidden / 256)): every device that
 * loads the library holds it (about 213 KB) until the process exits.  Larger sizes ->
 * KALM_ERR_INVALID_ARG.
 * Nothing is allocated: the call clears the counters it uses with an asynchronous
 * memset on `stream` and launches the fused kernel.
 * - The first call on a device looks up the array's device address (a runtime query);
 *   make that first call before any stream capture.
 * - Every call on a device shares the one array, and it keeps the last call's contents:
 *   calls whose work overlaps on the GPU (other streams, other host threads) race on it;
 *   order them on one stream. */
#define KALM_OUT_PROJ_STATIC_MAX_DOCS 4096
#define KALM_OUT_PROJ_STATIC_MAX_TILES 49152
kalm_status kalm_merged_attention_out_proj_static(const kalm_bf16* q, int64_t ldq,
                                                  const kalm_bf16* k_self, const kalm_bf16* v_self, int64_t ld_self,
                                                  const kalm_bf16* k_cross, const kalm_bf16* v_cross, int64_t ld_cross,
                                                  const int64_t* q_off, const int64_t* in_off, int64_t total_in,
                                                  const int64_t* pool_off, int32_t n_docs, int32_t max_q,
                                                  int64_t total_q, int64_t total_pool,
                                                  int32_t n_q, int32_t n_kv, int32_t head_dim, float scale,
                                                  const int32_t* order, kalm_bf16* out, int64_t ldo,
                                                  const kalm_bf16* w_o, int64_t ldw, kalm_bf16* x, int64_t ldx,
                                                  int32_t hidden, kalm_stream_t stream);

/* Entries of the sync array kalm_merged_attention_out_proj needs: n_docs + 2 +
 * n_docs * ceil(max_q / 128) * ceil(hidden / 256), or -1 for negative sizes or
 * hidden <= 0.  Host-only arithmetic. */
int64_t kalm_attention_out_proj_sync_len(int32_t n_docs, int32_t max_q, int32_t hidden);

/* Work items of one kalm_merged_attention call (one query tile of 128/(n_q/n_kv)
 * decoder positions x one KV head x one document): ceil(max_q / (128 n_kv / n_q))
 * * n_docs * n_kv, or n_docs * n_kv with last_tile_only.  Host-only
 * arithmetic; returns -1 for sizes kalm_merged_attention rejects.  Scheduling
 * aid for the step-3 kernel; the pages have no counterpart (they describe what
 * the attention computes, not how a GPU divides it). */
int64_t kalm_attention_items(int32_t n_docs, int32_t max_q, int32_t n_q, int32_t n_kv, int32_t last_tile_only);

/* Work order for kalm_merged_attention: writes order[0 .. items-1], a
 * permutation of the work items.  An item's cost is its K/V tiles (from q_off and
 * pool_off) plus a fixed per-item part; the items, sorted heaviest first, are
 * dealt out in rounds of one item per CTA, each to the CTA with the least total
 * cost so far, so that every CTA's total comes out close to the mean.  The costs
 * are the same for every layer of a query, so one order serves all its layers.
 * Scheduling aid; the pages have no counterpart.  order is caller-owned device
 * memory of at least order_len >= kalm_attention_items(...) entries; stream-
 * ordered, one single-CTA kernel; nothing allocated.  Errors: sizes as
 * kalm_merged_attention, order_len too small -> KALM_ERR_INVALID_ARG. */
kalm_status kalm_attention_schedule(const int64_t* q_off, const int64_t* pool_off, int32_t n_docs,
                                    int32_t max_q, int32_t n_q, int32_t n_kv, int32_t last_tile_only,
                                    int32_t* order, int64_t order_len, kalm_stream_t stream);

/* Step 4 - yes/no readout at each document's final decoder position.
 * "What this is": score = softmax([logit_yes, logit_no])[yes] at the final
 * position; "Score a pair" / "Frozen inference contract": margin = yes - no,
 * score = sigmoid(margin) (the same number).
 *
 * hidden  [q_off[n_docs]][ldh] bf16; document d's final row is q_off[d+1]-1
 * w_yes, w_no  [hidden_dim] bf16 (the two LM-head rows)
 * yes, no, score  fp32[n_docs]; margin fp32[n_docs] or NULL.  Documents with
 * no decoder rows get yes = no = margin = 0, score = 0.5.
 * Scores come back in input order. */
kalm_status kalm_yes_no_score(const kalm_bf16* hidden, int64_t ldh, const int64_t* q_off,
                              int32_t n_docs, int32_t hidden_dim,
                              const kalm_bf16* w_yes, const kalm_bf16* w_no,
                              float* yes, float* no, float* margin, float* score,
                              kalm_stream_t stream);

/* Copy rows of a shared [rows][ld_src] bf16 block into every document's slot:
 * dst[q_off[d] + i] = src[i] for i < q_off[d+1]-q_off[d] (<= rows).  Used to
 * start every document's decoder stream from the query's common input
 * (the decoder reads the same instruction + query for each passage). */
kalm_status kalm_broadcast_rows(const kalm_bf16* src, int64_t ld_src, int32_t rows,
                                int32_t width, const int64_t* q_off, int32_t n_docs,
                                kalm_bf16* dst, int64_t ld_dst, kalm_stream_t stream);

/* Rotary position embedding of the decoder's self Q and K, in place ("next"
 * step after the four above).  "KaLM-Reranker-V1-Nano - MLX (Apple Silicon)",
 * "Derivation": the rotary parameters and inverse-frequency tables are read
 * from the model config.  Reading taken (the pages give neither the pairing
 * nor which segments are rotated): element i < head_dim/2 of each head vector
 * pairs with element i + head_dim/2 and (a, b) turns by the angle
 * pos * theta^(-2i/head_dim): (a cos - b sin, b cos + a sin); the decoder's
 * self Q and K are rotated, the cross keys (pooled passage vectors, no decoder
 * position) are not.
 *
 * x       [rows][ldx] bf16, n_heads head vectors of head_dim elements at the
 *         start of each row (Q heads then self-K heads of the fused Q|K|V
 *         layout: one call covers both); rotated in place, one bf16 rounding.
 * q_off   int64[n_docs+1]: row r belongs to the document d with
 *         q_off[d] <= r < q_off[d+1] and sits at position r - q_off[d]
 *         (< KALM_MAX_QUERY_TOKENS; rows = q_off[n_docs]).
 * theta   rotary base (> 1).
 * Requirements: head_dim % 16 == 0, ldx % 8 == 0, x 16-byte aligned.  A row
 * whose position falls outside [0, KALM_MAX_QUERY_TOKENS) is left unchanged and
 * flagged in the device error word. */
kalm_status kalm_rope(kalm_bf16* x, int64_t ldx, int64_t rows, int32_t n_heads, int32_t head_dim,
                      const int64_t* q_off, int32_t n_docs, float theta, kalm_stream_t stream);

/* Table of the rotary angles' cosines and sines, built once per rotary base for
 * kalm_linear_rope.  Same passage and reading as kalm_rope: the angle of pair p
 * at position pos is pos * theta^(-2p/head_dim), its cosine and sine computed
 * exactly as kalm_rope computes them.
 *
 * table   float[head_dim/4][KALM_MAX_QUERY_TOKENS][4] device, caller-owned,
 *         16-byte aligned; entry [q][pos] = (cos, sin) of pair 2q, then
 *         (cos, sin) of pair 2q + 1 (position-minor, so that consecutive rows
 *         read consecutive entries).  Written entirely.
 * theta   rotary base (> 1); head_dim % 16 == 0. */
kalm_status kalm_rope_table(float theta, int32_t head_dim, float* table, kalm_stream_t stream);

/* The decoder's fused Q|K|V projection with the rotary embedding of its first
 * rot_cols output columns applied in the projection's epilogue: y = x . w^T,
 * then every head vector in columns [0, rot_cols) turns as kalm_rope turns it
 * (same pairing, angle and position rule), the angles read from a table that
 * kalm_rope_table built.  The result is bit-identical to kalm_linear followed
 * by kalm_rope over rot_cols / head_dim heads: the accumulator is rounded to
 * bf16 first, rotated in fp32, rounded again.  Saves the rotation's separate
 * read and write of Q and K_self.  Same passages as kalm_rope for the rotation,
 * as kalm_linear for the product.
 *
 * x, w, y, ldx, ldw, ldy, m, n, k   as kalm_linear (no residual).
 * rot_cols  multiple of head_dim, <= n: the Q heads and self-K heads.
 * head_dim  256 (one head per 256-column output tile).
 * q_off     int64[n_docs+1] device, as kalm_rope (rows [0, m) covered).
 * table     kalm_rope_table's output for head_dim 256 and the rotary base,
 *           16-byte aligned; read only.
 * Requirements: those of kalm_linear, and n % 256 == 0.  A row below m whose
 * position falls outside [0, KALM_MAX_QUERY_TOKENS) is flagged in the device
 * error word (its output is then unspecified). */
kalm_status kalm_linear_rope(const kalm_bf16* x, int64_t ldx, const kalm_bf16* w, int64_t ldw, kalm_bf16* y,
                             int64_t ldy, int64_t m, int32_t n, int32_t k, int32_t rot_cols, int32_t head_dim,
                             const int64_t* q_off, int32_t n_docs, const float* table, kalm_stream_t stream);

/* Failure-detection self-test: one CTA waits on a shared-memory barrier that
 * nothing completes, with a bound of `wait_ns` nanoseconds; on expiry it
 * records a timeout in the device error word and returns.  Lets tests check
 * the bounded-wait path without faulting or hanging the GPU. */
kalm_status kalm_selftest_wait_timeout(uint64_t wait_ns, kalm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif  /* KALM_H_ */
