// Step 1: masked-mean chunk pooling of cached passage encoder states into the
// document cache ("KaLM-Reranker-V1-Nano - MLX", "What this is": chunk size 4,
// masked mean per chunk; "KaLM-Reranker-V1-Large-Q8_0-GGUF", "Frozen inference
// contract": masked mean pooling over consecutive groups of 4 tokens).
//
// HBM-bound streaming kernel: one thread produces one 16-byte vector (8 bf16
// columns) of one pooled row, reading the same 16-byte column slice of up to
// `chunk` consecutive encoder rows.  Consecutive threads take consecutive column
// slices of a row, then the next pooled row, so every warp reads and writes
// contiguous runs of memory.  Algorithmic bytes per pooled row: (valid tokens
// + 1) * hidden * 2.
#include "kalm.h"
#include "kalm_internal.h"
#include "kalm_ptx.cuh"

namespace kalm {
namespace {

// Document that owns pooled row r: the largest d with pool_off[d] <= r.
__device__ __forceinline__ int find_doc(const int64_t* __restrict__ pool_off, int n_docs, int64_t r) {
  int lo = 0, hi = n_docs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(pool_off + mid) <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int CHUNK>
__global__ void __launch_bounds__(256, 8) chunk_pool_kernel(const uint4* __restrict__ enc, int64_t enc_ld_v,
                                                         const int64_t* __restrict__ tok_off,
                                                         const int32_t* __restrict__ len, int n_docs, int vec_per_row,
                                                         int chunk_rt, uint4* __restrict__ pooled,
                                                         int64_t pooled_ld_v, const int64_t* __restrict__ pool_off,
                                                         int64_t total_vec, uint32_t* err) {
  pdl_launch_dependents();
  pdl_wait_predecessor();
  const int chunk = CHUNK > 0 ? CHUNK : chunk_rt;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total_vec;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / vec_per_row;
    const int v = static_cast<int>(i - r * vec_per_row);
    const int d = find_doc(pool_off, n_docs, r);
    const int64_t c = r - __ldg(pool_off + d);
    int n = __ldg(len + d);
    if (n > KALM_MAX_DOC_TOKENS) {
      record_error(err, kErrDeviceArg | kSitePool);
      n = KALM_MAX_DOC_TOKENS;
    }
    const int t0 = static_cast<int>(c) * chunk;
    int cnt = n - t0;
    if (cnt > chunk) cnt = chunk;
    if (cnt <= 0) {  // pool_off inconsistent with len: flag, write nothing
      record_error(err, kErrDeviceArg | kSitePool);
      continue;
    }
    const uint4* src = enc + (__ldg(tok_off + d) + t0) * enc_ld_v + v;
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    if (CHUNK > 0) {
      uint4 x[CHUNK > 0 ? CHUNK : 1];
#pragma unroll
      for (int t = 0; t < (CHUNK > 0 ? CHUNK : 1); ++t)
        if (t < cnt) x[t] = __ldg(src + t * enc_ld_v);
#pragma unroll
      for (int t = 0; t < (CHUNK > 0 ? CHUNK : 1); ++t) {
        if (t < cnt) {
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x[t]);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(h[k]);
            acc[2 * k] += f.x;
            acc[2 * k + 1] += f.y;
          }
        }
      }
    } else {
      for (int t = 0; t < cnt; ++t) {
        const uint4 x = __ldg(src + t * enc_ld_v);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(h[k]);
          acc[2 * k] += f.x;
          acc[2 * k + 1] += f.y;
        }
      }
    }
    const float fc = static_cast<float>(cnt);
    uint4 out;
    out.x = pack_bf16x2(__fdiv_rn(acc[0], fc), __fdiv_rn(acc[1], fc));
    out.y = pack_bf16x2(__fdiv_rn(acc[2], fc), __fdiv_rn(acc[3], fc));
    out.z = pack_bf16x2(__fdiv_rn(acc[4], fc), __fdiv_rn(acc[5], fc));
    out.w = pack_bf16x2(__fdiv_rn(acc[6], fc), __fdiv_rn(acc[7], fc));
    pooled[r * pooled_ld_v + v] = out;
  }
}

}  // namespace
}  // namespace kalm

using namespace kalm;

extern "C" kalm_status kalm_chunk_pool(const kalm_bf16* enc, int64_t enc_ld, const int64_t* tok_off,
                                       const int32_t* len, int32_t n_docs, int32_t hidden, int32_t chunk,
                                       kalm_bf16* pooled, int64_t pooled_ld, const int64_t* pool_off,
                                       int64_t total_pooled, kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (n_docs < 0 || hidden <= 0 || total_pooled < 0)
    return fail(KALM_ERR_INVALID_ARG, "kalm_chunk_pool: n_docs=%d hidden=%d total_pooled=%lld", n_docs, hidden,
                (long long)total_pooled);
  if (chunk < 1 || chunk > 64) return fail(KALM_ERR_INVALID_ARG, "kalm_chunk_pool: chunk=%d not in [1,64]", chunk);
  if (hidden % 8 || enc_ld % 8 || pooled_ld % 8 || enc_ld < hidden || pooled_ld < hidden)
    return fail(KALM_ERR_INVALID_ARG, "kalm_chunk_pool: hidden and strides must be multiples of 8 (hidden=%d)",
                hidden);
  if (n_docs == 0 || total_pooled == 0) return KALM_OK;
  if (!enc || !tok_off || !len || !pooled || !pool_off)
    return fail(KALM_ERR_INVALID_ARG, "kalm_chunk_pool: NULL pointer");
  if (!aligned16(enc) || !aligned16(pooled))
    return fail(KALM_ERR_INVALID_ARG, "kalm_chunk_pool: enc/pooled must be 16-byte aligned");
  const int vpr = hidden / 8;
  const int64_t total_vec = total_pooled * vpr;
  int64_t blocks = (total_vec + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* err = device_error_word();
  const uint4* e = reinterpret_cast<const uint4*>(enc);
  uint4* p = reinterpret_cast<uint4*>(pooled);
  // chunk 4 (the runtime contract) and 2 have unrolled kernels; other sizes take the generic loop
  const cudaError_t ce =
      chunk == 4   ? launch_pdl(chunk_pool_kernel<4>, dim3((unsigned)blocks), dim3(256), 0, s, e, enc_ld / 8, tok_off,
                                len, n_docs, vpr, chunk, p, pooled_ld / 8, pool_off, total_vec, err)
      : chunk == 2 ? launch_pdl(chunk_pool_kernel<2>, dim3((unsigned)blocks), dim3(256), 0, s, e, enc_ld / 8, tok_off,
                                len, n_docs, vpr, chunk, p, pooled_ld / 8, pool_off, total_vec, err)
                   : launch_pdl(chunk_pool_kernel<0>, dim3((unsigned)blocks), dim3(256), 0, s, e, enc_ld / 8, tok_off,
                                len, n_docs, vpr, chunk, p, pooled_ld / 8, pool_off, total_vec, err);
  return check_cuda(ce, "launch chunk_pool_kernel");
}
