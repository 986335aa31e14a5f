// Step 1: masked-mean chunk pooling of cached passage encoder states into the
// document cache ("KaLM-Reranker-V1-Nano - MLX", "What this is": chunk size 4,
// masked mean per chunk; "KaLM-Reranker-V1-Large-Q8_0-GGUF", "Frozen inference
// contract": masked mean pooling over consecutive groups of 4 tokens).
//
// HBM-bound streaming kernel.  Each warp owns a contiguous range of pooled rows and
// walks it in order: it finds the document of its first row once (binary search over
// pool_off) and then advances to the next document when a row crosses its end, so no
// per-row search.  For one pooled row the lanes take consecutive 16-byte column slices
// (8 bf16 columns) and read the same slice of the group's `chunk` encoder rows, each
// lane issuing all its loads of the row before it sums them: every warp-wide load reads
// 512 contiguous bytes of one encoder row, and every store writes 512 contiguous bytes
// of the pooled row.  Algorithmic bytes per pooled row: (valid tokens + 1) * hidden * 2.
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

constexpr int kPoolThreads = 256;
constexpr int kRowsPerWarp = 2;      // target work per warp when the grid is not capped
constexpr int kVecUnroll = 2;        // 16-byte column slices a lane keeps in flight per pooled row
constexpr int kPoolBlocksPerSm = 3;  // resident blocks per SM (80 registers a thread)

// mean = sum / cnt with one rounding: a power-of-two count multiplies by its exact
// reciprocal (the same value as the division), other counts divide
__device__ __forceinline__ float mean_of(float sum, float cnt, float inv, bool exact) {
  return exact ? sum * inv : __fdiv_rn(sum, cnt);
}

__device__ __forceinline__ uint4 pack_mean(const float (&a)[8], float fc, float inv, bool exact) {
  uint4 out;
  out.x = pack_bf16x2(mean_of(a[0], fc, inv, exact), mean_of(a[1], fc, inv, exact));
  out.y = pack_bf16x2(mean_of(a[2], fc, inv, exact), mean_of(a[3], fc, inv, exact));
  out.z = pack_bf16x2(mean_of(a[4], fc, inv, exact), mean_of(a[5], fc, inv, exact));
  out.w = pack_bf16x2(mean_of(a[6], fc, inv, exact), mean_of(a[7], fc, inv, exact));
  return out;
}

__device__ __forceinline__ void add_bf16x8(float (&a)[8], const uint4& x) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __bfloat1622float2(h[k]);
    a[2 * k] += f.x;
    a[2 * k + 1] += f.y;
  }
}

// One lane's share of one pooled row: column slices v, v + 32, ... (kVecUnroll at a time),
// every load of a step issued before any is summed.
template <int CHUNK>
__device__ __forceinline__ void pool_row(const uint4* __restrict__ src, int64_t enc_ld_v, int cnt, int vec_per_row,
                                         int lane, uint4* __restrict__ dst) {
  const float fc = static_cast<float>(cnt);
  const bool exact = (cnt & (cnt - 1)) == 0;
  const float inv = exact ? 1.f / fc : 0.f;  // exact for a power of two
  for (int v0 = lane; v0 < vec_per_row; v0 += 32 * kVecUnroll) {
    if (CHUNK > 0) {
      uint4 x[kVecUnroll][CHUNK > 0 ? CHUNK : 1];
#pragma unroll
      for (int u = 0; u < kVecUnroll; ++u)
#pragma unroll
        for (int t = 0; t < (CHUNK > 0 ? CHUNK : 1); ++t)
          if (t < cnt && v0 + 32 * u < vec_per_row) x[u][t] = __ldg(src + t * enc_ld_v + v0 + 32 * u);
      // one slice at a time: sum, mean, store (keeps one slice's sums live)
#pragma unroll
      for (int u = 0; u < kVecUnroll; ++u) {
        if (v0 + 32 * u >= vec_per_row) break;
        float a[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) a[k] = 0.f;
#pragma unroll
        for (int t = 0; t < (CHUNK > 0 ? CHUNK : 1); ++t)
          if (t < cnt) add_bf16x8(a, x[u][t]);
        dst[v0 + 32 * u] = pack_mean(a, fc, inv, exact);
      }
    } else {
      // other chunk sizes: a run-time number of tokens, two at a time
      float a[kVecUnroll][8];
#pragma unroll
      for (int u = 0; u < kVecUnroll; ++u)
#pragma unroll
        for (int k = 0; k < 8; ++k) a[u][k] = 0.f;
      int t = 0;
      for (; t + 1 < cnt; t += 2) {
        uint4 x[kVecUnroll][2];
#pragma unroll
        for (int u = 0; u < kVecUnroll; ++u)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (v0 + 32 * u < vec_per_row) x[u][e] = __ldg(src + (t + e) * enc_ld_v + v0 + 32 * u);
#pragma unroll
        for (int u = 0; u < kVecUnroll; ++u)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (v0 + 32 * u < vec_per_row) add_bf16x8(a[u], x[u][e]);
      }
      if (t < cnt) {
#pragma unroll
        for (int u = 0; u < kVecUnroll; ++u)
          if (v0 + 32 * u < vec_per_row) add_bf16x8(a[u], __ldg(src + t * enc_ld_v + v0 + 32 * u));
      }
#pragma unroll
      for (int u = 0; u < kVecUnroll; ++u)
        if (v0 + 32 * u < vec_per_row) dst[v0 + 32 * u] = pack_mean(a[u], fc, inv, exact);
    }
  }
}

template <int CHUNK>
__global__ void __launch_bounds__(kPoolThreads, kPoolBlocksPerSm) chunk_pool_kernel(
    const uint4* __restrict__ enc, int64_t enc_ld_v, const int64_t* __restrict__ tok_off,
    const int32_t* __restrict__ len, int n_docs, int vec_per_row, int chunk_rt, uint4* __restrict__ pooled,
    int64_t pooled_ld_v, const int64_t* __restrict__ pool_off, int64_t total_rows, uint32_t* err) {
  pdl_launch_dependents();
  pdl_wait_predecessor();
  const int chunk = CHUNK > 0 ? CHUNK : chunk_rt;
  const int lane = threadIdx.x & 31;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * (kPoolThreads / 32);
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * (kPoolThreads / 32) + (threadIdx.x >> 5);
  // this warp's rows: a contiguous share of [0, total_rows)
  const int64_t per = (total_rows + n_warps - 1) / n_warps;
  int64_t r = gw * per;
  const int64_t r_end = min(total_rows, r + per);
  if (r >= r_end) return;
  int d = find_doc(pool_off, n_docs, r);
  int64_t d_begin = __ldg(pool_off + d), d_end = __ldg(pool_off + d + 1);
  for (; r < r_end; ++r) {
    while (r >= d_end && d + 1 < n_docs) {  // the row belongs to a later document (skips empty ones)
      ++d;
      d_begin = d_end;
      d_end = __ldg(pool_off + d + 1);
    }
    int n = __ldg(len + d);
    if (n > KALM_MAX_DOC_TOKENS) {
      if (lane == 0) record_error(err, kErrDeviceArg | kSitePool);
      n = KALM_MAX_DOC_TOKENS;
    }
    const int t0 = static_cast<int>(r - d_begin) * chunk;
    int cnt = n - t0;
    if (cnt > chunk) cnt = chunk;
    if (cnt <= 0 || r >= d_end) {  // pool_off inconsistent with len: flag, write nothing
      if (lane == 0) record_error(err, kErrDeviceArg | kSitePool);
      continue;
    }
    pool_row<CHUNK>(enc + (__ldg(tok_off + d) + t0) * enc_ld_v, enc_ld_v, cnt, vec_per_row, lane,
                    pooled + r * pooled_ld_v);
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
  // a few rows per warp, up to kPoolBlocksPerSm resident blocks per SM
  const int64_t warps = (total_pooled + kRowsPerWarp - 1) / kRowsPerWarp;
  int64_t blocks = (warps + kPoolThreads / 32 - 1) / (kPoolThreads / 32);
  const int64_t cap = static_cast<int64_t>(num_sms()) * kPoolBlocksPerSm;
  if (blocks > cap) blocks = cap;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* err = device_error_word();
  const uint4* e = reinterpret_cast<const uint4*>(enc);
  uint4* p = reinterpret_cast<uint4*>(pooled);
  // chunk 4 (the runtime contract) and 2 have unrolled kernels; other sizes take the generic loop
  const cudaError_t ce =
      chunk == 4   ? launch_pdl(chunk_pool_kernel<4>, dim3((unsigned)blocks), dim3(kPoolThreads), 0, s, e, enc_ld / 8, tok_off,
                                len, n_docs, vpr, chunk, p, pooled_ld / 8, pool_off, total_pooled, err)
      : chunk == 2 ? launch_pdl(chunk_pool_kernel<2>, dim3((unsigned)blocks), dim3(kPoolThreads), 0, s, e, enc_ld / 8, tok_off,
                                len, n_docs, vpr, chunk, p, pooled_ld / 8, pool_off, total_pooled, err)
                   : launch_pdl(chunk_pool_kernel<0>, dim3((unsigned)blocks), dim3(kPoolThreads), 0, s, e, enc_ld / 8, tok_off,
                                len, n_docs, vpr, chunk, p, pooled_ld / 8, pool_off, total_pooled, err);
  return check_cuda(ce, "launch chunk_pool_kernel");
}
