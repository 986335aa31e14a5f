// Rotary position embedding of the decoder's self Q and K, in place.
// "KaLM-Reranker-V1-Nano - MLX (Apple Silicon)", "Derivation": the rotary
// parameters and inverse-frequency tables come from the model config.  Element
// i (< D/2) of a head vector pairs with element i + D/2 and the pair turns by
// pos * theta^(-2i/D), pos being the row's position in its document's decoder
// stream (row - q_off[d]).
//
// Memory-bound elementwise kernel: one thread rotates 8 consecutive pairs of one
// head of one row (two 16-byte loads, two 16-byte stores).  Consecutive threads
// take consecutive pair groups of a row, so a warp covers two heads of a row in
// contiguous 16-byte runs.  fp32 arithmetic: the frequency from exp2 of the
// exact exponent, the angle's sine and cosine after a reduction by 2*pi, one
// bf16 rounding.
#include <cmath>

#include "kalm.h"
#include "kalm_internal.h"
#include "kalm_ptx.cuh"

namespace kalm {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) rope_kernel(uint4* __restrict__ x, int64_t ldx_v, int64_t rows,
                                                        int n_heads, int half_v, const int64_t* __restrict__ q_off,
                                                        int n_docs, float log2_theta, float inv_half_d,
                                                        uint32_t* err) {
  pdl_launch_dependents();
  pdl_wait_predecessor();
  const int64_t per_row = static_cast<int64_t>(n_heads) * half_v;
  const int64_t total = rows * per_row;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t r = i / per_row;
    const int rem = static_cast<int>(i - r * per_row);
    const int h = rem / half_v, g = rem - h * half_v;  // head, group of 8 pairs
    // document of row r: the largest d with q_off[d] <= r
    int lo = 0, hi = n_docs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(q_off + mid) <= r) lo = mid; else hi = mid - 1;
    }
    const int64_t pos64 = r - __ldg(q_off + lo);
    if (pos64 < 0 || pos64 >= KALM_MAX_QUERY_TOKENS) {  // row outside the offsets: flag, leave it
      record_error(err, kErrDeviceArg | kSiteRope);
      continue;
    }
    const float pos = static_cast<float>(pos64);
    uint4* base = x + r * ldx_v + static_cast<int64_t>(h) * (2 * half_v);
    uint4 va = base[g], vb = base[g + half_v];
    __nv_bfloat162* a2 = reinterpret_cast<__nv_bfloat162*>(&va);
    __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&vb);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 a = __bfloat1622float2(a2[k]);
      const float2 b = __bfloat1622float2(b2[k]);
      const int p0 = g * 8 + 2 * k;  // pair index of the first element
      float ra0, rb0, ra1, rb1;
      rope_pair(pos, p0, inv_half_d, log2_theta, a.x, b.x, &ra0, &rb0);
      rope_pair(pos, p0 + 1, inv_half_d, log2_theta, a.y, b.y, &ra1, &rb1);
      a2[k] = __floats2bfloat162_rn(ra0, ra1);
      b2[k] = __floats2bfloat162_rn(rb0, rb1);
    }
    base[g] = va;
    base[g + half_v] = vb;
  }
}

// Table of (cos, sin) for every decoder position below KALM_MAX_QUERY_TOKENS and
// every pair of a head, the same values rope_pair computes, so a kernel that looks
// them up rotates to the same bits.  Layout: float4 [half/2][KALM_MAX_QUERY_TOKENS],
// entry [q][pos] = (cos, sin) of pair 2q then of pair 2q + 1: threads holding
// consecutive positions read consecutive 16-byte entries.
__global__ void __launch_bounds__(kThreads) rope_table_kernel(float2* __restrict__ table, int total,
                                                              float log2_theta, float inv_half_d) {
  pdl_launch_dependents();
  pdl_wait_predecessor();
  for (int i = blockIdx.x * kThreads + threadIdx.x; i < total; i += gridDim.x * kThreads) {
    const int p = i / KALM_MAX_QUERY_TOKENS, pos = i - p * KALM_MAX_QUERY_TOKENS;
    float sn, cs;
    rope_angle(static_cast<float>(pos), p, inv_half_d, log2_theta, &sn, &cs);
    table[((p >> 1) * KALM_MAX_QUERY_TOKENS + pos) * 2 + (p & 1)] = make_float2(cs, sn);
  }
}

}  // namespace
}  // namespace kalm

using namespace kalm;

extern "C" kalm_status kalm_rope(kalm_bf16* x, int64_t ldx, int64_t rows, int32_t n_heads, int32_t head_dim,
                                 const int64_t* q_off, int32_t n_docs, float theta, kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (rows < 0 || n_heads <= 0 || n_docs < 0 || head_dim <= 0 || head_dim % 16)
    return fail(KALM_ERR_INVALID_ARG, "kalm_rope: rows=%lld n_heads=%d head_dim=%d n_docs=%d", (long long)rows,
                n_heads, head_dim, n_docs);
  if (ldx % 8 || ldx < static_cast<int64_t>(n_heads) * head_dim)
    return fail(KALM_ERR_INVALID_ARG, "kalm_rope: ldx=%lld must be a multiple of 8 covering all heads",
                (long long)ldx);
  if (!(theta > 1.f) || !std::isfinite(theta)) return fail(KALM_ERR_INVALID_ARG, "kalm_rope: theta must be > 1");
  if (rows == 0 || n_docs == 0) return KALM_OK;
  if (!x || !q_off) return fail(KALM_ERR_INVALID_ARG, "kalm_rope: NULL pointer");
  if (!aligned16(x)) return fail(KALM_ERR_INVALID_ARG, "kalm_rope: x must be 16-byte aligned");
  const int half_v = head_dim / 16;  // 8-pair groups per head
  const int64_t total = rows * n_heads * half_v;
  int64_t blocks = (total + kThreads - 1) / kThreads;
  if (blocks > static_cast<int64_t>(num_sms()) * 16) blocks = static_cast<int64_t>(num_sms()) * 16;
  return check_cuda(launch_pdl(rope_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0,
                               static_cast<cudaStream_t>(stream), reinterpret_cast<uint4*>(x), ldx / 8, rows, n_heads,
                               half_v, q_off, n_docs, log2f(theta), 2.0f / static_cast<float>(head_dim),
                               device_error_word()),
                    "launch rope_kernel");
}

extern "C" kalm_status kalm_rope_table(float theta, int32_t head_dim, float* table, kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (head_dim <= 0 || head_dim % 16) return fail(KALM_ERR_INVALID_ARG, "kalm_rope_table: head_dim=%d", head_dim);
  if (!(theta > 1.f) || !std::isfinite(theta)) return fail(KALM_ERR_INVALID_ARG, "kalm_rope_table: theta must be > 1");
  if (!table || !aligned16(table))
    return fail(KALM_ERR_INVALID_ARG, "kalm_rope_table: table must be non-NULL and 16-byte aligned");
  const int half = head_dim / 2, total = KALM_MAX_QUERY_TOKENS * half;
  const int blocks = (total + kThreads - 1) / kThreads;
  return check_cuda(launch_pdl(rope_table_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0,
                               static_cast<cudaStream_t>(stream), reinterpret_cast<float2*>(table), total,
                               log2f(theta), 2.0f / static_cast<float>(head_dim)),
                    "launch rope_table_kernel");
}
