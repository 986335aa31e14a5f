// Step 4: yes/no readout at each document's final decoder position.
// "KaLM-Reranker-V1-Nano - MLX", "What this is": score = softmax([logit_yes,
// logit_no])[yes] read at the final position; "KaLM-Reranker-V1-Small-Q4_K_M-
// GGUF", "Score a pair": margin = yes - no and score = sigmoid(margin).
//
// One warp per document: 16-byte loads of the final hidden row and of the two
// readout rows, fp32 dot products, a shuffle-tree reduction, and the logistic
// function evaluated without overflow.
#include "kalm.h"
#include "kalm_internal.h"
#include "kalm_ptx.cuh"

namespace kalm {
namespace {

__global__ void __launch_bounds__(128) yes_no_kernel(const uint4* __restrict__ hidden, int64_t ldh_v,
                                                     const int64_t* __restrict__ q_off, int n_docs, int vec,
                                                     const uint4* __restrict__ w_yes, const uint4* __restrict__ w_no,
                                                     float* __restrict__ yes, float* __restrict__ no,
                                                     float* __restrict__ margin, float* __restrict__ score) {
  pdl_launch_dependents();
  pdl_wait_predecessor();
  const int lane = threadIdx.x & 31;
  const int d = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (d >= n_docs) return;
  const int64_t a = q_off[d], b = q_off[d + 1];
  float sy = 0.f, sn = 0.f;
  if (b > a) {
    const uint4* x = hidden + (b - 1) * ldh_v;
    for (int v = lane; v < vec; v += 32) {
      const uint4 xv = __ldg(x + v), yv = __ldg(w_yes + v), nv = __ldg(w_no + v);
      const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xv);
      const __nv_bfloat162* yh = reinterpret_cast<const __nv_bfloat162*>(&yv);
      const __nv_bfloat162* nh = reinterpret_cast<const __nv_bfloat162*>(&nv);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 xf = __bfloat1622float2(xh[k]);
        const float2 yf = __bfloat1622float2(yh[k]);
        const float2 nf = __bfloat1622float2(nh[k]);
        sy = fmaf(xf.x, yf.x, sy);
        sy = fmaf(xf.y, yf.y, sy);
        sn = fmaf(xf.x, nf.x, sn);
        sn = fmaf(xf.y, nf.y, sn);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sy += __shfl_xor_sync(0xffffffffu, sy, o);
    sn += __shfl_xor_sync(0xffffffffu, sn, o);
  }
  if (lane == 0) {
    const float m = sy - sn;
    float s;
    if (m >= 0.f) {
      s = 1.f / (1.f + expf(-m));
    } else {
      const float e = expf(m);
      s = e / (1.f + e);
    }
    yes[d] = sy;
    no[d] = sn;
    if (margin) margin[d] = m;
    score[d] = s;
  }
}

}  // namespace
}  // namespace kalm

using namespace kalm;

extern "C" kalm_status kalm_yes_no_score(const kalm_bf16* hidden, int64_t ldh, const int64_t* q_off, int32_t n_docs,
                                         int32_t hidden_dim, const kalm_bf16* w_yes, const kalm_bf16* w_no,
                                         float* yes, float* no, float* margin, float* score, kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (n_docs < 0 || hidden_dim <= 0 || hidden_dim % 8 || ldh % 8 || ldh < hidden_dim)
    return fail(KALM_ERR_INVALID_ARG, "kalm_yes_no_score: n_docs=%d hidden=%d ldh=%lld", n_docs, hidden_dim,
                (long long)ldh);
  if (n_docs == 0) return KALM_OK;
  if (!hidden || !q_off || !w_yes || !w_no || !yes || !no || !score)
    return fail(KALM_ERR_INVALID_ARG, "kalm_yes_no_score: NULL pointer");
  if (!aligned16(hidden) || !aligned16(w_yes) || !aligned16(w_no))
    return fail(KALM_ERR_INVALID_ARG, "kalm_yes_no_score: bf16 pointers must be 16-byte aligned");
  const unsigned blocks = (unsigned)((n_docs + 3) / 4);
  return check_cuda(launch_pdl(yes_no_kernel, dim3(blocks), dim3(128), 0, static_cast<cudaStream_t>(stream),
                                reinterpret_cast<const uint4*>(hidden), ldh / 8, q_off, n_docs, hidden_dim / 8,
                                reinterpret_cast<const uint4*>(w_yes), reinterpret_cast<const uint4*>(w_no), yes,
                                no, margin, score),
                    "launch yes_no_kernel");
}
