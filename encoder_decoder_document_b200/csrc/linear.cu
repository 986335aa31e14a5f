// Dense projection y = x . w^T (+ residual) on the 5th-generation tensor cores.
//
// Used for the cross-attention K/V projection of the cached pooled vectors
// ("KaLM-Reranker-V1-Nano - MLX", "What this is": cross-attention KV computed
// over the cached passage encodings) and for the synthetic decoder's Q/K/V and
// output projections.
//
// Design (sm_100a): a persistent, warp-specialised kernel, one CTA per SM.
//   warps 0-3   TMA producers: 128 x 64 tiles of x and BN x 64 tiles of w (128-byte
//               swizzle) into a STAGES-deep shared-memory ring.  A warp's tile
//               copies are served one after another, so the copies are spread
//               over four warps (x or w, even or odd k-block) to keep enough of
//               them in flight;
//   warp 4      allocates tensor memory and issues tcgen05.mma (M=128, N=BN,
//               K=16 per instruction) from one thread; tcgen05.commit frees a
//               ring slot once the tensor core has read it;
//   warps 5..8  epilogue: tcgen05.ld of the fp32 accumulator (one TMEM lane =
//               one output row per thread) in 32-column chunks, optional bf16
//               residual add (the residual chunk is fetched by TMA ahead of
//               time), one rounding to bf16, then the 32 x 32 chunk is staged in
//               shared memory (64-byte swizzle, bank-conflict free) and written
//               by a TMA tile store, so global writes are full lines.
// The accumulator is double-buffered in TMEM (2 x BN columns) so the epilogue
// of tile i overlaps the main loop of tile i+1.  Out-of-range rows/columns of
// x and w are zero-filled by TMA; the epilogue masks their stores.
#include "kalm.h"
#include "kalm_internal.h"
#include "kalm_ptx.cuh"

namespace kalm {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;  // one 128-byte swizzle row of bf16
constexpr int kProdWarps = 4;
constexpr int kMmaWarp = 4;
constexpr int kEpiWarp0 = 5;
constexpr int kThreads = 32 * (kEpiWarp0 + 4);

constexpr int kChunkBytes = 32 * 32 * 2;  // one 32-row x 32-column bf16 epilogue chunk

template <int BN>
struct LinearCfg {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BN * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_BYTES = 4 * 2 * kChunkBytes;  // per epilogue warp: 2 staging chunks
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 2 * EPI_BYTES + BAR_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static constexpr uint32_t IDESC = idesc_bf16_f32(kBM, BN, false, false);
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    linear_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                  const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_r,
                  bool has_residual, int M, int N, int K, uint64_t wait_ns, uint32_t* err) {
  using C = LinearCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint8_t* sOut = sB + C::STAGES * C::B_BYTES;  // [4 warps][2][32 x 32 bf16]
  uint8_t* sRes = sOut + C::EPI_BYTES;          // [4 warps][2][32 x 32 bf16]
  uint64_t* full = reinterpret_cast<uint64_t*>(sRes + C::EPI_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* res_full = acc_empty + 2;  // [4 warps][2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(res_full + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 2);  // the x copy and the w copy each arrive with their bytes
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    for (int b = 0; b < 8; ++b) mbar_init(&res_full[b], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_m = (M + kBM - 1) / kBM;
  const int n_n = (N + BN - 1) / BN;
  const int tiles = n_m * n_n;
  const int kblocks = (K + kBK - 1) / kBK;

  if (warp < kProdWarps) {
    if (lane == 0) {
      const bool is_w = warp >= 2;      // which operand this warp copies
      const uint32_t mine = warp & 1;   // which k-blocks (by parity of the running count)
      const CUtensorMap* tm = is_w ? &tm_w : &tm_x;
      tma_prefetch_desc(tm);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t it = 0;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
        const int m0 = (t / n_n) * kBM, n0 = (t % n_n) * BN;
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          if ((it & 1u) == mine) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, wait_ns)) {
              record_error(err, kErrTimeout | kSiteLinear);
              *abort_flag = 1;
              break;
            }
            if (is_w) {
              mbar_arrive_expect_tx(&full[stage], C::B_BYTES);
              tma_load_2d(sB + stage * C::B_BYTES, tm, &full[stage], kb * kBK, n0);
            } else {
              mbar_arrive_expect_tx(&full[stage], C::A_BYTES);
              tma_load_2d(sA + stage * C::A_BYTES, tm, &full[stage], kb * kBK, m0);
            }
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, wait_ns)) {
          record_error(err, kErrTimeout | kSiteLinear);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, wait_ns)) {
            record_error(err, kErrTimeout | kSiteLinear);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = a_base + stage * C::A_BYTES, b0 = b_base + stage * C::B_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b0 + kk * 32, 16, 1024);
            umma_bf16_ss(d_tmem, ad, bd, C::IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    // epilogue warps 5..8: warp w may access TMEM lanes 32*(w%4) .. 32*(w%4)+31
    const int quarter = warp & 3;
    const int ew = warp - kEpiWarp0;
    uint8_t* obuf = sOut + ew * 2 * kChunkBytes;
    uint8_t* rbuf = sRes + ew * 2 * kChunkBytes;
    uint64_t* rbar = res_full + ew * 2;
    uint32_t rphase = 0u;  // bit b: parity of residual buffer b
    int acc = 0;
    uint32_t acc_phase = 0;
    int out_slot = 0;
    // 64-byte swizzle of a 32 x 64 B chunk: 16-byte unit i of row r sits at unit i ^ ((r >> 1) & 3)
    const uint32_t swz = static_cast<uint32_t>((lane >> 1) & 3);
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int m0 = (t / n_n) * kBM, n0 = (t % n_n) * BN;
      const int row0 = m0 + quarter * 32;
      const int nch = min(BN, N - n0) / 32;
      if (has_residual && lane == 0) {
        for (int c = 0; c < 2 && c < nch; ++c) {
          mbar_arrive_expect_tx(&rbar[c], kChunkBytes);
          tma_load_2d(rbuf + c * kChunkBytes, &tm_r, &rbar[c], n0 + c * 32, row0);
        }
      }
      bool ok = mbar_wait(&acc_full[acc], acc_phase, wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok || *abort_flag) {
        if (lane == 0) record_error(err, kErrTimeout | kSiteLinear);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN);
#pragma unroll 1
      for (int c = 0; c < nch; ++c) {
        uint32_t r[32];
        tmem_ld32(t_row + c * 32, r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (has_residual) {
          const int b = c & 1;
          bool okr = mbar_wait(&rbar[b], (rphase >> b) & 1u, wait_ns);
          rphase ^= 1u << b;
          if (!__all_sync(0xffffffffu, okr)) {
            if (lane == 0) record_error(err, kErrTimeout | kSiteLinear);
            *abort_flag = 1;
            break;
          }
          const uint8_t* rrow = rbuf + b * kChunkBytes + lane * 64;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 rv = *reinterpret_cast<const uint4*>(rrow + ((q ^ swz) << 4));
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&rv);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f = __bfloat1622float2(h[k]);
              v[q * 8 + 2 * k] += f.x;
              v[q * 8 + 2 * k + 1] += f.y;
            }
          }
          __syncwarp();
          if (lane == 0 && c + 2 < nch) {  // refill this residual buffer two chunks ahead
            mbar_arrive_expect_tx(&rbar[b], kChunkBytes);
            tma_load_2d(rbuf + b * kChunkBytes, &tm_r, &rbar[b], n0 + (c + 2) * 32, row0);
          }
        }
        // the staging slot is free once the store issued from it two chunks ago has read it
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        uint8_t* orow = obuf + out_slot * kChunkBytes + lane * 64;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 o;
          o.x = pack_bf16x2(v[q * 8 + 0], v[q * 8 + 1]);
          o.y = pack_bf16x2(v[q * 8 + 2], v[q * 8 + 3]);
          o.z = pack_bf16x2(v[q * 8 + 4], v[q * 8 + 5]);
          o.w = pack_bf16x2(v[q * 8 + 6], v[q * 8 + 7]);
          *reinterpret_cast<uint4*>(orow + ((q ^ swz) << 4)) = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_y, obuf + out_slot * kChunkBytes, n0 + c * 32, row0);
          bulk_commit_group();
        }
        out_slot ^= 1;
      }
      if (*abort_flag) break;
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_group<0>();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

int g_num_sms[64] = {0};

}  // namespace

kalm_status setup_linear_kernels() {
  kalm_status st = check_cuda(cudaFuncSetAttribute(linear_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   LinearCfg<256>::SMEM),
                              "cudaFuncSetAttribute(linear_kernel<256>)");
  if (st != KALM_OK) return st;
  st = check_cuda(cudaFuncSetAttribute(linear_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       LinearCfg<128>::SMEM),
                  "cudaFuncSetAttribute(linear_kernel<128>)");
  if (st != KALM_OK) return st;
  int dev = 0;
  cudaGetDevice(&dev);
  int sms = 0;
  st = check_cuda(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "SM count");
  if (st != KALM_OK) return st;
  if (dev < 64) g_num_sms[dev] = sms;
  return KALM_OK;
}

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev < 64 && g_num_sms[dev] > 0) ? g_num_sms[dev] : 148;
}

// Shared by kalm_linear and kalm_cross_kv_proj.
kalm_status launch_linear(const kalm_bf16* x, int64_t ldx, const kalm_bf16* w, int64_t ldw, const kalm_bf16* residual,
                          int64_t ldr, kalm_bf16* y, int64_t ldy, int64_t m, int32_t n, int32_t k,
                          cudaStream_t stream, const char* who) {
  if (m < 0 || n <= 0 || k <= 0) return fail(KALM_ERR_INVALID_ARG, "%s: m=%lld n=%d k=%d", who, (long long)m, n, k);
  if (m == 0) return KALM_OK;
  if (m > INT32_MAX - 256) return fail(KALM_ERR_INVALID_ARG, "%s: m=%lld too large", who, (long long)m);
  if (!x || !w || !y) return fail(KALM_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (n % 32) return fail(KALM_ERR_UNSUPPORTED, "%s: n=%d must be a multiple of 32", who, n);
  if (k % 8) return fail(KALM_ERR_INVALID_ARG, "%s: k=%d must be a multiple of 8", who, k);
  if (ldx % 8 || ldw % 8 || ldy % 8 || (residual && ldr % 8) || ldx < k || ldw < k || ldy < n ||
      (residual && ldr < n))
    return fail(KALM_ERR_INVALID_ARG, "%s: strides must be multiples of 8 and >= the row width", who);
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || (residual && !aligned16(residual)))
    return fail(KALM_ERR_INVALID_ARG, "%s: bf16 pointers must be 16-byte aligned", who);
  const bool wide = (n % 256) == 0;
  const int BN = wide ? 256 : 128;
  CUtensorMap tx, tw;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(k), static_cast<uint64_t>(m)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ldx) * 2};
    const uint32_t box[2] = {kBK, kBM};
    kalm_status st = make_tmap_bf16(&tx, x, 2, dims, strides, box);
    if (st != KALM_OK) return st;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(k), static_cast<uint64_t>(n)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ldw) * 2};
    const uint32_t box[2] = {kBK, static_cast<uint32_t>(BN)};
    kalm_status st = make_tmap_bf16(&tw, w, 2, dims, strides, box);
    if (st != KALM_OK) return st;
  }
  CUtensorMap ty, tr;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(n), static_cast<uint64_t>(m)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ldy) * 2};
    const uint32_t box[2] = {32, 32};
    kalm_status st = make_tmap_bf16(&ty, y, 2, dims, strides, box, 64);
    if (st != KALM_OK) return st;
    if (residual) {
      const uint64_t rstrides[1] = {static_cast<uint64_t>(ldr) * 2};
      st = make_tmap_bf16(&tr, residual, 2, dims, rstrides, box, 64);
      if (st != KALM_OK) return st;
    } else {
      tr = ty;  // never read
    }
  }
  const int64_t tiles = ((m + kBM - 1) / kBM) * ((n + BN - 1) / BN);
  const int grid = static_cast<int>(tiles < num_sms() ? tiles : num_sms());
  const bool has_r = residual != nullptr;
  if (wide)
    linear_kernel<256><<<grid, kThreads, LinearCfg<256>::SMEM, stream>>>(tx, tw, ty, tr, has_r, (int)m, n, k,
                                                                          kWaitNs, device_error_word());
  else
    linear_kernel<128><<<grid, kThreads, LinearCfg<128>::SMEM, stream>>>(tx, tw, ty, tr, has_r, (int)m, n, k,
                                                                          kWaitNs, device_error_word());
  return check_cuda(cudaGetLastError(), "launch linear_kernel");
}

}  // namespace kalm

using namespace kalm;

extern "C" kalm_status kalm_linear(const kalm_bf16* x, int64_t ldx, const kalm_bf16* w, int64_t ldw,
                                   const kalm_bf16* residual, int64_t ldr, kalm_bf16* y, int64_t ldy, int64_t m,
                                   int32_t n, int32_t k, kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  return launch_linear(x, ldx, w, ldw, residual, ldr, y, ldy, m, n, k, static_cast<cudaStream_t>(stream),
                       "kalm_linear");
}

extern "C" kalm_status kalm_cross_kv_proj(const kalm_bf16* pooled, int64_t pooled_ld, int64_t total_pooled,
                                          int32_t hidden, const kalm_bf16* w_kv, int32_t n_layers, int32_t n_kv,
                                          int32_t head_dim, kalm_bf16* kv_cross, kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (n_layers <= 0 || n_kv <= 0 || head_dim <= 0 || hidden <= 0 || total_pooled < 0)
    return fail(KALM_ERR_INVALID_ARG, "kalm_cross_kv_proj: bad sizes");
  const int64_t n = static_cast<int64_t>(n_layers) * 2 * n_kv * head_dim;
  if (n > INT32_MAX) return fail(KALM_ERR_INVALID_ARG, "kalm_cross_kv_proj: output width too large");
  return launch_linear(pooled, pooled_ld, w_kv, hidden, nullptr, 0, kv_cross, n, total_pooled,
                       static_cast<int32_t>(n), hidden, static_cast<cudaStream_t>(stream), "kalm_cross_kv_proj");
}
