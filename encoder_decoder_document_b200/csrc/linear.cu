// Dense projection y = x . w^T (+ residual) on the 5th-generation tensor cores.
//
// Used for the cross-attention K/V projection of the cached pooled vectors
// ("KaLM-Reranker-V1-Nano - MLX", "What this is": cross-attention KV computed
// over the cached passage encodings) and for the synthetic decoder's Q/K/V and
// output projections.
//
// Design (sm_100a): a persistent, warp-specialised kernel, one CTA per SM.
//   warps 0-1   TMA producers: 128 x 64 tiles of x (warp 0) and BN x 64 tiles of w
//               (warp 1, 128-byte swizzle) into a STAGES-deep shared-memory ring;
//   warp 2      allocates tensor memory and issues tcgen05.mma (M=128, N=BN,
//               K=16 per instruction) from one thread; tcgen05.commit frees a
//               ring slot once the tensor core has read it;
//   warps 3..6  epilogue: tcgen05.ld of the fp32 accumulator (one TMEM lane =
//               one output row per thread) in 32-column chunks, optional bf16
//               residual add (the residual chunk is fetched by TMA ahead of
//               time), one rounding to bf16, then the 32 x 32 chunk is staged in
//               shared memory (64-byte swizzle, bank-conflict free) and written
//               by a TMA tile store, so global writes are full lines.
// The accumulator is double-buffered in TMEM (2 x BN columns) so the epilogue
// of tile i overlaps the main loop of tile i+1.  Out-of-range rows/columns of
// x and w are zero-filled by TMA; the epilogue masks their stores.
// With a rotary table (Q|K|V projection) a 256-column tile is one head: the
// epilogue pairs chunk c with chunk c + 4 and turns them by the row's angles,
// read from a position-minor table (coalesced across a warp's consecutive rows)
// one chunk ahead of their use.  Seven warps leave 224 registers a thread for that.
#include <cmath>

#include "kalm.h"
#include "kalm_internal.h"
#include "kalm_ptx.cuh"

namespace kalm {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;  // one 128-byte swizzle row of bf16
constexpr int kProdWarps = 2;  // warp 0 copies x tiles, warp 1 w tiles
constexpr int kMmaWarp = 2;
constexpr int kEpiWarp0 = 3;
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

// Residual prefetch of the first two 32-column chunks of a tile (one lane per warp).
__device__ __forceinline__ void epi_prefetch_residual(const CUtensorMap* tm_r, uint8_t* rbuf, uint64_t* rbar,
                                                      int nch, int n0, int row0) {
  for (int c = 0; c < 2 && c < nch; ++c) {
    mbar_arrive_expect_tx(&rbar[c], kChunkBytes);
    tma_load_2d(rbuf + c * kChunkBytes, tm_r, &rbar[c], n0 + c * 32, row0);
  }
}

// Optional rotary embedding applied in the epilogue of a Q|K|V projection: output
// columns [0, rot_cols) are head vectors of 256 elements (one 256-column tile is one
// head) rotated by the row's decoder position (row - q_off[d] for its document d).
struct RopeArgs {
  const int64_t* q_off;
  int n_docs;
  int rot_cols;          // 0: no rotation
  const float4* table;   // angles: [64][KALM_MAX_QUERY_TOKENS], entry [q][pos] = (cos, sin) of pairs 2q, 2q+1
  int64_t rows;          // M: rows past it are clipped by the store
  uint32_t* err;         // device error word: a stored row whose position is out of range
};

// One 32-column chunk of one warp's 32 rows: bf16 into a 64-byte-swizzled staging
// slot, then a TMA tile store.  The slot is reused once the store issued from it two
// chunks ago has read it.
__device__ __forceinline__ void epi_emit(const float (&v)[32], int col, int row0, const CUtensorMap* tm_y,
                                         uint8_t* obuf, int& out_slot, int lane) {
  // 64-byte swizzle of a 32 x 64 B chunk: 16-byte unit i of row r sits at unit i ^ ((r >> 1) & 3)
  const uint32_t swz = static_cast<uint32_t>((lane >> 1) & 3);
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
    tma_store_2d(tm_y, obuf + out_slot * kChunkBytes, col, row0);
    bulk_commit_group();
  }
  out_slot ^= 1;
}

// Row of the angle table for this lane's row of a tile whose columns are rotated
// heads, or -1 when the tile is not rotated.  Called before the accumulator wait,
// so the offsets search overlaps the tile's MMAs.  A row past the last document
// (clipped by the store) reads position 0; a stored row whose position is out of
// range is flagged.
__device__ __forceinline__ int rope_row(const RopeArgs& rope, int n0, int nch, int row0, int lane) {
  if (!(n0 < rope.rot_cols && nch == 8)) return -1;
  const int64_t m = row0 + lane;
  int lo = 0, hi = rope.n_docs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(rope.q_off + mid) <= m) lo = mid; else hi = mid - 1;
  }
  const int64_t pos64 = m - __ldg(rope.q_off + lo);
  const bool in_range = pos64 >= 0 && pos64 < KALM_MAX_QUERY_TOKENS;
  if (m < rope.rows && !in_range) record_error(rope.err, kErrDeviceArg | kSiteRope);
  return in_range ? static_cast<int>(pos64) : 0;
}

// The first 32 pairs' angles of a rotated tile's row, loaded before the
// accumulator wait so that their latency hides behind the tile's MMAs.
__device__ __forceinline__ void rope_prefetch(const RopeArgs& rope, int rope_pos, float4 (&cs)[16]) {
  if (rope_pos >= 0) {
#pragma unroll
    for (int j = 0; j < 16; ++j) cs[j] = __ldg(rope.table + j * KALM_MAX_QUERY_TOKENS + rope_pos);
  }
}

// Epilogue of one tile for one warp: 32 rows (TMEM lanes of this warp) x nch
// 32-column chunks.  fp32 accumulator (+ residual) -> bf16 -> swizzled staging
// chunk -> TMA tile store.  A tile of rotated heads pairs chunk c with chunk c + 4
// (element i with element i + 128): both are rounded to bf16 (the stored
// projection), rotated in fp32 and rounded again.  Returns false if a bounded wait
// expired.
__device__ __forceinline__ bool epi_tile(uint32_t t_row, int nch, int n0, int row0, bool has_residual,
                                         const CUtensorMap* tm_y, const CUtensorMap* tm_r, uint8_t* obuf,
                                         uint8_t* rbuf, uint64_t* rbar, uint32_t& rphase, int& out_slot, int lane,
                                         uint64_t wait_ns, const RopeArgs& rope, int rope_pos, float4 (&cs)[16]) {
  if (rope_pos >= 0) {
    const float4* tcol = rope.table + rope_pos;  // lanes at consecutive positions read consecutive entries
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t ra[32], rb[32];
      tmem_ld32(t_row + c * 32, ra);
      tmem_ld32(t_row + (c + 4) * 32, rb);
      float4 nx[16];  // the next chunk's angles, in flight while this chunk is turned
      if (c < 3) {
#pragma unroll
        for (int j = 0; j < 16; ++j) nx[j] = __ldg(tcol + ((c + 1) * 16 + j) * KALM_MAX_QUERY_TOKENS);
      }
      tmem_ld_wait();
      float va[32], vb[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float a0 = __bfloat162float(__float2bfloat16_rn(__uint_as_float(ra[2 * j])));
        const float b0 = __bfloat162float(__float2bfloat16_rn(__uint_as_float(rb[2 * j])));
        const float a1 = __bfloat162float(__float2bfloat16_rn(__uint_as_float(ra[2 * j + 1])));
        const float b1 = __bfloat162float(__float2bfloat16_rn(__uint_as_float(rb[2 * j + 1])));
        rope_turn(a0, b0, cs[j].x, cs[j].y, &va[2 * j], &vb[2 * j]);
        rope_turn(a1, b1, cs[j].z, cs[j].w, &va[2 * j + 1], &vb[2 * j + 1]);
      }
      epi_emit(va, n0 + c * 32, row0, tm_y, obuf, out_slot, lane);
      epi_emit(vb, n0 + (c + 4) * 32, row0, tm_y, obuf, out_slot, lane);
#pragma unroll
      for (int j = 0; j < 16; ++j) cs[j] = nx[j];
    }
    return true;
  }
  // 64-byte swizzle of a 32 x 64 B chunk: 16-byte unit i of row r sits at unit i ^ ((r >> 1) & 3)
  const uint32_t swz = static_cast<uint32_t>((lane >> 1) & 3);
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
      const bool okr = mbar_wait(&rbar[b], (rphase >> b) & 1u, wait_ns);
      rphase ^= 1u << b;
      if (!__all_sync(0xffffffffu, okr)) return false;
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
        tma_load_2d(rbuf + b * kChunkBytes, tm_r, &rbar[b], n0 + (c + 2) * 32, row0);
      }
    }
    epi_emit(v, n0 + c * 32, row0, tm_y, obuf, out_slot, lane);
  }
  return true;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    linear_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                  const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_r,
                  bool has_residual, int M, int N, int K, uint64_t wait_ns, uint32_t* err, const RopeArgs rope) {
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
  pdl_launch_dependents();
  pdl_wait_predecessor();  // inputs of this GEMM are written by the previous kernel

  const int n_m = (M + kBM - 1) / kBM;
  const int n_n = (N + BN - 1) / BN;
  const int tiles = n_m * n_n;
  const int kblocks = (K + kBK - 1) / kBK;

  if (warp < kProdWarps) {
    if (lane == 0) {
      const bool is_w = warp == 1;  // which operand this warp copies
      const CUtensorMap* tm = is_w ? &tm_w : &tm_x;
      tma_prefetch_desc(tm);
      int stage = 0;
      uint32_t phase = 0;
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
        const int m0 = (t / n_n) * kBM, n0 = (t % n_n) * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
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
    // epilogue warps 3..6: warp w may access TMEM lanes 32*(w%4) .. 32*(w%4)+31
    const int quarter = warp & 3;
    const int ew = warp - kEpiWarp0;
    uint8_t* obuf = sOut + ew * 2 * kChunkBytes;
    uint8_t* rbuf = sRes + ew * 2 * kChunkBytes;
    uint64_t* rbar = res_full + ew * 2;
    uint32_t rphase = 0u;  // bit b: parity of residual buffer b
    int acc = 0;
    uint32_t acc_phase = 0;
    int out_slot = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      const int m0 = (t / n_n) * kBM, n0 = (t % n_n) * BN;
      const int row0 = m0 + quarter * 32;
      const int nch = min(BN, N - n0) / 32;
      if (has_residual && lane == 0) epi_prefetch_residual(&tm_r, rbuf, rbar, nch, n0, row0);
      const int rpos = rope_row(rope, n0, nch, row0, lane);
      float4 cs[16];
      rope_prefetch(rope, rpos, cs);
      bool ok = mbar_wait(&acc_full[acc], acc_phase, wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (ok && !*abort_flag) {
        tc_fence_after();
        const uint32_t t_row =
            tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN);
        ok = epi_tile(t_row, nch, n0, row0, has_residual, &tm_y, &tm_r, obuf, rbuf, rbar, rphase, out_slot, lane,
                      wait_ns, rope, rpos, cs);
      }
      if (!ok || *abort_flag) {
        if (lane == 0) record_error(err, kErrTimeout | kSiteLinear);
        *abort_flag = 1;
        break;
      }
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

// ---------------------------------------------------------------------------
// CTA-pair variant: a 2-CTA cluster computes a 256 x BN tile with tcgen05.mma
// cta_group::2.  Each CTA fetches its own 128 rows of x and its own BN/2 rows of
// w, so every SM moves fewer operand bytes per FLOP than a 128 x BN tile on one
// SM; the even CTA issues the MMAs, its commits arrive on both CTAs' barriers.
// ---------------------------------------------------------------------------
template <int BN>
struct Linear2Cfg {
  static constexpr int BNH = BN / 2;
  static constexpr int A_BYTES = kBM * kBK * 2;
  static constexpr int B_BYTES = BNH * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_BYTES = 4 * 2 * kChunkBytes;
  static constexpr int BAR_BYTES = 256;
  static constexpr int STAGES_FIT = (232448 - 1024 - BAR_BYTES - 2 * EPI_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 2 * EPI_BYTES + BAR_BYTES;
  static constexpr uint32_t TMEM_COLS = 512;  // two accumulators at columns 0 and 256
  static constexpr uint32_t ACC_STRIDE = 256;
  static constexpr uint32_t IDESC = idesc_bf16_f32(2 * kBM, BN, false, false);
  static_assert(BNH % 8 == 0, "B half-tile must be whole 8-row groups");
};

template <int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    linear_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                       const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_r,
                       bool has_residual, int M, int N, int K, uint64_t wait_ns, uint32_t* err, const RopeArgs rope) {
  using C = Linear2Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint8_t* sOut = sB + C::STAGES * C::B_BYTES;
  uint8_t* sRes = sOut + C::EPI_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sRes + C::EPI_BYTES);  // used in the even CTA
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;  // used in the even CTA
  uint64_t* res_full = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(res_full + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 2);  // the even CTA's x copy and w copy arrive with both CTAs' bytes
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);  // one arrival per epilogue warp of both CTAs
    }
    for (int b = 0; b < 8; ++b) mbar_init(&res_full[b], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait_predecessor();  // inputs of this GEMM are written by the previous kernel

  const int n_m = (M + 2 * kBM - 1) / (2 * kBM);
  const int n_n = (N + BN - 1) / BN;
  const int tiles = n_m * n_n;
  const int kblocks = (K + kBK - 1) / kBK;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (warp < kProdWarps) {
    if (lane == 0) {
      const bool is_w = warp == 1;
      const CUtensorMap* tm = is_w ? &tm_w : &tm_x;
      tma_prefetch_desc(tm);
      const uint32_t full0 = map_to_rank(smem_u32(full), 0);  // the even CTA's full barriers
      int stage = 0;
      uint32_t phase = 0;
      for (int t = pair; t < tiles && !*abort_flag; t += n_pairs) {
        const int m0 = (t / n_n) * 2 * kBM + static_cast<int>(rank) * kBM;
        const int n0 = (t % n_n) * BN + static_cast<int>(rank) * C::BNH;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, wait_ns)) {
            record_error(err, kErrTimeout | kSiteLinear);
            *abort_flag = 1;
            break;
          }
          const uint32_t bar = full0 + stage * 8;
          if (is_w) {
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::B_BYTES);
            tma_load_2d_pair(sB + stage * C::B_BYTES, tm, bar, kb * kBK, n0);
          } else {
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::A_BYTES);
            tma_load_2d_pair(sA + stage * C::A_BYTES, tm, bar, kb * kBK, m0);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      for (int t = pair; t < tiles && !*abort_flag; t += n_pairs) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, wait_ns)) {
          record_error(err, kErrTimeout | kSiteLinear);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc) * C::ACC_STRIDE;
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
            umma_bf16_ss_pair(d_tmem, ad, bd, C::IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair_multicast(&empty[stage], 0x3);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_multicast(&acc_full[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    // epilogue warps: this CTA's 128 rows of the pair tile
    const int quarter = warp & 3;
    const int ew = warp - kEpiWarp0;
    uint8_t* obuf = sOut + ew * 2 * kChunkBytes;
    uint8_t* rbuf = sRes + ew * 2 * kChunkBytes;
    uint64_t* rbar = res_full + ew * 2;
    const uint32_t acc_empty0 = map_to_rank(smem_u32(acc_empty), 0);
    uint32_t rphase = 0u;
    int acc = 0;
    uint32_t acc_phase = 0;
    int out_slot = 0;
    for (int t = pair; t < tiles; t += n_pairs) {
      const int m0 = (t / n_n) * 2 * kBM + static_cast<int>(rank) * kBM, n0 = (t % n_n) * BN;
      const int row0 = m0 + quarter * 32;
      const int nch = min(BN, N - n0) / 32;
      if (has_residual && lane == 0) epi_prefetch_residual(&tm_r, rbuf, rbar, nch, n0, row0);
      const int rpos = rope_row(rope, n0, nch, row0, lane);
      float4 cs[16];
      rope_prefetch(rope, rpos, cs);
      bool ok = mbar_wait(&acc_full[acc], acc_phase, wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (ok && !*abort_flag) {
        tc_fence_after();
        const uint32_t t_row =
            tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc) * C::ACC_STRIDE;
        ok = epi_tile(t_row, nch, n0, row0, has_residual, &tm_y, &tm_r, obuf, rbuf, rbar, rphase, out_slot, lane,
                      wait_ns, rope, rpos, cs);
      }
      if (!ok || *abort_flag) {
        if (lane == 0) record_error(err, kErrTimeout | kSiteLinear);
        *abort_flag = 1;
        break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + acc * 8);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (lane == 0) bulk_wait_group<0>();
  }
  tc_fence_before();
  cluster_sync_all();  // the peer's shared memory is read by the pair MMAs until here
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Two chained pair GEMMs in one persistent launch: Y1 = X1 . W1^T + R1 (the output
// projection with its residual, written in place), then Y2 = Y1 . W2^T (the next
// layer's Q|K|V projection).  Every tile is 256 rows (one CTA pair) by its phase's
// width (a runtime value up to 256); the launch walks the phase-1 tiles first and
// then the phase-2 tiles in row-block order, round robin over the pairs, so each
// pair finishes issuing its phase-1 tiles before it reaches a phase-2 tile.
// A phase-2 tile reads its 256 rows of Y1 only once every phase-1 tile of that row
// block has stored them: each epilogue warp of a phase-1 tile waits for its own tile
// stores to complete and adds 1 to the row block's counter (gpu-scope release), and
// the x producer of a phase-2 tile waits for the full count (acquire, bounded) before
// its first load.  Every waiter of a row block then counts itself in a second counter;
// the last one zeroes both, so each launch leaves the array at zero.  Phase-1 tiles
// wait on nothing, so no pair can wait on work that is not already issued.
// ---------------------------------------------------------------------------
struct ChainCfg {
  static constexpr int A_BYTES = kBM * kBK * 2;  // this CTA's 128 rows x 64 k
  static constexpr int B_BYTES = 128 * kBK * 2;  // its half of a tile up to 256 columns
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_BYTES = 4 * 2 * kChunkBytes;
  static constexpr int BAR_BYTES = 256;
  static constexpr int STAGES = (232448 - 1024 - BAR_BYTES - 2 * EPI_BYTES) / STAGE_BYTES;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + 2 * EPI_BYTES + BAR_BYTES;
  static constexpr uint32_t TMEM_COLS = 512;  // two accumulators at columns 0 and 256
  static constexpr uint32_t ACC_STRIDE = 256;
};

// One phase of the chained launch.
struct ChainPhase {
  int N, K;        // output columns and reduction length
  int BN;          // tile width: a multiple of 32 up to 256 whose half is whole 8-row groups
  uint32_t idesc;  // instruction descriptor of a 256 x BN product
  int n_n, kblocks;
};

template <bool ROPE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    linear_chain_kernel(const __grid_constant__ CUtensorMap tm_x1, const __grid_constant__ CUtensorMap tm_w1,
                        const __grid_constant__ CUtensorMap tm_y1, const __grid_constant__ CUtensorMap tm_r1,
                        const __grid_constant__ CUtensorMap tm_x2, const __grid_constant__ CUtensorMap tm_w2,
                        const __grid_constant__ CUtensorMap tm_y2, const ChainPhase p1, const ChainPhase p2, int M,
                        int* sync, uint64_t wait_ns, uint32_t* err, const RopeArgs rope) {
  using C = ChainCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint8_t* sOut = sB + C::STAGES * C::B_BYTES;
  uint8_t* sRes = sOut + C::EPI_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sRes + C::EPI_BYTES);  // used in the even CTA
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 2;  // used in the even CTA
  uint64_t* res_full = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(res_full + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 2);  // the even CTA's x copy and w copy arrive with both CTAs' bytes
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 8);  // one arrival per epilogue warp of both CTAs
    }
    for (int b = 0; b < 8; ++b) mbar_init(&res_full[b], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait_predecessor();  // X1 (and the buffer Y2 overwrites) belong to the previous kernel until here

  const int n_m = (M + 2 * kBM - 1) / (2 * kBM);
  const int tiles1 = n_m * p1.n_n;
  const int tiles = tiles1 + n_m * p2.n_n;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  int* done = sync;         // [n_m] phase-1 epilogue warps whose stores of the row block completed
  int* seen = sync + n_m;   // [n_m] phase-2 producers past their wait on the row block
  const int need = p1.n_n * 8;  // 4 epilogue warps in each CTA of every phase-1 tile of the row block

  if (warp < kProdWarps) {
    if (lane == 0) {
      const bool is_w = warp == 1;
      tma_prefetch_desc(is_w ? &tm_w1 : &tm_x1);
      tma_prefetch_desc(is_w ? &tm_w2 : &tm_x2);
      const uint32_t full0 = map_to_rank(smem_u32(full), 0);  // the even CTA's full barriers
      int stage = 0;
      uint32_t phase = 0;
      for (int t = pair; t < tiles && !*abort_flag; t += n_pairs) {
        const bool ph2 = t >= tiles1;
        const ChainPhase& P = ph2 ? p2 : p1;
        const int u = ph2 ? t - tiles1 : t;
        const int rb = u / P.n_n;
        const int m0 = rb * 2 * kBM + static_cast<int>(rank) * kBM;
        const int n0 = (u % P.n_n) * P.BN + static_cast<int>(rank) * (P.BN / 2);
        const CUtensorMap* tm = is_w ? (ph2 ? &tm_w2 : &tm_w1) : (ph2 ? &tm_x2 : &tm_x1);
        if (ph2 && !is_w) {
          // this row block's rows of Y1 are stored (bounded wait; the phase-1 tiles never wait)
          const uint64_t t0 = globaltimer_ns();
          bool ok = true;
          while (ld_acquire_gpu(done + rb) < need) {
            if (*abort_flag || globaltimer_ns() - t0 > wait_ns) {
              ok = false;
              break;
            }
          }
          if (!ok) {
            record_error(err, kErrTimeout | kSiteLinear);
            *abort_flag = 1;
            break;
          }
          fence_proxy_async_global();  // other CTAs wrote the rows through the async proxy
        }
        const int b_bytes = (P.BN / 2) * kBK * 2;
        for (int kb = 0; kb < P.kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, wait_ns)) {
            record_error(err, kErrTimeout | kSiteLinear);
            *abort_flag = 1;
            break;
          }
          const uint32_t bar = full0 + stage * 8;
          if (is_w) {
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * b_bytes);
            tma_load_2d_pair(sB + stage * C::B_BYTES, tm, bar, kb * kBK, n0);
          } else {
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::A_BYTES);
            tma_load_2d_pair(sA + stage * C::A_BYTES, tm, bar, kb * kBK, m0);
          }
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ph2 && !is_w && atomicAdd(seen + rb, 1) + 1 == 2 * P.n_n) {
          // (after the tile's loads, off their path) every producer that waits on this row
          // block is past its wait: zero both counters for the next launch
          done[rb] = 0;
          seen[rb] = 0;
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      for (int t = pair; t < tiles && !*abort_flag; t += n_pairs) {
        const ChainPhase& P = t >= tiles1 ? p2 : p1;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, wait_ns)) {
          record_error(err, kErrTimeout | kSiteLinear);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc) * C::ACC_STRIDE;
        bool ok = true;
        for (int kb = 0; kb < P.kblocks; ++kb) {
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
            umma_bf16_ss_pair(d_tmem, ad, bd, P.idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair_multicast(&empty[stage], 0x3);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_multicast(&acc_full[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    // epilogue warps: this CTA's 128 rows of the pair tile
    const int quarter = warp & 3;
    const int ew = warp - kEpiWarp0;
    uint8_t* obuf = sOut + ew * 2 * kChunkBytes;
    uint8_t* rbuf = sRes + ew * 2 * kChunkBytes;
    uint64_t* rbar = res_full + ew * 2;
    const uint32_t acc_empty0 = map_to_rank(smem_u32(acc_empty), 0);
    const RopeArgs no_rope{};
    uint32_t rphase = 0u;
    int acc = 0;
    uint32_t acc_phase = 0;
    int out_slot = 0;
    for (int t = pair; t < tiles; t += n_pairs) {
      const bool ph2 = t >= tiles1;
      const ChainPhase& P = ph2 ? p2 : p1;
      const int u = ph2 ? t - tiles1 : t;
      const int rb = u / P.n_n;
      const int m0 = rb * 2 * kBM + static_cast<int>(rank) * kBM, n0 = (u % P.n_n) * P.BN;
      const int row0 = m0 + quarter * 32;
      const int nch = min(P.BN, P.N - n0) / 32;
      if (!ph2 && lane == 0) epi_prefetch_residual(&tm_r1, rbuf, rbar, nch, n0, row0);
      // the second product's rotated heads (one 256-column tile is one head); compiled out
      // without rotation
      const RopeArgs& rp = (ROPE && ph2) ? rope : no_rope;
      const int rpos = ROPE ? rope_row(rp, n0, nch, row0, lane) : -1;
      float4 cs[16];
      if constexpr (ROPE) rope_prefetch(rp, rpos, cs);
      bool ok = mbar_wait(&acc_full[acc], acc_phase, wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (ok && !*abort_flag) {
        tc_fence_after();
        const uint32_t t_row =
            tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc) * C::ACC_STRIDE;
        ok = epi_tile(t_row, nch, n0, row0, !ph2, ph2 ? &tm_y2 : &tm_y1, &tm_r1, obuf, rbuf, rbar, rphase, out_slot,
                      lane, wait_ns, rp, rpos, cs);
      }
      if (!ok || *abort_flag) {
        if (lane == 0) record_error(err, kErrTimeout | kSiteLinear);
        *abort_flag = 1;
        break;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + acc * 8);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
      if (!ph2 && lane == 0) {
        // this warp's rows of the tile are in global memory: publish them to the phase-2
        // producers of the row block
        bulk_wait_group<0>();
        fence_proxy_async_global();
        red_release_gpu_add(done + rb, 1);
      }
    }
    if (lane == 0) bulk_wait_group<0>();
  }
  tc_fence_before();
  cluster_sync_all();  // the peer's shared memory is read by the pair MMAs until here
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

int g_num_sms[64] = {0};
int g_pair_slots[64][4] = {};  // co-resident CTA pairs for BN = 256, 192, 160, 224
int g_chain_slots[64] = {};    // co-resident CTA pairs of the chained kernel

template <int BN>
kalm_status setup_pair(int dev, int slot) {
  kalm_status st = check_cuda(cudaFuncSetAttribute(linear_pair_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   Linear2Cfg<BN>::SMEM),
                              "cudaFuncSetAttribute(linear_pair_kernel)");
  if (st != KALM_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 74, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Linear2Cfg<BN>::SMEM;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, linear_pair_kernel<BN>, &cfg) != cudaSuccess || clusters <= 0) {
    cudaGetLastError();
    clusters = g_num_sms[dev] / 2;
  }
  g_pair_slots[dev][slot] = clusters;
  return KALM_OK;
}

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
  if (dev >= 64) return fail(KALM_ERR_NO_DEVICE, "device index %d out of range", dev);
  int sms = 0;
  st = check_cuda(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "SM count");
  if (st != KALM_OK) return st;
  g_num_sms[dev] = sms;
  if ((st = setup_pair<256>(dev, 0)) != KALM_OK) return st;
  if ((st = setup_pair<192>(dev, 1)) != KALM_OK) return st;
  if ((st = setup_pair<160>(dev, 2)) != KALM_OK) return st;
  if ((st = setup_pair<224>(dev, 3)) != KALM_OK) return st;
  // the chained kernel: its shared memory and how many of its CTA pairs fit at once
  st = check_cuda(cudaFuncSetAttribute(linear_chain_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       ChainCfg::SMEM),
                  "cudaFuncSetAttribute(linear_chain_kernel)");
  if (st != KALM_OK) return st;
  st = check_cuda(cudaFuncSetAttribute(linear_chain_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       ChainCfg::SMEM),
                  "cudaFuncSetAttribute(linear_chain_kernel<rope>)");
  if (st != KALM_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 74, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = ChainCfg::SMEM;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, linear_chain_kernel<false>, &cfg) != cudaSuccess || clusters <= 0) {
    cudaGetLastError();
    clusters = sms / 2;
  }
  g_chain_slots[dev] = clusters;
  return KALM_OK;
}

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev < 64 && g_num_sms[dev] > 0) ? g_num_sms[dev] : 148;
}

namespace {

int pair_slots(int slot) {
  int dev = 0;
  cudaGetDevice(&dev);
  const int v = (dev < 64) ? g_pair_slots[dev][slot] : 0;
  return v > 0 ? v : num_sms() / 2;
}

kalm_status make_operand_maps(CUtensorMap* tx, CUtensorMap* tw, CUtensorMap* ty, CUtensorMap* tr, const kalm_bf16* x,
                              int64_t ldx, const kalm_bf16* w, int64_t ldw, const kalm_bf16* residual, int64_t ldr,
                              kalm_bf16* y, int64_t ldy, int64_t m, int32_t n, int32_t k, uint32_t w_box_rows) {
  kalm_status st;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(k), static_cast<uint64_t>(m)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ldx) * 2};
    const uint32_t box[2] = {kBK, kBM};
    if ((st = make_tmap_bf16(tx, x, 2, dims, strides, box)) != KALM_OK) return st;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(k), static_cast<uint64_t>(n)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ldw) * 2};
    const uint32_t box[2] = {kBK, w_box_rows};
    if ((st = make_tmap_bf16(tw, w, 2, dims, strides, box)) != KALM_OK) return st;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(n), static_cast<uint64_t>(m)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ldy) * 2};
    const uint32_t box[2] = {32, 32};
    if ((st = make_tmap_bf16(ty, y, 2, dims, strides, box, 64)) != KALM_OK) return st;
    if (residual) {
      const uint64_t rstrides[1] = {static_cast<uint64_t>(ldr) * 2};
      if ((st = make_tmap_bf16(tr, residual, 2, dims, rstrides, box, 64)) != KALM_OK) return st;
    } else {
      *tr = *ty;  // never read
    }
  }
  return KALM_OK;
}

template <int BN>
kalm_status launch_pair(const kalm_bf16* x, int64_t ldx, const kalm_bf16* w, int64_t ldw, const kalm_bf16* residual,
                        int64_t ldr, kalm_bf16* y, int64_t ldy, int64_t m, int32_t n, int32_t k, int slots,
                        cudaStream_t stream, const RopeArgs& rope) {
  CUtensorMap tx, tw, ty, tr;
  kalm_status st = make_operand_maps(&tx, &tw, &ty, &tr, x, ldx, w, ldw, residual, ldr, y, ldy, m, n, k, BN / 2);
  if (st != KALM_OK) return st;
  const int64_t tiles = ((m + 2 * kBM - 1) / (2 * kBM)) * ((n + BN - 1) / BN);
  const int pairs = static_cast<int>(tiles < slots ? tiles : slots);
  return check_cuda(launch_pdl(linear_pair_kernel<BN>, dim3(2 * pairs), dim3(kThreads), Linear2Cfg<BN>::SMEM,
                                stream, tx, tw, ty, tr, residual != nullptr, (int)m, n, k, kWaitNs,
                                device_error_word(), rope),
                    "launch linear_pair_kernel");
}

}  // namespace

// Shared by kalm_linear and kalm_cross_kv_proj.
kalm_status launch_linear(const kalm_bf16* x, int64_t ldx, const kalm_bf16* w, int64_t ldw, const kalm_bf16* residual,
                          int64_t ldr, kalm_bf16* y, int64_t ldy, int64_t m, int32_t n, int32_t k,
                          cudaStream_t stream, const char* who, const RopeArgs& rope = RopeArgs{}) {
  if (m < 0 || n <= 0 || k <= 0) return fail(KALM_ERR_INVALID_ARG, "%s: m=%lld n=%d k=%d", who, (long long)m, n, k);
  if (m == 0) return KALM_OK;
  if (m > INT32_MAX - 512) return fail(KALM_ERR_INVALID_ARG, "%s: m=%lld too large", who, (long long)m);
  if (!x || !w || !y) return fail(KALM_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (n % 32) return fail(KALM_ERR_UNSUPPORTED, "%s: n=%d must be a multiple of 32", who, n);
  if (k % 8) return fail(KALM_ERR_INVALID_ARG, "%s: k=%d must be a multiple of 8", who, k);
  if (ldx % 8 || ldw % 8 || ldy % 8 || (residual && ldr % 8) || ldx < k || ldw < k || ldy < n ||
      (residual && ldr < n))
    return fail(KALM_ERR_INVALID_ARG, "%s: strides must be multiples of 8 and >= the row width", who);
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || (residual && !aligned16(residual)))
    return fail(KALM_ERR_INVALID_ARG, "%s: bf16 pointers must be 16-byte aligned", who);
  if (rope.rot_cols > 0 && m >= 2 * kBM) {
    // rotated heads need one head per tile: 256-column pair tiles
    return launch_pair<256>(x, ldx, w, ldw, residual, ldr, y, ldy, m, n, k, pair_slots(0), stream, rope);
  }
  if (m >= 2 * kBM && n >= 128 && rope.rot_cols == 0) {
    // CTA-pair tiles of 256 x BN.  Time ~ rounds of co-resident pairs x (BN + fixed
    // per-tile cost); the fixed cost, measured at the Nano projection shapes, is worth
    // ~480 columns, so narrower tiles pay off only when they save a round.
    const int bns[4] = {256, 192, 160, 224};
    const int64_t n_m = (m + 2 * kBM - 1) / (2 * kBM);
    int best = 0;
    int64_t best_cost = INT64_MAX;
    for (int i = 0; i < 4; ++i) {
      const int64_t tiles = n_m * ((n + bns[i] - 1) / bns[i]);
      const int64_t slots = pair_slots(i);
      const int64_t cost = ((tiles + slots - 1) / slots) * (bns[i] + 480);
      if (cost < best_cost) {
        best_cost = cost;
        best = i;
      }
    }
    const int slots = pair_slots(best);
    if (best == 0) return launch_pair<256>(x, ldx, w, ldw, residual, ldr, y, ldy, m, n, k, slots, stream, rope);
    if (best == 1) return launch_pair<192>(x, ldx, w, ldw, residual, ldr, y, ldy, m, n, k, slots, stream, rope);
    if (best == 3) return launch_pair<224>(x, ldx, w, ldw, residual, ldr, y, ldy, m, n, k, slots, stream, rope);
    return launch_pair<160>(x, ldx, w, ldw, residual, ldr, y, ldy, m, n, k, slots, stream, rope);
  }
  const bool wide = (n % 256) == 0;
  const int BN = wide ? 256 : 128;
  CUtensorMap tx, tw, ty, tr;
  kalm_status st = make_operand_maps(&tx, &tw, &ty, &tr, x, ldx, w, ldw, residual, ldr, y, ldy, m, n, k, BN);
  if (st != KALM_OK) return st;
  const int64_t tiles = ((m + kBM - 1) / kBM) * ((n + BN - 1) / BN);
  const int grid = static_cast<int>(tiles < num_sms() ? tiles : num_sms());
  const bool has_r = residual != nullptr;
  const cudaError_t ce =
      wide ? launch_pdl(linear_kernel<256>, dim3(grid), dim3(kThreads), LinearCfg<256>::SMEM, stream, tx, tw, ty, tr,
                        has_r, (int)m, n, k, kWaitNs, device_error_word(), rope)
           : launch_pdl(linear_kernel<128>, dim3(grid), dim3(kThreads), LinearCfg<128>::SMEM, stream, tx, tw, ty, tr,
                        has_r, (int)m, n, k, kWaitNs, device_error_word(), rope);
  return check_cuda(ce, "launch linear_kernel");
}

namespace {

// Tile width of one phase of the chained launch (widths whose half is whole 8-row
// groups).  Both phases share one tile list, so a phase need not fill whole rounds of
// pairs: the widest width that divides n (no partial last tile, fewest operand bytes
// per output) is taken; otherwise the same rounds x (width + fixed cost) model as the
// separate projections.
int chain_width(int64_t n_m, int32_t n, int64_t slots) {
  for (int bn : {256, 224, 192, 160})
    if (n % bn == 0) return bn;
  const int bns[4] = {256, 192, 160, 224};
  int best = 256;
  int64_t best_cost = INT64_MAX;
  for (int bn : bns) {
    const int64_t tiles = n_m * ((n + bn - 1) / bn);
    const int64_t cost = ((tiles + slots - 1) / slots) * (bn + 480);
    if (cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

}  // namespace

int64_t linear_chain_sync_len(int64_t m) { return m < 0 ? -1 : 2 * ((m + 2 * kBM - 1) / (2 * kBM)); }

// y1 <- x1 . w1^T + y1 (in place), then y2 <- y1 . w2^T, in one launch (kalm_linear_chain).
kalm_status launch_linear_chain(const kalm_bf16* x1, int64_t ldx1, const kalm_bf16* w1, int64_t ldw1, kalm_bf16* y1,
                                int64_t ldy1, const kalm_bf16* w2, int64_t ldw2, kalm_bf16* y2, int64_t ldy2,
                                int64_t m, int32_t n1, int32_t k1, int32_t n2, int32_t* sync, int64_t sync_len,
                                cudaStream_t stream, const char* who, const RopeArgs& rope = RopeArgs{}) {
  if (m < 0 || n1 <= 0 || k1 <= 0 || n2 <= 0)
    return fail(KALM_ERR_INVALID_ARG, "%s: m=%lld n1=%d k1=%d n2=%d", who, (long long)m, n1, k1, n2);
  if (m == 0) return KALM_OK;
  if (m > INT32_MAX - 512) return fail(KALM_ERR_INVALID_ARG, "%s: m=%lld too large", who, (long long)m);
  if (!x1 || !w1 || !y1 || !w2 || !y2) return fail(KALM_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (n1 % 32 || n2 % 32) return fail(KALM_ERR_UNSUPPORTED, "%s: n1=%d and n2=%d must be multiples of 32", who, n1, n2);
  if (k1 % 8) return fail(KALM_ERR_INVALID_ARG, "%s: k1=%d must be a multiple of 8", who, k1);
  if (ldx1 % 8 || ldw1 % 8 || ldy1 % 8 || ldw2 % 8 || ldy2 % 8 || ldx1 < k1 || ldw1 < k1 || ldy1 < n1 ||
      ldw2 < n1 || ldy2 < n2)
    return fail(KALM_ERR_INVALID_ARG, "%s: strides must be multiples of 8 and >= the row width", who);
  if (!aligned16(x1) || !aligned16(w1) || !aligned16(y1) || !aligned16(w2) || !aligned16(y2))
    return fail(KALM_ERR_INVALID_ARG, "%s: bf16 pointers must be 16-byte aligned", who);
  if (m < 2 * kBM) {
    // below one CTA pair's rows: the two projections one after the other
    kalm_status st = launch_linear(x1, ldx1, w1, ldw1, y1, ldy1, y1, ldy1, m, n1, k1, stream, who);
    if (st != KALM_OK) return st;
    return launch_linear(y1, ldy1, w2, ldw2, nullptr, 0, y2, ldy2, m, n2, n1, stream, who, rope);
  }
  if (!sync || (reinterpret_cast<uintptr_t>(sync) & 3u))
    return fail(KALM_ERR_INVALID_ARG, "%s: sync must be a 4-byte aligned int32 array", who);
  if (sync_len < linear_chain_sync_len(m))
    return fail(KALM_ERR_INVALID_ARG, "%s: sync_len=%lld < %lld", who, (long long)sync_len,
                (long long)linear_chain_sync_len(m));
  int dev = 0;
  cudaGetDevice(&dev);
  const int64_t slots = (dev < 64 && g_chain_slots[dev] > 0) ? g_chain_slots[dev] : num_sms() / 2;
  const int64_t n_m = (m + 2 * kBM - 1) / (2 * kBM);
  ChainPhase p1{}, p2{};
  p1.N = n1;
  p1.K = k1;
  p1.BN = chain_width(n_m, n1, slots);
  p1.idesc = idesc_bf16_f32(2 * kBM, p1.BN, false, false);
  p1.n_n = (n1 + p1.BN - 1) / p1.BN;
  p1.kblocks = (k1 + kBK - 1) / kBK;
  p2.N = n2;
  p2.K = n1;
  p2.BN = rope.rot_cols > 0 ? 256 : chain_width(n_m, n2, slots);  // rotated heads: one head per tile
  p2.idesc = idesc_bf16_f32(2 * kBM, p2.BN, false, false);
  p2.n_n = (n2 + p2.BN - 1) / p2.BN;
  p2.kblocks = (n1 + kBK - 1) / kBK;
  CUtensorMap tx1, tw1, ty1, tr1, tx2, tw2, ty2, tr2;
  kalm_status st = make_operand_maps(&tx1, &tw1, &ty1, &tr1, x1, ldx1, w1, ldw1, y1, ldy1, y1, ldy1, m, n1, k1,
                                     static_cast<uint32_t>(p1.BN / 2));
  if (st != KALM_OK) return st;
  st = make_operand_maps(&tx2, &tw2, &ty2, &tr2, y1, ldy1, w2, ldw2, nullptr, 0, y2, ldy2, m, n2, n1,
                         static_cast<uint32_t>(p2.BN / 2));
  if (st != KALM_OK) return st;
  const int64_t tiles = n_m * (p1.n_n + p2.n_n);
  const int pairs = static_cast<int>(tiles < slots ? tiles : slots);
  const cudaError_t ce =
      rope.rot_cols > 0
          ? launch_pdl(linear_chain_kernel<true>, dim3(2 * pairs), dim3(kThreads), ChainCfg::SMEM, stream, tx1, tw1,
                       ty1, tr1, tx2, tw2, ty2, p1, p2, static_cast<int>(m), sync, kWaitNs, device_error_word(), rope)
          : launch_pdl(linear_chain_kernel<false>, dim3(2 * pairs), dim3(kThreads), ChainCfg::SMEM, stream, tx1, tw1,
                       ty1, tr1, tx2, tw2, ty2, p1, p2, static_cast<int>(m), sync, kWaitNs, device_error_word(), rope);
  return check_cuda(ce, "launch linear_chain_kernel");
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

extern "C" int64_t kalm_linear_chain_sync_len(int64_t m) { return linear_chain_sync_len(m); }

extern "C" kalm_status kalm_linear_chain(const kalm_bf16* x1, int64_t ldx1, const kalm_bf16* w1, int64_t ldw1,
                                         kalm_bf16* y1, int64_t ldy1, const kalm_bf16* w2, int64_t ldw2,
                                         kalm_bf16* y2, int64_t ldy2, int64_t m, int32_t n1, int32_t k1, int32_t n2,
                                         int32_t* sync, int64_t sync_len, kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  return launch_linear_chain(x1, ldx1, w1, ldw1, y1, ldy1, w2, ldw2, y2, ldy2, m, n1, k1, n2, sync, sync_len,
                             static_cast<cudaStream_t>(stream), "kalm_linear_chain");
}

extern "C" kalm_status kalm_linear_chain_rope(const kalm_bf16* x1, int64_t ldx1, const kalm_bf16* w1, int64_t ldw1,
                                              kalm_bf16* y1, int64_t ldy1, const kalm_bf16* w2, int64_t ldw2,
                                              kalm_bf16* y2, int64_t ldy2, int64_t m, int32_t n1, int32_t k1,
                                              int32_t n2, int32_t rot_cols, int32_t head_dim, const int64_t* q_off,
                                              int32_t n_docs, const float* table, int32_t* sync, int64_t sync_len,
                                              kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  const char* who = "kalm_linear_chain_rope";
  if (head_dim != 256) return fail(KALM_ERR_UNSUPPORTED, "%s: head_dim=%d (only 256)", who, head_dim);
  if (n2 % 256) return fail(KALM_ERR_UNSUPPORTED, "%s: n2=%d must be a multiple of 256", who, n2);
  if (rot_cols <= 0 || rot_cols % head_dim || rot_cols > n2)
    return fail(KALM_ERR_INVALID_ARG, "%s: rot_cols=%d must be a positive multiple of %d <= n2=%d", who, rot_cols,
                head_dim, n2);
  if (!table || !aligned16(table)) return fail(KALM_ERR_INVALID_ARG, "%s: table must be non-NULL and 16-byte aligned", who);
  if (n_docs <= 0 || !q_off) return fail(KALM_ERR_INVALID_ARG, "%s: q_off/n_docs required", who);
  RopeArgs rope{q_off, n_docs, rot_cols, reinterpret_cast<const float4*>(table), m, device_error_word()};
  return launch_linear_chain(x1, ldx1, w1, ldw1, y1, ldy1, w2, ldw2, y2, ldy2, m, n1, k1, n2, sync, sync_len,
                             static_cast<cudaStream_t>(stream), who, rope);
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

extern "C" kalm_status kalm_linear_rope(const kalm_bf16* x, int64_t ldx, const kalm_bf16* w, int64_t ldw, kalm_bf16* y,
                                        int64_t ldy, int64_t m, int32_t n, int32_t k, int32_t rot_cols,
                                        int32_t head_dim, const int64_t* q_off, int32_t n_docs, const float* table,
                                        kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (head_dim != 256) return fail(KALM_ERR_UNSUPPORTED, "kalm_linear_rope: head_dim=%d (only 256)", head_dim);
  if (n % 256) return fail(KALM_ERR_UNSUPPORTED, "kalm_linear_rope: n=%d must be a multiple of 256", n);
  if (rot_cols <= 0 || rot_cols % head_dim || rot_cols > n)
    return fail(KALM_ERR_INVALID_ARG, "kalm_linear_rope: rot_cols=%d must be a positive multiple of %d <= n=%d",
                rot_cols, head_dim, n);
  if (!table || !aligned16(table))
    return fail(KALM_ERR_INVALID_ARG, "kalm_linear_rope: table must be non-NULL and 16-byte aligned");
  if (n_docs <= 0 || !q_off) return fail(KALM_ERR_INVALID_ARG, "kalm_linear_rope: q_off/n_docs required");
  RopeArgs rope{q_off, n_docs, rot_cols, reinterpret_cast<const float4*>(table), m, device_error_word()};
  return launch_linear(x, ldx, w, ldw, nullptr, 0, y, ldy, m, n, k, static_cast<cudaStream_t>(stream),
                       "kalm_linear_rope", rope);
}
