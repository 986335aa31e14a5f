// Step 3: merged self + cross attention for a ragged batch of documents.
//
// "KaLM-Reranker-V1-Nano - MLX (Apple Silicon)", "What this is": the decoder runs
// a single scaled-dot-product attention whose keys and values are the
// concatenation of its own (causal) self-attention K/V and the cross-attention
// K/V of the document's cached pooled vectors.  One softmax covers both parts.
//
// Design (sm_100a): a persistent kernel, one CTA per SM, each CTA walking a list
// of work items (query tile, KV head, document), heaviest tiles first:
//   * 128 packed rows = (128 / G) decoder positions x G query heads of one KV
//     head (GQA), so every K/V tile is fetched once for the G heads sharing it.
//     The Q tile (128 x 256 bf16) is one 4-D TMA box (64 columns x heads x
//     positions x 4 column slabs).
//   * The KV loop walks the self segment (64-key tiles up to the tile's last
//     position, causal mask inside) and then the cross segment (64-key tiles,
//     only the ragged tail masked).  The concatenation exists only as this
//     loop order; nothing is materialised in memory.
//   * S = Q K^T and O += P V run on the tensor cores (tcgen05.mma, fp32
//     accumulators in tensor memory: O = 256 columns, S double-buffered 2 x 64).
//     The Q tile is copied once per item from shared memory into the last 128
//     tensor-memory columns (tcgen05.cp) and the S products read it from there,
//     so each S product reads only the 64-key K tile from shared memory and the
//     shared-memory Q tile is free for the next item's copy right away.
//   * Softmax: the two warp groups (warps 0-3, 4-7) take alternate tiles, one
//     thread per row with all 64 scores, so two tiles' exponentials overlap.  A
//     tile's running max goes to the next tile's group through shared memory as
//     soon as its row max is known.  The running max is only raised when it grows
//     by more than 2^8 in the exponent; otherwise P keeps the stale max (values
//     stay below 256), so O is rescaled in tensor memory only on such rare jumps.
//     Each group keeps its partial row sum relative to the max it last used; the
//     epilogue brings both to the final max.  P goes as bf16 into a 128-byte-
//     swizzled shared tile (the A operand of P V).
//   * The K/V rings, S/P buffers and their barriers run over one tile counter
//     for all items of the CTA, so the next item's Q load (issued as soon as the
//     current Q is in tensor memory) and its first S product overlap the current
//     item's tiles, last softmax, P V and O write-out.
//   * Every role loads the next item's offsets while it works on the current one.
//   * Epilogue: each warp stages its 32 rows x 64 columns of O / l as bf16 in the idle
//     P buffers and copies them out row-major, so every store writes whole lines.
//   * Warp roles: warps 0-7 softmax + epilogue, warp 8 TMA producer of Q and K,
//     warp 10 TMA producer of V, warp 9 tensor-memory allocation, the Q copy and
//     the S products, warp 11 the P V products.  With two issuing threads, S of the
//     next tiles goes out while P V waits for the softmax, so the tensor pipe does
//     not idle behind one thread's waits.
#include <cmath>
#include <mutex>

#include "kalm.h"
#include "kalm_internal.h"
#include "kalm_ptx.cuh"

namespace kalm {
namespace {

constexpr int kD = 256;
constexpr int kBM = 128;
constexpr int kBKV = 64;
constexpr int kThreads = 384;
constexpr int kSoftmaxThreads = 256;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kTmaWarpV = 10;
constexpr int kMmaWarpPV = 11;
constexpr int kQBytes = kBM * kD * 2;          // 4 slabs of 128 rows x 128 B
constexpr int kKVBytes = kBKV * kD * 2;        // 4 slabs of 64 rows x 128 B
constexpr int kQSlab = kBM * 128;              // 16 KB
constexpr int kKVSlab = kBKV * 128;            // 8 KB
constexpr int kPBytes = kBM * kBKV * 2;        // 1 slab of 128 rows x 128 B
constexpr int kBarBytes = 512;
constexpr int kSmem = 1024 + kQBytes + 2 * kKVBytes + 2 * kKVBytes + 2 * kPBytes + kBarBytes + 2 * 128 * 4 + 128 * 4;
static_assert(kSmem <= 227 * 1024, "attention shared memory");
constexpr uint32_t kTmemCols = 512;            // O: [0,256), S0: [256,320), S1: [320,384), Q: [384,512)
constexpr uint32_t kTmemQ = 384;               // the Q tile as bf16 pairs (A operand of S = Q K^T)
constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBKV, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, kD, false, true);
constexpr float kRescaleThreshold = 8.0f;      // log2 units

struct AttnParams {
  const int64_t* q_off;
  const int64_t* in_off;  // first q / self-K/V row of each document; NULL: q_off
  int last_only;          // compute only the query tile holding each document's last row
  const int64_t* pool_off;
  __nv_bfloat16* out;
  float* lse;
  int64_t ldo;
  int n_docs;
  int n_q;
  int n_kv;
  int G;            // query heads per KV head
  int P;            // decoder positions per tile = 128 / G
  int tiles_per_doc;
  int n_items;
  const int32_t* order;  // work items sorted heaviest first (kalm_attention_schedule); NULL: index order
  float scale_log2;  // scale * log2(e)
  uint64_t wait_ns;
  uint32_t* err;
};

// The fused launch's output projection (X += O . Wo^T over each document's rows).
struct ProjParams {
  __nv_bfloat16* x;   // residual stream [total_q][ldx], updated in place
  int64_t ldx;
  int hidden;         // N of the projection (multiple of 64)
  int kdim;           // K of the projection = n_q * 256
  int n_chunks;       // 256-column chunks of hidden
  int m_tiles;        // 128-row tiles of max_q
  int n_otiles;       // n_docs * m_tiles * n_chunks (tiles of rows past a document's end are skipped)
  // [n_docs] per-document item counters, [n_docs] ready-queue tail, [n_docs + 1] its head,
  // [n_docs + 2, + n_otiles) the ready queue (tile id + 1, 0 = empty); all zero between launches
  int* sync;
};

// One work item: query tile t of KV head g of document d, with its extents.
struct Item {
  int t, g, d, Lq, Nc, pos0, pos1, n_self, nt;
  int64_t q0, qi, c0;
};

__device__ __forceinline__ Item make_item(const AttnParams& p, int w) {
  Item it;
  const int per_t = p.n_docs * p.n_kv;
  const int rem = w % per_t;
  it.g = rem % p.n_kv;
  it.d = rem / p.n_kv;
  it.q0 = p.q_off[it.d];
  it.Lq = static_cast<int>(p.q_off[it.d + 1] - it.q0);
  it.qi = p.in_off ? p.in_off[it.d] : it.q0;
  it.t = p.last_only ? (it.Lq > 0 ? (it.Lq - 1) / p.P : 0) : p.tiles_per_doc - 1 - w / per_t;
  it.c0 = p.pool_off[it.d];
  it.Nc = static_cast<int>(p.pool_off[it.d + 1] - it.c0);
  it.pos0 = it.t * p.P;
  it.pos1 = min(it.pos0 + p.P, it.Lq);
  it.n_self = it.pos0 < it.Lq ? (it.pos1 + kBKV - 1) / kBKV : 0;
  it.nt = it.pos0 < it.Lq ? it.n_self + (it.Nc + kBKV - 1) / kBKV : 0;  // 0: nothing to do
  return it;
}

constexpr int kNoMore = -2;  // item_at: this CTA has no further items
constexpr int kSkip = -1;    // item_at: no item at this pass

// Work item of this CTA's k-th pass: entry k * grid + c of the work order
// (kalm_attention_schedule lays it out so that the CTAs' total costs come out
// even), or without one item k * grid + c itself.
__device__ __forceinline__ int item_at(const AttnParams& p, int k) {
  const int64_t base = static_cast<int64_t>(k) * gridDim.x;
  if (base >= p.n_items) return kNoMore;
  const int64_t idx = base + static_cast<int>(blockIdx.x);
  if (idx >= p.n_items) return kSkip;
  if (!p.order) return static_cast<int>(idx);
  const int w = p.order[idx];
  if (w < 0 || w >= p.n_items) {  // not a work order of this launch: flag it, skip the entry
    record_error(p.err, kErrDeviceArg | kSiteAttention);
    return kSkip;
  }
  return w;
}

__device__ __forceinline__ Item load_item(const AttnParams& p, int w) {
  if (w >= 0) return make_item(p, w);
  Item it{};
  it.nt = 0;
  return it;
}

// ------------------------------------------------------------------------------
// Output projection phase of the fused decoder layer: X[rows of d] += O[rows of d] . Wo^T.
// Tiles are (document, 128-row block, 256-column chunk).  When a document's last attention
// item is counted (by whichever CTA computed it), its tiles go into a ready queue; CTAs
// that have finished their own attention items pop tiles from it in that order, so no CTA
// waits on a document that is still being computed while finished ones wait.  1-CTA tcgen05 GEMM:
// warp 8 lane 0 claims tiles and loads A (O rows) and B (Wo rows) by TMA into a 4-deep
// ring, warp 9 lane 0 issues M=128 x N=256 products into one of two TMEM
// accumulators, warps 0-7 add the residual and write X (warp w: rows 32 (w % 4) ..,
// columns 128 (w / 4) .. of the tile).
constexpr int kGStages = 4;
constexpr int kGABytes = kBM * 64 * 2;   // 128 rows x 64 k
constexpr int kGBBytes = 256 * 64 * 2;   // 256 rows x 64 k
constexpr int kGStageBytes = kGABytes + kGBBytes;
constexpr uint32_t kIdescG = idesc_bf16_f32(kBM, 256, false, false);
static_assert(kGStages * kGStageBytes + 8 * 4096 <= kQBytes + 4 * kKVBytes + 2 * kPBytes,
              "projection ring and staging fit in the attention buffers");

struct GemmBars {
  uint64_t* full;       // [kGStages]
  uint64_t* empty;      // [kGStages]
  uint64_t* acc_full;   // [2]
  uint64_t* acc_empty;  // [2] one arrival per epilogue warp
  uint64_t* tq_full;    // [2] tile id published
  uint64_t* tq_empty;   // [2] tile id slot free (one arrival per epilogue warp)
  volatile int* tq;     // [2] tile ids (-1: no more)
};

__device__ __forceinline__ GemmBars gemm_bars(uint64_t* bars) {
  return GemmBars{bars + 22, bars + 26, bars + 30, bars + 32, bars + 34, bars + 36,
                  reinterpret_cast<volatile int*>(bars + 38)};
}

__device__ __forceinline__ void decode_otile(const ProjParams& f, int t, int& d, int& mi, int& ni) {
  const int per_doc = f.m_tiles * f.n_chunks;
  d = t / per_doc;
  const int rem = t - d * per_doc;
  mi = rem / f.n_chunks;
  ni = rem - mi * f.n_chunks;
}

__device__ __forceinline__ void out_proj_phase(const AttnParams& p, const ProjParams& f, const CUtensorMap* tm_oa,
                                               const CUtensorMap* tm_wo, uint8_t* smem, const GemmBars& gb,
                                               uint32_t tmem, int warp, int lane, volatile int* abort_flag) {
  int* tail = f.sync + p.n_docs;      // pushes (by the CTAs that complete documents)
  int* head = f.sync + p.n_docs + 1;  // pops
  int* queue = f.sync + p.n_docs + 2;
  const int kblocks = f.kdim / 64;
  if (warp == kTmaWarp) {
    if (lane != 0) return;
    // ---------------------------------------------------- tile pops and A/B loads
    tma_prefetch_desc(tm_oa);
    tma_prefetch_desc(tm_wo);
    int published = 0, stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    int d = 0, mi = 0, ni = 0;
    // documents without decoder rows have no attention items to complete them: this CTA
    // queues the (empty) tiles of those in its stripe, so every queue slot gets filled
    const int per_doc = f.m_tiles * f.n_chunks;
    for (int e = blockIdx.x; e < p.n_docs; e += gridDim.x)
      if (p.q_off[e + 1] == p.q_off[e])
        for (int u = 0; u < per_doc; ++u) st_release_gpu(queue + atomicAdd(tail, 1), e * per_doc + u + 1);
    while (true) {
      const int pos = atomicAdd(head, 1);
      if (pos == f.n_otiles + static_cast<int>(gridDim.x) - 1) {
        // the launch's last pop: every CTA is past its attention items (so every push is
        // done) and every slot has been taken; the queue starts empty in the next launch
        atomicExch(head, 0);
        atomicExch(tail, 0);
      }
      int id = -1;
      if (pos < f.n_otiles && ok && !*abort_flag) {
        // the slot is filled once the document it belongs to is complete
        int v = 0;
        const uint64_t t0 = globaltimer_ns();
        while ((v = ld_acquire_gpu(queue + pos)) == 0) {
          if (*abort_flag || globaltimer_ns() - t0 > p.wait_ns) {
            record_error(p.err, kErrTimeout | kSiteAttention);
            *abort_flag = 1;
            ok = false;
            break;
          }
        }
        if (ok) {
          queue[pos] = 0;
          decode_otile(f, v - 1, d, mi, ni);
          if (mi * kBM >= static_cast<int>(p.q_off[d + 1] - p.q_off[d])) continue;  // no rows in the block
          id = v - 1;
        }
      }
      // publish the tile (or the end) to the MMA and epilogue warps
      const int k = published & 1;
      if (published >= 2 && !mbar_wait(&gb.tq_empty[k], ((published - 2) >> 1) & 1, p.wait_ns)) {
        record_error(p.err, kErrTimeout | kSiteAttention);
        *abort_flag = 1;
        ok = false;
      }
      gb.tq[k] = id;
      mbar_arrive(&gb.tq_full[k]);
      ++published;
      if (id < 0) break;
      if (!ok) continue;
      fence_proxy_async_global();  // O rows written by other CTAs, read below by TMA
      const int32_t row0 = static_cast<int32_t>(p.q_off[d] + mi * kBM);
      for (int kb = 0; kb < kblocks && ok; ++kb) {
        if (!mbar_wait(&gb.empty[stage], phase ^ 1u, p.wait_ns)) {
          record_error(p.err, kErrTimeout | kSiteAttention);
          *abort_flag = 1;
          ok = false;
          break;
        }
        uint8_t* sa = smem + stage * kGStageBytes;
        mbar_arrive_expect_tx(&gb.full[stage], kGStageBytes);
        tma_load_2d(sa, tm_oa, &gb.full[stage], kb * 64, row0);
        tma_load_2d(sa + kGABytes, tm_wo, &gb.full[stage], kb * 64, ni * 256);
        if (++stage == kGStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane != 0) return;
    // ---------------------------------------------------- products into TMEM
    int k = 0, stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    const uint32_t base = smem_u32(smem);
    while (true) {
      if (!mbar_wait(&gb.tq_full[k & 1], (k >> 1) & 1, p.wait_ns)) {
        record_error(p.err, kErrTimeout | kSiteAttention);
        *abort_flag = 1;
        break;
      }
      const int id = gb.tq[k & 1];
      ++k;
      if (id < 0) break;
      if (!mbar_wait(&gb.acc_empty[acc], acc_phase ^ 1u, p.wait_ns)) {
        record_error(p.err, kErrTimeout | kSiteAttention);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc) * 256u;
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait(&gb.full[stage], phase, p.wait_ns)) {
          record_error(p.err, kErrTimeout | kSiteAttention);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad0 = sdesc_sw128(base + stage * kGStageBytes, 16, 1024);
        const uint64_t bd0 = sdesc_sw128(base + stage * kGStageBytes + kGABytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_ss(d_tmem, ad0 + static_cast<uint64_t>(kk * 2), bd0 + static_cast<uint64_t>(kk * 2), kIdescG,
                       (kb | kk) != 0 ? 1u : 0u);
        umma_commit(&gb.empty[stage]);
        if (++stage == kGStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      umma_commit(&gb.acc_full[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  } else if (warp < kSoftmaxThreads / 32) {
    // ---------------------------------------------------- epilogue: + residual, bf16, X
    const int quarter = warp & 3, half = warp >> 2;
    uint8_t* stage_buf = smem + kGStages * kGStageBytes + warp * 4096;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int k = 0, acc = 0;
    uint32_t acc_phase = 0;
    while (true) {
      bool wt = mbar_wait(&gb.tq_full[k & 1], (k >> 1) & 1, p.wait_ns);
      if (!__all_sync(0xffffffffu, wt)) {
        if (lane == 0) record_error(p.err, kErrTimeout | kSiteAttention);
        *abort_flag = 1;
        break;
      }
      const int id = gb.tq[k & 1];
      const int kslot = k & 1;
      ++k;
      if (id < 0) break;
      int d, mi, ni;
      decode_otile(f, id, d, mi, ni);
      const int64_t q0 = p.q_off[d];
      const int lq = static_cast<int>(p.q_off[d + 1] - q0);
      wt = mbar_wait(&gb.acc_full[acc], acc_phase, p.wait_ns);
      if (!__all_sync(0xffffffffu, wt) || *abort_flag) {
        if (lane == 0) record_error(p.err, kErrTimeout | kSiteAttention);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int rloc = mi * kBM + quarter * 32;  // first row of this warp, within the document
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int col0 = ni * 256 + half * 128 + c * 64;
        uint32_t o[2][32];
        tmem_ld32(lane_base + static_cast<uint32_t>(acc * 256 + half * 128 + c * 64), o[0]);
        tmem_ld32(lane_base + static_cast<uint32_t>(acc * 256 + half * 128 + c * 64 + 32), o[1]);
        tmem_ld_wait();
        const bool row_ok = rloc + lane < lq && col0 < f.hidden;
        uint4 vv[8];
        const __nv_bfloat16* xr = f.x + (q0 + rloc + lane) * f.ldx + col0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint4 rv = make_uint4(0u, 0u, 0u, 0u);
          if (row_ok) rv = *reinterpret_cast<const uint4*>(xr + u * 8);
          const __nv_bfloat162* rh = reinterpret_cast<const __nv_bfloat162*>(&rv);
          const uint32_t* oc = o[u >> 2] + (u & 3) * 8;
          float f[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 r2 = __bfloat1622float2(rh[e]);
            f[2 * e] = __uint_as_float(oc[2 * e]) + r2.x;
            f[2 * e + 1] = __uint_as_float(oc[2 * e + 1]) + r2.y;
          }
          vv[u].x = pack_bf16x2(f[0], f[1]);
          vv[u].y = pack_bf16x2(f[2], f[3]);
          vv[u].z = pack_bf16x2(f[4], f[5]);
          vv[u].w = pack_bf16x2(f[6], f[7]);
        }
        // staged (swizzled) and written row-major, 8 lanes per 128-byte row
        uint8_t* row = stage_buf + lane * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) *reinterpret_cast<uint4*>(row + ((u ^ (lane & 7)) << 4)) = vv[u];
        __syncwarp();
        const int cu = lane & 7;
#pragma unroll
        for (int kq = 0; kq < 8; ++kq) {
          const int rr = (lane >> 3) + 4 * kq;
          const uint4 val = *reinterpret_cast<const uint4*>(stage_buf + rr * 128 + ((cu ^ (rr & 7)) << 4));
          if (rloc + rr < lq && col0 < f.hidden)
            *reinterpret_cast<uint4*>(f.x + (q0 + rloc + rr) * f.ldx + col0 + cu * 8) = val;
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&gb.acc_empty[acc]);
        mbar_arrive(&gb.tq_empty[kslot]);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }
}

template <bool FUSED>
__global__ void __launch_bounds__(kThreads, 1)
    merged_attention_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_ks,
                            const __grid_constant__ CUtensorMap tm_vs, const __grid_constant__ CUtensorMap tm_kc,
                            const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_oa,
                            const __grid_constant__ CUtensorMap tm_wo, const AttnParams p, const ProjParams f) {
  pdl_launch_dependents();
  pdl_wait_predecessor();  // q/K/V come from the previous kernel; offsets are read by every role

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kQBytes;
  uint8_t* sV = sK + 2 * kKVBytes;
  uint8_t* sP = sV + 2 * kKVBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * kPBytes);
  uint64_t* bar_q = bars;        // Q landed (per item)
  uint64_t* bar_qfree = bars + 1;  // Q copied into tensor memory: shared-memory Q tile reusable (per item)
  uint64_t* bar_k = bars + 2;    // [2] K tile landed
  uint64_t* bar_v = bars + 4;    // [2] V tile landed
  uint64_t* bar_s = bars + 6;    // [2] S ready
  uint64_t* bar_p = bars + 8;    // [2] P written (and O rescaled)
  uint64_t* bar_pv = bars + 10;  // [2] P V done
  uint64_t* bar_l = bars + 12;   // partial row sums published (per item)
  uint64_t* bar_ofree = bars + 13;  // O read out by the epilogue (per item)
  uint64_t* bar_m = bars + 14;   // [2] running max after a tile published (one per tile parity)
  uint64_t* bar_sdone = bars + 16;  // every S of an item done: the Q columns of tensor memory reusable
  uint64_t* bar_sfree = bars + 17;  // [2] S buffer loaded into registers by its softmax group (per tile parity)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // fused output projection only: an item's O stores done (softmax warps) / counted (signaller)
  uint64_t* bar_ostored = bars + 20;
  uint64_t* bar_osig = bars + 21;
  float* l_part = reinterpret_cast<float*>(sP + 2 * kPBytes + kBarBytes);  // [2][128]
  // running max after the latest tile, per row: written by the tile's group, read by the next
  // tile's group after bar_m; the bar_m waits order every write after the previous read
  float* m_pub = l_part + 2 * 128;                                         // [128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_qfree, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_k[i], 1);
      mbar_init(&bar_v[i], 1);
      mbar_init(&bar_s[i], 1);
      mbar_init(&bar_p[i], kSoftmaxThreads / 2);  // one warp group writes each tile's P
      mbar_init(&bar_sfree[i], kSoftmaxThreads / 2);
      mbar_init(&bar_pv[i], 1);
      mbar_init(&bar_m[i], 4);                    // the four warps of that group
    }
    mbar_init(bar_l, kSoftmaxThreads);
    mbar_init(bar_ofree, kSoftmaxThreads);
    mbar_init(bar_sdone, 1);
    if constexpr (FUSED) {
      const GemmBars gb = gemm_bars(bars);
      mbar_init(bar_ostored, kSoftmaxThreads / 32);
      mbar_init(bar_osig, 1);
      for (int i = 0; i < kGStages; ++i) {
        mbar_init(&gb.full[i], 1);
        mbar_init(&gb.empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&gb.acc_full[i], 1);
        mbar_init(&gb.acc_empty[i], kSoftmaxThreads / 32);
        mbar_init(&gb.tq_full[i], 1);
        mbar_init(&gb.tq_empty[i], kSoftmaxThreads / 32);
      }
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail_wait = [&]() {
    record_error(p.err, kErrTimeout | kSiteAttention);
    *abort_flag = 1;
  };

  if (warp == kTmaWarp || warp == kTmaWarpV) {
    // ------------------------------------------------------------ TMA producers (Q+K, V)
    if (lane == 0) {
      const bool is_v = warp == kTmaWarpV;
      uint64_t* bar_free = is_v ? bar_pv : bar_s;   // slot reusable once S (for K) / PV (for V) is done
      uint64_t* bar_full = is_v ? bar_v : bar_k;
      uint8_t* ring = is_v ? sV : sK;
      uint32_t J = 0;  // tile counter over all items of this CTA
      int n_it = 0;
      bool ok = true;
      bool q_ready = false;  // the current item's Q was issued during the previous item
      int64_t last_j = -1;   // last K/V tile issued (for the drain at the end)
      int q_issued = 0;      // Q tiles issued
      int wc = item_at(p, 0);
      Item nxt = load_item(p, wc);
      for (int pass = 0; wc != kNoMore && ok && !*abort_flag; ++pass) {
        const Item it = nxt;  // offsets are loaded one item ahead
        wc = item_at(p, pass + 1);
        nxt = load_item(p, wc);
        if (it.nt == 0) continue;
        // The shared-memory Q tile is free once the previous item's Q is in tensor memory,
        // which happens at that item's start, so the Q+K producer normally issues an
        // item's Q during the previous item (q_ready); here only if that did not happen.
        if (!is_v && !q_ready) {
          if (n_it >= 1 && !mbar_wait(bar_qfree, (n_it - 1) & 1, p.wait_ns)) {
            fail_wait();
            break;
          }
          mbar_arrive_expect_tx(bar_q, kQBytes);
          tma_load_4d(sQ, &tm_q, bar_q, 0, it.g * p.G, static_cast<int32_t>(it.qi + it.pos0), 0);
          ++q_issued;
        }
        q_ready = false;
        for (int j = 0; j < it.nt; ++j, ++J) {
          const int s = J & 1;
          const bool self = j < it.n_self;
          const int32_t row = self ? static_cast<int32_t>(it.qi + j * kBKV)
                                   : static_cast<int32_t>(it.c0 + (j - it.n_self) * kBKV);
          const CUtensorMap* m = is_v ? (self ? &tm_vs : &tm_vc) : (self ? &tm_ks : &tm_kc);
          if (J >= 2 && !mbar_wait(&bar_free[s], ((J - 2) >> 1) & 1, p.wait_ns)) {
            fail_wait();
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_full[s], kKVBytes);
          tma_load_3d(ring + s * kKVBytes, m, &bar_full[s], 0, row, it.g * 4);
          last_j = J;
          if (!is_v && j == 0 && nxt.nt > 0) {
            // next item's Q as soon as this item's Q is in tensor memory
            if (!mbar_wait(bar_qfree, n_it & 1, p.wait_ns)) {
              fail_wait();
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar_q, kQBytes);
            tma_load_4d(sQ, &tm_q, bar_q, 0, nxt.g * p.G, static_cast<int32_t>(nxt.qi + nxt.pos0), 0);
            ++q_issued;
            q_ready = true;
          }
        }
        ++n_it;
      }
      // Drain (matters when a role gave up on a wait): every copy this thread issued has
      // landed before the CTA tears down.  Each barrier waited on here is at most one
      // phase behind the issue it waits for, so the parity waits are exact.
      for (int64_t jj = last_j; jj >= 0 && jj >= last_j - 1; --jj)
        mbar_wait(&bar_full[jj & 1], static_cast<uint32_t>(jj >> 1) & 1, p.wait_ns);
      if (q_issued > 0) mbar_wait(bar_q, (q_issued - 1) & 1, p.wait_ns);
    } else if (FUSED && warp == kTmaWarpV && lane == 1) {  // (compiled out when not FUSED)
      // Fused output projection: count each finished item for its document.  The softmax
      // warps arrive once their O stores of the item are done; the release add then makes
      // those stores visible, at gpu scope, to the CTA that projects the document.
      int n_it = 0;
      int wc = item_at(p, 0);
      Item nxt = load_item(p, wc);
      for (int pass = 0; wc != kNoMore; ++pass) {
        const Item it = nxt;
        wc = item_at(p, pass + 1);
        nxt = load_item(p, wc);
        if (it.nt == 0) continue;
        if (!mbar_wait(bar_ostored, n_it & 1, p.wait_ns) || *abort_flag) {
          fail_wait();
          break;
        }
        // count the item; the count that completes the document (acquiring the other
        // counters' releases) queues its tiles, each slot written with release order
        const int items = p.n_kv * ((it.Lq + p.P - 1) / p.P);
        if (atom_add_acq_rel_gpu(f.sync + it.d, 1) + 1 == items) {
          f.sync[it.d] = 0;  // no further count this launch: zero for the next one
          const int per_doc = f.m_tiles * f.n_chunks;
          for (int u = 0; u < per_doc; ++u) {
            const int pos = atomicAdd(f.sync + p.n_docs, 1);
            st_release_gpu(f.sync + p.n_docs + 2 + pos, it.d * per_doc + u + 1);
          }
        }
        mbar_arrive(bar_osig);
        ++n_it;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ S issuer: Q copy and S = Q K^T
    // S of tile J goes out as soon as K_J has landed and the softmax has loaded S_{J-2}
    // (same buffer) into registers, independently of the P V products, which warp 11
    // issues.
    if (lane == 0) {
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK);
      uint32_t J = 0;
      int n_it = 0;
      bool ok = true;
      uint64_t* last_bar = nullptr;  // barrier of this thread's last commit (for the drain)
      uint32_t last_par = 0;
      int wc = item_at(p, 0);
      Item nxt = load_item(p, wc);
      for (int pass = 0; wc != kNoMore && ok && !*abort_flag; ++pass) {
        const Item it = nxt;  // offsets are loaded one item ahead
        wc = item_at(p, pass + 1);
        nxt = load_item(p, wc);
        if (it.nt == 0) continue;
        // Q of this item: landed in shared memory, and the previous item's S products
        // no longer read the Q columns -> copy it into tensor memory, then release the
        // shared-memory tile so the next item's Q can load during this whole item
        ok = mbar_wait(bar_q, n_it & 1, p.wait_ns) && (n_it == 0 || mbar_wait(bar_sdone, (n_it - 1) & 1, p.wait_ns));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          tmem_cp_128x256b(tmem + kTmemQ + static_cast<uint32_t>(kk * 8),
                           sdesc_sw128(q_base + (kk >> 2) * kQSlab + static_cast<uint32_t>((kk & 3) * 32), 16, 1024));
        umma_commit(bar_qfree);
        last_bar = bar_qfree;
        last_par = n_it & 1;
        for (int j = 0; j < it.nt && ok && !*abort_flag; ++j) {
          const uint32_t Jc = J + j;
          const int s = Jc & 1;
          if (!mbar_wait(&bar_k[s], (Jc >> 1) & 1, p.wait_ns) ||
              (Jc >= 2 && !mbar_wait(&bar_sfree[s], ((Jc - 2) >> 1) & 1, p.wait_ns))) {  // S_{Jc-2} loaded
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_s = tmem + 256u + static_cast<uint32_t>(s * kBKV);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = static_cast<uint32_t>((kk & 3) * 32);  // 16-element step inside a swizzle row
            const uint64_t bd = sdesc_sw128(k_base + s * kKVBytes + (kk >> 2) * kKVSlab + off, 16, 1024);
            // Q from tensor memory: only the K tile is read from shared memory
            umma_bf16_ts(d_s, tmem + kTmemQ + static_cast<uint32_t>(kk * 8), bd, kIdescS, kk != 0 ? 1u : 0u);
          }
          umma_commit(&bar_s[s]);
          last_bar = &bar_s[s];
          last_par = (Jc >> 1) & 1;
          if (j + 1 == it.nt) {
            umma_commit(bar_sdone);  // every S of this item done
            last_bar = bar_sdone;
            last_par = n_it & 1;
          }
        }
        J += it.nt;
        ++n_it;
      }
      if (!ok) fail_wait();
      // Drain: tensor-core operations complete in issue order, so once the last commit's
      // barrier completes nothing this thread issued still reads shared or tensor memory
      if (last_bar) mbar_wait(last_bar, last_par, p.wait_ns);
    }
  } else if (warp == kMmaWarpPV) {
    // ------------------------------------------------------------ P V issuer
    if (lane == 0) {
      const uint32_t v_base = smem_u32(sV), p_base = smem_u32(sP);
      uint32_t J = 0;
      int n_it = 0;
      bool ok = true;
      int64_t last_j = -1;  // last P V issued (for the drain)
      int wc = item_at(p, 0);
      Item nxt = load_item(p, wc);
      for (int pass = 0; wc != kNoMore && ok && !*abort_flag; ++pass) {
        const Item it = nxt;
        wc = item_at(p, pass + 1);
        nxt = load_item(p, wc);
        if (it.nt == 0) continue;
        for (int j = 0; j < it.nt && ok && !*abort_flag; ++j) {
          const uint32_t Jc = J + j;
          const int s = Jc & 1;
          if (!mbar_wait(&bar_p[s], (Jc >> 1) & 1, p.wait_ns) ||
              !mbar_wait(&bar_v[s], (Jc >> 1) & 1, p.wait_ns) ||
              (j == 0 && n_it >= 1 && !mbar_wait(bar_ofree, (n_it - 1) & 1, p.wait_ns))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBKV / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(p_base + s * kPBytes + kk * 32, 16, 1024);
            // V is MN-major: 64-column slabs kKVSlab apart (LBO), 8-key groups 1024 B apart (SBO)
            const uint64_t bd = sdesc_sw128(v_base + s * kKVBytes + kk * 16 * 128, kKVSlab, 1024);
            umma_bf16_ss(tmem, ad, bd, kIdescPV, (j | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&bar_pv[s]);
          last_j = Jc;
        }
        J += it.nt;
        ++n_it;
      }
      if (!ok) fail_wait();
      if (last_j >= 0) mbar_wait(&bar_pv[last_j & 1], static_cast<uint32_t>(last_j >> 1) & 1, p.wait_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0..7
    // Two warp groups take alternate tiles (group = tile parity = S and P buffer), one
    // thread per row with all 64 scores, so two tiles' exponentials run at once.  The
    // running max passes from each tile to the next through shared memory as soon as
    // the tile's row max is known; each group keeps its partial row sum relative to the
    // max it last used, and the epilogue brings both to the final max.
    const int quarter = warp & 3;             // TMEM lane quarter
    const int half = warp >> 2;               // warp group; in the epilogue, which 128 O columns
    const int r = quarter * 32 + lane;        // packed row = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float c2 = p.scale_log2;
    uint32_t J = 0;
    int n_it = 0;
    bool ok = true;
    int wc = item_at(p, 0);
    Item nxt = load_item(p, wc);
    for (int pass = 0; wc != kNoMore && ok; ++pass) {
      const Item it = nxt;
      wc = item_at(p, pass + 1);
      nxt = load_item(p, wc);
      if (it.nt == 0) continue;
      const int pos = it.pos0 + r / p.G;      // decoder position of this row
      const int hh = r % p.G;                 // query head within the KV group
      float m_ref = -INFINITY, l_own = 0.f;   // this group's partial sum and the max it is relative to
      for (int j = 0; j < it.nt; ++j) {
        const uint32_t Jc = J + j;
        const int s = Jc & 1;
        if (s != half) continue;              // the other group's tile
        bool wt = mbar_wait(&bar_s[s], (Jc >> 1) & 1, p.wait_ns);
        if (!__all_sync(0xffffffffu, wt) || *abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(lane_base + 256u + s * kBKV, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(lane_base + 256u + s * kBKV + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&bar_sfree[s]);  // the scores are in registers: the buffer may take S_{Jc+2}
        // visible keys of this tile: self keys k <= pos, cross keys k < Nc
        int n_vis = (j < it.n_self) ? pos + 1 - j * kBKV : it.Nc - (j - it.n_self) * kBKV;
        n_vis = max(0, min(kBKV, n_vis));
        const bool masked = !__all_sync(0xffffffffu, n_vis == kBKV);
        if (masked) {
#pragma unroll
          for (int k = 0; k < 64; ++k)
            if (k >= n_vis) sr[k] = __float_as_uint(-INFINITY);
        }
        // row max of the raw scores (scale > 0 keeps the order), as a tree
        float t32[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) t32[k] = fmaxf(__uint_as_float(sr[k]), __uint_as_float(sr[k + 32]));
#pragma unroll
        for (int w2 = 16; w2 > 0; w2 >>= 1)
#pragma unroll
          for (int k = 0; k < w2; ++k) t32[k] = fmaxf(t32[k], t32[k + w2]);
        const float mx = t32[0] * c2;
        // running max after the previous tile (the other group's), or none at an item's start
        float m_prev = -INFINITY;
        if (j > 0) {
          const bool wm = mbar_wait(&bar_m[s ^ 1], ((Jc - 1) >> 1) & 1, p.wait_ns);
          if (!__all_sync(0xffffffffu, wm)) {
            ok = false;
            break;
          }
          m_prev = m_pub[r];
        }
        // lazy max: raised only when it grows by more than 2^8 (j == 0: every row sees self key 0)
        const bool rescale = j > 0 && mx > m_prev + kRescaleThreshold;
        const float m_run = (j == 0 || rescale) ? mx : m_prev;
        m_pub[r] = m_run;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_m[s]);
        if (m_ref != m_run) {  // this group's sum so far was relative to an older max
          l_own = (m_ref == -INFINITY) ? 0.f : l_own * ex2_approx(m_ref - m_run);
          m_ref = m_run;
        }
        // P buffer s is free once PV_{Jc-2} has completed (also when this warp's epilogue
        // staging, which lives in the same rows of the same buffer, is done: program order)
        if (Jc >= 2) {
          const bool wp = mbar_wait(&bar_pv[s], ((Jc - 2) >> 1) & 1, p.wait_ns);
          if (!__all_sync(0xffffffffu, wp)) {
            ok = false;
            break;
          }
        }
        // the row's 64 probabilities 2^(s * scale_log2 - m_run), written as bf16 into the
        // 128-byte swizzled K-major row (16-byte unit u of row r sits at unit u ^ (r & 7)),
        // 32 at a time
        const float neg_m = -m_run;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        uint8_t* prow = sP + s * kPBytes + r * 128;
#pragma unroll
        for (int hp = 0; hp < 2; ++hp) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float e0 = ex2_approx(fmaf(__uint_as_float(sr[32 * hp + k]), c2, neg_m));
            const float e1 = ex2_approx(fmaf(__uint_as_float(sr[32 * hp + k + 1]), c2, neg_m));
            acc[(k >> 1) & 3] += e0 + e1;
            pk[k >> 1] = pack_bf16x2(e0, e1);
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint4 v;
            v.x = pk[4 * c + 0];
            v.y = pk[4 * c + 1];
            v.z = pk[4 * c + 2];
            v.w = pk[4 * c + 3];
            *reinterpret_cast<uint4*>(prow + (((4 * hp + c) ^ (r & 7)) << 4)) = v;
          }
        }
        l_own += (acc[0] + acc[1]) + (acc[2] + acc[3]);
        fence_proxy_async_smem();
        if (__any_sync(0xffffffffu, rescale)) {
          // O must hold the result of PV_{Jc-1} before it is rescaled in place
          const bool wr = mbar_wait(&bar_pv[s ^ 1], ((Jc - 1) >> 1) & 1, p.wait_ns);
          if (!__all_sync(0xffffffffu, wr)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = rescale ? ex2_approx(m_prev - m_run) : 1.f;
#pragma unroll 1
          for (int c = 0; c < kD; c += 32) {
            uint32_t o[32];
            tmem_ld32(lane_base + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(lane_base + c, o);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(&bar_p[s]);
      }
      if (!ok) break;
      // both groups' sums relative to the final running max (published by the last tile)
      const uint32_t Jl = J + it.nt - 1;
      float m_fin = m_ref;
      if (static_cast<int>(Jl & 1) != half) {
        const bool wm = mbar_wait(&bar_m[Jl & 1], (Jl >> 1) & 1, p.wait_ns);
        if (!__all_sync(0xffffffffu, wm)) {
          ok = false;
          break;
        }
        m_fin = m_pub[r];
      }
      const float l_run = (m_ref == -INFINITY) ? 0.f : l_own * ex2_approx(m_ref - m_fin);
      const float m_run = m_fin;
      // ---- epilogue of this item: O / l -> bf16, this half's 128 columns
      // l_part holds one item: the other group must have read the previous item's sums,
      // which it does before it loads that item's O (bar_ofree)
      if (n_it >= 1) {
        const bool wo = mbar_wait(bar_ofree, (n_it - 1) & 1, p.wait_ns);
        if (!__all_sync(0xffffffffu, wo)) {
          ok = false;
          break;
        }
      }
      l_part[half * 128 + r] = l_run;
      mbar_arrive(bar_l);
      // the item's last P V.  A parity wait is exact only when the barrier is at most one
      // phase behind it; the group whose own last tile is Jl - 1 never waited on P V_{Jl-2}
      // (same barrier), so it first waits on P V_{Jl-1} (other barrier, one phase at most),
      // after which P V_{Jl-2} has completed too (P V products complete in order)
      bool wt = (Jl == 0 || mbar_wait(&bar_pv[(Jl - 1) & 1], ((Jl - 1) >> 1) & 1, p.wait_ns)) &&
                mbar_wait(&bar_pv[Jl & 1], (Jl >> 1) & 1, p.wait_ns) && mbar_wait(bar_l, n_it & 1, p.wait_ns);
      if (!__all_sync(0xffffffffu, wt)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float l_tot = l_part[r] + l_part[128 + r];
      const float inv_l = 1.f / l_tot;
      const bool valid = pos < it.pos1;
      const int head = it.g * p.G + hh;
      // This warp's 32 rows go out through its own 4 KB staging tile in the (now idle)
      // P buffers, one 64-column slab at a time: each lane writes its row (swizzled,
      // so the writes are bank-conflict free), then reads it back row-major, 8 lanes
      // per 128-byte row, so every global store instruction writes 4 whole lines.
      const int r0 = quarter * 32;
      uint8_t* stage = sP + warp * 4096;
      // this thread's 128 O columns, two 32-column loads per wait, packed to bf16; O is
      // then free for the next item's P V before any store is issued
      uint4 vv[2][8];
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        uint32_t o[2][32];
        tmem_ld32(lane_base + half * 128 + hs * 64, o[0]);
        tmem_ld32(lane_base + half * 128 + hs * 64 + 32, o[1]);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4& v = vv[hs][c * 4 + q];
            v.x = pack_bf16x2(__uint_as_float(o[c][8 * q + 0]) * inv_l, __uint_as_float(o[c][8 * q + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[c][8 * q + 2]) * inv_l, __uint_as_float(o[c][8 * q + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[c][8 * q + 4]) * inv_l, __uint_as_float(o[c][8 * q + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[c][8 * q + 6]) * inv_l, __uint_as_float(o[c][8 * q + 7]) * inv_l);
          }
      }
      tc_fence_before();
      mbar_arrive(bar_ofree);  // O read out: the next item's first P V may overwrite it
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const int sl = 2 * half + hs;
        const uint4* v = vv[hs];
        uint8_t* row = stage + lane * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u) *reinterpret_cast<uint4*>(row + ((u ^ (lane & 7)) << 4)) = v[u];
        __syncwarp();
        const int cu = lane & 7;  // 16-byte unit of the row this lane copies
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = (lane >> 3) + 4 * k;  // row of the warp's 32
          const uint4 val = *reinterpret_cast<const uint4*>(stage + rr * 128 + ((cu ^ (rr & 7)) << 4));
          const int prow = r0 + rr;            // packed row = position x head
          const int ppos = it.pos0 + prow / p.G;
          if (ppos < it.pos1) {
            __nv_bfloat16* dst = p.out + (it.q0 + ppos) * p.ldo +
                                 static_cast<int64_t>(it.g * p.G + prow % p.G) * kD + sl * 64 + cu * 8;
            *reinterpret_cast<uint4*>(dst) = val;
          }
        }
        __syncwarp();  // staging tile read before it is refilled
      }
      if (valid && half == 0 && p.lse) {
        // natural-log softmax denominator in scaled-logit units
        p.lse[(it.q0 + pos) * p.n_q + head] = (m_run + log2f(l_tot)) * 0.69314718055994531f;
      }
      if constexpr (FUSED) {
        // this warp's O stores of the item are done; the signaller counts the item once all
        // eight warps have arrived (and only after it counted the previous one: at most one
        // item in flight on the barrier)
        __syncwarp();
        if (lane == 0) {
          const bool ws = n_it == 0 || mbar_wait(bar_osig, (n_it - 1) & 1, p.wait_ns);
          if (!ws) {
            record_error(p.err, kErrTimeout | kSiteAttention);
            *abort_flag = 1;
          }
          mbar_arrive(bar_ostored);
        }
      }
      J += it.nt;
      ++n_it;
    }
    if (!ok) {
      if (lane == 0) record_error(p.err, kErrTimeout | kSiteAttention);
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (FUSED) {
    // every attention product, read and store of this CTA is done: the buffers and the
    // tensor memory now serve the output projection
    tc_fence_after();
    out_proj_phase(p, f, &tm_oa, &tm_wo, smem, gemm_bars(bars), tmem, warp, lane, abort_flag);
    tc_fence_before();
    __syncthreads();
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Work order for the persistent kernel (one CTA).  An item's cost is its K/V tiles
// plus a fixed per-item part (the Q copy, the pipeline refill and the output write
// at the item's end, about three tiles' time); items without tiles cost nothing.
// The items are counting-sorted by cost, heaviest first, and dealt out in rounds
// of `grid` (the attention launch's CTA count): in each round the heaviest
// remaining item goes to the CTA with the least total cost so far, the next to the
// next least loaded, and so on (longest-processing-time-first, one item per CTA
// per round).  The result is laid out so that the attention kernel's CTA c takes
// entry k * grid + c in its k-th pass: the CTAs that receive an item in a last,
// partial round are renumbered 0 .. cnt - 1.  The order of equal costs is whatever
// the atomics give; each item's result does not depend on which CTA computes it.
constexpr int kSchedThreads = 1024;
constexpr int kSchedBins = 64;
constexpr int kItemFixedCost = 3;

__device__ __forceinline__ int item_cost(const AttnParams& p, int w) {
  const Item it = make_item(p, w);
  return it.nt > 0 ? min(it.nt + kItemFixedCost, kSchedBins - 1) : 0;
}

__global__ void __launch_bounds__(kSchedThreads) attention_schedule_kernel(const AttnParams p, int32_t* order,
                                                                          int grid) {
  __shared__ int hist[kSchedBins];
  __shared__ int next[kSchedBins];
  __shared__ int load[kSchedThreads];      // total cost dealt to each CTA so far
  __shared__ int seg_item[kSchedThreads];  // this round's items, heaviest first
  __shared__ int seg_cost[kSchedThreads];
  __shared__ int who[kSchedThreads];       // CTA that takes this round's i-th item
  __shared__ int label[kSchedThreads];     // final CTA number of each CTA
  pdl_launch_dependents();
  pdl_wait_predecessor();
  const int tid = threadIdx.x;
  const int n = p.n_items;
  if (tid < kSchedBins) hist[tid] = 0;
  __syncthreads();
  for (int w = tid; w < n; w += kSchedThreads) atomicAdd(&hist[kSchedBins - 1 - item_cost(p, w)], 1);
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int b = 0; b < kSchedBins; ++b) {
      next[b] = run;
      run += hist[b];
    }
  }
  __syncthreads();
  for (int w = tid; w < n; w += kSchedThreads) order[atomicAdd(&next[kSchedBins - 1 - item_cost(p, w)], 1)] = w;
  __syncthreads();  // the sorted list is in `order`: every thread reads it back below

  if (tid < grid) {
    load[tid] = 0;
    label[tid] = tid;
  }
  const int rounds = (n + grid - 1) / grid;
  int last_cnt = grid;
  for (int k = 0; k < rounds; ++k) {
    const int base = k * grid;
    const int cnt = min(grid, n - base);
    __syncthreads();
    if (tid < cnt) {
      seg_item[tid] = order[base + tid];
      seg_cost[tid] = item_cost(p, seg_item[tid]);
    }
    __syncthreads();
    if (tid < grid) {  // rank of this CTA by (cost so far, number), ascending
      const int l = load[tid];
      int rk = 0;
      for (int c = 0; c < grid; ++c) {
        const int lc = load[c];
        rk += (lc < l || (lc == l && c < tid)) ? 1 : 0;
      }
      if (rk < cnt) who[rk] = tid;
    }
    __syncthreads();
    if (tid < cnt) {
      const int v = who[tid];
      load[v] += seg_cost[tid];
      if (cnt == grid) order[base + v] = seg_item[tid];  // a full round: entry base + CTA
    }
    last_cnt = cnt;
  }
  if (last_cnt == grid) return;  // every round full: the CTA numbers stand
  // A partial last round: the CTA that takes its i-th item becomes CTA i (so the
  // round's entries, still in sorted order, stay where they are), the others keep
  // their relative order after them, and every full round is renumbered.
  __syncthreads();
  if (tid == 0) {
    for (int c = 0; c < grid; ++c) label[c] = -1;
    for (int i = 0; i < last_cnt; ++i) label[who[i]] = i;
    int nxt = last_cnt;
    for (int c = 0; c < grid; ++c)
      if (label[c] < 0) label[c] = nxt++;
  }
  __syncthreads();
  for (int k = 0; k + 1 < rounds; ++k) {
    const int base = k * grid;
    if (tid < grid) seg_item[tid] = order[base + tid];
    __syncthreads();
    if (tid < grid) order[base + label[tid]] = seg_item[tid];
    __syncthreads();
  }
}

}  // namespace

kalm_status setup_attention_kernels() {
  kalm_status st = check_cuda(
      cudaFuncSetAttribute(merged_attention_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem),
      "cudaFuncSetAttribute(merged_attention_kernel)");
  if (st != KALM_OK) return st;
  return check_cuda(
      cudaFuncSetAttribute(merged_attention_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem),
      "cudaFuncSetAttribute(merged_attention_kernel<fused>)");
}

}  // namespace kalm

using namespace kalm;

namespace {

// Output projection of the fused launch (kalm_merged_attention_out_proj); null: none.
struct OutProj {
  const kalm_bf16* w_o;
  int64_t ldw;
  kalm_bf16* x;
  int64_t ldx;
  int32_t hidden;
  int32_t* sync;
};

kalm_status launch_attention(const kalm_bf16* q, int64_t ldq, const kalm_bf16* k_self, const kalm_bf16* v_self,
                             int64_t ld_self, const kalm_bf16* k_cross, const kalm_bf16* v_cross, int64_t ld_cross,
                             const int64_t* q_off, const int64_t* in_off, int64_t total_in, const int64_t* pool_off,
                             int32_t n_docs, int32_t max_q, int64_t total_q, int64_t total_pool, int32_t n_q,
                             int32_t n_kv, int32_t head_dim, float scale, int32_t last_tile_only,
                             const int32_t* order, kalm_bf16* out, int64_t ldo, float* lse, const OutProj* op,
                             kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (head_dim != kD) return fail(KALM_ERR_UNSUPPORTED, "kalm_merged_attention: head_dim=%d (only 256)", head_dim);
  if (n_docs < 0 || n_q <= 0 || n_kv <= 0 || n_q % n_kv || max_q < 0 || max_q > KALM_MAX_QUERY_TOKENS ||
      total_q < 0 || total_pool < 0)
    return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention: bad sizes (n_docs=%d n_q=%d n_kv=%d max_q=%d)", n_docs,
                n_q, n_kv, max_q);
  const int G = n_q / n_kv;
  if (kBM % G) return fail(KALM_ERR_UNSUPPORTED, "kalm_merged_attention: n_q/n_kv=%d must divide 128", G);
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention: bad scale");
  if (n_docs == 0 || max_q == 0 || total_q == 0) return KALM_OK;
  if (!q || !k_self || !v_self || !out || !q_off || !pool_off || (total_pool > 0 && (!k_cross || !v_cross)))
    return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention: NULL pointer");
  if (ldq % 8 || ld_self % 8 || ld_cross % 8 || ldo % 8 || ldq < (int64_t)n_q * kD || ld_self < (int64_t)n_kv * kD ||
      (total_pool > 0 && ld_cross < (int64_t)n_kv * kD) || ldo < (int64_t)n_q * kD)
    return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention: strides must be multiples of 8 covering all heads");
  if (!aligned16(q) || !aligned16(k_self) || !aligned16(v_self) || !aligned16(out) ||
      (total_pool > 0 && (!aligned16(k_cross) || !aligned16(v_cross))))
    return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention: bf16 pointers must be 16-byte aligned");
  if (!in_off) total_in = total_q;
  if (total_in <= 0) return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention: total_in=%lld", (long long)total_in);
  if (total_q > INT32_MAX - 1024 || total_pool > INT32_MAX - 1024 || total_in > INT32_MAX - 1024)
    return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention: too many rows");

  // Q: a 4-D view (64 columns, head, row, 64-column slab) so one box moves a whole
  // 128-row x 256-column tile in the slab-major order the tensor-core descriptors read.
  CUtensorMap tq, tks, tvs, tkc, tvc;
  {
    const uint64_t dims[4] = {64, static_cast<uint64_t>(n_q), static_cast<uint64_t>(total_in), 4};
    const uint64_t strides[3] = {kD * 2, static_cast<uint64_t>(ldq) * 2, 128};
    const uint32_t box[4] = {64, static_cast<uint32_t>(G), static_cast<uint32_t>(kBM / G), 4};
    if ((st = make_tmap_bf16(&tq, q, 4, dims, strides, box)) != KALM_OK) return st;
  }
  // K and V: 3-D views (64 columns, row, 64-column slab over all KV heads); a box is
  // one 64-key x 256-column tile of one KV head.
  auto kv_map = [&](CUtensorMap* m, const kalm_bf16* base, int64_t ld, int64_t rows) -> kalm_status {
    const uint64_t dims[3] = {64, static_cast<uint64_t>(rows > 0 ? rows : 1), static_cast<uint64_t>(n_kv) * 4};
    const uint64_t strides[2] = {static_cast<uint64_t>(ld) * 2, 128};
    const uint32_t box[3] = {64, kBKV, 4};
    return make_tmap_bf16(m, base, 3, dims, strides, box);
  };
  if ((st = kv_map(&tks, k_self, ld_self, total_in)) != KALM_OK) return st;
  if ((st = kv_map(&tvs, v_self, ld_self, total_in)) != KALM_OK) return st;
  // with no cross rows at all, the cross maps are never read; point them at the self tensors
  if ((st = kv_map(&tkc, total_pool > 0 ? k_cross : k_self, total_pool > 0 ? ld_cross : ld_self,
                   total_pool > 0 ? total_pool : total_in)) != KALM_OK)
    return st;
  if ((st = kv_map(&tvc, total_pool > 0 ? v_cross : v_self, total_pool > 0 ? ld_cross : ld_self,
                   total_pool > 0 ? total_pool : total_in)) != KALM_OK)
    return st;

  AttnParams prm;
  prm.q_off = q_off;
  prm.in_off = in_off;
  prm.last_only = last_tile_only ? 1 : 0;
  prm.pool_off = pool_off;
  prm.out = reinterpret_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.ldo = ldo;
  prm.n_docs = n_docs;
  prm.n_q = n_q;
  prm.n_kv = n_kv;
  prm.G = G;
  prm.P = kBM / G;
  prm.tiles_per_doc = (max_q + prm.P - 1) / prm.P;
  prm.order = order;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wait_ns = kWaitNs;
  prm.err = device_error_word();
  const int64_t items = static_cast<int64_t>(last_tile_only ? 1 : prm.tiles_per_doc) * n_docs * n_kv;
  if (items > INT32_MAX) return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention: too many work items");
  prm.n_items = static_cast<int>(items);
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  const int64_t grid = items < sms ? items : sms;  // persistent: one CTA per SM
  if (!op) {
    return check_cuda(launch_pdl(merged_attention_kernel<false>, dim3(static_cast<unsigned>(grid)), dim3(kThreads),
                                 kSmem, static_cast<cudaStream_t>(stream), tq, tks, tvs, tkc, tvc, tq, tq, prm,
                                 ProjParams{}),
                      "launch merged_attention_kernel");
  }
  // fused output projection: A = O rows of a document (the `out` written above), B = Wo
  CUtensorMap toa, two;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(n_q) * kD, static_cast<uint64_t>(total_q)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ldo) * 2};
    const uint32_t box[2] = {64, kBM};
    if ((st = make_tmap_bf16(&toa, out, 2, dims, strides, box)) != KALM_OK) return st;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(n_q) * kD, static_cast<uint64_t>(op->hidden)};
    const uint64_t strides[1] = {static_cast<uint64_t>(op->ldw) * 2};
    const uint32_t box[2] = {64, 256};
    if ((st = make_tmap_bf16(&two, op->w_o, 2, dims, strides, box)) != KALM_OK) return st;
  }
  ProjParams fp{};
  fp.x = reinterpret_cast<__nv_bfloat16*>(op->x);
  fp.ldx = op->ldx;
  fp.hidden = op->hidden;
  fp.kdim = n_q * kD;
  fp.n_chunks = (op->hidden + 255) / 256;
  fp.m_tiles = (max_q + kBM - 1) / kBM;
  const int64_t otiles = static_cast<int64_t>(n_docs) * fp.m_tiles * fp.n_chunks;
  if (otiles + grid > INT32_MAX) return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention_out_proj: too many tiles");
  fp.n_otiles = static_cast<int>(otiles);
  fp.sync = op->sync;
  return check_cuda(launch_pdl(merged_attention_kernel<true>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), kSmem,
                               static_cast<cudaStream_t>(stream), tq, tks, tvs, tkc, tvc, toa, two, prm, fp),
                    "launch merged_attention_kernel<fused>");
}

}  // namespace

extern "C" kalm_status kalm_merged_attention(const kalm_bf16* q, int64_t ldq, const kalm_bf16* k_self,
                                             const kalm_bf16* v_self, int64_t ld_self, const kalm_bf16* k_cross,
                                             const kalm_bf16* v_cross, int64_t ld_cross, const int64_t* q_off,
                                             const int64_t* in_off, int64_t total_in, const int64_t* pool_off,
                                             int32_t n_docs, int32_t max_q, int64_t total_q, int64_t total_pool,
                                             int32_t n_q, int32_t n_kv, int32_t head_dim, float scale,
                                             int32_t last_tile_only, const int32_t* order, kalm_bf16* out,
                                             int64_t ldo, float* lse, kalm_stream_t stream) {
  return launch_attention(q, ldq, k_self, v_self, ld_self, k_cross, v_cross, ld_cross, q_off, in_off, total_in,
                          pool_off, n_docs, max_q, total_q, total_pool, n_q, n_kv, head_dim, scale, last_tile_only,
                          order, out, ldo, lse, nullptr, stream);
}

extern "C" int64_t kalm_attention_out_proj_sync_len(int32_t n_docs, int32_t max_q, int32_t hidden) {
  if (n_docs < 0 || max_q < 0 || hidden <= 0) return -1;
  const int64_t tiles = static_cast<int64_t>(n_docs) * ((max_q + kBM - 1) / kBM) * ((hidden + 255) / 256);
  return static_cast<int64_t>(n_docs) + 2 + tiles;
}

extern "C" kalm_status kalm_merged_attention_out_proj(
    const kalm_bf16* q, int64_t ldq, const kalm_bf16* k_self, const kalm_bf16* v_self, int64_t ld_self,
    const kalm_bf16* k_cross, const kalm_bf16* v_cross, int64_t ld_cross, const int64_t* q_off, const int64_t* in_off,
    int64_t total_in, const int64_t* pool_off, int32_t n_docs, int32_t max_q, int64_t total_q, int64_t total_pool,
    int32_t n_q, int32_t n_kv, int32_t head_dim, float scale, const int32_t* order, kalm_bf16* out, int64_t ldo,
    const kalm_bf16* w_o, int64_t ldw, kalm_bf16* x, int64_t ldx, int32_t hidden, int32_t* sync, int64_t sync_len,
    kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (n_docs < 0 || hidden <= 0 || hidden % 64)
    return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention_out_proj: hidden=%d must be a positive multiple of 64",
                hidden);
  if (n_docs == 0 || max_q == 0 || total_q == 0) return KALM_OK;
  if (!w_o || !x || !sync) return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention_out_proj: NULL pointer");
  if (sync_len < kalm_attention_out_proj_sync_len(n_docs, max_q, hidden))
    return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention_out_proj: sync_len=%lld < %lld", (long long)sync_len,
                (long long)kalm_attention_out_proj_sync_len(n_docs, max_q, hidden));
  if ((reinterpret_cast<uintptr_t>(sync) & 3u) || !aligned16(w_o) || !aligned16(x) || ldw % 8 || ldx % 8 ||
      ldw < static_cast<int64_t>(n_q) * head_dim || ldx < hidden)
    return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention_out_proj: bad alignment or stride");
  const OutProj op{w_o, ldw, x, ldx, hidden, sync};
  return launch_attention(q, ldq, k_self, v_self, ld_self, k_cross, v_cross, ld_cross, q_off, in_off, total_in,
                          pool_off, n_docs, max_q, total_q, total_pool, n_q, n_kv, head_dim, scale, 0, order, out, ldo,
                          nullptr, &op, stream);
}

// ----------------------------------------------------------------------------------
// The fused layer for callers that cannot allocate device memory.  Its counters live in a
// fixed array in the library's own device memory instead of a caller-provided buffer:
// every device that loads the library holds the array (4096 documents' counters and a queue of
// 49,152 projection tiles: 213,000 bytes) until the process exits.
namespace {

constexpr int kStaticSyncDocs = KALM_OUT_PROJ_STATIC_MAX_DOCS;    // documents per call
constexpr int kStaticSyncTiles = KALM_OUT_PROJ_STATIC_MAX_TILES;  // projection tiles per call
constexpr int kStaticSyncLen = kStaticSyncDocs + 2 + kStaticSyncTiles;
static __device__ __align__(256) int32_t g_out_proj_sync[kStaticSyncLen];

// Device address of g_out_proj_sync, looked up once per device (host code only sees a
// stand-in symbol, not a device address).
std::mutex g_static_sync_mutex;
int32_t* g_static_sync_ptr[64] = {};

kalm_status static_sync_ptr(int dev, int32_t** out) {
  if (dev < 0 || dev >= 64) return fail(KALM_ERR_NO_DEVICE, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_static_sync_mutex);
  if (!g_static_sync_ptr[dev]) {
    void* ptr = nullptr;
    kalm_status st = check_cuda(cudaGetSymbolAddress(&ptr, g_out_proj_sync), "cudaGetSymbolAddress(out-proj counters)");
    if (st != KALM_OK) return st;
    g_static_sync_ptr[dev] = static_cast<int32_t*>(ptr);
  }
  *out = g_static_sync_ptr[dev];
  return KALM_OK;
}

}  // namespace

extern "C" kalm_status kalm_merged_attention_out_proj_static(
    const kalm_bf16* q, int64_t ldq, const kalm_bf16* k_self, const kalm_bf16* v_self, int64_t ld_self,
    const kalm_bf16* k_cross, const kalm_bf16* v_cross, int64_t ld_cross, const int64_t* q_off, const int64_t* in_off,
    int64_t total_in, const int64_t* pool_off, int32_t n_docs, int32_t max_q, int64_t total_q, int64_t total_pool,
    int32_t n_q, int32_t n_kv, int32_t head_dim, float scale, const int32_t* order, kalm_bf16* out, int64_t ldo,
    const kalm_bf16* w_o, int64_t ldw, kalm_bf16* x, int64_t ldx, int32_t hidden, kalm_stream_t stream) {
  int dev = -1;
  kalm_status st = ensure_device(&dev);
  if (st != KALM_OK) return st;
  if (n_docs < 0 || max_q < 0 || hidden <= 0)
    return fail(KALM_ERR_INVALID_ARG, "kalm_merged_attention_out_proj_static: n_docs=%d max_q=%d hidden=%d", n_docs,
                max_q, hidden);
  const int64_t len = kalm_attention_out_proj_sync_len(n_docs, max_q, hidden);
  if (n_docs > kStaticSyncDocs || len - n_docs - 2 > kStaticSyncTiles)
    return fail(KALM_ERR_INVALID_ARG,
                "kalm_merged_attention_out_proj_static: %d documents and %lld projection tiles exceed what its "
                "built-in counters hold (%d documents, %d tiles); pass a counter array to "
                "kalm_merged_attention_out_proj instead",
                n_docs, (long long)(len - n_docs - 2), kStaticSyncDocs, kStaticSyncTiles);
  int32_t* sync = nullptr;
  if ((st = static_sync_ptr(dev, &sync)) != KALM_OK) return st;
  // the counters must start at zero: clear the part this call uses (a call cut short by a
  // device error may have left values behind)
  st = check_cuda(cudaMemsetAsync(sync, 0, static_cast<size_t>(len) * sizeof(int32_t),
                                  static_cast<cudaStream_t>(stream)),
                  "clear out-proj counters");
  if (st != KALM_OK) return st;
  return kalm_merged_attention_out_proj(q, ldq, k_self, v_self, ld_self, k_cross, v_cross, ld_cross, q_off, in_off,
                                        total_in, pool_off, n_docs, max_q, total_q, total_pool, n_q, n_kv, head_dim,
                                        scale, order, out, ldo, w_o, ldw, x, ldx, hidden, sync, len, stream);
}

extern "C" int64_t kalm_attention_items(int32_t n_docs, int32_t max_q, int32_t n_q, int32_t n_kv,
                                        int32_t last_tile_only) {
  if (n_docs < 0 || n_q <= 0 || n_kv <= 0 || n_q % n_kv || max_q < 0 || max_q > KALM_MAX_QUERY_TOKENS) return -1;
  const int G = n_q / n_kv;
  if (kBM % G) return -1;
  const int P = kBM / G;
  const int64_t tiles = last_tile_only ? 1 : (max_q + P - 1) / P;
  return max_q == 0 ? 0 : tiles * n_docs * n_kv;
}

extern "C" kalm_status kalm_attention_schedule(const int64_t* q_off, const int64_t* pool_off, int32_t n_docs,
                                               int32_t max_q, int32_t n_q, int32_t n_kv, int32_t last_tile_only,
                                               int32_t* order, int64_t order_len, kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  const int64_t items = kalm_attention_items(n_docs, max_q, n_q, n_kv, last_tile_only);
  if (items < 0)
    return fail(KALM_ERR_INVALID_ARG, "kalm_attention_schedule: bad sizes (n_docs=%d n_q=%d n_kv=%d max_q=%d)", n_docs,
                n_q, n_kv, max_q);
  if (items > INT32_MAX) return fail(KALM_ERR_INVALID_ARG, "kalm_attention_schedule: too many work items");
  if (order_len < items)
    return fail(KALM_ERR_INVALID_ARG, "kalm_attention_schedule: order_len=%lld < %lld work items",
                (long long)order_len, (long long)items);
  if (items == 0) return KALM_OK;
  if (!q_off || !pool_off || !order) return fail(KALM_ERR_INVALID_ARG, "kalm_attention_schedule: NULL pointer");
  AttnParams prm{};
  prm.q_off = q_off;
  prm.in_off = nullptr;
  prm.last_only = last_tile_only ? 1 : 0;
  prm.pool_off = pool_off;
  prm.n_docs = n_docs;
  prm.n_q = n_q;
  prm.n_kv = n_kv;
  prm.G = n_q / n_kv;
  prm.P = kBM / prm.G;
  prm.tiles_per_doc = (max_q + prm.P - 1) / prm.P;
  prm.n_items = static_cast<int>(items);
  prm.err = device_error_word();
  // the attention launch's CTA count for these sizes (one CTA per SM, at most one per item)
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms <= 0) sms = 148;
  int grid = items < sms ? static_cast<int>(items) : sms;
  if (grid > kSchedThreads) grid = kSchedThreads;  // only the balance depends on it
  return check_cuda(launch_pdl(attention_schedule_kernel, dim3(1), dim3(kSchedThreads), 0,
                               static_cast<cudaStream_t>(stream), prm, order, grid),
                    "launch attention_schedule_kernel");
}
