// Runtime plumbing of libkalm: status strings, device check, device error word,
// tensor-map encoding, ragged offsets, row broadcast and the bounded-wait
// self-test.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "kalm.h"
#include "kalm_internal.h"
#include "kalm_ptx.cuh"

namespace kalm {

namespace {

thread_local char g_last_error[512] = {0};

// One error word per device (each device that loads the module holds its own copy).
__device__ uint32_t g_device_error_word;
// Where the read-and-clear kernel leaves the word it took (one per device as well).
__device__ uint32_t g_error_word_taken;

constexpr int kMaxDevices = 64;
// `ready` is published with release order after every other field of the
// device's set-up (and the per-kernel tables written by the set-up hooks), so a
// thread that reads it true with acquire order also sees those writes.
struct DeviceState {
  std::atomic<bool> ready{false};
  bool ok = false;
  uint32_t* err = nullptr;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mutex;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

}  // namespace

kalm_status fail(kalm_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

kalm_status check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return KALM_OK;
  return fail(KALM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Per-kernel set-up hooks defined in the other translation units.
kalm_status setup_linear_kernels();
kalm_status setup_attention_kernels();

kalm_status ensure_device(int* device_out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return fail(KALM_ERR_NO_DEVICE, "no CUDA device: %s", cudaGetErrorString(e));
  }
  if (dev >= kMaxDevices) return fail(KALM_ERR_NO_DEVICE, "device index %d out of range", dev);
  if (device_out) *device_out = dev;
  DeviceState& s = g_dev[dev];
  if (s.ready.load(std::memory_order_acquire))
    return s.ok ? KALM_OK : fail(KALM_ERR_NO_DEVICE, "device %d is not an sm_100 device", dev);
  std::lock_guard<std::mutex> lock(g_mutex);
  if (s.ready.load(std::memory_order_relaxed))
    return s.ok ? KALM_OK : fail(KALM_ERR_NO_DEVICE, "device %d is not an sm_100 device", dev);
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return fail(KALM_ERR_NO_DEVICE, "cannot query device %d", dev);
  }
  if (major != 10 || minor != 0) {
    s.ok = false;
    s.ready.store(true, std::memory_order_release);
    return fail(KALM_ERR_NO_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a only", dev, major,
                minor);
  }
  void* p = nullptr;
  kalm_status st = check_cuda(cudaGetSymbolAddress(&p, g_device_error_word), "cudaGetSymbolAddress(error word)");
  if (st != KALM_OK) return st;
  s.err = static_cast<uint32_t*>(p);
  st = check_cuda(cudaMemset(s.err, 0, sizeof(uint32_t)), "clear error word");
  if (st != KALM_OK) return st;
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    st = check_cuda(cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q),
                    "cudaGetDriverEntryPointByVersion(cuTensorMapEncodeTiled)");
    if (st != KALM_OK) return st;
    if (q != cudaDriverEntryPointSuccess || !fn)
      return fail(KALM_ERR_CUDA, "driver entry point cuTensorMapEncodeTiled not found");
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  if ((st = setup_linear_kernels()) != KALM_OK) return st;
  if ((st = setup_attention_kernels()) != KALM_OK) return st;
  s.ok = true;
  s.ready.store(true, std::memory_order_release);
  return KALM_OK;
}

uint32_t* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  return g_dev[dev].err;
}

kalm_status make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
  if (!g_encode) return fail(KALM_ERR_CUDA, "tensor-map encoder not initialised");
  cuuint64_t gdim[5];
  cuuint64_t gstride[4];
  cuuint32_t bdim[5];
  cuuint32_t estride[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estride[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gstride[i] = strides_bytes[i];
  const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                        gdim, gstride, bdim, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KALM_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return KALM_OK;
}

// ---------------------------------------------------------------------------
// kernels
// ---------------------------------------------------------------------------
namespace {

// Single-CTA exclusive scan of len and ceil(len/chunk).  n is a few thousand
// documents at most, so one CTA of 1024 threads walks it in 1024-wide steps.
__global__ void __launch_bounds__(1024) ragged_offsets_kernel(const int32_t* __restrict__ len, int32_t n,
                                                              int32_t chunk, int64_t* __restrict__ tok_off,
                                                              int64_t* __restrict__ pool_off, uint32_t* err) {
  pdl_launch_dependents();
  pdl_wait_predecessor();
  __shared__ int64_t warp_tok[32];
  __shared__ int64_t warp_pool[32];
  __shared__ int64_t carry[2];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) {
    carry[0] = 0;
    carry[1] = 0;
  }
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + tid;
    int64_t t = 0, p = 0;
    if (i < n) {
      int32_t v = len[i];
      if (v < 0 || v > KALM_MAX_DOC_TOKENS) {
        record_error(err, kErrDeviceArg | kSiteOffsets);
        v = v < 0 ? 0 : KALM_MAX_DOC_TOKENS;
      }
      t = v;
      p = (v + chunk - 1) / chunk;
    }
    // inclusive warp scan
    int64_t it = t, ip = p;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t a = __shfl_up_sync(0xffffffffu, it, o);
      int64_t b = __shfl_up_sync(0xffffffffu, ip, o);
      if (lane >= o) {
        it += a;
        ip += b;
      }
    }
    if (lane == 31) {
      warp_tok[wid] = it;
      warp_pool[wid] = ip;
    }
    __syncthreads();
    if (wid == 0) {
      int64_t a = warp_tok[lane], b = warp_pool[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int64_t x = __shfl_up_sync(0xffffffffu, a, o);
        int64_t y = __shfl_up_sync(0xffffffffu, b, o);
        if (lane >= o) {
          a += x;
          b += y;
        }
      }
      warp_tok[lane] = a;  // inclusive over warps
      warp_pool[lane] = b;
    }
    __syncthreads();
    const int64_t wt = wid ? warp_tok[wid - 1] : 0, wp = wid ? warp_pool[wid - 1] : 0;
    const int64_t c0 = carry[0], c1 = carry[1];
    if (i < n) {
      // exclusive value at i, inclusive written at i+1
      if (tok_off) tok_off[i + 1] = c0 + wt + it;
      if (pool_off) pool_off[i + 1] = c1 + wp + ip;
    }
    __syncthreads();
    if (tid == 0) {
      carry[0] = c0 + warp_tok[31];
      carry[1] = c1 + warp_pool[31];
    }
    __syncthreads();
  }
  if (tid == 0) {
    if (tok_off) tok_off[0] = 0;
    if (pool_off) pool_off[0] = 0;
  }
}

__global__ void broadcast_rows_kernel(const uint4* __restrict__ src, int64_t ld_src_v, int32_t rows, int32_t width_v,
                                      const int64_t* __restrict__ q_off, int32_t n_docs, uint4* __restrict__ dst,
                                      int64_t ld_dst_v) {
  pdl_launch_dependents();
  pdl_wait_predecessor();
  const int d = blockIdx.y;
  const int64_t r0 = q_off[d];
  int64_t nr = q_off[d + 1] - r0;
  if (nr > rows) nr = rows;
  const int64_t total = nr * width_v;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / width_v, c = i - r * width_v;
    dst[(r0 + r) * ld_dst_v + c] = src[r * ld_src_v + c];
  }
}

// Reads and clears the error word in one atomic step, so a bit that another
// stream's kernel sets at the same moment lands either in this read or in the
// next one, never in neither.
__global__ void take_error_word_kernel() { g_error_word_taken = atomicExch(&g_device_error_word, 0u); }

// Waits on a barrier that is never completed; the bounded wait must expire.
__global__ void selftest_wait_kernel(uint64_t wait_ns, uint32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(&bar, 0, wait_ns)) record_error(err, kErrTimeout | kSiteSelftest);
  }
  __syncthreads();
}

}  // namespace
}  // namespace kalm

using namespace kalm;

extern "C" {

int kalm_version(void) { return 100; }

const char* kalm_status_string(int status) {
  switch (status) {
    case KALM_OK: return "KALM_OK";
    case KALM_ERR_INVALID_ARG: return "KALM_ERR_INVALID_ARG";
    case KALM_ERR_UNSUPPORTED: return "KALM_ERR_UNSUPPORTED";
    case KALM_ERR_NO_DEVICE: return "KALM_ERR_NO_DEVICE";
    case KALM_ERR_CUDA: return "KALM_ERR_CUDA";
    case KALM_ERR_TIMEOUT: return "KALM_ERR_TIMEOUT";
    case KALM_ERR_DEVICE_ARG: return "KALM_ERR_DEVICE_ARG";
    default: return "KALM_ERR_UNKNOWN";
  }
}

const char* kalm_last_error(void) { return kalm::g_last_error; }

kalm_status kalm_device_check(void) { return ensure_device(nullptr); }

kalm_status kalm_check_device_errors(kalm_stream_t stream, uint32_t* word_out) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  // stream-ordered after the work already queued on `stream`: take the word atomically,
  // copy it out, wait for both
  take_error_word_kernel<<<1, 1, 0, s>>>();
  st = check_cuda(cudaGetLastError(), "launch take_error_word_kernel");
  if (st != KALM_OK) return st;
  uint32_t w = 0;
  st = check_cuda(cudaMemcpyFromSymbolAsync(&w, kalm::g_error_word_taken, sizeof(w), 0, cudaMemcpyDeviceToHost, s),
                  "read error word");
  if (st != KALM_OK) return st;
  st = check_cuda(cudaStreamSynchronize(s), "cudaStreamSynchronize");
  if (st != KALM_OK) return st;
  if (word_out) *word_out = w;
  if (w & kErrTimeout) return fail(KALM_ERR_TIMEOUT, "device wait expired (error word 0x%x)", w);
  if (w & kErrDeviceArg) return fail(KALM_ERR_DEVICE_ARG, "invalid device data (error word 0x%x)", w);
  return KALM_OK;
}

kalm_status kalm_ragged_offsets(const int32_t* len, int32_t n, int32_t chunk, int64_t* tok_off, int64_t* pool_off,
                                kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (n < 0 || chunk < 1) return fail(KALM_ERR_INVALID_ARG, "kalm_ragged_offsets: n=%d chunk=%d", n, chunk);
  if (n > 0 && !len) return fail(KALM_ERR_INVALID_ARG, "kalm_ragged_offsets: len is NULL");
  if (!tok_off && !pool_off) return KALM_OK;
  return check_cuda(launch_pdl(ragged_offsets_kernel, dim3(1), dim3(1024), 0, static_cast<cudaStream_t>(stream), len,
                                n, chunk, tok_off, pool_off, device_error_word()),
                    "launch ragged_offsets_kernel");
}

kalm_status kalm_broadcast_rows(const kalm_bf16* src, int64_t ld_src, int32_t rows, int32_t width,
                                const int64_t* q_off, int32_t n_docs, kalm_bf16* dst, int64_t ld_dst,
                                kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (n_docs < 0 || rows < 0 || width < 0) return fail(KALM_ERR_INVALID_ARG, "kalm_broadcast_rows: negative size");
  if (n_docs == 0 || rows == 0 || width == 0) return KALM_OK;
  if (!src || !dst || !q_off) return fail(KALM_ERR_INVALID_ARG, "kalm_broadcast_rows: NULL pointer");
  if (width % 8 || ld_src % 8 || ld_dst % 8 || ld_src < width || ld_dst < width || !aligned16(src) ||
      !aligned16(dst))
    return fail(KALM_ERR_INVALID_ARG, "kalm_broadcast_rows: width/strides must be multiples of 8, 16-B aligned");
  if (n_docs > 65535) return fail(KALM_ERR_INVALID_ARG, "kalm_broadcast_rows: n_docs > 65535");
  const int32_t wv = width / 8;
  const int64_t per_doc = (int64_t)rows * wv;
  int bx = (int)((per_doc + 255) / 256);
  if (bx > 64) bx = 64;
  dim3 grid(bx, n_docs);
  return check_cuda(launch_pdl(broadcast_rows_kernel, grid, dim3(256), 0, static_cast<cudaStream_t>(stream),
                                reinterpret_cast<const uint4*>(src), ld_src / 8, rows, wv, q_off, n_docs,
                                reinterpret_cast<uint4*>(dst), ld_dst / 8),
                    "launch broadcast_rows_kernel");
}

kalm_status kalm_selftest_wait_timeout(uint64_t wait_ns, kalm_stream_t stream) {
  kalm_status st = ensure_device(nullptr);
  if (st != KALM_OK) return st;
  if (wait_ns > 2000000000ull) return fail(KALM_ERR_INVALID_ARG, "wait_ns above 2 s");
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(wait_ns, device_error_word());
  return check_cuda(cudaGetLastError(), "launch selftest_wait_kernel");
}

}  // extern "C"
