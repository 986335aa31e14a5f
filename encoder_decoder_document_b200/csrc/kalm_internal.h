// Host-side helpers shared by the entry points of libkalm (not part of the ABI).
#pragma once

#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kalm.h"

namespace kalm {

// Record a detail message for kalm_last_error() and return `st`.
kalm_status fail(kalm_status st, const char* fmt, ...);

// Check that the current device is sm_100 and run its one-time set-up (kernel
// attributes, device error word address).  Returns KALM_OK or an error.
kalm_status ensure_device(int* device_out);

// Device address of the current device's error word (valid after ensure_device).
uint32_t* device_error_word();

// Streaming multiprocessors of the current device (cached at set-up).
int num_sms();

// Map a CUDA runtime error to KALM_ERR_CUDA with its message; KALM_OK if none.
kalm_status check_cuda(cudaError_t e, const char* what);

// Tiled bf16 tensor maps with zero fill outside the tensor.  `dims`/`box` list
// the innermost dimension first; `strides_bytes` holds the byte strides of
// dimensions 1.. (rank-1 values); `swizzle_bytes` is 128 (default), 64, 32 or 0.
kalm_status make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                           const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes = 128);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch with programmatic stream serialization (the kernel must call
// pdl_wait_predecessor() before it touches global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace kalm
