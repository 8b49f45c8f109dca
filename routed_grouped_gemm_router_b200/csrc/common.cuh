// Shared device helpers: the device status word, bf16 packing, warp utilities.
#pragma once
#include <atomic>
#include <cstdint>
#include <utility>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/moe.h"
#include "sm100.cuh"

namespace moe {

// Device-side error word: the first kernel that detects a problem (a wait that
// ran out, an expert id outside [0, E)) stores its code here; the host reads
// and clears it with moe_last_device_status. Kernels never trap.
__device__ int g_device_status = 0;

__device__ __forceinline__ void report(int code) { atomicCAS(&g_device_status, 0, code); }

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Round two floats to bf16 (nearest-even) and pack them, lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Inclusive prefix sum across the 32 lanes of a warp.
__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Kernels this library has launched in the process (every launch goes
// through launch_pdl_clustered; read with moe_launch_count).
inline std::atomic<unsigned long long>& launch_count() {
  static std::atomic<unsigned long long> n{0};
  return n;
}

// Launches `kernel` on stream `s` with programmatic stream serialisation, so
// its set-up may overlap the tail of the previous kernel on the stream (the
// kernel itself waits for that kernel's results, see griddep_wait).
// cluster_x > 1 launches clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_clustered(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                        cudaStream_t s, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
#ifndef MOE_PDL
#define MOE_PDL 1
#endif
  attr[0].val.programmaticStreamSerializationAllowed = MOE_PDL;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster_x > 1 ? 2 : 1;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (err == cudaSuccess) launch_count().fetch_add(1, std::memory_order_relaxed);
  return err;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  return launch_pdl_clustered(kernel, grid, block, smem, s, 1u, std::forward<Args>(args)...);
}

}  // namespace moe
