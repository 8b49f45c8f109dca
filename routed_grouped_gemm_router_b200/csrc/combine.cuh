// K-CB: un-permute and sum each token's k expert results.
//
// modelopt moe helpers, a2a_moe Flow: after the experts run, each token's
// top-k results are summed and returned in the hidden dtype. The routing
// weight is already applied in the down-GEMM epilogue, so this is a plain
// gather-sum: Y[t] = sum_j O[pair_pos[t*k+j]], fp32 in j order, one bf16
// rounding. One warp per token, 16-byte vectors (8 bf16), all k rows of a
// vector loaded before the adds so k loads are in flight per lane.
#pragma once
#include "common.cuh"

// The expert outputs are read once: load them with the streaming hint
// (evict-first) so they do not displace reused data from L2.
#ifndef MOE_COMBINE_STREAM_LOADS
#define MOE_COMBINE_STREAM_LOADS 1
#endif

namespace moe {

template <int KMAX>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ O, const int32_t* __restrict__ pair_pos,
                                                      int64_t T, int k, int vec_per_row, uint4* __restrict__ Y) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t P = T * k;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    int64_t rows[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      const int32_t r = (j < k) ? pair_pos[t * k + j] : -1;
      rows[j] = (r >= 0 && r < P) ? r : -1;
    }
    for (int c = lane; c < vec_per_row; c += 32) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      uint4 v[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
#if MOE_COMBINE_STREAM_LOADS
        v[j] = (rows[j] >= 0) ? __ldcs(O + rows[j] * vec_per_row + c) : make_uint4(0, 0, 0, 0);
#else
        v[j] = (rows[j] >= 0) ? __ldg(O + rows[j] * vec_per_row + c) : make_uint4(0, 0, 0, 0);
#endif
      }
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (rows[j] >= 0) {
          const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] += bf16lo(w[i]);
            acc[2 * i + 1] += bf16hi(w[i]);
          }
        }
      }
      uint4 out;
      out.x = pack_bf16(acc[0], acc[1]);
      out.y = pack_bf16(acc[2], acc[3]);
      out.z = pack_bf16(acc[4], acc[5]);
      out.w = pack_bf16(acc[6], acc[7]);
      Y[t * vec_per_row + c] = out;
    }
  }
}

// Generic path for large k: rows are read one after another.
__global__ void __launch_bounds__(256) combine_kernel_any_k(const uint4* __restrict__ O,
                                                            const int32_t* __restrict__ pair_pos, int64_t T, int k,
                                                            int vec_per_row, uint4* __restrict__ Y) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t P = T * k;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    for (int c = lane; c < vec_per_row; c += 32) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      for (int j = 0; j < k; ++j) {
        const int32_t r = pair_pos[t * k + j];
        if (r < 0 || r >= P) continue;
        const uint4 v = __ldg(O + static_cast<int64_t>(r) * vec_per_row + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] += bf16lo(w[i]);
          acc[2 * i + 1] += bf16hi(w[i]);
        }
      }
      uint4 out;
      out.x = pack_bf16(acc[0], acc[1]);
      out.y = pack_bf16(acc[2], acc[3]);
      out.z = pack_bf16(acc[4], acc[5]);
      out.w = pack_bf16(acc[6], acc[7]);
      Y[t * vec_per_row + c] = out;
    }
  }
}

inline cudaError_t launch_combine(const void* O, const int32_t* pair_pos, int T, int k, int H, void* Y,
                                  cudaStream_t s, int num_sms) {
  if (T == 0) return cudaSuccess;
  const int vec = H / 8;
  int blocks = (T + 7) / 8;
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  const uint4* o = static_cast<const uint4*>(O);
  uint4* y = static_cast<uint4*>(Y);
  const int64_t T64 = T;
  if (k <= 4) return launch_pdl(combine_kernel<4>, dim3(blocks), dim3(256), 0, s, o, pair_pos, T64, k, vec, y);
  if (k <= 8) return launch_pdl(combine_kernel<8>, dim3(blocks), dim3(256), 0, s, o, pair_pos, T64, k, vec, y);
  if (k <= 16) return launch_pdl(combine_kernel<16>, dim3(blocks), dim3(256), 0, s, o, pair_pos, T64, k, vec, y);
  return launch_pdl(combine_kernel_any_k, dim3(blocks), dim3(256), 0, s, o, pair_pos, T64, k, vec, y);
}

}  // namespace moe
