// Helpers of the expert-parallel layer (experts split over ranks; the rows
// travel to the rank that owns their expert and back). modelopt `moe`
// helpers, a2a_moe Flow: the (token, expert) pairs are expanded, sent to the
// experts, computed there, sent back, weighted and summed per token.
#pragma once
#include "common.cuh"

namespace moe {

// For every expert-sorted row r of expert e (rows [offsets[e], offsets[e+1])):
// the expert's index on its owner rank (experts are split into contiguous
// blocks of experts_per_rank) and the row's routing weight topk_w[pair],
// pair = sorted_pair[r]. One block per expert, its rows in order.
__global__ void __launch_bounds__(256) ep_pack_rows_kernel(const int32_t* __restrict__ offsets,
                                                           const int32_t* __restrict__ sorted_pair,
                                                           const float* __restrict__ topk_w, int64_t P,
                                                           int experts_per_rank, int32_t* __restrict__ local_expert,
                                                           float* __restrict__ row_w) {
  griddep_wait();
  griddep_launch_dependents();
  const int e = blockIdx.x;
  const int lo = offsets[e], hi = offsets[e + 1];
  const int le = e % experts_per_rank;
  for (int r = lo + threadIdx.x; r < hi; r += blockDim.x) {
    if (r < 0 || r >= P) {
      report(MOE_ERR_DEVICE_CHECK);
      continue;
    }
    const int32_t q = sorted_pair[r];
    local_expert[r] = le;
    row_w[r] = (q >= 0 && q < P) ? __ldg(topk_w + q) : 0.0f;
  }
}

// The routing-weight gradient of every pair q: the sum, in tile order, of
// the partial dot products <dY[t], h W_d^T> that the dgrad-down epilogue
// wrote for the pair's row pair_pos[q] (n_parts per row).
__global__ void __launch_bounds__(256) pair_dw_kernel(const float* __restrict__ dw_part,
                                                      const int32_t* __restrict__ pair_pos, int n_parts, int64_t P,
                                                      float* __restrict__ dw) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < P; q += stride) {
    const int32_t r = pair_pos[q];
    float s = 0.f;
    if (r >= 0 && r < P)
      for (int n = 0; n < n_parts; ++n) s += dw_part[static_cast<int64_t>(r) * n_parts + n];
    dw[q] = s;
  }
}

}  // namespace moe
