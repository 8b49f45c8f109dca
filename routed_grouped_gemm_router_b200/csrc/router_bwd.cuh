// K-RB: gradient of the router logits from the routing-weight gradients.
//
// Forward ("[WIP] Qwen3 MoE support", torchtune PR #2820, review comment):
//   p = softmax(l), S = sum_j p[idx_j] + 1e-20, w_j = p[idx_j] / S.
// With the selected set held constant:
//   dp[idx_j] = (dw_j - sum_i dw_i w_i) / S   (0 for unselected experts)
//   dl_e      = p_e (dp_e - sum_e' p_e' dp_e')
// dw_j itself is the sum over the down-GEMM N tiles of the partial dot
// products <dY[t], h W_d^T> written by the dgrad-down epilogue, read in fixed
// tile order. One warp per token; the logits row is built in shared memory
// and written out coalesced.
#pragma once
#include "common.cuh"

namespace moe {

__global__ void __launch_bounds__(256) router_bwd_kernel(const float* __restrict__ probs,
                                                         const int32_t* __restrict__ topk_idx,
                                                         const float* __restrict__ topk_w,
                                                         const float* __restrict__ dw_part,
                                                         const int32_t* __restrict__ pair_pos, int n_parts,
                                                         int64_t T, int E, int k, float* __restrict__ dlogits) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ float s_row[];  // [8 warps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* row = s_row + warp * E;
  const int64_t P = T * k;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp; t < T; t += warps) {
    const float* prow = probs + t * E;
    // pass 1: per selected slot j (lane-strided), dw_j, p_j, w_j
    float s_p = 0.f, s_dww = 0.f;
    for (int j = lane; j < k; j += 32) {
      const int64_t q = t * k + j;
      const int e = topk_idx[q];
      const int32_t r = pair_pos[q];
      float dw = 0.f;
      if (r >= 0 && r < P)
        for (int n = 0; n < n_parts; ++n) dw += dw_part[static_cast<int64_t>(r) * n_parts + n];
      const float pj = (e >= 0 && e < E) ? prow[e] : 0.f;
      s_p += pj;
      s_dww += dw * topk_w[q];
    }
    const float S = warp_sum_f(s_p) + 1e-20f;
    const float c1 = warp_sum_f(s_dww);
    // pass 2: dp on the selected slots and sum_e p_e dp_e
    float s_pdp = 0.f;
    for (int j = lane; j < k; j += 32) {
      const int64_t q = t * k + j;
      const int e = topk_idx[q];
      const int32_t r = pair_pos[q];
      float dw = 0.f;
      if (r >= 0 && r < P)
        for (int n = 0; n < n_parts; ++n) dw += dw_part[static_cast<int64_t>(r) * n_parts + n];
      const float pj = (e >= 0 && e < E) ? prow[e] : 0.f;
      s_pdp += pj * ((dw - c1) / S);
    }
    const float c2 = warp_sum_f(s_pdp);
    for (int e = lane; e < E; e += 32) row[e] = -prow[e] * c2;
    __syncwarp();
    for (int j = lane; j < k; j += 32) {
      const int64_t q = t * k + j;
      const int e = topk_idx[q];
      const int32_t r = pair_pos[q];
      float dw = 0.f;
      if (r >= 0 && r < P)
        for (int n = 0; n < n_parts; ++n) dw += dw_part[static_cast<int64_t>(r) * n_parts + n];
      if (e >= 0 && e < E) row[e] = prow[e] * ((dw - c1) / S - c2);
    }
    __syncwarp();
    float* drow = dlogits + t * E;
    for (int e = lane; e < E; e += 32) drow[e] = row[e];
    __syncwarp();
  }
}

}  // namespace moe
