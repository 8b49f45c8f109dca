// K-RB: gradient of the router logits from the routing-weight gradients.
//
// Forward ("[WIP] Qwen3 MoE support", torchtune PR #2820, review comment):
//   p = softmax(l), S = sum_j p[idx_j] + 1e-20, w_j = p[idx_j] / S.
// With the selected set held constant:
//   dp[idx_j] = (dw_j - sum_i dw_i w_i) / S   (0 for unselected experts)
//   dl_e      = p_e (dp_e - sum_e' p_e' dp_e')
// dw_j itself is the sum over the down-GEMM N tiles of the partial dot
// products <dY[t], h W_d^T> written by the dgrad-down epilogue, read in fixed
// tile order.
#pragma once
#include "common.cuh"

namespace moe {

// One warp per token. For k <= 32 each top-k slot j has R = 32 / kp lanes
// (kp = k rounded up to a power of two) that read the slot's partials in
// parallel (lane sub of the group takes parts sub, sub + R, ...) and add them
// in a fixed butterfly. The probs row is read once, coalesced, into
// registers (lane l holds experts l + 32 v), and the d logits row is written
// from them, coalesced: -p_e c2 everywhere, p_e (dp_j - c2) at the k selected
// experts (each slot's expert and dp broadcast from its group's first lane).
// k > 32: one lane per slot, parts in order.
template <int VPL>
__global__ void __launch_bounds__(256) router_bwd_kernel(const float* __restrict__ probs,
                                                         const int32_t* __restrict__ topk_idx,
                                                         const float* __restrict__ topk_w,
                                                         const float* __restrict__ dw_part,
                                                         const int32_t* __restrict__ pair_pos, int n_parts,
                                                         int64_t T, int E, int k, float* __restrict__ dlogits) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t P = T * k;
  int kp = 1;
  while (kp < k && kp < 32) kp <<= 1;
  const int R = (k <= 32) ? 32 / kp : 1;         // lanes per slot
  const int j0 = (k <= 32) ? lane / R : lane;     // first slot of this lane
  const int sub = (k <= 32) ? lane % R : 0;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    const float* prow = probs + t * E;
    float pe[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int e = lane + 32 * v;
      pe[v] = (e < E) ? __ldg(prow + e) : 0.f;
    }
    float out[VPL];
    if (k <= 32) {
      // this lane's slot: its expert, weight, probability and dw
      const bool act = j0 < k;
      const int64_t q = t * k + (act ? j0 : 0);
      const int e = act ? __ldg(topk_idx + q) : -1;
      const bool valid = act && e >= 0 && e < E;
      const int32_t r = act ? __ldg(pair_pos + q) : -1;
      float dw = 0.f;
      if (act && r >= 0 && r < P)
        for (int n = sub; n < n_parts; n += R) dw += __ldg(dw_part + static_cast<int64_t>(r) * n_parts + n);
      for (int o = R >> 1; o > 0; o >>= 1) dw += __shfl_xor_sync(0xffffffffu, dw, o);
      const bool lead = act && sub == 0;
      const float pj = valid ? __ldg(prow + e) : 0.f;
      const float wj = act ? __ldg(topk_w + q) : 0.f;
      const float S = warp_sum_f(lead ? pj : 0.f) + 1e-20f;
      const float c1 = warp_sum_f(lead ? dw * wj : 0.f);
      const float dpj = (dw - c1) / S;
      const float c2 = warp_sum_f(lead ? pj * dpj : 0.f);
#pragma unroll
      for (int v = 0; v < VPL; ++v) out[v] = -pe[v] * c2;
      for (int j = 0; j < k; ++j) {
        const int ej = __shfl_sync(0xffffffffu, valid ? e : -1, j * R);
        const float dj = __shfl_sync(0xffffffffu, dpj, j * R);
#pragma unroll
        for (int v = 0; v < VPL; ++v)
          if (lane + 32 * v == ej) out[v] = pe[v] * (dj - c2);
      }
    } else {
      float s_p = 0.f, s_dww = 0.f;
      for (int j = lane; j < k; j += 32) {
        const int64_t q = t * k + j;
        const int e = topk_idx[q];
        const int32_t r = pair_pos[q];
        float dw = 0.f;
        if (r >= 0 && r < P)
          for (int n = 0; n < n_parts; ++n) dw += dw_part[static_cast<int64_t>(r) * n_parts + n];
        s_p += (e >= 0 && e < E) ? prow[e] : 0.f;
        s_dww += dw * topk_w[q];
      }
      const float S = warp_sum_f(s_p) + 1e-20f;
      const float c1 = warp_sum_f(s_dww);
      float s_pdp = 0.f;
      for (int j = lane; j < k; j += 32) {
        const int64_t q = t * k + j;
        const int e = topk_idx[q];
        const int32_t r = pair_pos[q];
        float dw = 0.f;
        if (r >= 0 && r < P)
          for (int n = 0; n < n_parts; ++n) dw += dw_part[static_cast<int64_t>(r) * n_parts + n];
        s_pdp += ((e >= 0 && e < E) ? prow[e] : 0.f) * ((dw - c1) / S);
      }
      const float c2 = warp_sum_f(s_pdp);
#pragma unroll
      for (int v = 0; v < VPL; ++v) out[v] = -pe[v] * c2;
      // slots in groups of 32: each lane owns one slot per group, broadcast in turn
      for (int jb = 0; jb < k; jb += 32) {
        const int j = jb + lane;
        int e = -1;
        float dpj = 0.f;
        if (j < k) {
          const int64_t q = t * k + j;
          e = topk_idx[q];
          const int32_t r = pair_pos[q];
          float dw = 0.f;
          if (r >= 0 && r < P)
            for (int n = 0; n < n_parts; ++n) dw += dw_part[static_cast<int64_t>(r) * n_parts + n];
          dpj = (dw - c1) / S;
          if (e < 0 || e >= E) e = -1;
        }
        const int nj = (k - jb < 32) ? k - jb : 32;
        for (int i = 0; i < nj; ++i) {
          const int ej = __shfl_sync(0xffffffffu, e, i);
          const float dj = __shfl_sync(0xffffffffu, dpj, i);
#pragma unroll
          for (int v = 0; v < VPL; ++v)
            if (lane + 32 * v == ej) out[v] = pe[v] * (dj - c2);
        }
      }
    }
    float* drow = dlogits + t * E;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int e = lane + 32 * v;
      if (e < E) drow[e] = out[v];
    }
  }
}

inline cudaError_t launch_router_bwd(const float* probs, const int32_t* topk_idx, const float* topk_w,
                                     const float* dw_part, const int32_t* pair_pos, int n_parts, int64_t T, int E,
                                     int k, float* dlogits, int num_sms, cudaStream_t s) {
  int64_t blocks = (T + 7) / 8;
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  const int vpl = (E + 31) / 32;
#define MOE_ROUTER_BWD_CASE(V)                                                                                 \
  if (vpl <= V)                                                                                                \
    return launch_pdl(router_bwd_kernel<V>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, probs, topk_idx, \
                      topk_w, dw_part, pair_pos, n_parts, T, E, k, dlogits);
  MOE_ROUTER_BWD_CASE(1)
  MOE_ROUTER_BWD_CASE(2)
  MOE_ROUTER_BWD_CASE(4)
  MOE_ROUTER_BWD_CASE(8)
  MOE_ROUTER_BWD_CASE(16)
  MOE_ROUTER_BWD_CASE(32)
#undef MOE_ROUTER_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace moe
