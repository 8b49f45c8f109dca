// Low-rank adapter helper kernel (the adapter GEMMs themselves run in the
// grouped GEMM: its K extension and its plain and weight-gradient kinds).
// Source: fused-MoE Triton project summary (sourcepulse), Highlighted
// Details: LoRA on the fused expert weights; the update is the published LoRA
// form W + scale * B A, per expert.
#pragma once
#include <cstdint>

#include "common.cuh"

namespace moe {

// out[r, :] = topk_w[sorted_pair[r]] * in[r, :] over the P permuted rows of a
// [P, R] bf16 matrix, R = 8 * r8 (one 16-byte piece per thread): the routing-
// weighted copy of the down adapter's activations scale * (h A_d^T), whose
// product with the permuted upstream gradient is that adapter's B gradient.
// A pair id outside [0, P) gives weight 0.
__global__ void __launch_bounds__(256) lora_weight_rows_kernel(const uint4* __restrict__ in,
                                                               const int32_t* __restrict__ sorted_pair,
                                                               const float* __restrict__ topk_w, int64_t P, int r8,
                                                               uint4* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t n = P * r8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / r8;
    const int32_t q = sorted_pair[row];
    const float w = (q >= 0 && q < P) ? __ldg(topk_w + q) : 0.0f;
    const uint4 v = in[i];
    uint4 o;
    o.x = pack_bf16(w * bf16lo(v.x), w * bf16hi(v.x));
    o.y = pack_bf16(w * bf16lo(v.y), w * bf16hi(v.y));
    o.z = pack_bf16(w * bf16lo(v.z), w * bf16hi(v.z));
    o.w = pack_bf16(w * bf16lo(v.w), w * bf16hi(v.w));
    out[i] = o;
  }
}

}  // namespace moe
