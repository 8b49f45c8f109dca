// K-RT: router softmax -> top-k -> renormalise, one warp per token.
//
// fused-MoE Triton project summary, Highlighted Details: softmax and top-k are
// fused into one kernel; "[WIP] Qwen3 MoE support" (torchtune PR #2820),
// review comment: top-k scores are divided by their sum + 1e-20.
//
// Lane l holds experts e = l + 32*v (v < VPL) in registers, so the logits row
// is read once, coalesced. With n_part > 0 the logits are not read from
// `logits` but summed from the router GEMM's split-K partials
// (part[s * part_stride + t * part_ld + e], s = 0..n_part-1 in order) and
// written to `logits_out` (if not null). Selection compares the fp32 logits themselves
// (logit descending, lower expert index on ties), which makes the chosen set
// and its order exactly reproducible on any processor given the same logits.
#pragma once
#include "common.cuh"

namespace moe {

// Most split-K partials of the router logits the routing kernel sums.
constexpr int kRouteMaxParts = 8;

// Routes token t with one warp: softmax, top-k on the logits, renormalised
// weights (written to topk_idx / topk_w / probs). On return, lane l holds in
// isel[v] the expert of top-k slot j = l + 32 v (for j < k).
template <int VPL>
__device__ __forceinline__ void route_token(const float* __restrict__ logits, int64_t t, int E, int k,
                                            int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                            float* __restrict__ probs, const float* __restrict__ part, int n_part,
                                            int part_ld, int64_t part_stride, float* __restrict__ logits_out,
                                            int (&isel)[VPL]) {
  const int lane = threadIdx.x & 31;
  float l[VPL];
  float m = -INFINITY;
  if (n_part == 0) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int e = lane + 32 * v;
      l[v] = (e < E) ? __ldg(logits + static_cast<int64_t>(t) * E + e) : -INFINITY;
    }
  } else if constexpr (VPL > 4) {
    // wide rows: one partial at a time, the row's values in parallel
#pragma unroll
    for (int v = 0; v < VPL; ++v) l[v] = 0.0f;
    for (int s = 0; s < n_part; ++s) {
      float pv[VPL];
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int e = lane + 32 * v;
        pv[v] = (e < E) ? __ldg(part + s * part_stride + static_cast<int64_t>(t) * part_ld + e) : 0.0f;
      }
#pragma unroll
      for (int v = 0; v < VPL; ++v) l[v] += pv[v];
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int e = lane + 32 * v;
      if (e < E && logits_out != nullptr) logits_out[static_cast<int64_t>(t) * E + e] = l[v];
      if (e >= E) l[v] = -INFINITY;
    }
  } else {
    // every partial of every value is requested before the first add
    float pv[kRouteMaxParts][VPL];
#pragma unroll
    for (int s = 0; s < kRouteMaxParts; ++s)
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int e = lane + 32 * v;
        pv[s][v] = (s < n_part && e < E) ? __ldg(part + s * part_stride + static_cast<int64_t>(t) * part_ld + e)
                                         : 0.0f;
      }
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int e = lane + 32 * v;
      float acc = pv[0][v];
#pragma unroll
      for (int s = 1; s < kRouteMaxParts; ++s)
        if (s < n_part) acc += pv[s][v];
      l[v] = (e < E) ? acc : -INFINITY;
      if (e < E && logits_out != nullptr) logits_out[static_cast<int64_t>(t) * E + e] = acc;
    }
  }
#pragma unroll
  for (int v = 0; v < VPL; ++v) m = fmaxf(m, l[v]);
  m = warp_max_f(m);
  float z[VPL];
  float zsum = 0.f;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int e = lane + 32 * v;
    z[v] = (e < E) ? expf(l[v] - m) : 0.f;
    zsum += z[v];
  }
  zsum = warp_sum_f(zsum);
  const float inv = 1.0f / zsum;
  if (probs != nullptr) {
    float* prow = probs + static_cast<int64_t>(t) * E;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int e = lane + 32 * v;
      if (e < E) prow[e] = z[v] * inv;
    }
  }
  float psel[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    psel[v] = 0.f;
    isel[v] = 0;
  }
  float psum = 0.f;
  if constexpr (VPL <= 8) {
    // Each lane sorts its VPL logits by (logit descending, expert ascending)
    // as order-preserving integer keys (-0.0 folded into +0.0 so signed
    // zeros tie); then k rounds of a warp-wide argmax over the lanes' heads:
    // the largest key, then the smallest expert among the lanes holding it.
    // The winning lane drops its head. A lane's equal keys stay in expert
    // order (only strictly larger keys move up), so the smallest expert of a
    // tie is always at the head of its lane.
    uint32_t key[VPL];
    int ev[VPL];
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int e = lane + 32 * v;
      const float cv = (l[v] == 0.0f) ? 0.0f : l[v];
      const uint32_t bits = __float_as_uint(cv);
      key[v] = (e < E) ? ((bits & 0x80000000u) ? ~bits : (bits | 0x80000000u)) : 0u;
      ev[v] = (e < E) ? e : 0x7fffffff;
    }
    // odd-even transposition sort, VPL rounds (swaps only on strictly larger keys: stable)
#pragma unroll
    for (int r = 0; r < VPL; ++r) {
#pragma unroll
      for (int v = (r & 1); v + 1 < VPL; v += 2) {
        const bool sw = key[v + 1] > key[v];
        const uint32_t ka = key[v], kb = key[v + 1];
        const int ea = ev[v], eb = ev[v + 1];
        key[v] = sw ? kb : ka;
        key[v + 1] = sw ? ka : kb;
        ev[v] = sw ? eb : ea;
        ev[v + 1] = sw ? ea : eb;
      }
    }
    if (k <= 32) {
      // lane j keeps the key and expert of round j's winner; the k winners'
      // probabilities are then computed at once, one per lane, exactly as
      // probs is (exp(l - m) / sum, the logit recovered from its key)
      uint32_t ksel = 0u;
      int esel = 0;
      for (int j = 0; j < k; ++j) {
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, key[0]);
        const int be = static_cast<int>(
            __reduce_min_sync(0xffffffffu, key[0] == kmax ? static_cast<uint32_t>(ev[0]) : 0xffffffffu));
        if ((be & 31) == lane) {  // the winner's lane drops its head
#pragma unroll
          for (int v = 0; v + 1 < VPL; ++v) {
            key[v] = key[v + 1];
            ev[v] = ev[v + 1];
          }
          key[VPL - 1] = 0u;
          ev[VPL - 1] = 0x7fffffff;
        }
        if (j == lane) {
          ksel = kmax;
          esel = be;
        }
      }
      float pj = 0.f;
      if (lane < k) {
        const uint32_t wb = (ksel & 0x80000000u) ? (ksel & 0x7fffffffu) : ~ksel;
        pj = expf(__uint_as_float(wb) - m) * inv;
      }
      psum = warp_sum_f(pj);
      psel[0] = pj;
      isel[0] = esel;
    } else {
      for (int j = 0; j < k; ++j) {
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, key[0]);
        const int be = static_cast<int>(
            __reduce_min_sync(0xffffffffu, key[0] == kmax ? static_cast<uint32_t>(ev[0]) : 0xffffffffu));
        if ((be & 31) == lane) {
#pragma unroll
          for (int v = 0; v + 1 < VPL; ++v) {
            key[v] = key[v + 1];
            ev[v] = ev[v + 1];
          }
          key[VPL - 1] = 0u;
          ev[VPL - 1] = 0x7fffffff;
        }
        const uint32_t wb = (kmax & 0x80000000u) ? (kmax & 0x7fffffffu) : ~kmax;
        const float pwin = expf(__uint_as_float(wb) - m) * inv;
        psum += pwin;
        if ((j & 31) == lane) {
          const int vj = j >> 5;
#pragma unroll
          for (int v = 0; v < VPL; ++v)
            if (v == vj) {
              psel[v] = pwin;
              isel[v] = be;
            }
        }
      }
    }
  } else {
    // k rounds of a warp-wide argmax over the not-yet-taken experts.
    uint32_t taken = 0;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int e = lane + 32 * v;
        const bool avail = (e < E) && !((taken >> v) & 1u);
        // within a lane e grows with v, so strict > keeps the lower index on ties
        if (avail && (l[v] > bv || be == 0x7fffffff)) {
          bv = l[v];
          be = e;
        }
      }
      // Warp argmax in two reductions: the largest logit (as an order-
      // preserving integer key; -0.0 is folded into +0.0 so signed zeros tie),
      // then the smallest expert index among the lanes holding it.
      const float cv = (bv == 0.0f) ? 0.0f : bv;
      const uint32_t bits = __float_as_uint(cv);
      const uint32_t key = (be == 0x7fffffff) ? 0u : ((bits & 0x80000000u) ? ~bits : (bits | 0x80000000u));
      const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
      be = static_cast<int>(__reduce_min_sync(0xffffffffu, key == kmax ? static_cast<uint32_t>(be) : 0xffffffffu));
      // owner lane marks the winner taken; every lane learns its probability
      float pwin = 0.f;
      if ((be & 31) == lane) {
        const int vw = be >> 5;
#pragma unroll
        for (int v = 0; v < VPL; ++v)
          if (v == vw) {
            taken |= 1u << v;
            pwin = z[v] * inv;
          }
      }
      pwin = __shfl_sync(0xffffffffu, pwin, be & 31);
      psum += pwin;
      if ((j & 31) == lane) {
        const int vj = j >> 5;
#pragma unroll
        for (int v = 0; v < VPL; ++v)
          if (v == vj) {
            psel[v] = pwin;
            isel[v] = be;
          }
      }
    }
  }
  const float denom = psum + 1e-20f;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int j = lane + 32 * v;
    if (j < k) {
      topk_idx[static_cast<int64_t>(t) * k + j] = isel[v];
      topk_w[static_cast<int64_t>(t) * k + j] = psel[v] / denom;
    }
  }
}

template <int VPL>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                    int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                                    float* __restrict__ probs, const float* __restrict__ part,
                                                    int n_part, int part_ld, int64_t part_stride,
                                                    float* __restrict__ logits_out) {
  griddep_wait();
  griddep_launch_dependents();
  const int warps_per_block = blockDim.x >> 5;
  for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < T; t += gridDim.x * warps_per_block) {
    int isel[VPL];
    route_token<VPL>(logits, t, E, k, topk_idx, topk_w, probs, part, n_part, part_ld, part_stride, logits_out,
                     isel);
  }
}

// Routing fused with the first pass of the permutation: block b routes the
// kRouteChunkTokens tokens [b * 32, b * 32 + 32) (two per warp, in order) and
// writes how many of their pairs chose each expert to hist8[b * ld + e]
// (bytes: a chunk holds at most 32 pairs of one expert, since a token's top-k
// experts are distinct; entries e in [E, ld) are written as 0). Each warp
// counts into its own byte row in shared memory; within one token the lanes
// holding its k experts touch distinct bytes, so no atomics are needed.
constexpr int kRouteChunkTokens = 32;
constexpr int kRouteHistWarps = 16;
// Up to 128 experts (VPL <= 4) the kernel is held to 32 registers, so four
// blocks fit an SM: the grid of a 16384-token batch is resident at once
// (measured per routing front-end call: 14.5 against 15.7 us at T 8192,
// 22.9 against 23.3 us at T 16384, E 128).
constexpr int route_hist_min_blocks(int vpl) { return vpl <= 4 ? 4 : 1; }

template <int VPL>
__global__ void __launch_bounds__(32 * kRouteHistWarps, route_hist_min_blocks(VPL)) route_hist_kernel(
    const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w, float* __restrict__ probs, uint8_t* __restrict__ hist8, int ld) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ __align__(16) uint8_t s_rows[];  // [kRouteHistWarps][ld]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kPerWarp = kRouteChunkTokens / kRouteHistWarps;
  uint8_t* row = s_rows + warp * ld;
  for (int i = lane; i < ld / 4; i += 32) reinterpret_cast<uint32_t*>(row)[i] = 0u;
  __syncwarp();
  const int t0 = blockIdx.x * kRouteChunkTokens + warp * kPerWarp;
  for (int i = 0; i < kPerWarp; ++i) {
    const int t = t0 + i;
    if (t >= T) break;
    int isel[VPL];
    route_token<VPL>(logits, t, E, k, topk_idx, topk_w, probs, nullptr, 0, 0, 0, nullptr, isel);
#pragma unroll
    for (int v = 0; v < VPL; ++v)
      if (lane + 32 * v < k) row[isel[v]] += 1;
    __syncwarp();
  }
  __syncthreads();
  for (int e = threadIdx.x; e < ld; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kRouteHistWarps; ++w) c += s_rows[w * ld + e];
    hist8[static_cast<int64_t>(blockIdx.x) * ld + e] = static_cast<uint8_t>(c);
  }
}

inline int route_hist_ld(int E) { return (E + 15) / 16 * 16; }
inline int route_hist_chunks(int T) { return (T + kRouteChunkTokens - 1) / kRouteChunkTokens; }

inline cudaError_t launch_route_hist(const float* logits, int T, int E, int k, int32_t* idx, float* w, float* probs,
                                     uint8_t* hist8, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int blocks = route_hist_chunks(T);
  const int ld = route_hist_ld(E);
  const size_t smem = static_cast<size_t>(kRouteHistWarps) * ld;  // <= 16 KB (E <= 1024)
  const int vpl = (E + 31) / 32;
#define MOE_ROUTE_HIST_CASE(V)                                                                              \
  if (vpl <= V) {                                                                                           \
    return launch_pdl(route_hist_kernel<V>, dim3(blocks), dim3(32 * kRouteHistWarps), smem, s, logits, T, E, k, \
                      idx, w, probs, hist8, ld);                                                            \
  }
  MOE_ROUTE_HIST_CASE(1)
  MOE_ROUTE_HIST_CASE(2)
  MOE_ROUTE_HIST_CASE(4)
  MOE_ROUTE_HIST_CASE(8)
  MOE_ROUTE_HIST_CASE(16)
  MOE_ROUTE_HIST_CASE(32)
#undef MOE_ROUTE_HIST_CASE
  return cudaErrorInvalidValue;
}

// One-pass launch: picks the register width from E.
inline cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* idx, float* w, float* probs,
                                cudaStream_t s, const float* part = nullptr, int n_part = 0, int part_ld = 0,
                                int64_t part_stride = 0, float* logits_out = nullptr) {
  if (T == 0) return cudaSuccess;
  const int threads = 256;
  const int warps = threads / 32;
  int blocks = (T + warps - 1) / warps;
  if (blocks > 148 * 32) blocks = 148 * 32;
  const int vpl = (E + 31) / 32;
#define MOE_ROUTE_CASE(V)                                                                    \
  if (vpl <= V) {                                                                            \
    return launch_pdl(route_kernel<V>, dim3(blocks), dim3(threads), 0, s, logits, T, E, k, idx, w, probs, part, \
                      n_part, part_ld, part_stride, logits_out);                                                \
  }
  MOE_ROUTE_CASE(1)
  MOE_ROUTE_CASE(2)
  MOE_ROUTE_CASE(4)
  MOE_ROUTE_CASE(8)
  MOE_ROUTE_CASE(16)
  MOE_ROUTE_CASE(32)
#undef MOE_ROUTE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace moe
