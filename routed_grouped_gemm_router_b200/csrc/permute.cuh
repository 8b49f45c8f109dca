// K-PM: expert histogram -> prefix sum -> stable scatter, and the row gather.
//
// "[MoE] Improve moe kernels for unsloth fine tuning #3812", review of the
// token-routing logic: the counts are bincount(flat ids, minlength=E) and the
// gather order is the stable argsort of the flat ids. The result here is
// bit-identical to those definitions, computed without atomics:
//
//  1. count   : the P pair ids are cut into chunks of kChunk; inside a block
//               each warp owns a contiguous slice and counts it 32 ids at a
//               time with __match_any_sync (one leader lane per distinct
//               expert updates the warp's private histogram, so no two lanes
//               ever write the same counter).
//  2. scan    : one block turns the chunk histograms into, per (chunk,
//               expert), the first output row of that chunk's pairs of that
//               expert, and writes counts and offsets.
//  3. scatter : each block recounts its chunk, derives per-warp bases and
//               writes every pair at base + (rank among equal ids before it),
//               so pairs of one expert keep ascending pair-id order.
//  4. gather  : Xp[pair_pos[q]] = X[q / k] in pair order, 16-byte vectors.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kPermThreads = 256;
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kPermIters = 8;                              // 32-id steps per warp
constexpr int kChunk = kPermWarps * 32 * kPermIters;       // 2048 pairs per block

__host__ __device__ inline int perm_num_chunks(int64_t P) { return static_cast<int>((P + kChunk - 1) / kChunk); }

// Counts the warp's slice into hist_w[E] (shared, zeroed by the caller).
__device__ __forceinline__ void warp_count_slice(const int32_t* __restrict__ flat, int64_t P, int E,
                                                 int64_t slice_begin, int* hist_w) {
  const int lane = threadIdx.x & 31;
  for (int it = 0; it < kPermIters; ++it) {
    const int64_t q = slice_begin + it * 32 + lane;
    int e = -1;
    if (q < P) {
      e = flat[q];
      if (e < 0 || e >= E) {
        report(MOE_ERR_DEVICE_CHECK);
        e = -1;
      }
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    if (e >= 0 && lane == leader) hist_w[e] += __popc(peers);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kPermThreads) permute_count_kernel(const int32_t* __restrict__ flat, int64_t P,
                                                                     int E, int* __restrict__ chunk_hist) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ int s_hist[];  // [kPermWarps][E]
  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) s_hist[i] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kChunk + warp * 32 * kPermIters;
  warp_count_slice(flat, P, E, base, s_hist + warp * E);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
#pragma unroll
    for (int w = 0; w < kPermWarps; ++w) s += s_hist[w * E + e];
    chunk_hist[static_cast<int64_t>(blockIdx.x) * E + e] = s;
  }
}

// One block of 1024 threads; thread e owns expert e (E <= 1024). Leaves in
// chunk_hist[c][e] the number of expert-e pairs in chunks before c; the
// scatter adds offsets[e] to it.
__global__ void __launch_bounds__(1024) permute_scan_kernel(int* __restrict__ chunk_hist, int nchunks, int E,
                                                            int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ int s_warp[32];
  const int e = threadIdx.x;
  int total = 0;
  if (e < E) {
    constexpr int B = 16;  // independent loads in flight per thread
    for (int c0 = 0; c0 < nchunks; c0 += B) {
      int v[B];
#pragma unroll
      for (int i = 0; i < B; ++i) v[i] = (c0 + i < nchunks) ? chunk_hist[static_cast<int64_t>(c0 + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < B; ++i) {
        if (c0 + i < nchunks) chunk_hist[static_cast<int64_t>(c0 + i) * E + e] = total;
        total += v[i];
      }
    }
    counts[e] = total;
  }
  // exclusive scan of the totals over experts
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int incl = warp_inclusive_scan(total);
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = s_warp[lane];
    const int sc = warp_inclusive_scan(v);
    s_warp[lane] = sc - v;
  }
  __syncthreads();
  const int excl = s_warp[warp] + incl - total;
  if (e < E) offsets[e] = excl;
  if (e == E - 1) offsets[E] = excl + total;
}

__global__ void __launch_bounds__(kPermThreads) permute_scatter_kernel(const int32_t* __restrict__ flat, int64_t P,
                                                                       int E, const int* __restrict__ chunk_base,
                                                                       const int32_t* __restrict__ offsets,
                                                                       int32_t* __restrict__ sorted_pair,
                                                                       int32_t* __restrict__ pair_pos) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ int s_hist[];  // [kPermWarps][E] -> per-warp running bases
  for (int i = threadIdx.x; i < kPermWarps * E; i += blockDim.x) s_hist[i] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kChunk + warp * 32 * kPermIters;
  warp_count_slice(flat, P, E, base, s_hist + warp * E);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = chunk_base[static_cast<int64_t>(blockIdx.x) * E + e] + offsets[e];
#pragma unroll
    for (int w = 0; w < kPermWarps; ++w) {
      const int c = s_hist[w * E + e];
      s_hist[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  int* run_w = s_hist + warp * E;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int it = 0; it < kPermIters; ++it) {
    const int64_t q = base + it * 32 + lane;
    int e = -1;
    if (q < P) {
      e = flat[q];
      if (e < 0 || e >= E) e = -1;  // already reported by the count pass
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int pos = 0;
    if (e >= 0) pos = run_w[e] + __popc(peers & lt_mask);
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) run_w[e] += __popc(peers);
    __syncwarp();
    if (e >= 0) {
      sorted_pair[pos] = static_cast<int32_t>(q);
      pair_pos[q] = pos;
    }
  }
}

// Xp[pair_pos[q], :] = X[q / k, :] for every pair q: the rows are visited in
// pair order, so the k copies of a token row are made by consecutive warps
// while the row is in L1/L2 and every row of X is read from DRAM once even
// when X is larger than L2. One warp per pair, 16-byte vectors, four loads in
// flight per lane. Pairs whose row is out of range (only possible after an
// invalid expert id was reported) are skipped.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ X,
                                                          const int32_t* __restrict__ pair_pos, int64_t P,
                                                          int k, int vec_per_row, uint4* __restrict__ Xp) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); q < P; q += warps) {
    const int32_t r = pair_pos[q];
    if (r < 0 || r >= P) continue;
    const uint4* src = X + (q / k) * vec_per_row;
    uint4* dst = Xp + static_cast<int64_t>(r) * vec_per_row;
    for (int c0 = 0; c0 < vec_per_row; c0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = c0 + 32 * i + lane;
        if (c < vec_per_row) v[i] = __ldg(src + c);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = c0 + 32 * i + lane;
        if (c < vec_per_row) dst[c] = v[i];
      }
    }
  }
}

}  // namespace moe
