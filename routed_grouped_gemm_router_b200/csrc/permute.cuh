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

namespace moe {

// Scan and scatter in one kernel, from the per-chunk expert counts written by
// the routing kernel (route_hist_kernel: chunk c = tokens [32 c, 32 c + 32),
// hist8[c * ld + e] = its pairs of expert e, ld >= E). Block b owns the 8
// chunks [8 b, 8 b + 8), one per warp (small blocks, so that the pairs'
// scattered stores spread over many SMs). Every block sums the whole count
// table itself (a few tens of KB from L2), so no block waits on another:
//   total[e]  = sum over all chunks          -> counts, offsets (block 0 writes them)
//   before[e] = sum over the chunks before b's first
// Warp w's first row for expert e is then offsets[e] + before[e] + the counts
// of the block's chunks before w, and the warp places its chunk's pairs in
// ascending pair order, so each expert's rows keep ascending pair ids: the
// stable argsort of the flat ids. The ids must come from routing (each token's k
// experts distinct), as in moe_route_permute. Block width, measured with the
// routing kernel before it: 4 warps is much slower (each block sums the whole
// table with fewer threads); 16 warps take a whole SM's registers, so its
// blocks cannot start beside the routing kernel's and end no sooner.
constexpr int kScanScatterWarps = 8;
constexpr int kScanScatterThreads = 32 * kScanScatterWarps;

__global__ void __launch_bounds__(kScanScatterThreads) permute_scan_scatter_kernel(
    const uint8_t* __restrict__ hist8, int ld, int nchunks, const int32_t* __restrict__ flat, int T, int E, int k,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ sorted_pair,
    int32_t* __restrict__ pair_pos) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ int s_mem[];
  int* s_run = s_mem;                                     // [warps][E] running first rows
  int* s_tot = s_run + kScanScatterWarps * E;             // [groups][ld] partial totals
  int* s_pre = s_tot + 4 * kScanScatterThreads;           // [groups][ld] partial prefixes
  __shared__ int s_warp[kScanScatterWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c0 = blockIdx.x * kScanScatterWarps;
  const int words = ld / 4;                               // ld is a multiple of 16, at most 1024
  const int groups = kScanScatterThreads / words;         // >= 1
  // the ids this warp places in step 4 (k <= 32: lane j < k holds slot j of
  // each of its chunk's 32 tokens), requested first: they depend on nothing
  // computed here, so their latency overlaps the count-table sum
  const int c = c0 + warp;
  const int tc0 = c * 32;
  const int tc1 = (tc0 + 32 < T) ? tc0 + 32 : T;
  int ids[32];
#pragma unroll
  for (int i = 0; i < 32; ++i)
    ids[i] = (k <= 32 && lane < k && tc0 + i < tc1) ? __ldg(flat + static_cast<int64_t>(tc0 + i) * k + lane) : 0;

  // 1. per expert: total over all chunks and the prefix before this block.
  // Thread (word wi, group g) reads 4 experts' bytes of chunks g, g + groups,
  // ..., summed two at a time in 16-bit fields (even bytes, odd bytes). A
  // field takes at most 1024 counts of at most 32 (32768 < 2^16) before it
  // is folded into a 32-bit sum, so it never overflows.
  {
    const int wi = tid % words, g = tid / words;
    if (g < groups) {
      int tot[4] = {0, 0, 0, 0}, pre[4] = {0, 0, 0, 0};
      for (int cs = g; cs < nchunks; cs += 1024 * groups) {
        const int ce = (cs + 1024 * groups < nchunks) ? cs + 1024 * groups : nchunks;
        uint32_t tot_e = 0, tot_o = 0, pre_e = 0, pre_o = 0;
        constexpr int kU = 16;
        for (int cb = cs; cb < ce; cb += kU * groups) {
          uint32_t v[kU];
#pragma unroll
          for (int i = 0; i < kU; ++i) {
            const int c = cb + i * groups;
            v[i] = (c < ce) ? __ldg(reinterpret_cast<const uint32_t*>(hist8 + static_cast<int64_t>(c) * ld) + wi)
                            : 0u;
          }
#pragma unroll
          for (int i = 0; i < kU; ++i) {
            const uint32_t ev = v[i] & 0x00ff00ffu, od = (v[i] >> 8) & 0x00ff00ffu;
            tot_e += ev;
            tot_o += od;
            if (cb + i * groups < c0) {
              pre_e += ev;
              pre_o += od;
            }
          }
        }
        tot[0] += tot_e & 0xffffu, tot[1] += tot_o & 0xffffu, tot[2] += tot_e >> 16, tot[3] += tot_o >> 16;
        pre[0] += pre_e & 0xffffu, pre[1] += pre_o & 0xffffu, pre[2] += pre_e >> 16, pre[3] += pre_o >> 16;
      }
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        s_tot[g * ld + 4 * wi + b] = tot[b];
        s_pre[g * ld + 4 * wi + b] = pre[b];
      }
    }
  }
  // 3a. this block's chunk counts of the thread's four experts, requested now
  uint32_t own[kScanScatterWarps];
  if (tid < words) {
#pragma unroll
    for (int w = 0; w < kScanScatterWarps; ++w) {
      const int c = c0 + w;
      own[w] = (c < nchunks) ? __ldg(reinterpret_cast<const uint32_t*>(hist8 + static_cast<int64_t>(c) * ld) + tid)
                             : 0u;
    }
  }
  __syncthreads();
  // thread t owns experts 4t .. 4t + 3 (those >= E count zero)
  int tot[4] = {0, 0, 0, 0}, pre[4] = {0, 0, 0, 0};
  if (tid < words) {
    for (int g = 0; g < groups; ++g)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        tot[b] += s_tot[g * ld + 4 * tid + b];
        pre[b] += s_pre[g * ld + 4 * tid + b];
      }
  }
  // 2. exclusive scan of the totals over experts
  const int mine = tot[0] + tot[1] + tot[2] + tot[3];
  const int incl = warp_inclusive_scan(mine);
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = (lane < kScanScatterWarps) ? s_warp[lane] : 0;
    const int sc = warp_inclusive_scan(v) - v;
    if (lane < kScanScatterWarps) s_warp[lane] = sc;
  }
  __syncthreads();
  if (tid < words) {
    int off = s_warp[warp] + incl - mine;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int e = 4 * tid + b;
      if (e < E) {
        if (blockIdx.x == 0) {
          counts[e] = tot[b];
          offsets[e] = off;
          if (e == E - 1) offsets[E] = off + tot[b];
        }
        // 3b. each warp's first rows: the block's chunks in order
        int run = off + pre[b];
#pragma unroll
        for (int w = 0; w < kScanScatterWarps; ++w) {
          s_run[w * E + e] = run;
          run += (own[w] >> (8 * b)) & 0xff;
        }
      }
      off += tot[b];
    }
  }
  __syncthreads();
  // 4. warp w places the pairs of chunk c0 + w token by token, in pair
  // order. The ids come from the routing kernel, so a token's k experts are
  // distinct: the lanes holding them bump distinct running counters, and
  // only consecutive tokens are ordered (by __syncwarp).
  if (c >= nchunks) return;
  int* run_w = s_run + warp * E;
  const int64_t P = static_cast<int64_t>(T) * k;
  auto place = [&](int64_t q, int e) {
    if (e < 0 || e >= E) {
      report(MOE_ERR_DEVICE_CHECK);
      return;
    }
    const int pos = run_w[e];
    run_w[e] = pos + 1;
    if (pos < P) {  // counts that disagree with the ids: never written out of range
      sorted_pair[pos] = static_cast<int32_t>(q);
      pair_pos[q] = pos;
    } else {
      report(MOE_ERR_DEVICE_CHECK);
    }
  };
  if (k <= 32) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (tc0 + i >= tc1) break;
      if (lane < k) place(static_cast<int64_t>(tc0 + i) * k + lane, ids[i]);
      __syncwarp();
    }
  } else {  // wide top-k: a token's slots in groups of 32, tokens in order
    for (int t = tc0; t < tc1; ++t) {
      for (int jb = 0; jb < k; jb += 32) {
        const int j = jb + lane;
        if (j < k) place(static_cast<int64_t>(t) * k + j, __ldg(flat + static_cast<int64_t>(t) * k + j));
        __syncwarp();
      }
    }
  }
}

inline size_t scan_scatter_smem(int E) {
  return sizeof(int) * (static_cast<size_t>(kScanScatterWarps) * E + 8 * kScanScatterThreads);
}

}  // namespace moe
