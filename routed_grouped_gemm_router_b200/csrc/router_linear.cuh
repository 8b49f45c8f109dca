// Router Linear on the tensor cores: logits = X W_r^T (forward), and its
// backward dW_r = dlogits^T X and dX += dlogits W_r.
//
// The router is a Linear(H -> E) with weight W_r [E, H] ("Integration of
// fused moe kernel (e.g., megablocks) for efficient moe training", axolotl
// issue #3155, discussion of the router's weight shape) and runs in fp32.
// X is bf16; W_r and dlogits are fp32. Every fp32 value v splits exactly into
// three bf16 terms, v = v0 + v1 + v2 with v0 = bf16(v), v1 = bf16(v - v0),
// v2 = v - v0 - v1 (8 + 8 + 8 significant bits cover fp32's 24), so
//   X W_r^T        = sum_s X W_s^T                    (3 bf16 products, exact)
//   dlogits^T X    = sum_s dl_s^T X                   (3 bf16 products, exact)
//   dlogits W_r   ~= dl0 W0 + dl0 W1 + dl1 W0          (relative error ~2^-16,
//                                                       128x below the bf16
//                                                       rounding of dX)
// and each sum runs as one GEMM whose K loop walks the terms one after the
// other into a single fp32 accumulator in TMEM.
//
// All three are skinny (one dimension is E <= 1024, or the K extent is E), so
// the kernel is a one-CTA tcgen05 GEMM (M = 128 rows per tile) with split-K:
// unit = (M tile, N tile, K range); the fp32 partial sums of the splits are
// added in a fixed order by the consumer (the routing kernel for the logits,
// a summing kernel for dW_r), so results do not depend on scheduling.
//
// Roles: warp 0 issues the TMA loads, warp 1 allocates TMEM and issues the
// MMAs, warps 2..5 read the accumulator (warp w owns TMEM lanes 32*(w%4)..).
#pragma once
#include "common.cuh"

namespace moe {

enum RouterGemmKind : int {
  kRgLogits = 0,  // out[split][t][e]   = sum_k X[t,k] W3[term*E + e, k]           (fp32 partials)
  kRgWgrad = 1,   // out[split][e][h]   = sum_t dl3[term*T + t, e] X[t, h]        (fp32 partials of dW_r)
  kRgDgrad = 2,   // dX[t][h] += sum_e dl3[a*T + t, e] W3[b*E + e, h], (a,b) pairs (bf16 in/out)
  // logits as kRgLogits, K split over the two CTAs of a cluster; the odd CTA
  // adds its partial into the even CTA's shared memory, which then routes
  // (softmax, top-k, renormalisation) in the epilogue (E <= 128, k <= KMAX)
  kRgLogitsRoute = 3,
};

constexpr int kRgBM = 128;
constexpr int kRgBK = 64;
constexpr int kRgMaxStages = 4;
constexpr int kRgThreads = 192;
constexpr int kRgATileBytes = kRgBM * kRgBK * 2;  // 16 KiB
constexpr int kRgStageWarpBytes = 32 * 128;       // 32 rows x 32 fp32 per epilogue warp
constexpr int kRgMaxSplitsLogits = 8;  // the routing kernel sums at most 8 partials
constexpr int kRgMaxSplitsWgrad = 32;
constexpr int kRgDgradBN = 128;  // N tile of the dX part (its epilogue prefetch is sized for it)

// (term of A, term of B) of the three products kept in the dX part.
__host__ __device__ constexpr int rg_dgrad_term_a(int j) { return j == 2 ? 1 : 0; }
__host__ __device__ constexpr int rg_dgrad_term_b(int j) { return j == 1 ? 1 : 0; }

struct RouterGemmParams {
  CUtensorMap tmA;
  CUtensorMap tmB;
  int M, N;          // output rows and columns
  int term_rows_a;   // rows between the terms of A's tensor (0 when A has one term)
  int term_rows_b;   // rows between the terms of B's tensor
  int nkb;           // 64-wide K blocks per term
  int n_terms;       // the K loop runs over n_terms * nkb blocks
  int splits;        // split-K parts
  int m_tiles, n_tiles;
  int bn;            // N tile (columns); multiple of 16 (K-major B) or 64 (MN-major B), <= 256
  int stages;        // ring depth, <= kRgMaxStages
  float* out;        // fp32 partials (logits, wgrad)
  int out_ld;        // row stride of `out` in floats
  int64_t out_split_stride;
  uint16_t* dx;      // bf16 in/out (dgrad)
  int dx_ld;
  // kRgLogitsRoute outputs (logits and probs may be null)
  int k;
  int32_t* topk_idx;
  float* topk_w;
  float* probs;
  float* logits;
};

// Fused routing: row stride (in floats) of the [E][128] logits buffer in
// shared memory; 129 keeps both row-wise and column-wise accesses free of
// bank conflicts.
constexpr int kRgLgStride = 129;
constexpr int kRgRouteMaxE = 128;

__host__ __device__ inline int rg_b_tile_bytes(int bn) { return bn * kRgBK * 2; }
__host__ __device__ inline int rg_tmem_cols(int bn) {
  int c = 32;
  while (c < bn) c <<= 1;
  return c;
}
// The epilogue's staging blocks (4 warps x 4 KiB) reuse stage 0's A tile: a
// CTA computes one tile, so every load and MMA is finished when its epilogue
// starts.
inline size_t rg_smem_bytes(int bn, int stages, int lg_rows = 0) {
  return 1024 /* alignment slack */ + static_cast<size_t>(stages) * (kRgATileBytes + rg_b_tile_bytes(bn)) +
         256 /* barriers, TMEM slot, flags */ + static_cast<size_t>(lg_rows) * kRgLgStride * 4;
}
static_assert(4 * kRgStageWarpBytes <= kRgATileBytes, "epilogue staging must fit in one A tile");

// Epilogue staging of one 32 x 32 fp32 block per warp: row r's 16-byte
// piece p lives at r*128 + 16*(p ^ (r & 7)), which keeps both the row-domain
// writes (lane = row) and the transposed reads (a quarter-warp per row)
// at four shared-memory wavefronts per instruction.
__device__ __forceinline__ void rg_stage_row(uint8_t* stg, int r, const uint32_t (&v)[32]) {
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    uint4 x = make_uint4(v[4 * p], v[4 * p + 1], v[4 * p + 2], v[4 * p + 3]);
    *reinterpret_cast<uint4*>(stg + r * 128 + 16 * (p ^ (r & 7))) = x;
  }
}
__device__ __forceinline__ void rg_read8(const uint8_t* stg, int r, int q, float (&f)[8]) {
  const uint4 a = *reinterpret_cast<const uint4*>(stg + r * 128 + 16 * ((2 * q) ^ (r & 7)));
  const uint4 b = *reinterpret_cast<const uint4*>(stg + r * 128 + 16 * ((2 * q + 1) ^ (r & 7)));
  f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y); f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
  f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y); f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
}

// Every lane polls; the warp proceeds together (false: the wait limit passed).
__device__ __forceinline__ bool rg_warp_wait(uint64_t* bar, uint32_t parity) {
  const bool ok = mbar_wait(bar, parity);
  return __all_sync(0xffffffffu, ok);
}

template <int KIND, int KMAX = 1>
__global__ void __launch_bounds__(kRgThreads, 1) router_gemm_kernel(const __grid_constant__ RouterGemmParams p) {
  constexpr bool kRoute = (KIND == kRgLogitsRoute);
  constexpr bool kAMN = (KIND == kRgWgrad);  // A = X^T: M (hidden) contiguous
  constexpr bool kBMN = (KIND == kRgWgrad || KIND == kRgDgrad);  // B = dl3 (wgrad) or W3 (dgrad): N contiguous
  constexpr uint32_t kALbo = kAMN ? 8192u : 16u;
  constexpr uint32_t kBLbo = kBMN ? 8192u : 16u;
  constexpr uint32_t kAStep = kAMN ? 2048u : 32u;  // bytes per 16-deep K step
  constexpr uint32_t kBStep = kBMN ? 2048u : 32u;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int bn = p.bn;
  const int stages = p.stages;
  const int b_bytes = rg_b_tile_bytes(bn);
  uint8_t* sA = smem;
  uint8_t* sB = smem + stages * kRgATileBytes;
  uint8_t* s_stage = sA;  // epilogue staging, used only after the last MMA completed
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + stages * b_bytes);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + kRgMaxStages;
  uint64_t* tfull_bar = bars + 2 * kRgMaxStages;
  uint64_t* drain_bar = bars + 2 * kRgMaxStages + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * kRgMaxStages + 2);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  float* s_lg = reinterpret_cast<float*>(s_tmem + 16);  // kRgLogitsRoute: logits [E][kRgLgStride]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t tmem_cols = static_cast<uint32_t>(rg_tmem_cols(bn));

  // unit -> (M tile, N tile, K range); the splits of one output tile are
  // adjacent (for kRgLogitsRoute they are the two CTAs of a cluster)
  const int unit = blockIdx.x;
  const uint32_t crank = kRoute ? cluster_ctarank() : 0u;
  const int split = kRoute ? static_cast<int>(crank) : unit % p.splits;
  const int n_blk = kRoute ? 0 : (unit / p.splits) % p.n_tiles;
  const int m_blk = kRoute ? (unit >> 1) : unit / (p.splits * p.n_tiles);
  const int m0 = m_blk * kRgBM;
  const int n0 = n_blk * bn;
  const int64_t G = static_cast<int64_t>(p.n_terms) * p.nkb;
  const int g0 = static_cast<int>(G * split / p.splits);
  const int g1 = static_cast<int>(G * (split + 1) / p.splits);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, tmem_cols);
    tmem_relinquish();
  }
  griddep_wait();
  griddep_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int g = g0; g < g1 && !*s_abort; ++g) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) {
          report(MOE_ERR_TIMEOUT);
          *s_abort = 1;
          break;
        }
        const int term = g / p.nkb;
        const int kx = (g - term * p.nkb) * kRgBK;
        uint64_t* fb = &full_bar[stage];
        uint8_t* a_dst = sA + stage * kRgATileBytes;
        uint8_t* b_dst = sB + stage * b_bytes;
        mbar_arrive_expect_tx(fb, static_cast<uint32_t>(kRgATileBytes + b_bytes));
        if constexpr (KIND == kRgLogits || kRoute) {
          tma_load_2d(a_dst, &p.tmA, fb, kx, m0);
          tma_load_2d(b_dst, &p.tmB, fb, kx, term * p.term_rows_b + n0);
        } else if constexpr (KIND == kRgWgrad) {
          tma_load_2d(a_dst, &p.tmA, fb, m0, kx);
          tma_load_2d(a_dst + 8192, &p.tmA, fb, m0 + 64, kx);
          for (int c = 0; c < bn / 64; ++c)
            tma_load_2d(b_dst + 8192 * c, &p.tmB, fb, n0 + 64 * c, term * p.term_rows_b + kx);
        } else {
          tma_load_2d(a_dst, &p.tmA, fb, kx, rg_dgrad_term_a(term) * p.term_rows_a + m0);
          for (int c = 0; c < bn / 64; ++c)
            tma_load_2d(b_dst + 8192 * c, &p.tmB, fb, n0 + 64 * c, rg_dgrad_term_b(term) * p.term_rows_b + kx);
        }
        ++issued;
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // no load may still be landing in shared memory when the CTA leaves
      const int inflight = issued < stages ? issued : stages;
      for (int i = 0; i < inflight; ++i) {
        if (--stage < 0) {
          stage = stages - 1;
          phase ^= 1u;
        }
        mbar_wait(&full_bar[stage], phase);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kRgBM, bn, kAMN, kBMN);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int g = g0; g < g1 && !*s_abort; ++g) {
      if (!rg_warp_wait(&full_bar[stage], phase)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a_addr = smem_u32(sA + stage * kRgATileBytes);
        const uint32_t b_addr = smem_u32(sB + stage * b_bytes);
#pragma unroll
        for (int kk = 0; kk < kRgBK / 16; ++kk) {
          const uint64_t adesc = sdesc_sw128(a_addr + kk * kAStep, kALbo, 1024);
          const uint64_t bdesc = sdesc_sw128(b_addr + kk * kBStep, kBLbo, 1024);
          umma_bf16(tmem_base, adesc, bdesc, idesc, (g > g0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty_bar[stage]);
      }
      __syncwarp();
      if (++stage == stages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) {
      if (lane == 0) report(MOE_ERR_TIMEOUT);
      *s_abort = 1;
    }
    // the accumulator is complete (or abandoned) once every MMA above is done
    if (lane == 0) {
      umma_commit(tfull_bar);
      umma_commit(drain_bar);
    }
    __syncwarp();
    rg_warp_wait(drain_bar, 0);
  } else {
    // ------------------------------------------------------------ epilogue
    // Thread (warp w, lane l) owns accumulator row 32*(w%4) + l ("row
    // domain"). Logits and dX go through the warp's staging block and are
    // written from the transposed domain (lane l: rows 8i + l/4, columns
    // 8*(l%4)..+7 of the 32-column chunk), so each quarter-warp touches one
    // row's contiguous bytes. dW_r is written transposed straight from the
    // row domain: for a fixed column the 32 lanes cover 32 consecutive floats.
    const int sub = warp & 3;
    uint8_t* stg = s_stage + (warp - 2) * kRgStageWarpBytes;
    const int tr_row = lane >> 2;
    const int tr_q = lane & 3;
    // dX: the incoming values of this warp's rows are requested before the
    // wait, so their DRAM latency overlaps the main loop
    constexpr int kDxChunks = KIND == kRgDgrad ? kRgDgradBN / 32 : 1;
    uint4 dxv[kDxChunks][4];
    if constexpr (KIND == kRgDgrad) {
#pragma unroll
      for (int ch = 0; ch < kDxChunks; ++ch)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = m0 + sub * 32 + i * 8 + tr_row;
          const int col = n0 + ch * 32 + tr_q * 8;
          dxv[ch][i] = (row < p.M && col < p.N)
                           ? *reinterpret_cast<const uint4*>(p.dx + static_cast<int64_t>(row) * p.dx_ld + col)
                           : make_uint4(0, 0, 0, 0);
        }
    }
    const bool ok = rg_warp_wait(tfull_bar, 0);
    if (!ok) {
      if (lane == 0) report(MOE_ERR_TIMEOUT);
      *s_abort = 1;
    }
    tc_fence_after();
    if (kRoute && ok && !*s_abort && crank == 1) {
      // odd CTA of the cluster: its fp32 partial goes into the even CTA's
      // logits buffer (element [e][row]; lanes write consecutive rows)
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(sub * 32) << 16);
      const uint32_t peer_lg = mapa_shared(smem_u32(s_lg), 0);
      const int r = sub * 32 + lane;
#pragma unroll 1
      for (int ch = 0; ch < (bn + 31) / 32; ++ch) {
        if (ch * 32 >= p.N) break;
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + ch * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int e = ch * 32 + j;
          if (e < p.N) st_shared_cluster_f32(peer_lg + static_cast<uint32_t>(e * kRgLgStride + r) * 4u, __uint_as_float(v[j]));
        }
      }
    } else if (kRoute) {
      // even CTA: routes after the cluster barrier below
    } else if (ok && !*s_abort && KIND == kRgDgrad) {
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(sub * 32) << 16);
      const int row0 = m0 + sub * 32;
#pragma unroll
      for (int ch = 0; ch < kDxChunks; ++ch) {
        const int col0 = n0 + ch * 32;
        if (col0 < p.N) {  // warp-uniform
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + ch * 32, v);
          tmem_ld_wait();
          rg_stage_row(stg, lane, v);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int row = row0 + i * 8 + tr_row;
            const int col = col0 + tr_q * 8;
            if (row < p.M && col < p.N) {  // N is a multiple of 8: bf16(dX + acc)
              float f[8];
              rg_read8(stg, i * 8 + tr_row, tr_q, f);
              const uint4 old = dxv[ch][i];
              uint4 o;
              o.x = pack_bf16(bf16lo(old.x) + f[0], bf16hi(old.x) + f[1]);
              o.y = pack_bf16(bf16lo(old.y) + f[2], bf16hi(old.y) + f[3]);
              o.z = pack_bf16(bf16lo(old.z) + f[4], bf16hi(old.z) + f[5]);
              o.w = pack_bf16(bf16lo(old.w) + f[6], bf16hi(old.w) + f[7]);
              *reinterpret_cast<uint4*>(p.dx + static_cast<int64_t>(row) * p.dx_ld + col) = o;
            }
          }
          __syncwarp();
        }
      }
    } else if (ok && !*s_abort) {
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(sub * 32) << 16);
      const int row0 = m0 + sub * 32;
#pragma unroll 1
      // TMEM holds rg_tmem_cols(bn) >= 32 * ceil(bn / 32) columns, so a chunk
      // may run past bn; columns >= N are never written
      for (int ch = 0; ch < (bn + 31) / 32; ++ch) {
        const int col0 = n0 + ch * 32;
        if (col0 >= p.N) break;  // warp-uniform
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + ch * 32, v);
        tmem_ld_wait();
        if constexpr (KIND == kRgWgrad) {
          const int h = row0 + lane;
          float* o = p.out + split * p.out_split_stride + h;
          if (h < p.M) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < p.N) o[static_cast<int64_t>(col0 + j) * p.out_ld] = __uint_as_float(v[j]);
          }
        } else {
          rg_stage_row(stg, lane, v);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int row = row0 + i * 8 + tr_row;
            const int col = col0 + tr_q * 8;
            if (row < p.M && col < p.N) {
              float f[8];
              rg_read8(stg, i * 8 + tr_row, tr_q, f);
              if constexpr (KIND == kRgLogits) {
                float* o = p.out + split * p.out_split_stride + static_cast<int64_t>(row) * p.out_ld + col;
                if (col + 8 <= p.N) {
                  reinterpret_cast<float4*>(o)[0] = make_float4(f[0], f[1], f[2], f[3]);
                  reinterpret_cast<float4*>(o)[1] = make_float4(f[4], f[5], f[6], f[7]);
                } else {
#pragma unroll
                  for (int j = 0; j < 8; ++j)
                    if (col + j < p.N) o[j] = f[j];
                }
              }
            }
          }
          __syncwarp();
        }
      }
    }
    tc_fence_before();
  }

  if constexpr (kRoute) {
    // ------------------------------------------ routing (even CTA of the pair)
    __syncthreads();
    __syncwarp();
    cluster_sync_all();  // the odd CTA's partial has landed in s_lg
    if (crank == 0 && warp >= 2 && !*s_abort) {
      const int sub = warp & 3;
      const int r = sub * 32 + lane;  // row of the tile owned by this thread
      const int t = m0 + r;
      const int E = p.N;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(sub * 32) << 16);
      tc_fence_after();
      // logits = (even CTA's partial) + (odd CTA's partial), fp32
#pragma unroll 1
      for (int ch = 0; ch < (bn + 31) / 32; ++ch) {
        if (ch * 32 >= E) break;
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + ch * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int e = ch * 32 + j;
          if (e < E) s_lg[e * kRgLgStride + r] = __uint_as_float(v[j]) + s_lg[e * kRgLgStride + r];
        }
      }
      __syncwarp();
      if (p.logits != nullptr) {  // the warp's 32 rows, coalesced
        for (int i = 0; i < 32; ++i) {
          const int row = sub * 32 + i;
          if (m0 + row >= p.M) break;
          for (int e = lane; e < E; e += 32)
            p.logits[static_cast<int64_t>(m0 + row) * E + e] = s_lg[e * kRgLgStride + row];
        }
      }
      // max and top-k (logit descending, lower expert index on ties: an
      // entry moves down only for a strictly larger value) in one pass, 8
      // logits at a time with independent maxima; then z = exp(l - max) and
      // its sum the same way (partial sums added in a fixed order)
      float inv = 0.0f;
      if (t < p.M) {
        float vl[KMAX];
        int il[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          vl[j] = -INFINITY;
          il[j] = -1;
        }
        float mx[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
        for (int e0 = 0; e0 < E; e0 += 8) {
          float lv[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) lv[u] = (e0 + u < E) ? s_lg[(e0 + u) * kRgLgStride + r] : -INFINITY;
#pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = fmaxf(mx[u], lv[u]);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (e0 + u < E && (lv[u] > vl[KMAX - 1] || il[KMAX - 1] < 0)) {
              float cv = lv[u];
              int ci = e0 + u;
#pragma unroll
              for (int j = 0; j < KMAX; ++j) {
                if (ci >= 0 && (il[j] < 0 || cv > vl[j])) {
                  const float tv = vl[j];
                  const int ti = il[j];
                  vl[j] = cv;
                  il[j] = ci;
                  cv = tv;
                  ci = ti;
                }
              }
            }
          }
        }
        const float m = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                              fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        float zs[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) zs[u] = 0.0f;
        for (int e0 = 0; e0 < E; e0 += 8) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (e0 + u < E) {
              const float z = expf(s_lg[(e0 + u) * kRgLgStride + r] - m);
              s_lg[(e0 + u) * kRgLgStride + r] = z;
              zs[u] += z;
            }
          }
        }
        const float zsum = ((zs[0] + zs[1]) + (zs[2] + zs[3])) + ((zs[4] + zs[5]) + (zs[6] + zs[7]));
        inv = 1.0f / zsum;
        float psum = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          if (j < p.k) {
            vl[j] = expf(vl[j] - m) * inv;
            psum += vl[j];
          }
        const float denom = psum + 1e-20f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          if (j < p.k) {
            p.topk_idx[static_cast<int64_t>(t) * p.k + j] = il[j];
            p.topk_w[static_cast<int64_t>(t) * p.k + j] = vl[j] / denom;
          }
      }
      __syncwarp();
      if (p.probs != nullptr) {  // p = z / sum z, the warp's 32 rows, coalesced
        for (int i = 0; i < 32; ++i) {
          const int row = sub * 32 + i;
          const float inv_i = __shfl_sync(0xffffffffu, inv, i);
          if (m0 + row >= p.M) break;
          for (int e = lane; e < E; e += 32)
            p.probs[static_cast<int64_t>(m0 + row) * E + e] = s_lg[e * kRgLgStride + row] * inv_i;
        }
      }
      tc_fence_before();
    }
  }

  // ------------------------------------------------------------ tear-down
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// Exact three-way bf16 split of an fp32 matrix src [rows, cols] (row stride
// src_ld): dst[(s * term_rows + r) * dst_ld + c] = term s of src[r][c].
__global__ void __launch_bounds__(256) split3_bf16_kernel(const float* __restrict__ src, int64_t rows, int cols,
                                                          int src_ld, int dst_ld, int64_t term_rows,
                                                          uint16_t* __restrict__ dst) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t n = rows * cols;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / cols;
    const int c = static_cast<int>(i - r * cols);
    const float v = src[r * src_ld + c];
    const __nv_bfloat16 v0 = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(v0);
    const __nv_bfloat16 v1 = __float2bfloat16_rn(r1);
    const __nv_bfloat16 v2 = __float2bfloat16_rn(r1 - __bfloat162float(v1));
    dst[r * dst_ld + c] = __bfloat16_as_ushort(v0);
    dst[(term_rows + r) * dst_ld + c] = __bfloat16_as_ushort(v1);
    dst[(2 * term_rows + r) * dst_ld + c] = __bfloat16_as_ushort(v2);
  }
}

// out[i] = sum over s = 0..S-1 (in that order) of part[s * stride + i]; n and
// stride multiples of 4.
__global__ void __launch_bounds__(256) sum_splits_kernel(const float* __restrict__ part, int S, int64_t n,
                                                         int64_t stride, float* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t n4 = n / 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 a = reinterpret_cast<const float4*>(part)[i];
    for (int s = 1; s < S; ++s) {
      const float4 b = reinterpret_cast<const float4*>(part + s * stride)[i];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    reinterpret_cast<float4*>(out)[i] = a;
  }
}

}  // namespace moe
