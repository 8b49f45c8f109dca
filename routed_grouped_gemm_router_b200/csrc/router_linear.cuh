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
// Persistent: CTA c takes units c, c + gridDim.x, ...; the load ring runs on
// across units and the accumulator is double-buffered in TMEM, so a unit's
// epilogue overlaps the next unit's loads and MMAs.
// Roles: warp 0 issues the TMA loads, warp 1 allocates TMEM and issues the
// MMAs, warps 2..5 read the accumulator (warp w owns TMEM lanes 32*(w%4)..).
#pragma once
#include "common.cuh"

namespace moe {

enum RouterGemmKind : int {
  kRgLogits = 0,  // out[split][t][e]   = sum_k X[t,k] W3[term*E + e, k]           (fp32 partials)
  kRgWgrad = 1,   // out[split][e][h]   = sum_t dl3[term*T + t, e] X[t, h]        (fp32 partials of dW_r)
  kRgDgrad = 2,   // dX[t][h] += sum_e dl3[a*T + t, e] W3[b*E + e, h], (a,b) pairs (bf16 in/out)
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
};

__host__ __device__ inline int rg_b_tile_bytes(int bn) { return bn * kRgBK * 2; }
__host__ __device__ inline int rg_tmem_cols(int bn) {
  int c = 32;
  while (c < bn) c <<= 1;
  return c;
}
// Shared memory: the ring, the epilogue's staging blocks (4 warps x 4 KiB;
// their own space, since the ring keeps running into the next unit), then
// barriers, the TMEM slot and a flag.
inline size_t rg_smem_bytes(int bn, int stages) {
  return 1024 /* alignment slack */ + static_cast<size_t>(stages) * (kRgATileBytes + rg_b_tile_bytes(bn)) +
         4 * kRgStageWarpBytes + 256 /* barriers, TMEM slot, flags */;
}

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

template <int KIND>
__global__ void __launch_bounds__(kRgThreads, 1) router_gemm_kernel(const __grid_constant__ RouterGemmParams p) {
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
  uint8_t* s_stage = sB + stages * b_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_stage + 4 * kRgStageWarpBytes);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + kRgMaxStages;
  uint64_t* tfull_bar = bars + 2 * kRgMaxStages;       // [2]: accumulator buffer ready
  uint64_t* tempty_bar = bars + 2 * kRgMaxStages + 2;  // [2]: the 4 epilogue warps are done with it
  uint64_t* drain_bar = bars + 2 * kRgMaxStages + 4;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * kRgMaxStages + 5);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t buf_cols = static_cast<uint32_t>(rg_tmem_cols(bn));
  const uint32_t tmem_cols = 2 * buf_cols;

  // unit -> (M tile, N tile, K range); the splits of one output tile are
  // adjacent units
  const int units = p.m_tiles * p.n_tiles * p.splits;
  const int64_t G = static_cast<int64_t>(p.n_terms) * p.nkb;
  struct Unit {
    int m0, n0, split, g0, g1;
  };
  auto decode = [&](int unit) {
    Unit u;
    u.split = unit % p.splits;
    const int n_blk = (unit / p.splits) % p.n_tiles;
    const int m_blk = unit / (p.splits * p.n_tiles);
    u.m0 = m_blk * kRgBM;
    u.n0 = n_blk * bn;
    u.g0 = static_cast<int>(G * u.split / p.splits);
    u.g1 = static_cast<int>(G * (u.split + 1) / p.splits);
    return u;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 4);
    }
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
      for (int unit = blockIdx.x; unit < units && !*s_abort; unit += gridDim.x) {
        const Unit u = decode(unit);
        for (int g = u.g0; g < u.g1 && !*s_abort; ++g) {
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
          if constexpr (KIND == kRgLogits) {
            tma_load_2d(a_dst, &p.tmA, fb, kx, u.m0);
            tma_load_2d(b_dst, &p.tmB, fb, kx, term * p.term_rows_b + u.n0);
          } else if constexpr (KIND == kRgWgrad) {
            tma_load_2d(a_dst, &p.tmA, fb, u.m0, kx);
            tma_load_2d(a_dst + 8192, &p.tmA, fb, u.m0 + 64, kx);
            for (int c = 0; c < bn / 64; ++c)
              tma_load_2d(b_dst + 8192 * c, &p.tmB, fb, u.n0 + 64 * c, term * p.term_rows_b + kx);
          } else {
            tma_load_2d(a_dst, &p.tmA, fb, kx, rg_dgrad_term_a(term) * p.term_rows_a + u.m0);
            for (int c = 0; c < bn / 64; ++c)
              tma_load_2d(b_dst + 8192 * c, &p.tmB, fb, u.n0 + 64 * c, rg_dgrad_term_b(term) * p.term_rows_b + kx);
          }
          ++issued;
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
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
    int ucount = 0;
    for (int unit = blockIdx.x; unit < units && !*s_abort; unit += gridDim.x, ++ucount) {
      const Unit u = decode(unit);
      const int acc = ucount & 1;
      // the epilogue has read this buffer's previous unit (two units ago)
      if (!rg_warp_wait(&tempty_bar[acc], ((ucount >> 1) & 1) ^ 1u)) {
        if (lane == 0) report(MOE_ERR_TIMEOUT);
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * buf_cols;
      bool ok = true;
      for (int g = u.g0; g < u.g1; ++g) {
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
            umma_bf16(d_tmem, adesc, bdesc, idesc, (g > u.g0 || kk > 0) ? 1u : 0u);
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
      // the unit's accumulator is complete (or abandoned) once its MMAs are done
      if (lane == 0) umma_commit(&tfull_bar[acc]);
      __syncwarp();
      if (!ok) break;
    }
    if (lane == 0) umma_commit(drain_bar);
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
    constexpr int kDxChunks = KIND == kRgDgrad ? kRgDgradBN / 32 : 1;
    int ucount = 0;
    for (int unit = blockIdx.x; unit < units; unit += gridDim.x, ++ucount) {
      const Unit u = decode(unit);
      const int acc = ucount & 1;
      // dX: the incoming values of this warp's rows are requested before the
      // wait, so their DRAM latency overlaps the main loop
      uint4 dxv[kDxChunks][4];
      if constexpr (KIND == kRgDgrad) {
#pragma unroll
        for (int ch = 0; ch < kDxChunks; ++ch)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int row = u.m0 + sub * 32 + i * 8 + tr_row;
            const int col = u.n0 + ch * 32 + tr_q * 8;
            dxv[ch][i] = (row < p.M && col < p.N)
                             ? *reinterpret_cast<const uint4*>(p.dx + static_cast<int64_t>(row) * p.dx_ld + col)
                             : make_uint4(0, 0, 0, 0);
          }
      }
      if (!rg_warp_wait(&tfull_bar[acc], (ucount >> 1) & 1)) {
        if (lane == 0) report(MOE_ERR_TIMEOUT);
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      if (*s_abort) break;
      const uint32_t taddr = tmem_base + static_cast<uint32_t>(acc) * buf_cols + (static_cast<uint32_t>(sub * 32) << 16);
      const int row0 = u.m0 + sub * 32;
      if constexpr (KIND == kRgDgrad) {
#pragma unroll
        for (int ch = 0; ch < kDxChunks; ++ch) {
          const int col0 = u.n0 + ch * 32;
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
      } else {
        // TMEM holds rg_tmem_cols(bn) >= 32 * ceil(bn / 32) columns per
        // buffer, so a chunk may run past bn; columns >= N are never written
#pragma unroll 1
        for (int ch = 0; ch < (bn + 31) / 32; ++ch) {
          const int col0 = u.n0 + ch * 32;
          if (col0 >= p.N) break;  // warp-uniform
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + ch * 32, v);
          tmem_ld_wait();
          if constexpr (KIND == kRgWgrad) {
            const int h = row0 + lane;
            float* o = p.out + u.split * p.out_split_stride + h;
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
                float* o = p.out + u.split * p.out_split_stride + static_cast<int64_t>(row) * p.out_ld + col;
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
            __syncwarp();
          }
        }
      }
      // this warp's TMEM reads of the buffer are complete: hand it back
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
    }
  }

  // ------------------------------------------------------------ tear-down
  tc_fence_before();
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
