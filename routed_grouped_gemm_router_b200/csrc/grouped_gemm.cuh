// Persistent grouped GEMM over variable-size expert segments for sm_100a.
//
// fused-MoE Triton project summary, How It Works: one grouped GEMM with
// persistent workers over expert-sorted rows replaces the per-expert loop;
// unsloth PR #3812: stacked expert weights [E, 2I, H] / [E, H, I] and the
// routing-weight multiply fused after the GEMM ("fuse_mul_post").
//
// B200 design (not a translation of the Triton kernels):
//  * CTA pairs (clusters of 2 on one TPC) run tcgen05 MMAs of 256 x 256 x 16:
//    each CTA stages its own 128 rows of A and its half (128 rows) of B, the
//    even CTA issues the MMA for both, and each CTA's TMEM receives its 128
//    accumulator rows. Per CTA a 64-deep K step is 32 KiB, so a 6-deep
//    TMA ring fits in shared memory;
//  * 10 warps per CTA: warp 0 issues TMA loads, warp 1 issues MMAs (even
//    CTA) and owns the TMEM allocation,
//    warps 2-9 run the epilogue, two per TMEM sub-partition;
//  * both CTAs' loads complete on the even CTA's "full" mbarrier; the MMA
//    warp's commits release the "empty" barriers of both CTAs; the fp32
//    accumulator is double-buffered in TMEM (2 x 256 columns) so the
//    epilogue of tile i overlaps the main loop of tile i+1;
//  * the tile list is built on the device from the per-expert offsets, so the
//    host never learns the counts and experts without rows cost nothing;
//  * segment tails of 1..128 rows run in a second, one-CTA instance of the
//    kernel (CG = 1: 128 x 256 x 16 MMAs, each CTA staging all 256 B rows)
//    that is launched first on a few whole TPCs; the pair instance, launched
//    right after on the other SMs, runs concurrently with it (a 256-row pair
//    tile would spend at least half its tensor work on padding rows there).
//
// Variants (all D = A * B^T with bf16 operands and fp32 accumulation):
//  FwdGateUp   A = Xp[P,H] (K-major), B = gate rows (even CTA) and up rows
//              (odd CTA) of W_gu[e]; epilogue h = silu(g) * u.
//  FwdDown     A = h[P,I], B = W_d[e][H,I], epilogue O = w_q * acc.
//  BwdDgradDown   A = dYp[P,H], B = W_d[e] read MN-major ([H,I] as K x N);
//              epilogue: h = silu(g) * u from the saved g|u, partial
//              dw = <acc, h>, dh = w_q*acc, SwiGLU backward -> dGU = [dg | du],
//              and hw = w_q * h for the down wgrad.
//  BwdDgradGateUp A = dGU[P,2I], B = W_gu[e] MN-major ([2I,H] as K x N) -> dXp.
//  BwdWgrad    per expert dW[e] = A^T B with the expert's rows as K; both
//              operands MN-major, loaded through per-expert tensor maps whose
//              row extent ends at the segment end, so TMA reads the rows of
//              the next expert as zeros.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace moe {

enum GemmKind : int { kFwdGateUp = 0, kFwdDown = 1, kBwdDgradDown = 2, kBwdDgradGateUp = 3, kBwdWgrad = 4 };
// Which operand, if any, is read with row-gather TMA from a token-order
// tensor (tmG; row = sorted_pair[r] / gather_k) instead of a permuted copy.
enum GatherMode : int { kNoGather = 0, kGatherA = 1, kGatherB = 2 };

constexpr int kBM = 256;        // rows of a pair tile
constexpr int kBMc = 128;       // rows per CTA
constexpr int kBN = 256;        // columns of a tile (accumulator columns per CTA)
constexpr int kBNc = 128;       // B rows (N) staged per CTA
constexpr int kBK = 64;
constexpr int kUmmaK = 16;
constexpr int kStages = 6;                   // ring depth of the pair instance
constexpr int kATileBytes = kBMc * kBK * 2;  // 16 KiB
constexpr int kBTileBytes = kBNc * kBK * 2;  // 16 KiB per CTA of a pair
constexpr int kStageBytes = kATileBytes + kBTileBytes;
// Per CTA-group constants: ring depth, bytes of B staged per CTA.
template <int CG> struct CgCfg {
  static constexpr int kStages = CG == 2 ? 6 : 4;
  static constexpr int kBBytes = CG == 2 ? kBTileBytes : 2 * kBTileBytes;
  static constexpr int kStageBytes = kATileBytes + kBBytes;
};
// Segment tails of 1..128 rows run as one-CTA tiles (0: every row-grouped
// tile is a pair tile).
#ifndef MOE_TAIL_TILES
#define MOE_TAIL_TILES 1
#endif
constexpr bool kTailTiles = MOE_TAIL_TILES != 0;

// Row tiles of a segment of `rows` rows handled by the CG instance (tails
// split off only when `tails` is set).
template <int CG>
__host__ __device__ __forceinline__ int seg_row_tiles(int rows, bool tails) {
  if (!tails) return CG == 2 ? (rows + 255) / 256 : 0;
  const int full = rows / 256, tail = rows - 256 * (rows / 256);
  return CG == 2 ? full + (tail > 128 ? 1 : 0) : (tail > 0 && tail <= 128 ? 1 : 0);
}
// Epilogue warps: 4 (one per TMEM sub-partition) or 8 (two per sub-partition,
// each half of the columns).
#ifndef MOE_EPI_WARPS
#define MOE_EPI_WARPS 8
#endif
constexpr int kEpiWarps = MOE_EPI_WARPS;
static_assert(kEpiWarps == 4 || kEpiWarps == 8, "4 or 8 epilogue warps");
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
// Epilogue outputs are written with the streaming hint (evict-first in L2)
// so they do not push reused operand tiles out of L2.
#ifndef MOE_STREAM_STORES
#define MOE_STREAM_STORES 1
#endif
// dgrad through down: how many 32-column chunks ahead of its use the
// epilogue loads g|u into registers. 1 (the default) fits the 168 registers a
// thread of the 320-thread CTA gets; 2 spills 48 bytes and measured 2-7 %
// slower on this kernel.
#ifndef MOE_DGRAD_GU_AHEAD
#define MOE_DGRAD_GU_AHEAD 1
#endif
constexpr int kGuAhead = MOE_DGRAD_GU_AHEAD;
static_assert(kGuAhead == 1 || kGuAhead == 2, "g|u loads run 1 or 2 chunks ahead");
// Raster of the row-grouped tiles inside an expert: 0 = N block fastest
// (concurrent pairs share A rows), 1 = row block fastest (concurrent pairs
// share a weight tile).
#ifndef MOE_TILE_M_FASTEST
#define MOE_TILE_M_FASTEST 0
#endif
constexpr int kTmemCols = 2 * kBN;
constexpr int kMaxExperts = 1024;
constexpr int kNumBarriers = 2 * kStages + 5;  // sized for the deeper (pair) ring
// Epilogue staging: per epilogue warp 32 rows x 32 bf16 (64 bytes per row).
// The four 16-byte pieces of row r are stored at piece (m ^ ((r >> 1) & 3)),
// which keeps both the row-wise writes (8 rows per quarter-warp phase) and
// the transposed reads (2 rows x 4 pieces per phase) free of bank conflicts.
constexpr int kStageStrideBytes = 64;
// dgrad-down writes this many partial routing-weight sums per (row, N tile):
// one per column half of the tile. The workspace layout and the router
// backward read the same constant.
constexpr int kDwSlotsPerNTile = 2;
constexpr int kStageWarpBytes = 32 * kStageStrideBytes;

struct GemmParams {
  CUtensorMap tmA;
  CUtensorMap tmB;
  CUtensorMap tmG;                 // gathered operand: token-order [gather_rows, gather_cols], box 64 x 1
  const CUtensorMap* expert_maps;  // wgrad: [2][E] maps (A then B) clipped at each segment end
  const int32_t* offsets;      // [E+1] expert segment bounds in the permuted rows
  const int32_t* sorted_pair;  // [P]
  const float* topk_w;         // [P] routing weight per pair id (NULL: 1)
  int64_t P;
  int E;
  int N;        // output columns: I (gate/up), H (down), I (dgrad-down), H (dgrad-gate/up), N (wgrad)
  int K;        // reduction length of the row-grouped variants
  int M;        // wgrad: rows of dW[e]
  int I;        // intermediate size (gate/up row split)
  int b_rows;   // rows of the B tensor map that belong to one expert
  int n_tiles;  // tiles along N
  int m_tiles;  // wgrad: tiles along M
  uint16_t* out;             // output (bf16), row stride out_ld
  int64_t out_ld;
  int64_t out_expert_stride;  // wgrad: elements per expert
  uint16_t* gu;               // FwdGateUp: optional g|u save; BwdDgradDown: g|u input
  uint16_t* hw_out;           // BwdDgradDown: w_q * h
  float* dw_part;             // BwdDgradDown: [P, kDwSlotsPerNTile * n_tiles] partial routing-weight grads
  int gather_k;               // pair id -> token: q / gather_k
  int gather_rows;
  int gather_cols;
  int tails;                  // row-grouped kinds: segment tails of 1..128 rows go to the one-CTA instance
  int wait_at_end;            // pair instance launched after a one-CTA instance: wait for it at the end
  float* out_f32;             // wgrad: fp32 output in place of `out` (NULL: bf16 to `out`), same strides
  int accumulate;             // wgrad with out_f32: out_f32 += acc (fp32 add) instead of out_f32 = acc
  unsigned long long* clock_acc;  // profiling (NULL: off): [0] += SM cycles, [1] += ns of each MMA issuer's loop
  // K extension (row-grouped kinds): after the ceil(K / 64) K blocks of tmA /
  // tmB, nkb2 more come from tmA2 / tmB2 into the same accumulator, i.e. the
  // GEMM of [A | A2] and [B | B2] along K. Same row coordinates as the first
  // pair, except an MN-major B2, whose K rows are b_rows2 per expert. Used for
  // the low-rank adapter term (A2 = scale * Z, B2 = the adapter's B or A).
  CUtensorMap tmA2;
  CUtensorMap tmB2;
  int nkb2;
  int b_rows2;
  float out_scale;  // FwdDown / BwdDgradGateUp / bf16 wgrad epilogue: out = out_scale * (w *) acc
  // Narrow tiles for skinny products (FwdDown, BwdDgradGateUp, wgrad kinds):
  // bn = 64 (K-major B only) or 128 output columns per tile instead of 256;
  // the MMA's N shrinks with it, so a product with few columns does not pay
  // for 256. 0: 256.
  int bn;
  // wgrad with out_f32: store the tile transposed, out_f32[e][n][m] (ld =
  // out_ld = M), so that a product with few rows can be computed as its
  // transpose with the few rows as narrow columns.
  int out_transposed;
  // bf16 wgrad: write full 32 x 32 chunks with TMA stores through tmOut
  // ([E * M rows, N] bf16, 32 x 32 boxes, 64-byte swizzle: the staging
  // buffer's layout) instead of per-thread stores.
  int out_tma;
  CUtensorMap tmOut;
};

template <int CG>
__host__ __device__ inline size_t gemm_smem_bytes(int E) {
  return 1024 /*alignment slack*/ + static_cast<size_t>(CgCfg<CG>::kStages) * CgCfg<CG>::kStageBytes +
         kNumBarriers * 8 + 16 +
         2 * static_cast<size_t>(E + 1) * 4 + 512 /*staging alignment*/ +
         static_cast<size_t>(kEpiWarps) * kStageWarpBytes;
}

struct TileInfo {
  int e, m_blk, n_blk;
  int row0;     // first permuted row of the pair tile (row-grouped) / first K row (wgrad)
  int rows;     // rows of the segment from row0 on (row-grouped) / rows of the segment (wgrad)
  int num_kb;   // K blocks
};

template <int KIND, int CG>
__device__ __forceinline__ TileInfo decode_tile(int t, const GemmParams& p, const int* s_off,
                                                const int* s_tstart) {
  TileInfo ti;
  if constexpr (KIND == kBwdWgrad) {
    const int per_e = p.m_tiles * p.n_tiles;
    ti.e = t / per_e;
    const int local = t - ti.e * per_e;
    ti.m_blk = local / p.n_tiles;
    ti.n_blk = local - ti.m_blk * p.n_tiles;
    ti.row0 = s_off[ti.e];
    ti.rows = s_off[ti.e + 1] - ti.row0;
    ti.num_kb = (ti.rows + kBK - 1) / kBK;
  } else {
    int lo = 0, hi = p.E;  // s_tstart[lo] <= t < s_tstart[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_tstart[mid] <= t) lo = mid; else hi = mid;
    }
    ti.e = lo;
    const int local = t - s_tstart[lo];
#if MOE_TILE_M_FASTEST
    const int m_tiles_e = seg_row_tiles<CG>(s_off[lo + 1] - s_off[lo], p.tails != 0);
    ti.n_blk = local / m_tiles_e;
    ti.m_blk = local - ti.n_blk * m_tiles_e;
#else
    ti.m_blk = local / p.n_tiles;
    ti.n_blk = local - ti.m_blk * p.n_tiles;
#endif
    // pair tiles start at 256-row steps; the one-CTA tile is the segment's tail
    ti.row0 = s_off[lo] + (CG == 2 ? ti.m_blk * kBM : ((s_off[lo + 1] - s_off[lo]) / kBM) * kBM);
    ti.rows = s_off[lo + 1] - ti.row0;
    ti.num_kb = (p.K + kBK - 1) / kBK + p.nkb2;
  }
  return ti;
}

// Bounded wait done by every lane of a warp; the result is warp-uniform.
// (Measured: letting only lane 0 poll, with the others parked on a shuffle,
// costs ~10% on every GEMM.)
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
  const bool ok = mbar_wait(bar, parity);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void store16(uint16_t* dst, uint4 v) {
#if MOE_STREAM_STORES
  __stcs(reinterpret_cast<uint4*>(dst), v);
#else
  *reinterpret_cast<uint4*>(dst) = v;
#endif
}

__device__ __forceinline__ void store8_bf16(uint16_t* dst, const float* v) {
  uint4 o;
  o.x = pack_bf16(v[0], v[1]);
  o.y = pack_bf16(v[2], v[3]);
  o.z = pack_bf16(v[4], v[5]);
  o.w = pack_bf16(v[6], v[7]);
  store16(dst, o);
}

__device__ __forceinline__ void unpack8(const uint4 i, float* v) {
  v[0] = bf16lo(i.x); v[1] = bf16hi(i.x);
  v[2] = bf16lo(i.y); v[3] = bf16hi(i.y);
  v[4] = bf16lo(i.z); v[5] = bf16hi(i.z);
  v[6] = bf16lo(i.w); v[7] = bf16hi(i.w);
}

// Row domain -> staging: the thread's 32 values of its row, rounded to bf16.
__device__ __forceinline__ void stage_row(uint8_t* stg, int lane, const float (&v)[32]) {
  uint8_t* rp = stg + lane * kStageStrideBytes;
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    uint4 o;
    o.x = pack_bf16(v[8 * m + 0], v[8 * m + 1]);
    o.y = pack_bf16(v[8 * m + 2], v[8 * m + 3]);
    o.z = pack_bf16(v[8 * m + 4], v[8 * m + 5]);
    o.w = pack_bf16(v[8 * m + 6], v[8 * m + 7]);
    *reinterpret_cast<uint4*>(rp + 16 * (m ^ sw)) = o;
  }
}

// Transposed domain: 8 bf16 of staged row r starting at column 8*q.
__device__ __forceinline__ uint4 read_piece(const uint8_t* stg, int r, int q) {
  return *reinterpret_cast<const uint4*>(stg + r * kStageStrideBytes + 16 * (q ^ ((r >> 1) & 3)));
}

// Stores one 32-column chunk (row domain values v, thread = row) as bf16 to
// base[(row0 + r) * ld + col0 + c] for the warp's valid rows and c < ncols.
// In the transposed domain lane l writes row 8*i + l/4, columns 8*(l%4)..+7:
// every quarter-warp writes two rows of 64 contiguous bytes.
__device__ __forceinline__ void emit_chunk(uint8_t* stg, const float (&v)[32], uint16_t* base, int64_t row0,
                                           int64_t ld, int col0, int ncols, int wrows, int tr_row, int tr_q,
                                           int lane) {
  stage_row(stg, lane, v);
  __syncwarp();
  const int col = col0 + tr_q * 8;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i * 8 + tr_row;
    if (r < wrows && col < ncols) store16(base + (row0 + r) * ld + col, read_piece(stg, r, tr_q));
  }
  __syncwarp();
}

// fp32 variant of emit_chunk: the chunk's 32 columns go through the staging
// buffer as two halves of 16 fp32 (64 bytes per row, the bf16 chunk's
// footprint and swizzle); in the transposed domain lane l then owns rows
// 8*i + l/4 and columns 4*(l%4)..+3 of the half. accumulate: base += v.
__device__ __forceinline__ void emit_chunk_f32(uint8_t* stg, const uint32_t (&a)[32], float* base, int64_t row0,
                                               int64_t ld, int col0, int ncols, int wrows, int tr_row, int tr_q,
                                               int lane, bool accumulate) {
  uint8_t* rp = stg + lane * kStageStrideBytes;
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
#pragma unroll
    for (int m = 0; m < 4; ++m)
      *reinterpret_cast<uint4*>(rp + 16 * (m ^ sw)) =
          make_uint4(a[16 * half + 4 * m], a[16 * half + 4 * m + 1], a[16 * half + 4 * m + 2], a[16 * half + 4 * m + 3]);
    __syncwarp();
    const int col = col0 + 16 * half + 4 * tr_q;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = i * 8 + tr_row;
      if (r < wrows && col < ncols) {
        float4* dst = reinterpret_cast<float4*>(base + (row0 + r) * ld + col);
        const uint4 u = read_piece(stg, r, tr_q);
        float4 v = make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w));
        if (accumulate) {
          const float4 o = *dst;
          v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
        }
        *dst = v;
      }
    }
    __syncwarp();
  }
}

// dgrad-down epilogue operands in the transposed domain: for rows 8*i + tr_row
// of the warp, 8 columns from `col`: g and u (16 bytes each); zeros for rows
// or columns that do not exist. (h is recomputed as silu(g) * u, which saves a
// third of the epilogue's loads; the loads, not the math, bound this kernel.)
__device__ __forceinline__ void dgrad_down_load(const GemmParams& p, int64_t wrow0, int wrows, int col, int tr_row,
                                                uint4 (&b)[8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = i * 8 + tr_row;
    if (r < wrows && col < p.I) {
      const int64_t gr = wrow0 + r;
      // (streaming-hint loads measured 16% slower here)
      b[2 * i] = __ldg(reinterpret_cast<const uint4*>(p.gu + gr * (2 * p.I) + col));
      b[2 * i + 1] = __ldg(reinterpret_cast<const uint4*>(p.gu + gr * (2 * p.I) + p.I + col));
    } else {
      b[2 * i] = b[2 * i + 1] = make_uint4(0, 0, 0, 0);
    }
  }
}

// silu(x) = x / (1 + e^-x) and the logistic sigmoid, with CUDA's fast exp and
// division intrinsics (a few ulp; for x << 0 the denominator overflows to
// inf and both return 0).
__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

// CG = 2: CTA pairs (launched as clusters of two); CG = 1: one CTA per tile,
// the segment tails of 1..128 rows (row-grouped kinds without gathering;
// launched as clusters of two as well, so the pair instance gets whole TPCs).
template <int KIND, int GATHER, int CG = 2>
__global__ void __launch_bounds__(kGemmThreads, 1) grouped_gemm_kernel(const __grid_constant__ GemmParams p) {
  constexpr bool kWgrad = (KIND == kBwdWgrad);
  static_assert(CG == 2 || (!kWgrad && GATHER == kNoGather), "one-CTA tiles: row-grouped kinds, no gathering");
  using Cfg = CgCfg<CG>;
  constexpr int kSt = Cfg::kStages;
  constexpr bool kAMN = kWgrad;
  constexpr bool kBMN = (KIND == kBwdDgradDown || KIND == kBwdDgradGateUp || kWgrad);
  constexpr uint32_t kIdesc = idesc_bf16_f32(CG == 2 ? kBM : kBMc, kBN, kAMN, kBMN);
  constexpr bool kNarrowOk = (KIND == kFwdDown || KIND == kBwdDgradGateUp || KIND == kBwdWgrad) && GATHER == kNoGather;
  // tile width along N: every coordinate below uses it; the TMEM buffers and
  // the staged B rows keep their 256-column size (the MMA reads the first bn)
  const int bn = (kNarrowOk && p.bn > 0) ? p.bn : kBN;
  const uint32_t idesc = bn == kBN ? kIdesc : idesc_bf16_f32(CG == 2 ? kBM : kBMc, bn, kAMN, kBMN);
  // B bytes each CTA stages per K block: its bn/2 (pair) or bn columns only
  // (a K-major B map's box is bn/2 rows high; MN-major boxes are 64 columns)
  const int b_bytes_cta = KIND == kFwdGateUp ? Cfg::kBBytes : (CG == 2 ? bn / 2 : bn) * kBK * 2;
  const uint32_t stage_tx = static_cast<uint32_t>(CG * (kATileBytes + b_bytes_cta));
  constexpr uint32_t kALbo = kAMN ? 8192u : 16u;
  constexpr uint32_t kBLbo = kBMN ? 8192u : 16u;
  constexpr uint32_t kAStep = kAMN ? 2048u : 32u;  // bytes per UMMA_K step
  constexpr uint32_t kBStep = kBMN ? 2048u : 32u;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kSt * kATileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSt * Cfg::kStageBytes);
  uint64_t* full_bar = bars;                 // even CTA: both CTAs' TMA bytes of a stage
  uint64_t* empty_bar = bars + kStages;      // each CTA: its stage may be refilled
  uint64_t* tfull_bar = bars + 2 * kStages;  // each CTA: accumulator buffer ready
  uint64_t* tempty_bar = bars + 2 * kStages + 2;  // even CTA: both epilogues done with a buffer
  uint64_t* drain_bar = bars + 2 * kStages + 4;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + kNumBarriers);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_off = reinterpret_cast<int*>(s_tmem + 4);
  int* s_tstart = s_off + (p.E + 1);
  // staging buffers 512-byte aligned: the 64-byte swizzle of the TMA stores
  // takes its pattern from the shared-memory address bits
  uint8_t* s_stage = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(s_tstart + (p.E + 1)) + 511) &
                                                ~uintptr_t(511));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CG = 2: 0 = even CTA (issues the MMAs), 1 = odd CTA; CG = 1: always 0
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const int pair = CG == 2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int num_pairs = CG == 2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  // ------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], CG * kEpiWarps);  // one arrival per epilogue warp of the pair / CTA
    }
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
    if constexpr (GATHER != kNoGather) tma_prefetch_desc(&p.tmG);
    if (p.nkb2 > 0) {
      tma_prefetch_desc(&p.tmA2);
      tma_prefetch_desc(&p.tmB2);
    }
  }
  if (warp == 1) {
    if constexpr (CG == 2) {
      tmem_alloc_pair(s_tmem, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(s_tmem, kTmemCols);
      tmem_relinquish();
    }
  }
  // Everything above touches no global memory; from here on this kernel
  // reads its predecessors' results, so it waits for them first. A pair
  // instance launched right after a one-CTA instance (wait_at_end) starts
  // only once every one-CTA CTA has passed this wait, so its inputs are
  // complete already: it runs concurrently with the one-CTA instance and
  // waits for it at its end instead, so the next kernel sees both.
  if (!(CG == 2 && p.wait_at_end)) griddep_wait();
  griddep_launch_dependents();
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) s_off[i] = p.offsets[i];
  __syncthreads();
  // The segment bounds come from the caller. Unless 0 <= offsets[0] <= ... <=
  // offsets[E] <= P, tiles would reach rows outside the operands: such a call
  // runs no tile (every segment emptied; a weight gradient writes zeros) and
  // reports MOE_ERR_DEVICE_CHECK.
  {
    int bad = 0;
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
      const int v = s_off[i];
      bad |= (v < 0) | (static_cast<int64_t>(v) > p.P) | (i < p.E && v > s_off[i + 1]);
    }
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0) report(MOE_ERR_DEVICE_CHECK);
      for (int i = threadIdx.x; i <= p.E; i += blockDim.x) s_off[i] = 0;
      __syncthreads();
    }
  }
  if (warp == 0 && !kWgrad) {
    // pair tiles of expert e = ceil(rows_e / 256) * n_tiles; exclusive prefix over experts
    const int per = (p.E + 31) / 32;
    const int e0 = lane * per;
    int local = 0;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < p.E) local += seg_row_tiles<CG>(s_off[e + 1] - s_off[e], p.tails != 0) * p.n_tiles;
    }
    const int incl = warp_inclusive_scan(local);
    int run = incl - local;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < p.E) {
        s_tstart[e] = run;
        run += seg_row_tiles<CG>(s_off[e + 1] - s_off[e], p.tails != 0) * p.n_tiles;
      }
    }
    if (lane == 31) s_tstart[p.E] = incl;
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync_all();  // the peer's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total_tiles = kWgrad ? p.E * p.m_tiles * p.n_tiles : s_tstart[p.E];

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    // Loads K block kb of tile ti (this CTA's A rows and its share of B: half
    // of the 256 B rows in a pair, all of them in a one-CTA tile) into a
    // ring stage. In a pair both CTAs' bytes complete on the even CTA's full
    // barrier (a cluster address); a one-CTA tile uses its own. A gathered
    // operand (GATHER) is not loaded here but by the gathering producer below.
    auto issue = [&](const TileInfo& ti, int kb, bool prefetch_only, uint8_t* a_dst, uint8_t* b_dst, uint32_t fb,
                     uint64_t* fb_local) {
      (void)prefetch_only;
      const CUtensorMap* mapA = &p.tmA;
      const CUtensorMap* mapB = &p.tmB;
      int kb_local = kb;
      int b_rows = p.b_rows;
      if constexpr (kWgrad) {
        mapA = p.expert_maps + ti.e;
        mapB = p.expert_maps + p.E + ti.e;
      } else {
        const int nkb1 = (p.K + kBK - 1) / kBK;
        if (kb >= nkb1) {  // K extension
          mapA = &p.tmA2;
          mapB = &p.tmB2;
          kb_local = kb - nkb1;
          b_rows = p.b_rows2;
        }
      }
      const int kx = kb_local * kBK;
      const int r = static_cast<int>(rank);
      // box c of B lands 8 KiB (MN-major boxes of 64 x 64) or 16 KiB
      // (K-major boxes of 128 rows) after the previous one
      int ax, ay, bx, by, nbox_a = 1, nbox_b = 1, b_step_x = 0, b_step_y = 0, b_step_bytes = 0;
      if constexpr (KIND == kFwdGateUp) {
        ax = kx; ay = ti.row0 + r * kBMc;
        // gate rows of the N block (even CTA / first box), then the matching up rows
        bx = kx; by = ti.e * p.b_rows + ti.n_blk * kBNc + r * p.I;
        if constexpr (CG == 1) { nbox_b = 2; b_step_y = p.I; b_step_bytes = kBTileBytes; }
      } else if constexpr (KIND == kFwdDown) {
        ax = kx; ay = ti.row0 + r * kBMc;
        bx = kx; by = ti.e * p.b_rows + ti.n_blk * bn + r * (bn / 2);
        if constexpr (CG == 1) { nbox_b = 2; b_step_y = bn / 2; b_step_bytes = (bn / 2) * kBK * 2; }
      } else if constexpr (KIND == kBwdDgradDown || KIND == kBwdDgradGateUp) {
        ax = kx; ay = ti.row0 + r * kBMc;
        bx = ti.n_blk * bn + r * (bn / 2); by = ti.e * b_rows + kx;
        nbox_b = (CG == 2 ? bn / 2 : bn) / 64; b_step_x = 64; b_step_bytes = 8192;
      } else {  // wgrad: K rows are the expert's permuted rows
        ax = ti.m_blk * kBM + r * kBMc; ay = ti.row0 + kx;
        bx = ti.n_blk * bn + r * (bn / 2); by = ay;
        nbox_a = 2;
        nbox_b = (bn / 2) / 64; b_step_x = 64; b_step_bytes = 8192;
      }
      if constexpr (GATHER != kGatherA) {
        for (int c = 0; c < nbox_a; ++c) {
          if constexpr (CG == 2) tma_load_2d_pair(a_dst + 8192 * c, mapA, fb, ax + 64 * c, ay);
          else tma_load_2d(a_dst + 8192 * c, mapA, fb_local, ax + 64 * c, ay);
        }
      }
      if constexpr (GATHER != kGatherB) {
        for (int c = 0; c < nbox_b; ++c) {
          if constexpr (CG == 2)
            tma_load_2d_pair(b_dst + b_step_bytes * c, mapB, fb, bx + b_step_x * c, by + b_step_y * c);
          else
            tma_load_2d(b_dst + b_step_bytes * c, mapB, fb_local, bx + b_step_x * c, by + b_step_y * c);
        }
      }
    };
    if (GATHER == kNoGather && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int t = pair; t < total_tiles && !*s_abort; t += num_pairs) {
        const TileInfo ti = decode_tile<KIND, CG>(t, p, s_off, s_tstart);
        if constexpr (kWgrad) {
          if (ti.num_kb == 0) continue;
          tensormap_acquire(p.expert_maps + ti.e);
          tensormap_acquire(p.expert_maps + p.E + ti.e);
        }
        for (int kb = 0; kb < ti.num_kb; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) {
            report(MOE_ERR_TIMEOUT);
            *s_abort = 1;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], stage_tx);
          issue(ti, kb, false, sA + stage * kATileBytes, sB + stage * Cfg::kBBytes,
                CG == 2 ? mapa_shared(smem_u32(&full_bar[stage]), 0) : 0u, &full_bar[stage]);
          ++issued;
          if (++stage == kSt) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // The even CTA's full barriers count both CTAs' bytes: waiting on the
      // last phases there means no load of the pair is still in flight when
      // the pair leaves (immediate in normal operation).
      if (rank == 0) {
        const int inflight = issued < kSt ? issued : kSt;
        for (int i = 0; i < inflight; ++i) {
          if (--stage < 0) {
            stage = kSt - 1;
            phase ^= 1u;
          }
          mbar_wait(&full_bar[stage], phase);
        }
      }
    }
    if constexpr (GATHER != kNoGather) {
      // ------------------------------------- producer with a gathered operand
      // Lane 0 loads the other operand with TMA exactly as above. The
      // gathered operand's tile is loaded by all 32 lanes with row-gather
      // TMA (four 128-byte rows per load, 512 bytes apart in the 128-byte
      // swizzled tile), completing on the even CTA's full barrier like every
      // other load of the pair. K-major A (row-grouped kinds): lane l loads
      // rows 4l..4l+3 of the CTA's 128 tile rows at K block kb. MN-major
      // operand (weight gradients): lane l loads K rows 4(l%16)..+3 of the
      // block into MN chunk l/16 of the CTA's 128 MN columns; a chunk wholly
      // past the tensor's columns (it only feeds masked outputs) reads chunk
      // 0 instead. Rows past the segment end read token 0: their outputs are
      // masked, or the other operand is zero there.
      constexpr bool kMN = kWgrad;
      if (p.sorted_pair == nullptr || p.gather_rows < 1) {  // no row map: nothing to gather
        if (lane == 0) report(MOE_ERR_DEVICE_CHECK);
        *s_abort = 1;
      }
      const int gk = p.gather_k > 0 ? p.gather_k : 1;
      const int gcols = p.gather_cols;
      auto tok_of = [&](int32_t q) {
        const int t = q / gk;
        return t < 0 ? 0 : (t >= p.gather_rows ? p.gather_rows - 1 : t);
      };
      auto tile_pairs = [&](int t, int32_t (&q)[4]) {
        const TileInfo tn = decode_tile<KIND, CG>(t, p, s_off, s_tstart);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int r = static_cast<int>(rank) * kBMc + 4 * lane + m;
          q[m] = r < tn.rows ? __ldg(p.sorted_pair + tn.row0 + r) : 0;
        }
      };
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      int32_t q_nxt[4] = {0, 0, 0, 0};
      if constexpr (!kMN) {
        if (pair < total_tiles && !*s_abort) tile_pairs(pair, q_nxt);
      }
      for (int t = pair; t < total_tiles && !__any_sync(0xffffffffu, *s_abort != 0); t += num_pairs) {
        const TileInfo ti = decode_tile<KIND, CG>(t, p, s_off, s_tstart);
        if constexpr (kWgrad) {
          if (ti.num_kb == 0) continue;
          if (lane == 0) {
            tensormap_acquire(p.expert_maps + ti.e);
            tensormap_acquire(p.expert_maps + p.E + ti.e);
          }
        }
        // gathered pair ids: the tile's (row-grouped; requested one tile
        // ahead) or those of K blocks kb and kb+1 (wgrad; two blocks ahead)
        int32_t q_cur[4] = {0, 0, 0, 0}, q_k1[4] = {0, 0, 0, 0}, q_k2[4] = {0, 0, 0, 0};
        auto block_pairs = [&](int kb, int32_t (&q)[4]) {
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int r = kb * kBK + 4 * (lane & 15) + m;
            q[m] = (kb < ti.num_kb && r < ti.rows) ? __ldg(p.sorted_pair + ti.row0 + r) : 0;
          }
        };
        if constexpr (!kMN) {
#pragma unroll
          for (int m = 0; m < 4; ++m) q_cur[m] = q_nxt[m];
          if (t + num_pairs < total_tiles) tile_pairs(t + num_pairs, q_nxt);
        } else {
          block_pairs(0, q_k1);
          block_pairs(1, q_k2);
        }
        bool ok = true;
        for (int kb = 0; kb < ti.num_kb; ++kb) {
          if constexpr (kMN) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              q_cur[m] = q_k1[m];
              q_k1[m] = q_k2[m];
            }
            block_pairs(kb + 2, q_k2);
          }
          if (!warp_wait(&empty_bar[stage], phase ^ 1u)) {
            if (lane == 0) report(MOE_ERR_TIMEOUT);
            *s_abort = 1;
            ok = false;
            break;
          }
          const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
          if (lane == 0) {
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * kStageBytes);
            issue(ti, kb, false, sA + stage * kATileBytes, sB + stage * kBTileBytes, fb, &full_bar[stage]);
          }
          uint8_t* g_tile = (GATHER == kGatherA) ? sA + stage * kATileBytes : sB + stage * kBTileBytes;
          int gx = kb * kBK, goff = 512 * lane;
          if constexpr (kMN) {
            const int chunk = lane >> 4;
            gx = (GATHER == kGatherA ? ti.m_blk * kBM : ti.n_blk * kBN) + static_cast<int>(rank) * kBMc + 64 * chunk;
            if (gx >= gcols) gx = 0;
            goff = 8192 * chunk + 512 * (lane & 15);
          }
          tma_gather4_pair(g_tile + goff, &p.tmG, fb, gx, tok_of(q_cur[0]), tok_of(q_cur[1]), tok_of(q_cur[2]),
                           tok_of(q_cur[3]));
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // no load of the pair may still be in flight when it leaves
      if (lane == 0 && rank == 0) {
        const int inflight = issued < kStages ? issued : kStages;
        for (int i = 0; i < inflight; ++i) {
          if (--stage < 0) {
            stage = kStages - 1;
            phase ^= 1u;
          }
          mbar_wait(&full_bar[stage], phase);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer (even CTA)
    if (rank == 0) {
      const uint32_t peer_empty0 = CG == 2 ? mapa_shared(smem_u32(&empty_bar[0]), 1) : 0u;
      const uint32_t peer_tfull0 = CG == 2 ? mapa_shared(smem_u32(&tfull_bar[0]), 1) : 0u;
      int stage = 0;
      uint32_t phase = 0;
      int tcount = 0;
      // effective SM clock over the main loop (profiling only): SM cycles
      // against global nanoseconds; the power limit lowers the first
      const long long clk0 = clock64();
      const unsigned long long ns0 = globaltimer_ns();
      for (int t = pair; t < total_tiles && !*s_abort; t += num_pairs) {
        const TileInfo ti = decode_tile<KIND, CG>(t, p, s_off, s_tstart);
        if (ti.num_kb == 0) continue;  // empty expert (wgrad): the epilogues write zeros
        const int acc = tcount & 1;
        if (!warp_wait(&tempty_bar[acc], ((tcount >> 1) & 1) ^ 1u)) {
          if (lane == 0) report(MOE_ERR_TIMEOUT);
          *s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        bool ok = true;
        for (int kb = 0; kb < ti.num_kb; ++kb) {
          if (!warp_wait(&full_bar[stage], phase)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t a_addr = smem_u32(sA + stage * kATileBytes);
            const uint32_t b_addr = smem_u32(sB + stage * Cfg::kBBytes);
#pragma unroll
            for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
              const uint64_t adesc = sdesc_sw128(a_addr + kk * kAStep, kALbo, 1024);
              const uint64_t bdesc = sdesc_sw128(b_addr + kk * kBStep, kBLbo, 1024);
              if constexpr (CG == 2) umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
              else umma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            if constexpr (CG == 2) {
              umma_commit_pair(smem_u32(&empty_bar[stage]));
              umma_commit_pair(peer_empty0 + stage * 8);
            } else {
              umma_commit(&empty_bar[stage]);
            }
          }
          __syncwarp();
          if (++stage == kSt) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) {
          if (lane == 0) report(MOE_ERR_TIMEOUT);
          *s_abort = 1;
          break;
        }
        if (lane == 0) {
          if constexpr (CG == 2) {
            umma_commit_pair(smem_u32(&tfull_bar[acc]));
            umma_commit_pair(peer_tfull0 + acc * 8);
          } else {
            umma_commit(&tfull_bar[acc]);
          }
        }
        __syncwarp();
        ++tcount;
      }
      if (p.clock_acc != nullptr && lane == 0) {
        atomicAdd(p.clock_acc, static_cast<unsigned long long>(clock64() - clk0));
        atomicAdd(p.clock_acc + 1, globaltimer_ns() - ns0);
      }
      // all MMAs of the pair must finish before TMEM is released
      if (lane == 0) {
        if constexpr (CG == 2) umma_commit_pair(smem_u32(drain_bar));
        else umma_commit(drain_bar);
      }
      __syncwarp();
      warp_wait(drain_bar, 0);
    }
  } else {
    // ------------------------------------------------------- epilogue
    // Thread (warp w, lane l) reads TMEM lane 32*(w%4)+l: one accumulator row
    // ("row domain"); the two warps of a sub-partition split the columns.
    // Every 32-column chunk is rounded to bf16, staged through the warp's own
    // shared buffer and read back transposed ("transposed domain"): lane l
    // then owns rows 8*i + l/4, i = 0..3, and columns 8*(l%4)..+7 of the
    // chunk, so each quarter-warp of a 16-byte global access covers two rows
    // of 64 contiguous bytes.
    const int sub = warp & 3;
    const int half = kEpiWarps == 8 ? (warp - 2) >> 2 : 0;  // which half of the tile's columns
    const int tr_row = lane >> 2;  // transposed domain: row 8*i + tr_row
    const int tr_q = lane & 3;     // transposed domain: columns 8*tr_q..+7 of the chunk
    uint8_t* stg = s_stage + (warp - 2) * kStageWarpBytes;
    const uint32_t leader_tempty0 = CG == 2 ? mapa_shared(smem_u32(&tempty_bar[0]), 0) : 0u;
    constexpr int kChunks = (KIND == kFwdGateUp ? 128 : kBN) / 32 / (kEpiWarps / 4);  // chunks per warp
    int tcount = 0;
    for (int t = pair; t < total_tiles && !*s_abort; t += num_pairs) {
      const TileInfo ti = decode_tile<KIND, CG>(t, p, s_off, s_tstart);
      // this CTA's 128 rows of the pair tile, this warp's 32 of them
      const int cta_row0 = static_cast<int>(rank) * kBMc + sub * 32;
      const int tile_rows = kWgrad ? p.M - ti.m_blk * kBM : ti.rows;
      const int wrows = max(0, min(32, tile_rows - cta_row0));
      // first output row of this warp: permuted row (row-grouped) or dW row (wgrad)
      const int64_t wrow0 = kWgrad ? static_cast<int64_t>(ti.m_blk) * kBM + cta_row0
                                   : static_cast<int64_t>(ti.row0) + cta_row0;
      uint16_t* out_base = kWgrad ? (p.out_f32 != nullptr ? nullptr : p.out + ti.e * p.out_expert_stride) : p.out;
      float* out_f32 = kWgrad && p.out_f32 != nullptr ? p.out_f32 + ti.e * p.out_expert_stride : nullptr;
      const int ch0 = half * kChunks;  // first 32-column chunk of this warp
      if constexpr (kWgrad) {
        if (ti.num_kb == 0) {  // expert without rows: its weight gradient is zero (unchanged if accumulating)
          if (out_f32 != nullptr && p.accumulate) continue;
          for (int ch = ch0; ch < ch0 + kChunks && ch * 32 < bn; ++ch) {
            const int col = ti.n_blk * bn + ch * 32 + tr_q * 8;
            if (p.out_transposed && out_f32 != nullptr) {  // rows of the transposed tile: columns here
              if (lane < wrows) {
                for (int j = 0; j < 32 && ti.n_blk * bn + ch * 32 + j < p.N; ++j)
                  out_f32[static_cast<int64_t>(ti.n_blk * bn + ch * 32 + j) * p.out_ld + wrow0 + lane] = 0.f;
              }
              continue;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = i * 8 + tr_row;
              if (r < wrows && col < p.N) {
                if (out_f32 != nullptr) {
                  float4* dst = reinterpret_cast<float4*>(out_f32 + (wrow0 + r) * p.out_ld + col);
                  dst[0] = make_float4(0.f, 0.f, 0.f, 0.f);
                  dst[1] = make_float4(0.f, 0.f, 0.f, 0.f);
                } else {
                  *reinterpret_cast<uint4*>(out_base + (wrow0 + r) * p.out_ld + col) = make_uint4(0, 0, 0, 0);
                }
              }
            }
          }
          continue;
        }
      }
      // per-row routing weight, row domain (lane = row within the warp)
      float wq = 1.0f;
      if constexpr (KIND == kFwdDown || KIND == kBwdDgradDown) {
        if (lane < wrows && p.topk_w != nullptr) {
          const int32_t q = p.sorted_pair[wrow0 + lane];
          wq = (q >= 0 && q < p.P) ? __ldg(p.topk_w + q) : 0.0f;
        }
      }
      // dgrad-down: g|u of the first kGuAhead chunks are requested before
      // the wait, so their latency hides behind the main loop; each later
      // chunk's kGuAhead chunks ahead of its use
      uint4 dd_cur[8], dd_nxt[8];
      if constexpr (KIND == kBwdDgradDown) {
        dgrad_down_load(p, wrow0, wrows, ti.n_blk * kBN + ch0 * 32 + tr_q * 8, tr_row, dd_cur);
        if constexpr (kGuAhead == 2)
          dgrad_down_load(p, wrow0, wrows, ti.n_blk * kBN + (ch0 + 1) * 32 + tr_q * 8, tr_row, dd_nxt);
      }

      const int acc = tcount & 1;
      if (!warp_wait(&tfull_bar[acc], (tcount >> 1) & 1)) {
        if (lane == 0) report(MOE_ERR_TIMEOUT);
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + static_cast<uint32_t>(acc * kBN) + (static_cast<uint32_t>(sub * 32) << 16);

      if constexpr (KIND == kFwdGateUp) {
        const int I = p.I;
#pragma unroll 1
        for (int ch = ch0; ch < ch0 + kChunks; ++ch) {
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(taddr + ch * 32, g);
          tmem_ld_32x32b_x32(taddr + 128 + ch * 32, u);
          tmem_ld_wait();
          const int col0 = ti.n_blk * 128 + ch * 32;
          if (col0 >= I) continue;  // warp-uniform
          float v[32];
          if (p.out != nullptr) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = silu_f(__uint_as_float(g[j])) * __uint_as_float(u[j]);
            emit_chunk(stg, v, out_base, wrow0, p.out_ld, col0, I, wrows, tr_row, tr_q, lane);
          }
          if (p.gu != nullptr) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(g[j]);
            emit_chunk(stg, v, p.gu, wrow0, 2 * I, col0, I, wrows, tr_row, tr_q, lane);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(u[j]);
            emit_chunk(stg, v, p.gu + I, wrow0, 2 * I, col0, I, wrows, tr_row, tr_q, lane);
          }
        }
      } else if constexpr (KIND == kBwdDgradDown) {
        const int I = p.I;
        float dwp[4] = {0.f, 0.f, 0.f, 0.f};
        float wrow[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) wrow[i] = __shfl_sync(0xffffffffu, wq, i * 8 + tr_row);
#pragma unroll 1
        for (int ch = ch0; ch < ch0 + kChunks; ++ch) {
          const int col = ti.n_blk * kBN + ch * 32 + tr_q * 8;
          [[maybe_unused]] uint4 nxt2[8];  // used when kGuAhead == 2
          if constexpr (kGuAhead == 2) {
            if (ch + 2 < ch0 + kChunks) dgrad_down_load(p, wrow0, wrows, col + 64, tr_row, nxt2);
          } else {
            if (ch + 1 < ch0 + kChunks) dgrad_down_load(p, wrow0, wrows, col + 32, tr_row, dd_nxt);
          }
          uint32_t a[32];
          tmem_ld_32x32b_x32(taddr + ch * 32, a);
          tmem_ld_wait();
          float av[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) av[j] = __uint_as_float(a[j]);
          stage_row(stg, lane, av);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = i * 8 + tr_row;
            if (r < wrows && col < I) {
              float dhp[8], gv[8], uv[8], dg[8], du[8], hw[8];
              unpack8(read_piece(stg, r, tr_q), dhp);
              unpack8(dd_cur[2 * i], gv);
              unpack8(dd_cur[2 * i + 1], uv);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float sg = sigmoid_f(gv[j]);
                const float hv = gv[j] * sg * uv[j];  // h = silu(g) * u
                dwp[i] += dhp[j] * hv;
                const float dh = wrow[i] * dhp[j];
                du[j] = dh * gv[j] * sg;
                dg[j] = dh * uv[j] * sg * (1.0f + gv[j] * (1.0f - sg));
                hw[j] = wrow[i] * hv;
              }
              const int64_t gr = wrow0 + r;
              store8_bf16(p.out + gr * p.out_ld + col, dg);
              store8_bf16(p.out + gr * p.out_ld + I + col, du);
              store8_bf16(p.hw_out + gr * I + col, hw);
            }
          }
          __syncwarp();
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            dd_cur[x] = dd_nxt[x];
            if constexpr (kGuAhead == 2) dd_nxt[x] = nxt2[x];
          }
        }
        // each row's partial dot product is spread over the 4 lanes with the
        // same l/4; the two column halves write separate slots
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          dwp[i] += __shfl_xor_sync(0xffffffffu, dwp[i], 1);
          dwp[i] += __shfl_xor_sync(0xffffffffu, dwp[i], 2);
          const int r = i * 8 + tr_row;
          if (tr_q == 0 && r < wrows)
            p.dw_part[(wrow0 + r) * (kDwSlotsPerNTile * p.n_tiles) + kDwSlotsPerNTile * ti.n_blk + half] = dwp[i];
          if (kEpiWarps == 4 && tr_q == 0 && r < wrows)
            p.dw_part[(wrow0 + r) * (kDwSlotsPerNTile * p.n_tiles) + kDwSlotsPerNTile * ti.n_blk + 1] = 0.f;
        }
      } else {  // FwdDown (weighted), BwdDgradGateUp, BwdWgrad: plain bf16 store of (scale * w *) acc
        wq *= p.out_scale;
#pragma unroll 1
        for (int ch = ch0; ch < ch0 + kChunks; ch += 2) {
          uint32_t a0[32], a1[32];
          tmem_ld_32x32b_x32(taddr + ch * 32, a0);
          tmem_ld_32x32b_x32(taddr + (ch + 1) * 32, a1);
          tmem_ld_wait();
          const int col0 = ti.n_blk * bn + ch * 32;
          const bool in0 = ch * 32 < bn && col0 < p.N;              // warp-uniform
          const bool in1 = (ch + 1) * 32 < bn && col0 + 32 < p.N;
          if (kWgrad && out_f32 != nullptr) {  // fp32 weight gradient: the accumulator unrounded
            const bool accum = p.accumulate != 0;
            if (p.out_transposed) {
              // thread = tile row m; for each column n the warp's 32 rows are
              // 32 consecutive floats of out[n][.]: 128-byte stores
              float* col_base = out_f32 + wrow0 + lane;
              if (lane < wrows && in0) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  if (col0 + j < p.N) {
                    float* dst = col_base + static_cast<int64_t>(col0 + j) * p.out_ld;
                    float v = __uint_as_float(a0[j]);
                    if (accum) v += *dst;
                    *dst = v;
                  }
                }
              }
              if (lane < wrows && in1) {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  if (col0 + 32 + j < p.N) {
                    float* dst = col_base + static_cast<int64_t>(col0 + 32 + j) * p.out_ld;
                    float v = __uint_as_float(a1[j]);
                    if (accum) v += *dst;
                    *dst = v;
                  }
                }
              }
              continue;
            }
            if (in0) emit_chunk_f32(stg, a0, out_f32, wrow0, p.out_ld, col0, p.N, wrows, tr_row, tr_q, lane, accum);
            if (in1)
              emit_chunk_f32(stg, a1, out_f32, wrow0, p.out_ld, col0 + 32, p.N, wrows, tr_row, tr_q, lane, accum);
            continue;
          }
          float v[32];
          if (kWgrad && p.out_tma) {
            // bf16 weight gradient through TMA stores: the chunk is staged
            // once in the store box's layout and one thread stores it; a
            // partial box (fewer than 32 rows left in dW[e]) goes the
            // per-thread way, which must not overlap a store still reading
            // the buffer either
            const bool full = wrows == 32;
            const int row_g = ti.e * p.M + static_cast<int>(wrow0);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if (!(hh == 0 ? in0 : in1)) continue;  // warp-uniform
              const uint32_t* a = hh == 0 ? a0 : a1;
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = wq * __uint_as_float(a[j]);
              if (lane == 0) bulk_wait_group_read0();
              __syncwarp();
              if (full) {
                stage_row(stg, lane, v);
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                  tma_store_2d(&p.tmOut, stg, col0 + 32 * hh, row_g);
                  bulk_commit_group();
                }
              } else {
                emit_chunk(stg, v, out_base, wrow0, p.out_ld, col0 + 32 * hh, p.N, wrows, tr_row, tr_q, lane);
              }
            }
            continue;
          }
          if (in0) {  // warp-uniform
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = wq * __uint_as_float(a0[j]);
            emit_chunk(stg, v, out_base, wrow0, p.out_ld, col0, p.N, wrows, tr_row, tr_q, lane);
          }
          if (in1) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = wq * __uint_as_float(a1[j]);
            emit_chunk(stg, v, out_base, wrow0, p.out_ld, col0 + 32, p.N, wrows, tr_row, tr_q, lane);
          }
        }
      }
      // The warp's TMEM reads are complete (tcgen05.wait::ld); the arrival
      // only hands the accumulator buffer back to the MMA issuer, so it does
      // not wait for the tile's global stores to drain.
      tc_fence_before();
      __syncwarp();
#ifndef MOE_TEMPTY_RELAXED
#define MOE_TEMPTY_RELAXED 1
#endif
      if (lane == 0) {
        if constexpr (CG == 1) mbar_arrive(&tempty_bar[acc]);
        else if (MOE_TEMPTY_RELAXED) mbar_arrive_cluster_relaxed(leader_tempty0 + acc * 8);
        else mbar_arrive_cluster(leader_tempty0 + acc * 8);
      }
      ++tcount;
    }
    // this warp's TMA stores are complete before the CTA leaves
    if (kWgrad && p.out_tma && lane == 0) bulk_wait_group0();
    __syncwarp();
  }

  // ------------------------------------------------------------- tear-down
  tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync_all();  // the pair's MMAs, loads and TMEM reads are all finished
  if (warp == 1) {
    tc_fence_after();
    if constexpr (CG == 2) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
  // a pair instance that did not wait at its start completes only after the
  // one-CTA instance launched before it
  if (CG == 2 && p.wait_at_end) griddep_wait();
}

// Writes, for each expert e, copies of the A and B tensor maps of the weight
// gradient whose row extent ends at offsets[e+1] (the end of the expert's
// segment): out[e] for A, out[E + e] for B. One warp per map.
__global__ void __launch_bounds__(256) build_expert_maps_kernel(const __grid_constant__ CUtensorMap base_a,
                                                                const __grid_constant__ CUtensorMap base_b,
                                                                const int32_t* __restrict__ offsets, int E,
                                                                CUtensorMap* __restrict__ out) {
  __shared__ alignas(128) CUtensorMap s_map[8];
  griddep_wait();
  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 8 + warp;
  if (m >= 2 * E) return;  // warp-uniform
  const int e = m < E ? m : m - E;
  const CUtensorMap& src = m < E ? base_a : base_b;
  if (lane < 8)
    reinterpret_cast<uint4*>(&s_map[warp])[lane] = reinterpret_cast<const uint4*>(&src)[lane];
  __syncwarp();
  if (lane == 0) {
    const int end = offsets[e + 1];
    tensormap_set_rows(&s_map[warp], static_cast<uint32_t>(end > 0 ? end : 1));
  }
  __syncwarp();
  tensormap_copy_release(out + m, &s_map[warp]);
}

}  // namespace moe
