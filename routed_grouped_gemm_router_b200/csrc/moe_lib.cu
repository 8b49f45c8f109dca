// C ABI of the fused MoE expert layer (declared in include/moe.h).
//
// This file validates arguments, sizes the caller's workspace, encodes the TMA
// tensor maps and enqueues the kernels of route.cuh, permute.cuh,
// grouped_gemm.cuh, combine.cuh, router_bwd.cuh and ep.cuh on the caller's
// stream.
// It allocates no device memory and never synchronises (except the status
// read and the profiling read, which say so).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/moe.h"
#include "combine.cuh"
#include "common.cuh"
#include "ep.cuh"
#include "grouped_gemm.cuh"
#include "lora.cuh"
#include "permute.cuh"
#include "route.cuh"
#include "router_bwd.cuh"
#include "router_linear.cuh"

// bf16 weight gradients leave the wgrad epilogue through TMA stores (0: per-
// thread stores from the staging buffer, as the other outputs).
#ifndef MOE_WGRAD_TMA_STORE
#define MOE_WGRAD_TMA_STORE 1
#endif

namespace moe {

// Waits on an mbarrier that nothing ever arrives at, with the library's
// bounded wait shortened to `limit_ns`; when the limit passes it records
// MOE_ERR_TIMEOUT in the device status word and returns. Exercises the
// failure path of every pipeline wait without hanging the device.
__global__ void wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbarrier_init();
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(&bar, 0)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      report(MOE_ERR_TIMEOUT);
      return;
    }
  }
}

namespace {

// ------------------------------------------------------------------ helpers
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
inline bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }
inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kMaxDevices = 64;

// Device facts, looked up once per device.
struct DeviceInfo {
  int checked = 0;
  int supported = 0;
  int num_sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);
    d.num_sms = sms;
    d.checked = 1;
  }
  *out = &d;
  return d.supported ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// bf16 2-D row-major tensor [rows, inner], 128-byte swizzled boxes of
// box_inner x box_rows; out-of-range elements read as zero.
// row_stride_elems (0: = inner) is the distance between rows in elements.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
              uint32_t box_rows, uint64_t row_stride_elems = 0,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {(row_stride_elems ? row_stride_elems : inner) * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- profiling
enum ProfSlot : int {
  kProfRoute = 0,
  kProfPermCount,
  kProfPermScan,
  kProfPermScatter,
  kProfGatherX,
  kProfFwdGateUp,
  kProfFwdDown,
  kProfCombineY,
  kProfGatherDy,
  kProfRecomputeGateUp,
  kProfDgradDown,
  kProfDgradGateUp,
  kProfCombineDx,
  kProfWgradGateUp,
  kProfWgradDown,
  kProfRouterBwd,
  kProfRouterSplitW,
  kProfRouterLogits,
  kProfRouterSplitDl,
  kProfRouterWgrad,
  kProfRouterSumSplits,
  kProfRouterDgrad,
  kProfLoraZGateUp,
  kProfLoraZDown,
  kProfLoraVDown,
  kProfLoraVGateUp,
  kProfLoraWeightRows,
  kProfLoraDAGateUp,
  kProfLoraDBGateUp,
  kProfLoraDADown,
  kProfLoraDBDown,
  kProfRouteHist,
  kProfPermScanScatter,
  kProfPairDw,
  kProfEpPack,
  kProfSlots
};
const char* const kProfNames[kProfSlots] = {
    "route",          "permute_count",       "permute_scan",           "permute_scatter",
    "gather_x",       "gemm_fwd_gate_up",    "gemm_fwd_down",          "combine_y",
    "gather_dy",      "gemm_recompute_gate_up", "gemm_bwd_dgrad_down", "gemm_bwd_dgrad_gate_up",
    "combine_dx",     "gemm_bwd_wgrad_gate_up", "gemm_bwd_wgrad_down", "router_bwd",
    "router_split_w", "gemm_router_logits",  "router_split_dlogits",   "gemm_router_wgrad",
    "router_sum_splits", "gemm_router_dgrad", "gemm_lora_z_gate_up", "gemm_lora_z_down", "gemm_lora_v_down",
    "gemm_lora_v_gate_up", "lora_weight_rows", "gemm_lora_da_gate_up", "gemm_lora_db_gate_up", "gemm_lora_da_down",
    "gemm_lora_db_down", "route_hist", "permute_scan_scatter", "pair_dw", "ep_pack_rows"};

struct Profiler {
  std::mutex mu;
  bool on = false;
  int only = -1;  // record only this slot (-1: every slot)
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> recs[kProfSlots];
  std::vector<cudaEvent_t> pool;
  cudaEvent_t take() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  void clear() {
    for (auto& v : recs) {
      for (auto& pr : v) {
        pool.push_back(pr.first);
        pool.push_back(pr.second);
      }
      v.clear();
    }
  }
};
Profiler g_prof;

// Per-slot effective SM clock of the GEMMs while profiling: [slot][0] SM
// cycles, [slot][1] nanoseconds, summed over the MMA issuers' main loops.
// A static device array: profiling allocates no device memory.
__device__ unsigned long long g_gemm_clock[kProfSlots][2];

// Device address of g_gemm_clock on the current device, looked up once per
// device (NULL if the lookup fails); the cache is guarded by its own mutex so
// host threads may call in concurrently.
unsigned long long* gemm_clock_base() {
  constexpr int kMaxDevices = 64;
  static unsigned long long* base[kMaxDevices] = {};
  static std::mutex mu;
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (base[d] == nullptr) {
    void* b = nullptr;
    if (cudaGetSymbolAddress(&b, g_gemm_clock) != cudaSuccess) return nullptr;
    base[d] = static_cast<unsigned long long*>(b);
  }
  return base[d];
}

// Device address of the slot's clock counters when that slot is being
// profiled, else NULL (the kernels then skip the accounting).
unsigned long long* gemm_clock_slot(int slot) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  if (!g_prof.on || (g_prof.only >= 0 && g_prof.only != slot)) return nullptr;
  unsigned long long* base = gemm_clock_base();
  return base != nullptr ? base + 2 * slot : nullptr;
}

// Brackets one kernel launch with events on its stream when profiling is on.
struct ProfScope {
  int slot;
  cudaStream_t s;
  cudaEvent_t end = nullptr;
  ProfScope(int slot_, cudaStream_t s_) : slot(slot_), s(s_) {
    std::lock_guard<std::mutex> lock(g_prof.mu);
    if (!g_prof.on || (g_prof.only >= 0 && g_prof.only != slot)) return;
    cudaEvent_t start = g_prof.take();
    end = g_prof.take();
    cudaEventRecord(start, s);
    g_prof.recs[slot].push_back({start, end});
  }
  ~ProfScope() {
    if (end != nullptr) cudaEventRecord(end, s);
  }
};

int launch_status() { return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

template <int KIND, int GATHER, int CG>
int launch_gemm_instance(const GemmParams& p, int grid, cudaStream_t s) {
  const size_t smem = gemm_smem_bytes<CG>(p.E);
  if (cudaFuncSetAttribute(grouped_gemm_kernel<KIND, GATHER, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  // both instances run as clusters of two, so each takes whole TPCs
  if (launch_pdl_clustered(grouped_gemm_kernel<KIND, GATHER, CG>, dim3(grid), dim3(kGemmThreads), smem, s, 2u, p) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_status();
}

// One grouped GEMM. Row-grouped kinds without gathering with tail_ctas > 0:
// the one-CTA instance over the segment tails of 1..128 rows on tail_ctas
// CTAs, then the pair instance over the rest on the other SMs, concurrently
// (grid is the pair instance's grid without tails). Otherwise the pair
// instance alone over every tile.
template <int KIND, int GATHER = kNoGather>
int launch_gemm(GemmParams p, int grid, cudaStream_t s, int slot, int tail_ctas = 0, int num_sms = 0) {
  ProfScope ps(slot, s);
  p.clock_acc = gemm_clock_slot(slot);
  if constexpr (KIND != kBwdWgrad && GATHER == kNoGather) {
    if (kTailTiles && tail_ctas > 0) {
      p.tails = 1;
      p.wait_at_end = 0;
      if (int st = launch_gemm_instance<KIND, GATHER, 1>(p, tail_ctas, s)) return st;
      p.wait_at_end = 1;
      int pg = num_sms - tail_ctas;
      pg = (pg < grid ? pg : grid) & ~1;
      return launch_gemm_instance<KIND, GATHER, 2>(p, pg > 2 ? pg : 2, s);
    }
  }
  p.tails = 0;
  p.wait_at_end = 0;
  return launch_gemm_instance<KIND, GATHER, 2>(p, grid, s);
}

inline int cdiv(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

// Persistent grid for the GEMMs: CTA pairs, at most one CTA per SM and no
// more pairs than tiles. Always even (clusters of two).
inline int pair_grid(int64_t tiles, int num_sms) {
  const int64_t pairs = num_sms / 2;
  const int64_t n = tiles < pairs ? tiles : pairs;
  return static_cast<int>(2 * (n > 0 ? n : 1));
}
inline int rowgrouped_grid(int64_t P, int E, int n_tiles, int num_sms) {
  return pair_grid((static_cast<int64_t>(cdiv(P, kBM)) + E) * n_tiles, num_sms);
}
// CTAs (even) for the one-CTA tail instance, from the expected work split:
// about w E segments end in a tail of 1..128 rows (half of them for evenly
// spread routing, more when a few experts take most rows and the rest are
// small), one CTA for one tile time each; the full tiles cost two CTAs each
// (P / 256 of them). When the average segment is 128 rows or less nearly
// every tile is a tail. The weight w also carries the tail tiles' lower
// efficiency per CTA (each stages all 256 B rows), and its best value grows
// with the segment length: measured 0.65 on 512-row segments (Qwen3-30B-A3B
// layer, 0.4-1.0 swept) and 0.8 on 1024-row ones (Qwen3-235B-A22B layer,
// 0.5-1.0 swept); in between it is interpolated. MOE_TAIL_WEIGHT fixes it.
inline double tail_weight(int64_t P, int E) {
#ifdef MOE_TAIL_WEIGHT
  (void)P;
  (void)E;
  return MOE_TAIL_WEIGHT;
#else
  const double rows = static_cast<double>(P) / E;
  const double f = rows <= 512.0 ? 0.0 : rows >= 1024.0 ? 1.0 : (rows - 512.0) / 512.0;
  return 0.65 + 0.15 * f;
#endif
}
inline int tail_ctas(int64_t P, int E, int num_sms) {
  if (!kTailTiles || P == 0) return 0;
  int c;
  if (P <= static_cast<int64_t>(128) * E) {
    c = num_sms - 4;
  } else {
    const double tail = tail_weight(P, E) * E, full = 2.0 * static_cast<double>(P) / kBM;
    c = static_cast<int>(num_sms * tail / (tail + full) + 0.5);
  }
  c &= ~1;
  if (c < 2) c = 2;
  if (c > num_sms - 4) c = (num_sms - 4) & ~1;
  return c;
}

// The gathered operand of a GEMM: token-order rows [T, H] picked by
// sorted_pair[r] / k, read through a row-gather map (64-column boxes one row
// high). The operand's own tensor map is not loaded from; the caller keeps a
// valid map in its place for the kernel's descriptor prefetch.
bool set_gather(GemmParams& g, const moe_bf16* src, const int32_t* sorted_pair, int T, int k, int H) {
  if (!make_map(&g.tmG, src, H, T, 64, 1)) return false;
  g.sorted_pair = sorted_pair;  // the gathering producer maps rows to tokens through it
  g.gather_k = k;
  g.gather_rows = T;
  g.gather_cols = H;
  return true;
}

GemmParams base_params(int E, int64_t P, const int32_t* offsets) {
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.E = E;
  p.P = P;
  p.offsets = offsets;
  p.out_scale = 1.0f;
  return p;
}

// ------------------------------------------------------------ LoRA adapters
// One adapter per expert on each stacked weight: the layer uses
// W_gu + scale B_gu A_gu and W_d + scale B_d A_d. The forward keeps the
// adapter activations Z_gu = scale Xp A_gu^T and Z_d = scale h A_d^T [P, r].
struct LoraArgs {
  int r = 0;
  float scale = 1.0f;
  const moe_bf16* A_gu = nullptr;  // [E, r, H]
  const moe_bf16* B_gu = nullptr;  // [E, 2I, r]
  const moe_bf16* A_d = nullptr;   // [E, r, I]
  const moe_bf16* B_d = nullptr;   // [E, H, r]
  moe_bf16* Z_gu = nullptr;        // [P, r]
  moe_bf16* Z_d = nullptr;         // [P, r]
  float* dA_gu = nullptr;          // backward outputs, fp32
  float* dB_gu = nullptr;
  float* dA_d = nullptr;
  float* dB_d = nullptr;
  bool accumulate = false;
};
constexpr int kLoraMaxRank = 512;

bool lora_rank_ok(int r) { return r >= 8 && r <= kLoraMaxRank && r % 8 == 0; }

// Tile width for a product with n output columns: the narrowest of 64
// (K-major B only: its rows are the columns), 128 and 256 that holds them.
// An MN-major B keeps at least 128 (64 per CTA, a whole 128-byte swizzle row).
int narrow_bn(int n, bool b_mn) {
  if (n <= 64 && !b_mn) return 64;
  if (n <= 128) return 128;
  return kBN;
}

// K extension of a row-grouped GEMM by the adapter term: A2 [P, r] (K-major),
// and B2 either K-major [E * b_rows, r] (forward kinds, the base B's rows) or
// MN-major [E * r, N] (dgrad kinds: K rows = the adapter rank). Columns of A2
// past r read as zeros (out of the map), so B2 rows past r multiply zeros.
bool set_lora_ext(GemmParams& g, const moe_bf16* A2, int64_t P, const moe_bf16* B2, int E, int r, bool b_mn,
                  int b_rows_or_n) {
  if (!make_map(&g.tmA2, A2, r, P, 64, 128)) return false;
  if (b_mn) {
    if (!make_map(&g.tmB2, B2, b_rows_or_n, static_cast<uint64_t>(E) * r, 64, 64)) return false;
    g.b_rows2 = r;
  } else {
    if (!make_map(&g.tmB2, B2, r, static_cast<uint64_t>(E) * b_rows_or_n, 64, 128)) return false;
    g.b_rows2 = b_rows_or_n;
  }
  g.nkb2 = cdiv(r, kBK);
  return true;
}

bool shape_ok(int T, int E, int k) {
  return T >= 0 && k >= 1 && E >= k && E <= kMaxExperts && static_cast<int64_t>(T) * k < (int64_t(1) << 31);
}
bool dims_ok(int H) { return H > 0 && H % 8 == 0; }

struct BwdLayout {
  size_t dYp, dGU, hw, dXp, dw_part, maps, gu, V_d, V_gu, Zw_d, total;
};
// gather: the GEMMs read dY (and X) rows by token, so there is no dYp copy.
// lora_r > 0: room for the adapter terms V_d, V_gu, w * Z_d [P, r] and the
// tensor maps of the four adapter-gradient GEMMs.
BwdLayout bwd_layout(int T, int E, int k, int H, int I, bool recompute, bool gather = false, int lora_r = 0) {
  const size_t P = static_cast<size_t>(T) * k;
  BwdLayout L;
  size_t off = 0;
  L.dYp = off; off += gather ? 0 : round256(P * H * 2);
  L.dGU = off; off += round256(P * 2 * I * 2);
  L.hw = off; off += round256(P * I * 2);
  L.dXp = off; off += round256(P * H * 2);
  L.dw_part = off; off += round256(P * kDwSlotsPerNTile * cdiv(I, kBN) * 4);
  L.maps = off; off += round256(static_cast<size_t>(lora_r > 0 ? 12 : 4) * E * sizeof(CUtensorMap));
  L.gu = off; off += recompute ? round256(P * 2 * I * 2) : 0;
  const size_t zr = lora_r > 0 ? round256(P * lora_r * 2) : 0;
  L.V_d = off; off += zr;
  L.V_gu = off; off += zr;
  L.Zw_d = off; off += zr;
  L.total = off;
  return L;
}

// ------------------------------------------------------------ router Linear
static_assert(kRgMaxSplitsLogits <= kRouteMaxParts, "the routing kernel sums at most kRouteMaxParts partials");
inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Workspace of moe_router_fwd / moe_router_bwd: the bf16 terms of W_r
// [3E, H], those of dlogits [3T, E8] (rows padded to E8 = E rounded up to 8,
// so that rows start on 16 bytes) and the fp32 split-K partials (at most
// kRgMaxSplitsLogits x [T, E8] for the logits, kRgMaxSplitsWgrad x [E, H] for
// dW_r).
struct RouterLayout {
  size_t w3, dl3, part, total;
};
RouterLayout router_layout(int T, int H, int E) {
  const size_t E8 = static_cast<size_t>(round_up(E, 8));
  RouterLayout L;
  size_t off = 0;
  L.w3 = off; off += round256(size_t(3) * E * H * 2);
  L.dl3 = off; off += round256(size_t(3) * T * E8 * 2);
  const size_t part_fwd = size_t(kRgMaxSplitsLogits) * T * E8 * 4;
  const size_t part_bwd = size_t(kRgMaxSplitsWgrad) * E * H * 4;
  L.part = off; off += round256(part_fwd > part_bwd ? part_fwd : part_bwd);
  L.total = off;
  return L;
}

bool router_shape_ok(int T, int H, int E) {
  return T >= 0 && E >= 1 && E <= kMaxExperts && dims_ok(H) && 3 * static_cast<int64_t>(T) < (int64_t(1) << 31);
}

// CTAs of a router GEMM that fit on one SM (shared memory and TMEM).
int router_residency(int bn, int stages) {
  const size_t per = rg_smem_bytes(bn, stages) + 1024;  // + the per-CTA reservation
  int r = static_cast<int>((228 * 1024) / per);
  const int tmem = 512 / (2 * rg_tmem_cols(bn));  // two accumulator buffers per CTA
  if (r > tmem) r = tmem;
  return r < 1 ? 1 : r;
}

// Split-K count: about kRouterUnitsPerCta units for every resident CTA slot
// of the (persistent) device grid, at most `cap`, never more splits than K
// blocks.
#ifndef MOE_ROUTER_UNITS_PER_CTA
#define MOE_ROUTER_UNITS_PER_CTA 4
#endif
constexpr int kRouterUnitsPerCta = MOE_ROUTER_UNITS_PER_CTA;
int router_splits(int64_t tiles, int k_blocks, int cap, int slots) {
  const int64_t want = static_cast<int64_t>(slots) * kRouterUnitsPerCta;
  int64_t s = (want + tiles - 1) / tiles;
  if (s > cap) s = cap;
  if (s > k_blocks) s = k_blocks;
  return s < 1 ? 1 : static_cast<int>(s);
}

// Persistent grid: every resident CTA slot of the device, no more than the
// units.
template <int KIND>
int launch_router_gemm(const RouterGemmParams& p, cudaStream_t s, int slot, int num_sms) {
  const size_t smem = rg_smem_bytes(p.bn, p.stages);
  if (cudaFuncSetAttribute(router_gemm_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  ProfScope ps(slot, s);
  const int64_t units = static_cast<int64_t>(p.m_tiles) * p.n_tiles * p.splits;
  const int64_t slots = static_cast<int64_t>(num_sms) * router_residency(p.bn, p.stages);
  const int64_t grid = units < slots ? units : slots;
  if (launch_pdl(router_gemm_kernel<KIND>, dim3(static_cast<unsigned>(grid)), dim3(kRgThreads), smem, s, p) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_status();
}


int launch_split3(const float* src, int64_t rows, int cols, int src_ld, int dst_ld, int64_t term_rows,
                  uint16_t* dst, int num_sms, cudaStream_t s, int slot) {
  const int64_t n = rows * cols;
  if (n == 0) return MOE_OK;
  int64_t blocks = (n + 255) / 256;
  if (blocks > int64_t(num_sms) * 8) blocks = int64_t(num_sms) * 8;
  ProfScope ps(slot, s);
  if (launch_pdl(split3_bf16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, src, rows, cols, src_ld,
                 dst_ld, term_rows, dst) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_status();
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_str(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
    default: return "MOE_ERR_UNKNOWN";
  }
}

unsigned long long moe_launch_count(void) { return launch_count().load(std::memory_order_relaxed); }

int moe_last_device_status(moe_stream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  const int zero = 0;
  if (v != 0 && cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  return v;
}

int moe_route(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w, float* probs,
              moe_stream_t stream) {
  if (!shape_ok(T, E, k)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!ok_ptr(logits) || !ok_ptr(topk_idx) || !ok_ptr(topk_w) || !ok_opt(probs)) return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  ProfScope ps(kProfRoute, stream);
  if (launch_route(logits, T, E, k, topk_idx, topk_w, probs, stream) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

size_t moe_permute_workspace_bytes(int T, int E, int k) {
  if (!shape_ok(T, E, k)) return 0;
  const int64_t P = static_cast<int64_t>(T) * k;
  return round256(static_cast<size_t>(perm_num_chunks(P)) * E * 4);
}

int moe_permute(const int32_t* topk_idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                int32_t* sorted_pair, int32_t* pair_pos, const moe_bf16* X, int H, moe_bf16* Xp, void* ws,
                size_t ws_bytes, moe_stream_t stream) {
  if (!shape_ok(T, E, k)) return MOE_ERR_INVALID_ARG;
  if (!ok_ptr(counts) || !ok_ptr(offsets)) return MOE_ERR_INVALID_ARG;
  const bool gather = (X != nullptr || Xp != nullptr);
  if (gather && (!dims_ok(H) || (T > 0 && (!ok_ptr(X) || !ok_ptr(Xp))))) return MOE_ERR_INVALID_ARG;
  const int64_t P = static_cast<int64_t>(T) * k;
  if (P > 0 && (!ok_ptr(topk_idx) || !ok_ptr(sorted_pair) || !ok_ptr(pair_pos))) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_permute_workspace_bytes(T, E, k);
  if (ws_bytes < need || (need > 0 && !ok_ptr(ws))) return MOE_ERR_WORKSPACE;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  if (P == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  const int nchunks = perm_num_chunks(P);
  int* chunk_hist = static_cast<int*>(ws);
  const size_t hist_smem = sizeof(int) * kPermWarps * E;
  {
    ProfScope ps(kProfPermCount, stream);
    if (launch_pdl(permute_count_kernel, dim3(nchunks), dim3(kPermThreads), hist_smem, stream, topk_idx, P, E,
                   chunk_hist) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  {
    ProfScope ps(kProfPermScan, stream);
    if (launch_pdl(permute_scan_kernel, dim3(1), dim3(1024), 0, stream, chunk_hist, nchunks, E, counts, offsets) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  {
    ProfScope ps(kProfPermScatter, stream);
    if (launch_pdl(permute_scatter_kernel, dim3(nchunks), dim3(kPermThreads), hist_smem, stream, topk_idx, P, E,
                   static_cast<const int*>(chunk_hist), static_cast<const int32_t*>(offsets), sorted_pair,
                   pair_pos) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (gather) {
    ProfScope ps(kProfGatherX, stream);
    const int64_t want = (P + 7) / 8;
    const int blocks = static_cast<int>(want < dev->num_sms * 16 ? want : dev->num_sms * 16);
    if (launch_pdl(gather_rows_kernel, dim3(blocks), dim3(256), 0, stream, reinterpret_cast<const uint4*>(X),
                   static_cast<const int32_t*>(pair_pos), P, k, H / 8, reinterpret_cast<uint4*>(Xp)) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

size_t moe_route_permute_workspace_bytes(int T, int E, int k) {
  if (!shape_ok(T, E, k)) return 0;
  return round256(static_cast<size_t>(route_hist_chunks(T)) * route_hist_ld(E));
}

int moe_route_permute(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w, float* probs,
                      int32_t* counts, int32_t* offsets, int32_t* sorted_pair, int32_t* pair_pos, const moe_bf16* X,
                      int H, moe_bf16* Xp, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!shape_ok(T, E, k)) return MOE_ERR_INVALID_ARG;
  if (!ok_ptr(counts) || !ok_ptr(offsets)) return MOE_ERR_INVALID_ARG;
  const bool gather = (X != nullptr || Xp != nullptr);
  if (gather && (!dims_ok(H) || (T > 0 && (!ok_ptr(X) || !ok_ptr(Xp))))) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!ok_ptr(logits) || !ok_ptr(topk_idx) || !ok_ptr(topk_w) || !ok_opt(probs) ||
                !ok_ptr(sorted_pair) || !ok_ptr(pair_pos)))
    return MOE_ERR_INVALID_ARG;
  const size_t need = moe_route_permute_workspace_bytes(T, E, k);
  if (ws_bytes < need || (need > 0 && !ok_ptr(ws))) return MOE_ERR_WORKSPACE;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  uint8_t* hist8 = static_cast<uint8_t*>(ws);
  {
    ProfScope ps(kProfRouteHist, stream);
    if (launch_route_hist(logits, T, E, k, topk_idx, topk_w, probs, hist8, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  {
    ProfScope ps(kProfPermScanScatter, stream);
    const int nchunks = route_hist_chunks(T);
    const size_t smem = scan_scatter_smem(E);
    // always opted in: the kernel's static shared memory comes on top of this
    if (cudaFuncSetAttribute(permute_scan_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (launch_pdl(permute_scan_scatter_kernel, dim3(cdiv(nchunks, kScanScatterWarps)), dim3(kScanScatterThreads),
                   smem, stream, static_cast<const uint8_t*>(hist8), route_hist_ld(E), nchunks,
                   static_cast<const int32_t*>(topk_idx), T, E, k, counts, offsets, sorted_pair,
                   pair_pos) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (gather) {
    ProfScope ps(kProfGatherX, stream);
    const int64_t P = static_cast<int64_t>(T) * k;
    const int64_t want = (P + 7) / 8;
    const int blocks = static_cast<int>(want < dev->num_sms * 16 ? want : dev->num_sms * 16);
    if (launch_pdl(gather_rows_kernel, dim3(blocks), dim3(256), 0, stream, reinterpret_cast<const uint4*>(X),
                   static_cast<const int32_t*>(pair_pos), P, k, H / 8, reinterpret_cast<uint4*>(Xp)) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// moe_permute_noalloc: moe_permute for callers that cannot allocate device
// memory. Some callers have no way to obtain device scratch: a host program
// or plug-in that links only this C library and holds no device allocator,
// or code running where a device allocation would stall or is not allowed
// (cudaMalloc synchronises the device). This entry point takes its scratch
// from a fixed, file-scope device array instead of the caller's workspace.
//
// The array is a module global: every GPU that loads this library holds its
// 1 MiB until the process exits. All calls share it, so calls whose
// executions overlap on the GPU (different streams, or different host threads
// on one device) race on it; one stream at a time is safe because the
// kernels of one call finish before the next call's kernels start. The
// histogram pass overwrites every element it later reads, so the contents
// left by the previous call never need clearing.
constexpr int kNoAllocPermuteScratchInts = 262144;  // 1 MiB
static __device__ __align__(256) int g_permute_scratch[kNoAllocPermuteScratchInts];

namespace {
// Device address of g_permute_scratch for each device, looked up on the first
// call made with that device current (host code may not use the symbol's name
// as a device pointer).
int* g_permute_scratch_ptr[kMaxDevices] = {};
std::mutex g_permute_scratch_mu;

int permute_scratch_device_ptr(int** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_permute_scratch_mu);
  if (g_permute_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_permute_scratch_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_permute_scratch_ptr[dev];
  return MOE_OK;
}
}  // namespace

int moe_permute_noalloc(const int32_t* topk_idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                        int32_t* sorted_pair, int32_t* pair_pos, const moe_bf16* X, int H, moe_bf16* Xp,
                        moe_stream_t stream) {
  if (!shape_ok(T, E, k)) return MOE_ERR_INVALID_ARG;
  const size_t need = moe_permute_workspace_bytes(T, E, k);
  if (need > sizeof(int) * static_cast<size_t>(kNoAllocPermuteScratchInts)) return MOE_ERR_WORKSPACE;
  int* scratch = nullptr;
  if (int st = permute_scratch_device_ptr(&scratch)) return st;
  return moe_permute(topk_idx, T, E, k, counts, offsets, sorted_pair, pair_pos, X, H, Xp, scratch,
                     sizeof(int) * static_cast<size_t>(kNoAllocPermuteScratchInts), stream);
}

}  // extern "C"

namespace moe {
namespace {
// The two expert GEMMs of the forward. gather: `src` is X [T, H] in token
// order and the gate/up GEMM gathers its rows; otherwise `src` is Xp [P, H].
// lora (optional, permuted rows only): the adapted weights W + scale B A,
// with the adapter activations Z_gu, Z_d written for the backward.
int experts_fwd_impl(const moe_bf16* src, bool gather, const int32_t* offsets, const int32_t* sorted_pair,
                     const float* topk_w, int T, int E, int k, int H, int I, const moe_bf16* W_gu,
                     const moe_bf16* W_d, moe_bf16* h, moe_bf16* gu_save, moe_bf16* O, cudaStream_t stream,
                     const LoraArgs* lora = nullptr) {
  const moe_bf16* Xp = src;
  if (!shape_ok(T, E, k) || !dims_ok(H) || !dims_ok(I)) return MOE_ERR_INVALID_ARG;
  if (lora != nullptr && (gather || !lora_rank_ok(lora->r))) return MOE_ERR_INVALID_ARG;
  const int64_t P = static_cast<int64_t>(T) * k;
  if (P == 0) return MOE_OK;
  if (!ok_ptr(Xp) || !ok_ptr(offsets) || !ok_ptr(sorted_pair) || !ok_opt(topk_w) || !ok_ptr(W_gu) ||
      !ok_ptr(W_d) || !ok_ptr(h) || !ok_opt(gu_save) || !ok_ptr(O))
    return MOE_ERR_INVALID_ARG;
  if (lora != nullptr && (!ok_ptr(lora->A_gu) || !ok_ptr(lora->B_gu) || !ok_ptr(lora->A_d) || !ok_ptr(lora->B_d) ||
                          !ok_ptr(lora->Z_gu) || !ok_ptr(lora->Z_d)))
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  const int tails = tail_ctas(P, E, dev->num_sms);

  // Z = scale * act A^T [P, r]: a plain row-grouped GEMM with N = r whose B
  // is the adapter's A [E * r, K] (K-major)
  auto lora_z = [&](const moe_bf16* act, int K, const moe_bf16* A, moe_bf16* Z, int slot) -> int {
    GemmParams z = base_params(E, P, offsets);
    z.bn = narrow_bn(lora->r, false);
    // K-major B box: bn / 2 rows, the columns each CTA of a pair computes
    if (!make_map(&z.tmA, act, K, P, 64, 128) ||
        !make_map(&z.tmB, A, K, static_cast<uint64_t>(E) * lora->r, 64, static_cast<uint32_t>(z.bn / 2)))
      return MOE_ERR_CUDA;
    z.sorted_pair = sorted_pair;
    z.N = lora->r;
    z.K = K;
    z.I = I;
    z.b_rows = lora->r;
    z.n_tiles = cdiv(lora->r, z.bn);
    z.out = Z;
    z.out_ld = lora->r;
    z.out_scale = lora->scale;
    return launch_gemm<kFwdDown>(z, rowgrouped_grid(P, E, z.n_tiles, dev->num_sms), stream, slot, tails,
                                 dev->num_sms);
  };
  if (lora != nullptr) {
    if (int st = lora_z(Xp, H, lora->A_gu, lora->Z_gu, kProfLoraZGateUp)) return st;
  }

  GemmParams gu = base_params(E, P, offsets);
  if (!make_map(&gu.tmB, W_gu, H, static_cast<uint64_t>(E) * 2 * I, 64, 128)) return MOE_ERR_CUDA;
  if (gather) {
    if (!set_gather(gu, src, sorted_pair, T, k, H)) return MOE_ERR_CUDA;
    gu.tmA = gu.tmB;
  } else if (!make_map(&gu.tmA, Xp, H, P, 64, 128)) {
    return MOE_ERR_CUDA;
  }
  gu.sorted_pair = sorted_pair;
  gu.N = I;
  gu.K = H;
  gu.I = I;
  gu.b_rows = 2 * I;
  gu.n_tiles = cdiv(I, 128);
  gu.out = h;
  gu.out_ld = I;
  gu.gu = gu_save;
  if (lora != nullptr && !set_lora_ext(gu, lora->Z_gu, P, lora->B_gu, E, lora->r, false, 2 * I)) return MOE_ERR_CUDA;
  const int gu_grid = rowgrouped_grid(P, E, gu.n_tiles, dev->num_sms);
  if (int st = gather ? launch_gemm<kFwdGateUp, kGatherA>(gu, gu_grid, stream, kProfFwdGateUp)
                      : launch_gemm<kFwdGateUp>(gu, gu_grid, stream, kProfFwdGateUp, tails, dev->num_sms))
    return st;
  if (lora != nullptr) {
    if (int st = lora_z(h, I, lora->A_d, lora->Z_d, kProfLoraZDown)) return st;
  }

  GemmParams dn = base_params(E, P, offsets);
  if (!make_map(&dn.tmA, h, I, P, 64, 128) || !make_map(&dn.tmB, W_d, I, static_cast<uint64_t>(E) * H, 64, 128))
    return MOE_ERR_CUDA;
  dn.sorted_pair = sorted_pair;
  dn.topk_w = topk_w;
  dn.N = H;
  dn.K = I;
  dn.I = I;
  dn.b_rows = H;
  dn.n_tiles = cdiv(H, kBN);
  dn.out = O;
  dn.out_ld = H;
  if (lora != nullptr && !set_lora_ext(dn, lora->Z_d, P, lora->B_d, E, lora->r, false, H)) return MOE_ERR_CUDA;
  return launch_gemm<kFwdDown>(dn, rowgrouped_grid(P, E, dn.n_tiles, dev->num_sms), stream, kProfFwdDown, tails,
                               dev->num_sms);
}
}  // namespace
}  // namespace moe

extern "C" {

int moe_experts_fwd(const moe_bf16* Xp, const int32_t* offsets, const int32_t* sorted_pair, const float* topk_w,
                    int T, int E, int k, int H, int I, const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* h,
                    moe_bf16* gu_save, moe_bf16* O, moe_stream_t stream) {
  return experts_fwd_impl(Xp, false, offsets, sorted_pair, topk_w, T, E, k, H, I, W_gu, W_d, h, gu_save, O, stream);
}

int moe_experts_fwd_x(const moe_bf16* X, const int32_t* offsets, const int32_t* sorted_pair, const float* topk_w,
                      int T, int E, int k, int H, int I, const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* h,
                      moe_bf16* gu_save, moe_bf16* O, moe_stream_t stream) {
  return experts_fwd_impl(X, true, offsets, sorted_pair, topk_w, T, E, k, H, I, W_gu, W_d, h, gu_save, O, stream);
}

int moe_combine(const moe_bf16* O, const int32_t* pair_pos, int T, int k, int H, moe_bf16* Y, moe_stream_t stream) {
  if (T < 0 || k < 1 || static_cast<int64_t>(T) * k >= (int64_t(1) << 31) || !dims_ok(H)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!ok_ptr(O) || !ok_ptr(pair_pos) || !ok_ptr(Y)) return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  ProfScope ps(kProfCombineY, stream);
  return launch_combine(O, pair_pos, T, k, H, Y, stream, dev->num_sms) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

size_t moe_layer_bwd_workspace_bytes(int T, int E, int k, int H, int I, int recompute_gu) {
  if (!shape_ok(T, E, k) || !dims_ok(H) || !dims_ok(I)) return 0;
  return bwd_layout(T, E, k, H, I, recompute_gu != 0).total;
}

size_t moe_layer_bwd_x_workspace_bytes(int T, int E, int k, int H, int I, int recompute_gu) {
  if (!shape_ok(T, E, k) || !dims_ok(H) || !dims_ok(I)) return 0;
  return bwd_layout(T, E, k, H, I, recompute_gu != 0, true).total;
}

size_t moe_layer_bwd_lora_workspace_bytes(int T, int E, int k, int H, int I, int r, int recompute_gu) {
  if (!shape_ok(T, E, k) || !dims_ok(H) || !dims_ok(I) || !lora_rank_ok(r)) return 0;
  return bwd_layout(T, E, k, H, I, recompute_gu != 0, false, r).total;
}

int moe_experts_fwd_lora(const moe_bf16* Xp, const int32_t* offsets, const int32_t* sorted_pair, const float* topk_w,
                         int T, int E, int k, int H, int I, const moe_bf16* W_gu, const moe_bf16* W_d, int r,
                         float scale, const moe_bf16* A_gu, const moe_bf16* B_gu, const moe_bf16* A_d,
                         const moe_bf16* B_d, moe_bf16* h, moe_bf16* gu_save, moe_bf16* O, moe_bf16* Z_gu,
                         moe_bf16* Z_d, moe_stream_t stream) {
  LoraArgs a;
  a.r = r;
  a.scale = scale;
  a.A_gu = A_gu;
  a.B_gu = B_gu;
  a.A_d = A_d;
  a.B_d = B_d;
  a.Z_gu = Z_gu;
  a.Z_d = Z_d;
  return experts_fwd_impl(Xp, false, offsets, sorted_pair, topk_w, T, E, k, H, I, W_gu, W_d, h, gu_save, O, stream,
                          &a);
}

}  // extern "C"

namespace moe {
namespace {
void set_dw_out(GemmParams& p, void* dW, bool dw_f32, bool accumulate) {
  p.out = dw_f32 ? nullptr : static_cast<uint16_t*>(dW);
  p.out_f32 = dw_f32 ? static_cast<float*>(dW) : nullptr;
  p.accumulate = dw_f32 && accumulate ? 1 : 0;
}

// The layer's backward. gather: `src` is X [T, H] in token order and the
// GEMMs that read X or dY rows gather them (no dYp copy, no gather kernel);
// otherwise `src` is Xp [P, H] and dY is first gathered into dYp.
// dw_f32: dW_gu / dW_d are fp32 (the wgrad accumulators unrounded), else
// bf16; accumulate (fp32 only): dW += the gradient instead of dW = it.
// lora (optional, permuted rows only): backward of the adapted layer; the
// adapter gradients go to lora->dA_* / dB_* (fp32), and dW_gu / dW_d may then
// be NULL (frozen base weights: their GEMMs are skipped).
int layer_bwd_impl(const moe_bf16* dY, const moe_bf16* src, bool gather, const moe_bf16* gu_save,
                   const moe_bf16* h, const float* probs, const int32_t* topk_idx, const float* topk_w,
                   const int32_t* offsets, const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k,
                   int H, int I, const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* dX, void* dW_gu, void* dW_d,
                   bool dw_f32, bool accumulate, float* dlogits, void* ws, size_t ws_bytes, cudaStream_t stream,
                   const LoraArgs* lora = nullptr, bool pair_dw_out = false, float* pair_dw = nullptr) {
  const moe_bf16* Xp = src;
  if (!shape_ok(T, E, k) || !dims_ok(H) || !dims_ok(I)) return MOE_ERR_INVALID_ARG;
  if (lora != nullptr) {
    if (gather || !lora_rank_ok(lora->r) || !ok_opt(dW_gu) || !ok_opt(dW_d)) return MOE_ERR_INVALID_ARG;
    if (!ok_ptr(lora->A_gu) || !ok_ptr(lora->B_gu) || !ok_ptr(lora->A_d) || !ok_ptr(lora->B_d) ||
        !ok_ptr(lora->dA_gu) || !ok_ptr(lora->dB_gu) || !ok_ptr(lora->dA_d) || !ok_ptr(lora->dB_d))
      return MOE_ERR_INVALID_ARG;
  } else if (!ok_ptr(dW_gu) || !ok_ptr(dW_d)) {
    return MOE_ERR_INVALID_ARG;
  }
  if (!ok_ptr(offsets)) return MOE_ERR_INVALID_ARG;
  const int64_t P = static_cast<int64_t>(T) * k;
  // pair_dw_out: the routing-weight gradient of every pair (pair_dw [T*k])
  // is the output in place of the router backward (probs, topk_idx and
  // dlogits unused)
  const bool router = !pair_dw_out;
  if (P > 0 && (!ok_ptr(dY) || !ok_ptr(Xp) || !ok_opt(gu_save) || !ok_opt(h) || !ok_ptr(topk_w) ||
                !ok_ptr(sorted_pair) || !ok_ptr(pair_pos) || !ok_ptr(W_gu) || !ok_ptr(W_d) || !ok_ptr(dX)))
    return MOE_ERR_INVALID_ARG;
  if (P > 0 && (router ? (!ok_ptr(probs) || !ok_ptr(topk_idx) || !ok_ptr(dlogits)) : !ok_ptr(pair_dw)))
    return MOE_ERR_INVALID_ARG;
  if (P > 0 && lora != nullptr && (!ok_ptr(lora->Z_gu) || !ok_ptr(lora->Z_d))) return MOE_ERR_INVALID_ARG;
  (void)h;  // not read: the dgrad-down epilogue recomputes h = silu(g) * u from g|u
  const bool recompute = (gu_save == nullptr);
  const int lora_r = lora != nullptr ? lora->r : 0;
  const BwdLayout L = bwd_layout(T, E, k, H, I, recompute, gather, lora_r);
  if (P > 0 && (ws_bytes < L.total || !ok_ptr(ws))) return MOE_ERR_WORKSPACE;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  const size_t dw_elem = dw_f32 ? 4 : 2;
  const size_t dw_gu_bytes = static_cast<size_t>(E) * 2 * I * H * dw_elem;
  const size_t dw_d_bytes = static_cast<size_t>(E) * H * I * dw_elem;
  if (P == 0) {  // no rows: every expert is empty, all weight gradients are zero (dW += 0 if accumulating)
    if (!accumulate && ((dW_gu != nullptr && cudaMemsetAsync(dW_gu, 0, dw_gu_bytes, stream) != cudaSuccess) ||
                        (dW_d != nullptr && cudaMemsetAsync(dW_d, 0, dw_d_bytes, stream) != cudaSuccess)))
      return MOE_ERR_CUDA;
    if (lora != nullptr && !lora->accumulate) {
      const size_t r = static_cast<size_t>(lora->r), e = static_cast<size_t>(E);
      if (cudaMemsetAsync(lora->dA_gu, 0, e * r * H * 4, stream) != cudaSuccess ||
          cudaMemsetAsync(lora->dB_gu, 0, e * 2 * I * r * 4, stream) != cudaSuccess ||
          cudaMemsetAsync(lora->dA_d, 0, e * r * I * 4, stream) != cudaSuccess ||
          cudaMemsetAsync(lora->dB_d, 0, e * H * r * 4, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
  }
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  moe_bf16* dYp = reinterpret_cast<moe_bf16*>(w8 + L.dYp);
  moe_bf16* dGU = reinterpret_cast<moe_bf16*>(w8 + L.dGU);
  moe_bf16* hw = reinterpret_cast<moe_bf16*>(w8 + L.hw);
  moe_bf16* dXp = reinterpret_cast<moe_bf16*>(w8 + L.dXp);
  float* dw_part = reinterpret_cast<float*>(w8 + L.dw_part);
  const int nt_dgrad_down = cdiv(I, kBN);

  // 1. dYp[r] = dY[token of row r] (the GEMMs gather dY themselves when gather)
  if (!gather) {
    ProfScope ps(kProfGatherDy, stream);
    const int64_t want = (P + 7) / 8;
    const int blocks = static_cast<int>(want < dev->num_sms * 16 ? want : dev->num_sms * 16);
    if (launch_pdl(gather_rows_kernel, dim3(blocks), dim3(256), 0, stream, reinterpret_cast<const uint4*>(dY),
                   static_cast<const int32_t*>(pair_pos), P, k, H / 8, reinterpret_cast<uint4*>(dYp)) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  // 2. g|u when the forward did not keep them
  const moe_bf16* gu = gu_save;
  if (recompute) {
    moe_bf16* gu_ws = reinterpret_cast<moe_bf16*>(w8 + L.gu);
    GemmParams rc = base_params(E, P, offsets);
    if (!make_map(&rc.tmB, W_gu, H, static_cast<uint64_t>(E) * 2 * I, 64, 128)) return MOE_ERR_CUDA;
    if (gather) {
      if (!set_gather(rc, src, sorted_pair, T, k, H)) return MOE_ERR_CUDA;
      rc.tmA = rc.tmB;
    } else if (!make_map(&rc.tmA, Xp, H, P, 64, 128)) {
      return MOE_ERR_CUDA;
    }
    rc.sorted_pair = sorted_pair;
    rc.N = I;
    rc.K = H;
    rc.I = I;
    rc.b_rows = 2 * I;
    rc.n_tiles = cdiv(I, 128);
    rc.out = nullptr;
    rc.gu = gu_ws;
    if (lora != nullptr && !set_lora_ext(rc, lora->Z_gu, P, lora->B_gu, E, lora->r, false, 2 * I)) return MOE_ERR_CUDA;
    const int grid = rowgrouped_grid(P, E, rc.n_tiles, dev->num_sms);
    if (int st = gather ? launch_gemm<kFwdGateUp, kGatherA>(rc, grid, stream, kProfRecomputeGateUp)
                        : launch_gemm<kFwdGateUp>(rc, grid, stream, kProfRecomputeGateUp, tail_ctas(P, E, dev->num_sms), dev->num_sms))
      return st;
    gu = gu_ws;
  }
  // Adapter terms of the dgrad GEMMs: V = scale * act B [P, r], a plain
  // row-grouped GEMM (the dgrad-gate/up kind) whose MN-major B is the
  // adapter's B [E * K, r]. The dgrads then take [V] and the adapter's A as
  // their K extension.
  moe_bf16* V_d = reinterpret_cast<moe_bf16*>(w8 + L.V_d);
  moe_bf16* V_gu = reinterpret_cast<moe_bf16*>(w8 + L.V_gu);
  auto lora_v = [&](const moe_bf16* act, int K, const moe_bf16* Bm, moe_bf16* V, int slot) -> int {
    GemmParams v = base_params(E, P, offsets);
    if (!make_map(&v.tmA, act, K, P, 64, 128) ||
        !make_map(&v.tmB, Bm, lora->r, static_cast<uint64_t>(E) * K, 64, 64))
      return MOE_ERR_CUDA;
    v.N = lora->r;
    v.K = K;
    v.I = I;
    v.b_rows = K;
    v.bn = narrow_bn(lora->r, true);
    v.n_tiles = cdiv(lora->r, v.bn);
    v.out = V;
    v.out_ld = lora->r;
    v.out_scale = lora->scale;
    return launch_gemm<kBwdDgradGateUp>(v, rowgrouped_grid(P, E, v.n_tiles, dev->num_sms), stream, slot,
                                        tail_ctas(P, E, dev->num_sms), dev->num_sms);
  };
  if (lora != nullptr) {
    if (int st = lora_v(dYp, H, lora->B_d, V_d, kProfLoraVDown)) return st;
  }
  // 3. dgrad through down + SwiGLU backward: dGU, hw, partial dw
  {
    GemmParams bd = base_params(E, P, offsets);
    if (!make_map(&bd.tmB, W_d, I, static_cast<uint64_t>(E) * H, 64, 64)) return MOE_ERR_CUDA;
    if (gather) {
      if (!set_gather(bd, dY, sorted_pair, T, k, H)) return MOE_ERR_CUDA;
      bd.tmA = bd.tmB;
    } else if (!make_map(&bd.tmA, dYp, H, P, 64, 128)) {
      return MOE_ERR_CUDA;
    }
    bd.sorted_pair = sorted_pair;
    bd.topk_w = topk_w;
    bd.N = I;
    bd.K = H;
    bd.I = I;
    bd.b_rows = H;
    bd.n_tiles = nt_dgrad_down;
    bd.out = dGU;
    bd.out_ld = 2 * I;
    bd.gu = const_cast<moe_bf16*>(gu);
    bd.hw_out = hw;
    bd.dw_part = dw_part;
    if (lora != nullptr && !set_lora_ext(bd, V_d, P, lora->A_d, E, lora->r, true, I)) return MOE_ERR_CUDA;
    const int grid = rowgrouped_grid(P, E, bd.n_tiles, dev->num_sms);
    if (int st = gather ? launch_gemm<kBwdDgradDown, kGatherA>(bd, grid, stream, kProfDgradDown)
                        : launch_gemm<kBwdDgradDown>(bd, grid, stream, kProfDgradDown, tail_ctas(P, E, dev->num_sms), dev->num_sms))
      return st;
  }
  if (lora != nullptr) {
    if (int st = lora_v(dGU, 2 * I, lora->B_gu, V_gu, kProfLoraVGateUp)) return st;
  }
  // 4. dgrad through gate/up: dXp = dGU W_gu[e]
  {
    GemmParams bx = base_params(E, P, offsets);
    if (!make_map(&bx.tmA, dGU, 2 * I, P, 64, 128) ||
        !make_map(&bx.tmB, W_gu, H, static_cast<uint64_t>(E) * 2 * I, 64, 64))
      return MOE_ERR_CUDA;
    bx.N = H;
    bx.K = 2 * I;
    bx.I = I;
    bx.b_rows = 2 * I;
    bx.n_tiles = cdiv(H, kBN);
    bx.out = dXp;
    bx.out_ld = H;
    if (lora != nullptr && !set_lora_ext(bx, V_gu, P, lora->A_gu, E, lora->r, true, H)) return MOE_ERR_CUDA;
    if (int st = launch_gemm<kBwdDgradGateUp>(bx, rowgrouped_grid(P, E, bx.n_tiles, dev->num_sms), stream,
                                              kProfDgradGateUp, tail_ctas(P, E, dev->num_sms), dev->num_sms))
      return st;
  }
  // 5. dX[t] = sum_j dXp[pair_pos[t*k+j]]
  {
    ProfScope ps(kProfCombineDx, stream);
    if (launch_combine(dXp, pair_pos, T, k, H, dX, stream, dev->num_sms) != cudaSuccess) return MOE_ERR_CUDA;
  }
  // 6. weight gradients, K = the expert's rows. Each launch first writes
  //    per-expert copies of its two tensor maps, clipped at the segment end.
  CUtensorMap* maps = reinterpret_cast<CUtensorMap*>(w8 + L.maps);
  if (dW_gu != nullptr) {
    GemmParams wg = base_params(E, P, offsets);
    if (!make_map(&wg.tmA, dGU, 2 * I, P, 64, 64)) return MOE_ERR_CUDA;
    if (gather) {  // B = X rows by token (its per-expert map copy is unused)
      if (!set_gather(wg, src, sorted_pair, T, k, H)) return MOE_ERR_CUDA;
      wg.tmB = wg.tmA;
    } else if (!make_map(&wg.tmB, Xp, H, P, 64, 64)) {
      return MOE_ERR_CUDA;
    }
    if (launch_pdl(build_expert_maps_kernel, dim3(cdiv(2 * E, 8)), dim3(256), 0, stream, wg.tmA, wg.tmB, offsets, E,
                   maps) != cudaSuccess)
      return MOE_ERR_CUDA;
    wg.expert_maps = maps;
    wg.M = 2 * I;
    wg.N = H;
    wg.I = I;
    wg.m_tiles = cdiv(2 * I, kBM);
    wg.n_tiles = cdiv(H, kBN);
    set_dw_out(wg, dW_gu, dw_f32, accumulate);
    if (!dw_f32 && MOE_WGRAD_TMA_STORE) {  // bf16 dW: full 32 x 32 chunks leave through TMA stores
      if (!make_map(&wg.tmOut, dW_gu, H, static_cast<uint64_t>(E) * 2 * I, 32, 32, 0, CU_TENSOR_MAP_SWIZZLE_64B))
        return MOE_ERR_CUDA;
      wg.out_tma = 1;
    }
    wg.out_ld = H;
    wg.out_expert_stride = static_cast<int64_t>(2) * I * H;
    const int64_t tiles = static_cast<int64_t>(E) * wg.m_tiles * wg.n_tiles;
    const int grid = pair_grid(tiles, dev->num_sms);
    if (int st = gather ? launch_gemm<kBwdWgrad, kGatherB>(wg, grid, stream, kProfWgradGateUp)
                        : launch_gemm<kBwdWgrad>(wg, grid, stream, kProfWgradGateUp))
      return st;
  }
  if (dW_d != nullptr) {
    GemmParams wd = base_params(E, P, offsets);
    if (!make_map(&wd.tmB, hw, I, P, 64, 64)) return MOE_ERR_CUDA;
    if (gather) {  // A = dY rows by token (its per-expert map copy is unused)
      if (!set_gather(wd, dY, sorted_pair, T, k, H)) return MOE_ERR_CUDA;
      wd.tmA = wd.tmB;
    } else if (!make_map(&wd.tmA, dYp, H, P, 64, 64)) {
      return MOE_ERR_CUDA;
    }
    if (launch_pdl(build_expert_maps_kernel, dim3(cdiv(2 * E, 8)), dim3(256), 0, stream, wd.tmA, wd.tmB, offsets, E,
                   maps + 2 * E) != cudaSuccess)
      return MOE_ERR_CUDA;
    wd.expert_maps = maps + 2 * E;
    wd.M = H;
    wd.N = I;
    wd.I = I;
    wd.m_tiles = cdiv(H, kBM);
    wd.n_tiles = cdiv(I, kBN);
    set_dw_out(wd, dW_d, dw_f32, accumulate);
    if (!dw_f32 && MOE_WGRAD_TMA_STORE) {
      if (!make_map(&wd.tmOut, dW_d, I, static_cast<uint64_t>(E) * H, 32, 32, 0, CU_TENSOR_MAP_SWIZZLE_64B))
        return MOE_ERR_CUDA;
      wd.out_tma = 1;
    }
    wd.out_ld = I;
    wd.out_expert_stride = static_cast<int64_t>(H) * I;
    const int64_t tiles = static_cast<int64_t>(E) * wd.m_tiles * wd.n_tiles;
    const int grid = pair_grid(tiles, dev->num_sms);
    if (int st = gather ? launch_gemm<kBwdWgrad, kGatherA>(wd, grid, stream, kProfWgradDown)
                        : launch_gemm<kBwdWgrad>(wd, grid, stream, kProfWgradDown))
      return st;
  }
  // 6b. adapter gradients (fp32): per expert over its rows
  //   dA_gu = V_gu^T Xp, dB_gu = dGU^T Z_gu, dA_d = V_d^T hw, dB_d = dYp^T (w Z_d)
  // (V, Z carry the scale; hw and w Z_d the routing weight), each a weight-
  // gradient GEMM with its own per-expert tensor maps.
  if (lora != nullptr) {
    const int r = lora->r;
    moe_bf16* Zw_d = reinterpret_cast<moe_bf16*>(w8 + L.Zw_d);
    {
      ProfScope ps(kProfLoraWeightRows, stream);
      const int64_t n = P * (r / 8);
      const int blocks = static_cast<int>(cdiv(n, 256) < dev->num_sms * 8 ? cdiv(n, 256) : dev->num_sms * 8);
      if (launch_pdl(lora_weight_rows_kernel, dim3(blocks), dim3(256), 0, stream,
                     reinterpret_cast<const uint4*>(lora->Z_d), sorted_pair, topk_w, P, r / 8,
                     reinterpret_cast<uint4*>(Zw_d)) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    // Each is computed with the rank as its N (narrow tiles): dA as its
    // transpose (Xp^T V_gu, hw^T V_d) stored transposed into [r, K].
    struct Wg {
      const moe_bf16* a;  // [P, M]
      int M;
      const moe_bf16* b;  // [P, N]
      int N;
      float* out;
      int slot;
      bool transposed;
    };
    const Wg jobs[4] = {{Xp, H, V_gu, r, lora->dA_gu, kProfLoraDAGateUp, true},
                        {dGU, 2 * I, lora->Z_gu, r, lora->dB_gu, kProfLoraDBGateUp, false},
                        {hw, I, V_d, r, lora->dA_d, kProfLoraDADown, true},
                        {dYp, H, Zw_d, r, lora->dB_d, kProfLoraDBDown, false}};
    for (int j = 0; j < 4; ++j) {
      const Wg& w = jobs[j];
      GemmParams g = base_params(E, P, offsets);
      if (!make_map(&g.tmA, w.a, w.M, P, 64, 64) || !make_map(&g.tmB, w.b, w.N, P, 64, 64)) return MOE_ERR_CUDA;
      CUtensorMap* m = maps + (4 + 2 * j) * E;
      if (launch_pdl(build_expert_maps_kernel, dim3(cdiv(2 * E, 8)), dim3(256), 0, stream, g.tmA, g.tmB, offsets, E,
                     m) != cudaSuccess)
        return MOE_ERR_CUDA;
      g.expert_maps = m;
      g.M = w.M;
      g.N = w.N;
      g.I = I;
      g.bn = narrow_bn(w.N, true);
      g.m_tiles = cdiv(w.M, kBM);
      g.n_tiles = cdiv(w.N, g.bn);
      g.out_transposed = w.transposed ? 1 : 0;
      g.out_ld = w.transposed ? w.M : w.N;
      g.out_expert_stride = static_cast<int64_t>(w.M) * w.N;
      set_dw_out(g, w.out, true, lora->accumulate);
      const int64_t tiles = static_cast<int64_t>(E) * g.m_tiles * g.n_tiles;
      if (int st = launch_gemm<kBwdWgrad>(g, pair_grid(tiles, dev->num_sms), stream, w.slot)) return st;
    }
  }
  // 7. router logits gradient, or each pair's routing-weight gradient
  if (router) {
    ProfScope ps(kProfRouterBwd, stream);
    if (launch_router_bwd(probs, topk_idx, topk_w, static_cast<const float*>(dw_part), pair_pos,
                          kDwSlotsPerNTile * nt_dgrad_down, static_cast<int64_t>(T), E, k, dlogits, dev->num_sms,
                          stream) != cudaSuccess)
      return MOE_ERR_CUDA;
  } else {
    ProfScope ps(kProfPairDw, stream);
    const int64_t want = (P + 255) / 256;
    const int blocks = static_cast<int>(want < dev->num_sms * 8 ? want : dev->num_sms * 8);
    if (launch_pdl(pair_dw_kernel, dim3(blocks), dim3(256), 0, stream, static_cast<const float*>(dw_part), pair_pos,
                   kDwSlotsPerNTile * nt_dgrad_down, P, pair_dw) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
}  // namespace
}  // namespace moe

extern "C" {

int moe_layer_bwd(const moe_bf16* dY, const moe_bf16* Xp, const moe_bf16* gu_save, const moe_bf16* h,
                  const float* probs, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                  const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k, int H, int I,
                  const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* dX, moe_bf16* dW_gu, moe_bf16* dW_d,
                  float* dlogits, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return layer_bwd_impl(dY, Xp, false, gu_save, h, probs, topk_idx, topk_w, offsets, sorted_pair, pair_pos, T, E, k,
                        H, I, W_gu, W_d, dX, dW_gu, dW_d, false, false, dlogits, ws, ws_bytes, stream);
}

int moe_layer_bwd_pair_dw(const moe_bf16* dY, const moe_bf16* Xp, const moe_bf16* gu_save, const moe_bf16* h,
                          const float* topk_w, const int32_t* offsets, const int32_t* sorted_pair,
                          const int32_t* pair_pos, int T, int E, int k, int H, int I, const moe_bf16* W_gu,
                          const moe_bf16* W_d, moe_bf16* dX, moe_bf16* dW_gu, moe_bf16* dW_d, float* dw, void* ws,
                          size_t ws_bytes, moe_stream_t stream) {
  return layer_bwd_impl(dY, Xp, false, gu_save, h, nullptr, nullptr, topk_w, offsets, sorted_pair, pair_pos, T, E,
                        k, H, I, W_gu, W_d, dX, dW_gu, dW_d, false, false, nullptr, ws, ws_bytes, stream, nullptr,
                        true, dw);
}

int moe_router_bwd_from_dw(const float* dw_rows, const int32_t* pair_pos, const float* probs,
                           const int32_t* topk_idx, const float* topk_w, int T, int E, int k, float* dlogits,
                           moe_stream_t stream) {
  if (!shape_ok(T, E, k)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!ok_ptr(dw_rows) || !ok_ptr(pair_pos) || !ok_ptr(probs) || !ok_ptr(topk_idx) || !ok_ptr(topk_w) ||
      !ok_ptr(dlogits))
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  ProfScope ps(kProfRouterBwd, stream);
  if (launch_router_bwd(probs, topk_idx, topk_w, dw_rows, pair_pos, 1, static_cast<int64_t>(T), E, k, dlogits,
                        dev->num_sms, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_ep_pack_rows(const int32_t* offsets, const int32_t* sorted_pair, const float* topk_w, int T, int E, int k,
                     int experts_per_rank, int32_t* local_expert, float* row_w, moe_stream_t stream) {
  if (!shape_ok(T, E, k) || experts_per_rank < 1 || E % experts_per_rank != 0) return MOE_ERR_INVALID_ARG;
  const int64_t P = static_cast<int64_t>(T) * k;
  if (P == 0) return MOE_OK;
  if (!ok_ptr(offsets) || !ok_ptr(sorted_pair) || !ok_ptr(topk_w) || !ok_ptr(local_expert) || !ok_ptr(row_w))
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  ProfScope ps(kProfEpPack, stream);
  if (launch_pdl(ep_pack_rows_kernel, dim3(E), dim3(256), 0, stream, offsets, sorted_pair, topk_w, P,
                 experts_per_rank, local_expert, row_w) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

int moe_layer_bwd_dw_f32(const moe_bf16* dY, const moe_bf16* Xp, const moe_bf16* gu_save, const moe_bf16* h,
                         const float* probs, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                         const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k, int H, int I,
                         const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* dX, float* dW_gu, float* dW_d,
                         int accumulate, float* dlogits, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return layer_bwd_impl(dY, Xp, false, gu_save, h, probs, topk_idx, topk_w, offsets, sorted_pair, pair_pos, T, E, k,
                        H, I, W_gu, W_d, dX, dW_gu, dW_d, true, accumulate != 0, dlogits, ws, ws_bytes, stream);
}

int moe_layer_bwd_x(const moe_bf16* dY, const moe_bf16* X, const moe_bf16* gu_save, const moe_bf16* h,
                    const float* probs, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                    const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k, int H, int I,
                    const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* dX, moe_bf16* dW_gu, moe_bf16* dW_d,
                    float* dlogits, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return layer_bwd_impl(dY, X, true, gu_save, h, probs, topk_idx, topk_w, offsets, sorted_pair, pair_pos, T, E, k, H,
                        I, W_gu, W_d, dX, dW_gu, dW_d, false, false, dlogits, ws, ws_bytes, stream);
}

int moe_layer_bwd_lora(const moe_bf16* dY, const moe_bf16* Xp, const moe_bf16* gu_save, const moe_bf16* h,
                       const float* probs, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                       const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k, int H, int I,
                       const moe_bf16* W_gu, const moe_bf16* W_d, int r, float scale, const moe_bf16* A_gu,
                       const moe_bf16* B_gu, const moe_bf16* A_d, const moe_bf16* B_d, const moe_bf16* Z_gu,
                       const moe_bf16* Z_d, moe_bf16* dX, float* dA_gu, float* dB_gu, float* dA_d, float* dB_d,
                       int accumulate, moe_bf16* dW_gu, moe_bf16* dW_d, float* dlogits, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  LoraArgs a;
  a.r = r;
  a.scale = scale;
  a.A_gu = A_gu;
  a.B_gu = B_gu;
  a.A_d = A_d;
  a.B_d = B_d;
  a.Z_gu = const_cast<moe_bf16*>(Z_gu);
  a.Z_d = const_cast<moe_bf16*>(Z_d);
  a.dA_gu = dA_gu;
  a.dB_gu = dB_gu;
  a.dA_d = dA_d;
  a.dB_d = dB_d;
  a.accumulate = accumulate != 0;
  return layer_bwd_impl(dY, Xp, false, gu_save, h, probs, topk_idx, topk_w, offsets, sorted_pair, pair_pos, T, E, k,
                        H, I, W_gu, W_d, dX, dW_gu, dW_d, false, false, dlogits, ws, ws_bytes, stream, &a);
}

int moe_layer_bwd_x_dw_f32(const moe_bf16* dY, const moe_bf16* X, const moe_bf16* gu_save, const moe_bf16* h,
                           const float* probs, const int32_t* topk_idx, const float* topk_w, const int32_t* offsets,
                           const int32_t* sorted_pair, const int32_t* pair_pos, int T, int E, int k, int H, int I,
                           const moe_bf16* W_gu, const moe_bf16* W_d, moe_bf16* dX, float* dW_gu, float* dW_d,
                           int accumulate, float* dlogits, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return layer_bwd_impl(dY, X, true, gu_save, h, probs, topk_idx, topk_w, offsets, sorted_pair, pair_pos, T, E, k, H,
                        I, W_gu, W_d, dX, dW_gu, dW_d, true, accumulate != 0, dlogits, ws, ws_bytes, stream);
}

size_t moe_router_workspace_bytes(int T, int H, int E) {
  if (!router_shape_ok(T, H, E)) return 0;
  return router_layout(T, H, E).total;
}

int moe_router_fwd(const moe_bf16* X, const float* W_r, int T, int H, int E, int k, float* logits,
                   int32_t* topk_idx, float* topk_w, float* probs, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!router_shape_ok(T, H, E) || !shape_ok(T, E, k)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!ok_ptr(X) || !ok_ptr(W_r) || !ok_opt(logits) || !ok_ptr(topk_idx) || !ok_ptr(topk_w) || !ok_opt(probs))
    return MOE_ERR_INVALID_ARG;
  const RouterLayout L = router_layout(T, H, E);
  if (ws_bytes < L.total || !ok_ptr(ws)) return MOE_ERR_WORKSPACE;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* w3 = reinterpret_cast<uint16_t*>(w + L.w3);
  float* part = reinterpret_cast<float*>(w + L.part);
  const int E8 = round_up(E, 8);
  if (int st = launch_split3(W_r, E, H, H, H, E, w3, dev->num_sms, stream, kProfRouterSplitW)) return st;

  RouterGemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = T;
  p.N = E;
  p.bn = E < 256 ? round_up(E, 16) : 256;
  p.stages = kRgMaxStages;
  p.m_tiles = cdiv(T, kRgBM);
  p.n_tiles = cdiv(E, p.bn);
  p.nkb = cdiv(H, kRgBK);
  p.n_terms = 3;
  p.term_rows_b = E;
  p.splits = router_splits(int64_t(p.m_tiles) * p.n_tiles, 3 * p.nkb, kRgMaxSplitsLogits,
                           dev->num_sms * router_residency(p.bn, p.stages));
  p.out = part;
  p.out_ld = E8;
  p.out_split_stride = int64_t(T) * E8;
  if (!make_map(&p.tmA, X, H, T, 64, kRgBM) || !make_map(&p.tmB, w3, H, 3 * int64_t(E), 64, p.bn))
    return MOE_ERR_CUDA;
  if (int st = launch_router_gemm<kRgLogits>(p, stream, kProfRouterLogits, dev->num_sms)) return st;
  ProfScope ps(kProfRoute, stream);
  if (launch_route(nullptr, T, E, k, topk_idx, topk_w, probs, stream, part, p.splits, E8, int64_t(T) * E8, logits) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_status();
}

int moe_router_bwd(const float* dlogits, const moe_bf16* X, const float* W_r, int T, int H, int E, float* dW_r,
                   moe_bf16* dX, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!router_shape_ok(T, H, E)) return MOE_ERR_INVALID_ARG;
  if (!ok_opt(dW_r) || !ok_opt(dX)) return MOE_ERR_INVALID_ARG;
  if (dW_r == nullptr && dX == nullptr) return MOE_OK;
  if (T > 0 && (!ok_ptr(dlogits) || (dW_r != nullptr && !ok_ptr(X)) || (dX != nullptr && !ok_ptr(W_r))))
    return MOE_ERR_INVALID_ARG;
  const RouterLayout L = router_layout(T, H, E);
  if (T > 0 && (ws_bytes < L.total || !ok_ptr(ws))) return MOE_ERR_WORKSPACE;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  if (T == 0) {  // no tokens: dW_r = 0, dX is empty
    if (dW_r != nullptr && cudaMemsetAsync(dW_r, 0, sizeof(float) * size_t(E) * H, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* w3 = reinterpret_cast<uint16_t*>(w + L.w3);
  uint16_t* dl3 = reinterpret_cast<uint16_t*>(w + L.dl3);
  float* part = reinterpret_cast<float*>(w + L.part);
  const int E8 = round_up(E, 8);
  if (int st = launch_split3(dlogits, T, E, E, E8, T, dl3, dev->num_sms, stream, kProfRouterSplitDl)) return st;

  if (dW_r != nullptr) {  // dW_r^T [H, E] = X^T dl, split over K = tokens
    RouterGemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.M = H;
    p.N = E;
    p.bn = E < 256 ? round_up(E, 64) : 256;
    p.stages = kRgMaxStages;
    p.m_tiles = cdiv(H, kRgBM);
    p.n_tiles = cdiv(E, p.bn);
    p.nkb = cdiv(T, kRgBK);
    p.n_terms = 3;
    p.term_rows_b = T;
    p.splits = router_splits(int64_t(p.m_tiles) * p.n_tiles, 3 * p.nkb, kRgMaxSplitsWgrad,
                             dev->num_sms * router_residency(p.bn, p.stages));
    p.out = p.splits > 1 ? part : dW_r;
    p.out_ld = H;
    p.out_split_stride = int64_t(E) * H;
    if (!make_map(&p.tmA, X, H, T, 64, 64) || !make_map(&p.tmB, dl3, E, 3 * int64_t(T), 64, 64, E8))
      return MOE_ERR_CUDA;
    if (int st = launch_router_gemm<kRgWgrad>(p, stream, kProfRouterWgrad, dev->num_sms)) return st;
    if (p.splits > 1) {
      const int64_t n = int64_t(E) * H;
      int64_t blocks = (n / 4 + 255) / 256;
      if (blocks > int64_t(dev->num_sms) * 8) blocks = int64_t(dev->num_sms) * 8;
      ProfScope ps(kProfRouterSumSplits, stream);
      if (launch_pdl(sum_splits_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                     static_cast<const float*>(part), p.splits, n, n, dW_r) != cudaSuccess)
        return MOE_ERR_CUDA;
      if (int st = launch_status()) return st;
    }
  }
  if (dX != nullptr) {  // dX [T, H] += dl W_r over the term pairs (0,0), (0,1), (1,0)
    if (int st = launch_split3(W_r, E, H, H, H, E, w3, dev->num_sms, stream, kProfRouterSplitW)) return st;
    RouterGemmParams p;
    std::memset(&p, 0, sizeof(p));
    p.M = T;
    p.N = H;
    p.bn = kRgDgradBN;
    p.stages = kRgMaxStages;
    p.m_tiles = cdiv(T, kRgBM);
    p.n_tiles = cdiv(H, p.bn);
    p.nkb = cdiv(E, kRgBK);
    p.n_terms = 3;
    p.term_rows_a = T;
    p.term_rows_b = E;
    p.splits = 1;
    p.dx = dX;
    p.dx_ld = H;
    if (!make_map(&p.tmA, dl3, E, 3 * int64_t(T), 64, kRgBM, E8) || !make_map(&p.tmB, w3, H, 3 * int64_t(E), 64, 64))
      return MOE_ERR_CUDA;
    if (int st = launch_router_gemm<kRgDgrad>(p, stream, kProfRouterDgrad, dev->num_sms)) return st;
  }
  return MOE_OK;
}

int moe_selftest_wait_timeout(int limit_ms, moe_stream_t stream) {
  if (limit_ms < 1 || limit_ms > 2000) return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev;
  if (int st = current_device_info(&dev)) return st;
  wait_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<unsigned long long>(limit_ms) * 1000000ull);
  launch_count().fetch_add(1, std::memory_order_relaxed);
  return launch_status();
}

int moe_profile_enable(int on) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  g_prof.clear();
  g_prof.on = (on != 0);
  g_prof.only = -1;
  if (on) {
    unsigned long long* base = gemm_clock_base();
    if (base == nullptr || cudaMemset(base, 0, sizeof(unsigned long long) * 2 * kProfSlots) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int moe_profile_read_clock(const char* name, double* sm_mhz) {
  if (name == nullptr || sm_mhz == nullptr) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < kProfSlots; ++i) {
    if (std::strcmp(name, kProfNames[i]) != 0) continue;
    unsigned long long c[kProfSlots][2];
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpyFromSymbol(c, g_gemm_clock, sizeof(c)) != cudaSuccess)
      return MOE_ERR_CUDA;
    *sm_mhz = c[i][1] > 0 ? 1e3 * static_cast<double>(c[i][0]) / static_cast<double>(c[i][1]) : 0.0;
    return MOE_OK;
  }
  return MOE_ERR_INVALID_ARG;
}

int moe_profile_only(const char* name) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  if (name == nullptr) {
    g_prof.only = -1;
    return MOE_OK;
  }
  for (int i = 0; i < kProfSlots; ++i) {
    if (std::strcmp(name, kProfNames[i]) == 0) {
      g_prof.only = i;
      return MOE_OK;
    }
  }
  return MOE_ERR_INVALID_ARG;
}

int moe_profile_read(const char* name, double* total_ms, int* launches) {
  if (name == nullptr || total_ms == nullptr || launches == nullptr) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_prof.mu);
  for (int i = 0; i < kProfSlots; ++i) {
    if (std::strcmp(name, kProfNames[i]) != 0) continue;
    double sum = 0.0;
    for (auto& pr : g_prof.recs[i]) {
      if (cudaEventSynchronize(pr.second) != cudaSuccess) return MOE_ERR_CUDA;
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, pr.first, pr.second) != cudaSuccess) return MOE_ERR_CUDA;
      sum += ms;
    }
    *total_ms = sum;
    *launches = static_cast<int>(g_prof.recs[i].size());
    return MOE_OK;
  }
  return MOE_ERR_INVALID_ARG;
}

const char* moe_profile_kernel_name(int i) { return (i >= 0 && i < kProfSlots) ? kProfNames[i] : nullptr; }

}  // extern "C"
