// grouped_gemm.cu - launches of the grouped expert GEMM (one round's gate/up or down GEMM, or
// the router logits GEMM), optionally carrying the neighbouring round's copy step on extra
// warps, and the host-side tensor-map cache. The GEMM device code is in gemm_sm100.cuh.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "copy_phases.cuh"
#include "gemm_sm100.cuh"
#include "kernels.h"

namespace moe {

namespace gemm {

// Copy work that rides along with a GEMM launch on warps 6..9 ("copy warps"), overlapping
// the tensor-core work: the previous round's combine next to a gate/up GEMM, the next round's
// dispatch next to a down GEMM. It shares no data with the GEMM it rides with.
constexpr int kCopyWarps = 4;
constexpr int kLaunchThreads = kThreads + 32 * kCopyWarps;

enum SideKind : int { kSideNone = 0, kSideDispatch = 1, kSideCombine = 2 };

// The copy warps' accesses carry an L2 evict-first policy (copy_phases.cuh, kStream).
#ifndef MOE_STREAM_SIDE
#define MOE_STREAM_SIDE 1
#endif
constexpr bool kStreamSide = MOE_STREAM_SIDE != 0;
// Columns per lane per pass of a combine on the copy warps (copy_phases.cuh, accumulate_token).
#ifndef MOE_SIDE_LANE_COLS
#define MOE_SIDE_LANE_COLS 16
#endif
constexpr int kSideLaneCols = MOE_SIDE_LANE_COLS;

struct SideArgs {
  int kind;
  int r;                       // round the side work belongs to
  const int32_t* row_start;
  const int32_t* row_token;
  const int32_t* row_dst;
  const uint4* x;              // dispatch
  uint4* buf;
  int vecs;
  copy::CombineArgs comb;      // combine
  int by_rows;
  int32_t* dbg;                // debug bounds checks: the workspace header, else null
  int T;
  long long buf_rows;
};

__device__ __forceinline__ void side_work(const SideArgs& sa) {
  const int cw = blockIdx.x * kCopyWarps + ((threadIdx.x >> 5) - kThreads / 32);
  const int warps = gridDim.x * kCopyWarps;
  if (sa.kind == kSideDispatch) {
    copy::dispatch_rows<kStreamSide>(sa.x, sa.buf, sa.row_token, sa.row_dst, sa.row_start[sa.r],
                                     sa.row_start[sa.r + 1], sa.vecs, cw, warps, sa.dbg, sa.T, sa.buf_rows);
  } else if (sa.kind == kSideCombine) {
    if (sa.by_rows) {
      const int begin = sa.row_start[sa.r], end = sa.row_start[sa.r + 1];
      for (int row = begin + cw; row < end; row += warps) {
        const int t = sa.row_token[row];
        if (sa.dbg != nullptr && (t < 0 || t >= sa.T)) {
          if ((threadIdx.x & 31) == 0) record_bad(sa.dbg, kBadCombineToken, row);
          continue;
        }
        copy::combine_token<kSideLaneCols, kStreamSide>(sa.comb, t, sa.r, sa.row_dst[row]);
      }
    } else {
      for (int t = cw; t < sa.comb.T; t += warps) copy::combine_token<kSideLaneCols, kStreamSide>(sa.comb, t, sa.r);
    }
  }
}

struct KernelArgs {
  int mode;
  int widths[3];
  int width_idx;
  const int32_t* rows;
  int rows_const;
  int groups;
  int num_k_blocks;
  int n_total;
  int b_second_row;
  void* out;
  long long out_group_stride;
  int out_ld;
  const float* bias;
  int n_valid;
  int32_t* status;
  const int32_t* group_row;        // pooled rows (see Phase), or null
  const int32_t* group_row_base;
  int rows_cap;                    // debug bounds checks (see Phase): 0 = unchecked
  int tma_out;                     // CTA-pair form: store through the output map (see Phase)
  const int32_t* group_expert;     // weights of each group (see Phase), or null
  int half_tiles;                  // CTA-pair form: half-height tiles for short last row blocks
};

__global__ void __launch_bounds__(kLaunchThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb0,
                        const __grid_constant__ CUtensorMap tb1, const __grid_constant__ CUtensorMap tb2,
                        const KernelArgs args, const SideArgs side) {
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve(smem_raw);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&ta);
    tma_prefetch_desc(&tb0);
  }
  const uint32_t tmem = setup(s);
  Phase p;
  p.mode = args.mode;
  p.a = &ta;
  p.b[0] = &tb0;
  p.b[1] = &tb1;
  p.b[2] = &tb2;
  for (int i = 0; i < 3; ++i) p.widths[i] = args.widths[i];
  p.width_idx = args.width_idx;
  p.rows = args.rows;
  p.rows_const = args.rows_const;
  p.groups = args.groups;
  p.num_k_blocks = args.num_k_blocks;
  p.n_total = args.n_total;
  p.b_second_row = args.b_second_row;
  p.out = args.out;
  p.out_group_stride = args.out_group_stride;
  p.out_ld = args.out_ld;
  p.bias = args.bias;
  p.n_valid = args.n_valid;
  p.group_row = args.group_row;
  p.group_row_base = args.group_row_base;
  p.rows_cap = args.rows_cap;
  p.dbg = args.rows_cap > 0 ? args.status - kHdrStatus : nullptr;
  p.out_map = nullptr;
  p.group_expert = args.group_expert;
  p.a_rows64 = nullptr;
  p.b_rows64 = nullptr;
  plan_phase(s, p, 0);              // reads only the row counts (plan data)
  __syncthreads();
  // Everything above overlaps the previous kernel; the operands, and the output buffer that
  // earlier kernels of the round may still read, are touched only after it completes.
  grid_dependency_wait();
  pdl_trigger_early();
  Pipe pipe;
  if (threadIdx.x < kThreads)
    run_phase(s, tmem, p, 0, pipe, args.status);
  else
    side_work(side);
  tc_fence_before();
  __syncthreads();
  pdl_trigger_late();               // after every role of this CTA is done
  release_tmem(tmem);
}

// The CTA-pair form (gemm_sm100.cuh, run_phase_pair), launched as clusters of two CTAs: 256 x
// 256 tiles, one B map with 128-row boxes, a fixed width (SwiGLU 128 gate columns, Bf16Out 256);
// ta64 / tb64 are the A operand and the weights with 64-row boxes, read by the half-height tiles
// of a group's short last row block (tb64 by SwiGLU only).
__global__ void __launch_bounds__(kLaunchThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                             const __grid_constant__ CUtensorMap tout, const __grid_constant__ CUtensorMap ta64,
                             const __grid_constant__ CUtensorMap tb64, const KernelArgs args, const SideArgs side,
                             int width) {
  extern __shared__ uint8_t smem_raw[];
  const Smem s = carve(smem_raw);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&ta);
    tma_prefetch_desc(&tb);
    if (args.tma_out) tma_prefetch_desc(&tout);
  }
  const uint32_t tmem = setup_pair(s);
  Phase p;
  p.mode = args.mode;
  p.a = &ta;
  p.b[0] = &tb;
  p.b[1] = &tb;
  p.b[2] = &tb;
  for (int i = 0; i < 3; ++i) p.widths[i] = args.widths[i];
  p.width_idx = 0;
  p.rows = args.rows;
  p.rows_const = args.rows_const;
  p.groups = args.groups;
  p.num_k_blocks = args.num_k_blocks;
  p.n_total = args.n_total;
  p.b_second_row = args.b_second_row;
  p.out = args.out;
  p.out_group_stride = args.out_group_stride;
  p.out_ld = args.out_ld;
  p.bias = args.bias;
  p.n_valid = args.n_valid;
  p.group_row = args.group_row;
  p.group_row_base = args.group_row_base;
  p.rows_cap = args.rows_cap;
  p.dbg = args.rows_cap > 0 ? args.status - kHdrStatus : nullptr;
  p.out_map = args.tma_out ? &tout : nullptr;
  p.group_expert = args.group_expert;
  p.a_rows64 = args.half_tiles ? &ta64 : nullptr;
  p.b_rows64 = args.half_tiles ? &tb64 : nullptr;
  plan_phase_pair(s, p, 0, width);
  __syncthreads();
  grid_dependency_wait();
  pdl_trigger_early();
  Pipe pipe;
  if (threadIdx.x < kThreads)
    run_phase_pair(s, tmem, p, 0, width, blockIdx.x >> 1, gridDim.x >> 1, pipe, args.status);
  else
    side_work(side);
  tc_fence_before();
  __syncthreads();
  pdl_trigger_late();
  release_tmem_pair(tmem);
}

// ------------------------------------------------------------------ tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// box_inner == BK: operand tiles (64 columns, 128-byte swizzle); box_inner == kOutChunkCols: the
// TMA-store epilogue's output chunks (32 columns, 64-byte swizzle).
static cudaError_t encode_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                              uint64_t groups, uint32_t box_rows, uint32_t box_inner) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {inner, rows, groups};
  const cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult res = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          box_inner == BK ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Maps depend only on (pointer, extents, box), which repeat every round and every step,
// so encoded maps are kept in a small direct-mapped cache.
namespace {
struct MapKey {
  const void* base;
  uint64_t inner, rows, groups;
  uint32_t box_rows, box_inner;
  bool operator==(const MapKey& o) const {
    return base == o.base && inner == o.inner && rows == o.rows && groups == o.groups &&
           box_rows == o.box_rows && box_inner == o.box_inner;
  }
};
constexpr int kMapCacheSize = 128;
struct MapCacheEntry {
  bool used = false;
  MapKey key{};
  CUtensorMap map{};
};
MapCacheEntry g_map_cache[kMapCacheSize];
std::mutex g_map_mutex;
}  // namespace

cudaError_t make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                     uint64_t groups, uint32_t box_rows, uint32_t box_inner) {
  const MapKey key{base, inner, rows, groups, box_rows, box_inner};
  const uint64_t h = ((reinterpret_cast<uintptr_t>(base) >> 8) * 0x9E3779B97F4A7C15ull) ^
                     ((inner * 31 + rows) * 131 + groups * 7 + box_rows + box_inner * 3) * 0xC2B2AE3D27D4EB4Full;
  MapCacheEntry& slot = g_map_cache[(h >> 40) % kMapCacheSize];
  std::lock_guard<std::mutex> lock(g_map_mutex);
  if (slot.used && slot.key == key) {
    *map = slot.map;
    return cudaSuccess;
  }
  const cudaError_t e = encode_map(map, base, inner, rows, groups, box_rows, box_inner);
  if (e == cudaSuccess) {
    slot.used = true;
    slot.key = key;
    slot.map = *map;
  }
  return e;
}

// fp32 output map [groups][rows][inner] with box_inner x box_rows x 1 boxes and the 64-byte
// swizzle (box_inner * 4 must be 64): the backward's weight-gradient tiles. Cached like the bf16 maps.
cudaError_t make_map_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t groups,
                         uint32_t box_inner, uint32_t box_rows) {
  const MapKey key{base, inner, rows, groups, box_rows, box_inner | 0x80000000u};
  const uint64_t h = ((reinterpret_cast<uintptr_t>(base) >> 8) * 0x9E3779B97F4A7C15ull) ^
                     ((inner * 31 + rows) * 131 + groups * 7 + box_rows + box_inner * 5 + 1) * 0xC2B2AE3D27D4EB4Full;
  MapCacheEntry& slot = g_map_cache[(h >> 40) % kMapCacheSize];
  std::lock_guard<std::mutex> lock(g_map_mutex);
  if (slot.used && slot.key == key) {
    *map = slot.map;
    return cudaSuccess;
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {inner, rows, groups};
  const cuuint64_t strides[2] = {inner * 4, inner * rows * 4};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult res = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (res != CUDA_SUCCESS) return cudaErrorInvalidValue;
  slot.used = true;
  slot.key = key;
  slot.map = *map;
  return cudaSuccess;
}

// B maps for the candidate widths; a candidate that does not divide the N extent (never chosen
// on the device) repeats the map of the first one that does.
static cudaError_t make_b_maps(CUtensorMap* mb, const void* base, uint64_t inner, uint64_t rows,
                               uint64_t groups, const int* widths, int n_total) {
  int fallback = widths[0];
  for (int i = 0; i < 3; ++i)
    if (widths[i] > 0 && n_total % widths[i] == 0) {
      fallback = widths[i];
      break;
    }
  for (int i = 0; i < 3; ++i) {
    const int w = (widths[i] > 0 && n_total % widths[i] == 0) ? widths[i] : fallback;
    const cudaError_t e = make_map(&mb[i], base, inner, rows, groups, static_cast<uint32_t>(w));
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Host copy of the device's width rule (gemm_sm100.cuh, plan_phase): the widest candidate
// whose tile count reaches the SM count, else the narrowest that divides n_total. Sets the
// chosen index and returns the tile count (the launch then uses min(tiles, SMs) CTAs).
static long long choose_width(const int32_t* n_host, int groups, int rows_const, int n_total,
                              KernelArgs& args) {
  long long mt = 0;
  for (int g = 0; g < groups; ++g) mt += ((n_host ? n_host[g] : rows_const) + BM - 1) / BM;
  int wi = -1, last = -1;
  for (int i = 0; i < 3; ++i) {
    const int w = args.widths[i];
    if (w <= 0 || n_total % w != 0) continue;
    last = i;
    if (mt * (n_total / w) >= num_sms()) {
      wi = i;
      break;
    }
  }
  if (wi < 0) wi = last;
  args.width_idx = wi;
  return wi < 0 ? 0 : mt * (n_total / args.widths[wi]);
}

static cudaError_t run(const CUtensorMap& a, const CUtensorMap* b, const KernelArgs& args, long long tiles,
                       const SideArgs& side, int kind, cudaStream_t stream) {
  if (tiles <= 0 && side.kind == kSideNone) return cudaSuccess;
  static std::atomic<uint64_t> configured{0};   // one bit per device ordinal
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    const cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               kSmemBytes);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  launch_begin(kind, stream);
  // with side work every SM takes part in the copy; otherwise one CTA per tile, at most one per SM
  const int grid = side.kind != kSideNone ? num_sms() : static_cast<int>(tiles < num_sms() ? tiles : num_sms());
  const cudaError_t err = launch_pdl(grouped_gemm_kernel, dim3(grid), dim3(kLaunchThreads), kSmemBytes, stream,
                                     a, b[0], b[1], b[2], args, side);
  launch_end(kind, stream);
  return err;
}

#ifndef MOE_TMA_OUT_GATE_UP
#define MOE_TMA_OUT_GATE_UP 1   // 0: the pair gate/up GEMM stores h with per-thread stores
#endif

#ifndef MOE_GEMM_PAIR
#define MOE_GEMM_PAIR 1   // 0: never use the CTA-pair form
#endif

// Clusters of two that fit on the device at once (one CTA per SM), per device ordinal.
static int pair_clusters() {
  static std::atomic<int> cached[64];
  int dev = 0;
  cudaGetDevice(&dev);
  dev &= 63;
  int v = cached[dev].load();
  if (v > 0) return v;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  cfg.blockDim = dim3(kLaunchThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaFuncSetAttribute(grouped_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, grouped_gemm_pair_kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = -1;   // no pair form on this device
  }
  cached[dev].store(n);
  return n;
}

#ifndef MOE_GEMM_HALF
#define MOE_GEMM_HALF 1   // 0: no half-height tiles; a short last row block takes a 256-row tile
#endif

// Whether a round's GEMM runs in the CTA-pair form: its tiles must keep every cluster busy and
// cover at most 15 % more rows than the 128-row tiles of the single-CTA form (a short last row
// block, at most 128 rows, costs 128 rows with half-height tiles, else 256).
static bool use_pair(const int32_t* n_host, int groups, int n_total, int width) {
  if (!MOE_GEMM_PAIR || n_host == nullptr || n_total % width != 0) return false;
  long long pair_tiles = 0, rows_pair = 0, rows_single = 0;
  for (int g = 0; g < groups; ++g) {
    const long long blocks = (n_host[g] + kPairRows - 1) / kPairRows;
    const long long tail = n_host[g] - (blocks - 1) * kPairRows;
    pair_tiles += blocks;
    rows_pair += blocks * kPairRows - ((MOE_GEMM_HALF && blocks > 0 && tail <= BM) ? BM : 0);
    rows_single += static_cast<long long>((n_host[g] + BM - 1) / BM) * BM;
  }
  pair_tiles *= n_total / width;
  const int clusters = pair_clusters();
  return clusters > 0 && pair_tiles >= clusters && rows_pair * 100 <= rows_single * 115;
}

// a64, b64: the A operand's and the weights' maps with 64-row boxes (half-height tiles; b64 is
// read for SwiGLU only).
static cudaError_t run_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& out, const CUtensorMap& a64,
                            const CUtensorMap& b64, KernelArgs args, int width, const SideArgs& side, int kind,
                            cudaStream_t stream) {
  args.half_tiles = MOE_GEMM_HALF;
  const int clusters = pair_clusters();   // every cluster takes part; the device counts the tiles
  launch_begin(kind, stream);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kLaunchThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = MOE_PDL;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel, a, b, out, a64, b64, args, side, width);
  launch_end(kind, stream);
  return err;
}

}  // namespace gemm

extern const int kGateUpWidths[3] = {128, 64, 32};   // gate columns per tile (MMA N = 2x)
extern const int kDownWidths[3] = {256, 128, 64};

cudaError_t make_gate_up_maps(const uint16_t* buf, const uint16_t* w_gate_up, int E, int C, int d, int F,
                              CUtensorMap* ma, CUtensorMap* mb, bool pooled) {
  // A: [E][C][d] per expert, or pooled [1][E*C][d] (rows located by the group offsets)
  cudaError_t e = pooled ? gemm::make_map(ma, buf, d, static_cast<uint64_t>(E) * C, 1, gemm::BM)
                         : gemm::make_map(ma, buf, d, C, E, gemm::BM);
  if (e != cudaSuccess) return e;
  return gemm::make_b_maps(mb, w_gate_up, d, 2ull * F, E, kGateUpWidths, F);
}

// A round buffer ([E][C][inner] per expert, or pooled [1][E*C][inner]) with 64-row boxes.
static cudaError_t make_rows64_map(CUtensorMap* m, const uint16_t* rows, int inner, int E, int C, bool pooled) {
  return pooled ? gemm::make_map(m, rows, inner, static_cast<uint64_t>(E) * C, 1, gemm::kHalfRows)
                : gemm::make_map(m, rows, inner, C, E, gemm::kHalfRows);
}

cudaError_t make_down_maps(const uint16_t* h, const uint16_t* w_down, int E, int C, int d, int F,
                           CUtensorMap* ma, CUtensorMap* mb, bool pooled) {
  cudaError_t e = pooled ? gemm::make_map(ma, h, F, static_cast<uint64_t>(E) * C, 1, gemm::BM)
                         : gemm::make_map(ma, h, F, C, E, gemm::BM);
  if (e != cudaSuccess) return e;
  return gemm::make_b_maps(mb, w_down, F, d, E, kDownWidths, d);
}

static gemm::SideArgs make_side(const RoundCopy* copy) {
  gemm::SideArgs sd{};
  sd.kind = gemm::kSideNone;
  if (copy == nullptr) return sd;
  sd.kind = copy->combine ? gemm::kSideCombine : gemm::kSideDispatch;
  sd.r = copy->r;
  sd.row_start = copy->row_start;
  sd.row_token = copy->row_token;
  sd.row_dst = copy->row_dst;
  sd.x = reinterpret_cast<const uint4*>(copy->x);
  sd.buf = reinterpret_cast<uint4*>(copy->buf);
  sd.vecs = copy->d / 8;
  sd.comb = copy::CombineArgs{copy->out, copy->y, copy->idx, copy->gate, copy->round, copy->slot,
                              copy->T, copy->k, copy->C, copy->d, copy->row_off,
                              copy->row_off ? copy->row_start : nullptr, copy->E, copy->dbg,
                              static_cast<long long>(copy->E) * copy->C};
  sd.dbg = copy->dbg;
  sd.T = copy->T;
  sd.buf_rows = static_cast<long long>(copy->E) * copy->C;
  sd.by_rows = copy->rows < copy->T ? 1 : 0;
  return sd;
}

cudaError_t launch_gate_up(const uint16_t* buf, const uint16_t* w_gate_up, uint16_t* h,
                           const int32_t* n_dev, const int32_t* n_host, int E, int C, int d, int F,
                           int32_t* status, const RoundCopy* copy, const int32_t* group_row,
                           const int32_t* group_row_base, cudaStream_t stream, int rows_cap) {
  CUtensorMap ma, mb[3];
  cudaError_t e = make_gate_up_maps(buf, w_gate_up, E, C, d, F, &ma, mb, group_row != nullptr);
  if (e != cudaSuccess) return e;
  gemm::KernelArgs a{};
  a.mode = gemm::kSwiGLU;
  for (int i = 0; i < 3; ++i) a.widths[i] = kGateUpWidths[i];
  a.rows = n_dev;
  a.groups = E;
  a.num_k_blocks = d / gemm::BK;
  a.n_total = F;
  a.b_second_row = F;
  a.out = h;
  a.out_group_stride = static_cast<long long>(C) * F;
  a.out_ld = F;
  a.status = status;
  a.group_row = group_row;
  a.group_row_base = group_row_base;
  a.rows_cap = rows_cap;
  if (gemm::use_pair(n_host, E, F, 128)) {   // mb[0]: 128-row boxes of W1 and of W3
    CUtensorMap mo{};
    a.tma_out = MOE_TMA_OUT_GATE_UP && group_row == nullptr;   // per-expert h [E][C][F]: stored by TMA
    if (a.tma_out && (e = gemm::make_map(&mo, h, F, C, E, 32, gemm::kOutChunkCols)) != cudaSuccess) return e;
    CUtensorMap ma64, mb64;   // 64-row boxes of the rows and of W1 / W3 (half-height tiles)
    if ((e = make_rows64_map(&ma64, buf, d, E, C, group_row != nullptr)) != cudaSuccess ||
        (e = gemm::make_map(&mb64, w_gate_up, d, 2ull * F, E, gemm::kHalfRows)) != cudaSuccess)
      return e;
    return gemm::run_pair(ma, mb[0], mo, ma64, mb64, a, 128, make_side(copy), kKindGateUp, stream);
  }
  const long long tiles = gemm::choose_width(n_host, E, 0, F, a);
  return gemm::run(ma, mb, a, tiles, make_side(copy), kKindGateUp, stream);
}

cudaError_t launch_down(const uint16_t* h, const uint16_t* w_down, uint16_t* out, const int32_t* n_dev,
                        const int32_t* n_host, int E, int C, int d, int F, int32_t* status,
                        const RoundCopy* copy, const int32_t* group_row, const int32_t* group_row_base,
                        cudaStream_t stream, int rows_cap) {
  CUtensorMap ma, mb[3];
  cudaError_t e = make_down_maps(h, w_down, E, C, d, F, &ma, mb, group_row != nullptr);
  if (e != cudaSuccess) return e;
  gemm::KernelArgs a{};
  a.mode = gemm::kBf16Out;
  for (int i = 0; i < 3; ++i) a.widths[i] = kDownWidths[i];
  a.rows = n_dev;
  a.groups = E;
  a.num_k_blocks = F / gemm::BK;
  a.n_total = d;
  a.out = out;
  a.out_group_stride = static_cast<long long>(C) * d;
  a.out_ld = d;
  a.status = status;
  a.group_row = group_row;
  a.group_row_base = group_row_base;
  a.rows_cap = rows_cap;
  if (gemm::use_pair(n_host, E, d, gemm::kPairBn)) {   // each CTA loads 128 of the tile's 256 W2 rows
    CUtensorMap mb_half, mo{};
    if ((e = gemm::make_map(&mb_half, w_down, F, d, E, gemm::kPairBHalf)) != cudaSuccess) return e;
    a.tma_out = group_row == nullptr;          // per-expert out [E][C][d]: stored by TMA
    if (a.tma_out && (e = gemm::make_map(&mo, out, d, C, E, 32, gemm::kOutChunkCols)) != cudaSuccess) return e;
    CUtensorMap ma64;   // 64-row boxes of h (half-height tiles)
    if ((e = make_rows64_map(&ma64, h, F, E, C, group_row != nullptr)) != cudaSuccess) return e;
    return gemm::run_pair(ma, mb_half, mo, ma64, mb_half, a, gemm::kPairBn, make_side(copy), kKindDown, stream);
  }
  const long long tiles = gemm::choose_width(n_host, E, 0, d, a);
  return gemm::run(ma, mb, a, tiles, make_side(copy), kKindDown, stream);
}

cudaError_t launch_ep_experts(const uint16_t* recv, const uint16_t* w_gate_up, const uint16_t* w_down, uint16_t* h,
                              uint16_t* out, int groups, const int32_t* rows_dev, const int32_t* rows_host,
                              const int32_t* group_row_dev, const int32_t* group_expert_dev, long long buf_rows,
                              int E_local, int d, int F, int32_t* status, cudaStream_t stream) {
  // gate/up: h[rows of group g] = bf16(silu(recv W1_e^T) * (recv W3_e^T)), e = group_expert[g]
  CUtensorMap ma, mb[3];
  cudaError_t e = gemm::make_map(&ma, recv, d, static_cast<uint64_t>(buf_rows), 1, gemm::BM);
  if (e != cudaSuccess) return e;
  if ((e = gemm::make_b_maps(mb, w_gate_up, d, 2ull * F, E_local, kGateUpWidths, F)) != cudaSuccess) return e;
  gemm::KernelArgs a{};
  a.mode = gemm::kSwiGLU;
  for (int i = 0; i < 3; ++i) a.widths[i] = kGateUpWidths[i];
  a.rows = rows_dev;
  a.groups = groups;
  a.num_k_blocks = d / gemm::BK;
  a.n_total = F;
  a.b_second_row = F;
  a.out = h;
  a.out_ld = F;
  a.status = status;
  a.group_row = group_row_dev;        // groups are packed from row 0: group 0 starts at offset 0,
  a.group_row_base = group_row_dev;   // so its entry doubles as the base
  a.group_expert = group_expert_dev;
  const gemm::SideArgs none = make_side(nullptr);
  if (gemm::use_pair(rows_host, groups, F, 128)) {
    CUtensorMap unused{}, ma64, mb64;
    if ((e = gemm::make_map(&ma64, recv, d, static_cast<uint64_t>(buf_rows), 1, gemm::kHalfRows)) != cudaSuccess ||
        (e = gemm::make_map(&mb64, w_gate_up, d, 2ull * F, E_local, gemm::kHalfRows)) != cudaSuccess)
      return e;
    e = gemm::run_pair(ma, mb[0], unused, ma64, mb64, a, 128, none, kKindGateUp, stream);
  } else {
    const long long tiles = gemm::choose_width(rows_host, groups, 0, F, a);
    e = gemm::run(ma, mb, a, tiles, none, kKindGateUp, stream);
  }
  if (e != cudaSuccess) return e;
  // down: out[rows of group g] = bf16(h W2_e^T)
  if ((e = gemm::make_map(&ma, h, F, static_cast<uint64_t>(buf_rows), 1, gemm::BM)) != cudaSuccess) return e;
  gemm::KernelArgs b{};
  b.mode = gemm::kBf16Out;
  for (int i = 0; i < 3; ++i) b.widths[i] = kDownWidths[i];
  b.rows = rows_dev;
  b.groups = groups;
  b.num_k_blocks = F / gemm::BK;
  b.n_total = d;
  b.out = out;
  b.out_ld = d;
  b.status = status;
  b.group_row = group_row_dev;
  b.group_row_base = group_row_dev;
  b.group_expert = group_expert_dev;
  if (gemm::use_pair(rows_host, groups, d, gemm::kPairBn)) {
    CUtensorMap mb_half, unused{};
    if ((e = gemm::make_map(&mb_half, w_down, F, d, E_local, gemm::kPairBHalf)) != cudaSuccess) return e;
    CUtensorMap ma64;
    if ((e = gemm::make_map(&ma64, h, F, static_cast<uint64_t>(buf_rows), 1, gemm::kHalfRows)) != cudaSuccess) return e;
    return gemm::run_pair(ma, mb_half, unused, ma64, mb_half, b, gemm::kPairBn, none, kKindDown, stream);
  }
  if ((e = gemm::make_b_maps(mb, w_down, F, d, E_local, kDownWidths, d)) != cudaSuccess) return e;
  const long long tiles = gemm::choose_width(rows_host, groups, 0, d, b);
  return gemm::run(ma, mb, b, tiles, none, kKindDown, stream);
}

cudaError_t launch_router_gemm(const uint16_t* x, const uint16_t* w_router, const float* bias,
                               float* logits, int T, int d, int E, int32_t* status,
                               cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int bn = E <= 64 ? 64 : E <= 128 ? 128 : 256;
  CUtensorMap ma, mb[3];
  cudaError_t e = gemm::make_map(&ma, x, d, T, 1, gemm::BM);
  if (e != cudaSuccess) return e;
  const int widths[3] = {bn, 0, 0};
  if ((e = gemm::make_b_maps(mb, w_router, d, E, 1, widths, bn)) != cudaSuccess) return e;
  gemm::KernelArgs a{};
  a.mode = gemm::kF32Bias;
  a.widths[0] = bn;
  a.rows = nullptr;
  a.rows_const = T;
  a.groups = 1;
  a.num_k_blocks = d / gemm::BK;
  a.n_total = bn;
  a.n_valid = E;
  a.out = logits;
  a.out_ld = E;
  a.bias = bias;
  a.status = status;
  const long long tiles = gemm::choose_width(nullptr, 1, T, bn, a);
  return gemm::run(ma, mb, a, tiles, make_side(nullptr), kKindRouterGemm, stream);
}

}  // namespace moe
