// grouped_gemm.cu - the expert GEMMs of one round on the 5th-generation tensor cores.
//
// "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, item on reducing
// per-expert overhead [section "Reducing per-expert overhead"]: the experts of a group
// run as one grouped GEMM. Here one launch covers every expert that has rows in the
// round; each expert e multiplies its n[r][e] rows of the fixed [E, C, d] round buffer.
//
// Kernel shape (one persistent CTA per SM, 192 threads, warp-specialised):
//   warp 0      TMA producer: 3-D tiled loads (128-byte swizzle) of the A tile
//               (128 rows x 64 K) and the B tile into a ring of shared-memory stages.
//   warp 1      MMA issuer: one thread issues tcgen05.mma (kind::f16, bf16 x bf16 ->
//               fp32, M=128, N=BN, K=16) into a TMEM accumulator; tcgen05.commit frees
//               each stage and, after the last K block, hands the accumulator over.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator rows (warp w reads TMEM lanes
//               32*(w%4) .. +31), then the mode's math and 16-byte global stores.
// Two TMEM accumulators alternate, so the epilogue of tile i overlaps the main loop of
// tile i+1. Tiles are (expert, 128-row block, N block), enumerated from the device-side
// row counts, so empty experts cost nothing and the host needs no synchronisation.
//
// Modes:
//   SwiGLU  (gate/up): B holds BN/2 rows of W1 (gate) and the same BN/2 rows of W3 (up),
//           loaded as two boxes into one B tile, so one MMA of width BN computes both
//           halves; the epilogue writes bf16(silu(gate) * up).
//   Bf16Out (down):    bf16(A W2^T).
//   F32Bias (router):  fp32 A W_r^T + bias, for logits = x W_r^T + b.
//
// Rows of a tile beyond the expert's n[r][e] read stale buffer rows or TMA zero fill;
// they only reach accumulator rows that are never stored (an MMA row depends on its own
// A row only). No TMA multicast is used anywhere.
#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>
#include <mutex>

#include "kernels.h"
#include "sm100.cuh"

namespace moe {

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 64;       // bf16 elements in one 128-byte swizzle row
constexpr int UMMA_K = 16;
constexpr int kThreads = 192;
constexpr int kStageBudget = 192 * 1024;

enum Mode : int { kSwiGLU = 0, kBf16Out = 1, kF32Bias = 2 };

struct GemmArgs {
  const int32_t* rows;        // [groups] valid rows of each group (device), or nullptr
  int rows_const;             // rows of every group when rows == nullptr
  int groups;
  int num_k_blocks;           // K / 64
  int n_tiles;                // N blocks per (group, 128-row block)
  int b_second_row;           // SwiGLU: first row of the up projection inside B (= d_ff)
  int n_valid;                // F32Bias: valid output columns
  void* out;
  long long out_group_stride; // elements between groups of the output
  int out_ld;                 // elements between output rows
  const float* bias;          // F32Bias
  int32_t* status;            // workspace status word
};

template <int BN>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (kStageBudget / STAGE_BYTES) > 8 ? 8 : (kStageBudget / STAGE_BYTES);
  static constexpr int TMEM_COLS = 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 2 * BN <= 128 ? 128
                                                     : 2 * BN <= 256 ? 256 : 512;
  static constexpr int BAR_BYTES = (2 * STAGES + 5) * 8;
  static constexpr int MISC_BYTES = 16 + (MOE_MAX_E_PLAN + 1) * 4;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + MISC_BYTES;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float silu_f(float a) { return a / (1.0f + __expf(-a)); }

template <int MODE, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB, const GemmArgs args) {
  using Cf = Cfg<BN>;
  constexpr int S = Cf::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * Cf::STAGE_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* tile_start = reinterpret_cast<int*>(tmem_holder + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_addr(&full[s]), 1);
      mbar_init(smem_addr(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_addr(&tfull[a]), 1);
      mbar_init(smem_addr(&tempty[a]), 128);
    }
    mbar_init(smem_addr(drain), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
    // Tile enumeration: prefix over groups of ceil(rows / BM) * n_tiles.
    int running = 0;
    for (int g0 = 0; g0 < args.groups; g0 += 32) {
      const int g = g0 + lane;
      int cnt = 0;
      if (g < args.groups) {
        const int rows = args.rows ? args.rows[g] : args.rows_const;
        cnt = ((rows + BM - 1) / BM) * args.n_tiles;
      }
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      if (g < args.groups) tile_start[g] = running + incl - cnt;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tile_start[args.groups] = running;
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_holder), Cf::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total_tiles = tile_start[args.groups];

  auto decode = [&](int tile, int& g, int& mt, int& nt) {
    int lo = 0, hi = args.groups - 1;   // largest g with tile_start[g] <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tile_start[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int local = tile - tile_start[g];
    mt = local / args.n_tiles;
    nt = local - mt * args.n_tiles;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int g, mt, nt;
        decode(tile, g, mt, nt);
        for (int kb = 0; kb < args.num_k_blocks; ++kb) {
          if (!mbar_wait(smem_addr(&empty[stage]), phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t sA = smem_addr(smem + stage * Cf::STAGE_BYTES);
          const uint32_t sB = sA + Cf::A_BYTES;
          const uint32_t fb = smem_addr(&full[stage]);
          mbar_arrive_expect_tx(fb, Cf::STAGE_BYTES);
          tma_load_3d(sA, &tmA, fb, kb * BK, mt * BM, g);
          if constexpr (MODE == kSwiGLU) {
            tma_load_3d(sB, &tmB, fb, kb * BK, nt * (BN / 2), g);
            tma_load_3d(sB + (BN / 2) * BK * 2, &tmB, fb, kb * BK, args.b_second_row + nt * (BN / 2), g);
          } else {
            tma_load_3d(sB, &tmB, fb, kb * BK, nt * BN, g);
          }
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        atomicOr(args.status, kStatusTimeoutProducer);
        *abort_flag = 1;
        for (int s = 0; s < S; ++s)   // let issued loads land before shared memory is released
          if ((issued >> s) & 1u) mbar_wait(smem_addr(&full[s]), (issued_parity >> s) & 1u, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t kIdesc = idesc_bf16_f32(BM, BN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        if (!mbar_wait(smem_addr(&tempty[acc]), acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < args.num_k_blocks; ++kb) {
          if (!mbar_wait(smem_addr(&full[stage]), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_addr(smem + stage * Cf::STAGE_BYTES);
          const uint64_t adesc = smem_desc_sw128(sA);
          const uint64_t bdesc = smem_desc_sw128(sA + Cf::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)   // +32 bytes along K per step
            mma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, kIdesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit(smem_addr(&empty[stage]));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(smem_addr(&tfull[acc]));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) {
        atomicOr(args.status, kStatusTimeoutMma);
        *abort_flag = 1;
        mma_commit(smem_addr(drain));   // wait for every MMA already issued
        mbar_wait(smem_addr(drain), 0, nullptr);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      int g, mt, nt;
      decode(tile, g, mt, nt);
      if (!mbar_wait(smem_addr(&tfull[acc]), acc_phase, abort_flag)) {
        atomicOr(args.status, kStatusTimeoutEpilogue);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int row = mt * BM + q * 32 + lane;
      const int rows_g = args.rows ? args.rows[g] : args.rows_const;
      const bool valid = row < rows_g;
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      if constexpr (MODE == kSwiGLU) {
        constexpr int HALF = BN / 2;
        uint16_t* orow = static_cast<uint16_t*>(args.out) + g * args.out_group_stride +
                         static_cast<long long>(row) * args.out_ld + nt * HALF;
#pragma unroll 1
        for (int c = 0; c < HALF; c += 32) {
          uint32_t gv[32], uv[32];
          tmem_ld32(tb + c, gv);
          tmem_ld32(tb + HALF + c, uv);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float h0 = silu_f(__uint_as_float(gv[2 * i])) * __uint_as_float(uv[2 * i]);
            const float h1 = silu_f(__uint_as_float(gv[2 * i + 1])) * __uint_as_float(uv[2 * i + 1]);
            pk[i] = pack_bf16x2(h0, h1);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      } else if constexpr (MODE == kBf16Out) {
        uint16_t* orow = static_cast<uint16_t*>(args.out) + g * args.out_group_stride +
                         static_cast<long long>(row) * args.out_ld + nt * BN;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(tb + c, v);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      } else {
        float* orow = static_cast<float*>(args.out) + static_cast<long long>(row) * args.out_ld;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(tb + c, v);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int col = nt * BN + c + i;
              if (col < args.n_valid) orow[col] = __uint_as_float(v[i]) + (args.bias ? args.bias[col] : 0.f);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_addr(&tempty[acc]));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cf::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// 3-D bf16 tensor [groups][rows][inner] (inner contiguous); box = 64 x box_rows x 1,
// 128-byte swizzle, zero fill out of bounds.
cudaError_t make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                     uint64_t groups, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {inner, rows, groups};
  const cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult res = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int MODE, int BN>
cudaError_t run_gemm(const CUtensorMap& a, const CUtensorMap& b, const GemmArgs& args, long long tiles,
                     int kind, cudaStream_t stream) {
  if (tiles <= 0) return cudaSuccess;
  auto kern = grouped_gemm_kernel<MODE, BN>;
  static std::atomic<uint64_t> configured{0};   // one bit per device ordinal
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               Cfg<BN>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  const int grid = static_cast<int>(tiles < num_sms() ? tiles : num_sms());
  launch_begin(kind, stream);
  kern<<<grid, kThreads, Cfg<BN>::SMEM_BYTES, stream>>>(a, b, args);
  launch_end(kind, stream);
  return cudaGetLastError();
}

long long count_tiles(const int32_t* n_host, int E, int n_tiles) {
  long long t = 0;
  for (int e = 0; e < E; ++e) t += static_cast<long long>((n_host[e] + BM - 1) / BM) * n_tiles;
  return t;
}

}  // namespace

cudaError_t launch_gate_up(const uint16_t* buf, const uint16_t* w_gate_up, uint16_t* h,
                           const int32_t* n_dev, const int32_t* n_host, int E, int C, int d, int F,
                           int32_t* status, cudaStream_t stream) {
  const int half = (F % 128 == 0) ? 128 : 64;
  CUtensorMap ma, mb;
  cudaError_t e;
  if ((e = make_map(&ma, buf, d, C, E, BM)) != cudaSuccess) return e;
  if ((e = make_map(&mb, w_gate_up, d, 2ull * F, E, half)) != cudaSuccess) return e;
  GemmArgs a{};
  a.rows = n_dev;
  a.groups = E;
  a.num_k_blocks = d / BK;
  a.n_tiles = F / half;
  a.b_second_row = F;
  a.out = h;
  a.out_group_stride = static_cast<long long>(C) * F;
  a.out_ld = F;
  a.status = status;
  const long long tiles = count_tiles(n_host, E, a.n_tiles);
  return half == 128 ? run_gemm<kSwiGLU, 256>(ma, mb, a, tiles, kKindGateUp, stream)
                     : run_gemm<kSwiGLU, 128>(ma, mb, a, tiles, kKindGateUp, stream);
}

cudaError_t launch_down(const uint16_t* h, const uint16_t* w_down, uint16_t* out,
                        const int32_t* n_dev, const int32_t* n_host, int E, int C, int d, int F,
                        int32_t* status, cudaStream_t stream) {
  const int bn = (d % 256 == 0) ? 256 : (d % 128 == 0) ? 128 : 64;
  CUtensorMap ma, mb;
  cudaError_t e;
  if ((e = make_map(&ma, h, F, C, E, BM)) != cudaSuccess) return e;
  if ((e = make_map(&mb, w_down, F, d, E, bn)) != cudaSuccess) return e;
  GemmArgs a{};
  a.rows = n_dev;
  a.groups = E;
  a.num_k_blocks = F / BK;
  a.n_tiles = d / bn;
  a.out = out;
  a.out_group_stride = static_cast<long long>(C) * d;
  a.out_ld = d;
  a.status = status;
  const long long tiles = count_tiles(n_host, E, a.n_tiles);
  if (bn == 256) return run_gemm<kBf16Out, 256>(ma, mb, a, tiles, kKindDown, stream);
  if (bn == 128) return run_gemm<kBf16Out, 128>(ma, mb, a, tiles, kKindDown, stream);
  return run_gemm<kBf16Out, 64>(ma, mb, a, tiles, kKindDown, stream);
}

cudaError_t launch_router_gemm(const uint16_t* x, const uint16_t* w_router, const float* bias,
                               float* logits, int T, int d, int E, int32_t* status,
                               cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int bn = E <= 64 ? 64 : E <= 128 ? 128 : 256;
  CUtensorMap ma, mb;
  cudaError_t e;
  if ((e = make_map(&ma, x, d, T, 1, BM)) != cudaSuccess) return e;
  if ((e = make_map(&mb, w_router, d, E, 1, bn)) != cudaSuccess) return e;
  GemmArgs a{};
  a.rows = nullptr;
  a.rows_const = T;
  a.groups = 1;
  a.num_k_blocks = d / BK;
  a.n_tiles = 1;
  a.n_valid = E;
  a.out = logits;
  a.out_ld = E;
  a.bias = bias;
  a.status = status;
  const long long tiles = (T + BM - 1) / BM;
  if (bn == 64) return run_gemm<kF32Bias, 64>(ma, mb, a, tiles, kKindRouterGemm, stream);
  if (bn == 128) return run_gemm<kF32Bias, 128>(ma, mb, a, tiles, kKindRouterGemm, stream);
  return run_gemm<kF32Bias, 256>(ma, mb, a, tiles, kKindRouterGemm, stream);
}

}  // namespace moe
