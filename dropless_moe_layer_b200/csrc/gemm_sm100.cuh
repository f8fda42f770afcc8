// gemm_sm100.cuh - device side of the grouped expert GEMM on the 5th-generation tensor
// cores (launched by grouped_gemm.cu).
//
// "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, item on reducing
// per-expert overhead [section "Reducing per-expert overhead"]: the experts of a group run
// as one grouped GEMM. One GEMM phase covers every expert with rows in the round; expert e
// multiplies its n[r][e] rows of the fixed [E, C, K] round buffer by its own weights.
//
// CTA layout (192 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: 3-D tiled loads (128-byte swizzle, no multicast) of the
//               A tile (128 rows x 64 K) and the B tile into a 192 KB shared-memory ring of
//               4 to 8 stages (more stages when the tile is narrower).
//   warp 1      MMA issuer: one thread issues tcgen05.mma.cta_group::1.kind::f16 (bf16 x
//               bf16 -> fp32, M = 128, N = bn <= 256, K = 16) into a TMEM accumulator;
//               tcgen05.commit frees each stage and, after the last K block, hands the
//               accumulator to the epilogue.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4)..+31, one output row per thread), the phase's math, 16-byte stores.
// Two accumulators of 256 TMEM columns alternate, so tile i's epilogue overlaps tile i+1's
// main loop. The pipeline counters live in the role threads (struct Pipe).
//
// Tiles are (group, 128-row block, N block). The N width is chosen per launch: the widest
// candidate that still gives every SM a tile, else the narrowest, so thin rounds (few active
// experts) spread over more SMs. Rows of a tile past the group's row count read
// stale rows or TMA zero fill; they reach only accumulator rows that are never stored (an
// MMA output row depends on its own A row only).
//
// Modes: SwiGLU (B = `width` rows of W1 (gate) stacked on the same rows of W3 (up), one MMA
// of N = 2 * width; out = bf16(silu(gate) * up)), Bf16Out (out = bf16(A B^T)) and F32Bias
// (out = fp32 A B^T + bias, for the router logits).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace moe {
namespace gemm {

using namespace sm100;

constexpr int BM = 128;
constexpr int BK = 64;            // bf16 elements in one 128-byte swizzle row
constexpr int UMMA_K = 16;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;
constexpr int kBMaxRows = 256;
constexpr int kStageBytes = kABytes + kBMaxRows * BK * 2;   // 48 KB
constexpr int kAccCols = 256;
constexpr int kTmemCols = 512;
constexpr int kMaxGroups = MOE_MAX_E_PLAN;
constexpr int kThreads = 192;
constexpr int kMaxStages = 8;
constexpr int kRingBytes = kStages * kStageBytes;           // 192 KB, re-cut per phase width
// TMA-store epilogue: each epilogue warp stages 32 rows x 32 columns of bf16 (2 KB, 64-byte
// swizzle) in one of its two buffers, then stores them with one bulk tensor store.
constexpr int kOutChunkCols = 32;
constexpr int kOutChunkBytes = 32 * kOutChunkCols * 2;
constexpr int kOutStagingBytes = 4 * 2 * kOutChunkBytes;    // 16 KB
constexpr int kBarBytes = (2 * kMaxStages + 5) * 8;
constexpr int kMiscWords = 8;
constexpr int kSmemBytes =
    1024 + kRingBytes + kOutStagingBytes + kBarBytes + kMiscWords * 4 + 2 * (kMaxGroups + 1) * 4;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

enum Mode : int { kSwiGLU = 0, kBf16Out = 1, kF32Bias = 2 };

struct Smem {
  uint8_t* stage;
  uint8_t* out_stage;       // TMA-store staging of the epilogue warps (1024-byte aligned)
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* drain;
  uint32_t* tmem_holder;
  volatile int* abort;      // raised by any role of this CTA that gives up
  int* width_idx;           // [2] chosen width of the two planned phases
  int* tile_start[2];       // [groups + 1] tile prefix of the two planned phases
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* base = raw + ((1024u - (smem_addr(raw) & 1023u)) & 1023u);
  s.stage = base;
  s.out_stage = base + kRingBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + kRingBytes + kOutStagingBytes);
  s.full = bars;
  s.empty = bars + kMaxStages;
  s.tfull = bars + 2 * kMaxStages;
  s.tempty = s.tfull + 2;
  s.drain = s.tempty + 2;
  uint32_t* misc = reinterpret_cast<uint32_t*>(s.drain + 1);
  s.tmem_holder = misc;
  s.abort = reinterpret_cast<volatile int*>(misc + 1);
  s.width_idx = reinterpret_cast<int*>(misc + 2);
  s.tile_start[0] = reinterpret_cast<int*>(misc + kMiscWords);
  s.tile_start[1] = s.tile_start[0] + kMaxGroups + 1;
  return s;
}

// CTA set-up: barriers (thread 0) and the TMEM accumulators (warp 1). Ends synchronised.
__device__ __forceinline__ uint32_t setup(const Smem& s) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(smem_addr(&s.full[i]), 1);
      mbar_init(smem_addr(&s.empty[i]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_addr(&s.tfull[a]), 1);
      mbar_init(smem_addr(&s.tempty[a]), 128);
    }
    mbar_init(smem_addr(s.drain), 1);
    *s.abort = 0;
    mbar_fence_init();
  }
  __syncwarp();   // every warp reconverges before the (aligned) CTA barrier
  if ((threadIdx.x >> 5) == 1) {
    tmem_alloc(smem_addr(s.tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return *s.tmem_holder;
}

// CTA tear-down after every role is done: frees the TMEM accumulators.
__device__ __forceinline__ void release_tmem(uint32_t tmem_base) {
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// One grouped GEMM.
struct Phase {
  int mode;
  const CUtensorMap* a;
  const CUtensorMap* b[3];     // B maps, one per candidate width
  int widths[3];               // candidate N widths (SwiGLU: gate columns), widest first; 0 = none
  int width_idx;               // >= 0: use widths[width_idx]; < 0: pick on the device
  const int32_t* rows;         // rows of each group (device), or nullptr: rows_const for all
  int rows_const;
  int groups;
  int num_k_blocks;            // K / 64
  int n_total;                 // output columns (SwiGLU: d_ff)
  int b_second_row;            // SwiGLU: first row of W3 inside B (= d_ff)
  void* out;
  long long out_group_stride;  // elements
  int out_ld;                  // elements
  const float* bias;           // F32Bias
  int n_valid;                 // F32Bias: stored columns
  // Pooled rows (capacity borrowing): group g's rows start at row group_row[g] - *group_row_base
  // of a single [rows, K] operand and output, instead of at row 0 of group g. Null: per group.
  const int32_t* group_row;
  const int32_t* group_row_base;
  // Debug bounds checks (MOE_FLAG_DEBUG_BOUNDS): a group's row count above rows_cap (the buffer
  // rows a group may hold) is recorded in the header dbg and clamped. rows_cap 0: unchecked.
  int rows_cap;
  int32_t* dbg;
  // TMA-store epilogue (CTA-pair form, per-expert outputs only): the output as a 3-D map [groups]
  // [rows][n_total] with 32 x 32 boxes and the 64-byte swizzle. Null: 16-byte stores per thread.
  const CUtensorMap* out_map;
  // Weights of group g: expert group_expert[g] of the B map (expert parallelism: a group is one
  // source rank's rows of one local expert). Null: expert g.
  const int32_t* group_expert;
  // CTA-pair form: a group's last row block of at most 128 rows runs as half-height tiles (M =
  // 128; see run_phase_pair), read through these two maps with 64-row boxes: the A operand's,
  // and (SwiGLU) the weights'. Null: 256-row tiles throughout.
  const CUtensorMap* a_rows64;
  const CUtensorMap* b_rows64;
};

__device__ __forceinline__ int group_weights(const Phase& p, int g) { return p.group_expert ? p.group_expert[g] : g; }

// Rows of group g (clamped to rows_cap under the debug bounds checks).
__device__ __forceinline__ int group_rows(const Phase& p, int g) {
  const int r = p.rows ? p.rows[g] : p.rows_const;
  return (p.rows_cap > 0 && r > p.rows_cap) ? p.rows_cap : r;
}

// Pipeline counters; each role thread uses its own fields, and they persist across phases.
struct Pipe {
  int stage = 0;
  uint32_t phase = 0;
  int acc = 0;
  uint32_t acc_phase = 0;
  uint32_t issued = 0, issued_parity = 0;   // producer: stages with loads in flight
};

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Warp 0 picks the phase's N width and writes its tile prefix into slot `which`.
// The caller synchronises the CTA before run_phase.
// Warp 0 of CTA 0 records groups whose row count is above rows_cap (debug bounds checks).
__device__ __forceinline__ void check_group_rows(const Phase& p) {
  if (p.rows_cap <= 0 || p.dbg == nullptr || p.rows == nullptr || blockIdx.x != 0) return;
  for (int g = threadIdx.x & 31; g < p.groups; g += 32)
    if (p.rows[g] < 0 || p.rows[g] > p.rows_cap) record_bad(p.dbg, kBadGemmRows, g);
}

__device__ __forceinline__ void plan_phase(const Smem& s, const Phase& p, int which) {
  if ((threadIdx.x >> 5) != 0) return;
  const int lane = threadIdx.x & 31;
  check_group_rows(p);
  int mt = 0;
  for (int g = lane; g < p.groups; g += 32) {
    const int rows = group_rows(p, g);
    mt += (rows + BM - 1) / BM;
  }
  mt = warp_sum(mt);
  int wi = p.width_idx;          // chosen by the host when it knows the row counts
  if (wi < 0) {
    int last = -1;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const int w = p.widths[i];
      if (w <= 0 || p.n_total % w != 0) continue;
      last = i;
      if (static_cast<long long>(mt) * (p.n_total / w) >= gridDim.x) {
        wi = i;
        break;
      }
    }
    if (wi < 0) wi = last;
  }
  const int n_tiles = p.n_total / (wi == 0 ? p.widths[0] : wi == 1 ? p.widths[1] : p.widths[2]);
  int* ts = s.tile_start[which];
  int running = 0;
  for (int g0 = 0; g0 < p.groups; g0 += 32) {
    const int g = g0 + lane;
    int cnt = 0;
    if (g < p.groups) {
      const int rows = group_rows(p, g);
      cnt = ((rows + BM - 1) / BM) * n_tiles;
    }
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (g < p.groups) ts[g] = running + incl - cnt;
    running += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    ts[p.groups] = running;
    s.width_idx[which] = wi;
  }
  __syncwarp();
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// silu(a) = a * sigmoid(a) = a / (1 + e^-a), with the fast division (at most 2 ulp; it returns 0
// once 1 + e^-a exceeds 2^126, where silu(a) is below 1e-36 in magnitude anyway).
__device__ __forceinline__ float silu_f(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

// Epilogue of one accumulator row (this thread's TMEM lane; tb = lane base + accumulator
// column): SwiGLU of `width` gate columns (TMEM columns [0, width)) with the matching up
// columns ([width, 2 width)), bf16, 16-byte stores to orow[0, width). The TMEM loads are
// warp-wide, so every lane runs them; only rows with `valid` store.
__device__ __forceinline__ void store_swiglu(uint32_t tb, int width, uint16_t* orow, bool valid) {
  for (int c = 0; c < width; c += 32) {
    uint32_t gv[32], uv[32];
    tmem_ld32(tb + c, gv);
    tmem_ld32(tb + width + c, uv);
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
}

// Same for a plain bf16 result of `cols` columns.
__device__ __forceinline__ void store_bf16(uint32_t tb, int cols, uint16_t* orow, bool valid) {
  for (int c = 0; c < cols; c += 32) {
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
}

// Runs the CTA's share of the tiles of the phase planned in slot `which`. Returns when this
// warp's role work is issued/done (the epilogue warps return after their last store). Every warp
// leaves converged: a CTA barrier (which requires whole warps) may follow directly.
__device__ __forceinline__ void run_phase(const Smem& s, uint32_t tmem_base, const Phase& p, int which,
                                          Pipe& pipe, int32_t* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int* ts = s.tile_start[which];
  const int wi = s.width_idx[which];
  // explicit selects instead of indexing p.widths / p.b with wi: the Phase then stays in registers
  const int width = wi == 0 ? p.widths[0] : wi == 1 ? p.widths[1] : p.widths[2];
  const CUtensorMap* const b_map = wi == 0 ? p.b[0] : wi == 1 ? p.b[1] : p.b[2];
  const int bn = p.mode == kSwiGLU ? 2 * width : width;
  const int n_tiles = p.n_total / width;
  const int total = ts[p.groups];
  // the 192 KB ring is cut into as many stages as this width allows (4 at N = 256, 8 at N <= 64)
  const int stage_bytes = kABytes + bn * BK * 2;
  const int nstages = min(kMaxStages, kRingBytes / stage_bytes);
  auto decode = [&](int tile, int& g, int& mt, int& nt) {
    int lo = 0, hi = p.groups - 1;   // largest g with ts[g] <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ts[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int local = tile - ts[g];
    mt = local / n_tiles;
    nt = local - mt * n_tiles;
  };

  if (warp == 0) {
    if (lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    const CUtensorMap* mb = b_map;
    const uint32_t tx = static_cast<uint32_t>(kABytes + bn * BK * 2);
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      int g, mt, nt;
      decode(tile, g, mt, nt);
      int a_row = mt * BM, a_grp = g;
      if (p.group_row) {
        a_row += p.group_row[g] - *p.group_row_base;
        a_grp = 0;
      }
      for (int kb = 0; kb < p.num_k_blocks; ++kb) {
        if (!mbar_wait(smem_addr(&s.empty[pipe.stage]), pipe.phase ^ 1u, s.abort)) {
          ok = false;
          break;
        }
        const uint32_t sA = smem_addr(s.stage + pipe.stage * stage_bytes);
        const uint32_t sB = sA + kABytes;
        const uint32_t fb = smem_addr(&s.full[pipe.stage]);
        mbar_arrive_expect_tx(fb, tx);
        tma_load_3d(sA, p.a, fb, kb * BK, a_row, a_grp);
        if (p.mode == kSwiGLU) {
          tma_load_3d(sB, mb, fb, kb * BK, nt * width, group_weights(p, g));
          tma_load_3d(sB + width * BK * 2, mb, fb, kb * BK, p.b_second_row + nt * width, group_weights(p, g));
        } else {
          tma_load_3d(sB, mb, fb, kb * BK, nt * width, group_weights(p, g));
        }
        pipe.issued |= 1u << pipe.stage;
        pipe.issued_parity = (pipe.issued_parity & ~(1u << pipe.stage)) | (pipe.phase << pipe.stage);
        if (++pipe.stage == nstages) {
          pipe.stage = 0;
          pipe.phase ^= 1u;
        }
      }
    }
    if (!ok) {
      atomicOr(status, kStatusTimeoutProducer);
      *s.abort = 1;
      for (int i = 0; i < nstages; ++i)   // let issued loads land before shared memory is reused
        if ((pipe.issued >> i) & 1u) mbar_wait(smem_addr(&s.full[i]), (pipe.issued_parity >> i) & 1u, nullptr);
    }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(BM, bn);
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      if (!mbar_wait(smem_addr(&s.tempty[pipe.acc]), pipe.acc_phase ^ 1u, s.abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(pipe.acc * kAccCols);
      for (int kb = 0; kb < p.num_k_blocks; ++kb) {
        if (!mbar_wait(smem_addr(&s.full[pipe.stage]), pipe.phase, s.abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sA = smem_addr(s.stage + pipe.stage * stage_bytes);
        const uint64_t adesc = smem_desc_sw128(sA);
        const uint64_t bdesc = smem_desc_sw128(sA + kABytes);
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk)   // +32 bytes along K per step
          mma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
        mma_commit(smem_addr(&s.empty[pipe.stage]));
        if (++pipe.stage == nstages) {
          pipe.stage = 0;
          pipe.phase ^= 1u;
        }
      }
      if (!ok) break;
      mma_commit(smem_addr(&s.tfull[pipe.acc]));
      pipe.acc ^= 1;
      if (pipe.acc == 0) pipe.acc_phase ^= 1u;
    }
    if (!ok) {
      atomicOr(status, kStatusTimeoutMma);
      *s.abort = 1;
      mma_commit(smem_addr(s.drain));   // wait for every MMA already issued
      mbar_wait(smem_addr(s.drain), 0, nullptr);
    }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int g, mt, nt;
      decode(tile, g, mt, nt);
      // every lane waits; the outcome is made warp-uniform before the warp-wide TMEM loads
      const bool ready = __all_sync(0xffffffffu, mbar_wait(smem_addr(&s.tfull[pipe.acc]), pipe.acc_phase, s.abort));
      if (!ready) {
        if (lane == 0) atomicOr(status, kStatusTimeoutEpilogue);
        *s.abort = 1;
        break;
      }
      tc_fence_after();
      const int row = mt * BM + q * 32 + lane;
      const int rows_g = group_rows(p, g);
      const bool valid = row < rows_g;
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(pipe.acc * kAccCols);
      const long long orow_off = p.group_row
                                     ? static_cast<long long>(p.group_row[g] - *p.group_row_base + row) * p.out_ld
                                     : g * p.out_group_stride + static_cast<long long>(row) * p.out_ld;
      if (p.mode == kSwiGLU) {
        uint16_t* orow = static_cast<uint16_t*>(p.out) + orow_off + nt * width;
        store_swiglu(tb, width, orow, valid);
      } else if (p.mode == kBf16Out) {
        uint16_t* orow = static_cast<uint16_t*>(p.out) + orow_off + nt * width;
        store_bf16(tb, bn, orow, valid);
      } else {
        float* orow = static_cast<float*>(p.out) + static_cast<long long>(row) * p.out_ld;
        for (int c = 0; c < bn; c += 32) {
          uint32_t v[32];
          tmem_ld32(tb + c, v);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int col = nt * width + c + i;
              if (col < p.n_valid) orow[col] = __uint_as_float(v[i]) + (p.bias ? p.bias[col] : 0.f);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_addr(&s.tempty[pipe.acc]));
      pipe.acc ^= 1;
      if (pipe.acc == 0) pipe.acc_phase ^= 1u;
    }
    __syncwarp();
  }
}

// ================================================================ CTA-pair form (cta_group::2)
//
// The same grouped GEMM on tiles of 256 rows x 256 columns shared by the two CTAs of a cluster
// of two. CTA c of the pair loads A rows [128 c, 128 c + 128) of the tile and B rows
// [128 c, 128 c + 128) of its 256 (SwiGLU: c = 0 the tile's 128 gate rows, c = 1 the same 128
// up rows; Bf16Out: the two halves of the 256 output columns) into its own shared memory; the
// leader's one thread issues the M = 256, N = 256 MMA for both, which reads the peer's halves
// at the same offsets and leaves accumulator rows [128 c, 128 c + 128) in CTA c's TMEM. Per
// k block a CTA's shared memory then holds 32 KB for 2 x 128 x 256 x 64 flops, half the bytes
// per flop of the single-CTA tile, which is what lets the tensor pipe run near its peak: the
// single-CTA 128 x 256 tile needs more shared-memory bandwidth (TMA writes plus MMA reads)
// than an SM has. No load is multicast.
//
// Barriers: full[s] lives in the leader (one arrive with the pair's bytes, both CTAs' TMA
// loads complete on it); empty[s] and tfull[a] in both CTAs (the leader's commit arrives on
// both); tempty[a] in the leader (one arrive per epilogue warp of either CTA: 8).
constexpr int kPairRows = 2 * BM;        // rows of a pair tile
constexpr int kPairBn = 256;             // MMA N of a pair tile
constexpr int kPairBHalf = kPairBn / 2;  // B rows per CTA
constexpr int kPairStageBytes = kABytes + kPairBHalf * BK * 2;   // 32 KB
constexpr int kPairStages = kRingBytes / kPairStageBytes;        // 6
static_assert(kPairStages <= kMaxStages, "pair ring stages");
constexpr int kEpiWarpsPair = 8;         // arrivals on the leader's tempty per tile

// Half-height tiles. A group's last row block with at most 128 rows (an expert's leftover rows,
// common in a round that holds every expert) would leave at least half of a 256-row tile as
// padding. It runs instead as M = 128 tiles of the same columns: CTA c loads 64 A rows [64 c,
// 64 c + 64) of the block and the same 128 B rows as in a full tile, except that for SwiGLU CTA c
// takes W1 rows [64 c, 64 c + 64) of the tile's 128 gate columns and the same W3 rows (64-row
// boxes). In this shape the accumulator of each CTA holds its 64 rows twice over the TMEM lanes:
// lanes [0, 64) take the MMA's columns [0, 128) (CTA 0's B rows), lanes [64, 128) columns
// [128, 256) (CTA 1's), each at TMEM columns [0, 128). So epilogue warp q handles rows
// 32 (q & 1) .. + 32 of the CTA's 64 and the B half q >> 1: SwiGLU gate columns at [0, 64) and
// up at [64, 128) for the 64 gate columns 64 c' (c' = q >> 1) of the tile; Bf16Out the tile's
// columns 128 (q >> 1) .. + 128. Half the MMA work of a padded 256-row tile, the same weights.
constexpr int kHalfRows = BM / 2;        // A rows per CTA in a half-height tile
constexpr int kHalfStageBytes = kHalfRows * BK * 2 + kPairBHalf * BK * 2;   // 24 KB per CTA

// Whether row block mp of a group with `rows` rows is its short last block (half-height tiles).
__device__ __forceinline__ bool half_block(const Phase& p, int rows, int mp) {
  const int tail = rows - mp * kPairRows;
  return p.a_rows64 != nullptr && tail > 0 && tail <= BM;
}

// Set-up of both CTAs of a pair: barriers (thread 0 of each), the pair's TMEM (warp 1 of each),
// then a cluster barrier, so that no CTA signals its peer before the peer's barriers exist.
__device__ __forceinline__ uint32_t setup_pair(const Smem& s) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxStages; ++i) {
      mbar_init(smem_addr(&s.full[i]), 1);
      mbar_init(smem_addr(&s.empty[i]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_addr(&s.tfull[a]), 1);
      mbar_init(smem_addr(&s.tempty[a]), kEpiWarpsPair);
    }
    mbar_init(smem_addr(s.drain), 1);
    *s.abort = 0;
    mbar_fence_init();
  }
  __syncwarp();
  if ((threadIdx.x >> 5) == 1) {
    tmem_alloc_pair(smem_addr(s.tmem_holder), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  return *s.tmem_holder;
}

// Tear-down of both CTAs once every role of this CTA is done: a cluster barrier (no peer still
// reads this CTA's shared memory or signals its barriers), then the pair's TMEM is freed.
__device__ __forceinline__ void release_tmem_pair(uint32_t tmem_base) {
  tc_fence_before();
  cluster_sync();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// Warp 0 writes the phase's tile prefix over 256-row blocks into slot `which` (fixed width).
__device__ __forceinline__ void plan_phase_pair(const Smem& s, const Phase& p, int which, int width) {
  if ((threadIdx.x >> 5) != 0) return;
  const int lane = threadIdx.x & 31;
  check_group_rows(p);
  const int n_tiles = p.n_total / width;
  int* ts = s.tile_start[which];
  int running = 0;
  for (int g0 = 0; g0 < p.groups; g0 += 32) {
    const int g = g0 + lane;
    int cnt = 0;
    if (g < p.groups) {
      const int rows = group_rows(p, g);
      cnt = ((rows + kPairRows - 1) / kPairRows) * n_tiles;
    }
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (g < p.groups) ts[g] = running + incl - cnt;
    running += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) ts[p.groups] = running;
  __syncwarp();
}

// The pair's share of the tiles: pair `pair` of `pairs` takes tiles pair, pair + pairs, ...
// `width`: SwiGLU gate columns per tile (128; the B tile is those gate rows and the same up
// rows), Bf16Out output columns (256). Modes SwiGLU and Bf16Out only.
__device__ __forceinline__ void run_phase_pair(const Smem& s, uint32_t tmem_base, const Phase& p, int which,
                                               int width, int pair, int pairs, Pipe& pipe, int32_t* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t cta = cluster_rank();
  const int* ts = s.tile_start[which];
  const int n_tiles = p.n_total / width;
  const int total = ts[p.groups];
  auto decode = [&](int tile, int& g, int& mp, int& nt) {
    int lo = 0, hi = p.groups - 1;   // largest g with ts[g] <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (ts[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int local = tile - ts[g];
    mp = local / n_tiles;
    nt = local - mp * n_tiles;
  };
  // B rows of this CTA's half of a tile
  auto b_row = [&](int nt) {
    return p.mode == kSwiGLU ? static_cast<int>(cta) * p.b_second_row + nt * width
                             : nt * width + static_cast<int>(cta) * kPairBHalf;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    bool ok = true;
    for (int tile = pair; ok && tile < total; tile += pairs) {
      int g, mp, nt;
      decode(tile, g, mp, nt);
      const bool half = half_block(p, group_rows(p, g), mp);
      // the pair's bytes per stage, counted by the leader
      const uint32_t tx = 2u * (half ? kHalfStageBytes : kPairStageBytes);
      // this CTA's first A row
      int a_row = mp * kPairRows + static_cast<int>(cta) * (half ? kHalfRows : BM), a_grp = g;
      if (p.group_row) {
        a_row += p.group_row[g] - *p.group_row_base;
        a_grp = 0;
      }
      for (int kb = 0; kb < p.num_k_blocks; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(smem_addr(&s.empty[pipe.stage]), pipe.phase ^ 1u, s.abort))) {
          ok = false;
          break;
        }
        const uint32_t sA = smem_addr(s.stage + pipe.stage * kPairStageBytes);
        const uint32_t sB = sA + kABytes;
        const uint32_t fb_local = smem_addr(&s.full[pipe.stage]);
        const uint32_t fb = peer_addr(fb_local, 0);   // the leader's full barrier
        if (cta == 0 && lane == 0) mbar_arrive_expect_tx(fb_local, tx);
        __syncwarp();
        if (lane == 0) {
          if (!half) {
            tma_load_3d_pair(sA, p.a, fb, kb * BK, a_row, a_grp);
            tma_load_3d_pair(sB, p.b[0], fb, kb * BK, b_row(nt), group_weights(p, g));
          } else {
            tma_load_3d_pair(sA, p.a_rows64, fb, kb * BK, a_row, a_grp);
            if (p.mode == kSwiGLU) {   // 64 W1 rows, then the same 64 W3 rows
              const int w1 = nt * width + static_cast<int>(cta) * kHalfRows;
              tma_load_3d_pair(sB, p.b_rows64, fb, kb * BK, w1, group_weights(p, g));
              tma_load_3d_pair(sB + kHalfRows * BK * 2, p.b_rows64, fb, kb * BK, p.b_second_row + w1,
                               group_weights(p, g));
            } else {
              tma_load_3d_pair(sB, p.b[0], fb, kb * BK, b_row(nt), group_weights(p, g));
            }
          }
        }
        pipe.issued |= 1u << pipe.stage;
        if (++pipe.stage == kPairStages) {
          pipe.stage = 0;
          pipe.phase ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      atomicOr(status, kStatusTimeoutProducer);
      *s.abort = 1;
      // loads already issued complete on the leader's barriers, which this CTA cannot wait on:
      // give them time to land before the pair's shared memory is released
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 200000ull) {
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && cta == 0) {
    // ---------------------------------------------------------------- MMA issuer (leader only)
    bool ok = true;
    for (int tile = pair; ok && tile < total; tile += pairs) {
      int g, mp, nt;
      decode(tile, g, mp, nt);
      const uint32_t idesc = idesc_bf16_f32(half_block(p, group_rows(p, g), mp) ? BM : kPairRows, kPairBn);
      if (!mbar_wait(smem_addr(&s.tempty[pipe.acc]), pipe.acc_phase ^ 1u, s.abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(pipe.acc * kAccCols);
      for (int kb = 0; kb < p.num_k_blocks; ++kb) {
        if (!mbar_wait(smem_addr(&s.full[pipe.stage]), pipe.phase, s.abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sA = smem_addr(s.stage + pipe.stage * kPairStageBytes);
        const uint64_t adesc = smem_desc_sw128(sA);
        const uint64_t bdesc = smem_desc_sw128(sA + kABytes);
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk)
          mma_bf16_pair(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
        mma_commit_pair(smem_addr(&s.empty[pipe.stage]), 3);
        if (++pipe.stage == kPairStages) {
          pipe.stage = 0;
          pipe.phase ^= 1u;
        }
      }
      if (!ok) break;
      mma_commit_pair(smem_addr(&s.tfull[pipe.acc]), 3);
      pipe.acc ^= 1;
      if (pipe.acc == 0) pipe.acc_phase ^= 1u;
    }
    if (!ok) {
      atomicOr(status, kStatusTimeoutMma);
      *s.abort = 1;
      mma_commit_pair(smem_addr(s.drain), 1);   // wait for every MMA already issued
      mbar_wait(smem_addr(s.drain), 0, nullptr);
    }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    uint32_t ochunk = 0;   // chunks this warp has staged (alternates its two buffers)
    const uint32_t stage0 = smem_addr(s.out_stage + q * 2 * kOutChunkBytes);
    // the outputs stream out: first in line for eviction, behind the tiles the MMAs still reuse
    const uint64_t out_policy = policy_evict_first();
    for (int tile = pair; tile < total; tile += pairs) {
      int g, mp, nt;
      decode(tile, g, mp, nt);
      const bool ready = __all_sync(0xffffffffu, mbar_wait(smem_addr(&s.tfull[pipe.acc]), pipe.acc_phase, s.abort));
      if (!ready) {
        if (lane == 0) atomicOr(status, kStatusTimeoutEpilogue);
        *s.abort = 1;
        break;
      }
      tc_fence_after();
      const int rows_g = group_rows(p, g);
      const bool half = half_block(p, rows_g, mp);
      // this warp's first row, and the output columns it holds (from TMEM column 0 on): a full
      // tile's warp q has rows 32 q .. of the CTA's 128 and all the tile's columns; a half-height
      // tile's has rows 32 (q & 1) .. of the CTA's 64 and the columns of B half q >> 1
      const int row_base = mp * kPairRows + (half ? static_cast<int>(cta) * kHalfRows + (q & 1) * 32
                                                  : static_cast<int>(cta) * BM + q * 32);
      const int row = row_base + lane;
      const bool valid = row < rows_g;
      const int out_cols = (p.mode == kSwiGLU ? width : kPairBn) / (half ? 2 : 1);
      const int col0 = nt * width + (half ? (q >> 1) * out_cols : 0);
      const int up_off = out_cols;   // SwiGLU: TMEM offset of the up columns
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(pipe.acc * kAccCols);
      const long long orow_off = p.group_row
                                     ? static_cast<long long>(p.group_row[g] - *p.group_row_base + row) * p.out_ld
                                     : g * p.out_group_stride + static_cast<long long>(row) * p.out_ld;
      uint16_t* orow = static_cast<uint16_t*>(p.out) + orow_off + col0;
      if (p.out_map != nullptr) {
        // 32-column chunks: TMEM -> registers -> this warp's staging buffer -> one bulk store of
        // its 32 rows. Rows of the box past the group's rows hold junk; they fall in the expert's
        // unused rows [n, C) (never read) or past C (clipped by the map).
        const int chunks = out_cols / kOutChunkCols;
        for (int c = 0; c < chunks; ++c) {
          uint32_t pk[16];
          if (p.mode == kSwiGLU) {
            uint32_t gv[32], uv[32];
            tmem_ld32(tb + c * kOutChunkCols, gv);
            tmem_ld32(tb + up_off + c * kOutChunkCols, uv);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(silu_f(__uint_as_float(gv[2 * i])) * __uint_as_float(uv[2 * i]),
                                  silu_f(__uint_as_float(gv[2 * i + 1])) * __uint_as_float(uv[2 * i + 1]));
          } else {
            uint32_t v[32];
            tmem_ld32(tb + c * kOutChunkCols, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          }
          const uint32_t buf_off = (ochunk & 1u) * kOutChunkBytes;
          if (lane == 0) bulk_wait_read_1();   // the store that last used this buffer has read it
          __syncwarp();
          uint8_t* row_ptr = s.out_stage + q * 2 * kOutChunkBytes + buf_off + lane * 64;
#pragma unroll
          for (int j = 0; j < 4; ++j)   // 64-byte swizzle: piece j of row r at j ^ ((r >> 1) & 3)
            *reinterpret_cast<uint4*>(row_ptr + ((j ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(p.out_map, stage0 + buf_off, col0 + c * kOutChunkCols, row_base, g, out_policy);
            bulk_commit();
          }
          ++ochunk;
        }
      } else if (p.mode == kSwiGLU) {
        store_swiglu(tb, out_cols, orow, valid);
      } else {
        store_bf16(tb, out_cols, orow, valid);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(peer_addr(smem_addr(&s.tempty[pipe.acc]), 0));
      pipe.acc ^= 1;
      if (pipe.acc == 0) pipe.acc_phase ^= 1u;
    }
    if (lane == 0 && ochunk > 0) bulk_wait_all();   // this warp's stores are written before it exits
    __syncwarp();
  }
}

// Host side: tensor maps (cached) for a 3-D bf16 tensor [groups][rows][inner], box = box_inner
// x box_rows x 1, zero fill out of bounds; 128-byte swizzle for 64-column operand boxes, 64-byte
// swizzle for the 32-column output boxes of the TMA-store epilogue.
cudaError_t make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
                     uint64_t groups, uint32_t box_rows, uint32_t box_inner = BK);
// fp32 [groups][rows][inner], box box_inner x box_rows x 1, 64-byte swizzle (box_inner * 4 == 64).
cudaError_t make_map_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t groups,
                         uint32_t box_inner, uint32_t box_rows);

}  // namespace gemm
}  // namespace moe
