// backward.cu - backward pass of the multi-round dropless MoE layer, with per-round recompute.
//
// "Microsoft AI's MAI-Base-2 trained on 16K GPUs with Muon", section "Expert groups keep memory
// fixed when tokens pile up": the backward pass recomputes each expert group on the same round
// schedule as the forward, so its memory stays as static as the forward's. "Frontier
// Pre-training at Microsoft AI (MAI-Base-2)", Key claims, multi-round dropless MoE item
// [section "Scaling MoE", Fig. 6]: the backward uses fine-grained per-expert-group recompute.
//
// Per expert e and row x (a pair (t, j) of the round): a = W1 x, b = W3 x, s = silu(a),
// h = s * b, out = W2 h, y[t] += gate * out. Given dy (fp32):
//   dgate = <dy, out> = <W2^T dy, h>        dh = gate * W2^T dy
//   db = dh * s, da = dh * b * silu'(a)     dx[t] += W1^T da + W3^T db
//   dW2_e += (gate dy) h^T = dy (gate h)^T  dW1_e += da x^T, dW3_e += db x^T
//   dz = softmax Jacobian applied to dgate (renormalised gates: the quotient rule first).
//
// Per round r, with the forward's plan. The round's rows live in buffers of E * C rows, expert
// e's at e * C + slot; with capacity borrowing in buffers of E * C + 64 E rows, expert e's at
// seg_off[r][e] + slot, where each expert's segment starts at a multiple of 64:
//   gather     x rows -> xbuf, bf16(dy) rows -> dybuf; the pair's gate -> row_gate
//   recompute  [a | b] = xbuf W13^T (tensor cores); epilogue keeps a, b (bf16) and writes
//              hg = bf16(gate * h), through TMA stores of 32 x 32 chunks
//   dh         W2^T dy as dybuf (W2^T)^T (tensor cores, B = W2 read MN-major as stored);
//              epilogue: the SwiGLU backward (da, db from a, b and the gate), dgate partial sums
//              <W2^T dy, h> per 64..256-column tile, dab = [da | db] (TMA stores)
//              Rounds whose GEMMs run in the single-CTA form may run recompute and dh as one
//              launch (kRecDh, when it streams less per SM than two launches): a tile of 64 d_ff
//              columns accumulates [a | b] and W2^T dy side by side in TMEM, and one epilogue
//              writes hg and dab from fp32 a and b (ab is not written).
//   dx         dab W13 (tensor cores, B = W13 read MN-major as stored) -> dxbuf (bf16)
//   combine    dx[t] = (first round of t ? 0 : dx[t]) + sum of the token's dxbuf rows, ascending
//              j; dgate[t, j] = sum of its row's partials in tile order (no atomics anywhere);
//              the next round's gather runs in the same launch (other blocks), so a round after
//              the first takes four launches
//   wgrad      dW2 += dy^T hg and dW13 += dab^T x over K = the round's rows of each expert
//              (tensor cores, both operands the row-major round buffers read MN-major; the fp32
//              gradient tiles are stored in round 0, which holds every expert that has rows,
//              and reduce-added through TMA after); one launch with the dx GEMM, as the three
//              are independent
// After the last round: dz from dgate and the logits (one warp per token).
//
// Every operand of a tensor-core step is bf16 (fp32 accumulate); a and b are kept as bf16 between
// the recompute and the dh epilogue (fp32 in TMEM in the fused launch). Rows of a tile past the expert's row count never reach a
// store, except that the rows from the count up to the next multiple of 64 (within the expert's
// C rows, or its segment) are written as zeros in xbuf, dybuf, hg and dab: the weight-gradient
// GEMMs read K, the rows, in blocks of 64 without a mask, and with pooled rows the next expert's
// segment starts right after.
#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>

#include "copy_phases.cuh"
#include "gemm_sm100.cuh"
#include "backward.h"
#include "kernels.h"

namespace moe {
namespace bwd {

using namespace sm100;
using gemm::BK;
using gemm::BM;
using gemm::Pipe;
using gemm::Smem;

enum Mode : int { kRecompute = 0, kDh = 1, kDx = 2, kWgrad = 3, kRecDh = 4 };

// kRecDh (single-CTA form only): the recompute and dh of the same 64 d_ff columns in one tile.
// K blocks [0, num_k_blocks) accumulate [a | b] = x W13^T (MMA N = 128) into accumulator columns
// [0, 128), K blocks [num_k_blocks, 2 num_k_blocks) accumulate W2^T dy (N = 64, W2 read
// MN-major) into columns [128, 192); the epilogue has a, b and W2^T dy of its rows at once, so
// a and b are never stored.
constexpr int kRecDhWidth = 64;

struct GemmArgs {
  int mode;
  int width;                  // output columns per tile (kRecompute: gate columns, MMA N = 2x)
  const int32_t* rows;        // [E] rows of each expert in this round (the round's n)
  int groups;                 // E
  int m_total;                // kWgrad: output rows per expert (the M extent)
  int n_total;                // output columns per expert
  int num_k_blocks;           // K / 64 (all but kWgrad, whose K is the expert's rows)
  int C, F;
  // Pooled round rows (capacity borrowing): expert g's rows of the round start at row
  // group_row[g] - *group_row_base of the round buffers, a multiple of 64 (the backward's own
  // segment table). Null: rows at g * C.
  const int32_t* group_row;
  const int32_t* group_row_base;
  void* out;                  // kRecompute: ab; kDh: dab; kDx: dxbuf; kWgrad: the fp32 gradient
  long long out_group_stride; // elements (kWgrad)
  int out_ld;                 // elements (kWgrad, kDx)
  const uint16_t* ab;         // kDh: [E * C][2F] a | b
  const float* row_gate;      // kRecompute, kDh: [E * C] gate of the pair in each row
  float* dgate_part;          // kDh: [E * C][dgate_ld] partial sums of <W2^T dy, h>
  int dgate_ld;
  int overwrite;              // kWgrad: store the tile instead of adding it (round 0)
  int tma_out;                // kWgrad: write the tile through the phase's fp32 output map (TMA
                              // store, or TMA reduce-add) instead of per-thread read-add-write
  int b_mn;                   // B is MN-major ([K][N] in memory), loaded as 64 x 64 boxes (64 N
                              // by 64 K): kDh W2 [E][d][d_ff], kDx W13 [E][2 d_ff][d], kWgrad
                              // the round's row-major hg or xbuf ([rows][N], K = the rows)
  int a_mn;                   // A is MN-major the same way: kWgrad the round's dybuf or dab
  int32_t* status;
};

constexpr int kMnBox = 64;                         // MN-major boxes: 64 M or N x 64 K rows
constexpr int kMnBoxBytes = kMnBox * BK * 2;       // 8 KB

// Instruction descriptor bits of kind::f16: A MN-major (transpose A, bit 15), B MN-major (bit 16).
constexpr uint32_t kIdescAMn = 1u << 15;
constexpr uint32_t kIdescBMn = 1u << 16;

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<const uint16_t*>(&b);
}

// Tiles of expert g: row blocks of `bm` rows (128, or 256 in the CTA-pair form) x n_tiles.
__device__ __forceinline__ int tiles_of(const GemmArgs& p, int g, int n_tiles, int bm) {
  const int rows = p.rows[g];
  if (p.mode == kWgrad) return rows > 0 ? ((p.m_total + bm - 1) / bm) * n_tiles : 0;
  return ((rows + bm - 1) / bm) * n_tiles;
}

__device__ __forceinline__ int k_blocks_of(const GemmArgs& p, int g) {
  return p.mode == kWgrad ? (p.rows[g] + BK - 1) / BK : p.mode == kRecDh ? 2 * p.num_k_blocks : p.num_k_blocks;
}

// Exclusive prefix over the experts of cnt(g), written to out[0 .. groups] by warp 0.
template <typename Count>
__device__ __forceinline__ void warp_prefix(int* out, int groups, Count cnt_of) {
  const int lane = threadIdx.x & 31;
  int running = 0;
  for (int g0 = 0; g0 < groups; g0 += 32) {
    const int g = g0 + lane;
    const int cnt = g < groups ? cnt_of(g) : 0;
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (g < groups) out[g] = running + incl - cnt;
    running += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) out[groups] = running;
  __syncwarp();
}

// Warp 0 writes the tile prefix over the experts into ts[0 .. groups].
__device__ __forceinline__ void plan_tiles(int* ts, const GemmArgs& p, int n_tiles, int bm) {
  if ((threadIdx.x >> 5) != 0) return;
  warp_prefix(ts, p.groups, [&](int g) { return tiles_of(p, g, n_tiles, bm); });
}

// Row of expert g's row `row` in the round buffers.
__device__ __forceinline__ long long row_of(const GemmArgs& p, int g, int row) {
  return p.group_row ? static_cast<long long>(p.group_row[g] - *p.group_row_base) + row
                     : static_cast<long long>(g) * p.C + row;
}

// ---------------------------------------------------------------- epilogues (one row per thread)

// One 32 x 32 bf16 chunk of this warp's 32 rows (lane = row; pk = the lane's 32 values packed in
// pairs) through one of the warp's two staging buffers (64-byte swizzle) and one bulk tensor
// store at (col, row, grp) of `map`. ochunk counts the warp's staged chunks (alternates buffers).
__device__ __forceinline__ void store_chunk(const CUtensorMap* map, const uint32_t (&pk)[16], int col, int row,
                                            int grp, uint8_t* stage, uint32_t& ochunk) {
  const int lane = threadIdx.x & 31;
  const uint32_t buf_off = (ochunk & 1u) * gemm::kOutChunkBytes;
  if (lane == 0) bulk_wait_read_1();   // the store that last used this buffer has read it
  __syncwarp();
  uint8_t* row_ptr = stage + buf_off + lane * 64;
#pragma unroll
  for (int j = 0; j < 4; ++j)   // 64-byte swizzle: piece j of row r at j ^ ((r >> 1) & 3)
    *reinterpret_cast<uint4*>(row_ptr + ((j ^ ((lane >> 1) & 3)) << 4)) =
        make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
  fence_async_shared();
  __syncwarp();
  if (lane == 0) {
    tma_store_3d_plain(map, smem_addr(stage) + buf_off, col, row, grp);
    bulk_commit();
  }
  ++ochunk;
}

// Where this warp's 32 rows [row_base, row_base + 32) of expert g go, and which of them it
// stores: `rows_out` the map coordinates (row within the expert's C rows and group, or the
// pooled row and group 0); `keep_ab` whether the box holds a row of the expert (the ab box:
// rows past the expert's count in it are junk no one reads, and stay inside the expert's
// rows); `keep_pad` whether it starts below the count rounded up to 64 (the hg / dab box: rows
// past the count get zeros, and the box ends at or before that multiple of 64).
struct ChunkRows {
  int row, grp;
  bool keep_ab, keep_pad;
};

__device__ __forceinline__ ChunkRows chunk_rows(const GemmArgs& p, int g, int row_base) {
  ChunkRows c;
  const int n = p.rows[g];
  c.row = p.group_row ? static_cast<int>(row_of(p, g, row_base)) : row_base;
  c.grp = p.group_row ? 0 : g;
  c.keep_ab = row_base < n;
  c.keep_pad = row_base < (n + BK - 1) / BK * BK;
  return c;
}

// a, b of 32-column chunks into ab, and hg = bf16(gate * silu(a) * b), all row-major, through
// TMA stores of 32 x 32 chunks (maps: ab [.][2F], hg [.][F]). The expert's padding rows get
// zeros in hg.
__device__ __forceinline__ void epi_recompute(const GemmArgs& p, const CUtensorMap* ab_map, const CUtensorMap* hg_map,
                                              uint32_t tb, int g, int row_base, bool valid, int nt, uint8_t* stage,
                                              uint32_t& ochunk) {
  const int lane = threadIdx.x & 31;
  const ChunkRows cr = chunk_rows(p, g, row_base);
  const float gv = valid ? p.row_gate[row_of(p, g, row_base + lane)] : 0.f;
  for (int c = 0; c < p.width; c += 32) {
    uint32_t av[32], bv[32];
    tmem_ld32(tb + c, av);
    tmem_ld32(tb + p.width + c, bv);
    tmem_wait_ld();
    const int col0 = nt * p.width + c;
    uint32_t pa[16], pb[16], ph[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float a0 = __uint_as_float(av[2 * i]), a1 = __uint_as_float(av[2 * i + 1]);
      const float b0 = __uint_as_float(bv[2 * i]), b1 = __uint_as_float(bv[2 * i + 1]);
      pa[i] = gemm::pack_bf16x2(a0, a1);
      pb[i] = gemm::pack_bf16x2(b0, b1);
      ph[i] = valid ? gemm::pack_bf16x2(gv * gemm::silu_f(a0) * b0, gv * gemm::silu_f(a1) * b1) : 0u;
    }
    if (cr.keep_ab) {
      store_chunk(ab_map, pa, col0, cr.row, cr.grp, stage, ochunk);
      store_chunk(ab_map, pb, p.F + col0, cr.row, cr.grp, stage, ochunk);
    }
    if (cr.keep_pad) store_chunk(hg_map, ph, col0, cr.row, cr.grp, stage, ochunk);
  }
}

// The accumulator holds W2^T dy for 32-column chunks of the tile; a, b come from the recompute.
// [da | db] goes row-major into dab through TMA stores of 32 x 32 chunks (map dab [.][2F]); the
// expert's padding rows get zeros there.
__device__ __forceinline__ void epi_dh(const GemmArgs& p, const CUtensorMap* dab_map, uint32_t tb, int g, int row_base,
                                       bool valid, int nt, uint8_t* stage, uint32_t& ochunk) {
  const int lane = threadIdx.x & 31;
  const ChunkRows cr = chunk_rows(p, g, row_base);
  const long long rrow = row_of(p, g, row_base + lane);
  const float gv = valid ? p.row_gate[rrow] : 0.f;
  float part = 0.f;
  for (int c = 0; c < p.width; c += 32) {
    uint32_t v[32];
    tmem_ld32(tb + c, v);
    tmem_wait_ld();
    const int col0 = nt * p.width + c;
    uint32_t pda[16], pdb[16];
    if (valid) {
      const uint4* aq = reinterpret_cast<const uint4*>(p.ab + rrow * 2 * p.F + col0);
      const uint4* bq = reinterpret_cast<const uint4*>(p.ab + rrow * 2 * p.F + p.F + col0);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float af[8], bf[8];
        copy::bf16x8_to_f32(aq[u], af);
        copy::bf16x8_to_f32(bq[u], bf);
        float dav[8], dbv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float a = af[i], b = bf[i];
          const float dhu = __uint_as_float(v[8 * u + i]);
          const float sig = __fdividef(1.0f, 1.0f + __expf(-a));
          const float s = a * sig;
          part = __fmaf_rn(dhu, s * b, part);
          const float dh = gv * dhu;
          dbv[i] = dh * s;
          dav[i] = dh * b * (sig * (1.0f + a * (1.0f - sig)));
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          pda[4 * u + i] = gemm::pack_bf16x2(dav[2 * i], dav[2 * i + 1]);
          pdb[4 * u + i] = gemm::pack_bf16x2(dbv[2 * i], dbv[2 * i + 1]);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) pda[i] = pdb[i] = 0u;
    }
    if (cr.keep_pad) {
      store_chunk(dab_map, pda, col0, cr.row, cr.grp, stage, ochunk);
      store_chunk(dab_map, pdb, p.F + col0, cr.row, cr.grp, stage, ochunk);
    }
  }
  if (valid) p.dgate_part[rrow * p.dgate_ld + nt] = part;
}

// 16 accumulator columns of this warp's 32 lanes (one row each).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// kRecDh: a, b (accumulator columns [0, 64) and [64, 128)) and W2^T dy ([128, 192)) of 64 d_ff
// columns, all fp32, read 16 columns at a time. Per 32 columns: hg = bf16(gate * silu(a) * b)
// into hg, then [da | db] into dab (a and b read again), through TMA stores of 32 x 32 chunks
// (the expert's padding rows get zeros in both); the row's dgate partial <W2^T dy, h> over the
// tile's columns goes into dgate_part.
__device__ __forceinline__ void epi_recdh(const GemmArgs& p, const CUtensorMap* dab_map, const CUtensorMap* hg_map,
                                          uint32_t tb, int g, int row_base, bool valid, int nt, uint8_t* stage,
                                          uint32_t& ochunk) {
  const int lane = threadIdx.x & 31;
  const ChunkRows cr = chunk_rows(p, g, row_base);
  const long long rrow = row_of(p, g, row_base + lane);
  const float gv = valid ? p.row_gate[rrow] : 0.f;
  float part = 0.f;
  for (int c = 0; c < kRecDhWidth; c += 32) {
    const int col0 = nt * kRecDhWidth + c;
    {
      uint32_t ph[16];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t av[16], bv[16];
        tmem_ld16(tb + c + 16 * h, av);
        tmem_ld16(tb + kRecDhWidth + c + 16 * h, bv);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float a0 = __uint_as_float(av[2 * i]), a1 = __uint_as_float(av[2 * i + 1]);
          const float b0 = __uint_as_float(bv[2 * i]), b1 = __uint_as_float(bv[2 * i + 1]);
          ph[8 * h + i] = valid ? gemm::pack_bf16x2(gv * gemm::silu_f(a0) * b0, gv * gemm::silu_f(a1) * b1) : 0u;
        }
      }
      if (cr.keep_pad) store_chunk(hg_map, ph, col0, cr.row, cr.grp, stage, ochunk);
    }
    uint32_t pda[16], pdb[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t av[16], bv[16], dv[16];
      tmem_ld16(tb + c + 16 * h, av);
      tmem_ld16(tb + kRecDhWidth + c + 16 * h, bv);
      tmem_ld16(tb + 2 * kRecDhWidth + c + 16 * h, dv);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float dav[2], dbv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float a = __uint_as_float(av[2 * i + u]), b = __uint_as_float(bv[2 * i + u]);
          const float dhu = __uint_as_float(dv[2 * i + u]);
          const float sig = __fdividef(1.0f, 1.0f + __expf(-a));
          const float s = a * sig;
          part = __fmaf_rn(dhu, s * b, part);
          const float dh = gv * dhu;
          dbv[u] = dh * s;
          dav[u] = dh * b * (sig * (1.0f + a * (1.0f - sig)));
        }
        pda[8 * h + i] = valid ? gemm::pack_bf16x2(dav[0], dav[1]) : 0u;
        pdb[8 * h + i] = valid ? gemm::pack_bf16x2(dbv[0], dbv[1]) : 0u;
      }
    }
    if (cr.keep_pad) {
      store_chunk(dab_map, pda, col0, cr.row, cr.grp, stage, ochunk);
      store_chunk(dab_map, pdb, p.F + col0, cr.row, cr.grp, stage, ochunk);
    }
  }
  if (valid) p.dgate_part[rrow * p.dgate_ld + nt] = part;
}

// fp32 gradient tile row: out[g][row][nt * width + c] += accumulator (= accumulator when
// `overwrite`: round 0, the first round of every expert that has rows at all).
__device__ __forceinline__ void epi_wgrad(const GemmArgs& p, uint32_t tb, int g, int row, bool valid, int nt) {
  float* o = static_cast<float*>(p.out) + g * p.out_group_stride + static_cast<long long>(row) * p.out_ld +
             nt * p.width;
  for (int c = 0; c < p.width; c += 32) {
    uint32_t v[32];
    tmem_ld32(tb + c, v);
    tmem_wait_ld();
    if (valid) {
      float4* q = reinterpret_cast<float4*>(o + c);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float4 u = p.overwrite ? make_float4(0.f, 0.f, 0.f, 0.f) : q[i];
        u.x += __uint_as_float(v[4 * i]);
        u.y += __uint_as_float(v[4 * i + 1]);
        u.z += __uint_as_float(v[4 * i + 2]);
        u.w += __uint_as_float(v[4 * i + 3]);
        q[i] = u;
      }
    }
  }
}

// The same through TMA: each 32-column slice of the accumulator row goes to this warp's staging
// buffer as two 16-column fp32 chunks (64-byte swizzle, 32 rows by 64 bytes), which one bulk
// store (round 0) or one bulk reduce-add (later rounds) writes into the gradient. The add happens
// in the memory system; every element still gets one fp32 addition per round, in round order.
__device__ __forceinline__ void epi_wgrad_tma(const GemmArgs& p, const CUtensorMap* map, uint32_t tb, int g,
                                              int row_base, int nt, uint8_t* stage, uint32_t& ochunk) {
  const int lane = threadIdx.x & 31;
  const uint32_t stage_addr = smem_addr(stage);
  for (int c = 0; c < p.width; c += 32) {
    uint32_t v[32];
    tmem_ld32(tb + c, v);
    tmem_wait_ld();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t buf_off = (ochunk & 1u) * gemm::kOutChunkBytes;
      if (lane == 0) bulk_wait_read_1();   // the write that last used this buffer has read it
      __syncwarp();
      uint8_t* row_ptr = stage + buf_off + lane * 64;
#pragma unroll
      for (int j = 0; j < 4; ++j)   // 64-byte swizzle: piece j of row r at j ^ ((r >> 1) & 3)
        *reinterpret_cast<uint4*>(row_ptr + ((j ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(v[16 * h + 4 * j], v[16 * h + 4 * j + 1], v[16 * h + 4 * j + 2], v[16 * h + 4 * j + 3]);
      fence_async_shared();
      __syncwarp();
      if (lane == 0) {
        const int col = nt * p.width + c + 16 * h;
        if (p.overwrite)
          tma_store_3d_plain(map, stage_addr + buf_off, col, row_base, g);
        else
          tma_reduce_add_3d(map, stage_addr + buf_off, col, row_base, g);
        bulk_commit();
      }
      ++ochunk;
    }
  }
}

// ---------------------------------------------------------------- the GEMM kernel

// One launch runs up to three independent GEMMs ("phases") back to back over one tile list:
// phase 0's tiles, then phase 1's, then phase 2's. All phases share one stage geometry, because
// the ring's slot barriers assume that a slot always covers the same bytes.
//
// Two forms, as in the forward's grouped GEMM:
// - single CTA: 128-row tiles, a 128-row A tile and up to 256 B rows per stage (48 KB, 4
//   stages), M = 128 MMAs;
// - CTA pair (cta_group::2, clusters of two): 256-row tiles of 256 columns. CTA c of the pair
//   loads A rows [128 c, 128 c + 128) of the tile and B rows [128 c, 128 c + 128) of its 256
//   (recompute: c = 0 the tile's 128 W1 rows, c = 1 the same W3 rows, so that a and b land in
//   accumulator columns [0, 128) and [128, 256) as in the single-CTA form) into its own shared
//   memory (32 KB per stage, 6 stages); the leader's one thread issues the M = 256 MMAs for
//   both, and accumulator rows [128 c, 128 c + 128) land in CTA c's TMEM, where the same
//   epilogues as in the single-CTA form read them. Half the shared-memory bytes per flop.
//   Barriers: full[s] and tempty[a] in the leader, empty[s] and tfull[a] in both (the leader's
//   commits arrive on both). No load is multicast.
constexpr int kMaxPhases = 3;
constexpr int kStageBytes = gemm::kABytes + 256 * BK * 2;
constexpr int kStages = gemm::kRingBytes / kStageBytes;
static_assert(kStages >= 2 && kStages <= gemm::kMaxStages, "ring stages");
constexpr int kTileStride = gemm::kMaxGroups + 1;
// gemm::carve's layout (ring, output staging for the weight-gradient TMA writes, barriers, misc
// words), with room for a tile prefix and a pooled-column prefix per phase after the misc words.
constexpr int kSmemBytes = 1024 + gemm::kRingBytes + gemm::kOutStagingBytes + gemm::kBarBytes +
                           gemm::kMiscWords * 4 + 2 * kMaxPhases * kTileStride * 4;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

struct Launch {
  GemmArgs ph[kMaxPhases];
  int phases;
};

template <bool kPair>
__global__ void __launch_bounds__(gemm::kThreads, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap ta0, const __grid_constant__ CUtensorMap tb0,
                    const __grid_constant__ CUtensorMap ta1, const __grid_constant__ CUtensorMap tb1,
                    const __grid_constant__ CUtensorMap ta2, const __grid_constant__ CUtensorMap tb2,
                    const __grid_constant__ CUtensorMap tout1, const __grid_constant__ CUtensorMap tout2,
                    const __grid_constant__ Launch L) {
  constexpr int kRows = kPair ? gemm::kPairRows : BM;                   // rows of a tile
  constexpr int kSlot = kPair ? gemm::kPairStageBytes : kStageBytes;    // bytes of a ring slot
  constexpr int kSlots = kPair ? gemm::kPairStages : kStages;
  extern __shared__ uint8_t smem_raw[];
  const Smem s = gemm::carve(smem_raw);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&ta0);
    tma_prefetch_desc(&tb0);
  }
  const uint32_t tmem_base = kPair ? gemm::setup_pair(s) : gemm::setup(s);
  const uint32_t cta = kPair ? cluster_rank() : 0u;
  const int unit = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  int* ts[kMaxPhases];
  for (int q = 0; q < kMaxPhases; ++q) ts[q] = s.tile_start[0] + q * kTileStride;
  for (int q = 0; q < L.phases; ++q)     // reads only the round's row counts (plan data)
    plan_tiles(ts[q], L.ph[q], L.ph[q].n_total / L.ph[q].width, kRows);
  __syncthreads();
  grid_dependency_wait();
  pdl_trigger_early();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int first[kMaxPhases + 1];             // first tile of each phase in the launch's list
  first[0] = 0;
  for (int q = 0; q < kMaxPhases; ++q) first[q + 1] = first[q] + (q < L.phases ? ts[q][L.ph[q].groups] : 0);
  const int total = first[L.phases];
  auto decode = [&](int tile, int& q, int& g, int& mt, int& nt) {
    q = 0;
    while (q + 1 < L.phases && tile >= first[q + 1]) ++q;
    const GemmArgs& p = L.ph[q];
    const int* t = ts[q];
    const int local0 = tile - first[q];
    int lo = 0, hi = p.groups - 1;       // largest g with t[g] <= local0
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (t[mid] <= local0) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int n_tiles = p.n_total / p.width;
    const int local = local0 - t[g];
    mt = local / n_tiles;
    nt = local - mt * n_tiles;
  };
  auto map_a = [&](int q) { return q == 0 ? &ta0 : q == 1 ? &ta1 : &ta2; };
  auto map_b = [&](int q) { return q == 0 ? &tb0 : q == 1 ? &tb1 : &tb2; };
  auto bn_of = [&](const GemmArgs& p) { return p.mode == kRecompute || p.mode == kRecDh ? 2 * p.width : p.width; };
  Pipe pipe;
  int32_t* status = L.ph[0].status;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer (both CTAs)
      bool ok = true;
      for (int tile = unit; ok && tile < total; tile += units) {
        int q, g, mt, nt;
        decode(tile, q, g, mt, nt);
        const GemmArgs& p = L.ph[q];
        const CUtensorMap* ma = map_a(q);
        const CUtensorMap* mb = map_b(q);
        // The tile's load plan, in registers: the loop below issues only the loads and the
        // K coordinate (the TMA and barrier asm statements clobber memory, so anything read
        // from the launch arguments inside the loop would be read again at every stage).
        enum : int { kLdWgrad, kLdBmn, kLdB1, kLdB2, kLdRecDh };
        const int mode = p.mode;
        const int m0 = mt * kRows + static_cast<int>(cta) * BM;   // this CTA's first A row of the tile
        const int grp = p.group_row ? 0 : g;
        const int kbs = k_blocks_of(p, g);
        const int nkb = p.num_k_blocks;
        int ld, a_c = 0, b_c = 0, b_c2 = 0, nbox = 0;
        if (mode == kWgrad) {
          // both operands are the round's row-major buffers read MN-major, K = the expert's
          // rows (from row 0 of its C rows, or from its segment's first row): this CTA's 128
          // A columns and its B columns as 64-column boxes, 8 KB apart
          ld = kLdWgrad;
          a_c = static_cast<int>(row_of(p, g, 0)) - (p.group_row ? 0 : g * p.C);   // K base
          b_c = nt * p.width + (kPair ? static_cast<int>(cta) * gemm::kPairBHalf : 0);
          nbox = kPair ? gemm::kPairBHalf / kMnBox : p.width / kMnBox;
        } else {
          a_c = p.group_row ? static_cast<int>(row_of(p, g, m0)) : m0;   // A row
          if (!kPair && mode == kRecDh) {
            // K blocks of the recompute (x, W13 rows of the tile's gate and up columns), then
            // those of dh (dy, the tile's 64 columns of W2 as one MN-major box)
            ld = kLdRecDh;
            b_c = nt * kRecDhWidth;
            b_c2 = p.F + nt * kRecDhWidth;
          } else if (p.b_mn) {
            // MN-major weights: this CTA's B columns as 64-column boxes, 8 KB apart
            ld = kLdBmn;
            b_c = nt * p.width + (kPair ? static_cast<int>(cta) * gemm::kPairBHalf : 0);
            nbox = kPair ? gemm::kPairBHalf / kMnBox : p.width / kMnBox;
          } else if (kPair) {
            // recompute: CTA 0 the tile's W1 rows, CTA 1 the same W3 rows; else 128 of the 256
            ld = kLdB1;
            b_c = mode == kRecompute ? static_cast<int>(cta) * p.F + nt * p.width
                                     : nt * p.width + static_cast<int>(cta) * gemm::kPairBHalf;
          } else if (mode == kRecompute) {
            ld = kLdB2;
            b_c = nt * p.width;
            b_c2 = p.F + nt * p.width;
          } else {
            ld = kLdB1;
            b_c = nt * p.width;
          }
        }
        const uint32_t b2_off = static_cast<uint32_t>(p.width) * BK * 2;   // kLdB2: the up rows
        // the pair's bytes per stage land on the leader's barrier; the leader counts both halves
        const uint32_t tx0 = kPair ? 2u * gemm::kPairStageBytes
                                   : static_cast<uint32_t>(gemm::kABytes + bn_of(p) * BK * 2);
        const uint32_t tx_dh = static_cast<uint32_t>(gemm::kABytes + kMnBoxBytes);
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait(smem_addr(&s.empty[pipe.stage]), pipe.phase ^ 1u, s.abort)) {
            ok = false;
            break;
          }
          const uint32_t sA = smem_addr(s.stage + pipe.stage * kSlot);
          const uint32_t sB = sA + gemm::kABytes;
          const uint32_t fb_local = smem_addr(&s.full[pipe.stage]);
          const uint32_t fb = kPair ? peer_addr(fb_local, 0) : fb_local;
          // kRecDh's dh half: A and one 64 x 64 MN-major box of W2 per stage
          const bool dh_half = !kPair && ld == kLdRecDh && kb >= nkb;
          if (cta == 0) mbar_arrive_expect_tx(fb_local, dh_half ? tx_dh : tx0);
          auto load = [&](uint32_t dst, const CUtensorMap* m, int c0, int c1, int c2) {
            if (kPair)
              tma_load_3d_pair(dst, m, fb, c0, c1, c2);
            else
              tma_load_3d(dst, m, fb, c0, c1, c2);
          };
          const int k = kb * BK;
          if (ld == kLdWgrad) {
            for (int j = 0; j < BM / kMnBox; ++j) load(sA + j * kMnBoxBytes, ma, m0 + j * kMnBox, a_c + k, grp);
            for (int j = 0; j < nbox; ++j) load(sB + j * kMnBoxBytes, mb, b_c + j * kMnBox, a_c + k, grp);
          } else if (ld == kLdRecDh) {
            if (!dh_half) {
              load(sA, &ta0, k, a_c, grp);
              load(sB, &tb0, k, b_c, g);
              load(sB + kRecDhWidth * BK * 2, &tb0, k, b_c2, g);
            } else {
              load(sA, &ta1, k - nkb * BK, a_c, grp);
              load(sB, &tb1, b_c, k - nkb * BK, g);
            }
          } else {
            load(sA, ma, k, a_c, grp);
            if (ld == kLdBmn) {
              for (int j = 0; j < nbox; ++j) load(sB + j * kMnBoxBytes, mb, b_c + j * kMnBox, k, g);
            } else {
              load(sB, mb, k, b_c, g);
              if (ld == kLdB2) load(sB + b2_off, mb, k, b_c2, g);
            }
          }
          pipe.issued |= 1u << pipe.stage;
          pipe.issued_parity = (pipe.issued_parity & ~(1u << pipe.stage)) | (pipe.phase << pipe.stage);
          if (++pipe.stage == kSlots) {
            pipe.stage = 0;
            pipe.phase ^= 1u;
          }
        }
      }
      if (!ok) {
        atomicOr(status, kStatusTimeoutProducer);
        *s.abort = 1;
        if (kPair) {
          // loads already issued complete on the leader's barriers, which the peer cannot wait
          // on: give them time to land before the pair's shared memory is released
          const uint64_t t0 = global_timer_ns();
          while (global_timer_ns() - t0 < 200000ull) {
          }
        } else {
          for (int i = 0; i < kSlots; ++i)   // let issued loads land before the CTA exits
            if ((pipe.issued >> i) & 1u) mbar_wait(smem_addr(&s.full[i]), (pipe.issued_parity >> i) & 1u, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && cta == 0) {
      // ------------------------------------------------------------ MMA issuer (the leader)
      bool ok = true;
      for (int tile = unit; ok && tile < total; tile += units) {
        int q, g, mt, nt;
        decode(tile, q, g, mt, nt);
        const GemmArgs& p = L.ph[q];
        const uint32_t idesc =
            idesc_bf16_f32(kRows, bn_of(p)) | (p.a_mn ? kIdescAMn : 0u) | (p.b_mn ? kIdescBMn : 0u);
        // kRecDh's dh half: N = 64, B MN-major, accumulator columns from 128
        const uint32_t idesc_dh = idesc_bf16_f32(kRows, kRecDhWidth) | kIdescBMn;
        // one K step of 16: +32 B along a K-major row, +16 rows of 128 B in an MN-major box
        const uint32_t b_step = p.b_mn ? (16u * 128u) >> 4 : 2u;
        const uint32_t a_step = p.a_mn ? (16u * 128u) >> 4 : 2u;
        const int kbs = k_blocks_of(p, g);
        // in registers: the asm statements below clobber memory
        const bool a_mn = p.a_mn != 0, b_mn = p.b_mn != 0;
        const bool rec_dh = !kPair && p.mode == kRecDh;
        const int nkb = p.num_k_blocks;
        if (!mbar_wait(smem_addr(&s.tempty[pipe.acc]), pipe.acc_phase ^ 1u, s.abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(pipe.acc * gemm::kAccCols);
        for (int kb = 0; kb < kbs; ++kb) {
          if (!mbar_wait(smem_addr(&s.full[pipe.stage]), pipe.phase, s.abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_addr(s.stage + pipe.stage * kSlot);
          const uint64_t adesc = a_mn ? smem_desc_sw128_mn(sA, kMnBoxBytes) : smem_desc_sw128(sA);
          if (rec_dh && kb >= nkb) {
            const int kd = kb - nkb;
            const uint64_t bdesc = smem_desc_sw128_mn(sA + gemm::kABytes, kMnBoxBytes);
            const uint32_t mn_step = (16u * 128u) >> 4;
#pragma unroll
            for (int kk = 0; kk < BK / gemm::UMMA_K; ++kk)
              mma_bf16(d_tmem + 2 * kRecDhWidth, adesc + 2u * kk, bdesc + mn_step * kk, idesc_dh,
                       (kd | kk) != 0 ? 1u : 0u);
          } else {
            const uint64_t bdesc = b_mn ? smem_desc_sw128_mn(sA + gemm::kABytes, kMnBoxBytes)
                                        : smem_desc_sw128(sA + gemm::kABytes);
#pragma unroll
            for (int kk = 0; kk < BK / gemm::UMMA_K; ++kk) {
              if (kPair)
                mma_bf16_pair(d_tmem, adesc + a_step * kk, bdesc + b_step * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
              else
                mma_bf16(d_tmem, adesc + a_step * kk, bdesc + b_step * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
          }
          if (kPair)
            mma_commit_pair(smem_addr(&s.empty[pipe.stage]), 3);
          else
            mma_commit(smem_addr(&s.empty[pipe.stage]));
          if (++pipe.stage == kSlots) {
            pipe.stage = 0;
            pipe.phase ^= 1u;
          }
        }
        if (!ok) break;
        if (kPair)
          mma_commit_pair(smem_addr(&s.tfull[pipe.acc]), 3);
        else
          mma_commit(smem_addr(&s.tfull[pipe.acc]));
        pipe.acc ^= 1;
        if (pipe.acc == 0) pipe.acc_phase ^= 1u;
      }
      if (!ok) {
        atomicOr(status, kStatusTimeoutMma);
        *s.abort = 1;
        if (kPair)
          mma_commit_pair(smem_addr(s.drain), 1);   // wait for every MMA already issued
        else
          mma_commit(smem_addr(s.drain));
        mbar_wait(smem_addr(s.drain), 0, nullptr);
      }
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue (warps 2..5)
    const int qw = warp & 3;
    uint32_t ochunk = 0;   // fp32 chunks this warp has staged (alternates its two buffers)
    uint8_t* stage = s.out_stage + qw * 2 * gemm::kOutChunkBytes;
    for (int tile = unit; tile < total; tile += units) {
      int q, g, mt, nt;
      decode(tile, q, g, mt, nt);
      const GemmArgs& p = L.ph[q];
      const bool ready =
          __all_sync(0xffffffffu, mbar_wait(smem_addr(&s.tfull[pipe.acc]), pipe.acc_phase, s.abort));
      if (!ready) {
        if (lane == 0) atomicOr(status, kStatusTimeoutEpilogue);
        *s.abort = 1;
        break;
      }
      tc_fence_after();
      const int row0 = mt * kRows + static_cast<int>(cta) * BM + qw * 32;   // this warp's first row
      const int row = row0 + lane;
      const bool valid = row < (p.mode == kWgrad ? p.m_total : p.rows[g]);
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(qw * 32) << 16) +
                             static_cast<uint32_t>(pipe.acc * gemm::kAccCols);
      if (p.mode == kRecompute) {
        epi_recompute(p, &tout1, &tout2, tbase, g, row0, valid, nt, stage, ochunk);
      } else if (p.mode == kDh) {
        epi_dh(p, &tout1, tbase, g, row0, valid, nt, stage, ochunk);
      } else if (p.mode == kRecDh) {
        if constexpr (!kPair) epi_recdh(p, &tout1, &tout2, tbase, g, row0, valid, nt, stage, ochunk);
      } else if (p.mode == kDx) {
        uint16_t* orow = static_cast<uint16_t*>(p.out) + row_of(p, g, row) * p.out_ld + nt * p.width;
        gemm::store_bf16(tbase, p.width, orow, valid);
      } else if (p.tma_out) {
        epi_wgrad_tma(p, q == 1 ? &tout1 : &tout2, tbase, g, row0, nt, stage, ochunk);
      } else {
        epi_wgrad(p, tbase, g, row, valid, nt);
      }
      tc_fence_before();
      if (kPair) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(peer_addr(smem_addr(&s.tempty[pipe.acc]), 0));
      } else {
        mbar_arrive(smem_addr(&s.tempty[pipe.acc]));
      }
      pipe.acc ^= 1;
      if (pipe.acc == 0) pipe.acc_phase ^= 1u;
    }
    if (lane == 0 && ochunk > 0) bulk_wait_all();   // the gradient writes are done before exit
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  pdl_trigger_late();
  if (kPair)
    gemm::release_tmem_pair(tmem_base);
  else
    gemm::release_tmem(tmem_base);
}

// ---------------------------------------------------------------- copy and small kernels

constexpr int kWarps = 8;

// Dispatch of round r. A block takes 64 rows of one expert's rows in the round and 256 columns
// (c0 = 256 * blockIdx.y): the rows' tokens come from the round-major row list (row_off[r][e] +
// s); their x and dy slices are copied into xbuf and dybuf (dy as bf16). The expert's padding
// rows (from n[r][e] up to the next multiple of 64, within its C rows or its pooled segment) get
// zeros: the weight-gradient GEMMs read the rows as K in blocks of 64. The blocks of the first
// column slice also write each row's gate.
// The grid's x covers only the round's rows: block b is the b-th 64-row block in expert order
// (expert e holds ceil(n[r][e] / 64) of them), so a round with few rows launches few blocks.
// Rows s of expert e are at e * C + s, or with pooled rows at 64 b + (s mod 64): each expert's
// segment starts at a multiple of 64 (the table seg_off the GEMMs and the combine read).
constexpr int kGatherCols = 256;   // columns of a gather block (8 per lane)

struct GatherArgs {
  const uint16_t* x;
  const float* dy;
  const int32_t* idx;
  const float* gate;
  const int32_t* n;           // [max_rounds, E]
  const int32_t* row_off;     // [max_rounds, E] first row of (round, expert) in the row list
  const int32_t* row_token;
  uint16_t* xbuf;
  uint16_t* dybuf;
  float* row_gate;
  int r, E, C, d, k, pooled;
};

// Block (bx, by) of the gather: 64 rows (the bx-th 64-row block of the round) x kGatherCols
// columns (c0 = kGatherCols by). The whole block runs it (256 threads).
__device__ __forceinline__ void gather_block(const GatherArgs& a, int bx, int by) {
  __shared__ int tok[64];
  __shared__ int blk[3];      // expert, its first row in this block, its rows in the round
  const int c0 = by * kGatherCols;
  const int32_t* nr = a.n + static_cast<size_t>(a.r) * a.E;
  if (threadIdx.x < 32) {
    // warp 0: the expert whose 64-row blocks hold block b (a running prefix over the experts)
    const int lane = threadIdx.x;
    const int b = bx;
    int acc = 0, found = -1, first = 0, rows = 0;
    for (int x0 = 0; x0 < a.E; x0 += 32) {
      const int x = x0 + lane;
      const int nx = x < a.E ? nr[x] : 0;
      const int cnt = (nx + 63) / 64;
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const int excl = acc + incl - cnt;
      const unsigned hit = __ballot_sync(0xffffffffu, cnt > 0 && b >= excl && b < excl + cnt);
      if (hit != 0u) {
        const int src = __ffs(hit) - 1;
        found = x0 + src;
        first = (b - __shfl_sync(0xffffffffu, excl, src)) * 64;
        rows = __shfl_sync(0xffffffffu, nx, src);
        break;
      }
      acc += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      blk[0] = found;
      blk[1] = first;
      blk[2] = rows;
    }
  }
  __syncthreads();
  const int e = blk[0], s0 = blk[1], ne = blk[2];
  if (e >= 0) {
    const int base = a.row_off[static_cast<size_t>(a.r) * a.E + e];
    // row-major row of s = 0 (pooled: this block's first row is 64 b)
    const long long dst0 = a.pooled ? static_cast<long long>(bx) * 64 - s0
                                    : static_cast<long long>(e) * a.C;
    if (threadIdx.x < 64) {
      const int sr = s0 + threadIdx.x;
      tok[threadIdx.x] = sr < ne ? a.row_token[base + sr] : -1;
    }
    __syncthreads();
    // 32 x 8 threads: a lane takes 8 columns (16-byte x and bf16 dy stores, two 16-byte dy
    // loads), a warp 256 columns of one row at a time
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int c = c0 + 8 * tx;
    if (c < a.d) {
#pragma unroll 4
      for (int i = 0; i < 8; ++i) {
        const int rr = ty + 8 * i;
        const int sr = s0 + rr;
        if (!a.pooled && sr >= a.C) continue;   // past the expert's C rows: the next expert's
        const int t = tok[rr];
        uint4 xv = make_uint4(0u, 0u, 0u, 0u), yv = make_uint4(0u, 0u, 0u, 0u);
        if (t >= 0) {
          xv = __ldg(reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.d + c));
          const float4* dq = reinterpret_cast<const float4*>(a.dy + static_cast<size_t>(t) * a.d + c);
          const float4 d0 = __ldg(dq), d1 = __ldg(dq + 1);
          yv = make_uint4(gemm::pack_bf16x2(d0.x, d0.y), gemm::pack_bf16x2(d0.z, d0.w), gemm::pack_bf16x2(d1.x, d1.y),
                          gemm::pack_bf16x2(d1.z, d1.w));
        }
        const size_t orow = static_cast<size_t>(dst0 + sr) * a.d + c;
        *reinterpret_cast<uint4*>(a.xbuf + orow) = xv;
        *reinterpret_cast<uint4*>(a.dybuf + orow) = yv;
      }
    }
    if (c0 == 0 && threadIdx.x < 64) {
      const int t = tok[threadIdx.x];
      if (t >= 0) {
        int j = 0;
        while (j + 1 < a.k && a.idx[static_cast<size_t>(t) * a.k + j] != e) ++j;
        a.row_gate[dst0 + s0 + threadIdx.x] = a.gate[static_cast<size_t>(t) * a.k + j];
      }
    }
  }
}

__global__ void __launch_bounds__(256) bwd_gather_kernel(const __grid_constant__ GatherArgs a) {
  grid_dependency_wait();
  gather_block(a, static_cast<int>(blockIdx.x), static_cast<int>(blockIdx.y));
  pdl_trigger_early();
  pdl_trigger_late();
}

// The pooled segment table of rounds 0 .. R-1 (one block per round): seg_off[r][e] = the sum over
// e' < e of n[r][e'] rounded up to 64, and zeros[r] = 0 (zeros[R] too).
__global__ void __launch_bounds__(32) seg_table_kernel(const int32_t* __restrict__ n, int E, int32_t* seg_off,
                                                       int32_t* zeros) {
  grid_dependency_wait();
  const int r = blockIdx.x, lane = threadIdx.x;
  const int32_t* nr = n + static_cast<size_t>(r) * E;
  int running = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    const int cnt = e < E ? (nr[e] + 63) / 64 * 64 : 0;
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (e < E) seg_off[static_cast<size_t>(r) * E + e] = running + incl - cnt;
    running += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    zeros[r] = 0;
    if (r == static_cast<int>(gridDim.x) - 1) zeros[r + 1] = 0;
  }
  pdl_trigger_early();
  pdl_trigger_late();
}

// One warp per token with pairs in round r: dx[t] (+)= its pairs' dxbuf rows (gate 1, ascending j),
// dgate[t, j] = sum over the row's `parts` partials, in order.
// The combine's arguments besides the copy step's.
struct CombineExtra {
  int r;
  const float* dgate_part;
  int dgate_ld, parts;
  float* dgate;
};

// Block `block` of `blocks` blocks of the combine (kWarps warps each).
__device__ __forceinline__ void combine_blocks(const copy::CombineArgs& a, const CombineExtra& x, int block,
                                               int blocks) {
  const int r = x.r, parts = x.parts, dgate_ld = x.dgate_ld;
  const float* __restrict__ dgate_part = x.dgate_part;
  float* __restrict__ dgate = x.dgate;
  const int lane = threadIdx.x & 31;
  const int warps = blocks * kWarps;
  for (int t = block * kWarps + (threadIdx.x >> 5); t < a.T; t += warps) {
    const copy::PairLoads l = copy::load_pairs(a, t);
    const copy::TokenPairs tp = copy::token_pairs(a, l, r);
    if (tp.npairs == 0) continue;
    copy::accumulate_token<8>(a, t, tp);
    const uint32_t here = __ballot_sync(0xffffffffu, l.round == r);
    if (lane < tp.npairs) {
      const int j = static_cast<int>(__fns(here, 0, lane + 1));
      const float* pr = dgate_part + tp.prow * dgate_ld;
      float sum = 0.f;
      for (int i = 0; i < parts; ++i) sum += pr[i];
      dgate[static_cast<size_t>(t) * a.k + j] = sum;
    }
  }
}

__global__ void __launch_bounds__(32 * kWarps) bwd_combine_kernel(const copy::CombineArgs a, const CombineExtra x) {
  grid_dependency_wait();
  combine_blocks(a, x, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x));
  pdl_trigger_early();
  pdl_trigger_late();
}

// The combine of round r (blocks [0, comb_blocks)) and the gather of round r + 1 (the other
// blocks, gather block (b mod gx, b / gx) for b = blockIdx.x - comb_blocks) in one launch: the
// combine reads only dxbuf and the dgate partials, which the gather does not write, and the
// gather writes only what round r's GEMMs have finished reading.
__global__ void __launch_bounds__(32 * kWarps)
    bwd_combine_gather_kernel(const copy::CombineArgs a, const CombineExtra x, const __grid_constant__ GatherArgs g,
                              int comb_blocks, int gx) {
  static_assert(32 * kWarps == 256, "the gather's blocks are 256 threads");
  grid_dependency_wait();
  const int b = static_cast<int>(blockIdx.x);
  if (b < comb_blocks) {
    combine_blocks(a, x, b, comb_blocks);
  } else {
    const int bg = b - comb_blocks;
    gather_block(g, bg % gx, bg / gx);
  }
  pdl_trigger_early();
  pdl_trigger_late();
}

// One warp per token: dz[t, e] = p_e (dp_e - sum_e' p_e' dp_e'), p = softmax(z[t]) in fp32,
// dp_e = the token's dgate of expert e (0 if not selected); with renormalised gates
// dp_{e_j} = (dgate_j - sum_i g_i dgate_i) / sum_i p_{e_i}.
__global__ void __launch_bounds__(32 * kWarps)
    gate_grad_kernel(const float* __restrict__ z, const int32_t* __restrict__ idx,
                     const float* __restrict__ dgate, int T, int E, int k, int renorm, float* __restrict__ dz) {
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * kWarps;
  for (int t = blockIdx.x * kWarps + (threadIdx.x >> 5); t < T; t += warps) {
    const float* zt = z + static_cast<size_t>(t) * E;
    float m = __int_as_float(0xff800000);   // -inf
    for (int e = lane; e < E; e += 32) m = fmaxf(m, zt[e]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float S = 0.f;
    for (int e = lane; e < E; e += 32) S += __expf(zt[e] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) S += __shfl_xor_sync(0xffffffffu, S, off);
    const float invS = 1.0f / S;
    int ej = -1;
    float psel = 0.f, dg = 0.f;
    if (lane < k) {
      ej = idx[static_cast<size_t>(t) * k + lane];
      psel = __expf(zt[ej] - m) * invS;
      dg = dgate[static_cast<size_t>(t) * k + lane];
    }
    float dps = dg;
    if (renorm) {
      float ssel = psel;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ssel += __shfl_xor_sync(0xffffffffu, ssel, off);
      float gd = psel * dg;           // sum_i g_i dgate_i = (sum_i p_i dgate_i) / ssel
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) gd += __shfl_xor_sync(0xffffffffu, gd, off);
      dps = lane < k ? (dg - gd / ssel) / ssel : 0.f;
    }
    float c = psel * dps;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      float dpe = 0.f;
      for (int j = 0; j < k; ++j) {
        const int ejj = __shfl_sync(0xffffffffu, ej, j);
        const float dpj = __shfl_sync(0xffffffffu, dps, j);
        if (ejj == e) dpe = dpj;
      }
      if (e < E) dz[static_cast<size_t>(t) * E + e] = __expf(zt[e] - m) * invS * (dpe - c);
    }
  }
  pdl_trigger_early();
  pdl_trigger_late();
}

__global__ void __launch_bounds__(256) fill_kernel(float* __restrict__ p, long long n, float v) {
  grid_dependency_wait();
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n; i += static_cast<long long>(gridDim.x) * 256)
    p[i] = v;
  pdl_trigger_early();
  pdl_trigger_late();
}

}  // namespace bwd

// ---------------------------------------------------------------- host side

namespace {

int grid_for(long long warps_needed) {
  const long long blocks = (warps_needed + bwd::kWarps - 1) / bwd::kWarps;
  const long long cap = 8ll * num_sms();
  return static_cast<int>(blocks < 1 ? 1 : blocks < cap ? blocks : cap);
}

// The candidate N width (dividing n_total) with the least streaming time: each SM streams a
// tile's 128 A rows and its B rows (width x b_per_col) over the same K, once per wave of
// tiles, so the time goes as waves x (128 + width x b_per_col). Ties go to the wider tile
// (fewer A re-reads in all). b_per_col: 2 for the recompute (W1 and W3 rows), else 1.
int pick_width(const int* widths, int n_widths, long long mtiles, int n_total, int b_per_col = 1) {
  int best = -1;
  long long best_cost = 0;
  for (int i = 0; i < n_widths; ++i) {
    if (n_total % widths[i] != 0) continue;
    const long long tiles = mtiles * (n_total / widths[i]);
    const long long waves = (tiles + num_sms() - 1) / num_sms();
    const long long cost = waves * (gemm::BM + static_cast<long long>(widths[i]) * b_per_col);
    if (best < 0 || cost < best_cost || (cost == best_cost && widths[i] > best)) {
      best = widths[i];
      best_cost = cost;
    }
  }
  return best;
}

#ifndef MOE_BWD_PAIR
#define MOE_BWD_PAIR 1   // 0: the backward GEMMs never use the CTA-pair form
#endif

// Sets the kernels' shared-memory size once per device; false on failure.
bool configure_kernels() {
  static std::atomic<uint64_t> configured{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (configured.load() & bit) return true;
  if (cudaFuncSetAttribute(bwd::bwd_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           bwd::kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(bwd::bwd_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           bwd::kSmemBytes) != cudaSuccess)
    return false;
  configured.fetch_or(bit);
  return true;
}

// Clusters of two of the pair form that fit on the device at once (one CTA per SM), per device
// ordinal; -1 when the pair form cannot run.
int pair_clusters() {
  static std::atomic<int> cached[64];
  int dev = 0;
  cudaGetDevice(&dev);
  dev &= 63;
  int v = cached[dev].load();
  if (v != 0) return v;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  cfg.blockDim = dim3(gemm::kThreads);
  cfg.dynamicSmemBytes = bwd::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (!configure_kernels() || cudaOccupancyMaxActiveClusters(&n, bwd::bwd_gemm_kernel<true>, &cfg) != cudaSuccess ||
      n <= 0) {
    cudaGetLastError();
    n = -1;
  }
  cached[dev].store(n);
  return n;
}

// Row blocks of the round: 256-row blocks (pair form) and the rows that 256- and 128-row tiles
// cover.
struct RowBlocks {
  long long blocks256 = 0, rows256 = 0, rows128 = 0;
};

RowBlocks row_blocks(const int32_t* n_host, int E) {
  RowBlocks b;
  for (int g = 0; g < E; ++g) {
    const long long p = (n_host[g] + gemm::kPairRows - 1) / gemm::kPairRows;
    b.blocks256 += p;
    b.rows256 += p * gemm::kPairRows;
    b.rows128 += static_cast<long long>((n_host[g] + gemm::BM - 1) / gemm::BM) * gemm::BM;
  }
  return b;
}

// Whether a launch whose tiles are the round's 256-row blocks x n_tiles runs in the pair form:
// enough tiles for every cluster, and at most 15% more rows than 128-row tiles would cover.
bool use_pair(const RowBlocks& b, long long n_tiles) {
  if (!MOE_BWD_PAIR || n_tiles <= 0) return false;
  const int clusters = pair_clusters();
  return clusters > 0 && b.blocks256 * n_tiles >= clusters && b.rows256 * 100 <= b.rows128 * 115;
}

// One launch of up to three GEMM phases (maps a[q], b[q], args[q]); tiles = the sum of their tiles
// (single-CTA form; the pair form runs one cluster per pair of SMs and counts tiles on the device).
// out: the epilogues' TMA-store maps out[1] and out[2] (the recompute's ab and hg, dh's dab, or
// the fp32 weight gradients of phases 1 and 2), or null.
cudaError_t run_gemm(const CUtensorMap* a, const CUtensorMap* b, const bwd::GemmArgs* args, int phases,
                     long long tiles, int kind, cudaStream_t stream, const CUtensorMap* out = nullptr,
                     bool pair = false) {
  if (tiles <= 0) return cudaSuccess;
  if (!configure_kernels()) return cudaGetLastError();
  bwd::Launch L{};
  L.phases = phases;
  for (int q = 0; q < phases; ++q) L.ph[q] = args[q];
  // kRecDh (one phase) reads its dh operands through the second map pair
  const bool rec_dh = args[0].mode == bwd::kRecDh;
  const CUtensorMap& a1 = a[phases > 1 || rec_dh ? 1 : 0];
  const CUtensorMap& b1 = b[phases > 1 || rec_dh ? 1 : 0];
  const CUtensorMap& a2 = a[phases > 2 ? 2 : 0];
  const CUtensorMap& b2 = b[phases > 2 ? 2 : 0];
  const CUtensorMap& o1 = out ? out[1] : a[0];   // unused unless an epilogue stores through TMA
  const CUtensorMap& o2 = out ? out[2] : a[0];
  launch_begin(kind, stream);
  cudaError_t err;
  if (pair) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pair_clusters());
    cfg.blockDim = dim3(gemm::kThreads);
    cfg.dynamicSmemBytes = bwd::kSmemBytes;
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
    err = cudaLaunchKernelEx(&cfg, bwd::bwd_gemm_kernel<true>, a[0], b[0], a1, b1, a2, b2, o1, o2, L);
  } else {
    // the fewest CTAs that take the tiles in as many waves as one CTA per SM would: the SMs left
    // over serve the other stream's launches when two rounds overlap
    const long long waves = (tiles + num_sms() - 1) / num_sms();
    const int grid = static_cast<int>((tiles + waves - 1) / waves);
    err = launch_pdl(bwd::bwd_gemm_kernel<false>, dim3(grid), dim3(gemm::kThreads), bwd::kSmemBytes, stream, a[0],
                     b[0], a1, b1, a2, b2, o1, o2, L);
  }
  launch_end(kind, stream);
  return err;
}

}  // namespace

long long backward_rows(int E, int C, bool pooled) {
  return static_cast<long long>(E) * C + (pooled ? 64ll * E : 0ll);
}

long long backward_rows2(int E, int C) {
  const long long eighth = (static_cast<long long>(E) * C + 7) / 8;
  return (eighth + 63) / 64 * 64 + 64ll * E;
}

cudaError_t launch_backward_prepare(const BackwardArgs& a, const int32_t* load_host, int R, cudaStream_t stream) {
  const int E = a.E, d = a.d, F = a.F;
  cudaError_t e;
  // Round 0 holds every expert that has rows at all (an expert with rows in round r > 0 has C
  // in round 0), and its weight-gradient tiles are stored, not added: only experts without
  // rows need zeroing.
  const size_t per13 = static_cast<size_t>(2) * F * d, per2 = static_cast<size_t>(d) * F;
  for (int x = 0; x < E; ++x) {
    if (load_host[x] > 0) continue;
    if ((e = cudaMemsetAsync(a.dw_gate_up + x * per13, 0, per13 * 4, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.dw_down + x * per2, 0, per2 * 4, stream)) != cudaSuccess) return e;
  }
  if (R > 0) {   // the pooled segment table (read only with pooled rows; cheap either way)
    launch_begin(kKindBackwardCopy, stream);
    e = launch_pdl(bwd::seg_table_kernel, dim3(R), dim3(32), 0, stream, a.n, E, a.seg_off, a.zeros);
    launch_end(kKindBackwardCopy, stream);
    if (e != cudaSuccess) return e;
  }
  const long long pairs = static_cast<long long>(a.T) * a.k;
  if (pairs > 0) {
    launch_begin(kKindBackwardCopy, stream);
    e = launch_pdl(bwd::fill_kernel, dim3(static_cast<unsigned>((pairs + 255) / 256 < 4096 ? (pairs + 255) / 256 : 4096)),
                   dim3(256), 0, stream, a.ones, pairs, 1.0f);
    launch_end(kKindBackwardCopy, stream);
  }
  return e;
}

namespace {

// The gather of round r: its arguments and its 64-row blocks, expert by expert.
bwd::GatherArgs gather_args(const BackwardArgs& a, int r) {
  return bwd::GatherArgs{a.x, a.dy, a.idx, a.gate, a.n, a.row_off, a.row_token, a.xbuf, a.dybuf,
                         a.row_gate, r, a.E, a.C, a.d, a.k, a.pooled != 0 ? 1 : 0};
}

long long gather_blocks(const int32_t* n_host, int E) {
  long long blocks = 0;
  for (int x = 0; x < E; ++x) blocks += (n_host[x] + 63) / 64;
  return blocks;
}

}  // namespace

namespace {

// What the launches of one round share: the round's row counts, its row blocks and the GEMMs'
// common arguments, and the round buffers' 3-D map extents ([E][C][K] per expert, or pooled
// [1][rows][K]).
struct RoundGeom {
  long long mt = 0;     // 128-row blocks of the round
  int active = 0;       // experts with rows
  RowBlocks rb;
  bwd::GemmArgs base{};
  uint64_t a_rows = 0, groups = 0;
};

RoundGeom round_geom(const BackwardArgs& a, int r, const int32_t* n_host) {
  RoundGeom q;
  const int E = a.E;
  const bool pooled = a.pooled != 0;
  for (int g = 0; g < E; ++g) {
    q.mt += (n_host[g] + gemm::BM - 1) / gemm::BM;
    q.active += n_host[g] > 0 ? 1 : 0;
  }
  q.rb = row_blocks(n_host, E);
  q.base.rows = a.n + static_cast<size_t>(r) * E;
  q.base.groups = E;
  q.base.C = a.C;
  q.base.F = a.F;
  q.base.group_row = pooled ? a.seg_off + static_cast<size_t>(r) * E : nullptr;   // 64-aligned segments
  q.base.group_row_base = pooled ? a.zeros + r : nullptr;
  q.base.status = a.status;
  q.a_rows = pooled ? static_cast<uint64_t>(a.rows) : static_cast<uint64_t>(a.C);
  q.groups = pooled ? 1 : static_cast<uint64_t>(E);
  return q;
}

constexpr int kWide[3] = {256, 128, 64};

}  // namespace

namespace {

constexpr int kRecW[3] = {128, 64, 32};   // the recompute's tile widths (gate columns)

// How a round's front half runs: `pair` when either GEMM takes the CTA-pair form (then as two
// launches); else as one fused recompute + dh launch (kRecDh) when that streams less per SM than
// the two launches, counting a launch as 550 KB of streaming (about 5.5 us at 100 GB/s per SM).
// Costs are in rows of K = d per SM: waves x (A rows + B rows) of each launch. `tiles`: the most
// tiles of one of its launches.
struct FrontPlan {
  bool pair = false, fused = false;
  int w_rec = 0, w_dh = 0;
  long long tiles = 0;
};

FrontPlan front_plan(const int32_t* n_host, int E, int d, int F) {
  FrontPlan f;
  long long mt = 0;
  for (int g = 0; g < E; ++g) mt += (n_host[g] + gemm::BM - 1) / gemm::BM;
  const RowBlocks rb = row_blocks(n_host, E);
  f.pair = (F % 128 == 0 && use_pair(rb, F / 128)) || (F % 256 == 0 && use_pair(rb, F / 256));
  f.w_rec = pick_width(kRecW, 3, mt, F, 2);
  f.w_dh = pick_width(kWide, 3, mt, F);
  const long long sms = num_sms();
  auto waves = [&](long long tiles) { return (tiles + sms - 1) / sms; };
  const long long t_rec = mt * (F / f.w_rec), t_dh = mt * (F / f.w_dh), t_f = mt * (F / bwd::kRecDhWidth);
  const long long separate = waves(t_rec) * (gemm::BM + 2 * f.w_rec) + waves(t_dh) * (gemm::BM + f.w_dh) +
                             (550ll * 1024) / (2ll * d);
  const long long fused = waves(t_f) * (gemm::BM + 2 * bwd::kRecDhWidth + gemm::BM + bwd::kRecDhWidth);
  f.fused = !f.pair && F % bwd::kRecDhWidth == 0 && fused < separate;
  f.tiles = f.fused ? t_f : (t_rec > t_dh ? t_rec : t_dh);
  return f;
}

}  // namespace

bool backward_front_is_thin(const BackwardArgs& a, const int32_t* n_host) {
  const FrontPlan f = front_plan(n_host, a.E, a.d, a.F);
  return !f.pair && f.tiles <= num_sms();
}

cudaError_t launch_backward_front(const BackwardArgs& a, int r, const int32_t* n_host, bool gather, int* parts_out,
                                  cudaStream_t stream) {
  const int E = a.E, d = a.d, F = a.F;
  cudaError_t e;
  // dispatch x and dy; the rows' gates
  if (gather) {
    const long long blocks = gather_blocks(n_host, E);
    if (blocks > 0) {
      launch_begin(kKindBackwardCopy, stream);
      e = launch_pdl(bwd::bwd_gather_kernel, dim3(static_cast<unsigned>(blocks), (d + bwd::kGatherCols - 1) / bwd::kGatherCols), dim3(256), 0, stream,
                     gather_args(a, r));
      launch_end(kKindBackwardCopy, stream);
      if (e != cudaSuccess) return e;
    }
  }
  const RoundGeom q = round_geom(a, r, n_host);
  const long long mt = q.mt;
  const RowBlocks& rb = q.rb;
  const bwd::GemmArgs& base = q.base;
  const uint64_t a_rows = q.a_rows, groups = q.groups;
  // pair form: 256-row tiles, 128 B rows per CTA (recompute: 128 W1 rows and the same W3 rows)
  const uint32_t pair_box = gemm::kPairBHalf;

  const FrontPlan fp = front_plan(n_host, E, d, F);
  // single-CTA form: recompute and dh of the same 64 d_ff columns in one tile (a, b stay in TMEM)
  if (fp.fused) {
    constexpr int w = bwd::kRecDhWidth;
    bwd::GemmArgs g = base;
    g.mode = bwd::kRecDh;
    g.width = w;
    g.n_total = F;
    g.num_k_blocks = d / gemm::BK;
    g.out = a.dab;
    g.row_gate = a.row_gate;
    g.dgate_part = a.dgate_part;
    g.dgate_ld = F / 64;
    CUtensorMap ma[2], mb[2], mo[3];
    if ((e = gemm::make_map(&ma[0], a.xbuf, d, a_rows, groups, gemm::BM)) != cudaSuccess ||
        (e = gemm::make_map(&mb[0], a.w_gate_up, d, 2ull * F, E, w)) != cudaSuccess ||
        (e = gemm::make_map(&ma[1], a.dybuf, d, a_rows, groups, gemm::BM)) != cudaSuccess ||
        (e = gemm::make_map(&mb[1], a.w_down, F, d, E, bwd::kMnBox, bwd::kMnBox)) != cudaSuccess)
      return e;
    // the epilogue's TMA stores: 1 = dab [.][2F], 2 = hg [.][F], 32 x 32 chunks
    if ((e = gemm::make_map(&mo[1], a.dab, 2ull * F, a_rows, groups, 32, gemm::kOutChunkCols)) != cudaSuccess ||
        (e = gemm::make_map(&mo[2], a.hg, F, a_rows, groups, 32, gemm::kOutChunkCols)) != cudaSuccess)
      return e;
    mo[0] = mo[1];
    if ((e = run_gemm(ma, mb, &g, 1, mt * (F / w), kKindBackwardRecDh, stream, mo, false)) != cudaSuccess) return e;
    *parts_out = F / w;
    return cudaSuccess;
  }

  // recompute: [a | b] = xbuf W13^T
  {
    const bool pair = F % 128 == 0 && use_pair(rb, F / 128);
    bwd::GemmArgs g = base;
    g.mode = bwd::kRecompute;
    g.width = pair ? 128 : fp.w_rec;
    g.n_total = F;
    g.num_k_blocks = d / gemm::BK;
    g.out = a.ab;
    g.row_gate = a.row_gate;
    CUtensorMap ma, mb;
    if ((e = gemm::make_map(&ma, a.xbuf, d, a_rows, groups, gemm::BM)) != cudaSuccess) return e;
    if ((e = gemm::make_map(&mb, a.w_gate_up, d, 2ull * F, E, pair ? pair_box : static_cast<uint32_t>(g.width))) !=
        cudaSuccess)
      return e;
    CUtensorMap mo[3];   // the epilogue's TMA stores: 1 = ab [.][2F], 2 = hg [.][F], 32 x 32 chunks
    if ((e = gemm::make_map(&mo[1], a.ab, 2ull * F, a_rows, groups, 32, gemm::kOutChunkCols)) != cudaSuccess ||
        (e = gemm::make_map(&mo[2], a.hg, F, a_rows, groups, 32, gemm::kOutChunkCols)) != cudaSuccess)
      return e;
    mo[0] = mo[1];
    if ((e = run_gemm(&ma, &mb, &g, 1, mt * (F / g.width), kKindBackwardRecompute, stream, mo, pair)) !=
        cudaSuccess)
      return e;
  }
  // dh = W2^T dy with the SwiGLU backward in its epilogue
  int parts = 0;
  {
    const bool pair = F % 256 == 0 && use_pair(rb, F / 256);
    bwd::GemmArgs g = base;
    g.mode = bwd::kDh;
    g.width = pair ? 256 : fp.w_dh;
    parts = F / g.width;
    g.n_total = F;
    g.num_k_blocks = d / gemm::BK;
    g.out = a.dab;
    g.ab = a.ab;
    g.row_gate = a.row_gate;
    g.dgate_part = a.dgate_part;
    g.dgate_ld = F / 64;
    CUtensorMap ma, mb;
    if ((e = gemm::make_map(&ma, a.dybuf, d, a_rows, groups, gemm::BM)) != cudaSuccess) return e;
    g.b_mn = 1;   // B[n = column of d_ff][k = column of d] = W2[k][n]: W2 as stored, MN-major
    if ((e = gemm::make_map(&mb, a.w_down, F, d, E, bwd::kMnBox, bwd::kMnBox)) != cudaSuccess) return e;
    CUtensorMap mo[3];   // the epilogue's TMA stores: 1 = dab [.][2F], 32 x 32 chunks
    if ((e = gemm::make_map(&mo[1], a.dab, 2ull * F, a_rows, groups, 32, gemm::kOutChunkCols)) != cudaSuccess) return e;
    mo[0] = mo[2] = mo[1];
    if ((e = run_gemm(&ma, &mb, &g, 1, mt * parts, kKindBackwardDh, stream, mo, pair)) != cudaSuccess) return e;
  }
  *parts_out = parts;
  return cudaSuccess;
}

cudaError_t launch_backward_back(const BackwardArgs& a, int r, const int32_t* n_host, int parts,
                                 const BackwardArgs* a_next, const int32_t* n_next, cudaStream_t stream) {
  const int E = a.E, C = a.C, d = a.d, F = a.F;
  const bool pooled = a.pooled != 0;
  cudaError_t e;
  const RoundGeom q = round_geom(a, r, n_host);
  const long long mt = q.mt;
  const int active = q.active;
  const RowBlocks& rb = q.rb;
  const bwd::GemmArgs& base = q.base;
  const uint64_t a_rows = q.a_rows, groups = q.groups;
  // one launch: dx rows = dab W13, dW2 (+)= dy^T hg and dW13 (+)= dab^T x over K = the round's
  // rows of each expert (both operands the row-major round buffers, read MN-major)
  {
    // the weight gradients' tiles cover d x F and 2F x d per active expert whatever the round's
    // rows; the dx phase decides, as in the other launches
    const bool pair = d % 256 == 0 && F % 256 == 0 && use_pair(rb, d / 256);
    bwd::GemmArgs g[3] = {base, base, base};
    CUtensorMap ma[3], mb[3], mo[3];
    long long tiles = 0;
    g[0].mode = bwd::kDx;
    // single-CTA form: the widest tiles when they divide (each tile's fixed costs, its pipeline
    // fill and its epilogue, then cover the most columns), else the least streaming time
    g[0].width = pair || d % 256 == 0 ? 256 : pick_width(kWide, 3, mt, d);
    g[0].n_total = d;
    g[0].num_k_blocks = 2 * F / gemm::BK;
    g[0].out = a.dxbuf;
    g[0].out_ld = d;
    if ((e = gemm::make_map(&ma[0], a.dab, 2ull * F, a_rows, groups, gemm::BM)) != cudaSuccess) return e;
    g[0].b_mn = 1;   // B[n = column of d][k = row of W13] = W13[k][n]: W13 as stored, MN-major
    if ((e = gemm::make_map(&mb[0], a.w_gate_up, d, 2ull * F, E, bwd::kMnBox, bwd::kMnBox)) != cudaSuccess) return e;
    tiles += mt * (d / g[0].width);
    const long long mt_w2 = static_cast<long long>(active) * ((d + gemm::BM - 1) / gemm::BM);
    const long long mt_w13 = static_cast<long long>(active) * ((2 * F + gemm::BM - 1) / gemm::BM);
    g[1].mode = bwd::kWgrad;
    g[1].m_total = d;
    g[1].n_total = F;
    g[1].width = pair || F % 256 == 0 ? 256 : pick_width(kWide, 3, mt_w2, F);
    g[1].out = a.dw_down;
    g[1].overwrite = r == 0;
    g[1].out_group_stride = static_cast<long long>(d) * F;
    g[1].out_ld = F;
    g[1].tma_out = 1;   // dW2 [E][d][F] fp32 through TMA (store in round 0, reduce-add after)
    if ((e = gemm::make_map_f32(&mo[1], a.dw_down, F, d, E, 16, 32)) != cudaSuccess) return e;
    g[1].a_mn = g[1].b_mn = 1;   // A[m = column of d][k = row] = dybuf[k][m], B[n][k] = hg[k][n]
    if ((e = gemm::make_map(&ma[1], a.dybuf, d, a_rows, groups, bwd::kMnBox, bwd::kMnBox)) != cudaSuccess ||
        (e = gemm::make_map(&mb[1], a.hg, F, a_rows, groups, bwd::kMnBox, bwd::kMnBox)) != cudaSuccess)
      return e;
    tiles += mt_w2 * (F / g[1].width);
    g[2].mode = bwd::kWgrad;
    g[2].m_total = 2 * F;
    g[2].n_total = d;
    g[2].width = pair || d % 256 == 0 ? 256 : pick_width(kWide, 3, mt_w13, d);
    g[2].out = a.dw_gate_up;
    g[2].overwrite = r == 0;
    g[2].out_group_stride = 2ll * F * d;
    g[2].out_ld = d;
    g[2].tma_out = 1;   // dW13 [E][2F][d] fp32 through TMA
    if ((e = gemm::make_map_f32(&mo[2], a.dw_gate_up, d, 2ull * F, E, 16, 32)) != cudaSuccess) return e;
    g[2].a_mn = g[2].b_mn = 1;   // A[m = column of 2 d_ff][k = row] = dab[k][m], B[n][k] = xbuf[k][n]
    if ((e = gemm::make_map(&ma[2], a.dab, 2ull * F, a_rows, groups, bwd::kMnBox, bwd::kMnBox)) != cudaSuccess ||
        (e = gemm::make_map(&mb[2], a.xbuf, d, a_rows, groups, bwd::kMnBox, bwd::kMnBox)) != cudaSuccess)
      return e;
    tiles += mt_w13 * (d / g[2].width);
    mo[0] = ma[0];
    if ((e = run_gemm(ma, mb, g, 3, tiles, kKindBackwardDxWgrad, stream, mo, pair)) != cudaSuccess) return e;
  }
  // combine dx and gather dgate; with the next round's gather in the same launch
  {
    // pooled rows: the pair's row is seg_off[r][e] - zeros[r] + slot
    const copy::CombineArgs ca{a.dxbuf, a.dx, a.idx, a.ones, a.round, a.slot, a.T, a.k, C, d,
                               pooled ? a.seg_off : nullptr, pooled ? a.zeros : nullptr, E};
    const bwd::CombineExtra cx{r, a.dgate_part, F / 64, parts, a.dgate};
    const int comb_blocks = grid_for(a.T);
    const int gy = (d + bwd::kGatherCols - 1) / bwd::kGatherCols;   // column blocks of the gather
    const long long next_blocks = a_next && n_next ? gather_blocks(n_next, E) * gy : 0;
    launch_begin(kKindBackwardCopy, stream);
    if (next_blocks > 0)
      e = launch_pdl(bwd::bwd_combine_gather_kernel, dim3(static_cast<unsigned>(comb_blocks + next_blocks)),
                     dim3(32 * bwd::kWarps), 0, stream, ca, cx, gather_args(*a_next, r + 1), comb_blocks,
                     static_cast<int>(next_blocks / gy));
    else
      e = launch_pdl(bwd::bwd_combine_kernel, dim3(comb_blocks), dim3(32 * bwd::kWarps), 0, stream, ca, cx);
    launch_end(kKindBackwardCopy, stream);
  }
  return e;
}

cudaError_t launch_backward_gates(const BackwardArgs& a, cudaStream_t stream) {
  if (a.T <= 0) return cudaSuccess;
  launch_begin(kKindBackwardCopy, stream);
  const cudaError_t e = launch_pdl(bwd::gate_grad_kernel, dim3(grid_for(a.T)), dim3(32 * bwd::kWarps), 0, stream,
                                   a.logits, a.idx, static_cast<const float*>(a.dgate), a.T, a.E, a.k, a.renorm, a.dz);
  launch_end(kKindBackwardCopy, stream);
  return e;
}

}  // namespace moe
