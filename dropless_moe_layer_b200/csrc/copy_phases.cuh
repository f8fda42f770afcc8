// copy_phases.cuh - device side of the round's copy steps (dispatch and combine).
//
// "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, multi-round dropless
// MoE item [section "Scaling MoE", Fig. 6]: every round is dispatch -> compute -> collect
// with a fixed per-expert capacity, so the round's token buffer has a fixed size. With all
// experts on one GPU, dispatch is a gather of token rows into the fixed [E, C, d] buffer and
// collect is a gate-weighted gather back into the fp32 output.
//
// dispatch: one warp per row of the round's contiguous range of the round-major row list
//   (built by the planner, so no empty expert is ever visited); 16-byte vector loads and
//   stores, up to eight in flight per lane.
// combine: one warp per token. A ballot over the token's k round numbers finds its pairs in
//   this round; the token's first round starts from zero instead of reading y; the pairs'
//   gate * out[e][slot] are added in ascending j with fp32 FMAs. The order of additions is
//   fixed by (round, j), so y is bitwise reproducible; no atomics are used.
#pragma once

#include <climits>
#include <cstdint>

#include "kernels.h"

namespace moe {
namespace copy {

// Streaming accesses for copies that run beside a GEMM (the copy warps of a GEMM launch): an L2
// evict-first policy, so that the copy's bytes, each touched once, do not push the GEMM's weight
// and activation tiles out of the L2. kStream = false: plain accesses.
__device__ __forceinline__ uint64_t stream_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
template <bool kStream>
__device__ __forceinline__ uint4 ld_u4(const uint4* p, uint64_t pol) {
  if constexpr (!kStream) return __ldg(p);
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p), "l"(pol));
  return v;
}
template <bool kStream>
__device__ __forceinline__ void st_u4(uint4* p, const uint4& v, uint64_t pol) {
  if constexpr (!kStream) {
    *p = v;
  } else {
    asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w), "l"(pol)
                 : "memory");
  }
}
template <bool kStream>
__device__ __forceinline__ float4 ld_f4(const float* p, uint64_t pol) {
  if constexpr (!kStream) return *reinterpret_cast<const float4*>(p);
  float4 v;
  asm volatile("ld.global.L1::no_allocate.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p), "l"(pol));
  return v;
}
template <bool kStream>
__device__ __forceinline__ void st_f4(float* p, const float4& v, uint64_t pol) {
  if constexpr (!kStream) {
    *reinterpret_cast<float4*>(p) = v;
  } else {
    asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
  }
}

template <bool kStream = false>
__device__ __forceinline__ void dispatch_row(const uint4* __restrict__ x, uint4* __restrict__ buf, int t,
                                             int dst, int vecs, int lane) {
  const uint4* src = x + static_cast<size_t>(t) * vecs;
  uint4* out = buf + static_cast<size_t>(dst) * vecs;
  const uint64_t pol = kStream ? stream_policy() : 0;
  for (int v0 = 0; v0 < vecs; v0 += 8 * 32) {
    uint4 tmp[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vecs) tmp[u] = ld_u4<kStream>(src + v, pol);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vecs) st_u4<kStream>(out + v, tmp[u], pol);
    }
  }
}

// Rows [begin, end) of the round-major row list, spread over `warps` warps (this one is `w`).
// With dbg (debug bounds checks) a row whose token is not below T or whose destination is not
// below buf_rows is recorded and skipped.
template <bool kStream = false>
__device__ __forceinline__ void dispatch_rows(const uint4* __restrict__ x, uint4* __restrict__ buf,
                                              const int32_t* __restrict__ row_token,
                                              const int32_t* __restrict__ row_dst, int begin, int end,
                                              int vecs, int w, int warps, int32_t* dbg = nullptr, int T = 0,
                                              long long buf_rows = 0) {
  const int lane = threadIdx.x & 31;
  for (int row = begin + w; row < end; row += warps) {
    const int t = row_token[row], dst = row_dst[row];
    if (dbg != nullptr && (t < 0 || t >= T || dst < 0 || dst >= buf_rows)) {
      if (lane == 0) record_bad(dbg, kBadDispatchRow, row);
      continue;
    }
    dispatch_row<kStream>(x, buf, t, dst, vecs, lane);
  }
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& q, float (&f)[8]) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

struct CombineArgs {
  const uint16_t* buf;
  float* y;
  const int32_t* idx;
  const float* gate;
  const int32_t* round;
  const int32_t* slot;
  int T, k, C, d;
  // Pooled round rows (capacity borrowing): the pair (e, slot) of round r is row
  // row_off[r][e] - row_start[r] + slot of buf. Null: row e * C + slot.
  const int32_t* row_off;
  const int32_t* row_start;
  int E;
  // Debug bounds checks (MOE_FLAG_DEBUG_BOUNDS): the workspace header, else null; a pair whose
  // expert is not below E, whose slot is not below C (per-expert rows) or whose buffer row is not
  // below rows_cap makes the token skipped.
  int32_t* dbg;
  long long rows_cap;
};

// One token's pairs in one round, spread over the warp (every lane holds the same scalars;
// lane p < npairs holds pair p's source row and gate, pairs in ascending j).
struct TokenPairs {
  int npairs;                     // pairs of the token in round r (0: nothing to do)
  bool fresh;                     // r is the token's first round: y starts from zero
  int prev_round;                 // the token's latest round before r, or -1
  unsigned long long first_row;   // buffer row of the token's first pair in round r
  int e, s;                       // this lane's pair (expert, slot), lane < npairs
  unsigned long long prow;        // its buffer row: e * C + s, or the pooled row
  float pgate;                    // its gate (0 for lanes >= npairs)
};

// A token's plan entries as loaded: lane j < k holds pair j's round, expert, slot and gate.
struct PairLoads {
  int round, idx, slot;
  float gate;
};

// Issues the four independent loads; nothing waits for them until token_pairs() uses them, so
// a warp can fetch the next token's entries while it combines the current one.
__device__ __forceinline__ PairLoads load_pairs(const CombineArgs& a, int t) {
  const int lane = threadIdx.x & 31;
  PairLoads l{INT_MAX, 0, 0, 0.f};
  if (lane < a.k) {
    const size_t i = static_cast<size_t>(t) * a.k + lane;
    l.round = a.round[i];
    l.idx = a.idx[i];
    l.slot = a.slot[i];
    l.gate = a.gate[i];
  }
  return l;
}

__device__ __forceinline__ TokenPairs token_pairs(const CombineArgs& a, const PairLoads& l, int r) {
  const int lane = threadIdx.x & 31;
  const int my_round = l.round, my_idx = l.idx, my_slot = l.slot;
  const float my_gate = l.gate;
  TokenPairs tp;
  const uint32_t here = __ballot_sync(0xffffffffu, my_round == r);
  tp.npairs = __popc(here);
  tp.fresh = __reduce_min_sync(0xffffffffu, my_round) == r;
  tp.prev_round = __reduce_max_sync(0xffffffffu, my_round < r ? my_round : -1);
  const int jp = lane < tp.npairs ? static_cast<int>(__fns(here, 0, lane + 1)) : 0;
  tp.e = __shfl_sync(0xffffffffu, my_idx, jp);
  tp.s = __shfl_sync(0xffffffffu, my_slot, jp);
  const float g = __shfl_sync(0xffffffffu, my_gate, jp);
  unsigned long long row = 0ull;
  const bool e_ok = a.dbg == nullptr || (tp.e >= 0 && tp.e < a.E);   // checked before it indexes row_off
  if (lane < tp.npairs && e_ok)
    row = a.row_off ? static_cast<unsigned long long>(a.row_off[static_cast<size_t>(r) * a.E + tp.e] - a.row_start[r] + tp.s)
                    : static_cast<unsigned long long>(tp.e) * a.C + tp.s;
  tp.prow = row;
  tp.first_row = __shfl_sync(0xffffffffu, row, 0);
  tp.pgate = lane < tp.npairs ? g : 0.f;
  if (a.dbg != nullptr) {
    // a slot past C lands in the next expert's rows of the [E, C, d] buffer: checked on its own
    const bool bad = lane < tp.npairs && (!e_ok || tp.s < 0 || (a.row_off == nullptr && tp.s >= a.C) ||
                                          row >= static_cast<unsigned long long>(a.rows_cap));
    const uint32_t any = __ballot_sync(0xffffffffu, bad);
    if (any) {
      if (lane == __ffs(any) - 1) record_bad(a.dbg, kBadCombinePair, static_cast<int>(row));
      tp.npairs = 0;
    }
  }
  return tp;
}

// y[t] = (fresh ? 0 : y[t]) + sum over the round's pairs (ascending j) of gate * out row, fp32
// FMAs. kLaneCols columns per lane per pass (8, 16 or 32): wider passes mean fewer dependent
// passes over a row and more loads in flight, which matters when few warps do the work (the
// copy warps of a GEMM launch). The whole warp runs it.
template <int kLaneCols = 8, bool kStream = false>
__device__ __forceinline__ void accumulate_token(const CombineArgs& a, int t, const TokenPairs& tp) {
  static_assert(kLaneCols == 8 || kLaneCols == 16 || kLaneCols == 32, "lane width");
  constexpr int kVecs = kLaneCols / 8;   // bf16 x 8 per 16-byte load
  const int lane = threadIdx.x & 31;
  const uint64_t pol = kStream ? stream_policy() : 0;
  const int npairs = tp.npairs;
  float* yrow = a.y + static_cast<size_t>(t) * a.d;
  // Every lane runs the same iterations (the shuffles below need the whole warp); lanes past
  // the end of the row only skip the loads and stores.
  for (int c0 = 0; c0 < a.d; c0 += 32 * kLaneCols) {
    const int c = c0 + lane * kLaneCols;
    const bool col = c < a.d;
    float acc[kLaneCols];
    if (tp.fresh || !col) {
#pragma unroll
      for (int i = 0; i < kLaneCols; ++i) acc[i] = 0.f;
    } else {
#pragma unroll
      for (int i = 0; i < kLaneCols; i += 4) {
        const float4 u = ld_f4<kStream>(yrow + c + i, pol);
        acc[i] = u.x; acc[i + 1] = u.y; acc[i + 2] = u.z; acc[i + 3] = u.w;
      }
    }
    for (int p0 = 0; p0 < npairs; p0 += 4) {
      uint4 q[4][kVecs];
      float g[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {               // up to four rows in flight per lane
        const int p = p0 + u;
        const unsigned long long row = __shfl_sync(0xffffffffu, tp.prow, p & 31);
        g[u] = __shfl_sync(0xffffffffu, tp.pgate, p & 31);
#pragma unroll
        for (int v = 0; v < kVecs; ++v)
          q[u][v] = (p < npairs && col) ? ld_u4<kStream>(reinterpret_cast<const uint4*>(a.buf + row * a.d + c + 8 * v), pol)
                                        : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (p0 + u < npairs) {
#pragma unroll
          for (int v = 0; v < kVecs; ++v) {
            float f[8];
            bf16x8_to_f32(q[u][v], f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[8 * v + i] = __fmaf_rn(g[u], f[i], acc[8 * v + i]);
          }
        }
      }
    }
    if (col) {
#pragma unroll
      for (int i = 0; i < kLaneCols; i += 4)
        st_f4<kStream>(yrow + c + i, make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]), pol);
    }
  }
}

// The whole warp combines token t for round r (no-op if t has no pair in round r).
// With `only_row` >= 0 the warp stands for one buffer row of the round (one of token t's pairs)
// and does the work only if that row is t's first pair in the round, so that every active
// token is combined exactly once when the round is walked row by row.
template <int kLaneCols = 8, bool kStream = false>
__device__ __forceinline__ void combine_token(const CombineArgs& a, int t, int r, long long only_row = -1) {
  const TokenPairs tp = token_pairs(a, load_pairs(a, t), r);
  if (tp.npairs == 0) return;
  if (only_row >= 0 && tp.first_row != static_cast<unsigned long long>(only_row)) return;
  accumulate_token<kLaneCols, kStream>(a, t, tp);
}

// One warp copies rows [0, nr) (nr <= 32) of a slice of the round-major row list: row i goes
// from x[tok[i]] to buf[dst[i]]. The row list entries are read once (lane i holds row i) and the
// copy is flattened over (row, 16-byte vector) so that 16 loads per lane are in flight, whatever
// the row length. Every shuffle runs on all 32 lanes.
__device__ __forceinline__ void copy_rows_flat(const uint4* __restrict__ x, uint4* __restrict__ buf,
                                               int tok_lane, int dst_lane, int nr, int vecs) {
  const int lane = threadIdx.x & 31;
  const int units = nr * vecs;
  constexpr int kInFlight = 16;
  for (int u0 = 0; u0 < units; u0 += 32 * kInFlight) {
    uint4 v[kInFlight];
#pragma unroll
    for (int i = 0; i < kInFlight; ++i) {
      const int u = u0 + i * 32 + lane;
      const int uc = u < units ? u : units - 1;
      const int row = uc / vecs;
      const int t = __shfl_sync(0xffffffffu, tok_lane, row);
      if (u < units) v[i] = __ldg(x + static_cast<size_t>(t) * vecs + (uc - row * vecs));
    }
#pragma unroll
    for (int i = 0; i < kInFlight; ++i) {
      const int u = u0 + i * 32 + lane;
      const int uc = u < units ? u : units - 1;
      const int row = uc / vecs;
      const int dst = __shfl_sync(0xffffffffu, dst_lane, row);
      if (u < units) buf[static_cast<size_t>(dst) * vecs + (uc - row * vecs)] = v[i];
    }
  }
}

}  // namespace copy
}  // namespace moe
