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

__device__ __forceinline__ void dispatch_row(const uint4* __restrict__ x, uint4* __restrict__ buf, int t,
                                             int dst, int vecs, int lane) {
  const uint4* src = x + static_cast<size_t>(t) * vecs;
  uint4* out = buf + static_cast<size_t>(dst) * vecs;
  for (int v0 = 0; v0 < vecs; v0 += 8 * 32) {
    uint4 tmp[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vecs) tmp[u] = __ldg(src + v);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int v = v0 + u * 32 + lane;
      if (v < vecs) out[v] = tmp[u];
    }
  }
}

// Rows [begin, end) of the round-major row list, spread over `warps` warps (this one is `w`).
__device__ __forceinline__ void dispatch_rows(const uint4* __restrict__ x, uint4* __restrict__ buf,
                                              const int32_t* __restrict__ row_token,
                                              const int32_t* __restrict__ row_dst, int begin, int end,
                                              int vecs, int w, int warps) {
  const int lane = threadIdx.x & 31;
  for (int row = begin + w; row < end; row += warps)
    dispatch_row(x, buf, row_token[row], row_dst[row], vecs, lane);
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
};

// The whole warp combines token t for round r (no-op if t has no pair in round r).
// With `only_expert` >= 0 the warp stands for one row of the round (token t's pair with that
// expert) and does the work only if that pair is t's first pair in the round, so that every
// active token is combined exactly once when the round is walked row by row.
__device__ __forceinline__ void combine_token(const CombineArgs& a, int t, int r, int only_expert = -1) {
  const int lane = threadIdx.x & 31;
  const size_t pbase = static_cast<size_t>(t) * a.k;
  // lane j < k holds pair j's round, expert, slot and gate (four independent loads)
  int my_round = INT_MAX, my_idx = 0, my_slot = 0;
  float my_gate = 0.f;
  if (lane < a.k) {
    my_round = a.round[pbase + lane];
    my_idx = a.idx[pbase + lane];
    my_slot = a.slot[pbase + lane];
    my_gate = a.gate[pbase + lane];
  }
  const uint32_t here = __ballot_sync(0xffffffffu, my_round == r);
  if (here == 0u) return;
  if (only_expert >= 0 && __shfl_sync(0xffffffffu, my_idx, __ffs(here) - 1) != only_expert) return;
  const int first_round = __reduce_min_sync(0xffffffffu, my_round);
  const bool fresh = first_round == r;
  const int npairs = __popc(here);
  // Lane p holds the source row and gate of the p-th pair of this round (ascending j).
  const int jp = lane < npairs ? static_cast<int>(__fns(here, 0, lane + 1)) : 0;
  const int e_p = __shfl_sync(0xffffffffu, my_idx, jp);
  const int s_p = __shfl_sync(0xffffffffu, my_slot, jp);
  const float g_p = __shfl_sync(0xffffffffu, my_gate, jp);
  const unsigned long long prow = lane < npairs ? static_cast<unsigned long long>(e_p) * a.C + s_p : 0ull;
  const float pgate = lane < npairs ? g_p : 0.f;
  float* yrow = a.y + static_cast<size_t>(t) * a.d;
  // Every lane runs the same iterations (the shuffles below need the whole warp); lanes past
  // the end of the row (d < 256) only skip the loads and stores.
  for (int c0 = 0; c0 < a.d; c0 += 32 * 8) {
    const int c = c0 + lane * 8;
    const bool col = c < a.d;
    float acc[8];
    if (fresh || !col) {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    } else {
      const float4 u = *reinterpret_cast<const float4*>(yrow + c);
      const float4 v = *reinterpret_cast<const float4*>(yrow + c + 4);
      acc[0] = u.x; acc[1] = u.y; acc[2] = u.z; acc[3] = u.w;
      acc[4] = v.x; acc[5] = v.y; acc[6] = v.z; acc[7] = v.w;
    }
    for (int p0 = 0; p0 < npairs; p0 += 4) {
      uint4 q[4];
      float g[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {               // up to four rows in flight per lane
        const int p = p0 + u;
        const unsigned long long row = __shfl_sync(0xffffffffu, prow, p & 31);
        g[u] = __shfl_sync(0xffffffffu, pgate, p & 31);
        q[u] = (p < npairs && col) ? *reinterpret_cast<const uint4*>(a.buf + row * a.d + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (p0 + u < npairs) {
          float f[8];
          bf16x8_to_f32(q[u], f);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(g[u], f[i], acc[i]);
        }
      }
    }
    if (col) {
      *reinterpret_cast<float4*>(yrow + c) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      *reinterpret_cast<float4*>(yrow + c + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

}  // namespace copy
}  // namespace moe
