// dispatch_combine.cu - the copy steps around the expert GEMMs of one round.
//
// "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, multi-round dropless
// MoE item [section "Scaling MoE", Fig. 6]: every round is dispatch -> compute -> collect,
// with a fixed per-expert capacity, so the round's token buffer has a fixed size. Here all
// experts live on one GPU, so dispatch is a gather of token rows into the fixed
// [E, C, d] buffer and collect is a gate-weighted gather back into the fp32 output.
//
// dispatch: one warp per row of the round-major row list (built by the planner, so
//   the round's rows are one contiguous range with no empty experts to skip); 16-byte
//   vector loads and stores, four in flight per lane.
// combine:  one warp per token. It finds the token's pairs that fall in this round
//   (ballot over the k round numbers), starts from zero on the token's first round
//   and from the running y otherwise, and adds gate * out[e][slot] in ascending j.
//   The order of additions is fixed by (round, j), so y is bitwise reproducible; no
//   atomics are used.
#include <climits>

#include <cuda_bf16.h>

#include "kernels.h"

namespace moe {

namespace {

constexpr int kDispatchWarps = 8;
constexpr int kCombineWarps = 8;

__global__ void __launch_bounds__(32 * kDispatchWarps)
    dispatch_kernel(const uint4* __restrict__ x, uint4* __restrict__ buf,
                    const int32_t* __restrict__ row_start, const int32_t* __restrict__ row_token,
                    const int32_t* __restrict__ row_dst, int r, int vecs) {
  const int lane = threadIdx.x & 31;
  const int begin = row_start[r], end = row_start[r + 1];
  const int stride = gridDim.x * kDispatchWarps;
  for (int row = begin + blockIdx.x * kDispatchWarps + (threadIdx.x >> 5); row < end; row += stride) {
    const int t = row_token[row];
    const int dst = row_dst[row];
    const uint4* src = x + static_cast<size_t>(t) * vecs;
    uint4* out = buf + static_cast<size_t>(dst) * vecs;
    for (int v0 = 0; v0 < vecs; v0 += 4 * 32) {
      uint4 tmp[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < vecs) tmp[u] = __ldg(src + v);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * 32 + lane;
        if (v < vecs) out[v] = tmp[u];
      }
    }
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

__global__ void __launch_bounds__(32 * kCombineWarps)
    combine_kernel(const uint16_t* __restrict__ buf, float* __restrict__ y,
                   const int32_t* __restrict__ idx, const float* __restrict__ gate,
                   const int32_t* __restrict__ round, const int32_t* __restrict__ slot, int T, int k,
                   int C, int d, int r) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const size_t pbase = static_cast<size_t>(t) * k;
  const int my_round = lane < k ? round[pbase + lane] : INT_MAX;
  const uint32_t here = __ballot_sync(0xffffffffu, my_round == r);
  if (here == 0u) return;
  const int first_round = __reduce_min_sync(0xffffffffu, my_round);
  const bool fresh = first_round == r;
  // Per-pair source row and gate, held by lane j.
  size_t my_row = 0;
  float my_gate = 0.f;
  if (lane < k && my_round == r) {
    my_row = static_cast<size_t>(idx[pbase + lane]) * C + slot[pbase + lane];
    my_gate = gate[pbase + lane];
  }
  float* yrow = y + static_cast<size_t>(t) * d;
  for (int c = lane * 8; c < d; c += 32 * 8) {
    float acc[8];
    if (fresh) {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    } else {
      const float4 a = *reinterpret_cast<const float4*>(yrow + c);
      const float4 b = *reinterpret_cast<const float4*>(yrow + c + 4);
      acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
      acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
    }
    uint32_t rest = here;
    while (rest) {
      const int j = __ffs(rest) - 1;
      rest &= rest - 1;
      const size_t row = __shfl_sync(0xffffffffu, my_row, j);
      const float g = __shfl_sync(0xffffffffu, my_gate, j);
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(buf + row * d + c));
      float f[8];
      bf16x8_to_f32(q, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(g, f[i], acc[i]);
    }
    *reinterpret_cast<float4*>(yrow + c) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *reinterpret_cast<float4*>(yrow + c + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

}  // namespace

cudaError_t launch_dispatch(const uint16_t* x, uint16_t* buf, const int32_t* row_start,
                            const int32_t* row_token, const int32_t* row_dst, int r, int rows,
                            int d, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int vecs = d / 8;
  const int max_blocks = num_sms() * 8;
  int blocks = (rows + kDispatchWarps - 1) / kDispatchWarps;
  if (blocks > max_blocks) blocks = max_blocks;
  launch_begin(kKindDispatch, stream);
  dispatch_kernel<<<blocks, 32 * kDispatchWarps, 0, stream>>>(
      reinterpret_cast<const uint4*>(x), reinterpret_cast<uint4*>(buf), row_start, row_token,
      row_dst, r, vecs);
  launch_end(kKindDispatch, stream);
  return cudaGetLastError();
}

cudaError_t launch_combine(const uint16_t* buf, float* y, const int32_t* idx, const float* gate,
                           const int32_t* round, const int32_t* slot, int T, int k, int C, int d,
                           int r, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int blocks = (T + kCombineWarps - 1) / kCombineWarps;
  launch_begin(kKindCombine, stream);
  combine_kernel<<<blocks, 32 * kCombineWarps, 0, stream>>>(buf, y, idx, gate, round, slot, T, k, C,
                                                            d, r);
  launch_end(kKindCombine, stream);
  return cudaGetLastError();
}

}  // namespace moe
