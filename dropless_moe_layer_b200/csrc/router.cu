// router.cu - softmax + top-k selection, one warp per token.
//
// "Microsoft AI's MAI-Base-2 trained on 16K GPUs with Muon", section "Expert groups
// keep memory fixed when tokens pile up": a router sends each token to a few experts.
// The pages do not name the gate function; this library takes the softmax over all E
// logits and keeps the k largest, best first, equal logits going to the lower expert
// index (+0 and -0 compare equal). Selection compares the fp32 logits themselves, so
// the chosen experts are exact; gates are fp32 softmax probabilities.
//
// Each lane holds up to 8 logits (E <= 256) in registers. The softmax max and sum are
// warp butterfly reductions (fixed order, so deterministic). Top-k is k rounds of a
// warp arg-max under the total order (logit desc, index asc); the winner is marked
// taken in its owner lane. The kernel also counts, for the planner, the pairs of every block
// of 256 tokens per expert.
#include <cfloat>
#include <climits>

#include "kernels.h"
#include "sm100.cuh"

namespace moe {

template <int VPL>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ logits, int T,
                                                          int E, int k, int renorm,
                                                          int32_t* __restrict__ idx_out,
                                                          float* __restrict__ gate_out,
                                                          int32_t* __restrict__ block_counts) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  sm100::grid_dependency_wait();
  sm100::grid_launch_dependents();
  if (t >= T) return;
  const float* row = logits + static_cast<size_t>(t) * E;

  float v[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldg(row + e) : -FLT_MAX;
  }
  float m = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < VPL; ++i) m = fmaxf(m, v[i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) s += expf(v[i] - m);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);

  uint32_t taken = 0;      // bit i: v[i] already selected
  int my_idx = 0;          // lane j keeps the j-th selection
  float my_gate = 0.f;
  float gsum = 0.f;
  for (int j = 0; j < k; ++j) {
    float bv = -FLT_MAX;
    int be = INT_MAX;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !(taken & (1u << i)) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    const float g = expf(bv - m) / s;
    gsum += g;
    if (lane == j) {
      my_idx = be;
      my_gate = g;
    }
  }
  if (lane < k) {
    if (renorm) my_gate = my_gate / gsum;
    idx_out[static_cast<size_t>(t) * k + lane] = my_idx;
    gate_out[static_cast<size_t>(t) * k + lane] = my_gate;
    // the planner's per-block counts (integer adds: the order does not matter)
    atomicAdd(block_counts + static_cast<size_t>(t / kPlanTokensPerBlock) * E + my_idx, 1);
  }
}

cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int renorm, int32_t* idx,
                               float* gate, int32_t* block_counts, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int warps_per_block = 8;
  const dim3 grid((T + warps_per_block - 1) / warps_per_block), block(32 * warps_per_block);
  launch_begin(kKindTopk, stream);
  const int vpl = (E + 31) / 32;
  auto kern = vpl <= 1 ? router_topk_kernel<1> : vpl <= 2 ? router_topk_kernel<2>
            : vpl <= 4 ? router_topk_kernel<4> : router_topk_kernel<8>;
  const cudaError_t err = launch_pdl(kern, grid, block, 0, stream, logits, T, E, k, renorm, idx, gate,
                                     block_counts);
  launch_end(kKindTopk, stream);
  return err;
}

}  // namespace moe
