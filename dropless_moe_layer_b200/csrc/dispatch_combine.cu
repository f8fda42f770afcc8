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
//   vector loads and stores, eight in flight per lane.
// combine:  one warp per token. It finds the token's pairs that fall in this round
//   (ballot over the k round numbers), starts from zero on the token's first round
//   and from the running y otherwise, and adds gate * out[e][slot] in ascending j.
//   The order of additions is fixed by (round, j), so y is bitwise reproducible; no
//   atomics are used.
#include "copy_phases.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int kDispatchWarps = 8;
constexpr int kCombineWarps = 8;

__global__ void __launch_bounds__(32 * kDispatchWarps)
    dispatch_kernel(const uint4* __restrict__ x, uint4* __restrict__ buf,
                    const int32_t* __restrict__ row_start, const int32_t* __restrict__ row_token,
                    const int32_t* __restrict__ row_dst, int r, int vecs) {
  const int begin = row_start[r], end = row_start[r + 1];   // plan data: written before this forward
  const int w = blockIdx.x * kDispatchWarps + (threadIdx.x >> 5), warps = gridDim.x * kDispatchWarps;
  sm100::grid_dependency_wait();                              // buf is still read by the previous round
  sm100::pdl_trigger_early();
  copy::dispatch_rows(x, buf, row_token, row_dst, begin, end, vecs, w, warps);
  sm100::pdl_trigger_late();
}

__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(const copy::CombineArgs a, int r) {
  const int t = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  sm100::grid_dependency_wait();      // buf comes from the round's down GEMM, y from earlier rounds
  sm100::pdl_trigger_early();
  if (t < a.T) copy::combine_token(a, t, r);
  sm100::pdl_trigger_late();
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
  const cudaError_t err = launch_pdl(dispatch_kernel, dim3(blocks), dim3(32 * kDispatchWarps), 0, stream,
                                     reinterpret_cast<const uint4*>(x), reinterpret_cast<uint4*>(buf),
                                     row_start, row_token, row_dst, r, vecs);
  launch_end(kKindDispatch, stream);
  return err;
}

cudaError_t launch_combine(const uint16_t* buf, float* y, const int32_t* idx, const float* gate,
                           const int32_t* round, const int32_t* slot, int T, int k, int C, int d,
                           int r, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int blocks = (T + kCombineWarps - 1) / kCombineWarps;
  launch_begin(kKindCombine, stream);
  const copy::CombineArgs a{buf, y, idx, gate, round, slot, T, k, C, d};
  const cudaError_t err = launch_pdl(combine_kernel, dim3(blocks), dim3(32 * kCombineWarps), 0, stream, a, r);
  launch_end(kKindCombine, stream);
  return err;
}

}  // namespace moe
