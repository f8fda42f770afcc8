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
// combine:  one warp per token, or, when the round holds fewer rows than there are tokens,
//   one warp per row of the round (the row of a token's first pair in the round does the
//   token's work). It finds the token's pairs that fall in this round (ballot over the k
//   round numbers), starts from zero on the token's first round and from the running y
//   otherwise, and adds gate * out[e][slot] in ascending j. The order of additions is
//   fixed by (round, j), so y is bitwise reproducible; no atomics are used.
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
                    const int32_t* __restrict__ row_dst, int r, int vecs, int32_t* dbg, int T,
                    long long buf_rows) {
  const int begin = row_start[r], end = row_start[r + 1];   // plan data: written before this forward
  const int w = blockIdx.x * kDispatchWarps + (threadIdx.x >> 5), warps = gridDim.x * kDispatchWarps;
  sm100::grid_dependency_wait();                              // buf is still read by the previous round
  sm100::pdl_trigger_early();
  copy::dispatch_rows(x, buf, row_token, row_dst, begin, end, vecs, w, warps, dbg, T, buf_rows);
  sm100::pdl_trigger_late();
}

// by_rows == 0: warp w combines token w. by_rows == 1: warp w stands for row w of the round's
// contiguous row range (fewer warps when the round holds fewer rows than there are tokens).
__global__ void __launch_bounds__(32 * kCombineWarps)
    combine_kernel(const copy::CombineArgs a, int r, int by_rows, const int32_t* __restrict__ row_start,
                   const int32_t* __restrict__ row_token, const int32_t* __restrict__ row_dst) {
  const int w = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  int t = w;
  long long buf_row = -1;
  if (by_rows) {                       // plan data: written before this forward
    const int row = row_start[r] + w;
    t = row < row_start[r + 1] ? row_token[row] : a.T;
    if (row < row_start[r + 1] && a.dbg != nullptr && (t < 0 || t >= a.T)) {
      if ((threadIdx.x & 31) == 0) record_bad(a.dbg, kBadCombineToken, row);
      t = a.T;
    }
    if (t < a.T) buf_row = row_dst[row];
  }
  sm100::grid_dependency_wait();      // buf comes from the round's down GEMM, y from earlier rounds
  sm100::pdl_trigger_early();
  if (t >= 0 && t < a.T) copy::combine_token<16>(a, t, r, buf_row);   // 16 columns per lane: more loads in flight
  sm100::pdl_trigger_late();
}

// Guard words of the workspace (MOE_FLAG_DEBUG_BOUNDS): block b handles guard b. Fill writes
// kGuardWord ^ b into each of its 64 words; check records the first guard found changed.
constexpr uint32_t kGuardWord = 0x5AC3E10Fu;
__global__ void __launch_bounds__(64) guard_kernel(uint8_t* ws, const GuardList g, int check, int32_t* hdr) {
  sm100::grid_dependency_wait();
  sm100::grid_launch_dependents();
  if (static_cast<int>(blockIdx.x) >= g.n) return;
  uint32_t* w = reinterpret_cast<uint32_t*>(ws + g.off[blockIdx.x]) + threadIdx.x;
  if (!check) {
    *w = kGuardWord ^ blockIdx.x;
  } else if (*w != (kGuardWord ^ blockIdx.x)) {
    record_bad(hdr, kBadCanary, static_cast<int>(blockIdx.x));
  }
}

}  // namespace

cudaError_t launch_guards(uint8_t* ws, const GuardList& g, int check, int32_t* hdr, cudaStream_t stream) {
  if (g.n <= 0) return cudaSuccess;
  static_assert(kGuardBytes == 64 * 4, "one thread per guard word");
  launch_begin(kKindPlan, stream);
  const cudaError_t err = launch_pdl(guard_kernel, dim3(g.n), dim3(64), 0, stream, ws, g, check, hdr);
  launch_end(kKindPlan, stream);
  return err;
}

cudaError_t launch_dispatch(const uint16_t* x, uint16_t* buf, const int32_t* row_start,
                            const int32_t* row_token, const int32_t* row_dst, int r, int rows,
                            int d, cudaStream_t stream, int32_t* dbg, int T, long long buf_rows) {
  if (rows <= 0) return cudaSuccess;
  const int vecs = d / 8;
  const int max_blocks = num_sms() * 8;
  int blocks = (rows + kDispatchWarps - 1) / kDispatchWarps;
  if (blocks > max_blocks) blocks = max_blocks;
  launch_begin(kKindDispatch, stream);
  const cudaError_t err = launch_pdl(dispatch_kernel, dim3(blocks), dim3(32 * kDispatchWarps), 0, stream,
                                     reinterpret_cast<const uint4*>(x), reinterpret_cast<uint4*>(buf),
                                     row_start, row_token, row_dst, r, vecs, dbg, T, buf_rows);
  launch_end(kKindDispatch, stream);
  return err;
}

cudaError_t launch_combine(const uint16_t* buf, float* y, const int32_t* idx, const float* gate,
                           const int32_t* round, const int32_t* slot, const int32_t* row_start,
                           const int32_t* row_token, const int32_t* row_dst, int T, int k, int C, int d,
                           int r, int rows, const int32_t* row_off, int E, cudaStream_t stream,
                           int32_t* dbg) {
  if (T <= 0) return cudaSuccess;
  const int by_rows = rows < T ? 1 : 0;
  const int warps = by_rows ? rows : T;
  if (warps <= 0) return cudaSuccess;
  const int blocks = (warps + kCombineWarps - 1) / kCombineWarps;
  launch_begin(kKindCombine, stream);
  const copy::CombineArgs a{buf, y, idx, gate, round, slot, T, k, C, d, row_off, row_off ? row_start : nullptr, E,
                            dbg, static_cast<long long>(E) * C};
  const cudaError_t err = launch_pdl(combine_kernel, dim3(blocks), dim3(32 * kCombineWarps), 0, stream, a, r,
                                     by_rows, row_start, row_token, row_dst);
  launch_end(kKindCombine, stream);
  return err;
}

}  // namespace moe
