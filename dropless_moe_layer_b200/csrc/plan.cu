// plan.cu - the round planner: every (token, expert) pair gets a round and a slot.
//
// "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, multi-round
// dropless MoE item [section "Scaling MoE"]: each expert processes at most a fixed
// number C of tokens per round and the rest waits for further rounds, so memory is
// fixed; its summary of the per-expert overhead cuts keeps the token metadata on the
// device. The pages do not say which tokens go first; this planner takes them in
// ascending token order within each expert (a stable order), with no capacity
// borrowing between experts:
//   rank(t, j) = #{t' < t : expert idx[t, j] is among t's choices}
//   round = rank / C, slot = rank % C, R = ceil(max_e load_e / C)
//
// Integer work only (bit-exact, deterministic), after the top-k kernel has counted the pairs
// of every block of 256 tokens per expert (router.cu):
//   1. plan_scan:     one CTA per expert: exclusive scan of the block counts over
//                     blocks (the block's base rank) and the expert's load; the last CTA
//                     to finish then computes the expert offsets, max load, R, n[r][e],
//                     the round-major row positions row_off[r][e] and row_start[r].
//   2. plan_rank:     per block of 256 tokens: the stable rank of each pair inside its
//                     block from per-warp lane bitmasks (popcount of lower lanes and
//                     lower warps), plus the block base; writes round, slot and the
//                     pair's row in the round-major list (source token, destination
//                     e * C + slot) that dispatch copies from.
#include "kernels.h"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int kTPB = kPlanTokensPerBlock;   // tokens per block = threads per block
constexpr int kWarps = kTPB / 32;

// Block-wide inclusive scan of one int per thread (blockDim.x == 256).
__device__ int block_inclusive_scan(int v, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += o;
    }
    if (lane < (blockDim.x >> 5)) warp_sums[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v += warp_sums[warp - 1];
  __syncthreads();
  return v;
}

__device__ void finalize_plan(const int32_t* __restrict__ load, int E, int C, int max_rounds,
                              int32_t* __restrict__ offsets, int32_t* __restrict__ header,
                              int32_t* __restrict__ n, int32_t* __restrict__ row_off,
                              int32_t* __restrict__ row_start, int32_t* __restrict__ mb_prefix,
                              int* warp_sums, int borrow);

// Block-wide sum of one int per thread (blockDim.x == 256); every thread gets the total.
__device__ int block_sum(int v, int* warp_sums) {
  const int incl = block_inclusive_scan(v, warp_sums);
  __shared__ int total;
  if (threadIdx.x == blockDim.x - 1) total = incl;
  __syncthreads();
  const int t = total;
  __syncthreads();
  return t;
}

// Rounds with capacity borrowing ("Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key
// claims, multi-round dropless MoE item: overflow uses unused capacity of other experts of the
// group, otherwise an extra round). One CTA, thread e = expert e, round after round: every
// expert first takes up to C of its pending pairs; the rows of the E*C pool left unused by that
// go to experts with pairs still pending, in ascending expert index. Writes n[r][e],
// row_off[r][e], row_start[r], the block prefix and R. Never more rounds than without
// borrowing, so r < max_rounds throughout.
__device__ void finalize_borrow(int load_e, int E, int C, int max_rounds, int max_load,
                                int32_t* __restrict__ header, int32_t* __restrict__ n,
                                int32_t* __restrict__ row_off, int32_t* __restrict__ row_start,
                                int32_t* __restrict__ mb_prefix, int* warp_sums) {
  const int e = threadIdx.x;
  int pending = e < E ? load_e : 0;
  int r = 0, rows_before = 0;
  const long long pool = static_cast<long long>(E) * C;
  while (r < max_rounds && block_sum(pending > 0 ? 1 : 0, warp_sums) > 0) {
    const int own = pending < C ? pending : C;
    const long long spare = pool - block_sum(own, warp_sums);
    const int want = pending - own;
    const int want_before = block_inclusive_scan(want, warp_sums) - want;   // lower experts first
    long long extra = spare - want_before;
    extra = extra < 0 ? 0 : (extra > want ? want : extra);
    const int nv = own + static_cast<int>(extra);
    const int incl = block_inclusive_scan(nv, warp_sums);
    const int mb = (nv + kPipeRowBlock - 1) / kPipeRowBlock;
    const int incl_mb = block_inclusive_scan(mb, warp_sums);
    if (e < E) {
      n[static_cast<size_t>(r) * E + e] = nv;
      row_off[static_cast<size_t>(r) * E + e] = rows_before + incl - nv;
      if (mb_prefix) mb_prefix[static_cast<size_t>(r) * (E + 1) + e] = incl_mb - mb;
    }
    if (e == E - 1 && mb_prefix) mb_prefix[static_cast<size_t>(r) * (E + 1) + E] = incl_mb;
    if (e == 0) row_start[r] = rows_before;
    rows_before += block_sum(nv, warp_sums);
    pending -= nv;
    ++r;
  }
  if (e == 0) {
    row_start[r] = rows_before;
    header[kHdrR] = r;
    header[kHdrMaxLoad] = max_load;
  }
}

// One CTA per expert e: block_base[b][e] <- sum_{b' < b} count[b'][e]; load[e] <- total. The
// last CTA to finish (a counter in the header) then finalizes the plan.
__global__ void __launch_bounds__(kTPB) plan_scan_kernel(int32_t* __restrict__ block_base,
                                                         int blocks, int E, int C, int max_rounds,
                                                         int32_t* __restrict__ load,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ header,
                                                         int32_t* __restrict__ n,
                                                         int32_t* __restrict__ row_off,
                                                         int32_t* __restrict__ row_start,
                                                         int32_t* __restrict__ mb_prefix,
                                                         int borrow) {
  __shared__ int warp_sums[kWarps];
  __shared__ int chunk_total;
  __shared__ int is_last;
  const int e = blockIdx.x;
  int carry = 0;
  sm100::grid_dependency_wait();
  sm100::grid_launch_dependents();
  for (int b0 = 0; b0 < blocks; b0 += kTPB) {
    const int b = b0 + threadIdx.x;
    const int c = b < blocks ? block_base[static_cast<size_t>(b) * E + e] : 0;
    const int inc = block_inclusive_scan(c, warp_sums);
    if (b < blocks) block_base[static_cast<size_t>(b) * E + e] = carry + inc - c;
    if (threadIdx.x == kTPB - 1) chunk_total = inc;   // the chunk's total
    __syncthreads();
    carry += chunk_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    load[e] = carry;
    __threadfence();   // load[e] is visible before this CTA counts itself done
    is_last = atomicAdd(header + kHdrScanDone, 1) == E - 1;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  finalize_plan(load, E, C, max_rounds, offsets, header, n, row_off, row_start, mb_prefix, warp_sums, borrow);
}

// One CTA (the last expert scan to finish): offsets, max load, R, n[r][e], row_off[r][e],
// row_start[r], and the per-round 128-row block prefix.
__device__ void finalize_plan(const int32_t* __restrict__ load, int E, int C, int max_rounds,
                              int32_t* __restrict__ offsets, int32_t* __restrict__ header,
                              int32_t* __restrict__ n, int32_t* __restrict__ row_off,
                              int32_t* __restrict__ row_start, int32_t* __restrict__ mb_prefix,
                              int* warp_sums, int borrow) {
  __shared__ int s_load[MOE_MAX_E_PLAN];
  __shared__ int s_max;
  const int e = threadIdx.x;
  const int le = e < E ? __ldcg(load + e) : 0;   // written by the other CTAs of this grid
  if (e < MOE_MAX_E_PLAN) s_load[e] = le;
  if (threadIdx.x == 0) s_max = 0;
  const int inc = block_inclusive_scan(le, warp_sums);
  if (e < E) {
    offsets[e] = inc - le;
    header[kHdrLoad + e] = le;
    atomicMax(&s_max, le);
  }
  if (e == E - 1) offsets[E] = inc;
  __syncthreads();
  const int max_load = s_max;
  if (borrow) {
    finalize_borrow(le, E, C, max_rounds, max_load, header, n, row_off, row_start, mb_prefix, warp_sums);
    return;
  }
  const int R = (max_load + C - 1) / C;
  if (threadIdx.x == 0) {
    header[kHdrR] = R;
    header[kHdrMaxLoad] = max_load;
  }
  // row_start[r] = sum_e min(load_e, r*C): rows of all rounds before r.
  for (int r = threadIdx.x; r <= R && r <= max_rounds; r += blockDim.x) {
    const long long cap = static_cast<long long>(r) * C;
    long long s = 0;
    for (int x = 0; x < E; ++x) s += s_load[x] < cap ? s_load[x] : cap;
    row_start[r] = static_cast<int>(s);
  }
  __syncthreads();
  // n[r][e] and row_off[r][e] = row_start[r] + sum_{e' < e} n[r][e'], one warp per round;
  // with mb_prefix, also the prefix over experts of their 128-row blocks in the round.
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r = warp; r < R; r += kWarps) {
    const long long base_r = static_cast<long long>(r) * C;
    int running = row_start[r];
    int running_mb = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int x = e0 + lane;
      int nv = 0;
      if (x < E) {
        const long long rem = s_load[x] - base_r;
        nv = rem <= 0 ? 0 : (rem >= C ? C : static_cast<int>(rem));
      }
      const int mb = (nv + kPipeRowBlock - 1) / kPipeRowBlock;
      int incl = nv, incl_mb = mb;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        const int om = __shfl_up_sync(0xffffffffu, incl_mb, off);
        if (lane >= off) {
          incl += o;
          incl_mb += om;
        }
      }
      if (x < E) {
        n[static_cast<size_t>(r) * E + x] = nv;
        row_off[static_cast<size_t>(r) * E + x] = running + incl - nv;
        if (mb_prefix) mb_prefix[static_cast<size_t>(r) * (E + 1) + x] = running_mb + incl_mb - mb;
      }
      running += __shfl_sync(0xffffffffu, incl, 31);
      running_mb += __shfl_sync(0xffffffffu, incl_mb, 31);
    }
    if (mb_prefix && lane == 0) mb_prefix[static_cast<size_t>(r) * (E + 1) + E] = running_mb;
  }
}

__global__ void __launch_bounds__(kTPB) plan_rank_kernel(const int32_t* __restrict__ idx, int T, int k,
                                                         int E, int C,
                                                         const int32_t* __restrict__ block_base,
                                                         const int32_t* __restrict__ row_off,
                                                         int32_t* __restrict__ round_out,
                                                         int32_t* __restrict__ slot_out,
                                                         int32_t* __restrict__ row_token,
                                                         int32_t* __restrict__ row_dst,
                                                         const int32_t* __restrict__ n,
                                                         const int32_t* __restrict__ row_start,
                                                         int borrow, int max_rounds,
                                                         int32_t* __restrict__ sync, long long sync_words,
                                                         int32_t* dbg) {
  __shared__ uint32_t mask[kWarps][MOE_MAX_E_PLAN];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) mask[i / E][i % E] = 0u;
  sm100::grid_dependency_wait();
  sm100::grid_launch_dependents();
  __syncthreads();
  const int t = blockIdx.x * kTPB + threadIdx.x;
  const bool valid = t < T;
  // the pipelined-rounds kernel expects its counters at zero
  if (sync)
    for (long long i = t; i < sync_words; i += static_cast<long long>(gridDim.x) * kTPB) sync[i] = 0;
  if (valid)
    for (int j = 0; j < k; ++j) {
      const int e = idx[static_cast<size_t>(t) * k + j];
      if (dbg != nullptr && (e < 0 || e >= E)) {   // debug bounds checks: an expert out of range
        record_bad(dbg, kBadPlanPair, t * k + j);
        continue;
      }
      atomicOr(&mask[warp][e], 1u << lane);
    }
  __syncthreads();
  if (!valid) return;
  const uint32_t lower = (1u << lane) - 1u;
  for (int j = 0; j < k; ++j) {
    const size_t p = static_cast<size_t>(t) * k + j;
    const int e = idx[p];
    if (dbg != nullptr && (e < 0 || e >= E)) continue;   // recorded above
    int rank = block_base[static_cast<size_t>(blockIdx.x) * E + e];
    for (int w = 0; w < warp; ++w) rank += __popc(mask[w][e]);
    rank += __popc(mask[warp][e] & lower);
    int r, s;
    if (!borrow) {
      r = rank / C;
      s = rank - r * C;
    } else {   // the expert's rounds hold its pairs in token order: find the round of this rank
      r = 0;
      int before = 0;   // the planner placed every pair within max_rounds rounds
      while (r + 1 < max_rounds && rank >= before + n[static_cast<size_t>(r) * E + e])
        before += n[static_cast<size_t>(r++) * E + e];
      s = rank - before;
    }
    round_out[p] = r;
    slot_out[p] = s;
    if (dbg != nullptr && (r < 0 || r >= max_rounds)) {
      record_bad(dbg, kBadPlanPair, static_cast<int>(p));
      continue;
    }
    const int pos = row_off[static_cast<size_t>(r) * E + e] + s;
    if (dbg != nullptr && (pos < 0 || static_cast<long long>(pos) >= static_cast<long long>(T) * k)) {
      record_bad(dbg, kBadPlanPair, static_cast<int>(p));
      continue;
    }
    row_token[pos] = t;
    // round buffer row: expert e's C rows, or with borrowing the round's rows packed in order
    row_dst[pos] = borrow ? pos - row_start[r] : e * C + s;
  }
}

// dst[i] = src[i] for i < n, with the stores made visible system-wide (dst is host memory
// mapped into the device's address space).
__global__ void __launch_bounds__(kTPB) copy_words_kernel(const int32_t* __restrict__ src, int32_t* dst, int n) {
  sm100::grid_dependency_wait();
  for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = src[i];
  __threadfence_system();
  sm100::pdl_trigger_early();
  sm100::pdl_trigger_late();
}

}  // namespace

cudaError_t launch_copy_words(const int32_t* src, int32_t* dst, int n, cudaStream_t stream) {
  launch_begin(kKindPlan, stream);
  const cudaError_t err = launch_pdl(copy_words_kernel, dim3(1), dim3(kTPB), 0, stream, src, dst, n);
  launch_end(kKindPlan, stream);
  return err;
}

cudaError_t launch_plan(const PlanBuffers& b, int T, int k, int E, int C, int max_rounds,
                        cudaStream_t stream) {
  const int blocks = (T + kTPB - 1) / kTPB;
  launch_begin(kKindPlan, stream);
  cudaError_t err = launch_pdl(plan_scan_kernel, dim3(E), dim3(kTPB), 0, stream, b.block_base, blocks, E, C,
                               max_rounds, b.load, b.offsets, b.header, b.n, b.row_off, b.row_start,
                               b.mb_prefix, b.borrow);
  if (blocks > 0 && err == cudaSuccess)
    err = launch_pdl(plan_rank_kernel, dim3(blocks), dim3(kTPB), 0, stream, b.idx, T, k, E, C,
                     b.block_base, b.row_off, b.round, b.slot, b.row_token, b.row_dst, b.n, b.row_start,
                     b.borrow, max_rounds, b.sync, b.sync_words, b.dbg);
  launch_end(kKindPlan, stream, blocks > 0 ? 2 : 1);
  return err;
}

}  // namespace moe
