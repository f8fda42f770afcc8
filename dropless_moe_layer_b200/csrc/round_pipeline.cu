// round_pipeline.cu - several rounds of the layer as one persistent, dependency-driven launch.
//
// "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, multi-round dropless MoE
// item [section "Scaling MoE", Fig. 6]: every round is dispatch -> compute -> collect at a fixed
// per-expert capacity, and the collect of one round overlaps the dispatch of the next, so only
// the first dispatch and the last collect are exposed. Its per-expert-overhead item names kernel
// dispatch and metadata handling as what held the MoE layer's efficiency down. On one GPU the
// late rounds of a skewed batch are thin (a few experts, a few hundred rows), and as separate
// launches each step pays a launch, a prologue and a pipeline fill. Here one CTA per SM runs
// rounds [r0, R) and consecutive rounds overlap wherever the data allows.
//
// Roles of a CTA (320 threads):
//   warps 0..5  the tcgen05 GEMM pipeline of gemm_sm100.cuh (TMA producer, MMA issuer, four
//               epilogue warps) over the GEMM tile list below, tiles dealt round-robin to CTAs;
//   warps 6..9  copy warps: the dispatch rows and combine items of every round, dealt
//               round-robin over all copy warps of the grid.
// GEMM tile list, for r = r0..R-1: the gate/up tiles of round r (128 rows x 32 gate columns,
// MMA N = 64, every column slice of a 128-row block before the next block), then its down
// tiles (128 rows x 64 output columns). Copy steps: dispatch(r0), then for each r:
// dispatch(r + 1), combine(r).
//
// Dependencies, tracked by cumulative int32 counters in the workspace (zero before a launch;
// the last CTA to finish zeroes them again). Every wait is bounded in time.
//   gate/up(r, e, m)  after dispatch(r) rows of block (e, m)     buf is its A operand
//                     after down(r-1) of block (e, m)           it overwrites h
//   down(r, e, m)     after gate/up(r) of block (e, m)          h is its A operand
//                     after combine(r-1)                        it overwrites out
//   dispatch(r)       after every gate/up tile of round r-1     it overwrites buf
//   combine(r)        after every down tile of round r          it reads out
//                     after combine(r-1)                        y accumulates in round order
// Each dependency points to a step earlier in the order
//   D(r0) G(r0) N(r0) D(r0+1) C(r0) G(r0+1) N(r0+1) D(r0+2) C(r0+1) ...
// and every role takes its own steps in that order. With every CTA resident (a cooperative
// launch of one CTA per SM) the earliest unfinished step always has its inputs and a role that
// is working on it, so the launch cannot deadlock.
//
// Memory ordering: a producer of data issues its stores, a generic-to-async proxy fence and a
// gpu-scope fence, then a release add on the counter; a consumer acquires the counter and, before
// a TMA load, issues the proxy fence as well.
#include <cuda.h>

#include <atomic>

#include "copy_phases.cuh"
#include "gemm_sm100.cuh"
#include "kernels.h"
#include "moe.h"

namespace moe {

namespace {

using namespace gemm;

constexpr int kBN = 2 * kPipeGuWidth;                      // MMA N of both GEMMs
constexpr int kPStageBytes = kABytes + kBN * BK * 2;       // 24 KB
constexpr int kPStages = kRingBytes / kPStageBytes;        // 8
static_assert(kPStages <= kMaxStages, "ring stages");
static_assert(kPipeDnWidth == kBN, "both GEMMs use one stage geometry");
static_assert(kPipeRowBlock == BM, "row blocks are GEMM tiles");
constexpr int kPipeCopyWarps = 4;
constexpr int kPipeThreads = kThreads + 32 * kPipeCopyWarps;
constexpr int kEpiWarps = 4;

#ifdef MOE_TRACE
// Diagnostic build only (-DMOE_TRACE): %globaltimer stamps of the launch, written to a buffer
// that moe_trace_set() installs. Layout (u64): [0] first CTA start (min), [1] last CTA end
// (max); from 16, eight words per GEMM tile: inputs ready, first load issued, epilogue done,
// CTA, first stage consumed by the MMA, last MMA committed, accumulator seen by the epilogue,
// last load issued; from 16 + 8 * kTraceTasks, eight words per round: dispatch start (min),
// dispatch end (max), combine start (min), combine end (max).
constexpr int kTraceTasks = 1 << 16;
constexpr int kTraceRounds = 4096;
__device__ unsigned long long* g_trace = nullptr;
__device__ __forceinline__ void trace_min(long long i, unsigned long long v) {
  if (g_trace) atomicMin(g_trace + i, v);
}
__device__ __forceinline__ void trace_max(long long i, unsigned long long v) {
  if (g_trace) atomicMax(g_trace + i, v);
}
__device__ __forceinline__ void trace_task(int task, int word, unsigned long long v) {
  if (g_trace && task < kTraceTasks) g_trace[16 + 8ll * task + word] = v;
}
__device__ __forceinline__ long long trace_round(int r, int word) {
  return 16 + 8ll * kTraceTasks + 8ll * (r < kTraceRounds ? r : kTraceRounds - 1) + word;
}
#define MOE_TRACE_DO(x) x
#else
#define MOE_TRACE_DO(x)
#endif

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int ld_relaxed(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release(int32_t* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ int ld_acquire_cta_shared(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_cta_shared(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(p)), "r"(v) : "memory");
}

// Marks the launch as failed: status bit plus the abort word every wait watches.
__device__ __forceinline__ void give_up(const PipelineArgs& a) {
  atomicOr(a.status, kStatusTimeoutPipeline);
  atomicExch(a.sync + kSyncAbort, 1);
}

// Bounded wait (one thread) until *p >= target. False if the time limit passed or another CTA
// gave up first.
__device__ bool wait_counter(const PipelineArgs& a, const int32_t* p, int target) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  unsigned ns = 32;
  while (true) {
    __nanosleep(ns);
    if (ld_acquire(p) >= target) return true;
    if (ns < 256) ns <<= 1;
    if (ld_relaxed(a.sync + kSyncAbort) != 0) return false;
    if (global_timer_ns() - t0 > MOE_WAIT_LIMIT_NS) {
      give_up(a);
      return false;
    }
  }
}

// Same on a value that another warp of this CTA publishes in shared memory.
__device__ bool wait_shared(const PipelineArgs& a, const int* p, int target) {
  if (ld_acquire_cta_shared(p) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    __nanosleep(64);
    if (ld_acquire_cta_shared(p) >= target) return true;
    if (ld_relaxed(a.sync + kSyncAbort) != 0) return false;
    if (global_timer_ns() - t0 > MOE_WAIT_LIMIT_NS) {
      give_up(a);
      return false;
    }
  }
}

// Walks the GEMM tile list forward, one round at a time.
struct Cursor {
  int r = 0;            // round of the tiles in [base, end)
  int base = 0;
  int end = 0;
  int gu_tiles = 0;     // gate/up tiles of round r (the first ones of the round)
  int comb_before = 0;  // combine items of rounds r0..r-1
};

__device__ __forceinline__ void cursor_load(Cursor& c, const PipelineArgs& a) {
  const int mblocks = a.mb_prefix[static_cast<size_t>(c.r) * (a.E + 1) + a.E];
  c.gu_tiles = mblocks * (a.F / kPipeGuWidth);
  c.end = c.base + c.gu_tiles + mblocks * (a.d / kPipeDnWidth);
}

__device__ __forceinline__ void cursor_init(Cursor& c, const PipelineArgs& a) {
  c.r = a.r0;
  c.base = 0;
  c.comb_before = 0;
  cursor_load(c, a);
}

// Combine items of round r: its rows when there are fewer rows than tokens, else its tokens.
__device__ __forceinline__ int combine_items(const PipelineArgs& a, int r, bool* by_rows) {
  const int rows = a.row_start[r + 1] - a.row_start[r];
  *by_rows = rows < a.T;
  return rows < a.T ? rows : a.T;
}

// Moves the cursor to the round holding `task`; false past the last round.
__device__ __forceinline__ bool cursor_seek(Cursor& c, const PipelineArgs& a, int task) {
  while (task >= c.end) {
    bool by_rows;
    c.comb_before += combine_items(a, c.r, &by_rows);
    c.base = c.end;
    if (++c.r >= a.R) return false;
    cursor_load(c, a);
  }
  return true;
}

struct Tile {
  bool gu;   // gate/up (else down)
  int r, e, m, nt, kb;
};

__device__ __forceinline__ void decode(const Cursor& c, const PipelineArgs& a, int task, Tile& t) {
  int local = task - c.base;
  t.r = c.r;
  t.gu = local < c.gu_tiles;
  int per;
  if (t.gu) {
    per = a.F / kPipeGuWidth;
    t.kb = a.d / BK;
  } else {
    local -= c.gu_tiles;
    per = a.d / kPipeDnWidth;
    t.kb = a.F / BK;
  }
  const int blk = local / per;
  t.nt = local - blk * per;
  const int32_t* pre = a.mb_prefix + static_cast<size_t>(c.r) * (a.E + 1);
  int lo = 0, hi = a.E - 1;   // largest e with pre[e] <= blk (an expert with blocks)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= blk) lo = mid; else hi = mid - 1;
  }
  t.e = lo;
  t.m = blk - pre[lo];
}

struct Counters {
  int32_t* disp;   // [E * MB] dispatch rows written into block (e, m), all rounds
  int32_t* gu;     // [E * MB] gate/up tile quarters finished on block (e, m)
  int32_t* dn;     // [E * MB] down tile quarters finished on block (e, m)
  int mb;          // 128-row blocks per expert = ceil(C / 128)
};

__device__ __forceinline__ Counters counters(const PipelineArgs& a) {
  Counters k;
  k.mb = static_cast<int>(pipe_row_blocks(a.C));
  k.disp = a.sync + kSyncBlocks;
  k.gu = k.disp + static_cast<size_t>(a.E) * k.mb;
  k.dn = k.gu + static_cast<size_t>(a.E) * k.mb;
  return k;
}

// Producer: every input of tile t is in memory.
__device__ bool wait_inputs(const PipelineArgs& a, const Counters& cn, const Cursor& c, const Tile& t) {
  const int blk = t.e * cn.mb + t.m;
  const int rr = t.r - a.r0;   // rounds of this launch before t.r
  if (t.gu) {
    const int full = min(BM, a.C - t.m * BM);
    const int nv = a.n[static_cast<size_t>(t.r) * a.E + t.e] - t.m * BM;
    const int rows = nv < 0 ? 0 : (nv > BM ? BM : nv);
    if (!wait_counter(a, cn.disp + blk, rr * full + rows)) return false;
    if (rr > 0 && !wait_counter(a, cn.dn + blk, rr * kEpiWarps * (a.d / kPipeDnWidth))) return false;
  } else {
    if (!wait_counter(a, cn.gu + blk, (rr + 1) * kEpiWarps * (a.F / kPipeGuWidth))) return false;
    if (rr > 0 && !wait_counter(a, a.sync + kSyncCombTotal, c.comb_before)) return false;
  }
  return true;
}

// Copy warps: a round-level wait. Copy warp 0 of the CTA polls the global counter and publishes
// what it saw in shared memory; the other copy warps wait on that word.
__device__ bool round_wait(const PipelineArgs& a, int* seen, const int32_t* counter, int target, int cwarp) {
  const int lane = threadIdx.x & 31;
  int ok = 1;
  if (lane == 0) {
    if (cwarp == 0) {
      ok = wait_counter(a, counter, target);
      if (ok) st_release_cta_shared(seen, target);
    } else {
      ok = wait_shared(a, seen, target);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// The four copy warps of this CTA: dispatch rows and combine items of rounds r0..R-1.
__device__ void copy_role(const PipelineArgs& a, const Counters& cn, int* seen) {
  const int lane = threadIdx.x & 31;
  const int cwarp = (threadIdx.x >> 5) - kThreads / 32;
  const int gw = blockIdx.x * kPipeCopyWarps + cwarp;
  const int W = gridDim.x * kPipeCopyWarps;
  const int vecs = a.d / 8;
  const copy::CombineArgs comb{a.out, a.y, a.idx, a.gate, a.round, a.slot, a.T, a.k, a.C, a.d};

  auto dispatch_round = [&](int r) {
    const int begin = a.row_start[r], rows = a.row_start[r + 1] - begin;
    MOE_TRACE_DO(if (lane == 0 && gw < rows) trace_min(trace_round(r, 0), global_timer_ns()));
    for (int i = gw; i < rows; i += W) {
      const int row = begin + i;
      const int t = a.row_token[row], dst = a.row_dst[row];
      const int e = dst / a.C, m = (dst - e * a.C) / BM;
      copy::dispatch_row(reinterpret_cast<const uint4*>(a.x), reinterpret_cast<uint4*>(a.buf), t, dst, vecs, lane);
      fence_proxy_async();   // the row is read next by TMA (the async proxy)
      __threadfence();
      __syncwarp();
      if (lane == 0) red_release(cn.disp + e * cn.mb + m, 1);
    }
    MOE_TRACE_DO(if (lane == 0 && gw < rows) trace_max(trace_round(r, 1), global_timer_ns()));
  };

  dispatch_round(a.r0);
  int gu_through = 0, dn_through = 0, comb_before = 0;
  for (int r = a.r0; r < a.R; ++r) {
    const int mblocks = a.mb_prefix[static_cast<size_t>(r) * (a.E + 1) + a.E];
    gu_through += mblocks * kEpiWarps * (a.F / kPipeGuWidth);
    dn_through += mblocks * kEpiWarps * (a.d / kPipeDnWidth);
    if (r + 1 < a.R) {
      // buf is free once every gate/up tile of round r has read it
      if (!round_wait(a, &seen[0], a.sync + kSyncGuTotal, gu_through, cwarp)) return;
      fence_proxy_async();
      dispatch_round(r + 1);
    }
    if (!round_wait(a, &seen[1], a.sync + kSyncDnTotal, dn_through, cwarp)) return;
    if (!round_wait(a, &seen[2], a.sync + kSyncCombTotal, comb_before, cwarp)) return;
    bool by_rows;
    const int items = combine_items(a, r, &by_rows);
    MOE_TRACE_DO(if (lane == 0 && gw < items) trace_min(trace_round(r, 2), global_timer_ns()));
    int done = 0;
    for (int u = gw; u < items; u += W, ++done) {
      if (by_rows) {
        const int row = a.row_start[r] + u;
        copy::combine_token(comb, a.row_token[row], r, a.row_dst[row] / a.C);
      } else {
        copy::combine_token(comb, u, r);
      }
    }
    if (done > 0) {
      __threadfence();
      __syncwarp();
      if (lane == 0) red_release(a.sync + kSyncCombTotal, done);
      MOE_TRACE_DO(if (lane == 0) trace_max(trace_round(r, 3), global_timer_ns()));
    }
    comb_before += items;
  }
}

__global__ void __launch_bounds__(kPipeThreads, 1)
    round_pipeline_kernel(const __grid_constant__ CUtensorMap a_gu, const __grid_constant__ CUtensorMap b_gu,
                          const __grid_constant__ CUtensorMap a_dn, const __grid_constant__ CUtensorMap b_dn,
                          const PipelineArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int seen[3];
  __shared__ int last_cta;
  const Smem s = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&a_gu);
    tma_prefetch_desc(&b_gu);
    tma_prefetch_desc(&a_dn);
    tma_prefetch_desc(&b_dn);
    seen[0] = seen[1] = seen[2] = 0;
  }
  const uint32_t tmem = setup(s);
  grid_dependency_wait();
  const Counters cn = counters(a);
  MOE_TRACE_DO(if (threadIdx.x == 0) trace_min(0, global_timer_ns()));

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      Cursor c;
      cursor_init(c, a);
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      auto load_b = [&](const Tile& t, int kb, uint32_t sB, uint32_t fb) {
        if (t.gu) {
          tma_load_3d(sB, &b_gu, fb, kb * BK, t.nt * kPipeGuWidth, t.e);
          tma_load_3d(sB + kPipeGuWidth * BK * 2, &b_gu, fb, kb * BK, a.F + t.nt * kPipeGuWidth, t.e);
        } else {
          tma_load_3d(sB, &b_dn, fb, kb * BK, t.nt * kPipeDnWidth, t.e);
        }
      };
      for (int task = blockIdx.x; ok; task += gridDim.x) {
        if (!cursor_seek(c, a, task)) break;
        Tile t;
        decode(c, a, task, t);
        const CUtensorMap* ma = t.gu ? &a_gu : &a_dn;
        // Weights do not depend on earlier steps: the B tiles of the first stages are requested
        // before the wait for this tile's A rows, so they arrive while it waits.
        const int pre = t.kb < kPStages ? t.kb : kPStages;
        const int first = stage;
        MOE_TRACE_DO(trace_task(task, 1, global_timer_ns()); trace_task(task, 3, blockIdx.x));
        int armed = 0;
        for (; armed < pre; ++armed) {
          if (!mbar_wait(smem_addr(&s.empty[stage]), phase ^ 1u, s.abort)) {
            ok = false;
            break;
          }
          const uint32_t sA = smem_addr(s.stage + stage * kPStageBytes);
          const uint32_t fb = smem_addr(&s.full[stage]);
          mbar_arrive_expect_tx(fb, kPStageBytes);
          load_b(t, armed, sA + kABytes, fb);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kPStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        const bool inputs = ok && wait_inputs(a, cn, c, t);
        MOE_TRACE_DO(trace_task(task, 0, global_timer_ns()));
        fence_proxy_async();
        // A loads of the armed stages (issued even when giving up, so every armed stage completes)
        for (int i = 0; i < armed; ++i) {
          const int st = (first + i) % kPStages;
          tma_load_3d(smem_addr(s.stage + st * kPStageBytes), ma, smem_addr(&s.full[st]), i * BK, t.m * BM, t.e);
        }
        if (!inputs) {
          ok = false;
          break;
        }
        for (int kb = pre; kb < t.kb; ++kb) {
          if (!mbar_wait(smem_addr(&s.empty[stage]), phase ^ 1u, s.abort)) {
            ok = false;
            break;
          }
          const uint32_t sA = smem_addr(s.stage + stage * kPStageBytes);
          const uint32_t fb = smem_addr(&s.full[stage]);
          mbar_arrive_expect_tx(fb, kPStageBytes);
          load_b(t, kb, sA + kABytes, fb);
          tma_load_3d(sA, ma, fb, kb * BK, t.m * BM, t.e);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kPStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        MOE_TRACE_DO(trace_task(task, 7, global_timer_ns()));
      }
      if (!ok) {
        atomicOr(a.status, kStatusTimeoutProducer);
        atomicExch(a.sync + kSyncAbort, 1);
        *s.abort = 1;
        for (int i = 0; i < kPStages; ++i)   // let issued loads land before shared memory is reused
          if ((issued >> i) & 1u) mbar_wait(smem_addr(&s.full[i]), (issued_parity >> i) & 1u, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      Cursor c;
      cursor_init(c, a);
      const uint32_t idesc = idesc_bf16_f32(BM, kBN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int task = blockIdx.x; ok; task += gridDim.x) {
        if (!cursor_seek(c, a, task)) break;
        Tile t;
        decode(c, a, task, t);
        if (!mbar_wait(smem_addr(&s.tempty[acc]), acc_phase ^ 1u, s.abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kAccCols);
        for (int kb = 0; kb < t.kb; ++kb) {
          if (!mbar_wait(smem_addr(&s.full[stage]), phase, s.abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          MOE_TRACE_DO(if (kb == 0) trace_task(task, 4, global_timer_ns()));
          const uint32_t sA = smem_addr(s.stage + stage * kPStageBytes);
          const uint64_t adesc = smem_desc_sw128(sA);
          const uint64_t bdesc = smem_desc_sw128(sA + kABytes);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            mma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit(smem_addr(&s.empty[stage]));
          if (++stage == kPStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(smem_addr(&s.tfull[acc]));
        MOE_TRACE_DO(trace_task(task, 5, global_timer_ns()));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) {
        atomicOr(a.status, kStatusTimeoutMma);
        atomicExch(a.sync + kSyncAbort, 1);
        *s.abort = 1;
        mma_commit(smem_addr(s.drain));   // wait for every MMA already issued
        mbar_wait(smem_addr(s.drain), 0, nullptr);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    Cursor c;
    cursor_init(c, a);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int task = blockIdx.x;; task += gridDim.x) {
      if (!cursor_seek(c, a, task)) break;
      Tile t;
      decode(c, a, task, t);
      const bool ready = __all_sync(0xffffffffu, mbar_wait(smem_addr(&s.tfull[acc]), acc_phase, s.abort));
      if (!ready) {
        if (lane == 0) {
          atomicOr(a.status, kStatusTimeoutEpilogue);
          atomicExch(a.sync + kSyncAbort, 1);
        }
        *s.abort = 1;
        break;
      }
      tc_fence_after();
      MOE_TRACE_DO(if (warp == 2 && lane == 0) trace_task(task, 6, global_timer_ns()));
      const int row = t.m * BM + q * 32 + lane;
      const bool valid = row < a.n[static_cast<size_t>(t.r) * a.E + t.e];
      const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kAccCols);
      if (t.gu) {
        uint16_t* orow = a.h + (static_cast<size_t>(t.e) * a.C + row) * a.F + t.nt * kPipeGuWidth;
        store_swiglu(tb, kPipeGuWidth, orow, valid);
      } else {
        uint16_t* orow = a.out + (static_cast<size_t>(t.e) * a.C + row) * a.d + t.nt * kPipeDnWidth;
        store_bf16(tb, kPipeDnWidth, orow, valid);
      }
      tc_fence_before();
      mbar_arrive(smem_addr(&s.tempty[acc]));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
      // this warp's quarter of the tile is in memory
      fence_proxy_async();
      __threadfence();
      __syncwarp();
      if (lane == 0) {
        const int blk = t.e * cn.mb + t.m;
        red_release((t.gu ? cn.gu : cn.dn) + blk, 1);
        red_release(a.sync + (t.gu ? kSyncGuTotal : kSyncDnTotal), 1);
        MOE_TRACE_DO(if (warp == 2) trace_task(task, 2, global_timer_ns()));
      }
    }
    __syncwarp();
  } else {
    copy_role(a, cn, seen);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  MOE_TRACE_DO(if (threadIdx.x == 0) trace_max(1, global_timer_ns()));
  if (threadIdx.x == 0) {
    __threadfence();
    last_cta = atomicAdd(a.sync + kSyncExit, 1) == static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (last_cta) {   // every other CTA is done with the counters: leave them at zero
    __threadfence();
    const long long words = pipe_sync_words(a.E, a.C);
    for (long long i = threadIdx.x; i < words; i += blockDim.x) a.sync[i] = 0;
  }
  pdl_trigger_late();
  release_tmem(tmem);
}

}  // namespace

#ifdef MOE_TRACE
extern "C" MOE_API int moe_trace_set(void* buffer) {
  unsigned long long* p = static_cast<unsigned long long*>(buffer);
  return cudaMemcpyToSymbol(g_trace, &p, sizeof(p)) == cudaSuccess ? 0 : -5;
}
#endif

cudaError_t launch_round_pipeline(const PipelineArgs& a, cudaStream_t stream) {
  if (a.r0 >= a.R) return cudaSuccess;
  CUtensorMap m_agu, m_bgu, m_adn, m_bdn;
  cudaError_t e = gemm::make_map(&m_agu, a.buf, a.d, a.C, a.E, BM);
  if (e == cudaSuccess) e = gemm::make_map(&m_bgu, a.w_gate_up, a.d, 2ull * a.F, a.E, kPipeGuWidth);
  if (e == cudaSuccess) e = gemm::make_map(&m_adn, a.h, a.F, a.C, a.E, BM);
  if (e == cudaSuccess) e = gemm::make_map(&m_bdn, a.w_down, a.F, a.d, a.E, kPipeDnWidth);
  if (e != cudaSuccess) return e;
  static std::atomic<uint64_t> configured{0};   // one bit per device ordinal
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(round_pipeline_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured.fetch_or(bit);
  }
  // Cooperative: the CTAs wait on one another's counters, so all of them must be resident at
  // once (one per SM); the launch fails instead of starting if that cannot be guaranteed.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(kPipeThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  launch_begin(kKindPipeline, stream);
  e = cudaLaunchKernelEx(&cfg, round_pipeline_kernel, m_agu, m_bgu, m_adn, m_bdn, a);
  launch_end(kKindPipeline, stream);
  return e;
}

}  // namespace moe
