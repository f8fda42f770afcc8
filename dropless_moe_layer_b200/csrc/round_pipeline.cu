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
// Roles of a CTA (512 threads):
//   warps 0..5    the tcgen05 GEMM pipeline of gemm_sm100.cuh (TMA producer, MMA issuer, four
//                 epilogue warps) over the GEMM tile list below: the producer claims the next
//                 tile of the list (a global counter) when it is ready for one, and passes its
//                 index to the MMA and epilogue warps through a small shared-memory ring;
//   warps 6..9    dispatch warps: each round's rows, in contiguous slices per warp of the grid;
//   warps 10..15  combine warps: each owns a fixed set of tokens and combines them round by round.
// GEMM tile list: gate/up tiles (128 rows x GW gate columns, MMA N = 2 GW, every column slice
// of a 128-row block before the next block) and down tiles (128 rows x 2 GW output columns),
// phase by phase in the order G(r0) G(r0+1) N(r0) G(r0+2) N(r0+1) ... N(R-1). GW is 64 when d
// is a multiple of 128 (fewer, wider tiles: each tile's fixed costs are paid for twice the
// columns), else 32 (a template parameter of the kernel; both use the same 192 KB ring).
//
// Round r uses buffer set p = (r - r0) & 1 (buf, h and out exist twice), so a round's buffers
// are reused two rounds later and consecutive rounds do not wait on each other's reads.
// Dependencies, tracked by int32 counters per buffer set in the workspace (zero before a
// launch; the last CTA to finish zeroes them again). Every wait is bounded in time.
//   dispatch(r, e, m) after gate/up(r-2) of block (e, m)        it overwrites buf[p]
//   gate/up(r, e, m)  after dispatch(r) rows of block (e, m)     buf[p] is its A operand
//                     after down(r-2) of block (e, m)           it overwrites h[p]
//   down(r, e, m)     after gate/up(r) of block (e, m)          h[p] is its A operand
//                     after combine(r-2) read block (e, m)      it overwrites out[p]
//   combine(r, t)     after down(r) of the blocks holding t's    it reads out[p]
//                     round-r rows (y[t] accumulates in round order by construction: one
//                     warp owns token t for all rounds)
// A counter of set p only ever receives the contributions of rounds of set p in round order
// (round r+2 of a set cannot start its step before round r's is complete), so "count >=
// target" means exactly "the earlier rounds of the set are done". Each dependency points to a
// step earlier in the order
//   D(r0) G(r0)  D(r0+1) G(r0+1) N(r0)  D(r0+2) G(r0+2) N(r0+1) C(r0)  D(r0+3) G(r0+3) N(r0+2)
//   C(r0+1) ...
// and every role takes its own steps in that order (a combine warp its tokens round by round).
// With every CTA resident (a cooperative launch of one CTA per SM) the earliest unfinished step
// always has its inputs and a role that is working on it, so the launch cannot deadlock.
//
// Memory ordering: the threads that wrote a step's data issue a generic-to-async proxy fence
// (the data may next be read by TMA) and meet at __syncwarp; one lane then adds to the counter
// with release semantics (cumulative over the warp's writes). A consumer acquires the counter
// and, before a TMA load, issues the proxy fence as well.
#include <cuda.h>

#include <atomic>

#include "copy_phases.cuh"
#include "gemm_sm100.cuh"
#include "kernels.h"
#include "moe.h"

namespace moe {

namespace {

using namespace gemm;

// Stage geometry for GW gate columns per gate/up tile: MMA N = 2 GW for both GEMMs (a down
// tile has 2 GW output columns), so one ring serves both.
template <int GW>
struct Geom {
  static constexpr int kBN = 2 * GW;                               // MMA N of both GEMMs
  static constexpr int kStageBytes = kABytes + kBN * BK * 2;       // 24 KB (GW 32), 32 KB (GW 64)
  static constexpr int kStages = kRingBytes / kStageBytes;         // 8, 6
  static_assert(kStages >= 2 && kStages <= kMaxStages, "ring stages");
};
static_assert(kPipeRowBlock == BM, "row blocks are GEMM tiles");
constexpr int kDispWarps = 4;
constexpr int kCombWarps = 6;
constexpr int kFirstDispWarp = kThreads / 32;
constexpr int kFirstCombWarp = kFirstDispWarp + kDispWarps;
constexpr int kPipeThreads = kThreads + 32 * (kDispWarps + kCombWarps);
constexpr int kEpiWarps = 4;
constexpr int kRing = 4;   // claimed tiles in flight between the producer and the consumers

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
  for (uint32_t i = 1;; ++i) {
    __nanosleep(ns);
    if (ld_acquire(p) >= target) return true;
    if (ns < 256) ns <<= 1;
    if ((i & 7) == 0 && ld_relaxed(a.sync + kSyncAbort) != 0) return false;
    if (global_timer_ns() - t0 > MOE_WAIT_LIMIT_NS) {
      give_up(a);
      return false;
    }
  }
}

// Walks the GEMM tile list forward, one phase (the gate/up or the down tiles of one round) at a
// time. Phase order: G(r0), then for each r: G(r + 1), N(r) -- the gate/up tiles run one round
// ahead, so that CTAs waiting for a round's gate/up results are not the ones that could start
// the next round's gate/up.
struct Cursor {
  bool gu = true;        // phase kind: gate/up (else down)
  int r = 0;             // round of the phase
  int base = 0;          // first task of the phase
  int end = 0;           // one past its last task
};

__device__ __forceinline__ void cursor_load(Cursor& c, const PipelineArgs& a) {
  const int mblocks = a.mb_prefix[static_cast<size_t>(c.r) * (a.E + 1) + a.E];
  c.end = c.base + mblocks * (c.gu ? a.F / a.gw : a.d / (2 * a.gw));
}

__device__ __forceinline__ void cursor_init(Cursor& c, const PipelineArgs& a) {
  c.gu = true;
  c.r = a.r0;
  c.base = 0;
  cursor_load(c, a);
}

// The phase after the cursor's; false at the end of the list.
__device__ __forceinline__ bool cursor_next(Cursor& c, const PipelineArgs& a) {
  if (c.gu && c.r == a.r0) {          // G(r0) -> G(r0 + 1), or N(r0) with one round
    if (c.r + 1 < a.R) ++c.r; else c.gu = false;
  } else if (c.gu) {                  // G(r) -> N(r - 1)
    c.gu = false;
    --c.r;
  } else if (c.r + 2 < a.R) {         // N(r) -> G(r + 2)
    c.gu = true;
    c.r += 2;
  } else if (c.r + 1 < a.R) {         // N(r) -> N(r + 1) at the end of the list
    ++c.r;
  } else {
    return false;
  }
  c.base = c.end;
  cursor_load(c, a);
  return true;
}

// Moves the cursor to the phase holding `task`; false past the end of the list.
__device__ __forceinline__ bool cursor_seek(Cursor& c, const PipelineArgs& a, int task) {
  while (task >= c.end)
    if (!cursor_next(c, a)) return false;
  return true;
}

struct Tile {
  bool gu;   // gate/up (else down)
  int r, e, m, nt, kb;
};

__device__ __forceinline__ void decode(const Cursor& c, const PipelineArgs& a, int task, Tile& t) {
  const int local = task - c.base;
  t.r = c.r;
  t.gu = c.gu;
  const int per = c.gu ? a.F / a.gw : a.d / (2 * a.gw);
  t.kb = c.gu ? a.d / BK : a.F / BK;
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
  int32_t* disp[2];   // [E * MB] per set: dispatch rows written into block (e, m)
  int32_t* gu[2];     // [E * MB] per set: gate/up tile quarters finished on block (e, m)
  int32_t* dn[2];     // [E * MB] per set: down tile quarters finished on block (e, m)
  int32_t* rd[2];     // [E * MB] per set: rows of block (e, m) of out read by the combine
  int mb;             // 128-row blocks per expert = ceil(C / 128)
};

__device__ __forceinline__ Counters counters(const PipelineArgs& a) {
  Counters k;
  k.mb = static_cast<int>(pipe_row_blocks(a.C));
  const size_t n = static_cast<size_t>(a.E) * k.mb * kSyncStride;
  int32_t* base = a.sync + kSyncBlocks;
  for (int p = 0; p < 2; ++p) {
    k.disp[p] = base + p * n;
    k.gu[p] = base + (2 + p) * n;
    k.dn[p] = base + (4 + p) * n;
    k.rd[p] = base + (6 + p) * n;
  }
  return k;
}

// Producer: every input of tile t is in memory and its output buffer is free.
__device__ bool wait_inputs(const PipelineArgs& a, const Counters& cn, const Cursor& c, const Tile& t) {
  const int blk = (t.e * cn.mb + t.m) * kSyncStride;
  const int p = (t.r - a.r0) & 1;
  const int q = (t.r - a.r0) >> 1;   // earlier rounds of this launch on the same buffer set
  if (t.gu) {
    const int full = min(BM, a.C - t.m * BM);
    const int nv = a.n[static_cast<size_t>(t.r) * a.E + t.e] - t.m * BM;
    const int rows = nv < 0 ? 0 : (nv > BM ? BM : nv);
    // round r0's rows were dispatched by an earlier kernel: set 0 counts them as present
    const int pre = a.r0_dispatched && p == 0 ? full : 0;
    if (!wait_counter(a, cn.disp[p] + blk, q * full + rows - pre)) return false;
    if (q > 0 && !wait_counter(a, cn.dn[p] + blk, q * kEpiWarps * (a.d / (2 * a.gw)))) return false;
  } else {
    if (!wait_counter(a, cn.gu[p] + blk, (q + 1) * kEpiWarps * (a.F / a.gw))) return false;
    if (q > 0 && !wait_counter(a, cn.rd[p] + blk, q * min(BM, a.C - t.m * BM))) return false;
  }
  return true;
}

// Dispatch warps: round r's rows x[token] -> buf[p][e][slot], each warp a contiguous slice.
__device__ void dispatch_role(const PipelineArgs& a, const Counters& cn) {
  const int lane = threadIdx.x & 31;
  const int dw = (threadIdx.x >> 5) - kFirstDispWarp;
  const int gw = blockIdx.x * kDispWarps + dw;
  const int W = gridDim.x * kDispWarps;
  const int vecs = a.d / 8;
  for (int r = a.r0 + (a.r0_dispatched ? 1 : 0); r < a.R; ++r) {
    const int p = (r - a.r0) & 1;
    const int q = (r - a.r0) >> 1;
    // block (e, m) of buf[p] is free once every gate/up tile of it in round r-2 has read it
    const int war_target = q * kEpiWarps * (a.F / a.gw);
    const int begin = a.row_start[r], rows = a.row_start[r + 1] - begin;
    const int chunk = (rows + W - 1) / W;
    const int lo = gw * chunk, hi = min(rows, lo + chunk);
    for (int b = lo; b < hi; b += 32) {
      const int nr = min(32, hi - b);
      int tok = 0, dst = 0, blk = -1;
      if (lane < nr) {
        tok = a.row_token[begin + b + lane];
        dst = a.row_dst[begin + b + lane];
        const int e = dst / a.C;
        blk = (e * cn.mb + (dst - e * a.C) / BM) * kSyncStride;
      }
      // rows are in (expert, slot) order: runs of rows of the same block
      const int prev = __shfl_up_sync(0xffffffffu, blk, 1);
      const bool head = lane < nr && (lane == 0 || prev != blk);
      const uint32_t heads = __ballot_sync(0xffffffffu, head);
      const uint32_t later = lane == 31 ? 0u : (heads & ~((2u << lane) - 1u));
      const int run_end = later ? __ffs(later) - 1 : nr;
      if (q > 0) {
        int ok = 1;
        if (head) ok = wait_counter(a, cn.gu[p] + blk, war_target);
        if (!__all_sync(0xffffffffu, ok)) return;
        fence_proxy_async();
      }
      copy::copy_rows_flat(reinterpret_cast<const uint4*>(a.x), reinterpret_cast<uint4*>(a.buf[p]), tok, dst,
                           nr, vecs);
      fence_proxy_async();   // the rows are read next by TMA (the async proxy)
      __syncwarp();
      if (head) red_release(cn.disp[p] + blk, run_end - lane);
    }
  }
}

// Combine warps: y[t] (+)= gate * out[p][e][slot] for round r. Each warp owns the tokens
// t = gw + i * W and combines them round by round, so a token's y row is only ever touched by
// one warp, each lane always on the same columns: the rounds are added in order by program
// order alone. A token waits only for the down tiles of the blocks its round-r rows live in;
// once its rows are read it counts them on their blocks, which the down GEMM two rounds later
// waits for before it overwrites them.
__device__ void combine_role(const PipelineArgs& a, const Counters& cn) {
  const int lane = threadIdx.x & 31;
  const int cw = (threadIdx.x >> 5) - kFirstCombWarp;
  const int gw = blockIdx.x * kCombWarps + cw;
  const int W = gridDim.x * kCombWarps;
  const long long span = 32ll * W;   // tokens per chunk (lane i holds the chunk's i-th token)
  int dn_cum[2] = {0, 0};
  for (int r = a.r0; r < a.R; ++r) {
    const int p = (r - a.r0) & 1;
    const int q = (r - a.r0) >> 1;
    const int mblocks = a.mb_prefix[static_cast<size_t>(r) * (a.E + 1) + a.E];
    dn_cum[p] += mblocks * kEpiWarps * (a.d / (2 * a.gw));
    const int blk_target = (q + 1) * kEpiWarps * (a.d / (2 * a.gw));
    const copy::CombineArgs comb{a.out[p], a.y, a.idx, a.gate, a.round, a.slot, a.T, a.k, a.C, a.d};
    bool round_done = false;   // every down tile of round r seen finished
    for (long long c0 = gw; c0 < a.T; c0 += span) {
      const long long tl = c0 + static_cast<long long>(lane) * W;
      bool has = false;
      if (tl < a.T)
        for (int j = 0; j < a.k; ++j) has |= a.round[tl * a.k + j] == r;
      uint32_t todo = __ballot_sync(0xffffffffu, has);
      if (todo == 0u) continue;
      copy::PairLoads next = copy::load_pairs(comb, static_cast<int>(c0 + static_cast<long long>(__ffs(todo) - 1) * W));
      while (todo) {
        const int i = __ffs(todo) - 1;
        todo &= todo - 1;
        const int t = static_cast<int>(c0 + static_cast<long long>(i) * W);
        const copy::PairLoads cur = next;
        if (todo) next = copy::load_pairs(comb, static_cast<int>(c0 + static_cast<long long>(__ffs(todo) - 1) * W));
        const copy::TokenPairs tp = copy::token_pairs(comb, cur, r);
        const int blk = (tp.e * cn.mb + tp.s / BM) * kSyncStride;   // this lane's pair's block
        if (!round_done) {
          int ok = 1;
          if (lane == 0) round_done = ld_acquire(a.sync + kSyncDnTotal + p * kSyncSetStride) >= dn_cum[p];
          round_done = __shfl_sync(0xffffffffu, round_done ? 1 : 0, 0) != 0;
          if (!round_done && lane < tp.npairs) ok = wait_counter(a, cn.dn[p] + blk, blk_target);
          if (!__all_sync(0xffffffffu, ok)) return;
        }
        copy::accumulate_token<16>(comb, t, tp);
        __syncwarp();
        if (lane < tp.npairs) red_release(cn.rd[p] + blk, 1);   // this pair's out row is read
      }
    }
  }
}

template <int GW>
__global__ void __launch_bounds__(kPipeThreads, 1)
    round_pipeline_kernel(const __grid_constant__ CUtensorMap a_gu0, const __grid_constant__ CUtensorMap a_gu1,
                          const __grid_constant__ CUtensorMap b_gu, const __grid_constant__ CUtensorMap a_dn0,
                          const __grid_constant__ CUtensorMap a_dn1, const __grid_constant__ CUtensorMap b_dn,
                          const PipelineArgs a) {
  constexpr int kBN = Geom<GW>::kBN;
  constexpr int kPStageBytes = Geom<GW>::kStageBytes;
  constexpr int kPStages = Geom<GW>::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int last_cta;
  // tile ring: the producer publishes each claimed tile (-1: no more) to the MMA issuer and the
  // four epilogue warps
  __shared__ uint64_t ring_full[kRing], ring_empty[kRing];
  __shared__ int ring_task[kRing];
  const Smem s = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(smem_addr(&ring_full[i]), 1);
      mbar_init(smem_addr(&ring_empty[i]), 1 + kEpiWarps);
    }
    tma_prefetch_desc(&a_gu0);
    tma_prefetch_desc(&a_gu1);
    tma_prefetch_desc(&b_gu);
    tma_prefetch_desc(&a_dn0);
    tma_prefetch_desc(&a_dn1);
    tma_prefetch_desc(&b_dn);
  }
  const uint32_t tmem = setup(s);
  grid_dependency_wait();
  const Counters cn = counters(a);

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
          tma_load_3d(sB, &b_gu, fb, kb * BK, t.nt * GW, t.e);
          tma_load_3d(sB + GW * BK * 2, &b_gu, fb, kb * BK, a.F + t.nt * GW, t.e);
        } else {
          tma_load_3d(sB, &b_dn, fb, kb * BK, t.nt * kBN, t.e);
        }
      };
      int slot = 0;
      uint32_t rphase = 0;
      while (ok) {
        const int task = atomicAdd(a.sync + kSyncNextTask, 1);
        const bool have = cursor_seek(c, a, task);
        if (!mbar_wait(smem_addr(&ring_empty[slot]), rphase ^ 1u, s.abort)) {
          ok = false;
          break;
        }
        ring_task[slot] = have ? task : -1;
        mbar_arrive(smem_addr(&ring_full[slot]));
        if (++slot == kRing) {
          slot = 0;
          rphase ^= 1u;
        }
        if (!have) break;
        Tile t;
        decode(c, a, task, t);
        const bool set1 = ((t.r - a.r0) & 1) != 0;
        const CUtensorMap* ma = t.gu ? (set1 ? &a_gu1 : &a_gu0) : (set1 ? &a_dn1 : &a_dn0);
        // Weights do not depend on earlier steps: the B tiles of the first stages are requested
        // before the wait for this tile's A rows, so they arrive while it waits.
        const int pre = t.kb < kPStages ? t.kb : kPStages;
        const int first = stage;
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
      int slot = 0;
      uint32_t rphase = 0;
      while (ok) {
        if (!mbar_wait(smem_addr(&ring_full[slot]), rphase, s.abort)) {
          ok = false;
          break;
        }
        const int task = ring_task[slot];
        mbar_arrive(smem_addr(&ring_empty[slot]));
        if (++slot == kRing) {
          slot = 0;
          rphase ^= 1u;
        }
        if (task < 0 || !cursor_seek(c, a, task)) break;
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
    int slot = 0;
    uint32_t rphase = 0;
    while (true) {
      if (!__all_sync(0xffffffffu, mbar_wait(smem_addr(&ring_full[slot]), rphase, s.abort))) {
        if (lane == 0) {
          atomicOr(a.status, kStatusTimeoutEpilogue);
          atomicExch(a.sync + kSyncAbort, 1);
        }
        *s.abort = 1;
        break;
      }
      const int task = ring_task[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&ring_empty[slot]));
      if (++slot == kRing) {
        slot = 0;
        rphase ^= 1u;
      }
      if (task < 0 || !cursor_seek(c, a, task)) break;
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
      const int row = t.m * BM + q * 32 + lane;
      const bool valid = row < a.n[static_cast<size_t>(t.r) * a.E + t.e];
      const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kAccCols);
      const int p = (t.r - a.r0) & 1;
      if (t.gu) {
        uint16_t* orow = a.h[p] + (static_cast<size_t>(t.e) * a.C + row) * a.F + t.nt * GW;
        store_swiglu(tb, GW, orow, valid);
      } else {
        uint16_t* orow = a.out[p] + (static_cast<size_t>(t.e) * a.C + row) * a.d + t.nt * kBN;
        store_bf16(tb, kBN, orow, valid);
      }
      tc_fence_before();
      mbar_arrive(smem_addr(&s.tempty[acc]));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
      // this warp's quarter of the tile is in memory
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        const int blk = (t.e * cn.mb + t.m) * kSyncStride;
        red_release((t.gu ? cn.gu[p] : cn.dn[p]) + blk, 1);
        if (!t.gu) red_release(a.sync + kSyncDnTotal + p * kSyncSetStride, 1);
      }
    }
    __syncwarp();
  } else if (warp < kFirstCombWarp) {
    dispatch_role(a, cn);
    __syncwarp();
  } else {
    combine_role(a, cn);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
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

cudaError_t launch_round_pipeline(const PipelineArgs& a, cudaStream_t stream) {
  if (a.r0 >= a.R) return cudaSuccess;
  for (int p = 0; p < 2; ++p)
    if (a.buf[p] == nullptr || a.h[p] == nullptr || a.out[p] == nullptr) return cudaErrorInvalidValue;
  CUtensorMap m_agu[2], m_bgu, m_adn[2], m_bdn;
  cudaError_t e = cudaSuccess;
  for (int p = 0; p < 2 && e == cudaSuccess; ++p) {
    e = gemm::make_map(&m_agu[p], a.buf[p], a.d, a.C, a.E, BM);
    if (e == cudaSuccess) e = gemm::make_map(&m_adn[p], a.h[p], a.F, a.C, a.E, BM);
  }
  const int gw = a.gw;
  if (gw != pipe_gate_width(a.d) || a.F % gw != 0 || a.d % (2 * gw) != 0) return cudaErrorInvalidValue;
  if (e == cudaSuccess) e = gemm::make_map(&m_bgu, a.w_gate_up, a.d, 2ull * a.F, a.E, gw);
  if (e == cudaSuccess) e = gemm::make_map(&m_bdn, a.w_down, a.F, a.d, a.E, 2 * gw);
  if (e != cudaSuccess) return e;
  static std::atomic<uint64_t> configured{0};   // one bit per device ordinal
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(configured.load() & bit)) {
    e = cudaFuncSetAttribute(round_pipeline_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(round_pipeline_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
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
  if (gw == 64)
    e = cudaLaunchKernelEx(&cfg, round_pipeline_kernel<64>, m_agu[0], m_agu[1], m_bgu, m_adn[0], m_adn[1], m_bdn, a);
  else
    e = cudaLaunchKernelEx(&cfg, round_pipeline_kernel<32>, m_agu[0], m_agu[1], m_bgu, m_adn[0], m_adn[1], m_bdn, a);
  launch_end(kKindPipeline, stream);
  return e;
}

}  // namespace moe
