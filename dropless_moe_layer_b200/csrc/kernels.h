// kernels.h - internal launchers shared by the library's translation units.
// Not part of the public C ABI (that is include/moe.h).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#ifndef MOE_PDL
#define MOE_PDL 1   // 0: plain stream-ordered launches (the kernels' dependency waits are no-ops)
#endif

namespace moe {

// Launch `kernel` with programmatic stream serialization: it may begin (and run its
// prologue) while the previous kernel in the stream drains. Every kernel of this library
// calls grid_dependency_wait() before it touches memory that an earlier kernel writes or
// reads, so stream order is preserved for data; only launch latency is hidden.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = MOE_PDL;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Workspace status word bits (header[kHdrStatus]).
enum : int {
  kStatusTimeoutProducer = 1,
  kStatusTimeoutMma = 2,
  kStatusTimeoutEpilogue = 4,
  kStatusTimeoutPipeline = 8,   // a dependency wait of the pipelined-rounds kernel gave up
  kStatusBounds = 16,           // a debug bounds check failed (MOE_FLAG_DEBUG_BOUNDS)
  kStatusCanary = 32,           // a workspace guard word was overwritten (MOE_FLAG_DEBUG_BOUNDS)
};

// Header words inside the workspace.
enum : int {
  kHdrR = 0,
  kHdrMaxLoad = 1,
  kHdrStatus = 2,
  kHdrScanDone = 3,   // planner: expert scans finished (the last one finalizes the plan)
  kHdrBadKind = 4,    // first failed debug check: what failed (BadKind), 0 = none
  kHdrBadValue = 5,   // ... and the offending index or guard number
  kHdrLoad = 64,      // copy of load[0..E-1], so one small copy brings the plan summary home
  kHdrWords = 64 + 256,
};

// What a failed debug check was checking (header word kHdrBadKind).
enum BadKind : int {
  kBadPlanPair = 1,      // planner: a pair's expert, round or row position out of range
  kBadDispatchRow = 2,   // dispatch: a row's source token or destination row out of range
  kBadCombinePair = 3,   // combine: a pair's expert or buffer row out of range
  kBadCombineToken = 4,  // combine: a row's token out of range
  kBadGemmRows = 5,      // GEMM: an expert's row count above the buffer's rows
  kBadCanary = 6,        // a guard after a workspace region was overwritten (value: guard number)
};

// With MOE_FLAG_DEBUG_BOUNDS the kernels get the workspace header (else null) and check every
// plan index before they use it; a failed check lands here and the access is skipped. Never traps.
__device__ __forceinline__ void record_bad(int32_t* hdr, int kind, int value) {
  atomicOr(hdr + kHdrStatus, kind == kBadCanary ? kStatusCanary : kStatusBounds);
  if (atomicCAS(hdr + kHdrBadKind, 0, kind) == 0) atomicExch(hdr + kHdrBadValue, value);
}

constexpr int kPlanTokensPerBlock = 256;
#define MOE_MAX_E_PLAN 256

// Pipelined-rounds kernel (round_pipeline.cu): fixed tile widths and the layout of its
// dependency counters inside the workspace ("sync" region, int32, all zero between launches).
// Round r of a launch starting at round r0 uses buffer set p = (r - r0) & 1.
constexpr int kPipeRowBlock = 128;   // rows of a tile (one 128-row block of an expert's C rows)
// Gate columns per gate/up tile (MMA N = twice that); a down tile has twice as many output
// columns, so both GEMMs share one stage geometry. 64 when d is a multiple of 128, else 32.
__host__ __device__ inline int pipe_gate_width(int d) { return d % 128 == 0 ? 64 : 32; }
// Every counter has its own 32-byte sector (a stride of 8 words) and the round-level counters
// their own 256-byte slots, so that polls and atomic adds on different counters do not queue
// behind each other in one L2 line.
constexpr int kSyncStride = 8;       // words between per-block counters
enum : int {
  kSyncAbort = 128,        // raised by any CTA that gave up a wait
  kSyncExit = 160,         // CTAs that finished (the last one zeroes the region)
  kSyncDnTotal = 192,      // [2] (stride 64) down tile quarters finished, per buffer set
  kSyncNextTask = 384,     // next GEMM tile of the list to claim
  kSyncBlocks = 448,       // then disp, gu, dn, rd: [2][E * MB] each, MB = ceil(C / 128)
};
constexpr int kSyncSetStride = 64;
__host__ __device__ inline long long pipe_row_blocks(int C) { return (C + kPipeRowBlock - 1) / kPipeRowBlock; }
__host__ __device__ inline long long pipe_sync_words(int E, int C) {
  return kSyncBlocks + 8ll * E * pipe_row_blocks(C) * kSyncStride;
}

// Kernel kinds for profiling (same numbering as the public header).
enum KernelKind : int {
  kKindRouterGemm = 0,
  kKindTopk = 1,
  kKindPlan = 2,
  kKindDispatch = 3,
  kKindGateUp = 4,
  kKindDown = 5,
  kKindCombine = 6,
  kKindPipeline = 7,
};

// Called around every launch (profiling and launch accounting).
void launch_begin(int kind, cudaStream_t stream);
void launch_end(int kind, cudaStream_t stream, int kernels = 1);

int num_sms();

// ---- router / top-k (router.cu)
// block_counts: [ceil(T / 256), E] pair counts per block of 256 tokens and expert, added with
// atomics (the caller zeroes it first); the planner's first input.
cudaError_t launch_router_topk(const float* logits, int T, int E, int k, int renorm, int32_t* idx,
                               float* gate, int32_t* block_counts, cudaStream_t stream);

// ---- planner (plan.cu)
struct PlanBuffers {
  const int32_t* idx;     // [T, k]
  int32_t* header;        // [kHdrWords]
  int32_t* load;          // [E]
  int32_t* offsets;       // [E + 1]
  int32_t* block_base;    // [blocks, E]: per-block pair counts from the top-k kernel
  int32_t* n;             // [max_rounds, E]
  int32_t* row_off;       // [max_rounds, E]
  int32_t* row_start;     // [max_rounds + 1]
  int32_t* round;         // [T, k]
  int32_t* slot;          // [T, k]
  int32_t* row_token;     // [T * k]
  int32_t* row_dst;       // [T * k]
  int32_t* mb_prefix;     // [max_rounds, E + 1] 128-row blocks of experts < e in round r, or null
  int32_t* sync;          // pipelined-rounds counters to zero ([sync_words]), or null
  long long sync_words;
  int borrow;             // 1: capacity borrowing (rows packed per round, n[r][e] may exceed C)
  int32_t* dbg;           // the header when MOE_FLAG_DEBUG_BOUNDS is set, else null
};
cudaError_t launch_plan(const PlanBuffers& b, int T, int k, int E, int C, int max_rounds,
                        cudaStream_t stream);
// One block copies n words from device memory to dst, host memory mapped into the device's
// address space (a kernel's stores, not a copy engine).
cudaError_t launch_copy_words(const int32_t* src, int32_t* dst, int n, cudaStream_t stream);

// ---- dispatch / combine (dispatch_combine.cu)
// dbg: the workspace header when MOE_FLAG_DEBUG_BOUNDS is set (row checks against T tokens and
// buf_rows buffer rows), else null.
cudaError_t launch_dispatch(const uint16_t* x, uint16_t* buf, const int32_t* row_start,
                            const int32_t* row_token, const int32_t* row_dst, int r, int rows,
                            int d, cudaStream_t stream, int32_t* dbg = nullptr, int T = 0,
                            long long buf_rows = 0);
// rows: rows of round r (host copy); the kernel walks the round's rows instead of all T
// tokens when there are fewer of them.
// row_off: pooled round rows (capacity borrowing: pair (e, slot) of round r at buffer row
// row_off[r][e] - row_start[r] + slot), or null for the per-expert [E, C, d] buffer.
cudaError_t launch_combine(const uint16_t* buf, float* y, const int32_t* idx, const float* gate,
                           const int32_t* round, const int32_t* slot, const int32_t* row_start,
                           const int32_t* row_token, const int32_t* row_dst, int T, int k, int C, int d,
                           int r, int rows, const int32_t* row_off, int E, cudaStream_t stream,
                           int32_t* dbg = nullptr);

// Guard words after the workspace regions (MOE_FLAG_DEBUG_BOUNDS): fill writes the pattern into
// every guard; check compares it and records the first guard found changed.
constexpr int kMaxGuards = 32;
constexpr int kGuardBytes = 256;
struct GuardList {
  int n;
  unsigned long long off[kMaxGuards];   // byte offsets of the guards inside the workspace
};
cudaError_t launch_guards(uint8_t* ws, const GuardList& g, int check, int32_t* hdr, cudaStream_t stream);

// ---- grouped GEMMs (grouped_gemm.cu)
// gate_up: h[e][s] = bf16(silu(buf[e][s] W1_e^T) * (buf[e][s] W3_e^T)), s < n_dev[e]
// A copy step of a neighbouring round carried by a GEMM launch on extra warps: a dispatch
// (x -> buf rows of round r) or a combine (gate * out -> y for round r).
struct RoundCopy {
  bool combine;
  int r;
  int rows;                  // rows of round r (host copy)
  const int32_t* row_start;
  const int32_t* row_token;
  const int32_t* row_dst;
  const uint16_t* x;         // dispatch
  uint16_t* buf;
  const uint16_t* out;       // combine
  float* y;
  const int32_t* idx;
  const float* gate;
  const int32_t* round;
  const int32_t* slot;
  int T, k, C, d;
  const int32_t* row_off;    // pooled round rows (capacity borrowing), or null
  int E;
  int32_t* dbg;              // the header when MOE_FLAG_DEBUG_BOUNDS is set, else null
};

// rows_cap > 0 (debug bounds checks): an expert's device row count above it is recorded in the
// header and clamped.
// n_dev: rows per expert this round on the device (read by the kernel); n_host: the same on
// the host (picks the tile width and the grid). copy: optional side copy step, or null.
// group_row / group_row_base: pooled round rows (capacity borrowing: expert e's rows start at
// buffer row group_row[e] - *group_row_base), or null for the per-expert [E, C, .] buffers.
cudaError_t launch_gate_up(const uint16_t* buf, const uint16_t* w_gate_up, uint16_t* h,
                           const int32_t* n_dev, const int32_t* n_host, int E, int C, int d, int F,
                           int32_t* status, const RoundCopy* copy, const int32_t* group_row,
                           const int32_t* group_row_base, cudaStream_t stream, int rows_cap = 0);
// down: out[e][s] = bf16(h[e][s] W2_e^T), s < n_dev[e]
cudaError_t launch_down(const uint16_t* h, const uint16_t* w_down, uint16_t* out, const int32_t* n_dev,
                        const int32_t* n_host, int E, int C, int d, int F, int32_t* status,
                        const RoundCopy* copy, const int32_t* group_row, const int32_t* group_row_base,
                        cudaStream_t stream, int rows_cap = 0);

// ---- pipelined rounds (round_pipeline.cu)
// Rounds [r0, R) of the layer in one persistent launch (one CTA per SM): dispatch, gate/up
// GEMM, down GEMM and combine of consecutive rounds overlap, ordered by dependency counters
// instead of kernel boundaries. Expects rounds < r0 fully done (y holds their sums).
struct PipelineArgs {
  const uint16_t* x;
  const uint16_t* w_gate_up;
  const uint16_t* w_down;
  uint16_t* buf[2];          // two buffer sets: round r uses set (r - r0) & 1
  uint16_t* h[2];
  uint16_t* out[2];
  float* y;
  const int32_t* idx;
  const float* gate;
  const int32_t* round;
  const int32_t* slot;
  const int32_t* n;          // [max_rounds, E]
  const int32_t* row_start;  // [max_rounds + 1]
  const int32_t* row_token;
  const int32_t* row_dst;
  const int32_t* mb_prefix;  // [max_rounds, E + 1]
  int32_t* sync;
  int32_t* status;
  int T, k, E, C, d, F, r0, R;
  int r0_dispatched;         // 1: round r0's rows are already in buf (set 0) when the launch starts
  int gw;                    // gate columns per gate/up tile (pipe_gate_width(d)); down tiles 2 gw
};
cudaError_t launch_round_pipeline(const PipelineArgs& a, cudaStream_t stream);

// Expert parallelism, owner side of round r: both grouped GEMMs over the rows received from every
// source rank, one group per (source rank, local expert) in that order, packed from row 0 of
// recv (group g at row group_row[g], rows[g] rows), weights of local expert group_expert[g] of
// w_gate_up [E_local, 2 d_ff, d] and w_down [E_local, d, d_ff]; h and out hold the same rows.
// recv, h and out have buf_rows rows each.
cudaError_t launch_ep_experts(const uint16_t* recv, const uint16_t* w_gate_up, const uint16_t* w_down, uint16_t* h,
                              uint16_t* out, int groups, const int32_t* rows_dev, const int32_t* rows_host,
                              const int32_t* group_row_dev, const int32_t* group_expert_dev, long long buf_rows,
                              int E_local, int d, int F, int32_t* status, cudaStream_t stream);

// router GEMM: logits[t][e] = x[t] . w_router[e] + bias[e] (fp32 out)
cudaError_t launch_router_gemm(const uint16_t* x, const uint16_t* w_router, const float* bias,
                               float* logits, int T, int d, int E, int32_t* status,
                               cudaStream_t stream);

}  // namespace moe
