// moe_api.cu - the C ABI (include/moe.h): argument checks, the fixed workspace layout,
// the router -> planner sequence and the round loop.
//
// The memory of the layer is fixed by the shape alone ("Frontier Pre-training at
// Microsoft AI (MAI-Base-2)", Key claims, multi-round dropless MoE item: memory usage
// is static whatever the token imbalance). moe_workspace_bytes() depends on
// (T, d, E, k, d_ff, C) only; the routing decides how many rounds run, never how much
// memory they use.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "backward.h"
#include "kernels.h"
#include "moe.h"

namespace moe {

// ---------------------------------------------------------------- accounting / profiling

namespace {

std::atomic<uint64_t> g_launches{0};

constexpr int kProfMax = 4096;
struct Profiler {
  bool on = false;
  bool created = false;
  int n = 0;
  int kind[kProfMax];
  cudaEvent_t ev[2 * kProfMax];
};
Profiler g_prof;

std::mutex g_sm_mutex;
int g_sm_count[64] = {0};

}  // namespace

void launch_begin(int kind, cudaStream_t stream) {
  (void)kind;
  if (g_prof.on && g_prof.n < kProfMax) cudaEventRecord(g_prof.ev[2 * g_prof.n], stream);
}

void launch_end(int kind, cudaStream_t stream, int kernels) {
  g_launches.fetch_add(static_cast<uint64_t>(kernels));
  if (g_prof.on && g_prof.n < kProfMax) {
    cudaEventRecord(g_prof.ev[2 * g_prof.n + 1], stream);
    g_prof.kind[g_prof.n] = kind;
    ++g_prof.n;
  }
}

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  dev &= 63;
  std::lock_guard<std::mutex> lock(g_sm_mutex);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    g_sm_count[dev] = n > 0 ? n : 1;
  }
  return g_sm_count[dev];
}

}  // namespace moe

using namespace moe;

namespace {

// Host words mapped into the device's address space, for reading the plan summary without a
// copy engine (moe_plan). One buffer per host thread and device: moe_plan returns only after
// reading it, so a thread never has two reads of its buffer in flight. Allocated on first use
// (kHdrWords words of pinned host memory) and kept for the thread's lifetime; null if the
// allocation fails (moe_plan then copies with cudaMemcpyAsync).
struct MappedWords {
  volatile int32_t* host = nullptr;
  int32_t* dev = nullptr;
};

#ifndef MOE_PLAN_MAPPED
#define MOE_PLAN_MAPPED 1   // 0: moe_plan reads its summary back with cudaMemcpyAsync
#endif

const MappedWords* mapped_words() {
  if (!MOE_PLAN_MAPPED) return nullptr;
  thread_local MappedWords per_device[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  MappedWords& m = per_device[dev & 63];
  if (m.host == nullptr) {
    void* h = nullptr;
    void* d = nullptr;
    if (cudaHostAlloc(&h, kHdrWords * sizeof(int32_t), cudaHostAllocMapped) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    if (cudaHostGetDevicePointer(&d, h, 0) != cudaSuccess) {
      cudaGetLastError();
      cudaFreeHost(h);
      return nullptr;
    }
    m.host = static_cast<volatile int32_t*>(h);
    m.dev = static_cast<int32_t*>(d);
  }
  return &m;
}

int check_shape(const moe_shape_t* s) {
  if (s == nullptr) return MOE_ERR_INVALID_ARG;
  if (s->flags & ~static_cast<uint32_t>(MOE_FLAG_RENORM_TOPK | MOE_FLAG_PER_ROUND | MOE_FLAG_PIPELINE_ALL |
                                        MOE_FLAG_BORROW | MOE_FLAG_DEBUG_BOUNDS))
    return MOE_ERR_INVALID_ARG;
  if ((s->flags & MOE_FLAG_DEBUG_BOUNDS) && (s->flags & MOE_FLAG_PIPELINE_ALL)) return MOE_ERR_INVALID_ARG;
  if ((s->flags & MOE_FLAG_PER_ROUND) && (s->flags & MOE_FLAG_PIPELINE_ALL)) return MOE_ERR_INVALID_ARG;
  if ((s->flags & MOE_FLAG_BORROW) && (s->flags & MOE_FLAG_PIPELINE_ALL)) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->E < 1 || s->E > MOE_MAX_EXPERTS || s->k < 1 || s->k > MOE_MAX_TOPK ||
      s->k > s->E || s->C < 1)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (s->d < 64 || s->d > 16384 || s->d % 64 != 0 || s->d_ff < 64 || s->d_ff > 16384 ||
      s->d_ff % 64 != 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(s->T) * s->k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(s->E) * s->C >= (1ll << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
  const long long wide = s->d > s->d_ff ? s->d : s->d_ff;
  if (static_cast<long long>(s->C) * wide * 2 >= (1ll << 40)) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

int max_rounds_of(const moe_shape_t* s) { return s->T == 0 ? 0 : (s->T + s->C - 1) / s->C; }

bool debug_bounds(const moe_shape_t* s) { return (s->flags & MOE_FLAG_DEBUG_BOUNDS) != 0; }

// With MOE_FLAG_DEBUG_BOUNDS every region is followed by a guard of kGuardBytes (listed in
// *guards when given), which moe_plan fills and moe_device_status checks.
void make_layout(const moe_shape_t* s, moe_workspace_layout_t* L, GuardList* guards = nullptr) {
  std::memset(L, 0, sizeof(*L));
  size_t off = 0;
  const bool dbg = debug_bounds(s);
  if (guards) guards->n = 0;
  auto take = [&](long long bytes) {
    const size_t o = off;
    off += (static_cast<size_t>(bytes) + 255) & ~static_cast<size_t>(255);
    if (dbg) {
      if (guards && guards->n < kMaxGuards) guards->off[guards->n++] = off;
      off += kGuardBytes;
    }
    return o;
  };
  const long long T = s->T, E = s->E, k = s->k, C = s->C;
  const int mr = max_rounds_of(s);
  const int blocks = static_cast<int>((T + kPlanTokensPerBlock - 1) / kPlanTokensPerBlock);
  L->header = take(kHdrWords * 4ll);
  L->block_base = take(static_cast<long long>(blocks) * E * 4);   // right after the header: one memset
  L->logits = take(T * E * 4);
  L->topk_idx = take(T * k * 4);
  L->gate = take(T * k * 4);
  L->round = take(T * k * 4);
  L->slot = take(T * k * 4);
  L->load = take(E * 4);
  L->offsets = take((E + 1) * 4);
  L->n = take(static_cast<long long>(mr) * E * 4);
  L->row_off = take(static_cast<long long>(mr) * E * 4);
  L->row_start = take((mr + 1ll) * 4);
  L->row_token = take(T * k * 4);
  L->row_dst = take(T * k * 4);
  L->buf = take(E * C * s->d * 2);
  L->h = take(E * C * s->d_ff * 2);
  L->out = take(E * C * s->d * 2);
  L->mb_prefix = take(static_cast<long long>(mr) * (E + 1) * 4);
  L->sync = take(pipe_sync_words(s->E, s->C) * 4);
  if (!(s->flags & (MOE_FLAG_PER_ROUND | MOE_FLAG_BORROW | MOE_FLAG_DEBUG_BOUNDS))) {   // pipelined launch's 2nd set
    L->buf2 = take(E * C * s->d * 2);
    L->h2 = take(E * C * s->d_ff * 2);
    L->out2 = take(E * C * s->d * 2);
  }
  L->total_bytes = off;
  L->max_rounds = mr;
  L->plan_blocks = blocks;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  static std::atomic<uint64_t> ok_mask{0}, bad_mask{0};
  const uint64_t bit = 1ull << (dev & 63);
  if (ok_mask.load() & bit) return MOE_OK;
  if (bad_mask.load() & bit) return MOE_ERR_NO_DEVICE;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10) {
    bad_mask.fetch_or(bit);
    return MOE_ERR_NO_DEVICE;
  }
  ok_mask.fetch_or(bit);
  return MOE_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

bool borrowing(const moe_shape_t* s);

// Common argument checks of the calls that run a plan (no CUDA call).
int check_plan_args(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws, size_t ws_bytes,
                    moe_workspace_layout_t* L) {
  int st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (info == nullptr || ws == nullptr) return MOE_ERR_INVALID_ARG;
  make_layout(shape, L);
  if (ws_bytes < L->total_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned(ws, 256)) return MOE_ERR_MISALIGNED;
  if (info->R < 0 || info->R > L->max_rounds) return MOE_ERR_INVALID_ARG;
  // the plan was made for this kind of plan (with or without borrowing)
  if ((info->plan_flags ^ shape->flags) & MOE_FLAG_BORROW) return MOE_ERR_INVALID_ARG;
  if (debug_bounds(shape)) {
    // debug bounds checks, on the host before any launch: the plan summary must be one that the
    // planner can have produced for this shape
    long long sum = 0;
    int max_load = 0;
    for (int e = 0; e < shape->E; ++e) {
      if (info->load[e] < 0 || info->load[e] > shape->T) return MOE_ERR_INVALID_ARG;
      sum += info->load[e];
      max_load = info->load[e] > max_load ? info->load[e] : max_load;
    }
    if (sum != static_cast<long long>(shape->T) * shape->k || max_load != info->max_load) return MOE_ERR_INVALID_ARG;
    const int r_own = (max_load + shape->C - 1) / shape->C;   // rounds without borrowing
    if (!borrowing(shape) ? info->R != r_own : (info->R > r_own || (shape->T > 0 && info->R < 1)))
      return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

// The same, then the device check.
int check_run(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws, size_t ws_bytes,
              moe_workspace_layout_t* L) {
  const int st = check_plan_args(shape, info, ws, ws_bytes, L);
  return st != MOE_OK ? st : check_device();
}

bool borrowing(const moe_shape_t* s) { return (s->flags & MOE_FLAG_BORROW) != 0; }

// Rows of each expert in round r, on the host, from the loads: the same integer rule as the
// planner's (min(C, what is left) without borrowing; with borrowing, the planner's
// round-by-round lending of the E*C pool, replayed up to round r).
void round_rows(const moe_shape_t* s, const moe_plan_info_t* info, int r, int32_t* n_host, int* rows) {
  long long total = 0;
  if (!borrowing(s)) {
    const long long base = static_cast<long long>(r) * s->C;
    for (int e = 0; e < s->E; ++e) {
      const long long rem = info->load[e] - base;
      n_host[e] = rem <= 0 ? 0 : rem >= s->C ? s->C : static_cast<int32_t>(rem);
      total += n_host[e];
    }
    *rows = static_cast<int>(total);
    return;
  }
  long long pending[MOE_MAX_EXPERTS];
  for (int e = 0; e < s->E; ++e) pending[e] = info->load[e];
  const long long pool = static_cast<long long>(s->E) * s->C;
  for (int rr = 0; rr <= r; ++rr) {
    long long own_sum = 0;
    for (int e = 0; e < s->E; ++e) own_sum += pending[e] < s->C ? pending[e] : s->C;
    long long spare = pool - own_sum;
    total = 0;
    for (int e = 0; e < s->E; ++e) {
      const long long own = pending[e] < s->C ? pending[e] : s->C;
      const long long want = pending[e] - own;
      const long long extra = want < spare ? want : spare;
      spare -= extra;
      n_host[e] = static_cast<int32_t>(own + extra);
      pending[e] -= own + extra;
      total += n_host[e];
    }
  }
  *rows = static_cast<int>(total);
}

// The workspace header for the kernels' debug bounds checks, or null when they are off.
int32_t* debug_ptr(const moe_shape_t* s, void* ws, const moe_workspace_layout_t& L) {
  return debug_bounds(s) ? at<int32_t>(ws, L.header) : nullptr;
}

// Most rows one expert may hold in a round (checked by the GEMMs under debug bounds checks).
int rows_cap(const moe_shape_t* s) {
  if (!debug_bounds(s)) return 0;
  const long long cap = borrowing(s) ? static_cast<long long>(s->E) * s->C : s->C;
  return static_cast<int>(cap);
}

int do_dispatch(const moe_shape_t* s, const moe_plan_info_t* info, void* ws,
                const moe_workspace_layout_t& L, int r, const uint16_t* x, cudaStream_t stream) {
  int32_t n_host[MOE_MAX_EXPERTS];
  int rows = 0;
  round_rows(s, info, r, n_host, &rows);
  return cuda_status(launch_dispatch(x, at<uint16_t>(ws, L.buf), at<int32_t>(ws, L.row_start),
                                     at<int32_t>(ws, L.row_token), at<int32_t>(ws, L.row_dst), r, rows,
                                     s->d, stream, debug_ptr(s, ws, L), s->T,
                                     static_cast<long long>(s->E) * s->C));
}

// Copy steps up to this many bytes of rows ride on a GEMM launch (its 4 copy warps per SM);
// larger ones ride there only when the copy's estimated time, at about kSideCopyGBs, stays below
// the GEMM's at about kGemmTflops; otherwise they get their own kernel at full HBM bandwidth.
constexpr size_t kFuseCopyBytes = 32ull << 20;
#ifndef MOE_SIDE_COPY_GBS
#define MOE_SIDE_COPY_GBS 2000.0
#endif
constexpr double kSideCopyGBs = MOE_SIDE_COPY_GBS;
constexpr double kGemmTflops = 1100.0;

// The copy step of round `cr` carried by a GEMM launch (a combine, or a dispatch of x).
RoundCopy make_copy(const moe_shape_t* s, const moe_plan_info_t* info, void* ws, const moe_workspace_layout_t& L,
                    bool combine, int cr, const uint16_t* x, float* y) {
  int32_t n_host[MOE_MAX_EXPERTS];
  RoundCopy c{};
  c.combine = combine;
  c.r = cr;
  round_rows(s, info, cr, n_host, &c.rows);
  c.row_start = at<int32_t>(ws, L.row_start);
  c.row_token = at<int32_t>(ws, L.row_token);
  c.row_dst = at<int32_t>(ws, L.row_dst);
  c.x = x;
  c.buf = at<uint16_t>(ws, L.buf);
  c.out = at<uint16_t>(ws, L.out);
  c.y = y;
  c.idx = at<int32_t>(ws, L.topk_idx);
  c.gate = at<float>(ws, L.gate);
  c.round = at<int32_t>(ws, L.round);
  c.slot = at<int32_t>(ws, L.slot);
  c.T = s->T;
  c.k = s->k;
  c.C = s->C;
  c.d = s->d;
  c.row_off = borrowing(s) ? at<int32_t>(ws, L.row_off) : nullptr;
  c.E = s->E;
  c.dbg = debug_ptr(s, ws, L);
  return c;
}

int do_gate_up(const moe_shape_t* s, const moe_plan_info_t* info, void* ws,
               const moe_workspace_layout_t& L, int r, const uint16_t* w13, const RoundCopy* copy,
               cudaStream_t stream) {
  int32_t n_host[MOE_MAX_EXPERTS];
  int rows = 0;
  round_rows(s, info, r, n_host, &rows);
  const bool pooled = borrowing(s);
  return cuda_status(launch_gate_up(at<uint16_t>(ws, L.buf), w13, at<uint16_t>(ws, L.h),
                                    at<int32_t>(ws, L.n) + static_cast<size_t>(r) * s->E, n_host, s->E,
                                    s->C, s->d, s->d_ff, at<int32_t>(ws, L.header) + kHdrStatus, copy,
                                    pooled ? at<int32_t>(ws, L.row_off) + static_cast<size_t>(r) * s->E : nullptr,
                                    pooled ? at<int32_t>(ws, L.row_start) + r : nullptr, stream, rows_cap(s)));
}

int do_down(const moe_shape_t* s, const moe_plan_info_t* info, void* ws,
            const moe_workspace_layout_t& L, int r, const uint16_t* w2, const RoundCopy* copy,
            cudaStream_t stream) {
  int32_t n_host[MOE_MAX_EXPERTS];
  int rows = 0;
  round_rows(s, info, r, n_host, &rows);
  const bool pooled = borrowing(s);
  return cuda_status(launch_down(at<uint16_t>(ws, L.h), w2, at<uint16_t>(ws, L.out),
                                 at<int32_t>(ws, L.n) + static_cast<size_t>(r) * s->E, n_host, s->E,
                                 s->C, s->d, s->d_ff, at<int32_t>(ws, L.header) + kHdrStatus, copy,
                                 pooled ? at<int32_t>(ws, L.row_off) + static_cast<size_t>(r) * s->E : nullptr,
                                 pooled ? at<int32_t>(ws, L.row_start) + r : nullptr, stream, rows_cap(s)));
}

int do_combine(const moe_shape_t* s, const moe_plan_info_t* info, void* ws, const moe_workspace_layout_t& L,
               int r, float* y, cudaStream_t stream) {
  int32_t n_host[MOE_MAX_EXPERTS];
  int rows = 0;
  round_rows(s, info, r, n_host, &rows);
  return cuda_status(launch_combine(at<uint16_t>(ws, L.out), y, at<int32_t>(ws, L.topk_idx),
                                    at<float>(ws, L.gate), at<int32_t>(ws, L.round),
                                    at<int32_t>(ws, L.slot), at<int32_t>(ws, L.row_start),
                                    at<int32_t>(ws, L.row_token), at<int32_t>(ws, L.row_dst), s->T, s->k,
                                    s->C, s->d, r, rows, borrowing(s) ? at<int32_t>(ws, L.row_off) : nullptr,
                                    s->E, stream, debug_ptr(s, ws, L)));
}

void make_backward_layout(const moe_shape_t* s, moe_backward_layout_t* L) {
  std::memset(L, 0, sizeof(*L));
  size_t off = 0;
  auto take = [&](long long bytes) {
    const size_t o = off;
    off += (static_cast<size_t>(bytes) + 255) & ~static_cast<size_t>(255);
    return o;
  };
  const long long T = s->T, E = s->E, k = s->k, d = s->d, F = s->d_ff;
  const long long rows = backward_rows(s->E, s->C, (s->flags & MOE_FLAG_BORROW) != 0);
  const long long mr = max_rounds_of(s);
  L->xbuf = take(rows * d * 2);
  L->dybuf = take(rows * d * 2);
  L->row_gate = take(rows * 4);
  L->ab = take(rows * 2 * F * 2);
  L->hg = take(rows * F * 2);
  L->dab = take(rows * 2 * F * 2);
  L->dgate_part = take(rows * (F / 64) * 4);
  L->dxbuf = take(rows * d * 2);
  L->dgate = take(T * k * 4);
  L->ones = take(T * k * 4);
  L->seg_off = take(mr * E * 4);
  L->zeros = take((mr + 1) * 4);
  // the second buffer set (none with MOE_FLAG_PER_ROUND, which runs the rounds one at a time)
  const long long rows2 = (s->flags & MOE_FLAG_PER_ROUND) ? 0 : backward_rows2(s->E, s->C);
  L->xbuf2 = take(rows2 * d * 2);
  L->dybuf2 = take(rows2 * d * 2);
  L->row_gate2 = take(rows2 * 4);
  L->ab2 = take(rows2 * 2 * F * 2);
  L->hg2 = take(rows2 * F * 2);
  L->dab2 = take(rows2 * 2 * F * 2);
  L->dgate_part2 = take(rows2 * (F / 64) * 4);
  L->dxbuf2 = take(rows2 * d * 2);
  if (rows2 == 0) L->xbuf2 = L->dybuf2 = L->row_gate2 = L->ab2 = L->hg2 = L->dab2 = L->dgate_part2 = L->dxbuf2 = 0;
  L->total_bytes = off;
  L->rows = static_cast<int32_t>(rows);
  L->rows2 = static_cast<int32_t>(rows2);
}

// The per-round buffers' rows (and the element offsets within them) must fit int32.
// The backward's second stream (the highest priority: it carries the rounds' serial back
// halves) and its events, per host thread and device, created on first use.
struct SideStream {
  cudaStream_t stream;
  cudaEvent_t front, back[2];
};

cudaError_t side_stream(SideStream* out) {
  thread_local SideStream cache[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  SideStream& c = cache[dev & 63];
  if (c.stream == nullptr) {
    SideStream n{};
    int least = 0, greatest = 0;
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess ||
        (e = cudaStreamCreateWithPriority(&n.stream, cudaStreamNonBlocking, greatest)) != cudaSuccess)
      return e;
    if ((e = cudaEventCreateWithFlags(&n.front, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&n.back[0], cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&n.back[1], cudaEventDisableTiming)) != cudaSuccess) {
      cudaStreamDestroy(n.stream);
      return e;
    }
    c = n;
  }
  *out = c;
  return cudaSuccess;
}

bool backward_shape_ok(const moe_shape_t* s) {
  const long long rows = backward_rows(s->E, s->C, (s->flags & MOE_FLAG_BORROW) != 0);
  return rows * 2 * s->d_ff < (1ll << 31) && rows * s->d < (1ll << 31);
}

}  // namespace

extern "C" {

size_t moe_backward_workspace_bytes(const moe_shape_t* shape) {
  if (check_shape(shape) != MOE_OK || !backward_shape_ok(shape)) return 0;
  moe_backward_layout_t L;
  make_backward_layout(shape, &L);
  return L.total_bytes;
}

int moe_backward_workspace_layout(const moe_shape_t* shape, moe_backward_layout_t* layout) {
  const int st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (!backward_shape_ok(shape)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (layout == nullptr) return MOE_ERR_INVALID_ARG;
  make_backward_layout(shape, layout);
  return MOE_OK;
}

int moe_backward(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws, size_t ws_bytes,
                 void* bws, size_t bws_bytes, const uint16_t* x, const uint16_t* w_gate_up,
                 const uint16_t* w_down, const float* dy, float* dx, float* dw_gate_up, float* dw_down,
                 float* dz, moe_stream_t stream_) {
  moe_workspace_layout_t L;
  int st = check_plan_args(shape, info, ws, ws_bytes, &L);
  if (st != MOE_OK) return st;
  if (!backward_shape_ok(shape)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (bws == nullptr || w_gate_up == nullptr || w_down == nullptr || dw_gate_up == nullptr ||
      dw_down == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (shape->T > 0 && (x == nullptr || dy == nullptr || dx == nullptr || dz == nullptr))
    return MOE_ERR_INVALID_ARG;
  moe_backward_layout_t B;
  make_backward_layout(shape, &B);
  if (bws_bytes < B.total_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned(bws, 256) || !aligned(x, 16) || !aligned(w_gate_up, 16) || !aligned(w_down, 16) ||
      !aligned(dy, 16) || !aligned(dx, 16) || !aligned(dw_gate_up, 16) || !aligned(dw_down, 16) ||
      !aligned(dz, 16))
    return MOE_ERR_MISALIGNED;
  if ((st = check_device()) != MOE_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  BackwardArgs a{};
  a.x = x;
  a.w_gate_up = w_gate_up;
  a.w_down = w_down;
  a.dy = dy;
  a.logits = info->logits;
  a.idx = at<int32_t>(ws, L.topk_idx);
  a.gate = at<float>(ws, L.gate);
  a.round = at<int32_t>(ws, L.round);
  a.slot = at<int32_t>(ws, L.slot);
  a.n = at<int32_t>(ws, L.n);
  a.row_start = at<int32_t>(ws, L.row_start);
  a.row_off = at<int32_t>(ws, L.row_off);
  a.row_token = at<int32_t>(ws, L.row_token);
  a.row_dst = at<int32_t>(ws, L.row_dst);
  a.dx = dx;
  a.dw_gate_up = dw_gate_up;
  a.dw_down = dw_down;
  a.dz = dz;
  a.xbuf = at<uint16_t>(bws, B.xbuf);
  a.dybuf = at<uint16_t>(bws, B.dybuf);
  a.row_gate = at<float>(bws, B.row_gate);
  a.ab = at<uint16_t>(bws, B.ab);
  a.hg = at<uint16_t>(bws, B.hg);
  a.dab = at<uint16_t>(bws, B.dab);
  a.seg_off = at<int32_t>(bws, B.seg_off);
  a.zeros = at<int32_t>(bws, B.zeros);
  a.dgate_part = at<float>(bws, B.dgate_part);
  a.dxbuf = at<uint16_t>(bws, B.dxbuf);
  a.dgate = at<float>(bws, B.dgate);
  a.ones = at<float>(bws, B.ones);
  a.status = at<int32_t>(ws, L.header) + kHdrStatus;
  a.T = shape->T;
  a.k = shape->k;
  a.E = shape->E;
  a.C = shape->C;
  a.d = shape->d;
  a.F = shape->d_ff;
  a.renorm = (shape->flags & MOE_FLAG_RENORM_TOPK) ? 1 : 0;
  a.pooled = borrowing(shape) ? 1 : 0;
  a.rows = B.rows;
  // The second buffer set: a thin round (its front half's GEMMs have fewer tiles than the device
  // has SMs) whose pooled rows fit in it runs there when the round before ran in the first set,
  // so that its front half (dispatch, recompute, dh) on the caller's stream overlaps the round
  // before's back half (dx and weight gradients, combine) on a second stream. Large rounds are
  // not overlapped: two GEMM launches that each fill the device only slow each other down.
  // The back halves keep their round order on that stream (the fp32 weight gradients and dx are
  // accumulated round by round), so the results are those of running the rounds one at a time.
  BackwardArgs a2 = a;
  SideStream side{};
  bool overlap = B.rows2 > 0 && info->R > 1;
  if (overlap) {
    a2.xbuf = at<uint16_t>(bws, B.xbuf2);
    a2.dybuf = at<uint16_t>(bws, B.dybuf2);
    a2.row_gate = at<float>(bws, B.row_gate2);
    a2.ab = at<uint16_t>(bws, B.ab2);
    a2.hg = at<uint16_t>(bws, B.hg2);
    a2.dab = at<uint16_t>(bws, B.dab2);
    a2.dgate_part = at<float>(bws, B.dgate_part2);
    a2.dxbuf = at<uint16_t>(bws, B.dxbuf2);
    a2.pooled = 1;
    a2.rows = B.rows2;
    if ((st = cuda_status(side_stream(&side))) != MOE_OK) return st;
  }
  if ((st = cuda_status(launch_backward_prepare(a, info->load, info->R, stream))) != MOE_OK) return st;
  int32_t n_rounds[2][MOE_MAX_EXPERTS];
  int rows[2] = {0, 0};
  auto pooled_rows = [&](const int32_t* n) {
    long long p = 0;
    for (int e = 0; e < shape->E; ++e) p += (n[e] + 63) / 64 * 64;
    return p;
  };
  // set of round r + 1 given round r's: the second set only right after the first
  auto next_set = [&](int set, const int32_t* n_next) {
    return overlap && set == 0 && pooled_rows(n_next) <= B.rows2 && backward_front_is_thin(a2, n_next) ? 1 : 0;
  };
  if (info->R > 0) round_rows(shape, info, 0, n_rounds[0], &rows[0]);
  int set = 0;
  bool gathered = false;     // the round's dispatch ran in the previous round's combine launch
  bool back_used[2] = {false, false};
  cudaStream_t back_stream = overlap ? side.stream : stream;
  // the caller's stream waits for everything the second stream was given (also on an error
  // return, so that no work of this call is left unordered behind the caller's next launches)
  auto join = [&]() {
    if (!overlap) return cudaSuccess;
    const cudaError_t e = cudaEventRecord(side.front, back_stream);
    return e == cudaSuccess ? cudaStreamWaitEvent(stream, side.front, 0) : e;
  };
  auto fail = [&](int code) {
    join();
    return code;
  };
  for (int r = 0; r < info->R; ++r) {
    const int cur = r & 1, nxt = cur ^ 1;
    const bool more = r + 1 < info->R;
    if (more) round_rows(shape, info, r + 1, n_rounds[nxt], &rows[nxt]);
    const BackwardArgs& ar = set ? a2 : a;
    // front half on the caller's stream, after the last back half that read this set
    if (overlap && back_used[set] && (st = cuda_status(cudaStreamWaitEvent(stream, side.back[set], 0))) != MOE_OK)
      return fail(st);
    int parts = 0;
    if ((st = cuda_status(launch_backward_front(ar, r, n_rounds[cur], !gathered, &parts, stream))) != MOE_OK)
      return fail(st);
    // back half: the next round's dispatch joins its combine launch when the next round uses
    // the same set (its front half waits for this back half anyway)
    const int set_next = more ? next_set(set, n_rounds[nxt]) : 0;
    const bool merge = more && set_next == set;
    if (overlap) {
      if ((st = cuda_status(cudaEventRecord(side.front, stream))) != MOE_OK ||
          (st = cuda_status(cudaStreamWaitEvent(back_stream, side.front, 0))) != MOE_OK)
        return fail(st);
    }
    if ((st = cuda_status(launch_backward_back(ar, r, n_rounds[cur], parts, merge ? &ar : nullptr,
                                               merge ? n_rounds[nxt] : nullptr, back_stream))) != MOE_OK)
      return fail(st);
    if (overlap) {
      if ((st = cuda_status(cudaEventRecord(side.back[set], back_stream))) != MOE_OK) return fail(st);
      back_used[set] = true;
    }
    gathered = merge;
    set = set_next;
  }
  // dz after the last combine (the back halves ran in round order on the second stream)
  if ((st = cuda_status(join())) != MOE_OK) return st;
  return cuda_status(launch_backward_gates(a, stream));
}

size_t moe_workspace_bytes(const moe_shape_t* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  moe_workspace_layout_t L;
  make_layout(shape, &L);
  return L.total_bytes;
}

int moe_workspace_layout(const moe_shape_t* shape, moe_workspace_layout_t* layout) {
  const int st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (layout == nullptr) return MOE_ERR_INVALID_ARG;
  make_layout(shape, layout);
  return MOE_OK;
}

int moe_plan(const moe_shape_t* shape, const float* logits, const uint16_t* x,
             const uint16_t* w_router, const float* bias, void* ws, size_t ws_bytes,
             moe_plan_info_t* info, moe_stream_t stream_) {
  int st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (ws == nullptr || info == nullptr) return MOE_ERR_INVALID_ARG;
  if (logits == nullptr && shape->T > 0 && (x == nullptr || w_router == nullptr))
    return MOE_ERR_INVALID_ARG;
  moe_workspace_layout_t L;
  make_layout(shape, &L);
  if (ws_bytes < L.total_bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned(ws, 256) || !aligned(logits, 16) || !aligned(x, 16) || !aligned(w_router, 16) ||
      !aligned(bias, 4))
    return MOE_ERR_MISALIGNED;
  if ((st = check_device()) != MOE_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const moe_shape_t& s = *shape;
  int32_t* header = at<int32_t>(ws, L.header);
  // the header and the per-block pair counts start at zero (one memset: they are adjacent)
  if (cudaMemsetAsync(header, 0, L.block_base - L.header + static_cast<size_t>(L.plan_blocks) * s.E * 4, stream) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  if (debug_bounds(&s)) {   // the guards after every region (the memset above covers the first)
    GuardList guards;
    moe_workspace_layout_t L2;
    make_layout(&s, &L2, &guards);
    if ((st = cuda_status(launch_guards(static_cast<uint8_t*>(ws), guards, 0, header, stream))) != MOE_OK) return st;
  }

  const float* z = logits;
  if (z == nullptr && s.T > 0) {
    if ((st = cuda_status(launch_router_gemm(x, w_router, bias, at<float>(ws, L.logits), s.T, s.d,
                                             s.E, header + kHdrStatus, stream))) != MOE_OK)
      return st;
    z = at<float>(ws, L.logits);
  }
  if ((st = cuda_status(launch_router_topk(z, s.T, s.E, s.k, (s.flags & MOE_FLAG_RENORM_TOPK) ? 1 : 0,
                                           at<int32_t>(ws, L.topk_idx), at<float>(ws, L.gate),
                                           at<int32_t>(ws, L.block_base), stream))) != MOE_OK)
    return st;
  PlanBuffers pb;
  pb.idx = at<int32_t>(ws, L.topk_idx);
  pb.header = header;
  pb.load = at<int32_t>(ws, L.load);
  pb.offsets = at<int32_t>(ws, L.offsets);
  pb.block_base = at<int32_t>(ws, L.block_base);
  pb.n = at<int32_t>(ws, L.n);
  pb.row_off = at<int32_t>(ws, L.row_off);
  pb.row_start = at<int32_t>(ws, L.row_start);
  pb.round = at<int32_t>(ws, L.round);
  pb.slot = at<int32_t>(ws, L.slot);
  pb.row_token = at<int32_t>(ws, L.row_token);
  pb.row_dst = at<int32_t>(ws, L.row_dst);
  pb.mb_prefix = at<int32_t>(ws, L.mb_prefix);
  pb.sync = at<int32_t>(ws, L.sync);
  pb.sync_words = pipe_sync_words(s.E, s.C);
  pb.borrow = (s.flags & MOE_FLAG_BORROW) ? 1 : 0;
  pb.dbg = debug_bounds(&s) ? header : nullptr;
  if ((st = cuda_status(launch_plan(pb, s.T, s.k, s.E, s.C, L.max_rounds, stream))) != MOE_OK) return st;

  // The plan summary comes home through host memory mapped into the device, written by a
  // kernel: a copy-engine transfer would queue behind any large transfer the caller has in
  // flight in the same direction on another stream (a result going back to the host while
  // the next batch is planned), and moe_plan would wait for it.
  int32_t host[kHdrWords];
  const MappedWords* mw = mapped_words();
  if (mw != nullptr) {
    if ((st = cuda_status(launch_copy_words(header, mw->dev, kHdrWords, stream))) != MOE_OK) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    std::memcpy(host, const_cast<const int32_t*>(mw->host), sizeof(host));
  } else {
    if (cudaMemcpyAsync(host, header, sizeof(host), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (host[kHdrStatus] != 0) return MOE_ERR_TIMEOUT;

  info->R = host[kHdrR];
  info->max_load = host[kHdrMaxLoad];
  for (int e = 0; e < MOE_MAX_EXPERTS; ++e) info->load[e] = e < s.E ? host[kHdrLoad + e] : 0;
  info->logits = z;
  info->topk_idx = pb.idx;
  info->gate = at<float>(ws, L.gate);
  info->round = pb.round;
  info->slot = pb.slot;
  info->offsets = pb.offsets;
  info->n = pb.n;
  info->plan_flags = s.flags & MOE_FLAG_BORROW;
  return MOE_OK;
}

int moe_round_dispatch(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws, size_t ws_bytes,
                       int32_t r, const uint16_t* x, moe_stream_t stream) {
  moe_workspace_layout_t L;
  int st = check_run(shape, info, ws, ws_bytes, &L);
  if (st != MOE_OK) return st;
  if (r < 0 || r >= info->R || x == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16)) return MOE_ERR_MISALIGNED;
  return do_dispatch(shape, info, ws, L, r, x, reinterpret_cast<cudaStream_t>(stream));
}

int moe_round_gate_up(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws, size_t ws_bytes,
                      int32_t r, const uint16_t* w_gate_up, moe_stream_t stream) {
  moe_workspace_layout_t L;
  int st = check_run(shape, info, ws, ws_bytes, &L);
  if (st != MOE_OK) return st;
  if (r < 0 || r >= info->R || w_gate_up == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(w_gate_up, 16)) return MOE_ERR_MISALIGNED;
  return do_gate_up(shape, info, ws, L, r, w_gate_up, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int moe_round_down(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws, size_t ws_bytes,
                   int32_t r, const uint16_t* w_down, moe_stream_t stream) {
  moe_workspace_layout_t L;
  int st = check_run(shape, info, ws, ws_bytes, &L);
  if (st != MOE_OK) return st;
  if (r < 0 || r >= info->R || w_down == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(w_down, 16)) return MOE_ERR_MISALIGNED;
  return do_down(shape, info, ws, L, r, w_down, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int moe_round_combine(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws, size_t ws_bytes,
                      int32_t r, float* y, moe_stream_t stream) {
  moe_workspace_layout_t L;
  int st = check_run(shape, info, ws, ws_bytes, &L);
  if (st != MOE_OK) return st;
  if (r < 0 || r >= info->R || y == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(y, 16)) return MOE_ERR_MISALIGNED;
  return do_combine(shape, info, ws, L, r, y, reinterpret_cast<cudaStream_t>(stream));
}

int moe_forward(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws, size_t ws_bytes,
                const uint16_t* x, const uint16_t* w_gate_up, const uint16_t* w_down, float* y,
                moe_stream_t stream_) {
  moe_workspace_layout_t L;
  int st = check_run(shape, info, ws, ws_bytes, &L);
  if (st != MOE_OK) return st;
  if (shape->T > 0 && (x == nullptr || w_gate_up == nullptr || w_down == nullptr || y == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_gate_up, 16) || !aligned(w_down, 16) || !aligned(y, 16))
    return MOE_ERR_MISALIGNED;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const int R = info->R;
  if (R == 0) return MOE_OK;
  auto small = [&](int rr) {
    int32_t n_host[MOE_MAX_EXPERTS];
    int rows = 0;
    round_rows(shape, info, rr, n_host, &rows);
    return static_cast<size_t>(rows) * shape->d * 2 <= kFuseCopyBytes;
  };
  // Rounds [0, r0) run as per-round launches, [r0, R) in one pipelined launch.
  // A round is thin when even 128-column tiles of its gate/up GEMM would leave SMs idle: its
  // steps are latency-bound and gain from overlapping their neighbours. The pipelined launch
  // takes the trailing run of thin rounds (its 32-column tiles and its copy warps suit thin
  // rounds only; a large round's copies get full-bandwidth kernels of their own).
  auto thin = [&](int rr) {
    long long blocks = 0;
    const long long base = static_cast<long long>(rr) * shape->C;
    for (int e = 0; e < shape->E; ++e) {
      const long long rem = info->load[e] - base;
      const long long n = rem <= 0 ? 0 : (rem >= shape->C ? shape->C : rem);
      blocks += (n + kPipeRowBlock - 1) / kPipeRowBlock;
    }
    return blocks * (shape->d_ff / 128 > 0 ? shape->d_ff / 128 : 1) < num_sms();
  };
  int r0 = R;
  if (shape->flags & MOE_FLAG_PIPELINE_ALL) {
    r0 = 0;
  } else if (!(shape->flags & (MOE_FLAG_PER_ROUND | MOE_FLAG_BORROW | MOE_FLAG_DEBUG_BOUNDS))) {
    // borrowing and the debug bounds checks run per round only
    while (r0 > 0 && thin(r0 - 1)) --r0;
  }
  // Per-round launch order. A round's copy steps ride on the neighbouring GEMM launches as
  // their copy warps -- combine(r-1) on gate/up(r), dispatch(r+1) on down(r) -- when they are
  // small (at most kFuseCopyBytes of rows) or when their estimated time there stays below that
  // GEMM's; otherwise they run as their own full-bandwidth kernels, dispatch(r+1) right after
  // down(r), combine(r) after that. Each launch depends only on the one before it (PDL wait), and
  // no two steps of one launch touch the same buffer: dispatch writes buf, gate/up reads buf and
  // writes h, down reads h and writes out, combine reads out and updates y. The first pipelined
  // round is dispatched here too, so the pipelined launch starts with its rows in place.
  auto rows_of = [&](int rr) {
    int32_t n_host[MOE_MAX_EXPERTS];
    int rows = 0;
    round_rows(shape, info, rr, n_host, &rows);
    return rows;
  };
  // copy warps move about kSideCopyGBs while the GEMM runs at about kGemmTflops
  auto side_s = [&](double bytes) { return bytes / (kSideCopyGBs * 1e9); };
  auto gemm_s = [&](double flops) { return flops / (kGemmTflops * 1e12); };
  auto combine_rides = [&](int rc, int rg) {   // combine(rc) on gate/up(rg)
    if (small(rc)) return true;
    const double rows_c = rows_of(rc), tokens_c = rows_c < shape->T ? rows_c : shape->T;
    return side_s((2.0 * rows_c + 8.0 * tokens_c) * shape->d) <=
           gemm_s(4.0 * rows_of(rg) * shape->d * shape->d_ff);
  };
  auto dispatch_rides = [&](int rd, int rg) {   // dispatch(rd) on down(rg)
    if (small(rd)) return true;
    return side_s(4.0 * rows_of(rd) * shape->d) <= gemm_s(2.0 * rows_of(rg) * shape->d * shape->d_ff);
  };
  auto per_round = [&](int rb, int re) -> int {
    int rc = MOE_OK;
    for (int r = rb; r < re; ++r) {
      const bool fuse_combine = r > rb && combine_rides(r - 1, r);
      const RoundCopy comb = make_copy(shape, info, ws, L, true, r > 0 ? r - 1 : 0, x, y);
      if ((rc = do_gate_up(shape, info, ws, L, r, w_gate_up, fuse_combine ? &comb : nullptr, stream)) != MOE_OK)
        return rc;
      const bool next = r + 1 < R;
      const bool fuse_dispatch = next && dispatch_rides(r + 1, r);
      const RoundCopy disp = make_copy(shape, info, ws, L, false, next ? r + 1 : r, x, y);
      if ((rc = do_down(shape, info, ws, L, r, w_down, fuse_dispatch ? &disp : nullptr, stream)) != MOE_OK) return rc;
      if (next && !fuse_dispatch && (rc = do_dispatch(shape, info, ws, L, r + 1, x, stream)) != MOE_OK) return rc;
      if (!(r + 1 < re && combine_rides(r, r + 1)) && (rc = do_combine(shape, info, ws, L, r, y, stream)) != MOE_OK)
        return rc;
    }
    return rc;
  };
  if ((st = do_dispatch(shape, info, ws, L, 0, x, stream)) != MOE_OK) return st;
  if ((st = per_round(0, r0)) != MOE_OK) return st;
  if (r0 < R) {
    PipelineArgs p{};
    p.x = x;
    p.w_gate_up = w_gate_up;
    p.w_down = w_down;
    p.buf[0] = at<uint16_t>(ws, L.buf);
    p.h[0] = at<uint16_t>(ws, L.h);
    p.out[0] = at<uint16_t>(ws, L.out);
    p.buf[1] = at<uint16_t>(ws, L.buf2);
    p.h[1] = at<uint16_t>(ws, L.h2);
    p.out[1] = at<uint16_t>(ws, L.out2);
    p.y = y;
    p.idx = at<int32_t>(ws, L.topk_idx);
    p.gate = at<float>(ws, L.gate);
    p.round = at<int32_t>(ws, L.round);
    p.slot = at<int32_t>(ws, L.slot);
    p.n = at<int32_t>(ws, L.n);
    p.row_start = at<int32_t>(ws, L.row_start);
    p.row_token = at<int32_t>(ws, L.row_token);
    p.row_dst = at<int32_t>(ws, L.row_dst);
    p.mb_prefix = at<int32_t>(ws, L.mb_prefix);
    p.sync = at<int32_t>(ws, L.sync);
    p.status = at<int32_t>(ws, L.header) + kHdrStatus;
    p.T = shape->T;
    p.k = shape->k;
    p.E = shape->E;
    p.C = shape->C;
    p.d = shape->d;
    p.F = shape->d_ff;
    p.r0 = r0;
    p.R = R;
    p.r0_dispatched = 1;
    p.gw = pipe_gate_width(shape->d);
    const cudaError_t e = launch_round_pipeline(p, stream);
    if (e == cudaErrorCooperativeLaunchTooLarge) {
      // not every SM is available to this context (a partitioned GPU): run those rounds per round
      cudaGetLastError();
      return per_round(r0, R);
    }
    if ((st = cuda_status(e)) != MOE_OK) return st;
  }
  return MOE_OK;
}

int moe_device_status(const moe_shape_t* shape, void* ws, moe_stream_t stream_) {
  const int st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (ws == nullptr) return MOE_ERR_INVALID_ARG;
  moe_workspace_layout_t L;
  make_layout(shape, &L);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (debug_bounds(shape)) {   // compare every guard word first
    GuardList guards;
    make_layout(shape, &L, &guards);
    if (cuda_status(launch_guards(static_cast<uint8_t*>(ws), guards, 1, at<int32_t>(ws, L.header), stream)) !=
        MOE_OK)
      return MOE_ERR_CUDA;
  }
  int32_t word = 0;
  if (cudaMemcpyAsync(&word, at<int32_t>(ws, L.header) + kHdrStatus, 4, cudaMemcpyDeviceToHost, stream) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (word & (kStatusBounds | kStatusCanary)) return MOE_ERR_BOUNDS;
  return word != 0 ? MOE_ERR_TIMEOUT : MOE_OK;
}

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MOE_ERR_MISALIGNED: return "misaligned pointer";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "a kernel wait timed out";
    case MOE_ERR_NO_DEVICE: return "current device is not sm_100";
    case MOE_ERR_NOALLOC_LIMIT: return "shape needs more scratch than moe_plan_noalloc's static array";
    case MOE_ERR_BOUNDS: return "a debug bounds check failed or a workspace guard was overwritten";
    default: return "unknown status";
  }
}

uint64_t moe_launch_count(void) { return g_launches.load(); }

int moe_profile_enable(int on) {
  if (on && !g_prof.created) {
    for (int i = 0; i < 2 * kProfMax; ++i)
      if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) return MOE_ERR_CUDA;
    g_prof.created = true;
  }
  g_prof.on = on != 0;
  g_prof.n = 0;
  return MOE_OK;
}

int moe_profile_read(int32_t counts[MOE_PROFILE_KINDS], double ms[MOE_PROFILE_KINDS]) {
  if (counts == nullptr || ms == nullptr) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < MOE_PROFILE_KINDS; ++i) {
    counts[i] = 0;
    ms[i] = 0.0;
  }
  for (int i = 0; i < g_prof.n; ++i) {
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess) return MOE_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess) return MOE_ERR_CUDA;
    counts[g_prof.kind[i]] += 1;
    ms[g_prof.kind[i]] += t;
  }
  g_prof.n = 0;
  return MOE_OK;
}

}  // extern "C"
