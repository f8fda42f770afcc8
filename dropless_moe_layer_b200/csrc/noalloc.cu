// noalloc.cu - routing and round planning with no device allocation anywhere.
//
// Some callers cannot allocate device memory at the point where they route a batch:
// code running under a memory pool that owns every byte of the device, plugins handed
// only their input and output buffers by a host framework, or deployments that forbid
// cudaMalloc after start-up. moe_plan() needs a caller-allocated workspace; this entry
// point instead keeps the planner's scratch (plan header, per-block counts, expert
// loads and offsets, per-round row tables and the round-major row list) in one
// file-scope device array of fixed size. The caller passes only the logits and the
// four [T, k] output arrays.
//
// The array is MOE_NOALLOC_SCRATCH_BYTES large. CUDA reserves it on a device when it loads
// this file's code there: at context creation under eager module loading, and under lazy
// loading (the CUDA 12 default) at the first moe_plan_noalloc() on that device, whose address
// lookup loads it. From then on the device holds it until the process exits. So a caller that
// must not allocate later makes one call per device at start-up (a batch of T = 0 will do),
// before its memory pool takes the device and before any stream capture. All calls share the
// array: two calls whose work overlaps on the GPU (different streams, or different host
// threads) race on it. The contents left by the previous call are never trusted: the header
// (status word included) is cleared by every call and every other region is fully rewritten
// before it is read.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "moe.h"

namespace {

static __device__ __align__(256) uint8_t g_plan_scratch[MOE_NOALLOC_SCRATCH_BYTES];

// Device address of g_plan_scratch on the current device. Host code must not use the symbol
// itself as a device pointer. The address is looked up on every call, not cached: a cached
// address would outlive the context it belongs to (cudaDeviceReset tears the module down).
int scratch_for_current_device(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_plan_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
  *out = p;
  return MOE_OK;
}

size_t round_up(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

}  // namespace

extern "C" MOE_API int moe_plan_noalloc(const moe_shape_t* shape, const float* logits,
                                        int32_t* topk_idx, float* gate, int32_t* round,
                                        int32_t* slot, int32_t* R, int32_t* load,
                                        moe_stream_t stream_) {
  if (shape == nullptr || R == nullptr) return MOE_ERR_INVALID_ARG;
  if (moe_workspace_bytes(shape) == 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  const moe_shape_t& s = *shape;
  if (s.T > 0 && (logits == nullptr || topk_idx == nullptr || gate == nullptr || round == nullptr ||
                  slot == nullptr))
    return MOE_ERR_INVALID_ARG;
  auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (misaligned(logits) || misaligned(topk_idx) || misaligned(gate) || misaligned(round) ||
      misaligned(slot))
    return MOE_ERR_MISALIGNED;

  // Scratch layout (256-byte aligned regions) and the size limit.
  const long long T = s.T, E = s.E, k = s.k;
  const int max_rounds = s.T == 0 ? 0 : (s.T + s.C - 1) / s.C;
  const int blocks = static_cast<int>((T + moe::kPlanTokensPerBlock - 1) / moe::kPlanTokensPerBlock);
  size_t off = 0;
  auto take = [&](long long bytes) {
    const size_t o = off;
    off += round_up(static_cast<size_t>(bytes));
    return o;
  };
  const size_t o_header = take(moe::kHdrWords * 4ll);
  const size_t o_block = take(static_cast<long long>(blocks) * E * 4);   // adjacent: one memset
  const size_t o_load = take(E * 4);
  const size_t o_offsets = take((E + 1) * 4);
  const size_t o_n = take(static_cast<long long>(max_rounds) * E * 4);
  const size_t o_row_off = take(static_cast<long long>(max_rounds) * E * 4);
  const size_t o_row_start = take((max_rounds + 1ll) * 4);
  const size_t o_row_token = take(T * k * 4);
  const size_t o_row_dst = take(T * k * 4);
  if (off > static_cast<size_t>(MOE_NOALLOC_SCRATCH_BYTES)) return MOE_ERR_NOALLOC_LIMIT;

  int major = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10) return MOE_ERR_NO_DEVICE;
  void* base = nullptr;
  int st = scratch_for_current_device(&base);
  if (st != MOE_OK) return st;
  uint8_t* scratch = static_cast<uint8_t*>(base);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);

  int32_t* header = reinterpret_cast<int32_t*>(scratch + o_header);
  if (cudaMemsetAsync(header, 0, o_block - o_header + static_cast<size_t>(blocks) * E * 4, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::launch_router_topk(logits, s.T, s.E, s.k, (s.flags & MOE_FLAG_RENORM_TOPK) ? 1 : 0, topk_idx,
                              gate, reinterpret_cast<int32_t*>(scratch + o_block), stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  moe::PlanBuffers pb;
  pb.idx = topk_idx;
  pb.header = header;
  pb.load = reinterpret_cast<int32_t*>(scratch + o_load);
  pb.offsets = reinterpret_cast<int32_t*>(scratch + o_offsets);
  pb.block_base = reinterpret_cast<int32_t*>(scratch + o_block);
  pb.n = reinterpret_cast<int32_t*>(scratch + o_n);
  pb.row_off = reinterpret_cast<int32_t*>(scratch + o_row_off);
  pb.row_start = reinterpret_cast<int32_t*>(scratch + o_row_start);
  pb.round = round;
  pb.slot = slot;
  pb.row_token = reinterpret_cast<int32_t*>(scratch + o_row_token);
  pb.row_dst = reinterpret_cast<int32_t*>(scratch + o_row_dst);
  pb.mb_prefix = nullptr;   // planning only: no forward pass runs on this scratch
  pb.sync = nullptr;
  pb.sync_words = 0;
  pb.borrow = (s.flags & MOE_FLAG_BORROW) ? 1 : 0;
  pb.dbg = nullptr;
  if (moe::launch_plan(pb, s.T, s.k, s.E, s.C, max_rounds, stream) != cudaSuccess) return MOE_ERR_CUDA;

  int32_t host[moe::kHdrWords];
  if (cudaMemcpyAsync(host, header, sizeof(host), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (host[moe::kHdrStatus] != 0) return MOE_ERR_TIMEOUT;
  *R = host[moe::kHdrR];
  if (load != nullptr)
    for (int e = 0; e < s.E; ++e) load[e] = host[moe::kHdrLoad + e];
  return MOE_OK;
}
