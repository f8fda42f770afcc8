// ep_round.cu - device data path of the expert-parallel form of the layer, one round at a time.
//
// "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, the multi-round dropless
// MoE item [section "Scaling MoE", Fig. 6]: the experts are split into groups, one group per
// expert-parallel rank, every group runs dispatch -> compute -> collect rounds with a fixed
// per-expert capacity, and the token metadata stays on the device. Rank g owns the E/G
// contiguous experts [g E/G, (g+1) E/G); an expert's capacity C per round is shared by all
// source ranks, which fill it in (source rank, token) order (ep_plan.cu has the tables).
//
// Per rank and round r, the caller runs:
//   pack      this rank's pairs of round r, in (expert, slot) order, into a send buffer; the
//             rows for owner g form one contiguous chunk (moe_ep_exchange_plan's send counts)
//   exchange  (the caller's transport: an all-to-all of the chunks)
//   experts   on the owner: both grouped GEMMs straight over the received rows, one group per
//             (source rank, local expert), with no copy into a per-expert buffer
//   exchange  back, the same chunks in the other direction
//   combine   y[t] (+)= gate * result row, for this rank's pairs of round r, j ascending
//
// Plan of this rank (moe_ep_plan), from the pairs' ranks among this rank's own pairs of each
// expert (moe_plan without borrowing: local rank = round * C + slot) and the global offsets:
//   global rank g = base[e] + local rank;   round = g / C
//   slot within this rank's rows of (round, e) = g - max(base[e], round * C)
// and this rank's rows of round r are packed expert after expert at row_off[r][e].
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <vector>

#include "kernels.h"
#include "moe.h"
#include "sm100.cuh"

namespace moe {
namespace {

struct EpLayout {
  size_t base_all, loads_all, row_off, row_start, round, slot, row_token, row_dst, grp_rows, grp_row, grp_expert;
  size_t total;
  int max_rounds;
};

// Every rank has T tokens, so no expert receives more than G T pairs: at most ceil(G T / C) rounds.
EpLayout ep_layout(const moe_shape_t* s, int G) {
  EpLayout L{};
  size_t off = 0;
  auto take = [&](long long bytes) {
    const size_t o = off;
    off += (static_cast<size_t>(bytes) + 255) & ~static_cast<size_t>(255);
    return o;
  };
  const long long T = s->T, E = s->E, k = s->k;
  L.max_rounds = s->T == 0 ? 0 : static_cast<int>((static_cast<long long>(G) * T + s->C - 1) / s->C);
  L.base_all = take(G * E * 4);
  L.loads_all = take(G * E * 4);
  L.row_off = take(static_cast<long long>(L.max_rounds) * E * 4);
  L.row_start = take((L.max_rounds + 1ll) * 4);
  L.round = take(T * k * 4);
  L.slot = take(T * k * 4);
  L.row_token = take(T * k * 4);
  L.row_dst = take(T * k * 4);
  L.grp_rows = take(E * 4);   // G * (E / G) groups
  L.grp_row = take(E * 4);
  L.grp_expert = take(E * 4);
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

long long overlap(long long lo, long long hi, long long a, long long b) {
  const long long l = lo > a ? lo : a, h = hi < b ? hi : b;
  return h > l ? h - l : 0;
}

// Host view of the counts: base[s][e] = pairs of e on ranks before s; total[e]; R.
struct EpCounts {
  int G, E, C, R;
  std::vector<long long> base, total;
  const int32_t* loads;
  long long rows(int s, int e, int r) const {   // rank s's rows of expert e in round r
    const long long b = base[static_cast<size_t>(s) * E + e];
    return overlap(static_cast<long long>(r) * C, static_cast<long long>(r + 1) * C, b,
                   b + loads[static_cast<size_t>(s) * E + e]);
  }
};

int make_counts(const moe_shape_t* s, int G, int rank, const int32_t* loads, EpCounts* c) {
  if (moe_workspace_bytes(s) == 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (loads == nullptr || G < 1 || s->E % G != 0 || rank < 0 || rank >= G) return MOE_ERR_INVALID_ARG;
  if (s->flags & MOE_FLAG_BORROW) return MOE_ERR_INVALID_ARG;   // the pairs' local ranks need C-slot rounds
  c->G = G;
  c->E = s->E;
  c->C = s->C;
  c->loads = loads;
  c->base.assign(static_cast<size_t>(G) * s->E, 0);
  c->total.assign(s->E, 0);
  long long mine = 0, max_total = 0;
  for (int q = 0; q < G; ++q)
    for (int e = 0; e < s->E; ++e) {
      const int32_t v = loads[static_cast<size_t>(q) * s->E + e];
      if (v < 0) return MOE_ERR_INVALID_ARG;
      c->base[static_cast<size_t>(q) * s->E + e] = c->total[e];
      c->total[e] += v;
      if (q == rank) mine += v;
    }
  if (mine != static_cast<long long>(s->T) * s->k) return MOE_ERR_INVALID_ARG;
  for (int e = 0; e < s->E; ++e) max_total = c->total[e] > max_total ? c->total[e] : max_total;
  const long long R = (max_total + s->C - 1) / s->C;
  const long long cap = s->T == 0 ? 0 : (static_cast<long long>(G) * s->T + s->C - 1) / s->C;
  if (R > cap) return MOE_ERR_INVALID_ARG;   // some rank has more than T tokens
  c->R = static_cast<int>(R);
  return MOE_OK;
}

// One thread per pair: its global round, its slot within this rank's rows of (round, expert),
// and its place in this rank's packed row list.
__global__ void __launch_bounds__(256) ep_replan_kernel(const int32_t* __restrict__ idx,
                                                        const int32_t* __restrict__ local_round,
                                                        const int32_t* __restrict__ local_slot, int pairs, int k,
                                                        int E, int C, const int32_t* __restrict__ base,
                                                        const int32_t* __restrict__ row_off,
                                                        const int32_t* __restrict__ row_start,
                                                        int32_t* __restrict__ round_out, int32_t* __restrict__ slot_out,
                                                        int32_t* __restrict__ row_token, int32_t* __restrict__ row_dst) {
  sm100::grid_dependency_wait();
  sm100::grid_launch_dependents();
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= pairs) return;
  const int e = idx[p];
  const long long b = base[e];
  const long long g = b + static_cast<long long>(local_round[p]) * C + local_slot[p];
  const int r = static_cast<int>(g / C);
  const long long lo = b > static_cast<long long>(r) * C ? b : static_cast<long long>(r) * C;
  const int q = static_cast<int>(g - lo);
  round_out[p] = r;
  slot_out[p] = q;
  const int pos = row_off[static_cast<size_t>(r) * E + e] + q;
  row_token[pos] = p / k;
  row_dst[pos] = pos - row_start[r];
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

MOE_API size_t moe_ep_workspace_bytes(const moe_shape_t* shape, int32_t G) {
  if (shape == nullptr || moe_workspace_bytes(shape) == 0 || G < 1 || shape->E % G != 0) return 0;
  return ep_layout(shape, G).total;
}

MOE_API int moe_ep_plan(const moe_shape_t* shape, int32_t G, int32_t rank, const int32_t* loads,
                        const moe_plan_info_t* info, void* ws, size_t ws_bytes, void* ep_ws, size_t ep_bytes,
                        int32_t* R, moe_stream_t stream_) {
  if (shape == nullptr || info == nullptr || ws == nullptr || ep_ws == nullptr || R == nullptr)
    return MOE_ERR_INVALID_ARG;
  EpCounts c;
  int st = make_counts(shape, G, rank, loads, &c);
  if (st != MOE_OK) return st;
  moe_workspace_layout_t L;
  if ((st = moe_workspace_layout(shape, &L)) != MOE_OK) return st;
  if (ws_bytes < L.total_bytes || ep_bytes < ep_layout(shape, G).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(ws) | reinterpret_cast<uintptr_t>(ep_ws)) & 255u) return MOE_ERR_MISALIGNED;
  if (info->plan_flags & MOE_FLAG_BORROW) return MOE_ERR_INVALID_ARG;
  for (int e = 0; e < shape->E; ++e)   // the local plan was made from the same pairs
    if (info->load[e] != loads[static_cast<size_t>(rank) * shape->E + e]) return MOE_ERR_INVALID_ARG;
  const EpLayout P = ep_layout(shape, G);
  const int E = shape->E;
  // this rank's rows of round r, packed expert after expert
  std::vector<int32_t> row_off(static_cast<size_t>(c.R) * E), row_start(c.R + 1), base_all(c.base.size());
  long long running = 0;
  for (int r = 0; r < c.R; ++r) {
    row_start[r] = static_cast<int32_t>(running);
    for (int e = 0; e < E; ++e) {
      row_off[static_cast<size_t>(r) * E + e] = static_cast<int32_t>(running);
      running += c.rows(rank, e, r);
    }
  }
  row_start[c.R] = static_cast<int32_t>(running);
  for (size_t i = 0; i < c.base.size(); ++i) base_all[i] = static_cast<int32_t>(c.base[i]);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  auto up = [&](size_t off, const void* src, size_t bytes) {
    return bytes == 0 || cudaMemcpyAsync(at<uint8_t>(ep_ws, off), src, bytes, cudaMemcpyHostToDevice, stream) == cudaSuccess;
  };
  if (!up(P.row_off, row_off.data(), row_off.size() * 4) || !up(P.row_start, row_start.data(), row_start.size() * 4) ||
      !up(P.base_all, base_all.data(), base_all.size() * 4) ||
      !up(P.loads_all, loads, static_cast<size_t>(G) * E * 4))
    return MOE_ERR_CUDA;
  const int pairs = shape->T * shape->k;
  if (pairs > 0) {
    launch_begin(kKindPlan, stream);
    const cudaError_t e = launch_pdl(ep_replan_kernel, dim3((pairs + 255) / 256), dim3(256), 0, stream,
                                     at<int32_t>(ws, L.topk_idx), at<int32_t>(ws, L.round), at<int32_t>(ws, L.slot),
                                     pairs, shape->k, E, shape->C,
                                     at<int32_t>(ep_ws, P.base_all) + static_cast<size_t>(rank) * E,
                                     at<int32_t>(ep_ws, P.row_off), at<int32_t>(ep_ws, P.row_start),
                                     at<int32_t>(ep_ws, P.round), at<int32_t>(ep_ws, P.slot),
                                     at<int32_t>(ep_ws, P.row_token), at<int32_t>(ep_ws, P.row_dst));
    launch_end(kKindPlan, stream);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;   // the host tables are copied
  *R = c.R;
  return MOE_OK;
}

MOE_API int moe_ep_round_pack(const moe_shape_t* shape, int32_t G, int32_t rank, const int32_t* loads,
                              void* ep_ws, size_t ep_bytes, int32_t r, const uint16_t* x, uint16_t* sendbuf,
                              moe_stream_t stream) {
  EpCounts c;
  int st = make_counts(shape, G, rank, loads, &c);
  if (st != MOE_OK) return st;
  if (ep_ws == nullptr || r < 0 || r >= c.R || (shape->T > 0 && (x == nullptr || sendbuf == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (ep_bytes < ep_layout(shape, G).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  long long rows = 0;
  for (int e = 0; e < shape->E; ++e) rows += c.rows(rank, e, r);
  const EpLayout P = ep_layout(shape, G);
  return launch_dispatch(x, sendbuf, at<int32_t>(ep_ws, P.row_start), at<int32_t>(ep_ws, P.row_token),
                         at<int32_t>(ep_ws, P.row_dst), r, static_cast<int>(rows), shape->d,
                         reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

MOE_API int moe_ep_round_experts(const moe_shape_t* shape, int32_t G, int32_t rank, const int32_t* loads,
                                 void* ep_ws, size_t ep_bytes, int32_t r, const uint16_t* recvbuf,
                                 const uint16_t* w_gate_up, const uint16_t* w_down, uint16_t* h, uint16_t* out,
                                 int64_t buf_rows, void* ws, moe_stream_t stream_) {
  EpCounts c;
  int st = make_counts(shape, G, rank, loads, &c);
  if (st != MOE_OK) return st;
  if (ep_ws == nullptr || ws == nullptr || r < 0 || r >= c.R || w_gate_up == nullptr || w_down == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (ep_bytes < ep_layout(shape, G).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  const int per = shape->E / G, groups = G * per;
  std::vector<int32_t> rows(groups), grow(groups), gexp(groups);
  long long running = 0;
  for (int q = 0; q < G; ++q)
    for (int l = 0; l < per; ++l) {
      const int g = q * per + l;
      rows[g] = static_cast<int32_t>(c.rows(q, rank * per + l, r));
      grow[g] = static_cast<int32_t>(running);
      gexp[g] = l;
      running += rows[g];
    }
  if (running > buf_rows) return MOE_ERR_INVALID_ARG;   // at most E/G * C rows arrive per round
  if (running == 0) return MOE_OK;
  if (recvbuf == nullptr || h == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  const EpLayout P = ep_layout(shape, G);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (cudaMemcpyAsync(at<int32_t>(ep_ws, P.grp_rows), rows.data(), groups * 4, cudaMemcpyHostToDevice, stream) !=
          cudaSuccess ||
      cudaMemcpyAsync(at<int32_t>(ep_ws, P.grp_row), grow.data(), groups * 4, cudaMemcpyHostToDevice, stream) !=
          cudaSuccess ||
      cudaMemcpyAsync(at<int32_t>(ep_ws, P.grp_expert), gexp.data(), groups * 4, cudaMemcpyHostToDevice, stream) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  moe_workspace_layout_t L;
  if ((st = moe_workspace_layout(shape, &L)) != MOE_OK) return st;
  const cudaError_t e =
      launch_ep_experts(recvbuf, w_gate_up, w_down, h, out, groups, at<int32_t>(ep_ws, P.grp_rows), rows.data(),
                        at<int32_t>(ep_ws, P.grp_row), at<int32_t>(ep_ws, P.grp_expert), buf_rows, per, shape->d,
                        shape->d_ff, at<int32_t>(ws, L.header) + kHdrStatus, stream);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  // the host tables above are read by the copies before this call returns
  return cudaStreamSynchronize(stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

MOE_API int moe_ep_round_combine(const moe_shape_t* shape, int32_t G, int32_t rank, const int32_t* loads,
                                 void* ws, size_t ws_bytes, void* ep_ws, size_t ep_bytes, int32_t r,
                                 const uint16_t* retbuf, float* y, moe_stream_t stream) {
  EpCounts c;
  int st = make_counts(shape, G, rank, loads, &c);
  if (st != MOE_OK) return st;
  moe_workspace_layout_t L;
  if ((st = moe_workspace_layout(shape, &L)) != MOE_OK) return st;
  if (ws == nullptr || ep_ws == nullptr || r < 0 || r >= c.R || (shape->T > 0 && (retbuf == nullptr || y == nullptr)))
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < L.total_bytes || ep_bytes < ep_layout(shape, G).total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  const EpLayout P = ep_layout(shape, G);
  // token by token (rows = T): every token checks its pairs' rounds; pair (e, slot) of round r is
  // row row_off[r][e] - row_start[r] + slot of the returned rows
  return launch_combine(retbuf, y, at<int32_t>(ws, L.topk_idx), at<float>(ws, L.gate), at<int32_t>(ep_ws, P.round),
                        at<int32_t>(ep_ws, P.slot), at<int32_t>(ep_ws, P.row_start), at<int32_t>(ep_ws, P.row_token),
                        at<int32_t>(ep_ws, P.row_dst), shape->T, shape->k, shape->C, shape->d, r, shape->T,
                        at<int32_t>(ep_ws, P.row_off), shape->E, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

}  // extern "C"
