// backward.h - internal launchers of the backward pass (backward.cu), called by the C ABI in
// moe_api.cu. Not part of the public C ABI (that is include/moe.h).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"

namespace moe {

// Kernel kinds of the backward's launches for profiling (after the forward's KernelKind values;
// same numbering as the public header).
constexpr int kKindBackwardRecompute = 8;
constexpr int kKindBackwardDh = 9;
constexpr int kKindBackwardDxWgrad = 10;
constexpr int kKindBackwardCopy = 11;
constexpr int kKindBackwardRecDh = 12;

// ---- backward with per-round recompute (backward.cu)
// Device pointers of one backward call: the forward's plan (read only), the caller's tensors and
// gradients, and the backward workspace's buffers (moe_backward_layout_t).
struct BackwardArgs {
  const uint16_t* x;          // [T, d]
  const uint16_t* w_gate_up;  // [E, 2F, d]
  const uint16_t* w_down;     // [E, d, F]
  const float* dy;            // [T, d]
  const float* logits;        // [T, E] the logits the plan used
  const int32_t* idx;         // plan: [T, k]
  const float* gate;          // plan: [T, k]
  const int32_t* round;       // plan: [T, k]
  const int32_t* slot;        // plan: [T, k]
  const int32_t* n;           // plan: [max_rounds, E]
  const int32_t* row_start;   // plan: [max_rounds + 1]
  const int32_t* row_off;     // plan: [max_rounds, E] first row of (round, expert) in the row list
  const int32_t* row_token;   // plan: round-major row list
  const int32_t* row_dst;
  float* dx;                  // [T, d]
  float* dw_gate_up;          // [E, 2F, d]
  float* dw_down;             // [E, d, F]
  float* dz;                  // [T, E]
  // backward workspace: per-round buffers of `rows` rows (E * C, or with pooled rows E * C + 64 E:
  // expert e's rows of round r from seg_off[r][e], a multiple of 64)
  uint16_t* xbuf;             // [rows, d]
  uint16_t* dybuf;            // [rows, d]
  float* row_gate;            // [rows]
  uint16_t* ab;               // [rows, 2F]
  uint16_t* hg;               // [rows, F]
  uint16_t* dab;              // [rows, 2F]
  float* dgate_part;          // [rows, F / 64]
  uint16_t* dxbuf;            // [rows, d]
  float* dgate;               // [T, k]
  float* ones;                // [T, k]
  int32_t* seg_off;           // [max_rounds, E] pooled rows: each expert's first row in a round
  int32_t* zeros;             // [max_rounds + 1]
  int32_t* status;
  int T, k, E, C, d, F, renorm;
  int pooled;                 // capacity borrowing: pooled round rows (see the plan's row_off)
  int rows;                   // rows of the per-round buffers
};
// Rows of the per-round buffers: E * C per expert (expert e's rows at e * C), or with pooled rows
// E * C + 64 E (each expert's segment rounded up to 64 rows, in expert order).
long long backward_rows(int E, int C, bool pooled);
// Rows of the second, smaller buffer set (always pooled): E * C / 8 rounded up to 64, plus 64 E.
long long backward_rows2(int E, int C);
// Zeroes the weight gradients of experts without rows (load_host: host copy of the loads), fills
// the unit gates, and writes the segment table seg_off of the R rounds (from the plan's n on the
// device) and the zero words.
cudaError_t launch_backward_prepare(const BackwardArgs& a, const int32_t* load_host, int R, cudaStream_t stream);
// A round in two halves, each on a stream of its own choosing. n_host: the round's rows per
// expert. a: the round's buffer set (its pointers, pooled and rows).
// Whether a round's front half is one fused recompute + dh launch in the single-CTA form with at
// most as many tiles as the device has SMs (so that it leaves SMs to the round before's back
// half).
bool backward_front_is_thin(const BackwardArgs& a, const int32_t* n_host);
// Front: the dispatch of x and dy (when `gather`; else the previous round's combine launch ran
// it), the recompute and dh (+ the SwiGLU backward); *parts: dgate partials per row, for the back.
cudaError_t launch_backward_front(const BackwardArgs& a, int r, const int32_t* n_host, bool gather, int* parts,
                                  cudaStream_t stream);
// Back: the dx GEMM and the weight gradients (one launch), the dx combine and dgate. With a_next
// and n_next (the next round's buffer set and rows per expert) the next round's dispatch runs in
// the combine's launch.
cudaError_t launch_backward_back(const BackwardArgs& a, int r, const int32_t* n_host, int parts,
                                 const BackwardArgs* a_next, const int32_t* n_next, cudaStream_t stream);
// dz from dgate and the logits, after the last round.
cudaError_t launch_backward_gates(const BackwardArgs& a, cudaStream_t stream);

}  // namespace moe
