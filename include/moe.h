/*
 * moe.h - C ABI of the multi-round dropless MoE layer forward for NVIDIA B200 (sm_100a).
 *
 * The method (sources, by page and section):
 *   - "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, the multi-round
 *     dropless MoE item [section "Scaling MoE", Fig. 6]: each expert group runs one or
 *     more dispatch -> compute -> collect rounds with a fixed per-expert token capacity;
 *     overflow waits for another round; memory stays static whatever the imbalance;
 *     capacity is tunable.
 *   - "Microsoft AI's MAI-Base-2 trained on 16K GPUs with Muon", section "Expert groups
 *     keep memory fixed when tokens pile up": a router sends each token to a few experts;
 *     larger capacity costs memory, smaller capacity costs rounds.
 *   - "MAI-Base-2: Microsoft's 2.8T Model is a BREAKTHROUGH" (transcript, 03:11): no token
 *     is dropped.
 *
 * What this library computes (all experts on one GPU):
 *   z = logits [T,E] fp32 (given, or x @ w_router^T + bias)
 *   idx[t,0..k-1] = top-k experts of z[t] (logit descending, ties -> lower expert index)
 *   gate[t,j]     = softmax(z[t])[idx[t,j]] (fp32; divided by the k gates' sum with
 *                   MOE_FLAG_RENORM_TOPK)
 *   rank(t,j)     = number of tokens t' < t that selected the same expert
 *   round = rank / C, slot = rank % C, R = ceil(max_e load_e / C)
 *   for r in 0..R-1:
 *     dispatch: buf[e][slot] = x[t] for every pair in round r       (buf: [E, C, d] bf16)
 *     experts:  h = bf16(silu(buf W1^T) * (buf W3^T)); out = bf16(h W2^T)   (grouped GEMMs,
 *               out: [E, C, d] bf16)
 *     combine:  y[t] += gate[t,j] * out[e][slot] for the round's pairs, j ascending
 *   y [T, d] fp32 equals the capacity-free dropless MoE output up to bf16 rounding of the
 *   expert intermediates.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major, contiguous,
 *     16-byte aligned. bf16 is passed as its uint16_t bit pattern. The workspace must be
 *     256-byte aligned. The library allocates no device memory (moe_plan keeps one small
 *     pinned, device-mapped host buffer per host thread and device; see moe_plan).
 *   - Entry points return MOE_OK (0) or a negative moe_status; invalid arguments are found
 *     on the host before any kernel is launched, and no entry point aborts the process.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     Only moe_plan() synchronizes the stream (once, to learn the round count R).
 *   - Faults of earlier asynchronous work surface as MOE_ERR_CUDA from a later call.
 *   - Results are deterministic: the same inputs, C and GPU give the same bits.
 *   - Shape limits: T >= 0, 1 <= E <= 256, 1 <= k <= min(E, 16), d and d_ff multiples of
 *     64 in [64, 16384], C >= 1, T*k < 2^31, E*C < 2^31.
 */
#ifndef DROPLESS_MOE_H_
#define DROPLESS_MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* moe_stream_t;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,         /* null pointer, bad round index, inconsistent plan info */
  MOE_ERR_UNSUPPORTED_SHAPE = -2,   /* a shape limit above is violated */
  MOE_ERR_WORKSPACE_TOO_SMALL = -3, /* ws_bytes < moe_workspace_bytes(shape) */
  MOE_ERR_MISALIGNED = -4,          /* a pointer breaks the alignment rules */
  MOE_ERR_CUDA = -5,                /* a CUDA runtime call failed (includes earlier faults) */
  MOE_ERR_TIMEOUT = -6,             /* a kernel's bounded wait gave up; see moe_device_status */
  MOE_ERR_NO_DEVICE = -7,           /* current device is not an sm_100 GPU */
  MOE_ERR_NOALLOC_LIMIT = -8,       /* moe_plan_noalloc: shape needs more than its static scratch */
  MOE_ERR_BOUNDS = -9               /* MOE_FLAG_DEBUG_BOUNDS: a plan index was out of range, or a
                                       workspace guard was overwritten; see moe_device_status */
} moe_status;

/* moe_shape_t.flags */
#define MOE_FLAG_RENORM_TOPK 1u     /* divide the k selected gates of a token by their sum */
/* Launch schedule of moe_forward (results are identical; only the overlap of rounds differs).
 * Default: the trailing run of thin rounds (whose gate/up GEMM has fewer 128-row x 128-column
 * tiles than the GPU has SMs) runs in one pipelined launch, the rounds before it as per-round
 * launches. The pipelined launch
 * alternates two sets of round buffers, so the workspace holds a second set unless
 * MOE_FLAG_PER_ROUND is given. */
#define MOE_FLAG_PER_ROUND 2u       /* every round as per-round launches; moe_backward runs its
                                       rounds one after another on `stream`, without the second
                                       buffer set of its workspace (same results) */
#define MOE_FLAG_PIPELINE_ALL 4u    /* every round in the pipelined launch */
/* Capacity borrowing ("Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims,
 * multi-round dropless MoE item: overflow tokens use unused capacity of other experts of the
 * group, otherwise an extra round). Each round still holds at most E*C rows (the same fixed
 * buffers), but an overloaded expert takes the rows other experts leave unused: every expert
 * first takes up to C of its pending pairs, then the unused rows go to experts with pairs
 * pending, in ascending expert index. An expert may then hold more than C rows of a round, so
 * the round's rows are packed expert after expert (pair (e, slot) of round r at buffer row
 * row_off[r][e] - row_start[r] + slot, the layout's row lists) and `slot` counts from 0 within
 * the expert's rows of the round, up to n[r][e]-1. R never exceeds ceil(max_load / C) and is
 * 1 whenever T*k <= E*C. Runs as per-round launches (not with MOE_FLAG_PIPELINE_ALL); y is the
 * same layer output. Off by default: the default plan is R = ceil(max_load / C). */
#define MOE_FLAG_BORROW 8u
/* Debug bounds checks, a stand-in for a memory checker (off by default; slower). With this flag:
 *   - the calls that run a plan first check its summary on the host (loads non-negative, at most
 *     T and adding up to T*k, max_load their maximum, R the round count of those loads) and return
 *     MOE_ERR_INVALID_ARG, launching nothing, when it cannot be the planner's;
 *   - the planner, dispatch, combine and the GEMMs check every plan index before they use it
 *     (expert < E, round < the workspace's rounds, row-list position < T*k, source token < T,
 *     buffer row < E*C, rows of an expert in a round <= C, or <= E*C with MOE_FLAG_BORROW); a
 *     failed check is recorded in the workspace header and the access is skipped, never trapped;
 *   - the workspace holds a 256-byte guard after every region (moe_workspace_bytes grows by
 *     256 bytes per region), which moe_plan fills and moe_device_status verifies;
 *   - moe_forward runs every round as per-round launches (not with MOE_FLAG_PIPELINE_ALL);
 *   - moe_device_status returns MOE_ERR_BOUNDS after a failed check or a changed guard.
 * Results are bit-identical to the per-round schedule without the flag. The backward pass and
 * moe_plan_noalloc do not check. */
#define MOE_FLAG_DEBUG_BOUNDS 16u

#define MOE_MAX_EXPERTS 256
#define MOE_MAX_TOPK 16

/* Layer shape. T tokens, hidden size d, E experts, top-k, SwiGLU inner size d_ff,
 * per-expert capacity C of one round (the pages' tunable capacity). */
typedef struct moe_shape {
  int32_t T, d, E, k, d_ff, C;
  uint32_t flags;
} moe_shape_t;

/* Host-side result of moe_plan(). Caller-owned; pass it unchanged to the calls that
 * execute that plan on the same workspace. The device pointers point into the workspace. */
typedef struct moe_plan_info {
  int32_t R;                        /* number of rounds = ceil(max_load / C); 0 if T == 0 */
  int32_t max_load;                 /* largest number of tokens routed to one expert */
  int32_t load[MOE_MAX_EXPERTS];    /* tokens routed to each expert (first E entries) */
  const float* logits;              /* [T, E] fp32 logits the plan used (caller's or computed) */
  const int32_t* topk_idx;          /* [T, k] selected experts, best first */
  const float* gate;                /* [T, k] gates */
  const int32_t* round;             /* [T, k] round of each (token, expert) pair */
  const int32_t* slot;              /* [T, k] row of the pair inside its expert's C rows */
  const int32_t* offsets;           /* [E + 1] exclusive prefix sum of load */
  const int32_t* n;                 /* [max_rounds, E] rows of expert e in round r */
  uint32_t plan_flags;              /* the shape flags that decide the plan (MOE_FLAG_BORROW);
                                       calls that run the plan reject a shape whose flags differ */
} moe_plan_info_t;

/* Byte offsets of the sub-buffers inside the workspace (all 256-byte aligned). */
typedef struct moe_workspace_layout {
  size_t total_bytes;
  size_t header;      /* int32[64]: R, max_load, status word, ... */
  size_t logits;      /* f32 [T, E]   logits from the router GEMM */
  size_t topk_idx;    /* i32 [T, k] */
  size_t gate;        /* f32 [T, k] */
  size_t round;       /* i32 [T, k] */
  size_t slot;        /* i32 [T, k] */
  size_t load;        /* i32 [E] */
  size_t offsets;     /* i32 [E + 1] */
  size_t block_base;  /* i32 [plan_blocks, E] planner scratch: per-block per-expert counts */
  size_t n;           /* i32 [max_rounds, E] rows of expert e in round r */
  size_t row_off;     /* i32 [max_rounds, E] first row of (round r, expert e) in the row list */
  size_t row_start;   /* i32 [max_rounds + 1]: first row of round r in the round-major row list */
  size_t row_token;   /* i32 [T * k] round-major row list: source token */
  size_t row_dst;     /* i32 [T * k] round-major row list: destination e * C + slot */
  size_t buf;         /* bf16 [E, C, d]: dispatch buffer of the round */
  size_t h;           /* bf16 [E, C, d_ff]: SwiGLU activations of the round */
  size_t out;         /* bf16 [E, C, d]: expert outputs of the round */
  size_t mb_prefix;   /* i32 [max_rounds, E + 1]: 128-row blocks of experts < e in round r */
  size_t sync;        /* i32 [448 + 64 * E * ceil(C / 128)]: pipelined launch's dependency
                         counters (zero between calls) */
  size_t buf2;        /* second buffer set of the pipelined launch (rounds alternate sets); */
  size_t h2;          /* absent (0) with MOE_FLAG_PER_ROUND, which never uses it */
  size_t out2;
  int32_t max_rounds; /* ceil(T / C): no expert can receive more than T tokens */
  int32_t plan_blocks;
} moe_workspace_layout_t;

/* Bytes of device workspace for `shape`. Depends on the shape only, never on the
 * routing: this is the layer's fixed memory. Returns 0 for an invalid shape. */
MOE_API size_t moe_workspace_bytes(const moe_shape_t* shape);

/* Fills *layout for `shape`. Returns MOE_OK or MOE_ERR_UNSUPPORTED_SHAPE / INVALID_ARG. */
MOE_API int moe_workspace_layout(const moe_shape_t* shape, moe_workspace_layout_t* layout);

/* Router + round planner.
 *   logits   [T, E] fp32, or NULL to compute logits = x @ w_router^T + bias on tensor cores;
 *   x        [T, d] bf16 (needed only when logits == NULL);
 *   w_router [E, d] bf16 (nn.Linear layout; needed only when logits == NULL);
 *   bias     [E] fp32 or NULL (used only when logits == NULL).
 * Writes topk/gate/round/slot/load/offsets/n and the round-major row list into `ws`,
 * then synchronizes `stream` once and fills *info (R, max_load, load[], device pointers).
 * The summary (1280 bytes) comes home through pinned host memory mapped into the device,
 * written by a one-block kernel rather than by a copy engine, so that a large device-to-host
 * copy the caller has in flight on another stream does not delay moe_plan until it ends. That
 * buffer is allocated on the first call of each host thread on each device and kept for the
 * thread's lifetime; if it cannot be allocated, moe_plan copies with cudaMemcpyAsync instead.
 * Non-finite logits give undefined routing. */
MOE_API int moe_plan(const moe_shape_t* shape, const float* logits, const uint16_t* x,
             const uint16_t* w_router, const float* bias, void* ws, size_t ws_bytes,
             moe_plan_info_t* info, moe_stream_t stream);

/* Executes all R rounds of the plan in `info` (from moe_plan on this `ws`).
 * Per-round launches (programmatic dependent launch): per round the gate/up and the down GEMM;
 * a thin round's dispatch and combine ride on the neighbouring GEMM launches (extra warps), a
 * large round's get their own kernels. Pipelined launch: one persistent cooperative kernel (one
 * CTA per SM) runs a run of rounds, their dispatch, GEMM tiles and combine overlapping under
 * dependency counters kept in the workspace; a wait that exceeds 2 s sets the status word
 * (moe_device_status) and the launch unwinds. shape->flags choose the schedule. Arguments:
 *   x         [T, d] bf16
 *   w_gate_up [E, 2*d_ff, d] bf16: rows 0..d_ff-1 = W1 (gate), rows d_ff..2*d_ff-1 = W3 (up)
 *   w_down    [E, d, d_ff] bf16 (W2)
 *   y         [T, d] fp32 output; every row is written (rows of tokens with pairs are
 *             overwritten on their first round; T*k >= T pairs means every token has one).
 * Asynchronous: no synchronization. */
MOE_API int moe_forward(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws, size_t ws_bytes,
                const uint16_t* x, const uint16_t* w_gate_up, const uint16_t* w_down, float* y,
                moe_stream_t stream);

/* The four steps of round r (0 <= r < info->R), as moe_forward runs them. Exposed so that
 * each kernel can be checked and timed on its own; call them in this order per round.
 *   dispatch: buf[e][s] = x[token] for the round's rows (bf16 copy)
 *   gate_up:  h[e][s] = bf16(silu(buf[e][s] W1_e^T) * (buf[e][s] W3_e^T)) for s < n[r][e]
 *   down:     out[e][s] = bf16(h[e][s] W2_e^T) for s < n[r][e]
 *   combine:  y[t] = (t's first round ? 0 : y[t]) + sum_{j ascending, round(t,j)=r} gate*out */
MOE_API int moe_round_dispatch(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws,
                       size_t ws_bytes, int32_t r, const uint16_t* x, moe_stream_t stream);
MOE_API int moe_round_gate_up(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws,
                      size_t ws_bytes, int32_t r, const uint16_t* w_gate_up, moe_stream_t stream);
MOE_API int moe_round_down(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws,
                   size_t ws_bytes, int32_t r, const uint16_t* w_down, moe_stream_t stream);
MOE_API int moe_round_combine(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws,
                      size_t ws_bytes, int32_t r, float* y, moe_stream_t stream);

/* ---------------------------------------------------------------- backward pass
 *
 * "Microsoft AI's MAI-Base-2 trained on 16K GPUs with Muon", section "Expert groups keep
 * memory fixed when tokens pile up": the backward pass recomputes each expert group on the
 * forward's round schedule, so its memory is as static as the forward's. moe_backward runs
 * the R rounds of the plan in `info` again: per round it re-dispatches the round's x rows and
 * dy rows, recomputes the SwiGLU pre-activations on the tensor cores, and adds the round's
 * weight gradients into the caller's fp32 gradients; nothing it holds grows with the routing.
 *
 * Its own workspace `bws` (device, caller-owned, 256-byte aligned) holds the per-round buffers;
 * its size depends on the shape only. Weights and activations are read as they are stored: the
 * GEMMs that need an operand transposed load it MN-major, so no transposed copy is made. */
typedef struct moe_backward_layout {
  size_t total_bytes;
  /* The per-round buffers have `rows` rows: E * C, expert e's rows of the round at e * C + slot;
     with MOE_FLAG_BORROW E * C + 64 * E, expert e's rows at the round's seg_off[r][e] + slot,
     where each expert's segment starts at a multiple of 64 rows (the experts' rows rounded up to
     64, in expert order). Rows from an expert's count up to the next multiple of 64 (within its
     C rows, or within its segment) hold zeros in xbuf, dybuf, hg and dab: the weight-gradient
     GEMMs read K, the rows, in blocks of 64. */
  size_t xbuf;        /* bf16 [rows, d]      the round's x rows */
  size_t dybuf;       /* bf16 [rows, d]      the round's dy rows */
  size_t row_gate;    /* f32  [rows]         the gate of the pair in each row */
  size_t ab;          /* bf16 [rows, 2 d_ff] recomputed a = W1 x, b = W3 x */
  size_t hg;          /* bf16 [rows, d_ff]   gate * silu(a) * b */
  size_t dab;         /* bf16 [rows, 2 d_ff] [da | db] */
  size_t dgate_part;  /* f32  [rows, d_ff / 64] per-tile partial sums of dgate */
  size_t dxbuf;       /* bf16 [rows, d]      per-pair dx rows of the round */
  size_t dgate;       /* f32  [T, k]         dL/dgate */
  size_t ones;        /* f32  [T, k]         unit gates of the dx combine */
  size_t seg_off;     /* i32  [max_rounds, E] first row of each expert's segment in pooled rows */
  size_t zeros;       /* i32  [max_rounds + 1] zeros (row offsets of the segment tables) */
  int32_t rows;       /* rows of the per-round buffers (above) */
  /* A second, smaller set of the per-round buffers, laid out like the first but with rows2 =
     E * C / 8 (rounded up to 64) + 64 * E rows, always pooled (expert e's rows of the round at
     seg_off[r][e] + slot). A round whose pooled rows fit runs in it when the round before ran in
     the first set, so that its dispatch, recompute and dh overlap that round's dx, weight
     gradients and combine (unless MOE_FLAG_PER_ROUND). */
  size_t xbuf2, dybuf2, row_gate2, ab2, hg2, dab2, dgate_part2, dxbuf2;
  int32_t rows2;
} moe_backward_layout_t;

/* Bytes of the backward workspace for `shape` (0 for an invalid shape). */
MOE_API size_t moe_backward_workspace_bytes(const moe_shape_t* shape);
MOE_API int moe_backward_workspace_layout(const moe_shape_t* shape, moe_backward_layout_t* layout);

/* Gradients of the layer output y (moe_forward with the same plan, inputs and weights) given
 * dy = dL/dy:
 *   dx         [T, d] fp32 out: through the experts (the router's share, dz W_r, is the
 *              caller's: dz is returned for it)
 *   dw_gate_up [E, 2*d_ff, d] fp32 out (overwritten), same row order as w_gate_up
 *   dw_down    [E, d, d_ff] fp32 out (overwritten)
 *   dz         [T, E] fp32 out: dL/dlogits through the softmax gates of info->logits (the
 *              top-k selection passes no gradient)
 * ws holds the plan (moe_plan) and is only read, except for its status word; x, w_gate_up,
 * w_down as in moe_forward; dy [T, d] fp32. Operands of the tensor-core steps are bf16 (dy, a,
 * b, gate * h, da, db rounded to bf16) with fp32 accumulation. Plans made with MOE_FLAG_BORROW
 * run on their pooled round rows. A bounded wait that gives up sets the status word
 * (moe_device_status). Asynchronous: no synchronization. Thin rounds overlap the round before
 * them: their dispatch, recompute and dh run on `stream` while the round before's dx, weight
 * gradients and combine run on a second stream of the library's (one per host thread and
 * device, created on first use), joined back to `stream` before the call's last launch; the
 * results are those of one round at a time, bit for bit. */
MOE_API int moe_backward(const moe_shape_t* shape, const moe_plan_info_t* info, void* ws, size_t ws_bytes,
                         void* bws, size_t bws_bytes, const uint16_t* x, const uint16_t* w_gate_up,
                         const uint16_t* w_down, const float* dy, float* dx, float* dw_gate_up,
                         float* dw_down, float* dz, moe_stream_t stream);

/* Synchronizes `stream` and reads the workspace status word that kernels set when a
 * bounded wait gives up. With MOE_FLAG_DEBUG_BOUNDS it first verifies the workspace guards.
 * Returns MOE_OK, MOE_ERR_TIMEOUT, MOE_ERR_BOUNDS or MOE_ERR_CUDA. */
MOE_API int moe_device_status(const moe_shape_t* shape, void* ws, moe_stream_t stream);

/* Human-readable text for a moe_status value (static storage). */
MOE_API const char* moe_status_string(int status);

/* Number of kernels this library has launched in this process (for accounting). */
MOE_API uint64_t moe_launch_count(void);

/* Per-kernel timing with CUDA events. While enabled, every launch made by the calls above
 * is bracketed by two events on its stream; moe_profile_read() synchronizes on them and
 * reports, per kernel kind, the launch count and the summed milliseconds. Kinds:
 * 0 router GEMM, 1 top-k, 2 plan, 3 dispatch, 4 gate_up GEMM, 5 down GEMM, 6 combine,
 * 7 pipelined rounds (all four steps of its rounds in one launch); backward: 8 recompute GEMM,
 * 9 dh GEMM (with the SwiGLU backward), 10 dx and weight-gradient GEMMs (one launch a round),
 * 11 its other launches (gather, dx combine, gate gradient, segment table, fills), 12 recompute
 * and dh GEMMs in one launch (rounds whose GEMMs run in the single-CTA form).
 * Up to 4096 launches are recorded between enable and read. Not thread-safe. */
#define MOE_PROFILE_KINDS 13
MOE_API int moe_profile_enable(int on);
MOE_API int moe_profile_read(int32_t counts[MOE_PROFILE_KINDS], double ms[MOE_PROFILE_KINDS]);

/* ---------------------------------------------------------------- expert parallelism
 *
 * "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, the multi-round dropless
 * MoE item [section "Scaling MoE", Fig. 6]: the experts are split into groups, one group per
 * expert-parallel rank, and every group runs dispatch -> compute -> collect rounds with a fixed
 * per-expert capacity; the token metadata stays on the device. Over G ranks, rank g owns the
 * E/G contiguous experts [g E/G, (g+1) E/G). An expert's capacity C per round is shared by all
 * source ranks, which fill it in (source rank, token) order: the job's plan is the single-GPU
 * plan of the ranks' batches concatenated in rank order, and every rank runs the same
 * R = ceil(max_e total_e / C) rounds. In round r, rank s sends rank g its pairs of round r
 * whose expert g owns, in (expert, slot) order; rank g receives the chunks in source order.
 *
 * Exchange tables of rank `rank` from the pair counts of every rank. Host code only: no CUDA
 * call, no device memory; every rank computes its own tables from the same all-gathered counts.
 *   shape      this rank's layer shape (T = this rank's tokens; E, k, C as on every rank)
 *   loads      host in [G, E]: loads[s][e] = pairs of rank s routed to expert e (this rank's
 *              row must add up to T * k)
 *   max_rounds rows of the per-round arrays below
 *   R          host out: rounds of the job (filled even when it exceeds max_rounds)
 *   base       host out [E] or NULL: pairs of expert e on the ranks before this one (this rank's
 *              pairs of e hold the global ranks base[e] .. base[e] + loads[rank][e] - 1)
 *   send_counts, send_offsets  host out [max_rounds, G] or NULL: rows this rank sends rank g
 *              in round r, and their position in its packed round-r rows (exclusive prefix)
 *   recv_counts, recv_offsets  host out [max_rounds, G] or NULL: rows this rank receives from
 *              rank s in round r, and their position in its received rows (exclusive prefix)
 *   n_owned    host out [max_rounds, E / G] or NULL: rows of each expert this rank owns in
 *              round r, from all ranks (at most C)
 * Returns MOE_ERR_INVALID_ARG for G < 1, E not a multiple of G, a rank out of range, a
 * negative count, this rank's counts not adding up to T * k, or R > max_rounds with an
 * array to fill. */
MOE_API int moe_ep_exchange_plan(const moe_shape_t* shape, int32_t G, int32_t rank, const int32_t* loads,
                                 int32_t max_rounds, int32_t* R, int32_t* base, int32_t* send_counts,
                                 int32_t* send_offsets, int32_t* recv_counts, int32_t* recv_offsets,
                                 int32_t* n_owned);

/* Device data path of the expert-parallel layer, one round at a time (same sources and
 * readings as moe_ep_exchange_plan above). Every rank holds T tokens. Per round r, each rank:
 *   moe_ep_round_pack:     its pairs of round r, in (expert, slot) order, x rows -> sendbuf; the
 *                          rows for owner g are the chunk at send_offsets[r][g] (send_counts)
 *   (the caller's all-to-all: chunk g of every rank's sendbuf -> rank g's recvbuf, in source order)
 *   moe_ep_round_experts:  on the owner, both grouped GEMMs straight over the received rows, one
 *                          group per (source rank, local expert): h = bf16(silu(recv W1^T) *
 *                          (recv W3^T)), out = bf16(h W2^T), out in the order of recvbuf
 *   (the all-to-all back: chunk s of out -> rank s's retbuf)
 *   moe_ep_round_combine:  y[t] (+)= gate * retbuf row for its pairs of round r, j ascending
 * The rank's plan comes from moe_plan on its own tokens (without MOE_FLAG_BORROW) followed by
 * moe_ep_plan, which re-ranks every pair among all ranks' pairs of its expert. Buffers (device,
 * caller-owned, bf16, 16-byte aligned): sendbuf and retbuf hold min(T*k, E*C) rows of d; recvbuf
 * and out hold buf_rows >= E/G * C rows of d, h buf_rows rows of d_ff. loads is the host [G, E]
 * table of every rank's pair counts (all-gathered), the same on every rank.
 *
 * Bytes of the plan tables of one rank over G ranks (0 for an invalid shape or G). */
MOE_API size_t moe_ep_workspace_bytes(const moe_shape_t* shape, int32_t G);
/* Re-plans this rank's pairs (info/ws from moe_plan on this rank's tokens): global round, slot
 * within the rank's rows of (round, expert), packed row list. R: host out, the job's rounds.
 * Synchronizes `stream` once. MOE_ERR_INVALID_ARG if loads do not match info's loads, a rank
 * holds more than T tokens, or the plan used borrowing. */
MOE_API int moe_ep_plan(const moe_shape_t* shape, int32_t G, int32_t rank, const int32_t* loads,
                        const moe_plan_info_t* info, void* ws, size_t ws_bytes, void* ep_ws, size_t ep_bytes,
                        int32_t* R, moe_stream_t stream);
MOE_API int moe_ep_round_pack(const moe_shape_t* shape, int32_t G, int32_t rank, const int32_t* loads,
                              void* ep_ws, size_t ep_bytes, int32_t r, const uint16_t* x, uint16_t* sendbuf,
                              moe_stream_t stream);
/* w_gate_up [E/G, 2*d_ff, d] and w_down [E/G, d, d_ff]: this rank's own experts. ws: this rank's
 * workspace (its status word records bounded-wait time-outs). Synchronizes `stream` once. */
MOE_API int moe_ep_round_experts(const moe_shape_t* shape, int32_t G, int32_t rank, const int32_t* loads,
                                 void* ep_ws, size_t ep_bytes, int32_t r, const uint16_t* recvbuf,
                                 const uint16_t* w_gate_up, const uint16_t* w_down, uint16_t* h, uint16_t* out,
                                 int64_t buf_rows, void* ws, moe_stream_t stream);
MOE_API int moe_ep_round_combine(const moe_shape_t* shape, int32_t G, int32_t rank, const int32_t* loads,
                                 void* ws, size_t ws_bytes, void* ep_ws, size_t ep_bytes, int32_t r,
                                 const uint16_t* retbuf, float* y, moe_stream_t stream);

/* Routing and round plan with no device allocation at all.
 *
 * The pages have no counterpart to this call; it exists for callers that cannot
 * allocate device memory when they route a batch: code running under a memory pool
 * that already owns the device, plugins that a host framework hands only their input
 * and output buffers, or services that forbid cudaMalloc after start-up. moe_plan()
 * needs a caller-allocated workspace; this call keeps the planner's scratch in one
 * static device array of MOE_NOALLOC_SCRATCH_BYTES inside the library instead. A GPU
 * holds that array from the moment it loads the library's code (its first
 * moe_plan_noalloc() call under lazy module loading) until the process exits.
 *
 *   logits   [T, E] fp32 device input (the router-GEMM form is not offered here);
 *   topk_idx [T, k] int32, gate [T, k] fp32, round [T, k] int32, slot [T, k] int32:
 *            device outputs, identical to what moe_plan() writes into its workspace;
 *   R        host out: the number of rounds; load: host out [E] (may be NULL).
 * Returns MOE_ERR_NOALLOC_LIMIT, launching nothing, when the shape's scratch
 * (about 8*T*k + 8*ceil(T/C)*E + 4*ceil(T/256)*E bytes) exceeds the array. Calls no
 * cudaMalloc, cudaFree or other allocating routine. Every call looks up the array's
 * device address (cudaGetSymbolAddress) on the current device. Under CUDA's lazy module
 * loading (the default) that lookup is also what makes the device reserve the array, so
 * the FIRST call on each device may need 16 MiB of free device memory: make one call per
 * device at start-up (T = 0 will do), before a memory pool takes the device and before
 * any stream capture. All calls share the array and each one clears what must start at
 * zero, but calls whose GPU work overlaps (other streams, other threads) race on it.
 * Synchronizes `stream` once, like moe_plan(). */
#define MOE_NOALLOC_SCRATCH_BYTES (16u << 20)
MOE_API int moe_plan_noalloc(const moe_shape_t* shape, const float* logits, int32_t* topk_idx,
                             float* gate, int32_t* round, int32_t* slot, int32_t* R,
                             int32_t* load, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DROPLESS_MOE_H_ */
