// ep_plan.cu - exchange tables of the expert-parallel form of the layer (host code only).
//
// "Frontier Pre-training at Microsoft AI (MAI-Base-2)", Key claims, the multi-round dropless
// MoE item [section "Scaling MoE", Fig. 6]: the experts are split into groups, one group per
// expert-parallel rank, and every group runs dispatch -> compute -> collect rounds with a
// fixed per-expert capacity, its token metadata resident on the device. Here rank g owns the
// E/G contiguous experts [g E/G, (g+1) E/G). An expert's capacity C per round is shared by
// every rank that sends to it, and its pairs are taken in (source rank, token) order, so the
// job's plan is the single-GPU plan of the ranks' batches concatenated in rank order.
//
// Once every rank knows every rank's per-expert pair counts (one all-gather of G x E
// integers), each rank derives all the tables of the exchange by itself, with no further
// communication: rank s's pairs of expert e hold the global ranks [base_s[e], base_s[e] +
// load_s[e]) with base_s[e] = sum of load_s'[e] over s' < s, so their rows in round r are that
// range cut by [r C, (r+1) C). Integer work, identical on every rank.
#include <cstdint>
#include <cstring>
#include <vector>

#include "moe.h"

namespace {

int64_t overlap(int64_t lo, int64_t hi, int64_t a, int64_t b) {
  const int64_t l = lo > a ? lo : a, h = hi < b ? hi : b;
  return h > l ? h - l : 0;
}

}  // namespace

extern "C" MOE_API int moe_ep_exchange_plan(const moe_shape_t* shape, int32_t G, int32_t rank,
                                            const int32_t* loads, int32_t max_rounds, int32_t* R,
                                            int32_t* base, int32_t* send_counts, int32_t* send_offsets,
                                            int32_t* recv_counts, int32_t* recv_offsets, int32_t* n_owned) {
  if (shape == nullptr || loads == nullptr || R == nullptr) return MOE_ERR_INVALID_ARG;
  if (moe_workspace_bytes(shape) == 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  const int E = shape->E, C = shape->C;
  if (G < 1 || E % G != 0 || rank < 0 || rank >= G || max_rounds < 0) return MOE_ERR_INVALID_ARG;
  const int per = E / G;
  // every count is a pair count; this rank's add up to its T k pairs
  int64_t mine = 0;
  std::vector<int64_t> total(E, 0), base_all(static_cast<size_t>(G) * E, 0);
  for (int s = 0; s < G; ++s)
    for (int e = 0; e < E; ++e) {
      const int32_t v = loads[static_cast<size_t>(s) * E + e];
      if (v < 0) return MOE_ERR_INVALID_ARG;
      base_all[static_cast<size_t>(s) * E + e] = total[e];
      total[e] += v;
      if (s == rank) mine += v;
    }
  if (mine != static_cast<int64_t>(shape->T) * shape->k) return MOE_ERR_INVALID_ARG;
  int64_t max_total = 0;
  for (int e = 0; e < E; ++e) max_total = total[e] > max_total ? total[e] : max_total;
  const int64_t rounds = (max_total + C - 1) / C;
  if (rounds > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  *R = static_cast<int32_t>(rounds);
  if (base)
    for (int e = 0; e < E; ++e) {
      if (base_all[static_cast<size_t>(rank) * E + e] > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
      base[e] = static_cast<int32_t>(base_all[static_cast<size_t>(rank) * E + e]);
    }
  if (rounds > max_rounds) return (send_counts || send_offsets || recv_counts || recv_offsets || n_owned)
                                      ? MOE_ERR_INVALID_ARG : MOE_OK;
  for (int64_t r = 0; r < rounds; ++r) {
    const int64_t lo = r * C, hi = lo + C;
    int64_t s_run = 0, r_run = 0;
    for (int g = 0; g < G; ++g) {
      // this rank's rows of round r for owner g
      int64_t out = 0;
      for (int e = g * per; e < (g + 1) * per; ++e) {
        const int64_t b = base_all[static_cast<size_t>(rank) * E + e];
        out += overlap(lo, hi, b, b + loads[static_cast<size_t>(rank) * E + e]);
      }
      // rows of source rank g for the experts this rank owns
      int64_t in = 0;
      for (int e = rank * per; e < (rank + 1) * per; ++e) {
        const int64_t b = base_all[static_cast<size_t>(g) * E + e];
        in += overlap(lo, hi, b, b + loads[static_cast<size_t>(g) * E + e]);
      }
      const size_t at = static_cast<size_t>(r) * G + g;
      if (send_counts) send_counts[at] = static_cast<int32_t>(out);
      if (send_offsets) send_offsets[at] = static_cast<int32_t>(s_run);
      if (recv_counts) recv_counts[at] = static_cast<int32_t>(in);
      if (recv_offsets) recv_offsets[at] = static_cast<int32_t>(r_run);
      s_run += out;
      r_run += in;
    }
    if (n_owned)
      for (int l = 0; l < per; ++l) {
        const int64_t rem = total[rank * per + l] - lo;
        n_owned[static_cast<size_t>(r) * per + l] = static_cast<int32_t>(rem <= 0 ? 0 : rem >= C ? C : rem);
      }
  }
  return MOE_OK;
}
