// Expert-parallel exchange plan (host code only; no device work).
//
// "Scaling with experts" (jeff-ong.com), What you still pay for: with the
// experts partitioned over devices, a token travels to the device holding its
// assigned expert and the expert's output travels back.  Zen MoDE §7.2
// Communication Overhead (Distributed Training): that routing is an
// all-to-all exchange between the expert devices.
//
// Rank q of G holds the global experts [q*E_l, (q+1)*E_l), E_l = E/G.  Every
// rank routes and dispatches its own tokens exactly as a single device would
// (so its capacity cut and statistics are its own batch's), which leaves the
// kept rows of global expert e at x_perm[seg_off[e] .. seg_off[e+1]): the rows
// for the experts of peer q are ONE contiguous block of x_perm.  So the plan is
//   - one send chunk per peer (that block),
//   - one receive chunk per source rank, the blocks laid end to end in rank
//     order (source-major), and
//   - G * E_l row segments over that buffer, segment s*E_l + el holding source
//     s's rows for local expert el, which the grouped expert GEMM runs as
//     they lie (moe_expert_ffn_segments: segment i uses expert i % E_l).
// The return trip is the same table read backwards.  One message each way
// per pair of ranks.

#include <cstdint>

#include "../../include/moe_b200.h"

extern "C" int moe_ep_plan(int32_t n_ranks, int32_t rank, int32_t n_experts, const int32_t* seg_off_all,
                           int32_t* send, int32_t* recv, int32_t* local_seg_off) {
  if (n_ranks < 1 || n_experts < 1 || rank < 0 || rank >= n_ranks || n_experts % n_ranks != 0)
    return MOE_ERR_INVALID_ARG;
  if (!seg_off_all || !send || !recv || !local_seg_off) return MOE_ERR_INVALID_ARG;
  const int G = n_ranks, E = n_experts, El = E / G;
  // every rank's offsets must start at 0 and never decrease
  for (int s = 0; s < G; ++s) {
    const int32_t* so = seg_off_all + static_cast<int64_t>(s) * (E + 1);
    if (so[0] != 0) return MOE_ERR_INVALID_ARG;
    for (int e = 0; e < E; ++e)
      if (so[e + 1] < so[e]) return MOE_ERR_INVALID_ARG;
  }
  const int32_t* mine = seg_off_all + static_cast<int64_t>(rank) * (E + 1);
  for (int q = 0; q < G; ++q) {
    send[3 * q + 0] = q;
    send[3 * q + 1] = mine[q * El];
    send[3 * q + 2] = mine[(q + 1) * El] - mine[q * El];
  }
  int64_t off = 0;
  for (int s = 0; s < G; ++s) {
    const int32_t* so = seg_off_all + static_cast<int64_t>(s) * (E + 1);
    const int32_t first = so[rank * El];
    recv[3 * s + 0] = s;
    recv[3 * s + 1] = static_cast<int32_t>(off);
    recv[3 * s + 2] = so[(rank + 1) * El] - first;
    for (int el = 0; el < El; ++el) {
      local_seg_off[s * El + el] = static_cast<int32_t>(off + (so[rank * El + el] - first));
    }
    off += so[(rank + 1) * El] - first;
    if (off > INT32_MAX) return MOE_ERR_INVALID_ARG;
  }
  local_seg_off[G * El] = static_cast<int32_t>(off);
  return MOE_OK;
}
