// Expert-parallel exchange plan (host only): where every rank's kept
// dispatches land in each expert owner's receive buffer, and back.
//
// R ranks, N experts, expert e on rank e / (N / R).  The capacity of an
// expert counts the dispatches of all ranks in one global order (rank 0's
// tokens first, then rank 1's, each in token order), so the expert-parallel
// layer equals the single-device layer of "Mixture of Experts MoE: how sparse
// activation saves compute" (§3.5, §3.6, §3.8) on the ranks' batches laid end
// to end.  From the R x N dispatch counts every rank derives the same plan
// with no further communication.
#include <cstdint>
#include <vector>

#include "common.cuh"

extern "C" int moe_ep_plan(int32_t world, int32_t rank, int32_t N, int32_t capacity,
                           const int32_t* counts_all, int32_t* kept, int32_t* local_offsets,
                           int32_t* send_base, int32_t* send_counts, int32_t* recv_offsets,
                           int32_t* recv_src_base, int32_t* recv_counts, int32_t* overflow) {
  if (world < 1 || N < 1 || N % world != 0 || rank < 0 || rank >= world || capacity < 0)
    return MOE_ERR_INVALID_ARG;
  if (!counts_all || !kept || !local_offsets || !send_base || !send_counts || !recv_offsets ||
      !recv_src_base || !recv_counts)
    return MOE_ERR_INVALID_ARG;
  const int64_t R = world, E = N / world;
  for (int64_t i = 0; i < R * N; ++i)
    if (counts_all[i] < 0) return MOE_ERR_INVALID_ARG;
  // kept[r][e]: rank r's share of expert e's capacity, after the ranks before it
  std::vector<int64_t> kept_all((size_t)(R * N)), kept_before((size_t)(R * N));
  std::vector<int64_t> kept_tot((size_t)N, 0);
  for (int64_t e = 0; e < N; ++e) {
    int64_t before = 0, kbefore = 0;
    for (int64_t r = 0; r < R; ++r) {
      const int64_t c = counts_all[r * N + e];
      int64_t k = c;
      if (capacity > 0) {
        const int64_t room = (int64_t)capacity - before;
        k = room <= 0 ? 0 : (room < c ? room : c);
      }
      kept_all[(size_t)(r * N + e)] = k;
      kept_before[(size_t)(r * N + e)] = kbefore;
      before += c;
      kbefore += k;
    }
    kept_tot[(size_t)e] = kbefore;
    if (overflow) {
      const int64_t dropped = before - kbefore;
      if (dropped > INT32_MAX) return MOE_ERR_INVALID_ARG;
      overflow[e] = (int32_t)dropped;
    }
  }
  // first row of expert e in its owner's receive buffer (the owner's experts in order)
  std::vector<int64_t> expert_base((size_t)N);
  for (int64_t o = 0; o < R; ++o) {
    int64_t run = 0;
    for (int64_t e = o * E; e < (o + 1) * E; ++e) {
      expert_base[(size_t)e] = run;
      run += kept_tot[(size_t)e];
    }
    if (run > INT32_MAX) return MOE_ERR_INVALID_ARG;
  }
  int64_t run = 0;
  for (int64_t e = 0; e < N; ++e) {
    const int64_t k = kept_all[(size_t)(rank * N + e)];
    kept[e] = (int32_t)k;
    local_offsets[e] = (int32_t)run;
    run += k;
    send_base[e] = (int32_t)(expert_base[(size_t)e] + kept_before[(size_t)(rank * N + e)]);
  }
  if (run > INT32_MAX) return MOE_ERR_INVALID_ARG;
  local_offsets[N] = (int32_t)run;
  for (int64_t o = 0; o < R; ++o) {
    int64_t sent = 0;
    for (int64_t e = o * E; e < (o + 1) * E; ++e) sent += kept_all[(size_t)(rank * N + e)];
    send_counts[o] = (int32_t)sent;
  }
  run = 0;
  for (int64_t el = 0; el < E; ++el) {
    const int64_t e = rank * E + el;
    recv_offsets[el] = (int32_t)run;
    run += kept_tot[(size_t)e];
    for (int64_t r = 0; r < R; ++r)
      recv_src_base[el * R + r] =
          (int32_t)(expert_base[(size_t)e] + kept_before[(size_t)(r * N + e)]);
  }
  recv_offsets[E] = (int32_t)run;
  for (int64_t r = 0; r < R; ++r) {
    int64_t got = 0;
    for (int64_t el = 0; el < E; ++el) got += kept_all[(size_t)(r * N + rank * E + el)];
    recv_counts[r] = (int32_t)got;
  }
  return MOE_OK;
}
