// Runtime load balancing of heads (FVAttn blog summary, section "RLB：不搞全局重洗，只做P2P
// “微创手术”，修复临界路径"): the host-side greedy migration plan, and the device step that
// restricts the attention to the heads a rank keeps.
//
// The plan: with the per-head loads (selected block pairs) of every rank gathered, repeatedly
// take the most loaded rank as the sender and the least loaded as the receiver, and move the
// sender's heaviest head whose move keeps the receiver below the sender, until max / mean of
// the rank loads is at most the target or the sender has used its migration budget. Ties go
// to the lower rank / head index; a head moves at most once.
#include <math.h>
#include <stdint.h>

#include <vector>

#include "common.cuh"
#include "route.cuh"

namespace fv {

namespace {

// max / mean of the rank loads, as the correctly rounded quotient (max * R) / total.
double imbalance_of(const std::vector<int64_t>& L) {
  int64_t total = 0, mx = 0;
  for (int64_t x : L) {
    total += x;
    mx = x > mx ? x : mx;
  }
  if (total == 0) return 1.0;
  return (double)(mx * (int64_t)L.size()) / (double)total;
}

// Stable in-place compaction of the tile order to the tiles of active heads, one CTA of 1024
// threads walking the order in chunks; every read of a chunk precedes the chunk's writes, and
// writes only go to positions at or before the chunk.
__global__ void __launch_bounds__(1024) select_heads_kernel(int32_t* __restrict__ order, int64_t ntiles, int nt,
                                                            const uint8_t* __restrict__ active,
                                                            int32_t* __restrict__ control) {
  __shared__ int wcount[32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int64_t base = 0;
  bool bad = false;
  for (int64_t c0 = 0; c0 < ntiles; c0 += 1024) {
    const int64_t k = c0 + tid;
    int tile = -1;
    bool keep = false;
    if (k < ntiles) {
      tile = order[k];
      if (tile < 0 || tile >= ntiles) bad = true;
      else keep = active[tile / nt] != 0;
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, keep);
    const int rank = __popc(bal & lanemask_lt());
    if (lane == 0) wcount[warp] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = wcount[w];
      before += w < warp ? c : 0;
      total += c;
    }
    if (keep) order[base + before + rank] = tile;
    base += total;
    __syncthreads();
  }
  if (__syncthreads_or(bad) && tid == 0) report_error(control, FVATTN_ERR_INVALID, 21);
  if (tid == 0) control[3] = (int32_t)base;
}

}  // namespace

cudaError_t launch_select_heads(int32_t* tile_order, const Dims& m, const uint8_t* active, int32_t* control,
                                cudaStream_t st) {
  select_heads_kernel<<<1, 1024, 0, st>>>(tile_order, m.BH * m.nt, m.nt, active, control);
  return cudaGetLastError();
}

}  // namespace fv

extern "C" int fvattn_rlb_plan(const int64_t* loads, int32_t ranks, int32_t heads_per_rank, double target_imbalance,
                               int32_t max_moves_per_rank, int32_t* moves, int64_t moves_capacity,
                               int32_t* n_moves, int64_t* rank_loads) {
  if (loads == nullptr || n_moves == nullptr || ranks < 1 || heads_per_rank < 1 || max_moves_per_rank < 0)
    return FVATTN_ERR_INVALID;
  if (!(target_imbalance >= 1.0) || isinf(target_imbalance)) return FVATTN_ERR_INVALID;
  const int64_t per_rank = max_moves_per_rank < heads_per_rank ? max_moves_per_rank : heads_per_rank;
  if (moves_capacity < (int64_t)ranks * per_rank) return FVATTN_ERR_CAPACITY;
  if (moves == nullptr && moves_capacity > 0) return FVATTN_ERR_INVALID;
  const int64_t n = (int64_t)ranks * heads_per_rank;
  for (int64_t x = 0; x < n; ++x)
    if (loads[x] < 0 || loads[x] > ((int64_t)1 << 40)) return FVATTN_ERR_INVALID;

  std::vector<int64_t> L(ranks, 0);
  for (int r = 0; r < ranks; ++r)
    for (int h = 0; h < heads_per_rank; ++h) L[r] += loads[(int64_t)r * heads_per_rank + h];
  std::vector<char> moved(n, 0);
  std::vector<int32_t> sent(ranks, 0);
  int32_t count = 0;
  while (fv::imbalance_of(L) > target_imbalance) {
    int s = 0, d = 0;
    for (int r = 1; r < ranks; ++r) {
      if (L[r] > L[s]) s = r;
      if (L[r] < L[d]) d = r;
    }
    if (s == d || sent[s] >= max_moves_per_rank) break;
    int best = -1;
    for (int h = 0; h < heads_per_rank; ++h) {
      const int64_t w = loads[(int64_t)s * heads_per_rank + h];
      if (moved[(int64_t)s * heads_per_rank + h] || !(L[d] + w < L[s])) continue;
      if (best < 0 || w > loads[(int64_t)s * heads_per_rank + best]) best = h;
    }
    if (best < 0) break;
    const int64_t w = loads[(int64_t)s * heads_per_rank + best];
    L[s] -= w;
    L[d] += w;
    moved[(int64_t)s * heads_per_rank + best] = 1;
    ++sent[s];
    moves[3 * (int64_t)count + 0] = s;
    moves[3 * (int64_t)count + 1] = best;
    moves[3 * (int64_t)count + 2] = d;
    ++count;
  }
  *n_moves = count;
  if (rank_loads != nullptr)
    for (int r = 0; r < ranks; ++r) rank_loads[r] = L[r];
  return FVATTN_OK;
}
