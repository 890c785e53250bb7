// Expert placement with replicas (an expert-parallel load balancer).
//
// "什么是专家并行（Expert Parallelism）？", sections "工作机制" and
// "边界与常见误解" (third point): routing is dynamic, so per-expert token
// counts drift, and a balancer redistributes hot and cold experts over the
// GPUs to keep their utilisation balanced.  "Expert Parallelism (EP)",
// "Limitations" 3: the static contiguous layout has neither replication nor
// dynamic balancing.
//
// The plan (host, from measured per-expert loads) gives every expert one
// replica and each extra physical slot to the expert with the largest load
// per replica; splits an expert's load evenly over its replicas (integer
// shares, the remainder to the first ones); and places the replicas, largest
// share first, each on the least-loaded rank that has a free slot.  Every tie
// is broken by the lower expert id, replica index or rank, so the plan is an
// exact function of the loads.  The remap (device, every step) sends slot
// t*k + j of expert e to replica t mod n_e.  A replica holds the same weights
// as its expert, so the round trip's results do not change: only which
// physical expert (and rank) each row goes to.
#pragma once

#include <algorithm>
#include <cstdint>
#include <queue>
#include <vector>

#include "common.cuh"

namespace moe {

constexpr int kEplbMaxSlots = 1 << 20;          // physical expert slots in one plan
constexpr int64_t kEplbMaxLoad = int64_t(1) << 40;  // load * replicas stays below 2^63

// Returns false for sizes or loads outside the documented ranges.
inline bool eplb_plan_host(const int64_t* load, int E, int R, int slots, int32_t* phys_to_logical,
                           int32_t* replica_offsets, int32_t* replicas) {
  if (E < 1 || R < 1 || slots < 1 || (int64_t)R * slots > kEplbMaxSlots || R * slots < E) return false;
  for (int e = 0; e < E; ++e)
    if (load[e] < 0 || load[e] >= kEplbMaxLoad) return false;
  const int P = R * slots;

  // 1. replica counts: a max-heap of experts by load per replica
  std::vector<int> n(E, 1);
  auto before = [&](int a, int b) {  // a's load per replica is larger (ties: lower id)
    const int64_t lhs = load[a] * (int64_t)n[b], rhs = load[b] * (int64_t)n[a];
    return lhs != rhs ? lhs > rhs : a < b;
  };
  auto heap_less = [&](int a, int b) { return before(b, a); };  // top() = the expert that comes first
  std::priority_queue<int, std::vector<int>, decltype(heap_less)> heap(heap_less);
  for (int e = 0; e < E; ++e) heap.push(e);
  for (int extra = 0; extra < P - E; ++extra) {
    const int e = heap.top();
    heap.pop();
    ++n[e];
    heap.push(e);
  }

  // 2. shares: expert e's load split evenly over its n_e replicas
  struct Replica {
    int64_t share;
    int e, j;
  };
  std::vector<Replica> rep;
  rep.reserve(P);
  replica_offsets[0] = 0;
  for (int e = 0; e < E; ++e) {
    replica_offsets[e + 1] = replica_offsets[e] + n[e];
    const int64_t q = load[e] / n[e], rem = load[e] % n[e];
    for (int j = 0; j < n[e]; ++j) rep.push_back({q + (j < rem ? 1 : 0), e, j});
  }
  std::sort(rep.begin(), rep.end(), [](const Replica& a, const Replica& b) {
    if (a.share != b.share) return a.share > b.share;
    if (a.e != b.e) return a.e < b.e;
    return a.j < b.j;
  });

  // 3. placement: the least-loaded rank with a free slot (ties: lower rank)
  using RankKey = std::pair<int64_t, int>;  // (placed share, rank)
  std::priority_queue<RankKey, std::vector<RankKey>, std::greater<RankKey>> ranks;
  for (int r = 0; r < R; ++r) ranks.push({0, r});
  std::vector<int> used(R, 0);
  for (const Replica& x : rep) {
    const RankKey top = ranks.top();
    ranks.pop();
    const int r = top.second;
    const int phys = r * slots + used[r]++;
    phys_to_logical[phys] = x.e;
    replicas[replica_offsets[x.e] + x.j] = phys;
    if (used[r] < slots) ranks.push({top.first + x.share, r});
  }
  return true;
}

// phys_ids[t*k + j] = replicas[replica_offsets[e] + t % n_e] for e = ids[t*k + j].
// Ids outside [0, E) give -1 and set the bad-id bit; replica tables that are
// not consistent (an empty range, an offset or id outside [0, P)) give -1 and
// set the bad-offsets bit.  Never reads outside the tables.
__global__ void __launch_bounds__(256) eplb_remap_kernel(const int32_t* __restrict__ ids, int T, int k, int E,
                                                         const int32_t* __restrict__ replica_offsets,
                                                         const int32_t* __restrict__ replicas, int P,
                                                         int32_t* __restrict__ phys_ids) {
  pdl_wait();
  pdl_trigger();
  const int64_t S = (int64_t)T * k;
  for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < S; s += (int64_t)gridDim.x * blockDim.x) {
    const int e = __ldg(ids + s);
    int out = -1;
    if (e < 0 || e >= E) {
      flag_error(kErrBadId);
    } else {
      const int lo = __ldg(replica_offsets + e), hi = __ldg(replica_offsets + e + 1);
      if (lo < 0 || hi > P || hi <= lo) {
        flag_error(kErrBadOffsets);
      } else {
        const int t = (int)(s / k);
        const int p = __ldg(replicas + lo + t % (hi - lo));
        if (p < 0 || p >= P) flag_error(kErrBadOffsets);
        else out = p;
      }
    }
    phys_ids[s] = out;
  }
}

inline cudaError_t launch_eplb_remap(const int32_t* ids, int T, int k, int E, const int32_t* replica_offsets,
                                     const int32_t* replicas, int P, int32_t* phys_ids, cudaStream_t stream) {
  const int64_t S = (int64_t)T * k;
  if (S == 0) return cudaSuccess;
  const int grid = (int)std::min<int64_t>((S + 255) / 256, 148 * 8);
  cudaError_t err = launch_pdl(eplb_remap_kernel, grid, 256, 0, stream, ids, T, k, E, replica_offsets, replicas, P,
                               phys_ids);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
