// moe_route: top-k expert selection + softmax over the k selected logits.
//
// "EP: Partition Experts and Route Tokens", "Send tokens to experts and
// return their results": the router picks each token's experts from all E
// scores; "Return multiple expert results to the same token": the weights
// used at combine are kept apart from the choice.
//
// One warp per token (warp_topk_softmax); lane l loads logits l, l+32, ...
// (coalesced).
#pragma once

#include "common.cuh"

namespace moe {

// Total order on float32 logits as an unsigned key: larger logit -> larger
// key, -0 and +0 map to the same key, NaN sorts below every number (key 1),
// 0 is reserved for "no candidate".
__device__ __forceinline__ uint32_t logit_order_key(float f) {
  if (f != f) return 1u;
  uint32_t u = (f == 0.0f) ? 0u : __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k + softmax of one token by one warp.  Lane l holds the token's logits
// l, l+32, l+64, ... (val[v] for expert l + 32 v; key[v] = logit_order_key, or
// 0 for no expert).  Each of the k rounds takes a warp-wide arg-max with two
// redux ops: the largest order key, then the smallest expert id among lanes
// holding it, so equal logits resolve to the lower id.  Lane j < k gets the
// j-th expert and its weight exp(l_j - l_0) / sum_i exp(l_i - l_0), the sum
// taken in order i = 0..k-1.
template <int VPL>
__device__ __forceinline__ void warp_topk_softmax(uint32_t (&key)[VPL], const float (&val)[VPL], int k, int lane,
                                                  int& my_id, float& my_w) {
  my_id = 0;
  float my_val = 0.0f;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0;
    int bid = 0x7FFFFFFF;
    float bv = 0.0f;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      // ascending v visits ascending expert ids, so strict '>' keeps the lower id
      const bool better = key[v] > bk;
      bk = better ? key[v] : bk;
      bid = better ? lane + 32 * v : bid;
      bv = better ? val[v] : bv;
    }
    const uint32_t wk = __reduce_max_sync(0xFFFFFFFFu, bk);
    const int wid = __reduce_min_sync(0xFFFFFFFFu, bk == wk ? bid : 0x7FFFFFFF);
    const float wv = __shfl_sync(0xFFFFFFFFu, bv, wid & 31);  // the winner's logit, from its lane
    const bool mine = (wid & 31) == lane;
#pragma unroll
    for (int v = 0; v < VPL; ++v) key[v] = (mine && v == (wid >> 5)) ? 0u : key[v];  // taken
    if (lane == j) {
      my_id = wid;
      my_val = wv;
    }
  }
  // softmax over the selected logits, max-subtracted (the first pick is the max)
  const float l0 = __shfl_sync(0xFFFFFFFFu, my_val, 0);
  const float ex = lane < k ? expf(my_val - l0) : 0.0f;
  float sum = 0.0f;
  for (int j = 0; j < k; ++j) sum += __shfl_sync(0xFFFFFFFFu, ex, j);  // fixed order j = 0..k-1
  my_w = ex / sum;
}

template <int VPL>  // logits per lane: ceil(E / 32)
__global__ void __launch_bounds__(256) route_topk_softmax_kernel(const float* __restrict__ logits, int T, int E,
                                                                 int k, int32_t* __restrict__ topk_ids,
                                                                 float* __restrict__ topk_w) {
  pdl_wait();
  pdl_trigger();
  const int t = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = (int)lane_id();
  if (t >= T) return;  // whole warp exits together
  const float* row = logits + (size_t)t * E;

  uint32_t key[VPL];
  float val[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int e = lane + 32 * v;
    val[v] = (e < E) ? __ldg(row + e) : 0.0f;
    key[v] = (e < E) ? logit_order_key(val[v]) : 0u;
  }
  int my_id;
  float my_w;
  warp_topk_softmax<VPL>(key, val, k, lane, my_id, my_w);
  if (lane < k) {
    topk_ids[(size_t)t * k + lane] = my_id;
    topk_w[(size_t)t * k + lane] = my_w;
  }
}

inline cudaError_t launch_route(const float* logits, int T, int E, int k, int32_t* ids, float* w,
                                cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = (int)(((size_t)T * 32 + threads - 1) / threads);
  const int vpl = (E + 31) / 32;
  cudaError_t err = cudaSuccess;
#define MOE_ROUTE_CASE(V)                                                                  \
  case V:                                                                                  \
    err = launch_pdl(route_topk_softmax_kernel<V>, blocks, threads, 0, stream, logits, T, E, k, ids, w); \
    break;
  switch (vpl <= 1 ? 1 : vpl <= 2 ? 2 : vpl <= 4 ? 4 : vpl <= 8 ? 8 : vpl <= 16 ? 16 : 32) {
    MOE_ROUTE_CASE(1)
    MOE_ROUTE_CASE(2)
    MOE_ROUTE_CASE(4)
    MOE_ROUTE_CASE(8)
    MOE_ROUTE_CASE(16)
    MOE_ROUTE_CASE(32)
  }
#undef MOE_ROUTE_CASE
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
