// moe_combine: gather each token's k expert outputs, weight, sum, unpermute.
//
// "EP: Partition Experts and Route Tokens", "Send tokens to experts and
// return their results": each result returns to its source token, in the
// original order; "Return multiple expert results to the same token":
// y(t) = sum_j w_j u_j (e.g. 0.7 u0 + 0.3 u2).
//
// One warp per (token, slice of 64 16-byte columns).  Lanes j < k fetch
// (row_j, w_j) and broadcast them; then each lane walks its 16-byte column
// chunks, issuing all k row loads before the float32 multiply-adds (fixed
// order j = 0..k-1) and one rounded store.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kCombineSlice = 64;  // 16-byte column vectors of a row per warp (2 per lane)

template <typename T, int K>
__global__ void __launch_bounds__(256) combine_kernel(const T* __restrict__ y_disp, const float* __restrict__ topk_w,
                                                      const int32_t* __restrict__ slot_to_row, int T_, int H, int S,
                                                      int nslices, T* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const size_t gw = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5;
  const int t = (int)(gw / nslices), cs = (int)(gw - (size_t)t * nslices);
  const int lane = (int)lane_id();
  if (t >= T_) return;
  int my_row = -1;
  float my_w = 0.0f;
  if (lane < K) {
    my_row = __ldg(slot_to_row + (size_t)t * K + lane);
    my_w = __ldg(topk_w + (size_t)t * K + lane);
    if (my_row < 0 || my_row >= S) {
      if (my_row != -1 && cs == 0) flag_error(kErrBadRow);  // -1 marks a slot dispatch dropped
      my_row = -1;
    }
  }
  int rows[K];
  float w[K];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    rows[j] = __shfl_sync(0xFFFFFFFFu, my_row, j);
    w[j] = __shfl_sync(0xFFFFFFFFu, my_w, j);
  }
  constexpr int N = Vec16<T>::N;
  const int nvec = H / N;
  char* dst = reinterpret_cast<char*>(y + (size_t)t * H);
  const int i_end = min(nvec, (cs + 1) * kCombineSlice);
  for (int i = cs * kCombineSlice + lane; i < i_end; i += 32) {
    uint4 v[K];
#pragma unroll
    for (int j = 0; j < K; ++j)
      if (rows[j] >= 0) v[j] = ld_nc_v4(reinterpret_cast<const char*>(y_disp + (size_t)rows[j] * H) + (size_t)i * 16);
    float acc[N];
#pragma unroll
    for (int c = 0; c < N; ++c) acc[c] = 0.0f;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      if (rows[j] < 0) continue;
      float f[N];
      unpack16(v[j], f, T());
#pragma unroll
      for (int c = 0; c < N; ++c) acc[c] = fmaf(w[j], f[c], acc[c]);
    }
    st_v4(dst + (size_t)i * 16, pack16(acc, T()));
  }
}

template <typename T>
cudaError_t launch_combine(const T* y_disp, const float* topk_w, const int32_t* slot_to_row, int T_, int k, int H,
                           T* y, cudaStream_t stream) {
  if (T_ == 0) return cudaSuccess;
  const int threads = 256;
  const int nvec = H / Vec16<T>::N;
  const int nslices = (nvec + kCombineSlice - 1) / kCombineSlice;
  const int blocks = (int)(((size_t)T_ * nslices * 32 + threads - 1) / threads);
  const int S = T_ * k;
  cudaError_t err = cudaSuccess;
  switch (k) {
#define MOE_COMBINE_CASE(KK) \
  case KK:                   \
    err = launch_pdl(combine_kernel<T, KK>, blocks, threads, 0, stream, y_disp, topk_w, slot_to_row, T_, H, S, \
                     nslices, y);                                                                                \
    break;
    MOE_COMBINE_CASE(1)
    MOE_COMBINE_CASE(2)
    MOE_COMBINE_CASE(3)
    MOE_COMBINE_CASE(4)
    MOE_COMBINE_CASE(5)
    MOE_COMBINE_CASE(6)
    MOE_COMBINE_CASE(7)
    MOE_COMBINE_CASE(8)
#undef MOE_COMBINE_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
