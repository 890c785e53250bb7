// The masking form of expert parallelism: per-rank partial outputs and their
// reduction.
//
// "Expert Parallelism (EP)" (vLLM on Neuron), "Collective Patterns / Prefill
// (CTE kernel)" steps 5-6 and "Why a Single All-Reduce/Reduce-Scatter Works":
// every rank runs all tokens against its own experts only; a token whose
// chosen experts all sit elsewhere gets zeros from that rank; a reduce-scatter
// (prefill) or all-reduce (decode) over the ranks sums the partial outputs
// into the full weighted combination.  On one GPU the R logical ranks'
// partials are R [T, H] planes of one buffer and the reduction is a kernel.
//
// rank_partials_kernel: one warp per (token, slice of 64 16-byte columns),
// as combine_kernel.  Lanes j < k fetch (row_j, w_j, owner rank of id_j);
// each lane loads its column chunk of the k rows once, then for every rank r
// sums, in j order and in float32, the w_j-weighted chunks whose expert r
// owns, and stores the rounded sum (zero for a rank that owns none) into
// plane r.  y_disp is read once; the R planes are written once.
//
// reduce_ranks_kernel: one thread per 16-byte column chunk of y; sums the R
// planes' chunks in rank order in float32 and rounds once.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kPartialSlice = 64;  // 16-byte column vectors of a row per warp (2 per lane)

template <typename T, int K>
__global__ void __launch_bounds__(256) rank_partials_kernel(const T* __restrict__ y_disp,
                                                            const float* __restrict__ topk_w,
                                                            const int32_t* __restrict__ topk_ids,
                                                            const int32_t* __restrict__ slot_to_row, int T_, int H,
                                                            int S, int E, int EL, int R, int nslices,
                                                            T* __restrict__ part) {
  pdl_wait();
  pdl_trigger();
  const size_t gw = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5;
  const int t = (int)(gw / nslices), cs = (int)(gw - (size_t)t * nslices);
  const int lane = (int)lane_id();
  if (t >= T_) return;
  int my_row = -1, my_rank = -1;
  float my_w = 0.0f;
  if (lane < K) {
    const size_t s = (size_t)t * K + lane;
    my_row = __ldg(slot_to_row + s);
    const int e = __ldg(topk_ids + s);
    my_w = __ldg(topk_w + s);
    if (my_row < 0 || my_row >= S || e < 0 || e >= E) {
      // -1 marks a slot that dispatch dropped (its id was outside [0, E))
      if (my_row != -1 && cs == 0) flag_error(kErrBadRow);
      my_row = -1;
    } else {
      my_rank = e / EL;
    }
  }
  int rows[K], ranks[K];
  float w[K];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    rows[j] = __shfl_sync(0xFFFFFFFFu, my_row, j);
    ranks[j] = __shfl_sync(0xFFFFFFFFu, my_rank, j);
    w[j] = __shfl_sync(0xFFFFFFFFu, my_w, j);
  }
  constexpr int N = Vec16<T>::N;
  const int nvec = H / N;
  const size_t plane = (size_t)T_ * H;
  char* dst0 = reinterpret_cast<char*>(part + (size_t)t * H);
  const int i_end = min(nvec, (cs + 1) * kPartialSlice);
  for (int i = cs * kPartialSlice + lane; i < i_end; i += 32) {
    float f[K][N];
#pragma unroll
    for (int j = 0; j < K; ++j) {
      if (rows[j] >= 0) {
        const uint4 v = ld_nc_v4(reinterpret_cast<const char*>(y_disp + (size_t)rows[j] * H) + (size_t)i * 16);
        unpack16(v, f[j], T());
      }
    }
    for (int r = 0; r < R; ++r) {
      float acc[N];
#pragma unroll
      for (int c = 0; c < N; ++c) acc[c] = 0.0f;
#pragma unroll
      for (int j = 0; j < K; ++j) {
        if (ranks[j] != r) continue;  // also skips dropped slots (rank -1)
#pragma unroll
        for (int c = 0; c < N; ++c) acc[c] = fmaf(w[j], f[j][c], acc[c]);
      }
      st_v4(dst0 + ((size_t)r * plane) * sizeof(T) + (size_t)i * 16, pack16(acc, T()));
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) reduce_ranks_kernel(const T* __restrict__ part, size_t nvec_total, int R,
                                                           T* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  constexpr int N = Vec16<T>::N;
  const size_t plane_bytes = nvec_total * 16;
  const char* src = reinterpret_cast<const char*>(part);
  char* dst = reinterpret_cast<char*>(y);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nvec_total; i += (size_t)gridDim.x * blockDim.x) {
    float acc[N];
#pragma unroll
    for (int c = 0; c < N; ++c) acc[c] = 0.0f;
    int r = 0;
    for (; r + 4 <= R; r += 4) {  // four planes' loads in flight, summed in rank order
      uint4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = ld_nc_v4(src + (size_t)(r + q) * plane_bytes + i * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float f[N];
        unpack16(v[q], f, T());
#pragma unroll
        for (int c = 0; c < N; ++c) acc[c] += f[c];
      }
    }
    for (; r < R; ++r) {
      float f[N];
      unpack16(ld_nc_v4(src + (size_t)r * plane_bytes + i * 16), f, T());
#pragma unroll
      for (int c = 0; c < N; ++c) acc[c] += f[c];
    }
    st_v4(dst + i * 16, pack16(acc, T()));
  }
}

template <typename T>
cudaError_t launch_rank_partials(const T* y_disp, const float* topk_w, const int32_t* topk_ids,
                                 const int32_t* slot_to_row, int T_, int k, int H, int E, int R, T* part,
                                 cudaStream_t stream) {
  if (T_ == 0) return cudaSuccess;
  const int threads = 256;
  const int nvec = H / Vec16<T>::N;
  const int nslices = (nvec + kPartialSlice - 1) / kPartialSlice;
  const int blocks = (int)(((size_t)T_ * nslices * 32 + threads - 1) / threads);
  const int S = T_ * k, EL = E / R;
  cudaError_t err = cudaSuccess;
  switch (k) {
#define MOE_PARTIALS_CASE(KK)                                                                                   \
  case KK:                                                                                                      \
    err = launch_pdl(rank_partials_kernel<T, KK>, blocks, threads, 0, stream, y_disp, topk_w, topk_ids,       \
                     slot_to_row, T_, H, S, E, EL, R, nslices, part);                                           \
    break;
    MOE_PARTIALS_CASE(1)
    MOE_PARTIALS_CASE(2)
    MOE_PARTIALS_CASE(3)
    MOE_PARTIALS_CASE(4)
    MOE_PARTIALS_CASE(5)
    MOE_PARTIALS_CASE(6)
    MOE_PARTIALS_CASE(7)
    MOE_PARTIALS_CASE(8)
#undef MOE_PARTIALS_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return err != cudaSuccess ? err : cudaGetLastError();
}

template <typename T>
cudaError_t launch_reduce_ranks(const T* part, int T_, int H, int R, T* y, cudaStream_t stream) {
  if (T_ == 0) return cudaSuccess;
  const size_t nvec = (size_t)T_ * H / Vec16<T>::N;
  const int threads = 256;
  int sms = 0;
  cudaError_t err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, current_device());
  if (err != cudaSuccess) return err;
  // grid-stride over the column chunks, at most 8 CTAs of 256 threads per SM
  size_t blocks = (nvec + threads - 1) / threads;
  const size_t cap = (size_t)sms * 8;
  if (blocks > cap) blocks = cap;
  err = launch_pdl(reduce_ranks_kernel<T>, dim3((unsigned)blocks), dim3(threads), 0, stream, part, nvec, R, y);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
