// Expert-parallel exchange between ranks: the send plan of a source rank and
// the pack of its rows into per-destination buffers.
//
// "EP: Partition Experts and Route Tokens", "Send tokens to experts and
// return their results": each GPU routes its own tokens and sends each token
// vector to the GPU holding its selected expert (an exchange by destination
// with unequal counts); results return to the source GPU and token.  "Return
// multiple expert results to the same token": input delivery is shared when
// two selected experts sit on the same GPU.  "Expert Parallelism (EP)",
// "Limitations" 3-4: rank d holds experts [d*E/R, (d+1)*E/R).
//
// Plan (one source rank, T tokens): one send row per (token t, destination d
// holding any of t's experts), ordered by d then t; the row carries t's local
// expert ids on d (top-k order, -1 padded to k) and their weights.
//   ep_count_kernel: 1024-token chunks, a thread per token builds its
//     destination bit mask; per destination a warp ballot counts the chunk's
//     tokens -> chunk_counts[chunk][d].
//   ep_place_kernel: every CTA sums the chunk counts (its prefix and the
//     totals), scans the totals into send offsets, ranks its tokens per
//     destination (warp ballot prefix + a scan over the CTA's warps) and
//     writes, per token, its rows' ids and weights, the row of each slot, the
//     row of each slot's first choice on its destination (for the source's
//     final sum), and each row's token.
// Pack: a warp per (send row, slice of 128 16-byte columns) copies the token's
// row to its destination buffer with 16-byte vector accesses (peer stores
// over NVLink when the buffer is another GPU's), plus the row's ids and
// weights.  Rows whose destination row is beyond the buffer's capacity are
// skipped and flagged.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kEpMaxRanks = 64;      // destination masks are 64-bit
constexpr int kEpPlanThreads = 1024;  // tokens per plan chunk
constexpr int kEpPackThreads = 256;
constexpr int kEpPackSlice = 128;     // 16-byte vectors of a row per warp item (4 per lane)

inline int ep_plan_chunks(int T) { return (T + kEpPlanThreads - 1) / kEpPlanThreads; }

// Workspace: mask[T] uint64, then chunk_counts[chunks][R] int32.
inline size_t ep_plan_ws_bytes(int T, int R) {
  return ((size_t)T * 8 + 255) / 256 * 256 + (size_t)ep_plan_chunks(T) * R * 4;
}

struct EpPlanArgs {
  const int32_t* ids;
  const float* w;
  int T, k, E, R, EL, nchunks;
  uint64_t* mask;
  int32_t* chunk_counts;
  int32_t* send_counts;    // [R]
  int32_t* send_offsets;   // [R + 1]
  int32_t* slot_send_row;  // [T*k]
  int32_t* ret_row;        // [T*k]
  int32_t* row_token;      // [rows]
  int32_t* row_ids;        // [rows][k]
  float* row_w;            // [rows][k]
};

inline EpPlanArgs ep_plan_args(const int32_t* ids, const float* w, int T, int k, int E, int R, void* ws,
                               int32_t* send_counts, int32_t* send_offsets, int32_t* slot_send_row, int32_t* ret_row,
                               int32_t* row_token, int32_t* row_ids, float* row_w) {
  EpPlanArgs a;
  a.ids = ids;
  a.w = w;
  a.T = T;
  a.k = k;
  a.E = E;
  a.R = R;
  a.EL = E / R;
  a.nchunks = ep_plan_chunks(T);
  a.mask = reinterpret_cast<uint64_t*>(ws);
  a.chunk_counts = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + ((size_t)T * 8 + 255) / 256 * 256);
  a.send_counts = send_counts;
  a.send_offsets = send_offsets;
  a.slot_send_row = slot_send_row;
  a.ret_row = ret_row;
  a.row_token = row_token;
  a.row_ids = row_ids;
  a.row_w = row_w;
  return a;
}

__global__ void __launch_bounds__(kEpPlanThreads) ep_count_kernel(EpPlanArgs a) {
  __shared__ int32_t warp_cnt[kEpPlanThreads / 32][kEpMaxRanks];
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * kEpPlanThreads + threadIdx.x;
  uint64_t m = 0;
  if (t < a.T) {
    for (int j = 0; j < a.k; ++j) {
      const int e = __ldg(a.ids + (size_t)t * a.k + j);
      if (e < 0 || e >= a.E) {
        flag_error(kErrBadId);
        continue;
      }
      m |= 1ull << (e / a.EL);
    }
    a.mask[t] = m;
  }
  const int warp = threadIdx.x >> 5, lane = (int)lane_id();
  for (int d = 0; d < a.R; ++d) {
    const unsigned b = __ballot_sync(0xFFFFFFFFu, (unsigned)((m >> d) & 1ull));
    if (lane == 0) warp_cnt[warp][d] = __popc(b);
  }
  __syncthreads();
  for (int d = threadIdx.x; d < a.R; d += kEpPlanThreads) {
    int c = 0;
#pragma unroll 8
    for (int w = 0; w < kEpPlanThreads / 32; ++w) c += warp_cnt[w][d];
    a.chunk_counts[(size_t)blockIdx.x * a.R + d] = c;
  }
}

__global__ void __launch_bounds__(kEpPlanThreads) ep_place_kernel(EpPlanArgs a) {
  __shared__ int32_t warp_pre[kEpPlanThreads / 32][kEpMaxRanks];
  __shared__ int32_t base[kEpMaxRanks];  // send offset of d + this chunk's earlier chunks' rows for d
  __shared__ int32_t tot[kEpMaxRanks];
  __shared__ int32_t offs[kEpMaxRanks + 1];
  pdl_wait();
  pdl_trigger();
  const int c = blockIdx.x;
  if ((int)threadIdx.x < a.R) {
    const int d = threadIdx.x;
    int before = 0, total = 0;
    for (int cc = 0; cc < a.nchunks; ++cc) {
      const int v = __ldcg(a.chunk_counts + (size_t)cc * a.R + d);
      total += v;
      if (cc < c) before += v;
    }
    base[d] = before;
    tot[d] = total;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int d = 0; d < a.R; ++d) {
      offs[d] = run;
      run += tot[d];
    }
    offs[a.R] = run;
  }
  __syncthreads();
  if ((int)threadIdx.x < a.R) base[threadIdx.x] += offs[threadIdx.x];
  if (c == 0 && (int)threadIdx.x <= a.R) {
    a.send_offsets[threadIdx.x] = offs[threadIdx.x];
    if ((int)threadIdx.x < a.R) a.send_counts[threadIdx.x] = tot[threadIdx.x];
  }
  const int t = c * kEpPlanThreads + threadIdx.x;
  const uint64_t m = (t < a.T) ? __ldcg(reinterpret_cast<const unsigned long long*>(a.mask) + t) : 0ull;
  const int warp = threadIdx.x >> 5, lane = (int)lane_id();
  for (int d = 0; d < a.R; ++d) {
    const unsigned b = __ballot_sync(0xFFFFFFFFu, (unsigned)((m >> d) & 1ull));
    if (lane == 0) warp_pre[warp][d] = __popc(b);
  }
  __syncthreads();
  if ((int)threadIdx.x < a.R) {  // exclusive scan over the CTA's warps, per destination
    const int d = threadIdx.x;
    int run = base[d];
    for (int w = 0; w < kEpPlanThreads / 32; ++w) {
      const int v = warp_pre[w][d];
      warp_pre[w][d] = run;
      run += v;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  if (t < a.T) {
    for (int j = 0; j < a.k; ++j) {
      a.slot_send_row[(size_t)t * a.k + j] = -1;
      a.ret_row[(size_t)t * a.k + j] = -1;
    }
  }
  for (int d = 0; d < a.R; ++d) {  // uniform over the warp: every lane takes part in each ballot
    const bool mine = (m >> d) & 1ull;
    const unsigned b = __ballot_sync(0xFFFFFFFFu, (unsigned)mine);
    if (!mine) continue;
    const int row = warp_pre[warp][d] + __popc(b & lt);
    int n = 0;
    for (int j = 0; j < a.k; ++j) {
      const size_t s = (size_t)t * a.k + j;
      const int e = __ldg(a.ids + s);
      if (e < 0 || e >= a.E || e / a.EL != d) continue;
      a.row_ids[(size_t)row * a.k + n] = e - d * a.EL;
      a.row_w[(size_t)row * a.k + n] = __ldg(a.w + s);
      a.slot_send_row[s] = row;
      if (n == 0) a.ret_row[s] = row;
      ++n;
    }
    for (int i = n; i < a.k; ++i) {
      a.row_ids[(size_t)row * a.k + i] = -1;
      a.row_w[(size_t)row * a.k + i] = 0.0f;
    }
    a.row_token[row] = t;
  }
}

inline cudaError_t launch_ep_plan(const EpPlanArgs& a, cudaStream_t stream) {
  if (a.T == 0) return cudaSuccess;
  cudaError_t err = launch_pdl(ep_count_kernel, dim3(a.nchunks), dim3(kEpPlanThreads), 0, stream, a);
  if (err != cudaSuccess) return err;
  err = launch_pdl(ep_place_kernel, dim3(a.nchunks), dim3(kEpPlanThreads), 0, stream, a);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// The same plan, sequentially on the host (for host-side drivers and tests of
// the exchange protocol without a GPU).  Returns false for an id outside
// [0, E) (whose slot rows are then -1).
inline bool ep_plan_host(const int32_t* ids, const float* w, int T, int k, int E, int R, int32_t* send_counts,
                         int32_t* send_offsets, int32_t* slot_send_row, int32_t* ret_row, int32_t* row_token,
                         int32_t* row_ids, float* row_w) {
  const int EL = E / R;
  bool ok = true;
  for (int d = 0; d < R; ++d) send_counts[d] = 0;
  for (int t = 0; t < T; ++t) {
    uint64_t m = 0;
    for (int j = 0; j < k; ++j) {
      const int e = ids[(size_t)t * k + j];
      if (e < 0 || e >= E) {
        ok = false;
        continue;
      }
      m |= 1ull << (e / EL);
    }
    for (int d = 0; d < R; ++d) send_counts[d] += (int)((m >> d) & 1ull);
  }
  send_offsets[0] = 0;
  for (int d = 0; d < R; ++d) send_offsets[d + 1] = send_offsets[d] + send_counts[d];
  for (size_t s = 0; s < (size_t)T * k; ++s) slot_send_row[s] = ret_row[s] = -1;
  int next[kEpMaxRanks];
  for (int d = 0; d < R; ++d) next[d] = send_offsets[d];
  for (int t = 0; t < T; ++t) {
    int row_of[kEpMaxRanks];
    int n_of[kEpMaxRanks];
    for (int d = 0; d < R; ++d) row_of[d] = -1, n_of[d] = 0;
    for (int j = 0; j < k; ++j) {
      const size_t s = (size_t)t * k + j;
      const int e = ids[s];
      if (e < 0 || e >= E) continue;
      const int d = e / EL;
      if (row_of[d] < 0) {
        row_of[d] = next[d]++;
        row_token[row_of[d]] = t;
        ret_row[s] = row_of[d];
      }
      row_ids[(size_t)row_of[d] * k + n_of[d]] = e - d * EL;
      row_w[(size_t)row_of[d] * k + n_of[d]] = w[s];
      ++n_of[d];
      slot_send_row[s] = row_of[d];
    }
    for (int d = 0; d < R; ++d)
      if (row_of[d] >= 0)
        for (int i = n_of[d]; i < k; ++i) {
          row_ids[(size_t)row_of[d] * k + i] = -1;
          row_w[(size_t)row_of[d] * k + i] = 0.0f;
        }
  }
  return ok;
}

// Where the rows meet across ranks, from every source's send counts
// (counts[s][d], the all-gathered send_counts), for rank r:
//   dst_base[d]  = sum_{s < r} counts[s][d]: r's rows start there in d's receive buffer;
//   recv_base[s] = sum_{s' < s} counts[s'][r] (recv_base[R] = rows r receives);
//   ret_base[s]  = sum_{d < r} counts[s][d]: where r's partials for source s go in s's return buffer
//                  (= source s's send offset of destination r).
inline void ep_exchange_offsets_host(const int32_t* counts, int R, int r, int32_t* dst_base, int32_t* recv_base,
                                     int32_t* ret_base) {
  for (int d = 0; d < R; ++d) {
    int v = 0;
    for (int s = 0; s < r; ++s) v += counts[(size_t)s * R + d];
    dst_base[d] = v;
  }
  recv_base[0] = 0;
  for (int s = 0; s < R; ++s) recv_base[s + 1] = recv_base[s] + counts[(size_t)s * R + r];
  for (int s = 0; s < R; ++s) {
    int v = 0;
    for (int d = 0; d < r; ++d) v += counts[(size_t)s * R + d];
    ret_base[s] = v;
  }
}

// Destination buffers of a pack, one set per destination rank.
struct EpDest {
  void* x[kEpMaxRanks];         // [cap[d], H] rows
  int32_t* ids[kEpMaxRanks];    // [cap[d], k]
  float* w[kEpMaxRanks];        // [cap[d], k]
  int cap[kEpMaxRanks];         // rows each buffer holds
};

template <typename T>
__global__ void __launch_bounds__(kEpPackThreads) ep_pack_kernel(const T* __restrict__ x, int T_, int H, int k, int R,
                                                                 int nslices, const int32_t* __restrict__ send_offsets,
                                                                 const int32_t* __restrict__ dst_base,
                                                                 const int32_t* __restrict__ row_token,
                                                                 const int32_t* __restrict__ row_ids,
                                                                 const float* __restrict__ row_w, EpDest dst) {
  __shared__ int32_t offs[kEpMaxRanks + 1];
  __shared__ int32_t dbase[kEpMaxRanks];
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i <= R; i += blockDim.x) offs[i] = __ldcg(send_offsets + i);
  for (int i = threadIdx.x; i < R; i += blockDim.x) dbase[i] = __ldcg(dst_base + i);
  __syncthreads();
  const int rows = offs[R];
  const int lane = (int)lane_id();
  const size_t nitems = (size_t)rows * nslices;
  const size_t warps = (size_t)gridDim.x * (kEpPackThreads / 32);
  constexpr int N = Vec16<T>::N;
  const int nvec = H / N;
  for (size_t item = (blockIdx.x * (size_t)kEpPackThreads + threadIdx.x) >> 5; item < nitems; item += warps) {
    const int row = (int)(item / nslices), cs = (int)(item - (size_t)row * nslices);
    int d = 0;
    while (d + 1 < R && offs[d + 1] <= row) ++d;  // destination of the row (R <= 64)
    const int drow = dbase[d] + row - offs[d];
    const int t = __ldg(row_token + row);
    if (drow < 0 || drow >= dst.cap[d] || t < 0 || t >= T_) {
      if (cs == 0 && lane == 0) flag_error(kErrBadRow);
      continue;
    }
    const char* src = reinterpret_cast<const char*>(x + (size_t)t * H);
    char* out = reinterpret_cast<char*>(static_cast<T*>(dst.x[d]) + (size_t)drow * H);
    uint4 v[kEpPackSlice / 32];
#pragma unroll
    for (int u = 0; u < kEpPackSlice / 32; ++u) {
      const int i = cs * kEpPackSlice + u * 32 + lane;
      if (i < nvec) v[u] = ld_nc_v4(src + (size_t)i * 16);
    }
#pragma unroll
    for (int u = 0; u < kEpPackSlice / 32; ++u) {
      const int i = cs * kEpPackSlice + u * 32 + lane;
      if (i < nvec) st_v4(out + (size_t)i * 16, v[u]);
    }
    if (cs == 0 && lane < k) {
      dst.ids[d][(size_t)drow * k + lane] = __ldg(row_ids + (size_t)row * k + lane);
      dst.w[d][(size_t)drow * k + lane] = __ldg(row_w + (size_t)row * k + lane);
    }
  }
}

template <typename T>
cudaError_t launch_ep_pack(const T* x, int T_, int H, int k, int R, int max_rows, const int32_t* send_offsets,
                           const int32_t* dst_base, const int32_t* row_token, const int32_t* row_ids,
                           const float* row_w, const EpDest& dst, cudaStream_t stream) {
  if (max_rows == 0) return cudaSuccess;
  const int nvec = H / Vec16<T>::N;
  const int nslices = (nvec + kEpPackSlice - 1) / kEpPackSlice;
  int sms = 0;
  cudaError_t err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, current_device());
  if (err != cudaSuccess) return err;
  // a warp per item; enough CTAs for the largest possible row count, at most 8 per SM (grid-stride beyond)
  size_t blocks = ((size_t)max_rows * nslices + kEpPackThreads / 32 - 1) / (kEpPackThreads / 32);
  if (blocks > (size_t)sms * 8) blocks = (size_t)sms * 8;
  if (blocks < 1) blocks = 1;
  err = launch_pdl(ep_pack_kernel<T>, dim3((unsigned)blocks), dim3(kEpPackThreads), 0, stream, x, T_, H, k, R, nslices,
                   send_offsets, dst_base, row_token, row_ids, row_w, dst);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
