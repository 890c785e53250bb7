// moe_dispatch: expert histogram, exclusive scans, stable permutation and the
// row scatter into the expert-contiguous (= rank-major) buffer.
//
// "EP: Partition Experts and Route Tokens", "Send tokens to experts and
// return their results": dispatch groups token vectors by selected expert and
// keeps each row's association with its token; "Equal expert counts can
// receive different token counts": per-expert and per-rank loads differ.
// "Expert Parallelism (EP)", "Limitations" 3-4: rank r owns experts
// [r*E/R, (r+1)*E/R), so the expert-major row order is rank-major.
//
// Two launches:
//  1. dispatch_rank_kernel, one CTA per chunk of slots.  Chunks never straddle
//     a source rank (token t's source rank is t*R/T), so per-(source rank,
//     expert) counts are sums of whole chunks.  Each slot gets its stable rank
//     among same-expert slots of its chunk without atomics:
//     __match_any_sync groups a warp's lanes by expert, popc of the lower
//     peers gives the in-warp rank, and a per-expert scan over the warps adds
//     the earlier warps' counts.  The last CTA to finish (a fence + counter,
//     no waiting) turns the per-chunk counts into expert offsets, per-chunk
//     bases, rank counts and source-rank counts.
//  2. dispatch_scatter_kernel, one warp per (token, slice of 128 16-byte
//     columns): computes the token's k rows (the first slice also writes
//     slot_to_row / row_to_slot), reads its slice of the token row once and
//     stores it to the k rows with 16-byte vector accesses.
#pragma once

#include "common.cuh"

namespace moe {

struct DispatchGeom {
  int T, k, E, R, S;
  int chunk;    // slots per chunk (<= the 1024-thread CTA of kernel 1, a multiple of 32)
  int cpr;      // chunks per source rank
  int nchunks;  // R * cpr
  int counts_in_smem;  // the last CTA stages the [nchunks][E] counts in shared memory
};

constexpr size_t kDispatchCountsSmemMax = 96 * 1024;  // bytes of [nchunks][E] counts staged by the last CTA

// First token of source rank r: ceil(r*T/R), so that t*R/T == r on [lo(r), lo(r+1)).
__host__ __device__ __forceinline__ int src_rank_first_token(int r, int T, int R) {
  return (int)(((int64_t)r * T + R - 1) / R);
}

inline DispatchGeom make_dispatch_geom(int T, int k, int E, int R) {
  DispatchGeom g;
  g.T = T;
  g.k = k;
  g.E = E;
  g.R = R;
  g.S = T * k;
  const int max_tok = (T + R - 1) / R;  // largest source-rank range
  const int max_slots = max_tok * k;
  int ch = ((max_slots + 31) / 32) * 32;
  if (ch > 1024) ch = 1024;
  if (ch < 32) ch = 32;
  g.chunk = ch;
  g.cpr = (max_slots + ch - 1) / ch;
  if (g.cpr < 1) g.cpr = 1;
  g.nchunks = R * g.cpr;
  g.counts_in_smem = (size_t)g.nchunks * E * sizeof(int32_t) <= kDispatchCountsSmemMax;
  return g;
}

// Workspace layout (bytes): [0,256) control word; chunk_counts[nchunks][E];
// chunk_base[nchunks][E]; slot_rank[S].
struct DispatchWs {
  uint32_t* counter;
  int32_t* chunk_counts;
  int32_t* chunk_base;
  int32_t* slot_rank;
};

inline size_t dispatch_ws_bytes(const DispatchGeom& g) {
  return 256 + sizeof(int32_t) * ((size_t)2 * g.nchunks * g.E + (size_t)g.S);
}

inline DispatchWs dispatch_ws_carve(void* base, const DispatchGeom& g) {
  char* p = (char*)base;
  DispatchWs w;
  w.counter = (uint32_t*)p;
  w.chunk_counts = (int32_t*)(p + 256);
  w.chunk_base = w.chunk_counts + (size_t)g.nchunks * g.E;
  w.slot_rank = w.chunk_base + (size_t)g.nchunks * g.E;
  return w;
}

__device__ __forceinline__ void chunk_slot_range(const DispatchGeom& g, int c, int& s0, int& s1) {
  const int r = c / g.cpr, ci = c - r * g.cpr;
  const int lo = src_rank_first_token(r, g.T, g.R) * g.k;
  const int hi = src_rank_first_token(r + 1, g.T, g.R) * g.k;
  s0 = lo + ci * g.chunk;
  s1 = min(s0 + g.chunk, hi);
  if (s0 > hi) s0 = hi;
}

__device__ __forceinline__ int chunk_of_slot(const DispatchGeom& g, int s) {
  const int t = s / g.k;
  const int r = (int)(((int64_t)t * g.R) / g.T);
  const int lo = src_rank_first_token(r, g.T, g.R) * g.k;
  return r * g.cpr + (s - lo) / g.chunk;
}

// Dynamic shared memory: warp_counts[nwarps][E] int32, then E + 1 ints for the scan.
__global__ void __launch_bounds__(1024) dispatch_rank_kernel(
    DispatchGeom g, const int32_t* __restrict__ ids, DispatchWs ws, int32_t* __restrict__ expert_counts,
    int32_t* __restrict__ expert_offsets, int32_t* __restrict__ rank_counts, int32_t* __restrict__ rank_offsets,
    int32_t* __restrict__ src_expert_counts) {
  extern __shared__ int32_t smem_i32[];
  const int nwarps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = (int)lane_id();
  int32_t* warp_counts = smem_i32;  // [nwarps][E]
  size_t table = (size_t)nwarps * g.E;
  if (g.counts_in_smem && (size_t)g.nchunks * g.E > table) table = (size_t)g.nchunks * g.E;
  int32_t* scan = smem_i32 + table;  // [E + 1]
  __shared__ int s_is_last;

  pdl_wait();
  pdl_trigger();
  const int c = blockIdx.x;
  int s0, s1;
  chunk_slot_range(g, c, s0, s1);

  for (int i = threadIdx.x; i < nwarps * g.E; i += blockDim.x) warp_counts[i] = 0;
  __syncthreads();

  const int s = s0 + (int)threadIdx.x;
  int e = -2;  // -2: no slot; -1: bad id
  if (s < s1) {
    e = __ldg(ids + s);
    if (e < 0 || e >= g.E) {
      flag_error(kErrBadId);
      e = -1;
    }
  }
  const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
  const int rank_in_warp = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && lane == __ffs(peers) - 1) warp_counts[warp * g.E + e] = __popc(peers);
  __syncthreads();
  // exclusive scan over warps, per expert; totals are this chunk's counts
  for (int x = threadIdx.x; x < g.E; x += blockDim.x) {
    int run = 0;
    for (int w = 0; w < nwarps; ++w) {
      const int v = warp_counts[w * g.E + x];
      warp_counts[w * g.E + x] = run;
      run += v;
    }
    ws.chunk_counts[(size_t)c * g.E + x] = run;
  }
  __syncthreads();
  if (s < s1) ws.slot_rank[s] = (e >= 0) ? warp_counts[warp * g.E + e] + rank_in_warp : -1;

  // ---- last CTA: global scans (no CTA ever waits for another) ----
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_is_last = (atomicAdd(ws.counter, 1u) == (uint32_t)(g.nchunks - 1));
  __syncthreads();
  if (!s_is_last) return;
  __threadfence();

  // The per-chunk counts come back through L2; every read below is issued
  // independently of the running sums so that many are in flight at once.
  const int nce = g.nchunks * g.E;
  int32_t* cnt = smem_i32;  // warp_counts is dead here: reuse it for the [nchunks][E] counts
  if (g.counts_in_smem) {
#pragma unroll 4
    for (int i = threadIdx.x; i < nce; i += blockDim.x) cnt[i] = __ldcg(ws.chunk_counts + i);
    __syncthreads();
  }
  auto count_at = [&](int cc, int x) {
    return g.counts_in_smem ? cnt[cc * g.E + x] : __ldcg(ws.chunk_counts + (size_t)cc * g.E + x);
  };
  // 1. per-expert totals
  for (int x = threadIdx.x; x < g.E; x += blockDim.x) {
    int run = 0;
    for (int c0 = 0; c0 < g.nchunks; c0 += 8) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = (c0 + u < g.nchunks) ? count_at(c0 + u, x) : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) run += v[u];
    }
    scan[x] = run;
    expert_counts[x] = run;
  }
  __syncthreads();
  // 2. exclusive scan over experts (warp 0, 32 at a time)
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < g.E; base += 32) {
      const int v = (base + lane < g.E) ? scan[base + lane] : 0;
      int incl = v;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
      }
      if (base + lane < g.E) scan[base + lane] = carry + incl - v;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) scan[g.E] = carry;
  }
  __syncthreads();
  // 3. chunk bases = expert offset + counts of the same expert in earlier chunks
  for (int x = threadIdx.x; x < g.E; x += blockDim.x) {
    int run = scan[x];
    for (int c0 = 0; c0 < g.nchunks; c0 += 8) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = (c0 + u < g.nchunks) ? count_at(c0 + u, x) : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (c0 + u < g.nchunks) {
          ws.chunk_base[(size_t)(c0 + u) * g.E + x] = run;
          run += v[u];
        }
      }
    }
  }
  for (int x = threadIdx.x; x <= g.E; x += blockDim.x) expert_offsets[x] = scan[x];
  const int EL = g.E / g.R;
  for (int r = threadIdx.x; r < g.R; r += blockDim.x) {
    rank_counts[r] = scan[(r + 1) * EL] - scan[r * EL];
    rank_offsets[r] = scan[r * EL];
  }
  if (threadIdx.x == 0) rank_offsets[g.R] = scan[g.E];
  if (src_expert_counts) {
    for (int i = threadIdx.x; i < g.R * g.E; i += blockDim.x) {
      const int r = i / g.E, x = i - r * g.E;
      int sum = 0;
      for (int ci = 0; ci < g.cpr; ++ci) sum += count_at(r * g.cpr + ci, x);
      src_expert_counts[i] = sum;
    }
  }
  if (threadIdx.x == 0) *ws.counter = 0u;  // ready for the next call
}

constexpr int kScatterVecsPerLane = 4;                   // 16-byte vectors in flight per lane
constexpr int kScatterSlice = 32 * kScatterVecsPerLane;  // 16-byte vectors of a row per warp

template <typename T>
__global__ void __launch_bounds__(256) dispatch_scatter_kernel(DispatchGeom g, int H, int nslices,
                                                               const T* __restrict__ x,
                                                               const int32_t* __restrict__ ids, DispatchWs ws,
                                                               const int32_t* __restrict__ expert_offsets,
                                                               T* __restrict__ x_disp,
                                                               int32_t* __restrict__ slot_to_row,
                                                               int32_t* __restrict__ row_to_slot) {
  pdl_wait();
  pdl_trigger();
  const size_t gtid = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  // rows past the last placed row (only when ids were dropped) get row_to_slot = -1
  {
    const int placed = __ldg(expert_offsets + g.E);
    if (gtid < (size_t)(g.S - placed)) row_to_slot[placed + gtid] = -1;
  }
  // warp -> (token, column slice of kScatterSlice vectors)
  const size_t gw = gtid >> 5;
  const int t = (int)(gw / nslices), cs = (int)(gw - (size_t)t * nslices);
  const int lane = (int)lane_id();
  if (t >= g.T) return;

  int my_row = -1;
  if (lane < g.k) {
    const int s = t * g.k + lane;
    const int e = __ldg(ids + s);
    const int rk = ws.slot_rank[s];
    if (e >= 0 && e < g.E && rk >= 0) my_row = ws.chunk_base[(size_t)chunk_of_slot(g, s) * g.E + e] + rk;
    if (cs == 0) {
      slot_to_row[s] = my_row;
      if (my_row >= 0) row_to_slot[my_row] = s;
    }
  }
  int rows[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) rows[j] = __shfl_sync(0xFFFFFFFFu, my_row, j);

  constexpr int N = Vec16<T>::N;
  const int nvec = H / N;
  const char* src = reinterpret_cast<const char*>(x + (size_t)t * H);
  const int base = cs * kScatterSlice;
  uint4 v[kScatterVecsPerLane];
#pragma unroll
  for (int u = 0; u < kScatterVecsPerLane; ++u) {
    const int i = base + u * 32 + lane;
    if (i < nvec) v[u] = ld_nc_v4(src + (size_t)i * 16);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= g.k || rows[j] < 0) continue;
    char* dst = reinterpret_cast<char*>(x_disp + (size_t)rows[j] * H);
#pragma unroll
    for (int u = 0; u < kScatterVecsPerLane; ++u) {
      const int i = base + u * 32 + lane;
      if (i < nvec) st_v4(dst + (size_t)i * 16, v[u]);
    }
  }
}

template <typename T>
cudaError_t launch_dispatch(const DispatchGeom& g, int H, const T* x, const int32_t* ids, void* workspace,
                            T* x_disp, int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                            int32_t* rank_offsets, int32_t* slot_to_row, int32_t* row_to_slot,
                            int32_t* src_expert_counts, cudaStream_t stream) {
  DispatchWs ws = dispatch_ws_carve(workspace, g);
  const int threads1 = 1024;  // >= chunk: spare threads speed up the last CTA's scans
  size_t table = (size_t)(threads1 / 32) * g.E;  // warp_counts, later the staged chunk counts
  if (g.counts_in_smem && (size_t)g.nchunks * g.E > table) table = (size_t)g.nchunks * g.E;
  const size_t smem1 = sizeof(int32_t) * (table + g.E + 1);
  if (smem1 > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(dispatch_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem1);
    if (err != cudaSuccess) return err;
  }
  cudaError_t err = launch_pdl(dispatch_rank_kernel, g.nchunks, threads1, smem1, stream, g, ids, ws, expert_counts,
                               expert_offsets, rank_counts, rank_offsets, src_expert_counts);
  if (err == cudaSuccess) err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int threads2 = 256;
  const int nvec = H / Vec16<T>::N;
  const int nslices = (nvec + kScatterSlice - 1) / kScatterSlice;
  const size_t warps = (size_t)g.T * nslices;
  const int blocks2 = (int)((warps * 32 + threads2 - 1) / threads2);
  if (blocks2 > 0) {
    err = launch_pdl(dispatch_scatter_kernel<T>, blocks2, threads2, 0, stream, g, H, nslices, x, ids, ws,
                     expert_offsets, x_disp, slot_to_row, row_to_slot);
    if (err != cudaSuccess) return err;
  }
  return cudaGetLastError();
}

}  // namespace moe
