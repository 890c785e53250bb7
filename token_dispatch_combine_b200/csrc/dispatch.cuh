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
// One cooperative launch (every CTA resident at once), three phases split by
// one or two bounded grid barriers (a counted dispatch with a small count
// table has none, and is launched plainly):
//  1. per chunk of <= 512 slots (chunks never straddle a source rank, token
//     t's source rank being t*R/T): each slot's stable rank among the
//     same-expert slots of its chunk, without atomics -- __match_any_sync
//     groups a warp's lanes by expert, popc of the lower peers gives the
//     in-warp rank, a per-expert scan over the CTA's warps adds the earlier
//     warps' counts -- and the chunk's per-expert counts;
//  2. per-chunk bases (earlier chunks' counts of the same expert) and expert
//     offsets: when the [chunks][E] count table is small (<= 8192 entries)
//     every CTA loads it into shared memory and scans it itself; otherwise one
//     warp per expert scans its column (warp prefix sums, 32 chunks a round)
//     and, after a second barrier, every CTA scans the E totals;
//  3. each CTA owns a contiguous range of tokens: one thread per slot computes
//     the slot's row (offset + chunk base + in-chunk rank) into shared memory
//     and writes the permutation, then one warp per (token, slice of 128
//     16-byte columns) copies its slice of the token row to the k rows with
//     16-byte vector accesses.  Before phase 1 each CTA asks L2 for its token
//     rows of x and each warp loads its first slice, so those reads overlap
//     the counting and the barriers.
// With x_disp == nullptr (index-only dispatch, for a gate/up GEMM that gathers
// its rows from x itself) phase 3 writes only the permutation.
// A barrier that does not complete within its limit (1 s for moe_dispatch)
// sets the timeout bit of the device error word; the CTA then skips the rest
// of its work.  Every CTA, on every path, ends by arriving on an exit counter,
// and the last one out zeroes the barrier's arrival counter and the exit
// counter: a call that timed out leaves the workspace ready for the next one.
#pragma once

#include "common.cuh"
#include "route.cuh"

namespace moe {

constexpr int kDispatchThreads = 512;
// CTAs of the dispatch kernel resident per SM: 2 caps it at 64 registers per
// thread (no spills), twice the warps -- and the bytes in flight -- of the 84
// registers it takes unbounded (one CTA per SM).
#ifndef MOE_DISPATCH_MIN_BLOCKS
#define MOE_DISPATCH_MIN_BLOCKS 2
#endif
constexpr int kDispatchWarps = kDispatchThreads / 32;
constexpr int kScatterVecsPerLane = 4;                   // 16-byte vectors in flight per lane
constexpr int kScatterSlice = 32 * kScatterVecsPerLane;  // 16-byte vectors of a row per warp item
constexpr int kRowRound = kDispatchThreads / 8;          // tokens per phase-3 round: one slot per thread at k <= 8
constexpr uint64_t kGridBarrierLimitNs = 1000000000ull;   // 1 s: the limit of every moe_dispatch call
// Count tables up to this many entries are scanned by every CTA in shared
// memory, which saves the second grid barrier.
constexpr size_t kSmallCountTable = 8192;

// Chunk size of the counted pair (moe_route_count / moe_dispatch_counted):
// small chunks give the routing kernel, a CTA per chunk, a warp per token.
constexpr int kCountedChunk = 128;

// A small count table is held transposed in shared memory, expert-major with
// an odd row stride (no bank conflicts on either access pattern).
__host__ __device__ __forceinline__ int dispatch_table_ld(int nchunks) { return nchunks | 1; }

__host__ __device__ __forceinline__ size_t dispatch_smem_table(int nchunks, int E) {
  const size_t warps = (size_t)kDispatchWarps * E, table = (size_t)nchunks * E;
  const size_t held = (size_t)dispatch_table_ld(nchunks) * E;
  return (table <= kSmallCountTable && held > warps) ? held : warps;
}

struct DispatchGeom {
  int T, k, E, R, S;
  int chunk;    // slots per chunk (<= kDispatchThreads, a multiple of 32)
  int cpr;      // chunks per source rank
  int nchunks;  // R * cpr
};

// First token of source rank r: ceil(r*T/R), so that t*R/T == r on [lo(r), lo(r+1)).
__host__ __device__ __forceinline__ int src_rank_first_token(int r, int T, int R) {
  return (int)(((int64_t)r * T + R - 1) / R);
}

// max_chunk: kDispatchThreads (moe_dispatch), kCountedChunk (the counted pair).
inline DispatchGeom make_dispatch_geom(int T, int k, int E, int R, int max_chunk = kDispatchThreads) {
  DispatchGeom g;
  g.T = T;
  g.k = k;
  g.E = E;
  g.R = R;
  g.S = T * k;
  const int max_tok = (T + R - 1) / R;  // largest source-rank range
  const int max_slots = max_tok * k;
  int ch = ((max_slots + 31) / 32) * 32;
  if (ch > max_chunk) ch = max_chunk;
  if (ch < 32) ch = 32;
  g.chunk = ch;
  g.cpr = (max_slots + ch - 1) / ch;
  if (g.cpr < 1) g.cpr = 1;
  g.nchunks = R * g.cpr;
  return g;
}

// Workspace layout (bytes): [0,256) control words (grid-barrier arrival count
// at 64, generation at 128, exit count at 192; the two counts are zero
// between calls, the generation takes any value); chunk_counts[nchunks][E];
// chunk_base[nchunks][E] (relative to the expert's offset); slot_rank[S];
// totals[E].
constexpr size_t kDispatchBarCountOffset = 64;
struct DispatchWs {
  uint32_t* bar_count;
  uint32_t* bar_gen;
  uint32_t* exit_count;
  int32_t* chunk_counts;
  int32_t* chunk_base;
  int32_t* slot_rank;
  int32_t* totals;
};

inline size_t dispatch_ws_bytes(const DispatchGeom& g) {
  return 256 + sizeof(int32_t) * ((size_t)2 * g.nchunks * g.E + (size_t)g.S + (size_t)g.E);
}

inline DispatchWs dispatch_ws_carve(void* base, const DispatchGeom& g) {
  char* p = (char*)base;
  DispatchWs w;
  w.bar_count = (uint32_t*)(p + kDispatchBarCountOffset);
  w.bar_gen = (uint32_t*)(p + 128);
  w.exit_count = (uint32_t*)(p + 192);
  w.chunk_counts = (int32_t*)(p + 256);
  w.chunk_base = w.chunk_counts + (size_t)g.nchunks * g.E;
  w.slot_rank = w.chunk_base + (size_t)g.nchunks * g.E;
  w.totals = w.slot_rank + (size_t)g.S;
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

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier for a cooperative launch.  Thread 0 of each CTA reads the
// generation, arrives on the counter; the last arrival resets the counter and
// bumps the generation; the others wait (at most limit_ns) for the bump.
// Returns false, with the timeout bit set, if the wait gave up.
__device__ __forceinline__ bool grid_barrier(const DispatchWs& ws, int* s_ok, uint64_t limit_ns) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t gen = ld_acquire_u32(ws.bar_gen);
    __threadfence();
    const uint32_t arrived = atomicAdd(ws.bar_count, 1u);
    if (arrived == gridDim.x - 1) {
      atomicExch(ws.bar_count, 0u);
      __threadfence();
      atomicAdd(ws.bar_gen, 1u);
    } else {
      const uint64_t t0 = globaltimer_ns();
      while (ld_acquire_u32(ws.bar_gen) == gen) {
        if (globaltimer_ns() - t0 > limit_ns) {
          flag_error(kErrTimeout);
          *s_ok = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
  }
  __syncthreads();
  return *s_ok != 0;
}

// Phase 1 for chunk c: each slot's stable rank among the same-expert slots of
// the chunk, without atomics (__match_any_sync groups a warp's lanes by
// expert, popc of the lower peers gives the in-warp rank, a per-expert scan
// over the CTA's warps adds the earlier warps' counts), into ws.slot_rank; the
// chunk's per-expert counts into ws.chunk_counts.  id_of(s) is slot s's
// expert id; ids outside [0, E) are dropped and flagged (a -1 silently when
// allow_pad).  NW: warps of the block (at least kDispatchWarps, so that
// every slot of a chunk has a thread); warp_counts: [NW][E] ints of shared
// memory.
template <int NW, typename IdOf>
__device__ __forceinline__ void count_chunk(const DispatchGeom& g, int c, const DispatchWs& ws, int32_t* warp_counts,
                                            int allow_pad, IdOf id_of) {
  static_assert(NW >= kDispatchWarps, "a thread per slot of a chunk");
  constexpr int NT = NW * 32;
  const int warp = threadIdx.x >> 5, lane = (int)lane_id();
  int s0, s1;
  chunk_slot_range(g, c, s0, s1);
  for (int i = threadIdx.x; i < NW * g.E; i += NT) warp_counts[i] = 0;
  __syncthreads();
  const int s = s0 + (int)threadIdx.x;
  int e = -2;  // -2: no slot; -1: bad id
  if (s < s1) {
    e = id_of(s);
    if (e < 0 || e >= g.E) {
      if (!(allow_pad && e == -1)) flag_error(kErrBadId);  // -1 is padding where allowed
      e = -1;
    }
  }
  const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
  const int rank_in_warp = __popc(peers & ((1u << lane) - 1u));
  if (e >= 0 && lane == __ffs(peers) - 1) warp_counts[warp * g.E + e] = __popc(peers);
  __syncthreads();
  for (int xx = threadIdx.x; xx < g.E; xx += NT) {  // exclusive scan over warps, per expert
    int run = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const int v = warp_counts[w * g.E + xx];
      warp_counts[w * g.E + xx] = run;
      run += v;
    }
    ws.chunk_counts[(size_t)c * g.E + xx] = run;
  }
  __syncthreads();
  if (s < s1) ws.slot_rank[s] = (e >= 0) ? warp_counts[warp * g.E + e] + rank_in_warp : -1;
  __syncthreads();  // warp_counts is reused by the next chunk
}

// Last step of every CTA on every path (thread 0 only, after its last barrier
// operation): arrive on the exit counter; the last CTA out zeroes the arrival
// and exit counters.  A barrier that timed out leaves a partial arrival count
// behind, so without this the next call on the workspace would start from it.
__device__ __forceinline__ void dispatch_exit(const DispatchWs& ws) {
  if (threadIdx.x != 0) return;
  __threadfence();
  if (atomicAdd(ws.exit_count, 1u) == gridDim.x - 1) {
    atomicExch(ws.bar_count, 0u);
    atomicExch(ws.exit_count, 0u);
    __threadfence();
  }
}

// Dynamic shared memory: warp_counts[kDispatchWarps][E] int32 (or the whole
// [nchunks][E] table when it is small and larger), then offs[E + 1], then the
// rows of one round of this CTA's slots, rows[kDispatchThreads].
template <typename T>
__device__ __forceinline__ void dispatch_phases(
    const DispatchGeom& g, int H, int nslices, int tpc, const T* __restrict__ x, const int32_t* __restrict__ ids,
    const DispatchWs& ws, uint64_t limit_ns, int allow_pad, int counted, T* __restrict__ x_disp,
    int32_t* __restrict__ expert_counts,
    int32_t* __restrict__ expert_offsets, int32_t* __restrict__ rank_counts, int32_t* __restrict__ rank_offsets,
    int32_t* __restrict__ slot_to_row, int32_t* __restrict__ row_to_slot, int32_t* __restrict__ src_expert_counts) {
  extern __shared__ int32_t smem_i32[];
  int32_t* warp_counts = smem_i32;                                    // [kDispatchWarps][E]
  int32_t* offs = smem_i32 + dispatch_smem_table(g.nchunks, g.E);     // [E + 1]
  int32_t* s_rows = offs + g.E + 1;                                    // [kDispatchThreads]
  const bool small_table = (size_t)g.nchunks * g.E <= kSmallCountTable;
  const int ld = dispatch_table_ld(g.nchunks);
  int32_t* cbase = smem_i32;  // small_table: [E][ld] chunk bases, expert-major (reuses warp_counts)
  __shared__ int s_ok;
  // ---- this CTA's tokens [tb, te): ask L2 for their rows of x.  A prefetch
  // changes no data, so it may run before the previous kernel has finished.
  constexpr int N = Vec16<T>::N;
  const int nvec = H / N;
  const int tb = min(g.T, (int)blockIdx.x * tpc), te = min(g.T, tb + tpc);
  const bool copy_rows = x_disp != nullptr;  // index-only dispatch leaves the rows where they are
  if (copy_rows && threadIdx.x == 0 && te > tb) {
    const char* base = reinterpret_cast<const char*>(x + (size_t)tb * H);
    const size_t bytes = (size_t)(te - tb) * H * sizeof(T);  // a multiple of 16 (H * sizeof(T) is)
    for (size_t b = 0; b < bytes; b += 65536) {
      const uint32_t n = (uint32_t)min((size_t)65536, bytes - b);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + b), "r"(n) : "memory");
    }
  }
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = (int)lane_id();
  const size_t gwarp = (size_t)blockIdx.x * kDispatchWarps + warp;
  const size_t nwarps_grid = (size_t)gridDim.x * kDispatchWarps;
  const size_t gtid = (size_t)blockIdx.x * kDispatchThreads + threadIdx.x;
  const size_t nthreads_grid = (size_t)gridDim.x * kDispatchThreads;
  if (threadIdx.x == 0) s_ok = 1;

  // ---- each warp's first slice of x into registers (it does not depend on the counts)
  uint4 pre[kScatterVecsPerLane];
  const int pre_tok = tb + warp / nslices, pre_cs = warp % nslices;
  if (copy_rows && pre_tok < min(te, tb + kRowRound)) {
    const char* src = reinterpret_cast<const char*>(x + (size_t)pre_tok * H);
#pragma unroll
    for (int u = 0; u < kScatterVecsPerLane; ++u) {
      const int i = pre_cs * kScatterSlice + u * 32 + lane;
      if (i < nvec) pre[u] = ld_nc_v4(src + (size_t)i * 16);
    }
  }

  // ---- phase 1: per-chunk stable ranks and counts (already in the workspace when `counted`:
  // the routing kernel did them, route_count_kernel)
  if (!counted) {
    for (int c = blockIdx.x; c < g.nchunks; c += gridDim.x)
      count_chunk<kDispatchWarps>(g, c, ws, warp_counts, allow_pad, [&](int s) { return __ldg(ids + s); });
    if (!grid_barrier(ws, &s_ok, limit_ns)) return;
  }

  if (small_table) {
    // ---- phase 2 (small count table): every CTA scans the whole table itself
    for (int i = threadIdx.x; i < g.nchunks * g.E; i += kDispatchThreads) {  // transposed into shared memory
      const int c = i / g.E, xx = i - c * g.E;
      cbase[xx * ld + c] = __ldcg(ws.chunk_counts + i);
    }
    __syncthreads();
    for (int xx = warp; xx < g.E; xx += kDispatchWarps) {  // warp per expert, prefix over chunks
      int carry = 0;
      for (int base = 0; base < g.nchunks; base += 32) {
        const int c = base + lane;
        const int v = (c < g.nchunks) ? cbase[xx * ld + c] : 0;
        int incl = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
          if (lane >= d) incl += y;
        }
        if (c < g.nchunks) cbase[xx * ld + c] = carry + incl - v;
        carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
      if (lane == 0) {
        offs[xx] = carry;
        if (blockIdx.x == 0) expert_counts[xx] = carry;
      }
    }
  } else {
  // ---- phase 2a: one warp per expert, prefix over chunks
  for (size_t e = gwarp; e < (size_t)g.E; e += nwarps_grid) {
    int carry = 0;
    for (int base = 0; base < g.nchunks; base += 32) {
      const int c = base + lane;
      const int v = (c < g.nchunks) ? __ldcg(ws.chunk_counts + (size_t)c * g.E + e) : 0;
      int incl = v;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
      }
      if (c < g.nchunks) ws.chunk_base[(size_t)c * g.E + e] = carry + incl - v;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) {
      ws.totals[e] = carry;
      expert_counts[e] = carry;
    }
  }
  if (!grid_barrier(ws, &s_ok, limit_ns)) return;

  // ---- phase 2b: expert offsets (every CTA, in shared memory)
  for (int xx = threadIdx.x; xx < g.E; xx += kDispatchThreads) offs[xx] = __ldcg(ws.totals + xx);
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < g.E; base += 32) {
      const int v = (base + lane < g.E) ? offs[base + lane] : 0;
      int incl = v;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += y;
      }
      if (base + lane < g.E) offs[base + lane] = carry + incl - v;
      carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) offs[g.E] = carry;
  }
  __syncthreads();
  const int placed = offs[g.E];
  if (blockIdx.x == 0) {
    for (int xx = threadIdx.x; xx <= g.E; xx += kDispatchThreads) expert_offsets[xx] = offs[xx];
    const int EL = g.E / g.R;
    if (rank_counts != nullptr) {  // (NULL only from internal one-rank calls)
      for (int r = threadIdx.x; r < g.R; r += kDispatchThreads) {
        rank_counts[r] = offs[(r + 1) * EL] - offs[r * EL];
        rank_offsets[r] = offs[r * EL];
      }
      if (threadIdx.x == 0) rank_offsets[g.R] = placed;
    }
  }
  if (src_expert_counts) {  // a source rank's chunks are contiguous: differences of the chunk bases
    if (small_table) {
      if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < g.R * g.E; i += kDispatchThreads) {
          const int r = i / g.E, xx = i - r * g.E;
          const int lo = cbase[xx * ld + r * g.cpr];
          const int hi = (r + 1 < g.R) ? cbase[xx * ld + (r + 1) * g.cpr] : offs[xx + 1] - offs[xx];
          src_expert_counts[i] = hi - lo;
        }
      }
    } else {
      for (size_t i = gtid; i < (size_t)g.R * g.E; i += nthreads_grid) {
        const int r = (int)(i / g.E), xx = (int)(i - (size_t)r * g.E);
        const int lo = __ldcg(ws.chunk_base + (size_t)(r * g.cpr) * g.E + xx);
        const int hi = (r + 1 < g.R) ? __ldcg(ws.chunk_base + (size_t)((r + 1) * g.cpr) * g.E + xx)
                                     : offs[xx + 1] - offs[xx];
        src_expert_counts[i] = hi - lo;
      }
    }
  }
  // rows past the last placed row (only when ids were dropped) get row_to_slot = -1
  for (size_t i = gtid; i < (size_t)(g.S - placed); i += nthreads_grid) row_to_slot[placed + i] = -1;

  // ---- phase 3: this CTA's tokens, kRowRound at a time
  for (int r0 = tb; r0 < te; r0 += kRowRound) {
    const int r1 = min(r0 + kRowRound, te);
    const int nslot = (r1 - r0) * g.k;
    if ((int)threadIdx.x < nslot) {
      const int s = r0 * g.k + (int)threadIdx.x;
      const int e = __ldg(ids + s);
      const int rk = __ldcg(ws.slot_rank + s);
      int row = -1;
      if (e >= 0 && e < g.E && rk >= 0) {
        const int c = chunk_of_slot(g, s);
        row = offs[e] + (small_table ? cbase[e * ld + c] : __ldcg(ws.chunk_base + (size_t)c * g.E + e)) + rk;
        if (row >= offs[e + 1]) {  // counts that do not belong to these ids: never leave the segment
          flag_error(kErrBadOffsets);
          row = -1;
        }
      }
      s_rows[threadIdx.x] = row;
      slot_to_row[s] = row;
      if (row >= 0) row_to_slot[row] = s;
    }
    __syncthreads();
    const int nit = copy_rows ? (r1 - r0) * nslices : 0;
    for (int item = warp; item < nit; item += kDispatchWarps) {
      const int tl = item / nslices, cs = item - tl * nslices;
      uint4 v[kScatterVecsPerLane];
      if (r0 == tb && item == warp) {  // the slice loaded before phase 1
#pragma unroll
        for (int u = 0; u < kScatterVecsPerLane; ++u) v[u] = pre[u];
      } else {
        const char* src = reinterpret_cast<const char*>(x + (size_t)(r0 + tl) * H);
#pragma unroll
        for (int u = 0; u < kScatterVecsPerLane; ++u) {
          const int i = cs * kScatterSlice + u * 32 + lane;
          if (i < nvec) v[u] = ld_nc_v4(src + (size_t)i * 16);
        }
      }
      for (int j = 0; j < g.k; ++j) {
        const int row = s_rows[tl * g.k + j];
        if (row < 0) continue;
        char* dst = reinterpret_cast<char*>(x_disp + (size_t)row * H);
#pragma unroll
        for (int u = 0; u < kScatterVecsPerLane; ++u) {
          const int i = cs * kScatterSlice + u * 32 + lane;
          if (i < nvec) st_v4(dst + (size_t)i * 16, v[u]);
        }
      }
    }
    __syncthreads();  // s_rows is reused by the next round
  }
}

template <typename T>
__global__ void __launch_bounds__(kDispatchThreads, MOE_DISPATCH_MIN_BLOCKS) dispatch_kernel(
    DispatchGeom g, int H, int nslices, int tpc, const T* __restrict__ x, const int32_t* __restrict__ ids, DispatchWs ws,
    uint64_t limit_ns, int allow_pad, int counted, T* __restrict__ x_disp, int32_t* __restrict__ expert_counts,
    int32_t* __restrict__ expert_offsets, int32_t* __restrict__ rank_counts, int32_t* __restrict__ rank_offsets,
    int32_t* __restrict__ slot_to_row, int32_t* __restrict__ row_to_slot, int32_t* __restrict__ src_expert_counts) {
  dispatch_phases<T>(g, H, nslices, tpc, x, ids, ws, limit_ns, allow_pad, counted, x_disp, expert_counts,
                     expert_offsets, rank_counts, rank_offsets, slot_to_row, row_to_slot, src_expert_counts);
  dispatch_exit(ws);
}

// moe_route_count: the routing of moe_route fused with phase 1 of the
// dispatch.  One CTA per dispatch chunk (the same geometry, so the counts
// land where a counted dispatch reads them): its warps route the tokens that
// have slots in the chunk (a warp per token, warp_topk_softmax; a token whose
// slots straddle two chunks is routed by both, identically), write the
// chunk's slots of topk_ids / topk_w and keep their ids in shared memory;
// then count_chunk ranks and counts the chunk.  Each warp loads the logits of
// its next token before routing the current one (E <= 256).
// 1024 threads (512 above 256 experts, whose logits take twice the
// registers): that many routing warps, then the counting with a thread per
// slot.  Dynamic shared memory: warp_counts[warps][E], then ids[chunk].
template <int VPL>
struct RouteCountCfg {
  static constexpr int kThreads = VPL >= 16 ? 512 : 1024;
  static constexpr int kWarps = kThreads / 32;
};
template <int VPL>
__global__ void __launch_bounds__(RouteCountCfg<VPL>::kThreads) route_count_kernel(DispatchGeom g,
                                                                                  const float* __restrict__ logits,
                                                                                  int32_t* __restrict__ topk_ids,
                                                                                  float* __restrict__ topk_w,
                                                                                  DispatchWs ws) {
  constexpr int kRouteCountWarps = RouteCountCfg<VPL>::kWarps;
  extern __shared__ int32_t smem_i32[];
  int32_t* warp_counts = smem_i32;
  int32_t* s_ids = smem_i32 + kRouteCountWarps * g.E;
  pdl_wait();
  pdl_trigger();
  const int c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = (int)lane_id();
  int s0, s1;
  chunk_slot_range(g, c, s0, s1);
  const int t0 = s0 / g.k, t1 = s1 > s0 ? (s1 + g.k - 1) / g.k : t0;
  float val[VPL], nval[VPL];
  auto load = [&](int t, float (&v)[VPL]) {
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      const int e = lane + 32 * q;
      v[q] = (t < t1 && e < g.E) ? __ldg(logits + (size_t)t * g.E + e) : 0.0f;
    }
  };
  constexpr bool kPrefetch = VPL <= 8;  // (more experts: the second register set would spill)
  if (kPrefetch) load(t0 + warp, val);
  for (int t = t0 + warp; t < t1; t += kRouteCountWarps) {
    if (kPrefetch) load(t + kRouteCountWarps, nval);  // the next token's logits in flight while this one is routed
    else load(t, val);
    uint32_t key[VPL];
#pragma unroll
    for (int q = 0; q < VPL; ++q) key[q] = (lane + 32 * q < g.E) ? logit_order_key(val[q]) : 0u;
    int my_id;
    float my_w;
    warp_topk_softmax<VPL>(key, val, g.k, lane, my_id, my_w);
    const int s = t * g.k + lane;
    if (lane < g.k && s >= s0 && s < s1) {
      topk_ids[s] = my_id;
      topk_w[s] = my_w;
      s_ids[s - s0] = my_id;
    }
    if (kPrefetch) {
#pragma unroll
      for (int q = 0; q < VPL; ++q) val[q] = nval[q];
    }
  }
  __syncthreads();
  count_chunk<kRouteCountWarps>(g, c, ws, warp_counts, 0, [&](int s) { return s_ids[s - s0]; });
}

inline cudaError_t launch_route_count(const DispatchGeom& g, const float* logits, int32_t* ids, float* w,
                                      void* workspace, cudaStream_t stream) {
  if (g.T == 0) return cudaSuccess;
  const DispatchWs ws = dispatch_ws_carve(workspace, g);
  const int vpl = (g.E + 31) / 32;
  const int dev = current_device();
  cudaError_t err = cudaSuccess;
#define MOE_ROUTE_COUNT_CASE(V)                                                                              \
  case V: {                                                                                                  \
    constexpr int NW = RouteCountCfg<V>::kWarps;                                                             \
    const size_t smem = sizeof(int32_t) * ((size_t)NW * g.E + kDispatchThreads);                            \
    static PerDeviceOnce attr_once; /* shared memory for the largest E of this case */                      \
    err = attr_once.run(dev, [&] {                                                                           \
      return cudaFuncSetAttribute(route_count_kernel<V>, cudaFuncAttributeMaxDynamicSharedMemorySize,        \
                                  (int)(sizeof(int32_t) * ((size_t)NW * 32 * V + kDispatchThreads)));        \
    });                                                                                                      \
    if (err == cudaSuccess)                                                                                  \
      err = launch_pdl(route_count_kernel<V>, dim3(g.nchunks), dim3(NW * 32), smem, stream, g, logits, ids, w, ws); \
    break;                                                                                                   \
  }
  switch (vpl <= 1 ? 1 : vpl <= 2 ? 2 : vpl <= 4 ? 4 : vpl <= 8 ? 8 : vpl <= 16 ? 16 : 32) {
    MOE_ROUTE_COUNT_CASE(1)
    MOE_ROUTE_COUNT_CASE(2)
    MOE_ROUTE_COUNT_CASE(4)
    MOE_ROUTE_COUNT_CASE(8)
    MOE_ROUTE_COUNT_CASE(16)
    MOE_ROUTE_COUNT_CASE(32)
  }
#undef MOE_ROUTE_COUNT_CASE
  return err != cudaSuccess ? err : cudaGetLastError();
}

// limit_ns bounds each grid-barrier wait (kGridBarrierLimitNs for moe_dispatch).  allow_pad:
// an id of -1 is padding (dropped like a bad id, but not flagged).  counted: phase 1's counts
// and ranks are already in the workspace (route_count_kernel), so phase 1 and its barrier
// are skipped.
template <typename T>
cudaError_t launch_dispatch(const DispatchGeom& g, int H, const T* x, const int32_t* ids, void* workspace,
                            T* x_disp, int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                            int32_t* rank_offsets, int32_t* slot_to_row, int32_t* row_to_slot,
                            int32_t* src_expert_counts, cudaStream_t stream, uint64_t limit_ns = kGridBarrierLimitNs,
                            bool allow_pad = false, bool counted = false) {
  DispatchWs ws = dispatch_ws_carve(workspace, g);
  auto kern = dispatch_kernel<T>;
  const size_t smem = sizeof(int32_t) * (dispatch_smem_table(g.nchunks, g.E) + g.E + 1 + kDispatchThreads);
  const int dev = current_device();
  static PerDeviceOnce attr_once;  // raise the shared-memory limit once per device, for the largest E
  cudaError_t err = attr_once.run(dev, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(sizeof(int32_t) * (dispatch_smem_table(1, 1024) + 1025 + kDispatchThreads)));
    // (the largest need: the [16][1024] warp counts; a small table is at most 8192 + E entries)
  });
  if (err != cudaSuccess) return err;
  // Co-residency bound of the cooperative grid for this shared-memory size.
  int per_sm = 0, sms = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDispatchThreads, smem);
  if (err != cudaSuccess) return err;
  err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (err != cudaSuccess) return err;
  const long long cap = (long long)per_sm * sms;
  if (cap < 1) return cudaErrorCooperativeLaunchTooLarge;
  const int nvec = H / Vec16<T>::N;
  const int nslices = (nvec + kScatterSlice - 1) / kScatterSlice;
  // phase 3: a CTA takes a contiguous token range; as many CTAs as keep every
  // warp at one (token, slice) item, within the co-residency bound (index
  // only: one round of kRowRound tokens per CTA)
  int tpc_one = kDispatchWarps / nslices > 0 ? kDispatchWarps / nslices : 1;
  if (x_disp == nullptr) tpc_one = kRowRound;
  const long long item_ctas = ((long long)g.T + tpc_one - 1) / tpc_one;
  long long want = item_ctas > g.nchunks ? item_ctas : (long long)g.nchunks;
  if (want < 1) want = 1;
  const int grid = (int)(want < cap ? want : cap);
  const int tpc = (g.T + grid - 1) / grid;  // tokens per CTA in phase 3

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kDispatchThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // A counted dispatch with a small count table never waits on a grid barrier,
  // so it needs no co-residency: a plain launch lets its CTAs start as the
  // previous kernel's SMs free up.  Every other form is a cooperative launch.
  const bool grid_sync = !(counted && (size_t)g.nchunks * g.E <= kSmallCountTable);
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (grid_sync) {
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na].val.cooperative = 1;
    ++na;
  }
  if (MOE_PDL) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  err = cudaLaunchKernelEx(&cfg, kern, g, H, nslices, tpc, x, ids, ws, limit_ns, (int)allow_pad, (int)counted, x_disp,
                           expert_counts, expert_offsets, rank_counts, rank_offsets, slot_to_row, row_to_slot,
                           src_expert_counts);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
