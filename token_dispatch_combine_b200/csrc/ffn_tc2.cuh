// Grouped SwiGLU expert MLP on CTA pairs (tcgen05 cta_group::2), bf16 in,
// float32 accumulate.  Same arithmetic and operand layouts as ffn_tc.cuh; the
// difference is that two SMs of a cluster work on one 256-row tile:
//   - each CTA loads its own 128 rows of A and its half of the B tile into its
//     own shared memory: for the gate/up projection the gate and up columns of
//     64 h columns ([gate 64 | up 64]), for the down projection 128 output
//     columns;
//   - the leader CTA's single MMA thread issues M=256 N=256 UMMAs that read
//     both CTAs' shared memory and write each CTA's 128 rows into that CTA's
//     TMEM;
//   - both CTAs' TMA loads complete on the leader's "full" barrier; the
//     leader's commits arrive on both CTAs' "empty" and "accumulator full"
//     barriers (tcgen05.commit multicast); each CTA's epilogue reads its own
//     TMEM and arrives on the leader's "accumulator empty" barrier.
// An expert's last tile, when at most 128 rows are left, is an M=128 pair MMA
// (64 rows per CTA).
// Gathering form: each CTA's gather threads copy its own A rows from x
// (cp.async) and arrive on its own full barrier; in the peer an otherwise idle
// thread (warp 1) waits for that barrier and arrives on the leader's, which
// the MMA thread waits on.
// Per CTA a stage is 16 KB of A + 16 KB of B, so the ring holds 6 stages
// (half the weight bytes per SM of the single-CTA kernel, 50% more time of
// work in flight).  No TMA multicast: every load brings one CTA's own data.
// Every mbarrier wait is bounded as in ffn_tc.cuh.
#pragma once

#include "ffn_tc.cuh"

namespace moe {
namespace tc {

constexpr int BM2 = 256;  // rows of a pair tile (128 per CTA)

// Pair m-tiles per raster group (tiles of a group share weight columns in L2).
#ifndef MOE_TC2_GROUP_M
#define MOE_TC2_GROUP_M 8
#endif

// Gathering pair kernel: semantics of the peer relay's arrival on the
// leader's barrier: 0 release at CTA scope (mbarrier.arrive's default),
// 1 relaxed, 2 release at cluster scope (measured: 2.4x slower kernel, the
// cluster-scope release waits for the peer's copies still in flight).
#ifndef MOE_TC2_RELAY
#define MOE_TC2_RELAY 0
#endif

// An expert's last tile with at most 128 rows left runs as an M=128 pair MMA
// (64 rows per CTA) instead of a half-empty M=256 one.
#ifndef MOE_TC2_HALF
#define MOE_TC2_HALF 1
#endif
// TMEM layout of an M=128 pair MMA in each CTA: its 64 rows are folded over
// the 128 lanes, the D columns supplied by the leader's B half in lanes 0-63
// and those of the peer's B half in lanes 64-127, both in columns 0..N/2-1.

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Arrive on a barrier of another CTA of the cluster with release ordering at
// CTA scope only (the default semantics of mbarrier.arrive), or none.
__device__ __forceinline__ void mbar_arrive_remote_cta_release(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA into this CTA's shared memory, completion counted on an mbarrier that may
// live in the peer CTA (cta_group::2; not a multicast load).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the barrier at this shared-memory offset in every CTA of `mask`
// once all earlier MMAs of this thread have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

template <bool GATEUP>
struct Cfg2 {
  static constexpr int BN = GATEUP ? 128 : 256;     // output columns of a tile (gate/up: h columns)
  static constexpr int MMA_N = 256;                 // gate/up: [gate 128 | up 128]
  static constexpr int NBOX = 2;                    // 64-column B boxes per CTA (its half of MMA_N)
  static constexpr uint32_t kBBytes = NBOX * kBoxBytes;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;  // per CTA
  static constexpr int STAGES = 6;
  static constexpr size_t smem_bytes(int E) {
    return 1024 + (size_t)STAGES * kStageBytes + 256 + sizeof(int32_t) * (3 * ((size_t)E + 1) + 1);
  }
};

template <bool GATEUP, bool GATHER = false>
__global__ void __launch_bounds__(GATHER ? kThreads + kGatherThreads : kThreads, 1)
    grouped_gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_a64,
                            const __grid_constant__ CUtensorMap tmap_b0, const __grid_constant__ CUtensorMap tmap_b1,
                            Params p) {
  using C = Cfg2<GATEUP>;
  constexpr int STAGES = C::STAGES;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + (size_t)STAGES * kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + (size_t)STAGES * C::kBBytes);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int32_t* s_seg = reinterpret_cast<int32_t*>(smem + (size_t)STAGES * C::kStageBytes + 256);
  int32_t* s_pre = s_seg + (p.E + 1);
  int32_t* s_grp = s_pre + (p.E + 1);  // [E + 2]: raster group starts (m-tiles), count at [E + 1]

  const int warp = threadIdx.x >> 5, lane = (int)lane_id();
  const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs), 1: peer
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto tfull_bar = [&](int a) { return smem_u32(bars + 2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return smem_u32(bars + 2 * STAGES + 2 + a); };
  const uint32_t drain_bar = smem_u32(bars + 2 * STAGES + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // leader's copy: its own arrive_expect_tx (bytes of both CTAs); when gathering
      // also its gather threads' cp.async arrivals and the peer's relay.  The
      // peer's copy (gathering only) counts the peer's gather threads.
      mbar_init(full_bar(s), GATHER ? (rank == 0 ? 2 + kGatherThreads : kGatherThreads) : 1);
      mbar_init(empty_bar(s), 1);  // the leader's MMA commit, multicast to both CTAs
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 8);  // leader's copy: 4 epilogue warps in each CTA
    }
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (!GATHER) {
      prefetch_tmap(&tmap_a);
      if (MOE_TC2_HALF) prefetch_tmap(&tmap_a64);
    }
    prefetch_tmap(&tmap_b0);
    if (GATEUP) prefetch_tmap(&tmap_b1);
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(s_tmem), kTmemCols);  // same warp id in both CTAs
  pdl_wait();
  pdl_trigger();
  if (warp == 2) {
    // clamped segment starts and per-expert pair-tile (256-row) prefix sums
    const int E = p.E;
    bool bad = false;
    for (int e = lane; e <= E; e += 32) s_seg[e] = __ldg(p.offsets + e);
    __syncwarp();
    if (lane == 0) {
      int prev = 0;
      for (int e = 0; e <= E; ++e) {
        const int v = s_seg[e];
        int c = min(max(v, prev), p.S);
        if (e == 0) c = min(max(v, 0), p.S);
        if (c != v) bad = true;
        s_seg[e] = c;
        prev = c;
      }
      if (bad && rank == 0) flag_error(kErrBadOffsets);
    }
    __syncwarp();
    const int per = (E + 31) / 32;
    const int e0 = lane * per, e1 = min(e0 + per, E);
    int local = 0;
    for (int e = e0; e < e1; ++e) local += (s_seg[e + 1] - s_seg[e] + BM2 - 1) / BM2;
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= d) incl += y;
    }
    int run = incl - local;
    for (int e = e0; e < e1; ++e) {
      s_pre[e] = run;
      run += (s_seg[e + 1] - s_seg[e] + BM2 - 1) / BM2;
    }
    if (lane == 31) s_pre[E] = incl;
    if (MOE_TC_EXPERT_GROUPS) {
      // raster groups of whole experts: experts in order until a group holds at
      // least MOE_TC2_GROUP_M m-tiles, so that no expert's weights are streamed twice
      __syncwarp();
      if (lane == 0) {
        int ng = 0, start = 0;
        s_grp[0] = 0;
        for (int e = 0; e < E; ++e) {
          const int end = s_pre[e + 1];
          if (end - start >= MOE_TC2_GROUP_M) {
            s_grp[++ng] = end;
            start = end;
          }
        }
        if (start < s_pre[E]) s_grp[++ng] = s_pre[E];
        s_grp[E + 1] = ng;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total_tiles = s_pre[p.E] * p.ntn;
  const int num_kb = (p.K + BK - 1) / BK;

  auto tile_coords = [&](int tile, int& e, int& m0, int& mend, int& n0) {
    int mt, nt;
    const int total_mtiles = s_pre[p.E];
    if (MOE_TC_EXPERT_GROUPS) {
      // group g: m-tiles [s_grp[g], s_grp[g + 1]), n-tile-major inside
      int lo = 0, hi = s_grp[p.E + 1] - 1;  // largest g with s_grp[g] * ntn <= tile
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_grp[mid] * p.ntn <= tile) lo = mid;
        else hi = mid - 1;
      }
      const int gm0 = s_grp[lo], gm = s_grp[lo + 1] - gm0;
      const int r = tile - gm0 * p.ntn;
      nt = r / gm;
      mt = gm0 + (r - nt * gm);
    } else if (MOE_TC2_GROUP_M > 0) {
      const int per_group = MOE_TC2_GROUP_M * p.ntn;
      const int g = tile / per_group, r = tile - g * per_group;
      const int gm = min(MOE_TC2_GROUP_M, total_mtiles - g * MOE_TC2_GROUP_M);
      nt = r / gm;
      mt = g * MOE_TC2_GROUP_M + (r - nt * gm);
    } else {
      mt = tile / p.ntn;
      nt = tile - mt * p.ntn;
    }
    int lo = 0, hi = p.E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= mt) lo = mid;
      else hi = mid - 1;
    }
    e = lo;
    m0 = s_seg[e] + (mt - s_pre[e]) * BM2;
    mend = s_seg[e + 1];
    n0 = nt * BN;
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {  // (weights only when warps 6..9 gather the A rows)
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = cid; ok && tile < total_tiles; tile += ncl) {
        int e, m0, mend, n0;
        tile_coords(tile, e, m0, mend, n0);
        const bool half = MOE_TC2_HALF && (mend - m0 <= 128);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, s_abort)) {
            ok = false;
            break;
          }
          // a half tile brings 64 rows of A per CTA; gathered A rows are not TMA bytes
          if (rank == 0)
            mbar_arrive_expect_tx(full_bar(stage),
                                  GATHER ? 2 * C::kBBytes : 2 * (C::kStageBytes - (half ? kABytes / 2 : 0u)));
          const uint32_t fb = mapa_shared(full_bar(stage), 0);  // the leader's full barrier
          const uint32_t a_dst = smem_u32(sA + (size_t)stage * kABytes);
          const uint32_t b_dst = smem_u32(sB + (size_t)stage * C::kBBytes);
          if (!GATHER) {
            if (half) tma_load_2d_pair(a_dst, &tmap_a64, fb, kb * BK, m0 + 64 * (int)rank);
            else tma_load_2d_pair(a_dst, &tmap_a, fb, kb * BK, m0 + 128 * (int)rank);
          }
          if (GATEUP) {  // each CTA: [gate 64 | up 64] for h columns n0 + 64 * rank + [0, 64)
            const int c0 = n0 + 64 * (int)rank;
            tma_load_3d_pair(b_dst, &tmap_b0, fb, c0, kb * BK, e);
            tma_load_3d_pair(b_dst + kBoxBytes, &tmap_b1, fb, c0, kb * BK, e);
          } else {  // leader: columns [n0, n0+128), peer: [n0+128, n0+256)
            const int c0 = n0 + 128 * (int)rank;
            tma_load_3d_pair(b_dst, &tmap_b0, fb, c0, kb * BK, e);
            tma_load_3d_pair(b_dst + kBoxBytes, &tmap_b0, fb, c0 + 64, kb * BK, e);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (ok) {
        // Wait until the leader's MMAs have released every stage: their commit
        // arrivals land in this CTA's shared memory, which must outlive them.
        for (int i = 0; ok && i < STAGES; ++i) {
          ok = mbar_wait(empty_bar(stage), phase ^ 1u, s_abort);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Loads of this CTA may still be in flight, and only the leader's full
        // barriers count them: give them a fixed time (far above a load's
        // latency) to land before shared memory goes away.
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc256 = idesc_bf16_f32(BM2, C::MMA_N);
      constexpr uint32_t idesc128 = idesc_bf16_f32(128, C::MMA_N);
      int stage = 0, local = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int tile = cid; ok && tile < total_tiles; tile += ncl, ++local) {
        uint32_t idesc = idesc256;
        if (MOE_TC2_HALF) {
          int e_, m0_, mend_, n0_;
          tile_coords(tile, e_, m0_, mend_, n0_);
          if (mend_ - m0_ <= 128) idesc = idesc128;
        }
        const int acc = local & 1;
        const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)acc * kAccStride;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, s_abort)) {
            ok = false;
            break;
          }
          if (GATHER && MOE_TC_GATHER_FENCE) fence_proxy_async_smem();  // this CTA's A rows came through cp.async
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + (size_t)stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + (size_t)stage * C::kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, kBoxBytes, 1024);
            umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          issued = true;
          umma_commit_pair(empty_bar(stage), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit_pair(tfull_bar(acc), 0x3);
      }
      if (!ok && issued) {
        umma_commit_pair(drain_bar, 0x1);
        mbar_wait(drain_bar, 0, nullptr, 100000000ull);
      }
    } else if (GATHER && lane == 0 && rank == 1) {
      // ---------------------------------------------- relay (peer, gathering only):
      // once this CTA's gathered rows of a stage have landed, make them visible
      // to the async proxy and tell the leader's full barrier.
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = cid; ok && tile < total_tiles; tile += ncl) {
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, s_abort)) {
            ok = false;
            break;
          }
          if (MOE_TC_GATHER_FENCE) fence_proxy_async_smem();
          const uint32_t leader_full = mapa_shared(full_bar(stage), 0);
          if (MOE_TC2_RELAY == 0) mbar_arrive_remote_cta_release(leader_full);
          else if (MOE_TC2_RELAY == 1) mbar_arrive_cluster_relaxed(leader_full);
          else mbar_arrive_cluster(leader_full);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (GATHER && warp >= 6) {
    // ------------------------------------------------ A-row gather (warps 6..9, both CTAs):
    // this CTA's rows of the pair tile, arrivals on this CTA's full barrier
    const int gt = (int)threadIdx.x - 192;
    int stage = 0;
    uint32_t phase = 0;
    auto tile_rows = [&](int tile, int& r0, int& r_end) {
      int e, m0, mend, n0;
      tile_coords(tile, e, m0, mend, n0);
      const int arows = (MOE_TC2_HALF && (mend - m0 <= 128)) ? 64 : 128;  // rows of A per CTA
      r0 = m0 + arows * (int)rank;
      r_end = min(mend, r0 + arows);
    };
    int slot[kGatherRowsPerThread];
    int tile = cid;
    if (tile < total_tiles) {
      int r0, r_end;
      tile_rows(tile, r0, r_end);
      gather_load_slots(p, r0, r_end, gt, slot);
    }
    for (; tile < total_tiles; tile += ncl) {
      const char* src[kGatherRowsPerThread];
      uint32_t dst_off[kGatherRowsPerThread];
      const int nrows = gather_rows_of_thread(p, slot, gt, src, dst_off);
      if (tile + ncl < total_tiles) {  // next tile's slots, in flight during this one
        int r0, r_end;
        tile_rows(tile + ncl, r0, r_end);
        gather_load_slots(p, r0, r_end, gt, slot);
      }
      if (!gather_tile(p, num_kb, nrows, src, dst_off, smem_u32(sA), kABytes, STAGES, stage, phase,
                       [&](int s) { return empty_bar(s); }, [&](int s) { return full_bar(s); }, s_abort))
        break;
    }
    cp_async_wait_all();
  } else {
    // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    // the leader's "accumulator empty" barrier, seen from this CTA
    const uint32_t tempty_leader0 = mapa_shared(tempty_bar(0), 0);
    const uint32_t tempty_leader1 = mapa_shared(tempty_bar(1), 0);
    int local = 0;
    for (int tile = cid; tile < total_tiles; tile += ncl, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
      if (!mbar_wait(tfull_bar(acc), acc_phase, s_abort)) break;
      tc_fence_after();
      int e, m0, mend, n0;
      tile_coords(tile, e, m0, mend, n0);
      // D column j of the MMA: gate/up tiles hold [gate 64 | up 64] of h columns
      // n0 + [0, 64) in j < 128 and of n0 + [64, 128) in j >= 128.
      const bool half = MOE_TC2_HALF && (mend - m0 <= 128);
      // half tile: warp q holds rows 32 (q & 1) + lane of this CTA's 64 and
      // the D columns of B half q >> 1
      const int row = half ? m0 + 64 * (int)rank + 32 * (q & 1) + lane : m0 + 128 * (int)rank + 32 * q + lane;
      const bool row_ok = row < mend;
      const uint32_t t_base = tmem_base + (uint32_t)acc * kAccStride + ((uint32_t)(q * 32) << 16);
      const int out_base = n0 + (half ? (q >> 1) * (BN / 2) : 0);
      const int nch = half ? BN / 64 : BN / 32;  // 32-column output chunks of this warp
      __nv_bfloat16* out_row = p.out + (size_t)row * p.N;
#pragma unroll 1
      for (int c = 0; c < nch; ++c) {
        uint32_t r0[32];
        float v[32];
        if (GATEUP) {
          const int tcol = half ? c * 32 : (c >> 1) * 128 + (c & 1) * 32;
          uint32_t r1[32];
          tmem_ld32(t_base + tcol, r0);
          tmem_ld32(t_base + tcol + 64, r1);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float g = __uint_as_float(r0[i]), u = __uint_as_float(r1[i]);
            v[i] = __fdividef(g, 1.0f + __expf(-g)) * u;
          }
        } else {
          tmem_ld32(t_base + c * 32, r0);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r0[i]);
        }
        if (row_ok) {
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            const int col = out_base + c * 32 + g8 * 8;
            if (col < p.N) {
              const uint4 w = make_uint4(pack_bf16x2(v[g8 * 8 + 0], v[g8 * 8 + 1]),
                                         pack_bf16x2(v[g8 * 8 + 2], v[g8 * 8 + 3]),
                                         pack_bf16x2(v[g8 * 8 + 4], v[g8 * 8 + 5]),
                                         pack_bf16x2(v[g8 * 8 + 6], v[g8 * 8 + 7]));
              st_v4(out_row + col, w);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(tempty_bar(acc));
        else mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
      }
    }
  }
  // No CTA of the pair may leave while the other can still reach its shared
  // memory (peer MMA operand reads, commit and epilogue arrivals) or TMEM.
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------- host side
// Activations [rows, K] bf16, box 64 (K) x 64 (rows), 128-byte swizzle: the A
// operand of one CTA in a half tile.
inline bool make_tmap_act64(CUtensorMap* m, const void* base, int rows, int K) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, 64};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Number of 2-CTA clusters that can be resident at once (each CTA takes one
// SM), cached per device.
template <bool GATEUP, bool GATHER>
int max_pair_clusters(size_t smem) {
  static PerDeviceInt cached;
  return cached.get(current_device(), [&] {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    cfg.blockDim = dim3(GATHER ? kThreads + kGatherThreads : kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_tc2_kernel<GATEUP, GATHER>, &cfg) != cudaSuccess || n <= 0)
      n = num_sms() / 2;
    return n;
  });
}

template <bool GATEUP, bool GATHER = false>
cudaError_t launch_tc2(const CUtensorMap& ta, const CUtensorMap& ta64, const CUtensorMap& tb0, const CUtensorMap& tb1,
                       const Params& p, cudaStream_t stream) {
  using C = Cfg2<GATEUP>;
  auto kern = grouped_gemm_tc2_kernel<GATEUP, GATHER>;
  const size_t smem = C::smem_bytes(p.E);
  static PerDeviceOnce attr_once;  // the attribute is per device; set it once for the largest E
  cudaError_t err = attr_once.run(current_device(), [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::smem_bytes(1024));
  });
  if (err != cudaSuccess) return err;
  const long long max_tiles = ((long long)(p.S + BM2 - 1) / BM2 + p.E) * p.ntn;
  long long clusters = max_pair_clusters<GATEUP, GATHER>(C::smem_bytes(1024));
  if (max_tiles < clusters) clusters = max_tiles > 0 ? max_tiles : 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * clusters));
  cfg.blockDim = dim3(GATHER ? kThreads + kGatherThreads : kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = MOE_PDL ? 2 : 1;
  err = cudaLaunchKernelEx(&cfg, kern, ta, ta64, tb0, tb1, p);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// Pair-tile forms of launch_gate_up / launch_down (same arguments and outputs).
inline cudaError_t launch_gate_up_pair(const void* x_disp, const void* wg, const void* wu, const int32_t* off, int E,
                                       int H, int I, int S, void* h, cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  CUtensorMap ta, ta64, tg, tu;
  if (!make_tmap_act(&ta, x_disp, S, H) || !make_tmap_act64(&ta64, x_disp, S, H) ||
      !make_tmap_weight(&tg, wg, E, H, I) || !make_tmap_weight(&tu, wu, E, H, I))
    return cudaErrorInvalidValue;
  Params p{off, E, S, H, I, (I + 127) / 128, reinterpret_cast<__nv_bfloat16*>(h), nullptr, 1, 0, nullptr};
  return launch_tc2<true>(ta, ta64, tg, tu, p, stream);
}

// launch_gate_up_pair with the A rows gathered from x [T, H] (see launch_gate_up_gather).
inline cudaError_t launch_gate_up_pair_gather(const void* x, int T, const int32_t* row_to_slot, int k, const void* wg,
                                              const void* wu, const int32_t* off, int E, int H, int I, int S, void* h,
                                              cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  CUtensorMap tg, tu;  // the A rows come from x through cp.async: no activation tensor map
  if (!make_tmap_weight(&tg, wg, E, H, I) || !make_tmap_weight(&tu, wu, E, H, I)) return cudaErrorInvalidValue;
  Params p{off, E, S, H, I, (I + 127) / 128, reinterpret_cast<__nv_bfloat16*>(h), row_to_slot, k, T, x};
  return launch_tc2<true, true>(tg, tg, tg, tu, p, stream);
}

inline cudaError_t launch_down_pair(const void* h, const void* wd, const int32_t* off, int E, int H, int I, int S,
                                    void* y, cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  CUtensorMap ta, ta64, tb;
  if (!make_tmap_act(&ta, h, S, I) || !make_tmap_act64(&ta64, h, S, I) || !make_tmap_weight(&tb, wd, E, I, H))
    return cudaErrorInvalidValue;
  Params p{off, E, S, I, H, (H + 255) / 256, reinterpret_cast<__nv_bfloat16*>(y), nullptr, 1, 0, nullptr};
  return launch_tc2<false>(ta, ta64, tb, tb, p, stream);
}

}  // namespace tc
}  // namespace moe
