// moe_router_topk: the router's affinities and moe_route in one kernel.
//
// "Expert Parallelism (EP)", "Router Weights": every token is scored against
// all E experts, logits = x W_r^T (+ bias); "EP: Partition Experts and Route
// Tokens", "Send tokens to experts and return their results" / "Return
// multiple expert results to the same token": top-k selection and the
// combination weights, here the softmax over the k selected logits.
//
// Tiles of 128 tokens.  The affinity matrix is a dense contraction (M =
// tokens, N = experts <= 256, K = H), so it runs on tcgen05: warp 0 streams
// 64-deep k-blocks of the token tile and of W_r (both K-major, 128-byte
// swizzle) by TMA through a ring of mbarrier stages, warp 1 issues
// M=128 x N=E_pad UMMAs into float32 TMEM accumulators.  The K range is split
// over a cluster of SK CTAs per token tile: each drains its partial sums into
// shared memory, then CTA r sums rows [r*128/SK, (r+1)*128/SK) of all SK
// partials (cluster rank order, read over DSMEM) plus the bias, writes the
// logits (optional) and routes each of those tokens with
// moe_route's warp_topk_softmax (a warp per token, all 16 warps) -- so ids and
// weights are bit-identical to moe_route applied to the logits written.
// Every mbarrier wait is bounded; every thread reaches both cluster barriers.
#pragma once

#include "ffn_tc.cuh"
#include "route.cuh"

namespace moe {
namespace tc {

// 16 warps: warp 0 TMA, warp 1 MMA, warps 2-5 drain TMEM (one lane quarter
// each), and all 16 share the cross-CTA sums and the routing, so that the
// warp-wide selections of several warps hide each other's latency.
constexpr int kRouterThreads = 512;
constexpr int kRouterWarps = kRouterThreads / 32;

struct RouterParams {
  const float* bias;  // [E] or null
  int T, H, E, k;
  float* logits;      // [T, E] or null
  int32_t* topk_ids;  // [T, k]
  float* topk_w;      // [T, k]
};

// Instruction descriptor, kind::f16: D f32, A and B bf16, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_kk(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

template <int NPAD>
struct RouterCfg {
  static constexpr uint32_t kBBytes = NPAD * BK * 2;  // W_r rows of one k-block
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr int STAGES = (192 * 1024) / kStageBytes > 8 ? 8 : (192 * 1024) / kStageBytes;
  // Independent accumulators, K-step kk of a k-block into accumulator kk % NACC:
  // with few experts (small MMA N) one accumulation chain would wait on each
  // MMA's latency; NACC chains overlap it.  NACC * NPAD <= 512 TMEM columns.
  static constexpr int NACC = NPAD <= 128 ? 4 : 2;
  static constexpr uint32_t kAccCols = NPAD <= 32 ? 32 : NPAD <= 64 ? 64 : NPAD <= 128 ? 128 : 256;
  static constexpr uint32_t kTmemCols = kAccCols * NACC;
  static constexpr size_t smem_bytes = 1024 + (size_t)STAGES * kStageBytes + 256;
  static_assert((size_t)BM * (NPAD + 4) * 4 <= (size_t)STAGES * kStageBytes, "logit staging must fit in the ring");
};

__device__ __forceinline__ uint32_t router_cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void router_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 16 bytes at this (16-byte aligned) shared-memory address in CTA `rank` of the cluster
__device__ __forceinline__ float4 ld_peer_f32x4(uint32_t addr, uint32_t rank) {
  uint32_t peer;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(peer) : "r"(addr), "r"(rank));
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(peer)
               : "memory");
  return v;
}

// Grid: (token tiles) x SK CTAs, clusters of SK along x; CTA r of a cluster
// sums k-blocks [r*nkb/SK, (r+1)*nkb/SK) for the tile's 128 tokens.
template <int NPAD>
__global__ void __launch_bounds__(kRouterThreads, 1)
    router_topk_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                       RouterParams p, int SK) {
  using C = RouterCfg<NPAD>;
  constexpr int STAGES = C::STAGES;
  // staging rows 16-byte aligned (float4 stores and remote loads); the 4-word
  // pad spreads a warp's row-per-thread float4 stores over all banks
  constexpr int LD = NPAD + 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                              // STAGES x 16 KB token tile
  uint8_t* sB = smem + (size_t)STAGES * kABytes;   // STAGES x kBBytes router rows
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + (size_t)STAGES * C::kBBytes);
  // bars: full[STAGES], empty[STAGES], tfull, drain
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 2);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  float* s_part = reinterpret_cast<float*>(smem);  // [BM][LD] this CTA's partial sums (the idle ring)
  const int warp = threadIdx.x >> 5, lane = (int)lane_id();
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  const uint32_t tfull_bar = smem_u32(bars + 2 * STAGES);
  const uint32_t drain_bar = smem_u32(bars + 2 * STAGES + 1);
  const uint32_t rank = router_cluster_rank();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_w);
  }
  if (warp == 1) tmem_alloc(smem_u32(s_tmem), C::kTmemCols);
  pdl_wait();  // x and W_r may come from the previous kernel
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int m0 = (int)(blockIdx.x / SK) * BM;
  const int nkb = (p.H + BK - 1) / BK;
  const int kb0 = (int)rank * nkb / SK, kb1 = ((int)rank + 1) * nkb / SK;  // non-empty: SK <= nkb

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, armed_mask = 0, armed_par = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, s_abort)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(full_bar(stage), C::kStageBytes);
        armed_mask |= 1u << stage;
        armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
        tma_load_2d(smem_u32(sA + (size_t)stage * kABytes), &tmap_x, full_bar(stage), kb * BK, m0);
        tma_load_2d(smem_u32(sB + (size_t)stage * C::kBBytes), &tmap_w, full_bar(stage), kb * BK, 0);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {  // let in-flight loads land before the ring is reused or the CTA leaves
        for (int s = 0; s < STAGES; ++s)
          if (armed_mask & (1u << s)) mbar_wait(full_bar(s), (armed_par >> s) & 1u, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32_kk(BM, NPAD);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(full_bar(stage), phase, s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sA + (size_t)stage * kABytes);
        const uint32_t b_addr = smem_u32(sB + (size_t)stage * C::kBBytes);
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk) {
          // both operands K-major: rows of 128 B, 8-row atoms 1024 B apart; K step = 32 B
          const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 32, 16, 1024);
          umma_bf16(tmem_base + (uint32_t)(kk % C::NACC) * C::kAccCols, adesc, bdesc, idesc,
                    (kb != kb0 || kk >= C::NACC) ? 1u : 0u);
        }
        issued = true;
        umma_commit(empty_bar(stage));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) umma_commit(tfull_bar);
      else if (issued) {
        umma_commit(drain_bar);
        mbar_wait(drain_bar, 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------ drain: one token row per thread
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    if (mbar_wait(tfull_bar, 0, s_abort)) {
      tc_fence_after();
      const int r = q * 32 + lane;
#pragma unroll 1
      for (int c = 0; c < NPAD / 32; ++c) {
        float acc[32];
#pragma unroll
        for (int a = 0; a < C::NACC; ++a) {  // sum the accumulators in a fixed order
          uint32_t rr[32];
          tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + a * C::kAccCols + c * 32, rr);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = a == 0 ? __uint_as_float(rr[i]) : acc[i] + __uint_as_float(rr[i]);
        }
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(s_part + r * LD + c * 32 + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
      }
    }
    __syncwarp();
  }

  // ---- every CTA's partial sums are in its shared memory
  tc_fence_before();
  router_cluster_sync();
  tc_fence_after();
  // ---- this CTA's rows of the tile: sum the SK partials (cluster rank order)
  // plus the bias, in place over its own rows (which no peer reads) ...
  constexpr int VPL = NPAD / 32;
  const int rows = BM / SK, row0 = (int)rank * rows;
  if (*s_abort == 0) {
    // two float4 cells a thread per round, every remote load of a round issued before any sum
    constexpr int Q = NPAD / 4;  // float4 cells of a row
    const int n = rows * Q;
    for (int i0 = threadIdx.x; i0 < n; i0 += 2 * kRouterThreads) {
      float4 part[2][8];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = i0 + u * kRouterThreads;
        const int rl = i / Q, e4 = i - rl * Q;
        const uint32_t addr = smem_u32(s_part + (row0 + rl) * LD + 4 * e4);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (i < n && c < SK) part[u][c] = ld_peer_f32x4(addr, (uint32_t)c);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = i0 + u * kRouterThreads;
        if (i >= n) break;
        const int rl = i / Q, e4 = i - rl * Q;
        float4 sum = part[u][0];  // cluster rank order
#pragma unroll
        for (int c = 1; c < 8; ++c) {
          if (c < SK) {
            sum.x += part[u][c].x;
            sum.y += part[u][c].y;
            sum.z += part[u][c].z;
            sum.w += part[u][c].w;
          }
        }
        const float sv[4] = {sum.x, sum.y, sum.z, sum.w};
        float* cell = s_part + (row0 + rl) * LD + 4 * e4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = 4 * e4 + j;
          cell[j] = e < p.E ? sv[j] + (p.bias != nullptr ? __ldg(p.bias + e) : 0.0f) : 0.0f;
        }
      }
    }
  }
  __syncthreads();
  // ... then write the logits and route each token with a whole warp
  // (moe_route's warp_topk_softmax, lane = expert)
  if (*s_abort == 0) {
#pragma unroll 1
    for (int rl = warp; rl < rows; rl += kRouterWarps) {
      const int t = m0 + row0 + rl;
      if (t >= p.T) break;  // uniform in the warp
      uint32_t key[VPL];
      float val[VPL];
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const int e = lane + 32 * v;
        val[v] = s_part[(row0 + rl) * LD + e];
        key[v] = e < p.E ? logit_order_key(val[v]) : 0u;
        if (e < p.E && p.logits != nullptr) p.logits[(size_t)t * p.E + e] = val[v];
      }
      int my_id;
      float my_w;
      warp_topk_softmax<VPL>(key, val, p.k, lane, my_id, my_w);
      if (lane < p.k) {
        p.topk_ids[(size_t)t * p.k + lane] = my_id;
        p.topk_w[(size_t)t * p.k + lane] = my_w;
      }
    }
  }
  // ---- no CTA leaves (or frees TMEM) while a peer may still read its partials
  __syncwarp();
  router_cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Rows [rows, K] bf16, box 64 (K) x box_rows, 128-byte swizzle.
inline bool make_tmap_rows(CUtensorMap* m, const void* base, int rows, int K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NPAD>
cudaError_t launch_router_npad(const CUtensorMap& tx, const CUtensorMap& tw, const RouterParams& p,
                               cudaStream_t stream) {
  using C = RouterCfg<NPAD>;
  auto kern = router_topk_kernel<NPAD>;
  static PerDeviceOnce attr_once;
  cudaError_t err = attr_once.run(current_device(), [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::smem_bytes);
  });
  if (err != cudaSuccess) return err;
  // split K over a cluster of SK CTAs per token tile: as many as fill the SMs
  // once (at most 8, at least one k-block each)
  const int tiles = (p.T + BM - 1) / BM, nkb = (p.H + BK - 1) / BK;
  int sk = 1;
  while (sk < 8 && (long long)tiles * sk * 2 <= num_sms() && sk * 2 <= nkb) sk *= 2;
  static PerDeviceInt max_sk;  // the widest cluster of these CTAs the device can hold
  const int widest = max_sk.get(current_device(), [&] {
    int w = 8;
    for (; w > 1; w /= 2) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3((unsigned)w);
      q.blockDim = dim3(kRouterThreads);
      q.dynamicSmemBytes = C::smem_bytes;
      cudaLaunchAttribute a[1];
      a[0].id = cudaLaunchAttributeClusterDimension;
      a[0].val.clusterDim.x = (unsigned)w;
      a[0].val.clusterDim.y = 1;
      a[0].val.clusterDim.z = 1;
      q.attrs = a;
      q.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &q) == cudaSuccess && n > 0) break;
    }
    return w;
  });
  if (sk > widest) sk = widest;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(tiles * sk));
  cfg.blockDim = dim3(kRouterThreads);
  cfg.dynamicSmemBytes = C::smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)sk;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = MOE_PDL ? 2 : 1;
  err = cudaLaunchKernelEx(&cfg, kern, tx, tw, p, sk);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// x [T, H] bf16, w_router [E, H] bf16; E <= 256, H % 8 == 0.
inline cudaError_t launch_router(const void* x, const void* w_router, const RouterParams& p, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  const int npad = (p.E + 31) / 32 * 32;
  CUtensorMap tx, tw;
  if (!make_tmap_act(&tx, x, p.T, p.H) || !make_tmap_rows(&tw, w_router, p.E, p.H, npad))
    return cudaErrorInvalidValue;
  switch (npad) {
    case 32: return launch_router_npad<32>(tx, tw, p, stream);
    case 64: return launch_router_npad<64>(tx, tw, p, stream);
    case 96: return launch_router_npad<96>(tx, tw, p, stream);
    case 128: return launch_router_npad<128>(tx, tw, p, stream);
    case 160: return launch_router_npad<160>(tx, tw, p, stream);
    case 192: return launch_router_npad<192>(tx, tw, p, stream);
    case 224: return launch_router_npad<224>(tx, tw, p, stream);
    case 256: return launch_router_npad<256>(tx, tw, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace tc
}  // namespace moe
