// Grouped SwiGLU expert MLP on 5th-generation tensor cores (tcgen05 + TMEM +
// TMA), bf16 in, float32 accumulate.
//
// "EP: Partition Experts and Route Tokens", "Send tokens to experts and
// return their results": each expert's rows are stacked and multiplied by
// that expert's weights; rows never mix.  Expert form (Shazeer, "GLU Variants
// Improve Transformer"): h = SiLU(x Wg) * (x Wu), y = h Wd.
//
// Ragged expert segments: expert e owns rows [off[e], off[e+1]) of the
// dispatched buffer, unpadded.  An expert's last tile, when it holds at most
// 64 rows, runs as an M=64 UMMA (half the tensor time of M=128).  Every CTA rebuilds the tile list on the
// device from off[] (per-expert 128-row m-tiles, prefix-summed in shared
// memory) so the host never reads the counts.  A 128-row tile may run past
// its expert's last row: those extra rows are loaded (harmless: they belong to
// the next expert or lie past the buffer, where TMA fills zeros) and their
// results are never stored.  Stores are per-row predicated 16-byte st.global,
// because a TMA tile store would overwrite the neighbouring expert's rows.
//
// Persistent kernel, one CTA per SM, 192 threads:
//   warp 0      one lane issues TMA loads into a STAGES-deep shared-memory ring
//   warp 1      allocates 512 TMEM columns; one lane issues tcgen05.mma
//               (M=128, N=MMA_N, K=16) and tcgen05.commit
//   warps 2..5  epilogue: tcgen05.ld from TMEM (warp w reads lanes
//               32*(w%4)..+31), SwiGLU or bf16 rounding, predicated stores
// Two TMEM accumulators (columns 0 and 256) let the epilogue of one tile
// overlap the MMAs of the next.  Operand layouts, straight from the caller's
// buffers (no repacking):
//   A = activations [rows, K], K contiguous  -> K-major, 128-byte swizzle
//   B = weights [E, K, N], N contiguous      -> MN-major, 128-byte swizzle
// Gate/up fusion: the B tile of one stage holds 128 gate columns and the same
// 128 up columns side by side, so one N=256 MMA produces both halves of a
// 128-column h tile in one accumulator.
//
// Gathering form (gate/up only, moe_ffn_gate_up_gather): the A rows are not
// read from a dispatched buffer but copied from the token rows of x by 128
// extra threads (warps 6..9) with 16-byte cp.async into the same swizzled
// layout; each stage's full barrier then also counts one cp.async arrival
// per gather thread, and the MMA thread fences the proxy before reading.
// (TMA tile::gather4, four 128-byte rows per instruction, was measured first:
// 32 instructions per k-block made the kernel 2.5-3x slower.)
//
// Every mbarrier wait is bounded (globaltimer): on expiry the CTA sets the
// timeout bit of the device error word, the other roles stop, in-flight TMA
// loads and MMAs are waited for (bounded), TMEM is freed and the kernel
// returns.  No TMA multicast is used anywhere.
#pragma once

#include <cuda.h>

#include <climits>

#include "common.cuh"

// Tuning knobs (compile-time).
//  MOE_TC_GROUP_M: tiles are visited in groups of this many consecutive m-tiles,
//    all n-tiles of a group before the next group (0 = plain m-major order).
//  MOE_TC_HINT_A / MOE_TC_HINT_B: L2 eviction priority of the TMA loads of the
//    activation and weight tiles (0 normal, 1 evict-first, 2 evict-last).
#ifndef MOE_TC_GROUP_M
#define MOE_TC_GROUP_M 16
#endif
//  MOE_TC_EXPERT_GROUPS: raster groups end at expert boundaries (whole experts
//    until a group holds at least the group size in m-tiles) instead of every
//    group-size m-tiles, so an expert's m-tiles are never split across groups.
#ifndef MOE_TC_EXPERT_GROUPS
#define MOE_TC_EXPERT_GROUPS 1
#endif
#ifndef MOE_TC_HINT_A
#define MOE_TC_HINT_A 0
#endif
#ifndef MOE_TC_HINT_B
#define MOE_TC_HINT_B 0
#endif
//  MOE_TC_M64: tiles with at most 64 valid rows (an expert's last, partial
//    tile) issue M=64 UMMAs, which take about half the time of M=128; the
//    accumulator then sits in TMEM lanes 0-15 of each 32-lane quarter, so
//    epilogue warp q holds rows 16q..16q+15 in its lanes 0-15.
#ifndef MOE_TC_M64
#define MOE_TC_M64 1
#endif
//  MOE_TC_GATHER_FENCE: the MMA thread of a gathering kernel issues a
//    shared-memory proxy fence after each stage's full barrier, before its
//    UMMAs read the rows that cp.async wrote.
#ifndef MOE_TC_GATHER_FENCE
#define MOE_TC_GATHER_FENCE 1
#endif
//  MOE_TC_DOWN_BN: force the down-projection n-tile width (0 = chosen from H).
#ifndef MOE_TC_DOWN_BN
#define MOE_TC_DOWN_BN 0
#endif

namespace moe {
namespace tc {

constexpr int BM = 128;
constexpr int BK = 64;  // bf16 elements in one 128-byte swizzled row
constexpr int UMMA_K = 16;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccStride = 256;  // TMEM columns between the two accumulators
constexpr uint32_t kABytes = BM * BK * 2;  // 16 KB
constexpr uint32_t kBoxBytes = 64 * BK * 2;  // one 64-column x 64-row B box, 8 KB
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

// ------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity.  Returns false when the
// CTA is aborting (another role timed out) or this wait itself timed out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (abort_flag != nullptr && *abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        if (abort_flag != nullptr) *abort_flag = 1;
        flag_error(kErrTimeout);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// 16-byte global -> shared copy on the LSU path (cp.async); src_bytes = 0
// writes 16 zero bytes and reads nothing.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// Arrive on the mbarrier once all earlier cp.async of this thread have landed
// (the arrival counts toward the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Order shared-memory data made visible to this thread (written through the
// generic proxy, e.g. by cp.async) before its later async-proxy accesses
// (tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// L2 eviction-priority policy for cache-hinted TMA loads (1 evict-first, 2 evict-last).
template <int HINT>
__device__ __forceinline__ uint64_t l2_policy() {
  uint64_t pol = 0;
  if (HINT == 1) asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  if (HINT == 2) asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
template <int HINT>
__device__ __forceinline__ void tma_load_2d_h(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                              uint64_t pol) {
  if (HINT == 0) {
    tma_load_2d(dst, map, bar, c0, c1);
  } else {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(pol)
        : "memory");
  }
}
template <int HINT>
__device__ __forceinline__ void tma_load_3d_h(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                              int c2, uint64_t pol) {
  if (HINT == 0) {
    tma_load_3d(dst, map, bar, c0, c1, c2);
  } else {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "l"(pol)
        : "memory");
  }
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 inputs, f32 accumulate)
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The mbarrier completes one phase once every previously issued tcgen05.mma
// of this thread has finished.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns; thread i receives lane (base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100
// descriptor version 1 at bit 46.  lbo/sbo in bytes.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: D f32, A bf16 K-major, B bf16 MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(m >> 4) << 24);
}

// ------------------------------------------------------------- the kernel
struct Params {
  const int32_t* offsets;  // [E + 1]
  int E, S, K, N;          // N: output columns (I for gate/up, H for down)
  int ntn;                 // n-tiles per m-tile
  __nv_bfloat16* out;      // [S, N]
  // Gathering kernels only: A row r is token row row_to_slot[r] / gather_k of
  // x [gather_T, K] instead of row r of a dispatched buffer.
  const int32_t* gather_rows;  // [S] row_to_slot
  int gather_k, gather_T;
  const void* gather_x;        // [gather_T, K] bf16
  // Down projection with the combine in its epilogue (single-CTA tiles only):
  // row r's output, times comb_w[s], is added (float32 atomics) into
  // comb_acc[s / comb_k] for its slot s = comb_rows[r]; `out` is not written.
  const int32_t* comb_rows;  // [S] row_to_slot
  const float* comb_w;       // [comb_T * comb_k] topk_w
  float* comb_acc;           // [comb_T, N] float32
  int comb_k, comb_T;
};

// ---- A-row gather (dispatch fused into the gate/up projection)
// kGatherThreads extra threads per CTA copy the A tile rows of each k-block
// from x with 16-byte cp.async: thread t owns 16-byte chunk c = t % 8 of rows
// t / 8 + (kGatherThreads / 8) j of the 128-row tile, written to its 128-byte
// swizzled position (chunk c ^ (row % 8)).  Each thread then arrives on the
// stage's full barrier when its copies land (cp.async.mbarrier.arrive.noinc).
#ifndef MOE_TC_GATHER_THREADS
#define MOE_TC_GATHER_THREADS 128
#endif
constexpr int kGatherThreads = MOE_TC_GATHER_THREADS;       // 32, 64 or 128
constexpr int kGatherRowStep = kGatherThreads / 8;          // rows between a thread's rows
constexpr int kGatherRowsPerThread = 128 / kGatherRowStep;  // 8 at 128 threads
static_assert(kGatherThreads == 32 || kGatherThreads == 64 || kGatherThreads == 128, "gather threads");

// Slots (row_to_slot entries) of this thread's rows of the tile [r0, r_end),
// kNoGatherRow for rows past r_end.  Loaded one tile ahead, so their latency
// hides behind the previous tile's k-blocks.
constexpr int kNoGatherRow = INT_MIN;
__device__ __forceinline__ void gather_load_slots(const Params& p, int r0, int r_end, int gt,
                                                  int (&slot)[kGatherRowsPerThread]) {
  const int rr = gt >> 3;
#pragma unroll
  for (int j = 0; j < kGatherRowsPerThread; ++j) {
    const int r = r0 + rr + kGatherRowStep * j;
    slot[j] = r < r_end ? __ldg(p.gather_rows + r) : kNoGatherRow;
  }
}

// Source pointers (at the thread's chunk, k-block 0) and shared-memory byte
// offsets within a stage's A tile for the slots above; returns how many of
// the thread's rows are inside the tile.  A slot outside [0, gather_T *
// gather_k) is flagged and read as token 0 (the row's output is then
// meaningless but every load stays in bounds).  Rows past the tile are not
// copied: their accumulator rows are never stored.
__device__ __forceinline__ int gather_rows_of_thread(const Params& p, const int (&slot)[kGatherRowsPerThread], int gt,
                                                     const char* (&src)[kGatherRowsPerThread],
                                                     uint32_t (&dst_off)[kGatherRowsPerThread]) {
  const int c = gt & 7, rr = gt >> 3;  // chunk, first row (0 .. kGatherRowStep - 1)
  int n = 0;
#pragma unroll
  for (int j = 0; j < kGatherRowsPerThread; ++j) {
    const int row = rr + kGatherRowStep * j;
    src[j] = nullptr;
    dst_off[j] = (uint32_t)row * 128u + (uint32_t)((c ^ (row & 7)) << 4);
    if (slot[j] != kNoGatherRow) {
      int t = slot[j] / p.gather_k;
      if (slot[j] < 0 || t >= p.gather_T) {
        flag_error(kErrBadRow);
        t = 0;
      }
      src[j] = reinterpret_cast<const char*>(p.gather_x) + ((size_t)t * p.K + (size_t)c * 8) * 2;
      n = j + 1;
    }
  }
  return n;
}

// The k-blocks of one tile: wait for the stage to be free, copy this thread's
// rows of the k-block (16 zero bytes where the chunk lies past K), arrive on
// the stage's full barrier.  Returns false if a wait gave up.
template <typename EmptyBar, typename FullBar>
__device__ __forceinline__ bool gather_tile(const Params& p, int num_kb, int nrows,
                                            const char* const (&src)[kGatherRowsPerThread],
                                            const uint32_t (&dst_off)[kGatherRowsPerThread], uint32_t sA_base,
                                            uint32_t a_stage_bytes, int nstages, int& stage, uint32_t& phase,
                                            EmptyBar empty_bar, FullBar full_bar, volatile int* abort_flag) {
  const int c8 = (int)(threadIdx.x & 7) * 8;  // this thread's first K element within a k-block
  for (int kb = 0; kb < num_kb; ++kb) {
    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) return false;
    const uint32_t base = sA_base + (uint32_t)stage * a_stage_bytes;
    const uint32_t nbytes = kb * BK + c8 < p.K ? 16u : 0u;
    const size_t koff = (size_t)kb * BK * 2;
#pragma unroll
    for (int j = 0; j < kGatherRowsPerThread; ++j)
      if (j < nrows && src[j] != nullptr) cp_async16(base + dst_off[j], nbytes ? src[j] + koff : src[j], nbytes);
    cp_async_arrive_noinc(full_bar(stage));
    if (++stage == nstages) {
      stage = 0;
      phase ^= 1u;
    }
  }
  return true;
}

template <bool GATEUP, int BN, int STAGES>
struct Cfg {
  static constexpr int MMA_N = GATEUP ? 2 * BN : BN;  // gate/up: [gate BN | up BN]
  static constexpr int NBOX = GATEUP ? 2 * ((BN + 63) / 64) : (BN + 63) / 64;
  static constexpr uint32_t kBBytes = NBOX * kBoxBytes;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr size_t smem_bytes(int E) {
    return 1024 /* alignment slack */ + (size_t)STAGES * kStageBytes + 256 /* barriers etc */ +
           sizeof(int32_t) * (3 * ((size_t)E + 1) + 1);
  }
  static_assert(MMA_N % 16 == 0 && MMA_N >= 16 && MMA_N <= 256, "UMMA N for M=128");
  static_assert(!GATEUP || BN % 64 == 0, "gate/up halves must be whole 64-column boxes");
};

template <bool GATEUP, int BN, int STAGES, bool GATHER = false>
__global__ void __launch_bounds__(GATHER ? kThreads + kGatherThreads : kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b0,
                           const __grid_constant__ CUtensorMap tmap_b1, Params p) {
  using C = Cfg<GATEUP, BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                   // STAGES x 16 KB
  uint8_t* sB = smem + (size_t)STAGES * kABytes;        // STAGES x kBBytes
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + (size_t)STAGES * C::kBBytes);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int32_t* s_seg = reinterpret_cast<int32_t*>(smem + (size_t)STAGES * C::kStageBytes + 256);  // [E + 1]
  int32_t* s_pre = s_seg + (p.E + 1);                                                         // [E + 1]
  int32_t* s_grp = s_pre + (p.E + 1);  // [E + 2]: raster group starts (m-tiles), count at [E + 1]

  const int warp = threadIdx.x >> 5, lane = (int)lane_id();
  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + STAGES + s); };
  auto tfull_bar = [&](int a) { return smem_u32(bars + 2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return smem_u32(bars + 2 * STAGES + 2 + a); };
  const uint32_t drain_bar = smem_u32(bars + 2 * STAGES + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), GATHER ? 1 + kGatherThreads : 1);  // + one cp.async arrival per gather thread
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4);  // one arrive per epilogue warp
    }
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (!GATHER) prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b0);
    if (GATEUP) prefetch_tmap(&tmap_b1);
  }
  if (warp == 1) tmem_alloc(smem_u32(s_tmem), kTmemCols);
  // Everything above touches only this CTA's shared memory and TMEM; from here
  // on the kernel reads what earlier kernels wrote.
  pdl_wait();
  pdl_trigger();
  if (warp == 2) {
    // clamped segment starts and per-expert m-tile prefix sums (warp scan)
    const int E = p.E;
    bool bad = false;
    for (int e = lane; e <= E; e += 32) {
      int v = __ldg(p.offsets + e);
      s_seg[e] = v;
    }
    __syncwarp();
    if (lane == 0) {
      int prev = 0;
      for (int e = 0; e <= E; ++e) {  // clamp to a monotone sequence in [0, S]
        int v = s_seg[e];
        int c = min(max(v, prev), p.S);
        if (e == 0) c = min(max(v, 0), p.S);
        if (c != v) bad = true;
        s_seg[e] = c;
        prev = c;
      }
      if (bad) flag_error(kErrBadOffsets);
    }
    __syncwarp();
    const int per = (E + 31) / 32;
    const int e0 = lane * per, e1 = min(e0 + per, E);
    int local = 0;
    for (int e = e0; e < e1; ++e) local += (s_seg[e + 1] - s_seg[e] + BM - 1) / BM;
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= d) incl += y;
    }
    int run = incl - local;
    for (int e = e0; e < e1; ++e) {
      s_pre[e] = run;
      run += (s_seg[e + 1] - s_seg[e] + BM - 1) / BM;
    }
    if (lane == 31) s_pre[E] = incl;
    if (MOE_TC_EXPERT_GROUPS) {
      // raster groups of whole experts: experts in order until a group holds at
      // least MOE_TC_GROUP_M m-tiles, so that no expert's weights are streamed twice
      __syncwarp();
      if (lane == 0) {
        int ng = 0, start = 0;
        s_grp[0] = 0;
        for (int e = 0; e < E; ++e) {
          const int end = s_pre[e + 1];
          if (end - start >= MOE_TC_GROUP_M) {
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
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total_mtiles = s_pre[p.E];
  const int total_tiles = total_mtiles * p.ntn;
  const int num_kb = (p.K + BK - 1) / BK;

  // tile -> (expert, first row, end row, first output column)
  auto tile_coords = [&](int tile, int& e, int& m0, int& mend, int& n0) {
    int mt, nt;
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
    } else if (MOE_TC_GROUP_M > 0) {
      // groups of MOE_TC_GROUP_M m-tiles; inside a group, n-tile-major
      const int per_group = MOE_TC_GROUP_M * p.ntn;
      const int g = tile / per_group, r = tile - g * per_group;
      const int gm = min(MOE_TC_GROUP_M, total_mtiles - g * MOE_TC_GROUP_M);
      nt = r / gm;
      mt = g * MOE_TC_GROUP_M + (r - nt * gm);
    } else {
      mt = tile / p.ntn;
      nt = tile - mt * p.ntn;
    }
    int lo = 0, hi = p.E - 1;  // largest e with s_pre[e] <= mt
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= mt) lo = mid;
      else hi = mid - 1;
    }
    e = lo;
    m0 = s_seg[e] + (mt - s_pre[e]) * BM;
    mend = s_seg[e + 1];
    n0 = nt * BN;
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {  // (weights only when warps 6..9 gather the A rows)
      int stage = 0;
      uint32_t phase = 0, armed_mask = 0, armed_par = 0;
      bool ok = true;
      const uint64_t pol_a = l2_policy<MOE_TC_HINT_A>();
      const uint64_t pol_b = l2_policy<MOE_TC_HINT_B>();
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int e, m0, mend, n0;
        tile_coords(tile, e, m0, mend, n0);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, s_abort)) {
            ok = false;
            break;
          }
          const uint32_t fb = full_bar(stage);
          mbar_arrive_expect_tx(fb, GATHER ? C::kBBytes : C::kStageBytes);
          armed_mask |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          const uint32_t a_dst = smem_u32(sA + (size_t)stage * kABytes);
          const uint32_t b_dst = smem_u32(sB + (size_t)stage * C::kBBytes);
          if (!GATHER) tma_load_2d_h<MOE_TC_HINT_A>(a_dst, &tmap_a, fb, kb * BK, m0, pol_a);
          if (GATEUP) {
            constexpr int HB = C::NBOX / 2;  // boxes per half
#pragma unroll
            for (int i = 0; i < HB; ++i) {
              tma_load_3d_h<MOE_TC_HINT_B>(b_dst + i * kBoxBytes, &tmap_b0, fb, n0 + 64 * i, kb * BK, e, pol_b);
              tma_load_3d_h<MOE_TC_HINT_B>(b_dst + (HB + i) * kBoxBytes, &tmap_b1, fb, n0 + 64 * i, kb * BK, e,
                                           pol_b);
            }
          } else {
#pragma unroll
            for (int i = 0; i < C::NBOX; ++i)
              tma_load_3d_h<MOE_TC_HINT_B>(b_dst + i * kBoxBytes, &tmap_b0, fb, n0 + 64 * i, kb * BK, e, pol_b);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {  // let in-flight loads land before the CTA's shared memory goes away
        for (int s = 0; s < STAGES; ++s)
          if (armed_mask & (1u << s)) mbar_wait(full_bar(s), (armed_par >> s) & 1u, nullptr, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc128 = idesc_bf16_f32(BM, C::MMA_N);
      constexpr uint32_t idesc64 = idesc_bf16_f32(64, C::MMA_N);
      int stage = 0, local = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++local) {
        uint32_t idesc = idesc128;
        if (MOE_TC_M64) {
          int e_, m0_, mend_, n0_;
          tile_coords(tile, e_, m0_, mend_, n0_);
          if (mend_ - m0_ <= 64) idesc = idesc64;
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
          if (GATHER && MOE_TC_GATHER_FENCE) fence_proxy_async_smem();  // the A rows came through cp.async
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + (size_t)stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + (size_t)stage * C::kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk) {
            // A: K-major rows of 128 B, 8-row atoms 1024 B apart; K step = 32 B inside the row.
            const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            // B: MN-major, 64-column boxes 8 KB apart (LBO), 8-row K groups 1024 B apart (SBO);
            //    K step = 16 rows = 2048 B.
            const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, kBoxBytes, 1024);
            umma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          issued = true;
          umma_commit(empty_bar(stage));  // frees this stage once its MMAs are done
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(tfull_bar(acc));  // accumulator ready for the epilogue
      }
      if (!ok && issued) {  // wait for MMAs still reading shared memory / writing TMEM
        umma_commit(drain_bar);
        mbar_wait(drain_bar, 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else if (GATHER && warp >= 6) {
    // ------------------------------------------------ A-row gather (warps 6..9)
    const int gt = (int)threadIdx.x - 192;
    int stage = 0;
    uint32_t phase = 0;
    // rows of this CTA's part of a tile (an M=64 tile reads 64 rows)
    auto tile_rows = [&](int tile, int& r0, int& r_end) {
      int e, m0, mend, n0;
      tile_coords(tile, e, m0, mend, n0);
      r0 = m0;
      r_end = min(mend, m0 + ((MOE_TC_M64 && (mend - m0 <= 64)) ? 64 : BM));
    };
    int slot[kGatherRowsPerThread];
    int tile = blockIdx.x;
    if (tile < total_tiles) {
      int r0, r_end;
      tile_rows(tile, r0, r_end);
      gather_load_slots(p, r0, r_end, gt, slot);
    }
    for (; tile < total_tiles; tile += gridDim.x) {
      const char* src[kGatherRowsPerThread];
      uint32_t dst_off[kGatherRowsPerThread];
      const int nrows = gather_rows_of_thread(p, slot, gt, src, dst_off);
      if (tile + (int)gridDim.x < total_tiles) {  // next tile's slots, in flight during this one
        int r0, r_end;
        tile_rows(tile + (int)gridDim.x, r0, r_end);
        gather_load_slots(p, r0, r_end, gt, slot);
      }
      if (!gather_tile(p, num_kb, nrows, src, dst_off, smem_u32(sA), kABytes, STAGES, stage, phase,
                       [&](int s) { return empty_bar(s); }, [&](int s) { return full_bar(s); }, s_abort))
        break;
    }
    cp_async_wait_all();
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int local = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
      if (!mbar_wait(tfull_bar(acc), acc_phase, s_abort)) break;
      tc_fence_after();
      int e, m0, mend, n0;
      tile_coords(tile, e, m0, mend, n0);
      const bool m64 = MOE_TC_M64 && (mend - m0 <= 64);
      const int row = m64 ? m0 + q * 16 + lane : m0 + q * 32 + lane;
      const bool row_ok = row < mend && (!m64 || lane < 16);
      const uint32_t t_base = tmem_base + (uint32_t)acc * kAccStride + ((uint32_t)(q * 32) << 16);
      __nv_bfloat16* out_row = p.out + (size_t)row * p.N;
      constexpr int NCHUNK = (BN + 31) / 32;
      // combine in the epilogue: this row's slot, weight and token row of the accumulator
      float comb_wt = 0.0f;
      float* comb_row = nullptr;
      if (!GATEUP && p.comb_acc != nullptr && row_ok) {
        const int s = __ldg(p.comb_rows + row);
        if (s >= 0 && s < p.comb_T * p.comb_k) {
          comb_wt = __ldg(p.comb_w + s);
          comb_row = p.comb_acc + (size_t)(s / p.comb_k) * p.N;
        } else {
          flag_error(kErrBadRow);
        }
      }
#pragma unroll 1
      for (int c = 0; c < NCHUNK; ++c) {
        uint32_t r0[32];
        float v[32];
        if (GATEUP) {
          uint32_t r1[32];
          tmem_ld32(t_base + c * 32, r0);
          tmem_ld32(t_base + BN + c * 32, r1);
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
        if (!GATEUP && p.comb_acc != nullptr) {
          if (comb_row != nullptr) {
#pragma unroll
            for (int g4 = 0; g4 < 8; ++g4) {
              const int col = n0 + c * 32 + g4 * 4;
              if (c * 32 + g4 * 4 < BN && col < p.N)
                atomicAdd(reinterpret_cast<float4*>(comb_row + col),
                          make_float4(comb_wt * v[g4 * 4 + 0], comb_wt * v[g4 * 4 + 1], comb_wt * v[g4 * 4 + 2],
                                      comb_wt * v[g4 * 4 + 3]));
            }
          }
        } else if (row_ok) {
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            const int col = n0 + c * 32 + g8 * 8;
            if (c * 32 + g8 * 8 < BN && col < p.N) {
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
      if (lane == 0) mbar_arrive(tempty_bar(acc));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Second half of the combine done in the down projection's epilogue: y = the
// accumulator rounded to bf16, and the accumulator zeroed for the next call.
// A thread per 8 columns.
__global__ void __launch_bounds__(256) combine_finalize_kernel(float* __restrict__ acc, size_t n8,
                                                               __nv_bfloat16* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    float4* a = reinterpret_cast<float4*>(acc) + 2 * i;
    const float4 lo = __ldcg(a), hi = __ldcg(a + 1);
    const uint4 w = make_uint4(pack_bf16x2(lo.x, lo.y), pack_bf16x2(lo.z, lo.w), pack_bf16x2(hi.x, hi.y),
                               pack_bf16x2(hi.z, hi.w));
    st_v4(y + 8 * i, w);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    a[0] = z;
    a[1] = z;
  }
}

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// ever arrives on.  The wait gives up after limit_ns, sets the timeout bit of
// the device error word and the kernel returns normally.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns);
}

// ------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (thread-safe static init).
inline EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return (EncodeTiledFn) nullptr;
  }();
  return fn;
}

// Activations [rows, K] bf16, box 64 (K) x 128 (rows), 128-byte swizzle.
inline bool make_tmap_act(CUtensorMap* m, const void* base, int rows, int K) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)BM};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Weights [E, K, N] bf16 (N contiguous), box 64 (N) x 64 (K) x 1, 128-byte swizzle.
inline bool make_tmap_weight(CUtensorMap* m, const void* base, int E, int K, int N) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)K, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)N * 2, (cuuint64_t)K * N * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)BK, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// SMs of the current device.
inline int num_sms() {
  static PerDeviceInt sms;
  const int dev = current_device();
  return sms.get(dev, [&] {
    int n = 0;
    return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0 ? n : 148;
  });
}

template <bool GATEUP, int BN, int STAGES, bool GATHER = false>
cudaError_t launch_tc(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1, const Params& p,
                      cudaStream_t stream) {
  using C = Cfg<GATEUP, BN, STAGES>;
  auto kern = grouped_gemm_tc_kernel<GATEUP, BN, STAGES, GATHER>;
  const size_t smem = C::smem_bytes(p.E);
  static PerDeviceOnce attr_once;  // the attribute is per device; set it once for the largest E
  cudaError_t err = attr_once.run(current_device(), [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::smem_bytes(1024));
  });
  if (err != cudaSuccess) return err;
  const long long max_tiles = ((long long)(p.S + BM - 1) / BM + p.E) * p.ntn;
  int grid = num_sms();
  if (max_tiles < grid) grid = (int)(max_tiles > 0 ? max_tiles : 1);
  err = launch_pdl(kern, grid, GATHER ? kThreads + kGatherThreads : kThreads, smem, stream, ta, tb0, tb1, p);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// h = SiLU(x_disp Wg) * (x_disp Wu), 128-column h tiles (MMA N = 256)
inline cudaError_t launch_gate_up(const void* x_disp, const void* wg, const void* wu, const int32_t* off, int E,
                                  int H, int I, int S, void* h, cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  CUtensorMap ta, tg, tu;
  if (!make_tmap_act(&ta, x_disp, S, H) || !make_tmap_weight(&tg, wg, E, H, I) || !make_tmap_weight(&tu, wu, E, H, I))
    return cudaErrorInvalidValue;
  Params p{off, E, S, H, I, (I + 127) / 128, reinterpret_cast<__nv_bfloat16*>(h), nullptr, 1, 0, nullptr};
  return launch_tc<true, 128, 4>(ta, tg, tu, p, stream);
}

// launch_gate_up with the A rows gathered from x [T, H]: dispatched row r is
// token row_to_slot[r] / k (x_disp is never formed).
inline cudaError_t launch_gate_up_gather(const void* x, int T, const int32_t* row_to_slot, int k, const void* wg,
                                         const void* wu, const int32_t* off, int E, int H, int I, int S, void* h,
                                         cudaStream_t stream) {
  if (S == 0) return cudaSuccess;
  CUtensorMap tg, tu;  // the A rows come from x through cp.async: no activation tensor map
  if (!make_tmap_weight(&tg, wg, E, H, I) || !make_tmap_weight(&tu, wu, E, H, I)) return cudaErrorInvalidValue;
  Params p{off, E, S, H, I, (I + 127) / 128, reinterpret_cast<__nv_bfloat16*>(h), row_to_slot, k, T, x};
  return launch_tc<true, 128, 4, true>(tg, tg, tu, p, stream);
}

// y_disp = h Wd; n-tile width chosen to cover H with the least padding.
// With `comb` (comb_rows, comb_w, comb_acc, comb_k, comb_T set) the epilogue
// adds w * (h Wd) into comb_acc by token instead of writing y.
inline cudaError_t launch_down(const void* h, const void* wd, const int32_t* off, int E, int H, int I, int S,
                               void* y, cudaStream_t stream, const Params* comb = nullptr) {
  if (S == 0) return cudaSuccess;
  CUtensorMap ta, tb;
  if (!make_tmap_act(&ta, h, S, I) || !make_tmap_weight(&tb, wd, E, I, H)) return cudaErrorInvalidValue;
  // n-tile width: UMMA N that is a whole number of 64-column boxes runs best
  // (measured: N = 240 is slower than N = 256 even counting 256's padding), so
  // pick among 256 / 192 / 128 by padded width times a per-width cost.
  const int cands[3] = {256, 192, 128};
  const double cost[3] = {1.0, 1.08, 1.3};
  int best = 256;
  double best_cost = -1.0;
  for (int i = 0; i < 3; ++i) {
    const double c = (double)((H + cands[i] - 1) / cands[i]) * cands[i] * cost[i];
    if (best_cost < 0 || c < best_cost) {
      best_cost = c;
      best = cands[i];
    }
  }
  if (MOE_TC_DOWN_BN > 0) best = MOE_TC_DOWN_BN;
  Params p{off, E, S, I, H, (H + best - 1) / best, reinterpret_cast<__nv_bfloat16*>(y), nullptr, 1, 0, nullptr};
  if (comb != nullptr) {
    p.comb_rows = comb->comb_rows;
    p.comb_w = comb->comb_w;
    p.comb_acc = comb->comb_acc;
    p.comb_k = comb->comb_k;
    p.comb_T = comb->comb_T;
  }
  switch (best) {
    case 256:
      return launch_tc<false, 256, 4>(ta, tb, tb, p, stream);
    case 192:
      return launch_tc<false, 192, 5>(ta, tb, tb, p, stream);
    default:
      return launch_tc<false, 128, 6>(ta, tb, tb, p, stream);
  }
}

inline cudaError_t launch_combine_finalize(float* acc, int T, int H, void* y, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const size_t n8 = (size_t)T * H / 8;
  int sms = 0;
  cudaError_t err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, current_device());
  if (err != cudaSuccess) return err;
  size_t blocks = (n8 + 255) / 256;
  if (blocks > (size_t)sms * 8) blocks = (size_t)sms * 8;
  err = launch_pdl(combine_finalize_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, acc, n8,
                   reinterpret_cast<__nv_bfloat16*>(y));
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace tc
}  // namespace moe
