// C ABI of the MoE round trip (declared in include/moe_b200.h).
//
// Host side only validates arguments, picks kernel configurations and
// enqueues launches on the caller's stream.  It never allocates, never copies
// to the host and never synchronises (moe_get_error excepted).
#include <cuda.h>

#include <atomic>
#include <cstdio>
#include <mutex>
#include <string>

#include "combine.cuh"
#include "common.cuh"
#include "dispatch.cuh"
#include "ffn_simt.cuh"
#include "ffn_tc.cuh"
#include "ffn_tc2.cuh"
#include "route.cuh"
#include "ep.cuh"
#include "eplb.cuh"
#include "masked.cuh"
#include "router.cuh"

namespace {

std::atomic<int> g_ffn_tiling{MOE_FFN_TILING_AUTO};

// Pair tiles pad each expert's rows to 256 instead of 128; they pay off once
// the average expert holds enough rows (measured: 512 rows per expert gain,
// 256 lose).
// Auto tiling: pair tiles from this many rows per expert on.  An expert whose
// rows leave a remainder of at most 128 past a multiple of 256 ends in an
// M=128 pair tile that costs about as much as a full one, so the gate/up
// projection (the longer one) needs a few more rows per expert than down
// before the pair tiles' lower per-row cost wins.
constexpr int kPairMinRowsGateUp = 448;
constexpr int kPairMinRowsDown = 384;

int resolve_tiling(int E, int S, bool gate_up) {
  const int mode = g_ffn_tiling.load(std::memory_order_relaxed);
  if (mode != MOE_FFN_TILING_AUTO) return mode;
  const long long need = (long long)(gate_up ? kPairMinRowsGateUp : kPairMinRowsDown) * E;
  return (long long)S >= need ? MOE_FFN_TILING_PAIR : MOE_FFN_TILING_SINGLE;
}

thread_local std::string g_last_msg;

moe_status fail(moe_status st, const std::string& msg) {
  g_last_msg = msg;
  return st;
}

moe_status cuda_status(cudaError_t err, const char* where) {
  if (err == cudaSuccess) return MOE_OK;
  return fail(MOE_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(err));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t dtype_size(int dt) { return dt == MOE_F32 ? 4 : dt == MOE_BF16 ? 2 : 0; }

#define MOE_REQUIRE(cond, msg)                                   \
  do {                                                           \
    if (!(cond)) return fail(MOE_ERR_INVALID_ARG, (msg));        \
  } while (0)

#define MOE_REQUIRE_PTR(p, a, name)                                                              \
  do {                                                                                           \
    MOE_REQUIRE((p) != nullptr, std::string(name) + " is NULL");                                 \
    MOE_REQUIRE(aligned((p), (a)), std::string(name) + " is not " #a "-byte aligned");           \
  } while (0)

moe_status check_k_e(int k, int E) {
  MOE_REQUIRE(E >= 1 && E <= 1024, "E must be in [1, 1024]");
  MOE_REQUIRE(k >= 1 && k <= 8 && k <= E, "k must be in [1, min(E, 8)]");
  return MOE_OK;
}

}  // namespace

extern "C" {

int moe_abi_version(void) { return 2; }

moe_status moe_set_ffn_tiling(int mode) {
  if (mode != MOE_FFN_TILING_AUTO && mode != MOE_FFN_TILING_SINGLE && mode != MOE_FFN_TILING_PAIR)
    return fail(MOE_ERR_INVALID_ARG, "moe_set_ffn_tiling: mode must be 0 (auto), 1 (single) or 2 (pair)");
  g_ffn_tiling.store(mode, std::memory_order_relaxed);
  return MOE_OK;
}

int moe_get_ffn_tiling(void) { return g_ffn_tiling.load(std::memory_order_relaxed); }

int moe_ffn_tiling_for(int E, int S, int projection) {
  if (E <= 0 || S < 0 || (projection != MOE_FFN_GATE_UP && projection != MOE_FFN_DOWN)) return -1;
  return resolve_tiling(E, S, projection == MOE_FFN_GATE_UP);
}

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK:
      return "ok";
    case MOE_ERR_INVALID_ARG:
      return "invalid argument";
    case MOE_ERR_UNSUPPORTED:
      return "unsupported";
    case MOE_ERR_CUDA:
      return "CUDA error";
    case MOE_ERR_DEVICE:
      return "device flagged bad data";
    case MOE_ERR_TIMEOUT:
      return "device wait timed out";
    default:
      return "unknown status";
  }
}

const char* moe_last_error_message(void) { return g_last_msg.c_str(); }

moe_status moe_route(const float* logits, int T, int E, int k, int32_t* topk_ids, float* topk_w, void* stream) {
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  moe_status st = check_k_e(k, E);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  MOE_REQUIRE_PTR(logits, 4, "logits");
  MOE_REQUIRE_PTR(topk_ids, 4, "topk_ids");
  MOE_REQUIRE_PTR(topk_w, 4, "topk_w");
  return cuda_status(moe::launch_route(logits, T, E, k, topk_ids, topk_w, (cudaStream_t)stream), "moe_route");
}

moe_status moe_router_topk(const void* x, const void* w_router, const float* bias, int T, int H, int E, int k,
                           float* logits, int32_t* topk_ids, float* topk_w, void* stream) {
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  moe_status st = check_k_e(k, E);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(E <= 256, "moe_router_topk: E must be <= 256");
  MOE_REQUIRE(H >= 8 && H % 8 == 0, "moe_router_topk: H must be a positive multiple of 8");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE_PTR(x, 16, "x");
  MOE_REQUIRE_PTR(w_router, 16, "w_router");
  if (bias != nullptr) MOE_REQUIRE_PTR(bias, 4, "bias");
  if (logits != nullptr) MOE_REQUIRE_PTR(logits, 4, "logits");
  MOE_REQUIRE_PTR(topk_ids, 4, "topk_ids");
  MOE_REQUIRE_PTR(topk_w, 4, "topk_w");
  const moe::tc::RouterParams p{bias, T, H, E, k, logits, topk_ids, topk_w};
  return cuda_status(moe::tc::launch_router(x, w_router, p, (cudaStream_t)stream), "moe_router_topk");
}

size_t moe_dispatch_workspace_bytes(int T, int k, int E, int R) {
  if (T < 0 || k < 1 || E < 1 || R < 1) return 0;
  return moe::dispatch_ws_bytes(moe::make_dispatch_geom(T, k, E, R));
}

}  // extern "C"

namespace {

// Host-side checks of a dispatch call; nothing is enqueued.  The workspace
// pointer and size are checked only when `check_workspace` is set (the
// no-alloc form supplies its own).
moe_status check_dispatch(const void* x, int dtype, int T, int H, const int32_t* topk_ids, int k, int E, int R,
                          const void* x_disp, const int32_t* expert_counts, const int32_t* expert_offsets,
                          const int32_t* rank_counts, const int32_t* rank_offsets, const int32_t* slot_to_row,
                          const int32_t* row_to_slot, const int32_t* src_expert_counts, bool check_workspace,
                          const void* workspace, size_t workspace_bytes, int max_chunk = moe::kDispatchThreads) {
  const size_t es = dtype_size(dtype);
  MOE_REQUIRE(es != 0, "dtype must be MOE_F32 or MOE_BF16");
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  MOE_REQUIRE(H >= 1 && (H * es) % 16 == 0, "H * sizeof(dtype) must be a positive multiple of 16");
  moe_status st = check_k_e(k, E);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(R >= 1 && E % R == 0, "R must be >= 1 and divide E");
  MOE_REQUIRE((long long)T * k < (1LL << 31), "T * k must be < 2^31");
  MOE_REQUIRE_PTR(expert_counts, 4, "expert_counts");
  MOE_REQUIRE_PTR(expert_offsets, 4, "expert_offsets");
  MOE_REQUIRE_PTR(rank_counts, 4, "rank_counts");
  MOE_REQUIRE_PTR(rank_offsets, 4, "rank_offsets");
  MOE_REQUIRE(src_expert_counts == nullptr || aligned(src_expert_counts, 4), "src_expert_counts misaligned");
  if (check_workspace) {
    MOE_REQUIRE_PTR(workspace, 16, "workspace");
    MOE_REQUIRE(workspace_bytes >= moe::dispatch_ws_bytes(moe::make_dispatch_geom(T, k, E, R, max_chunk)),
                max_chunk == moe::kDispatchThreads ? "workspace_bytes smaller than moe_dispatch_workspace_bytes()"
                                                   : "workspace_bytes smaller than moe_route_count_workspace_bytes()");
  }
  MOE_REQUIRE((x == nullptr) == (x_disp == nullptr),
              "x and x_disp must both be given, or both be NULL (index-only dispatch)");
  if (T > 0) {
    if (x != nullptr) {
      MOE_REQUIRE_PTR(x, 16, "x");
      MOE_REQUIRE_PTR(x_disp, 16, "x_disp");
    }
    MOE_REQUIRE_PTR(topk_ids, 4, "topk_ids");
    MOE_REQUIRE_PTR(slot_to_row, 4, "slot_to_row");
    MOE_REQUIRE_PTR(row_to_slot, 4, "row_to_slot");
  }
  return MOE_OK;
}

// Enqueues the dispatch kernel of a call that passed check_dispatch.
cudaError_t enqueue_dispatch(const void* x, int dtype, int T, int H, const int32_t* topk_ids, int k, int E, int R,
                             void* x_disp, int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                             int32_t* rank_offsets, int32_t* slot_to_row, int32_t* row_to_slot,
                             int32_t* src_expert_counts, void* workspace, cudaStream_t s,
                             uint64_t limit_ns = moe::kGridBarrierLimitNs, bool counted = false) {
  const moe::DispatchGeom g =
      moe::make_dispatch_geom(T, k, E, R, counted ? moe::kCountedChunk : moe::kDispatchThreads);
  if (dtype == MOE_BF16)
    return moe::launch_dispatch(g, H, (const __nv_bfloat16*)x, topk_ids, workspace, (__nv_bfloat16*)x_disp,
                                expert_counts, expert_offsets, rank_counts, rank_offsets, slot_to_row, row_to_slot,
                                src_expert_counts, s, limit_ns, false, counted);
  return moe::launch_dispatch(g, H, (const float*)x, topk_ids, workspace, (float*)x_disp, expert_counts,
                              expert_offsets, rank_counts, rank_offsets, slot_to_row, row_to_slot, src_expert_counts,
                              s, limit_ns, false, counted);
}

}  // namespace

extern "C" {

moe_status moe_dispatch(const void* x, int dtype, int T, int H, const int32_t* topk_ids, int k, int E, int R,
                        void* x_disp, int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                        int32_t* rank_offsets, int32_t* slot_to_row, int32_t* row_to_slot,
                        int32_t* src_expert_counts, void* workspace, size_t workspace_bytes, void* stream) {
  moe_status st = check_dispatch(x, dtype, T, H, topk_ids, k, E, R, x_disp, expert_counts, expert_offsets,
                                 rank_counts, rank_offsets, slot_to_row, row_to_slot, src_expert_counts, true,
                                 workspace, workspace_bytes);
  if (st != MOE_OK) return st;
  return cuda_status(enqueue_dispatch(x, dtype, T, H, topk_ids, k, E, R, x_disp, expert_counts, expert_offsets,
                                      rank_counts, rank_offsets, slot_to_row, row_to_slot, src_expert_counts,
                                      workspace, (cudaStream_t)stream),
                     "moe_dispatch");
}

size_t moe_route_count_workspace_bytes(int T, int k, int E, int R) {
  if (T < 0 || k < 1 || E < 1 || R < 1) return 0;
  return moe::dispatch_ws_bytes(moe::make_dispatch_geom(T, k, E, R, moe::kCountedChunk));
}

moe_status moe_route_count(const float* logits, int T, int E, int k, int R, int32_t* topk_ids, float* topk_w,
                           void* workspace, size_t workspace_bytes, void* stream) {
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  moe_status st = check_k_e(k, E);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(R >= 1 && E % R == 0, "R must be >= 1 and divide E");
  MOE_REQUIRE((long long)T * k < (1LL << 31), "T * k must be < 2^31");
  MOE_REQUIRE_PTR(workspace, 16, "workspace");
  const moe::DispatchGeom g = moe::make_dispatch_geom(T, k, E, R, moe::kCountedChunk);
  MOE_REQUIRE(workspace_bytes >= moe::dispatch_ws_bytes(g),
              "workspace_bytes smaller than moe_route_count_workspace_bytes()");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE_PTR(logits, 4, "logits");
  MOE_REQUIRE_PTR(topk_ids, 4, "topk_ids");
  MOE_REQUIRE_PTR(topk_w, 4, "topk_w");
  return cuda_status(moe::launch_route_count(g, logits, topk_ids, topk_w, workspace, (cudaStream_t)stream),
                     "moe_route_count");
}

moe_status moe_dispatch_counted(const void* x, int dtype, int T, int H, const int32_t* topk_ids, int k, int E, int R,
                                void* x_disp, int32_t* expert_counts, int32_t* expert_offsets, int32_t* rank_counts,
                                int32_t* rank_offsets, int32_t* slot_to_row, int32_t* row_to_slot,
                                int32_t* src_expert_counts, void* workspace, size_t workspace_bytes, void* stream) {
  moe_status st = check_dispatch(x, dtype, T, H, topk_ids, k, E, R, x_disp, expert_counts, expert_offsets,
                                 rank_counts, rank_offsets, slot_to_row, row_to_slot, src_expert_counts, true,
                                 workspace, workspace_bytes, moe::kCountedChunk);
  if (st != MOE_OK) return st;
  return cuda_status(enqueue_dispatch(x, dtype, T, H, topk_ids, k, E, R, x_disp, expert_counts, expert_offsets,
                                      rank_counts, rank_offsets, slot_to_row, row_to_slot, src_expert_counts,
                                      workspace, (cudaStream_t)stream, moe::kGridBarrierLimitNs,
                                      /*counted=*/T > 0),  // no tokens: nothing was counted, count the empty chunks
                     "moe_dispatch_counted");
}

moe_status moe_selftest_dispatch_timeout(const void* x, int dtype, int T, int H, const int32_t* topk_ids, int k,
                                         int E, int R, void* x_disp, int32_t* expert_counts,
                                         int32_t* expert_offsets, int32_t* rank_counts, int32_t* rank_offsets,
                                         int32_t* slot_to_row, int32_t* row_to_slot, int32_t* src_expert_counts,
                                         void* workspace, size_t workspace_bytes, unsigned int limit_us,
                                         void* stream) {
  MOE_REQUIRE(limit_us >= 1 && limit_us <= 1000000u, "limit_us must be in [1, 1000000]");
  MOE_REQUIRE(T >= 1, "T must be >= 1 (a call with no tokens launches nothing)");
  moe_status st = check_dispatch(x, dtype, T, H, topk_ids, k, E, R, x_disp, expert_counts, expert_offsets,
                                 rank_counts, rank_offsets, slot_to_row, row_to_slot, src_expert_counts, true,
                                 workspace, workspace_bytes);
  if (st != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // An arrival count far above any grid size: no arrival can be the last, so
  // the first grid barrier runs out in every CTA.
  cudaError_t err = cudaMemsetAsync(static_cast<char*>(workspace) + moe::kDispatchBarCountOffset, 0x40, 4, s);
  if (err != cudaSuccess) return cuda_status(err, "moe_selftest_dispatch_timeout: preset arrival count");
  return cuda_status(enqueue_dispatch(x, dtype, T, H, topk_ids, k, E, R, x_disp, expert_counts, expert_offsets,
                                      rank_counts, rank_offsets, slot_to_row, row_to_slot, src_expert_counts,
                                      workspace, s, (uint64_t)limit_us * 1000ull),
                     "moe_selftest_dispatch_timeout");
}

// ---------------------------------------------------------------------------
// moe_dispatch_noalloc: moe_dispatch with its scratch in a fixed device array.
//
// Some callers cannot hand this library a workspace: their own interface has
// no slot for one, and they may not call cudaMalloc on their execution path
// (a host framework that owns every allocation, or code that must not risk
// the implicit device synchronisation and heap growth of cudaMalloc).  For
// them the dispatch scratch lives in the array below, which the CUDA module
// reserves on every GPU that loads this library and keeps until the process
// exits.  Host code never touches the array by name (that name is only a
// host-side stand-in); its device address is looked up with
// cudaGetSymbolAddress once per CUDA context (the device's primary context,
// or any other context current at the call) and passed to the kernels.
static __device__ __align__(256) unsigned char g_dispatch_noalloc_scratch[MOE_DISPATCH_NOALLOC_SCRATCH_BYTES];

namespace {
// cuCtxGetCurrent / cuCtxGetId, fetched from the driver through the runtime
// (no link against libcuda).  Context ids are unique for the life of the
// process, so a context created later (after cudaDeviceReset, or one a caller
// made current with the driver API) never matches an old entry.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct NoallocEntry {
  unsigned long long ctx_id;
  void* addr;
};
constexpr int kNoallocEntries = 64;
std::mutex g_noalloc_mu;
NoallocEntry g_noalloc_cache[kNoallocEntries] = {};
int g_noalloc_next = 0;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

moe_status current_context_id(unsigned long long* id) {
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) {
    void* f0 = nullptr;
    void* f1 = nullptr;
    cudaDriverEntryPointQueryResult q0, q1;
    cudaError_t err = cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f0, 12000, cudaEnableDefault, &q0);
    if (err == cudaSuccess)
      err = cudaGetDriverEntryPointByVersion("cuCtxGetId", &f1, 12000, cudaEnableDefault, &q1);
    if (err != cudaSuccess) return cuda_status(err, "moe_dispatch_noalloc: driver entry points");
    if (q0 != cudaDriverEntryPointSuccess || q1 != cudaDriverEntryPointSuccess || !f0 || !f1)
      return fail(MOE_ERR_CUDA, "moe_dispatch_noalloc: cuCtxGetCurrent/cuCtxGetId not available");
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f0);
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f1);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || g_ctx_get_id(ctx, id) != CUDA_SUCCESS)
    return fail(MOE_ERR_CUDA, "moe_dispatch_noalloc: no current CUDA context");
  return MOE_OK;
}

// Device address of the scratch array in the current context: looked up with
// cudaGetSymbolAddress on the first call in a context (the set-up step), then
// taken from the table.
moe_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);  // the runtime makes the device's primary context current if none is
  if (err != cudaSuccess) return cuda_status(err, "moe_dispatch_noalloc: cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long id = 0;
  moe_status st = current_context_id(&id);
  if (st != MOE_OK) {
    // A context the runtime has not created yet: the symbol lookup creates it.
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_dispatch_noalloc_scratch);
    if (err != cudaSuccess) return cuda_status(err, "moe_dispatch_noalloc: cudaGetSymbolAddress");
    st = current_context_id(&id);
    if (st != MOE_OK) return st;
  }
  for (const NoallocEntry& e : g_noalloc_cache)
    if (e.addr != nullptr && e.ctx_id == id) {
      *out = e.addr;
      return MOE_OK;
    }
  void* p = nullptr;
  err = cudaGetSymbolAddress(&p, g_dispatch_noalloc_scratch);
  if (err != cudaSuccess) return cuda_status(err, "moe_dispatch_noalloc: cudaGetSymbolAddress");
  g_noalloc_cache[g_noalloc_next] = NoallocEntry{id, p};
  g_noalloc_next = (g_noalloc_next + 1) % kNoallocEntries;
  *out = p;
  return MOE_OK;
}
}  // namespace

extern "C" moe_status moe_dispatch_noalloc(const void* x, int dtype, int T, int H, const int32_t* topk_ids, int k,
                                           int E, int R, void* x_disp, int32_t* expert_counts,
                                           int32_t* expert_offsets, int32_t* rank_counts, int32_t* rank_offsets,
                                           int32_t* slot_to_row, int32_t* row_to_slot, int32_t* src_expert_counts,
                                           void* stream) {
  // 1. sizes against the built-in scratch, 2. every other argument, 3. only
  // then any device work: a rejected call enqueues nothing.
  MOE_REQUIRE(T >= 0 && k >= 1 && E >= 1 && R >= 1, "T >= 0, k >= 1, E >= 1 and R >= 1 are required");
  MOE_REQUIRE((long long)T * k < (1LL << 31), "T * k must be < 2^31");
  const size_t need = moe_dispatch_workspace_bytes(T, k, E, R);
  MOE_REQUIRE(need <= (size_t)MOE_DISPATCH_NOALLOC_SCRATCH_BYTES,
              "moe_dispatch_noalloc: these sizes need " + std::to_string(need) +
                  " bytes of scratch, more than the built-in " +
                  std::to_string((size_t)MOE_DISPATCH_NOALLOC_SCRATCH_BYTES) + "; use moe_dispatch with a workspace");
  moe_status st = check_dispatch(x, dtype, T, H, topk_ids, k, E, R, x_disp, expert_counts, expert_offsets,
                                 rank_counts, rank_offsets, slot_to_row, row_to_slot, src_expert_counts, false,
                                 nullptr, 0);
  if (st != MOE_OK) return st;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  // The array keeps whatever the previous call left; the control words must start at zero.
  cudaError_t err = cudaMemsetAsync(scratch, 0, 256, s);
  if (err != cudaSuccess) return cuda_status(err, "moe_dispatch_noalloc: clear control words");
  return cuda_status(enqueue_dispatch(x, dtype, T, H, topk_ids, k, E, R, x_disp, expert_counts, expert_offsets,
                                      rank_counts, rank_offsets, slot_to_row, row_to_slot, src_expert_counts, scratch,
                                      s),
                     "moe_dispatch_noalloc");
}

static moe_status check_ffn(int dtype, int E, int H, int I, int S, const void* a, const char* a_name,
                            const int32_t* off) {
  const size_t es = dtype_size(dtype);
  MOE_REQUIRE(es != 0, "dtype must be MOE_F32 or MOE_BF16");
  MOE_REQUIRE(E >= 1 && E <= 1024, "E must be in [1, 1024]");
  MOE_REQUIRE(H >= 1 && I >= 1, "H and I must be >= 1");
  MOE_REQUIRE((H * es) % 16 == 0 && (I * es) % 16 == 0, "H * sizeof(dtype) and I * sizeof(dtype) must be multiples of 16");
  MOE_REQUIRE(S >= 0, "S must be >= 0");
  MOE_REQUIRE_PTR(off, 4, "expert_offsets");
  if (S > 0) MOE_REQUIRE_PTR(a, 16, a_name);
  return MOE_OK;
}

moe_status moe_ffn_gate_up(const void* x_disp, int dtype, const void* w_gate, const void* w_up,
                           const int32_t* expert_offsets, int E, int H, int I, int S, void* h, void* stream) {
  moe_status st = check_ffn(dtype, E, H, I, S, x_disp, "x_disp", expert_offsets);
  if (st != MOE_OK) return st;
  if (S == 0) return MOE_OK;
  MOE_REQUIRE_PTR(w_gate, 16, "w_gate");
  MOE_REQUIRE_PTR(w_up, 16, "w_up");
  MOE_REQUIRE_PTR(h, 16, "h");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t err;
  if (dtype == MOE_BF16)
    err = resolve_tiling(E, S, true) == MOE_FFN_TILING_PAIR
              ? moe::tc::launch_gate_up_pair(x_disp, w_gate, w_up, expert_offsets, E, H, I, S, h, s)
              : moe::tc::launch_gate_up(x_disp, w_gate, w_up, expert_offsets, E, H, I, S, h, s);
  else
    err = moe::launch_ffn_simt_gate_up((const float*)x_disp, (const float*)w_gate, (const float*)w_up,
                                       expert_offsets, E, H, I, S, (float*)h, s);
  return cuda_status(err, "moe_ffn_gate_up");
}

moe_status moe_ffn_down(const void* h, int dtype, const void* w_down, const int32_t* expert_offsets, int E, int H,
                        int I, int S, void* y_disp, void* stream) {
  moe_status st = check_ffn(dtype, E, H, I, S, h, "h", expert_offsets);
  if (st != MOE_OK) return st;
  if (S == 0) return MOE_OK;
  MOE_REQUIRE_PTR(w_down, 16, "w_down");
  MOE_REQUIRE_PTR(y_disp, 16, "y_disp");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t err;
  if (dtype == MOE_BF16)
    err = resolve_tiling(E, S, false) == MOE_FFN_TILING_PAIR
              ? moe::tc::launch_down_pair(h, w_down, expert_offsets, E, H, I, S, y_disp, s)
              : moe::tc::launch_down(h, w_down, expert_offsets, E, H, I, S, y_disp, s);
  else
    err = moe::launch_ffn_simt_down((const float*)h, (const float*)w_down, expert_offsets, E, H, I, S,
                                    (float*)y_disp, s);
  return cuda_status(err, "moe_ffn_down");
}

moe_status moe_ffn_down_combine(const void* h, int dtype, const void* w_down, const int32_t* expert_offsets, int E,
                                int H, int I, int S, const int32_t* row_to_slot, const float* topk_w, int T, int k,
                                float* y_acc, void* stream) {
  moe_status st = check_ffn(dtype, E, H, I, S, h, "h", expert_offsets);
  if (st != MOE_OK) return st;
  if (dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "moe_ffn_down_combine: bf16 only");
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= 8, "T >= 0 and k in [1, 8] are required");
  MOE_REQUIRE((long long)T * k < (1LL << 31) && S <= T * k, "S must be <= T * k < 2^31");
  if (S == 0) return MOE_OK;
  MOE_REQUIRE_PTR(w_down, 16, "w_down");
  MOE_REQUIRE_PTR(row_to_slot, 4, "row_to_slot");
  MOE_REQUIRE_PTR(topk_w, 4, "topk_w");
  MOE_REQUIRE_PTR(y_acc, 16, "y_acc");
  moe::tc::Params comb = {};
  comb.comb_rows = row_to_slot;
  comb.comb_w = topk_w;
  comb.comb_acc = y_acc;
  comb.comb_k = k;
  comb.comb_T = T;
  return cuda_status(moe::tc::launch_down(h, w_down, expert_offsets, E, H, I, S, nullptr, (cudaStream_t)stream, &comb),
                     "moe_ffn_down_combine");
}

moe_status moe_combine_finalize(float* y_acc, int dtype, int T, int H, void* y, void* stream) {
  MOE_REQUIRE(dtype == MOE_BF16 || dtype == MOE_F32, "dtype must be MOE_F32 or MOE_BF16");
  if (dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "moe_combine_finalize: bf16 only");
  MOE_REQUIRE(T >= 0 && H >= 8 && H % 8 == 0, "T >= 0 and H a positive multiple of 8 are required");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE_PTR(y_acc, 16, "y_acc");
  MOE_REQUIRE_PTR(y, 16, "y");
  return cuda_status(moe::tc::launch_combine_finalize(y_acc, T, H, y, (cudaStream_t)stream), "moe_combine_finalize");
}

moe_status moe_expert_ffn(const void* x_disp, int dtype, const void* w_gate, const void* w_up,
                          const void* w_down, const int32_t* expert_offsets, int E, int H, int I, int S, void* h,
                          void* y_disp, void* stream) {
  moe_status st = moe_ffn_gate_up(x_disp, dtype, w_gate, w_up, expert_offsets, E, H, I, S, h, stream);
  if (st != MOE_OK) return st;
  return moe_ffn_down(h, dtype, w_down, expert_offsets, E, H, I, S, y_disp, stream);
}

moe_status moe_ffn_gate_up_gather(const void* x, int dtype, int T, const int32_t* row_to_slot, int k,
                                  const void* w_gate, const void* w_up, const int32_t* expert_offsets, int E, int H,
                                  int I, int S, void* h, void* stream) {
  moe_status st = check_ffn(dtype, E, H, I, S, x, "x", expert_offsets);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  MOE_REQUIRE(k >= 1 && k <= 8, "k must be in [1, 8]");
  MOE_REQUIRE((long long)T * k < (1LL << 31), "T * k must be < 2^31");
  MOE_REQUIRE(S <= T * k, "S must be <= T * k");
  if (S == 0) return MOE_OK;
  MOE_REQUIRE_PTR(row_to_slot, 4, "row_to_slot");
  MOE_REQUIRE_PTR(w_gate, 16, "w_gate");
  MOE_REQUIRE_PTR(w_up, 16, "w_up");
  MOE_REQUIRE_PTR(h, 16, "h");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t err;
  if (dtype == MOE_BF16)
    err = resolve_tiling(E, S, true) == MOE_FFN_TILING_PAIR
              ? moe::tc::launch_gate_up_pair_gather(x, T, row_to_slot, k, w_gate, w_up, expert_offsets, E, H, I, S,
                                                    h, s)
              : moe::tc::launch_gate_up_gather(x, T, row_to_slot, k, w_gate, w_up, expert_offsets, E, H, I, S, h, s);
  else
    err = moe::launch_ffn_simt_gate_up_gather((const float*)x, T, row_to_slot, k, (const float*)w_gate,
                                              (const float*)w_up, expert_offsets, E, H, I, S, (float*)h, s);
  return cuda_status(err, "moe_ffn_gate_up_gather");
}

moe_status moe_expert_ffn_gather(const void* x, int dtype, int T, const int32_t* row_to_slot, int k,
                                 const void* w_gate, const void* w_up, const void* w_down,
                                 const int32_t* expert_offsets, int E, int H, int I, int S, void* h, void* y_disp,
                                 void* stream) {
  moe_status st =
      moe_ffn_gate_up_gather(x, dtype, T, row_to_slot, k, w_gate, w_up, expert_offsets, E, H, I, S, h, stream);
  if (st != MOE_OK) return st;
  return moe_ffn_down(h, dtype, w_down, expert_offsets, E, H, I, S, y_disp, stream);
}

moe_status moe_combine(const void* y_disp, int dtype, const float* topk_w, const int32_t* slot_to_row, int T, int k,
                       int H, void* y, void* stream) {
  const size_t es = dtype_size(dtype);
  MOE_REQUIRE(es != 0, "dtype must be MOE_F32 or MOE_BF16");
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  MOE_REQUIRE(k >= 1 && k <= 8, "k must be in [1, 8]");
  MOE_REQUIRE(H >= 1 && (H * es) % 16 == 0, "H * sizeof(dtype) must be a positive multiple of 16");
  MOE_REQUIRE((long long)T * k < (1LL << 31), "T * k must be < 2^31");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE_PTR(y_disp, 16, "y_disp");
  MOE_REQUIRE_PTR(topk_w, 4, "topk_w");
  MOE_REQUIRE_PTR(slot_to_row, 4, "slot_to_row");
  MOE_REQUIRE_PTR(y, 16, "y");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t err;
  if (dtype == MOE_BF16)
    err = moe::launch_combine((const __nv_bfloat16*)y_disp, topk_w, slot_to_row, T, k, H, (__nv_bfloat16*)y, s);
  else
    err = moe::launch_combine((const float*)y_disp, topk_w, slot_to_row, T, k, H, (float*)y, s);
  return cuda_status(err, "moe_combine");
}

moe_status moe_combine_rank_partials(const void* y_disp, int dtype, const float* topk_w, const int32_t* topk_ids,
                                    const int32_t* slot_to_row, int T, int k, int H, int E, int R, void* y_part,
                                    void* stream) {
  const size_t es = dtype_size(dtype);
  MOE_REQUIRE(es != 0, "dtype must be MOE_F32 or MOE_BF16");
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  MOE_REQUIRE(k >= 1 && k <= 8, "k must be in [1, 8]");
  MOE_REQUIRE(H >= 1 && (H * es) % 16 == 0, "H * sizeof(dtype) must be a positive multiple of 16");
  MOE_REQUIRE(E >= 1 && E <= 1024, "E must be in [1, 1024]");
  MOE_REQUIRE(R >= 1 && E % R == 0, "R must be >= 1 and divide E");
  MOE_REQUIRE((long long)T * k < (1LL << 31), "T * k must be < 2^31");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE_PTR(y_disp, 16, "y_disp");
  MOE_REQUIRE_PTR(topk_w, 4, "topk_w");
  MOE_REQUIRE_PTR(topk_ids, 4, "topk_ids");
  MOE_REQUIRE_PTR(slot_to_row, 4, "slot_to_row");
  MOE_REQUIRE_PTR(y_part, 16, "y_part");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t err;
  if (dtype == MOE_BF16)
    err = moe::launch_rank_partials((const __nv_bfloat16*)y_disp, topk_w, topk_ids, slot_to_row, T, k, H, E, R,
                                    (__nv_bfloat16*)y_part, s);
  else
    err = moe::launch_rank_partials((const float*)y_disp, topk_w, topk_ids, slot_to_row, T, k, H, E, R,
                                    (float*)y_part, s);
  return cuda_status(err, "moe_combine_rank_partials");
}

moe_status moe_reduce_rank_partials(const void* y_part, int dtype, int T, int H, int R, void* y, void* stream) {
  const size_t es = dtype_size(dtype);
  MOE_REQUIRE(es != 0, "dtype must be MOE_F32 or MOE_BF16");
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  MOE_REQUIRE(H >= 1 && (H * es) % 16 == 0, "H * sizeof(dtype) must be a positive multiple of 16");
  MOE_REQUIRE(R >= 1 && R <= 1024, "R must be in [1, 1024]");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE_PTR(y_part, 16, "y_part");
  MOE_REQUIRE_PTR(y, 16, "y");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t err;
  if (dtype == MOE_BF16)
    err = moe::launch_reduce_ranks((const __nv_bfloat16*)y_part, T, H, R, (__nv_bfloat16*)y, s);
  else
    err = moe::launch_reduce_ranks((const float*)y_part, T, H, R, (float*)y, s);
  return cuda_status(err, "moe_reduce_rank_partials");
}

static moe_status check_ep_plan(const int32_t* topk_ids, const float* topk_w, int T, int k, int E, int R,
                                const int32_t* send_counts, const int32_t* send_offsets, const int32_t* slot_send_row,
                                const int32_t* ret_row, const int32_t* row_token, const int32_t* row_ids,
                                const float* row_w) {
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  moe_status st = check_k_e(k, E);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(R >= 1 && R <= moe::kEpMaxRanks && E % R == 0, "R must be in [1, 64] and divide E");
  MOE_REQUIRE((long long)T * k < (1LL << 31), "T * k must be < 2^31");
  MOE_REQUIRE_PTR(send_counts, 4, "send_counts");
  MOE_REQUIRE_PTR(send_offsets, 4, "send_offsets");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE_PTR(topk_ids, 4, "topk_ids");
  MOE_REQUIRE_PTR(topk_w, 4, "topk_w");
  MOE_REQUIRE_PTR(slot_send_row, 4, "slot_send_row");
  MOE_REQUIRE_PTR(ret_row, 4, "ret_row");
  MOE_REQUIRE_PTR(row_token, 4, "row_token");
  MOE_REQUIRE_PTR(row_ids, 4, "row_ids");
  MOE_REQUIRE_PTR(row_w, 4, "row_w");
  return MOE_OK;
}

size_t moe_ep_plan_workspace_bytes(int T, int R) {
  if (T < 0 || R < 1) return 0;
  return moe::ep_plan_ws_bytes(T, R);
}

moe_status moe_ep_plan(const int32_t* topk_ids, const float* topk_w, int T, int k, int E, int R,
                       int32_t* send_counts, int32_t* send_offsets, int32_t* slot_send_row, int32_t* ret_row,
                       int32_t* row_token, int32_t* row_ids, float* row_w, void* workspace, size_t workspace_bytes,
                       void* stream) {
  moe_status st = check_ep_plan(topk_ids, topk_w, T, k, E, R, send_counts, send_offsets, slot_send_row, ret_row,
                                row_token, row_ids, row_w);
  if (st != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (T == 0) {  // nothing to send: zero counts and offsets
    cudaError_t err = cudaMemsetAsync(send_counts, 0, sizeof(int32_t) * R, s);
    if (err == cudaSuccess) err = cudaMemsetAsync(send_offsets, 0, sizeof(int32_t) * (R + 1), s);
    return cuda_status(err, "moe_ep_plan");
  }
  MOE_REQUIRE_PTR(workspace, 16, "workspace");
  MOE_REQUIRE(workspace_bytes >= moe::ep_plan_ws_bytes(T, R), "workspace_bytes smaller than moe_ep_plan_workspace_bytes()");
  const moe::EpPlanArgs a = moe::ep_plan_args(topk_ids, topk_w, T, k, E, R, workspace, send_counts, send_offsets,
                                              slot_send_row, ret_row, row_token, row_ids, row_w);
  return cuda_status(moe::launch_ep_plan(a, s), "moe_ep_plan");
}

moe_status moe_ep_plan_host(const int32_t* topk_ids, const float* topk_w, int T, int k, int E, int R,
                            int32_t* send_counts, int32_t* send_offsets, int32_t* slot_send_row, int32_t* ret_row,
                            int32_t* row_token, int32_t* row_ids, float* row_w) {
  moe_status st = check_ep_plan(topk_ids, topk_w, T, k, E, R, send_counts, send_offsets, slot_send_row, ret_row,
                                row_token, row_ids, row_w);
  if (st != MOE_OK) return st;
  if (!moe::ep_plan_host(topk_ids, topk_w, T, k, E, R, send_counts, send_offsets, slot_send_row, ret_row, row_token,
                         row_ids, row_w))
    return fail(MOE_ERR_DEVICE, "moe_ep_plan_host: expert ids outside [0, E) were dropped");
  return MOE_OK;
}

moe_status moe_ep_exchange_offsets(const int32_t* counts, int R, int rank, int32_t* dst_base, int32_t* recv_base,
                                   int32_t* ret_base) {
  MOE_REQUIRE(R >= 1 && R <= moe::kEpMaxRanks, "R must be in [1, 64]");
  MOE_REQUIRE(rank >= 0 && rank < R, "rank must be in [0, R)");
  MOE_REQUIRE(counts != nullptr && dst_base != nullptr && recv_base != nullptr && ret_base != nullptr,
              "moe_ep_exchange_offsets: host arrays must not be NULL");
  for (int i = 0; i < R * R; ++i) MOE_REQUIRE(counts[i] >= 0, "counts must be >= 0");
  moe::ep_exchange_offsets_host(counts, R, rank, dst_base, recv_base, ret_base);
  return MOE_OK;
}

moe_status moe_enable_peer_access(int peer_device) {
  MOE_REQUIRE(peer_device >= 0, "peer_device must be >= 0");
  int dev = 0, n = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_status(err, "cudaGetDevice");
  err = cudaGetDeviceCount(&n);
  if (err != cudaSuccess) return cuda_status(err, "cudaGetDeviceCount");
  MOE_REQUIRE(peer_device < n, "peer_device must be below the device count");
  if (peer_device == dev) return MOE_OK;
  int can = 0;
  err = cudaDeviceCanAccessPeer(&can, dev, peer_device);
  if (err != cudaSuccess) return cuda_status(err, "cudaDeviceCanAccessPeer");
  if (!can) return fail(MOE_ERR_UNSUPPORTED, "the current device cannot access peer_device's memory");
  err = cudaDeviceEnablePeerAccess(peer_device, 0);
  if (err == cudaErrorPeerAccessAlreadyEnabled) {
    (void)cudaGetLastError();  // clear the (non-sticky) error this call recorded
    return MOE_OK;
  }
  return cuda_status(err, "cudaDeviceEnablePeerAccess");
}

moe_status moe_ep_pack(const void* x, int dtype, int T, int H, int k, int R, const int32_t* send_offsets,
                       const int32_t* dst_base, const int32_t* row_token, const int32_t* row_ids, const float* row_w,
                       void* const* dst_x, int32_t* const* dst_ids, float* const* dst_w, const int32_t* dst_cap,
                       void* stream) {
  const size_t es = dtype_size(dtype);
  MOE_REQUIRE(es != 0, "dtype must be MOE_F32 or MOE_BF16");
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  MOE_REQUIRE(H >= 1 && (H * es) % 16 == 0, "H * sizeof(dtype) must be a positive multiple of 16");
  MOE_REQUIRE(k >= 1 && k <= 8, "k must be in [1, 8]");
  MOE_REQUIRE(R >= 1 && R <= moe::kEpMaxRanks, "R must be in [1, 64]");
  MOE_REQUIRE((long long)T * k < (1LL << 31), "T * k must be < 2^31");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE_PTR(x, 16, "x");
  MOE_REQUIRE_PTR(send_offsets, 4, "send_offsets");
  MOE_REQUIRE_PTR(dst_base, 4, "dst_base");
  MOE_REQUIRE_PTR(row_token, 4, "row_token");
  MOE_REQUIRE_PTR(row_ids, 4, "row_ids");
  MOE_REQUIRE_PTR(row_w, 4, "row_w");
  MOE_REQUIRE(dst_x != nullptr && dst_ids != nullptr && dst_w != nullptr && dst_cap != nullptr,
              "dst_x, dst_ids, dst_w and dst_cap (host arrays of R entries) must not be NULL");
  moe::EpDest dst = {};
  for (int d = 0; d < R; ++d) {
    MOE_REQUIRE(dst_cap[d] >= 0, "dst_cap entries must be >= 0");
    if (dst_cap[d] > 0) {
      MOE_REQUIRE_PTR(dst_x[d], 16, "dst_x[" + std::to_string(d) + "]");
      MOE_REQUIRE_PTR(dst_ids[d], 4, "dst_ids[" + std::to_string(d) + "]");
      MOE_REQUIRE_PTR(dst_w[d], 4, "dst_w[" + std::to_string(d) + "]");
    }
    dst.x[d] = dst_x[d];
    dst.ids[d] = dst_ids[d];
    dst.w[d] = dst_w[d];
    dst.cap[d] = dst_cap[d];
  }
  const int max_rows = T * (k < R ? k : R);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t err;
  if (dtype == MOE_BF16)
    err = moe::launch_ep_pack((const __nv_bfloat16*)x, T, H, k, R, max_rows, send_offsets, dst_base, row_token, row_ids,
                              row_w, dst, s);
  else
    err = moe::launch_ep_pack((const float*)x, T, H, k, R, max_rows, send_offsets, dst_base, row_token, row_ids, row_w,
                              dst, s);
  return cuda_status(err, "moe_ep_pack");
}

moe_status moe_ep_recv_index(const int32_t* recv_ids, int T_recv, int k, int EL, int32_t* expert_counts,
                             int32_t* expert_offsets, int32_t* slot_to_row, int32_t* row_to_slot, void* workspace,
                             size_t workspace_bytes, void* stream) {
  MOE_REQUIRE(T_recv >= 0, "T_recv must be >= 0");
  // a received row holds at most min(k, EL) local ids, padded with -1 to k columns: k may exceed EL
  MOE_REQUIRE(EL >= 1 && EL <= 1024, "EL must be in [1, 1024]");
  MOE_REQUIRE(k >= 1 && k <= 8, "k must be in [1, 8]");
  MOE_REQUIRE((long long)T_recv * k < (1LL << 31), "T_recv * k must be < 2^31");
  MOE_REQUIRE_PTR(expert_counts, 4, "expert_counts");
  MOE_REQUIRE_PTR(expert_offsets, 4, "expert_offsets");
  MOE_REQUIRE_PTR(workspace, 16, "workspace");
  const moe::DispatchGeom g = moe::make_dispatch_geom(T_recv, k, EL, 1);
  MOE_REQUIRE(workspace_bytes >= moe::dispatch_ws_bytes(g), "workspace_bytes smaller than moe_dispatch_workspace_bytes(T_recv, k, EL, 1)");
  if (T_recv > 0) {
    MOE_REQUIRE_PTR(recv_ids, 4, "recv_ids");
    MOE_REQUIRE_PTR(slot_to_row, 4, "slot_to_row");
    MOE_REQUIRE_PTR(row_to_slot, 4, "row_to_slot");
  }
  // the one-rank dispatch of the received rows, index only (no row width: H is unused), no rank
  // totals; -1 ids are padding
  return cuda_status(moe::launch_dispatch<__nv_bfloat16>(g, 8, nullptr, recv_ids, workspace, nullptr, expert_counts,
                                                         expert_offsets, nullptr, nullptr, slot_to_row, row_to_slot,
                                                         nullptr, (cudaStream_t)stream, moe::kGridBarrierLimitNs, true),
                     "moe_ep_recv_index");
}

moe_status moe_eplb_plan(const int64_t* load, int E, int R, int slots_per_rank, int32_t* phys_to_logical,
                         int32_t* replica_offsets, int32_t* replicas) {
  MOE_REQUIRE(E >= 1 && R >= 1 && slots_per_rank >= 1, "E, R and slots_per_rank must be >= 1");
  MOE_REQUIRE((long long)R * slots_per_rank <= moe::kEplbMaxSlots, "R * slots_per_rank must be <= 2^20");
  MOE_REQUIRE(R * slots_per_rank >= E, "R * slots_per_rank must be >= E (every expert needs a slot)");
  MOE_REQUIRE(load != nullptr && phys_to_logical != nullptr && replica_offsets != nullptr && replicas != nullptr,
              "moe_eplb_plan: host arrays must not be NULL");
  for (int e = 0; e < E; ++e)
    MOE_REQUIRE(load[e] >= 0 && load[e] < moe::kEplbMaxLoad, "loads must be in [0, 2^40)");
  if (!moe::eplb_plan_host(load, E, R, slots_per_rank, phys_to_logical, replica_offsets, replicas))
    return fail(MOE_ERR_INVALID_ARG, "moe_eplb_plan: invalid sizes");
  return MOE_OK;
}

moe_status moe_eplb_remap(const int32_t* topk_ids, int T, int k, int E, const int32_t* replica_offsets,
                          const int32_t* replicas, int P, int32_t* phys_ids, void* stream) {
  MOE_REQUIRE(T >= 0, "T must be >= 0");
  MOE_REQUIRE(k >= 1 && k <= 8, "k must be in [1, 8]");
  MOE_REQUIRE(E >= 1 && P >= E && P <= moe::kEplbMaxSlots, "need 1 <= E <= P <= 2^20");
  MOE_REQUIRE((long long)T * k < (1LL << 31), "T * k must be < 2^31");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE_PTR(topk_ids, 4, "topk_ids");
  MOE_REQUIRE_PTR(replica_offsets, 4, "replica_offsets");
  MOE_REQUIRE_PTR(replicas, 4, "replicas");
  MOE_REQUIRE_PTR(phys_ids, 4, "phys_ids");
  return cuda_status(moe::launch_eplb_remap(topk_ids, T, k, E, replica_offsets, replicas, P, phys_ids,
                                            (cudaStream_t)stream),
                     "moe_eplb_remap");
}

moe_status moe_eplb_replicate(const void* w, size_t expert_bytes, int E, const int32_t* phys_to_logical, int P,
                              void* w_phys, void* stream) {
  MOE_REQUIRE(E >= 1 && P >= 1, "E and P must be >= 1");
  MOE_REQUIRE(phys_to_logical != nullptr, "phys_to_logical (host array) must not be NULL");
  for (int p = 0; p < P; ++p)
    MOE_REQUIRE(phys_to_logical[p] >= 0 && phys_to_logical[p] < E, "phys_to_logical entries must be in [0, E)");
  if (expert_bytes == 0) return MOE_OK;
  MOE_REQUIRE(w != nullptr && w_phys != nullptr, "w and w_phys must not be NULL");
  const char* src = static_cast<const char*>(w);
  char* dst = static_cast<char*>(w_phys);
  MOE_REQUIRE(dst + (size_t)P * expert_bytes <= src || src + (size_t)E * expert_bytes <= dst,
              "w and w_phys must not overlap");
  for (int p = 0; p < P; ++p) {
    cudaError_t err = cudaMemcpyAsync(dst + (size_t)p * expert_bytes, src + (size_t)phys_to_logical[p] * expert_bytes,
                                      expert_bytes, cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
    if (err != cudaSuccess) return cuda_status(err, "moe_eplb_replicate");
  }
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(unsigned int limit_us, void* stream) {
  MOE_REQUIRE(limit_us >= 1 && limit_us <= 1000000u, "limit_us must be in [1, 1000000]");
  moe::tc::wait_timeout_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_us * 1000ull);
  return cuda_status(cudaGetLastError(), "moe_selftest_wait_timeout");
}

moe_status moe_get_error(void* stream, uint32_t* bits_out) {
  cudaError_t err = cudaStreamSynchronize((cudaStream_t)stream);
  if (err != cudaSuccess) return cuda_status(err, "moe_get_error: stream synchronize");
  uint32_t word = 0;
  err = cudaMemcpyFromSymbol(&word, moe::g_error_word, sizeof(word));
  if (err != cudaSuccess) return cuda_status(err, "moe_get_error: read error word");
  if (bits_out) *bits_out = word;
  if (word == 0) return MOE_OK;
  const uint32_t zero = 0;
  err = cudaMemcpyToSymbol(moe::g_error_word, &zero, sizeof(zero));
  if (err != cudaSuccess) return cuda_status(err, "moe_get_error: clear error word");
  if (word & moe::kErrTimeout) return fail(MOE_ERR_TIMEOUT, "a bounded device-side wait ran out");
  return fail(MOE_ERR_DEVICE, "device skipped bad data (error word " + std::to_string(word) + ")");
}

}  // extern "C"
