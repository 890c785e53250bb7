// Shared device helpers for the MoE round-trip kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "moe_b200.h"

namespace moe {

// Error-word bits (see moe_get_error in moe_b200.h).
constexpr uint32_t kErrBadId = 1u;
constexpr uint32_t kErrBadOffsets = 2u;
constexpr uint32_t kErrBadRow = 4u;
constexpr uint32_t kErrTimeout = 8u;

// One word per device, set by kernels that skip bad data, read and cleared
// by moe_get_error.
__device__ uint32_t g_error_word;

__device__ __forceinline__ void flag_error(uint32_t bits) { atomicOr(&g_error_word, bits); }

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }

// Programmatic dependent launch.  Every kernel of this library is launched
// with programmatic stream serialisation, so it may start while the previous
// kernel in the stream is still finishing.  pdl_wait() blocks until that
// kernel has completed and its memory is visible; no global memory that a
// predecessor touches may be read or written before it.  pdl_trigger() lets
// the next kernel in the stream begin launching (it still waits in its own
// pdl_wait() for this one to complete).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch with programmatic stream serialisation allowed (see pdl_wait).
// MOE_PDL=0 launches plainly (griddepcontrol.* then return at once).
#ifndef MOE_PDL
#define MOE_PDL 1
#endif
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = MOE_PDL ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---- host-side per-device setup, safe to call from several host threads
constexpr int kMaxDevices = 64;

// Runs a setup step (e.g. raising a kernel's shared-memory limit) once per
// device; a failed step is retried by the next call.
class PerDeviceOnce {
 public:
  template <typename F>
  cudaError_t run(int dev, F&& setup) {
    if (dev < 0 || dev >= kMaxDevices) return setup();
    if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(mu_);
    if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    const cudaError_t err = setup();
    if (err == cudaSuccess) done_[dev].store(true, std::memory_order_release);
    return err;
  }

 private:
  std::mutex mu_;
  std::atomic<bool> done_[kMaxDevices] = {};
};

// A positive per-device value computed once (e.g. an occupancy bound).
class PerDeviceInt {
 public:
  template <typename F>
  int get(int dev, F&& compute) {
    if (dev < 0 || dev >= kMaxDevices) return compute();
    int v = val_[dev].load(std::memory_order_acquire);
    if (v > 0) return v;
    v = compute();
    if (v > 0) val_[dev].store(v, std::memory_order_release);
    return v;
  }

 private:
  std::atomic<int> val_[kMaxDevices] = {};
};

inline int current_device() {
  int dev = 0;
  return cudaGetDevice(&dev) == cudaSuccess ? dev : 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

template <typename T>
struct Vec16;  // 16-byte vector of T
template <>
struct Vec16<float> {
  static constexpr int N = 4;
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
};

// Widen the N elements packed in a 16-byte word to float.
__device__ __forceinline__ void unpack16(const uint4& v, float* f, float) {
  f[0] = __uint_as_float(v.x);
  f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z);
  f[3] = __uint_as_float(v.w);
}
__device__ __forceinline__ void unpack16(const uint4& v, float* f, __nv_bfloat16) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ uint4 pack16(const float* f, float) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&p);
}
__device__ __forceinline__ uint4 pack16(const float* f, __nv_bfloat16) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void st_v4(void* p, const uint4& v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

}  // namespace moe
