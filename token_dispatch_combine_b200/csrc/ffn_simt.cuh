// Grouped SwiGLU expert MLP on CUDA cores, for float32 layers.
//
// "EP: Partition Experts and Route Tokens", "Send tokens to experts and
// return their results": an expert's rows are stacked and multiplied by that
// expert's weights, with no mixing across rows.  Expert form (Shazeer, "GLU
// Variants Improve Transformer"): h = SiLU(x Wg) * (x Wu), y = h Wd.
//
// float32 inputs need float32 products: tcgen05's tf32 kind keeps 10 mantissa
// bits, too few for a 1e-4 relative bound, so this path uses FFMA.  A CTA
// computes one 64x64 output tile of one expert's segment (4x4 per thread,
// K staged through shared memory 16 at a time).  The tile list is derived on
// the device from expert_offsets: CTA x maps to (expert, m-tile) by walking
// the per-expert tile counts; CTAs past the last tile exit.
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

// Clamped segment of expert e: [lo, hi) within [0, S); flags inconsistent offsets.
__device__ __forceinline__ void expert_segment(const int32_t* __restrict__ off, int e, int S, int& lo, int& hi) {
  int a = __ldg(off + e), b = __ldg(off + e + 1);
  if (a < 0 || b < a || b > S) {
    if (threadIdx.x == 0) flag_error(kErrBadOffsets);
    a = min(max(a, 0), S);
    b = min(max(b, a), S);
  }
  lo = a;
  hi = b;
}

// gather != nullptr (gate/up only): A row r is row gather[r] / gk of A [gT, K]
// (the token's row of x) instead of row r.
template <typename T, bool GATEUP>
__global__ void __launch_bounds__(256) ffn_simt_kernel(const T* __restrict__ A, const T* __restrict__ B0,
                                                       const T* __restrict__ B1, const int32_t* __restrict__ off,
                                                       int E, int K, int N, int S, T* __restrict__ out,
                                                       const int32_t* __restrict__ gather, int gk, int gT) {
  constexpr int BM = 64, BN = 64, BK = 16;
  __shared__ float As[BK][BM + 4];
  __shared__ int s_src[BM];  // source row of A for each tile row (-1: none)
  __shared__ float Bs0[BK][BN];
  __shared__ float Bs1[GATEUP ? BK : 1][GATEUP ? BN : 1];

  pdl_wait();
  pdl_trigger();
  // map blockIdx.x -> (expert, m-tile)
  int e = -1, row0 = 0, row_end = 0;
  {
    int acc = 0;
    for (int x = 0; x < E; ++x) {
      int lo, hi;
      expert_segment(off, x, S, lo, hi);
      const int nt = (hi - lo + BM - 1) / BM;
      if ((int)blockIdx.x < acc + nt) {
        e = x;
        row0 = lo + ((int)blockIdx.x - acc) * BM;
        row_end = hi;
        break;
      }
      acc += nt;
    }
  }
  if (e < 0) return;
  const int n0 = blockIdx.y * BN;
  const size_t wstride = (size_t)K * N;
  const T* b0 = B0 + (size_t)e * wstride;
  const T* b1 = GATEUP ? B1 + (size_t)e * wstride : nullptr;

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 x 16 threads, 4 x 4 outputs each
  float acc0[4][4] = {}, acc1[4][4] = {};
  if (threadIdx.x < BM) {
    const int row = row0 + (int)threadIdx.x;
    int src = row < row_end ? row : -1;
    if (gather != nullptr && src >= 0) {
      const int sl = __ldg(gather + row);
      src = sl / gk;
      if (sl < 0 || src >= gT) {
        flag_error(kErrBadRow);
        src = -1;
      }
    }
    s_src[threadIdx.x] = src;
  }
  __syncthreads();

  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = threadIdx.x; i < BM * BK; i += 256) {
      const int r = i / BK, kk = i % BK;
      const int src = s_src[r], kx = k0 + kk;
      As[kk][r] = (src >= 0 && kx < K) ? (float)A[(size_t)src * K + kx] : 0.0f;
    }
    for (int i = threadIdx.x; i < BK * BN; i += 256) {
      const int kk = i / BN, c = i % BN;
      const int kx = k0 + kk, col = n0 + c;
      const bool ok = kx < K && col < N;
      Bs0[kk][c] = ok ? (float)b0[(size_t)kx * N + col] : 0.0f;
      if constexpr (GATEUP) Bs1[kk][c] = ok ? (float)b1[(size_t)kx * N + col] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], bv0[4], bv1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bv0[j] = Bs0[kk][tx * 4 + j];
        if constexpr (GATEUP) bv1[j] = Bs1[kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], bv0[j], acc0[i][j]);
          if constexpr (GATEUP) acc1[i][j] = fmaf(a[i], bv1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = row0 + ty * 4 + i;
    if (row >= row_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + tx * 4 + j;
      if (col >= N) continue;
      const float v = GATEUP ? silu_mul(acc0[i][j], acc1[i][j]) : acc0[i][j];
      out[(size_t)row * N + col] = (T)v;
    }
  }
}

template <typename T>
cudaError_t launch_ffn_simt_gate_up(const T* x_disp, const T* wg, const T* wu, const int32_t* off, int E, int H,
                                    int I, int S, T* h, cudaStream_t stream) {
  const int max_mtiles = (S + 63) / 64 + E;  // bound on sum_e ceil(count_e / 64)
  if (S == 0) return cudaSuccess;
  dim3 grid(max_mtiles, (I + 63) / 64);
  cudaError_t err = launch_pdl(ffn_simt_kernel<T, true>, grid, 256, 0, stream, x_disp, wg, wu, off, E, H, I, S, h,
                               (const int32_t*)nullptr, 1, 0);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// launch_ffn_simt_gate_up with the A rows gathered from x [T, H] by row_to_slot / k.
template <typename T>
cudaError_t launch_ffn_simt_gate_up_gather(const T* x, int T_, const int32_t* row_to_slot, int k, const T* wg,
                                           const T* wu, const int32_t* off, int E, int H, int I, int S, T* h,
                                           cudaStream_t stream) {
  const int max_mtiles = (S + 63) / 64 + E;
  if (S == 0) return cudaSuccess;
  dim3 grid(max_mtiles, (I + 63) / 64);
  cudaError_t err = launch_pdl(ffn_simt_kernel<T, true>, grid, 256, 0, stream, x, wg, wu, off, E, H, I, S, h,
                               row_to_slot, k, T_);
  return err != cudaSuccess ? err : cudaGetLastError();
}

template <typename T>
cudaError_t launch_ffn_simt_down(const T* h, const T* wd, const int32_t* off, int E, int H, int I, int S, T* y,
                                 cudaStream_t stream) {
  const int max_mtiles = (S + 63) / 64 + E;
  if (S == 0) return cudaSuccess;
  dim3 grid(max_mtiles, (H + 63) / 64);
  cudaError_t err = launch_pdl(ffn_simt_kernel<T, false>, grid, 256, 0, stream, h, wd, (const T*)nullptr, off, E, I,
                               H, S, y, (const int32_t*)nullptr, 1, 0);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
