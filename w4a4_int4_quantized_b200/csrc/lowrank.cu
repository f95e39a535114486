// Low-rank down-projection T = X L1 of the SVDQuant branch.
//
// Method: "Krea 2 Turbo - SVDQuant" (sweettea.co), "What's included" -- a
// low-rank correction branch runs in parallel with the 4-bit matmul; reading:
// the branch takes the unrotated bf16 activations, T = X L1 accumulates in
// fp32 and is stored as bf16 for the up-projection folded into the GEMM
// epilogue.
//
// Shared-memory tiled fp32 kernel: a CTA computes a 64 x 64 tile of T with
// 256 threads (4 x 4 outputs each), staging 64 x 32 slabs of X and 32 x 64
// slabs of L1.  Rank r <= 256 keeps this a thin product (2 M K r flops).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace w4a4 {

namespace {

constexpr int TM = 64, TN = 64, TK = 32;

__device__ __forceinline__ float bf(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

__global__ void __launch_bounds__(256) lowrank_down_kernel(const uint16_t* __restrict__ X,
                                                           const uint16_t* __restrict__ L1, int M, int K, int r,
                                                           uint16_t* __restrict__ T) {
  __shared__ float xs[TK][TM + 1];
  __shared__ float ls[TK][TN + 1];
  grid_launch_dependents();
  const int m0 = blockIdx.y * TM, j0 = blockIdx.x * TN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int i = threadIdx.x; i < TM * TK; i += 256) {
      const int mm = i / TK, kk = i % TK;
      const long m = m0 + mm;
      xs[kk][mm] = (m < M) ? bf(X[m * K + k0 + kk]) : 0.0f;
    }
    for (int i = threadIdx.x; i < TK * TN; i += 256) {
      const int kk = i / TN, jj = i % TN;
      const int j = j0 + jj;
      ls[kk][jj] = (j < r) ? bf(L1[(long)(k0 + kk) * r + j]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i) b[i] = ls[kk][tx * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jv = 0; jv < 4; ++jv) acc[i][jv] = __fmaf_rn(a[i], b[jv], acc[i][jv]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int jv = 0; jv < 4; ++jv) {
      const int j = j0 + tx * 4 + jv;
      if (j < r) {
        __nv_bfloat16 h = __float2bfloat16_rn(acc[i][jv]);
        T[m * r + j] = *reinterpret_cast<uint16_t*>(&h);
      }
    }
  }
}

}  // namespace

cudaError_t launch_lowrank_down(const uint16_t* X, const uint16_t* L1, int M, int K, int r, uint16_t* T,
                                cudaStream_t st) {
  dim3 grid((r + TN - 1) / TN, (M + TM - 1) / TM);
  lowrank_down_kernel<<<grid, 256, 0, st>>>(X, L1, M, K, r, T);
  return cudaGetLastError();
}

}  // namespace w4a4
