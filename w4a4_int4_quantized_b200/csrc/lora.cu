// Runtime LoRA merged into the low-rank branch.
//
// "ComfyUI-INT4-Fast" (kongchang.com), "INT4 Quantized Inference Comes to
// ComfyUI": LoRAs apply on top of the 4-bit layers; "Krea 2 Turbo - SVDQuant"
// (sweettea.co), "What's included": the low-rank branch runs beside the
// 4-bit product.  A LoRA (A [K, rl], B [rl, N], scale s) is placed beside the
// SVDQuant pair (L1 [K, r], L2 [r, N]) as one branch of rank r + rl:
//   L1o = [L1 | A],  L2o = [L2 ; bf16(fl32(s * B))],
// so the GEMM's single epilogue low-rank MMA covers both.  Elementwise and
// memory-bound: 16-byte copies for the concatenation, one fp32 multiply and
// one round-to-nearest-even narrowing per scaled element.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace w4a4 {

namespace {

__global__ void lora_merge_kernel(const uint16_t* __restrict__ L1, const uint16_t* __restrict__ L2, int r,
                                  const uint16_t* __restrict__ A, const uint16_t* __restrict__ B, int rl,
                                  float scale, int K, int N, uint16_t* __restrict__ L1o,
                                  uint16_t* __restrict__ L2o) {
  const int rt = r + rl;
  const long n1 = (long)K * (rt / 8);          // 8-element chunks of L1o (r, rl multiples of 16)
  const long n2 = (long)rt * (N / 8);          // 8-element chunks of L2o (N multiple of 8)
  const long stride = (long)gridDim.x * blockDim.x;
  for (long c = (long)blockIdx.x * blockDim.x + threadIdx.x; c < n1 + n2; c += stride) {
    if (c < n1) {
      const long k = c / (rt / 8);
      const int j = (int)(c - k * (rt / 8)) * 8;
      const uint4 v = j < r ? *reinterpret_cast<const uint4*>(L1 + k * r + j)
                            : *reinterpret_cast<const uint4*>(A + k * rl + (j - r));
      *reinterpret_cast<uint4*>(L1o + k * rt + j) = v;
    } else {
      const long c2 = c - n1;
      const long j = c2 / (N / 8);
      const int n = (int)(c2 - j * (N / 8)) * 8;
      uint4 v;
      if (j < r) {
        v = *reinterpret_cast<const uint4*>(L2 + j * N + n);
      } else {
        const uint4 b = *reinterpret_cast<const uint4*>(B + (j - r) * N + n);
        const uint32_t w[4] = {b.x, b.y, b.z, b.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float lo = __fmul_rn(scale, __uint_as_float(w[q] << 16));
          const float hi = __fmul_rn(scale, __uint_as_float(w[q] & 0xFFFF0000u));
          __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
          o[q] = *reinterpret_cast<uint32_t*>(&h);
        }
        v = make_uint4(o[0], o[1], o[2], o[3]);
      }
      *reinterpret_cast<uint4*>(L2o + j * N + n) = v;
    }
  }
}

// Wb[n][k] = bf16(fl32(W[n][k] + fl32(scale * sum_j A[k][j] B[j][n]))), the
// sum as fp32 fused multiply-adds in index order (the reading of baking a
// LoRA into the weights before they are re-quantized).  A CTA computes a
// 64 (n) x 64 (k) tile; A and B are staged through shared memory in chunks
// of 32 ranks taken in order, so every output's FMA chain still runs
// j = 0, 1, 2, ... and the result is bit-exact.  Each thread owns 4 x 4
// outputs (k fastest, for coalesced stores).
constexpr int kBakeTile = 64;
constexpr int kBakeChunk = 32;

__global__ void __launch_bounds__(256) lora_bake_kernel(const uint16_t* __restrict__ W,
                                                        const uint16_t* __restrict__ A,
                                                        const uint16_t* __restrict__ B, int N, int K, int rl,
                                                        float scale, uint16_t* __restrict__ Wb) {
  __shared__ float As[kBakeChunk][kBakeTile + 1];   // [j][k]
  __shared__ float Bs[kBakeChunk][kBakeTile + 1];   // [j][n]
  const int k0 = blockIdx.x * kBakeTile, n0 = blockIdx.y * kBakeTile;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int j0 = 0; j0 < rl; j0 += kBakeChunk) {
    for (int t = threadIdx.x; t < kBakeChunk * kBakeTile; t += blockDim.x) {
      const int jj = t % kBakeChunk, kk = t / kBakeChunk;          // A[k][j]: j fastest in memory
      const int k = k0 + kk, j = j0 + jj;
      As[jj][kk] = (k < K && j < rl) ? __uint_as_float((uint32_t)A[(long)k * rl + j] << 16) : 0.0f;
      const int nn = t % kBakeTile, jb = t / kBakeTile;            // B[j][n]: n fastest in memory
      const int n = n0 + nn, j2 = j0 + jb;
      Bs[jb][nn] = (n < N && j2 < rl) ? __uint_as_float((uint32_t)B[(long)j2 * N + n] << 16) : 0.0f;
    }
    __syncthreads();
    const int jn = min(kBakeChunk, rl - j0);
    for (int jj = 0; jj < jn; ++jj) {
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = As[jj][tx * 4 + q];
        b[q] = Bs[jj][ty * 4 + q];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][q] = __fmaf_rn(a[q], b[i], acc[i][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = n0 + ty * 4 + i;
    if (n >= N) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = k0 + tx * 4 + q;
      if (k >= K) continue;
      const float w = __uint_as_float((uint32_t)W[(long)n * K + k] << 16);
      const __nv_bfloat16 h = __float2bfloat16_rn(__fadd_rn(w, __fmul_rn(scale, acc[i][q])));
      Wb[(long)n * K + k] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

}  // namespace

cudaError_t launch_lora_bake(const uint16_t* W, const uint16_t* A, const uint16_t* B, int N, int K, int rl,
                             float scale, uint16_t* Wb, cudaStream_t st) {
  const dim3 grid((unsigned)((K + kBakeTile - 1) / kBakeTile), (unsigned)((N + kBakeTile - 1) / kBakeTile));
  lora_bake_kernel<<<grid, 256, 0, st>>>(W, A, B, N, K, rl, scale, Wb);
  return cudaGetLastError();
}

cudaError_t launch_lora_merge(const uint16_t* L1, const uint16_t* L2, int r, const uint16_t* A, const uint16_t* B,
                              int rl, float scale, int K, int N, uint16_t* L1o, uint16_t* L2o, cudaStream_t st) {
  const long chunks = (long)K * ((r + rl) / 8) + (long)(r + rl) * (N / 8);
  const int threads = 256;
  const long blocks = (chunks + threads - 1) / threads;
  const int grid = (int)(blocks < 148L * 16 ? blocks : 148L * 16);
  lora_merge_kernel<<<grid > 0 ? grid : 1, threads, 0, st>>>(L1, L2, r, A, B, rl, scale, K, N, L1o, L2o);
  return cudaGetLastError();
}

}  // namespace w4a4
