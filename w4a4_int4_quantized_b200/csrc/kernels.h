// Internal launchers of libw4a4 (not part of the public C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace w4a4 {

cudaError_t launch_rotate_quantize(const uint16_t* X, int rows, int K, int group, int qmax, uint8_t* out,
                                   float* scale, cudaStream_t st);

struct GemmArgs {
  const uint8_t* A;        // activation codes [M, K/2] packed or [M, K] int8
  const float* a_scale;    // [M]
  const uint8_t* B;        // weight codes [N, K/2] packed or [N, K] int8
  const float* b_scale;    // [N]
  int M, N, K;
  float inv_group;         // 1/g (exact power of two), 1 when the rotation is off
  const uint16_t* T;       // low-rank activations [M, r] bf16, or null
  const uint16_t* L2;      // low-rank up-projection [r, N] bf16, or null
  int rank;
  const uint16_t* bias;    // [N] bf16 or null
  uint16_t* Y;             // [M, N] bf16
  int32_t* acc_debug;      // [M, N] int32 or null
};

cudaError_t launch_gemm(const GemmArgs& a, bool packed_int4, cudaStream_t st);

// T[M, r] (bf16) = X[M, K] (bf16) x L1[K, r] (bf16), fp32 accumulation.
cudaError_t launch_lowrank_down(const uint16_t* X, const uint16_t* L1, int M, int K, int r, uint16_t* T,
                                cudaStream_t st);

}  // namespace w4a4
