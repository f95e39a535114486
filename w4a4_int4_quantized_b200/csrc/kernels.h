// Internal launchers of libw4a4 (not part of the public C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace w4a4 {

// qmax 7: symmetric INT4 (packed); 127: symmetric INT8; 15: asymmetric 4-bit
// with a zero point per row (packed unsigned codes; `zero` [rows], else null).
cudaError_t launch_rotate_quantize(const uint16_t* X, int rows, int K, int group, int qmax, uint8_t* out,
                                   float* scale, uint8_t* zero, cudaStream_t st);

// Host-only planning of the rotate + quantize launch shape (no CUDA call):
// out = {rows per block, threads, dynamic shared memory, grid}.
bool plan_rotate_quantize_shape(int M, int K, int group, int sms, int resident_per_sm, bool cached, int out[4]);

// The GEMM's split-K decision without a CUDA call (the launcher feeds it the
// occupancy query): *split = 4, 2 or 1 (the persistent form), given how many
// clusters of 8 and of 4 CTAs fit on the device at once.
bool plan_gemm_split(int M, int N, int K, int rank, int sms, int clusters_of_8, int clusters_of_4, int* split);

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
  const uint8_t* w_zero;   // W4A8: zero point per weight row [N] (codes 0..15), else null
  int act;                 // W4A4: 0 none, 1 GELU (tanh approximation) applied before the bf16 store
};

// kW4A4: packed INT4 x packed INT4 (optional low-rank); kW8A8: int8 x int8;
// kW4A8: int8 activations x packed unsigned 4-bit weights with zero points.
enum class GemmMode { kW8A8 = 0, kW4A4 = 1, kW4A8 = 2 };

cudaError_t launch_gemm(const GemmArgs& a, GemmMode mode, cudaStream_t st);

// T[M, r] (bf16) = X[M, K] (bf16) x L1[K, r] (bf16), fp32 accumulation.
cudaError_t launch_lowrank_down(const uint16_t* X, const uint16_t* L1, int M, int K, int r, uint16_t* T,
                                cudaStream_t st);

// The same with an explicit limit for every bounded wait and, for the
// wait-timeout self-test, a producer that withholds every operand load (the
// consumer's first wait then runs out after wait_ns; T is left undefined).
cudaError_t launch_lowrank_down_ex(const uint16_t* X, const uint16_t* L1, int M, int K, int r, uint16_t* T,
                                   unsigned long long wait_ns, int withhold, cudaStream_t st);

// Symmetric INT4 codes of rotated rows with stochastic rounding: q =
// clamp(floor(y / s + u), -8, 7), u from Philox4x64-10 keyed by `seed`.
cudaError_t launch_rotate_quantize_sr(const uint16_t* X, int rows, int K, int group, uint8_t* out, float* scale,
                                      unsigned long long seed, cudaStream_t st);

// Wb [N, K] = bf16(W + scale * (A B)^T), fp32 FMA sums in index order.
cudaError_t launch_lora_bake(const uint16_t* W, const uint16_t* A, const uint16_t* B, int N, int K, int rl,
                             float scale, uint16_t* Wb, cudaStream_t st);

// [L1 | A] and [L2 ; bf16(fl32(scale * B))] (rank r + rl low-rank operands).
cudaError_t launch_lora_merge(const uint16_t* L1, const uint16_t* L2, int r, const uint16_t* A, const uint16_t* B,
                              int rl, float scale, int K, int N, uint16_t* L1o, uint16_t* L2o, cudaStream_t st);

}  // namespace w4a4
