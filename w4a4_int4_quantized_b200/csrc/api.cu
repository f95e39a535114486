// C ABI of libw4a4: host-side validation and launches.  Declarations and the
// contract of every entry point are in include/w4a4.h.
#include <atomic>
#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "plan_cache.h"
#include "w4a4.h"

namespace w4a4 {

// Per-device error word written by kernels whose bounded waits give up.
__device__ unsigned int g_device_error_word = 0u;

namespace {

constexpr int kMaxDevices = 64;
std::atomic<int> g_dev_ok[kMaxDevices];  // 0 unknown, 1 sm_100, 2 other

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

w4a4_status check_k_group(int K, int group) {
  if (group != 0 && group != 64 && group != 128) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if (K < 128 || K % 128 != 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  const int g = (group == 64) ? 64 : 128;
  if (K / g > 256) return W4A4_ERR_UNSUPPORTED_SHAPE;
  return W4A4_OK;
}

w4a4_status check_rank(int rank) {
  if (rank < 0 || rank > 256 || rank % 16 != 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  return W4A4_OK;
}

w4a4_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return W4A4_ERR_UNSUPPORTED_DEVICE;
  int state = g_dev_ok[dev].load(std::memory_order_relaxed);
  if (state == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      cudaGetLastError();
      return W4A4_ERR_CUDA;
    }
    state = (major == 10 && minor == 0) ? 1 : 2;
    g_dev_ok[dev].store(state, std::memory_order_relaxed);
  }
  return state == 1 ? W4A4_OK : W4A4_ERR_UNSUPPORTED_DEVICE;
}

w4a4_status cuda_status(cudaError_t e) { return e == cudaSuccess ? W4A4_OK : W4A4_ERR_CUDA; }

size_t round256(size_t x) { return (x + 255u) & ~size_t(255u); }

}  // namespace

unsigned int* device_error_word() {
  void* addr = nullptr;
  if (symbol_address_cached(reinterpret_cast<const void*>(&g_device_error_word), &addr) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return static_cast<unsigned int*>(addr);
}

}  // namespace w4a4

using namespace w4a4;

static_assert(kDevErrTimeoutFull == W4A4_DEVERR_WAIT_OPERANDS && kDevErrTimeoutEmpty == W4A4_DEVERR_WAIT_SLOT &&
                  kDevErrTimeoutAcc == W4A4_DEVERR_WAIT_ACCUM && kDevErrTimeoutDrain == W4A4_DEVERR_WAIT_DRAIN,
              "device error bits of the public header");

extern "C" {

int w4a4_version(void) { return 100; }

const char* w4a4_status_string(w4a4_status s) {
  switch (s) {
    case W4A4_OK: return "W4A4_OK";
    case W4A4_ERR_INVALID_ARG: return "W4A4_ERR_INVALID_ARG";
    case W4A4_ERR_UNSUPPORTED_SHAPE: return "W4A4_ERR_UNSUPPORTED_SHAPE";
    case W4A4_ERR_MISALIGNED: return "W4A4_ERR_MISALIGNED";
    case W4A4_ERR_CUDA: return "W4A4_ERR_CUDA";
    case W4A4_ERR_DEVICE_TIMEOUT: return "W4A4_ERR_DEVICE_TIMEOUT";
    case W4A4_ERR_UNSUPPORTED_DEVICE: return "W4A4_ERR_UNSUPPORTED_DEVICE";
    case W4A4_ERR_WORKSPACE: return "W4A4_ERR_WORKSPACE";
  }
  return "W4A4_ERR_UNKNOWN";
}

// ------------------------------------------------------------------ quantizers
static w4a4_status quantize_rows(const void* X, int rows, int K, int group, void* out, float* scale, int qmax,
                                 uint8_t* zero, w4a4_stream_t stream) {
  if (!X || !out || !scale || (qmax == 15 && !zero)) return W4A4_ERR_INVALID_ARG;
  if (rows < 1) return W4A4_ERR_UNSUPPORTED_SHAPE;
  w4a4_status s = check_k_group(K, group);
  if (s != W4A4_OK) return s;
  if (!aligned16(X) || !aligned16(out) || !aligned16(scale)) return W4A4_ERR_MISALIGNED;
  if ((s = check_device()) != W4A4_OK) return s;
  return cuda_status(launch_rotate_quantize(static_cast<const uint16_t*>(X), rows, K, group, qmax,
                                            static_cast<uint8_t*>(out), scale, zero,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

w4a4_status w4a4_quantize_weights(const void* W, int N, int K, int group, uint8_t* Wq, float* w_scale,
                                  w4a4_stream_t stream) {
  return quantize_rows(W, N, K, group, Wq, w_scale, 7, nullptr, stream);
}

w4a4_status w8a8_quantize_weights(const void* W, int N, int K, int group, int8_t* Wq, float* w_scale,
                                  w4a4_stream_t stream) {
  return quantize_rows(W, N, K, group, Wq, w_scale, 127, nullptr, stream);
}

w4a4_status w4a8_quantize_weights(const void* W, int N, int K, int group, uint8_t* Wq, float* w_scale,
                                  uint8_t* w_zero, w4a4_stream_t stream) {
  return quantize_rows(W, N, K, group, Wq, w_scale, 15, w_zero, stream);
}

w4a4_status w8a8_rotate_quantize_act(const void* X, int M, int K, int group, int8_t* Xq, float* x_scale,
                                     w4a4_stream_t stream) {
  return quantize_rows(X, M, K, group, Xq, x_scale, 127, nullptr, stream);
}

w4a4_status w4a4_rotate_quantize_act(const void* X, int M, int K, int group, uint8_t* Xq, float* x_scale,
                                     const void* L1, int rank, void* T, w4a4_stream_t stream) {
  if (!X || !Xq || !x_scale) return W4A4_ERR_INVALID_ARG;
  w4a4_status s = check_rank(rank);
  if (s != W4A4_OK) return s;
  if (rank > 0) {
    if (!L1 || !T) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(L1) || !aligned16(T)) return W4A4_ERR_MISALIGNED;
  }
  if (M < 1) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if ((s = check_k_group(K, group)) != W4A4_OK) return s;
  if (!aligned16(X) || !aligned16(Xq) || !aligned16(x_scale)) return W4A4_ERR_MISALIGNED;
  if ((s = check_device()) != W4A4_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_rotate_quantize(static_cast<const uint16_t*>(X), M, K, group, 7, Xq, x_scale, nullptr, st);
  if (e != cudaSuccess) return W4A4_ERR_CUDA;
  if (rank > 0) {
    e = launch_lowrank_down(static_cast<const uint16_t*>(X), static_cast<const uint16_t*>(L1), M, K, rank,
                            static_cast<uint16_t*>(T), st);
    if (e != cudaSuccess) return W4A4_ERR_CUDA;
  }
  return W4A4_OK;
}

// ------------------------------------------------------------------ GEMMs
static w4a4_status gemm_common(const void* Xq, const float* x_scale, const void* Wq, const float* w_scale,
                               const uint8_t* w_zero, int M, int N, int K, int group, const void* T, const void* L2,
                               int rank, const void* bias, void* Y, int32_t* acc_debug, GemmMode mode,
                               w4a4_stream_t stream, int act = 0) {
  if (!Xq || !x_scale || !Wq || !w_scale || !Y) return W4A4_ERR_INVALID_ARG;
  if (mode == GemmMode::kW4A8 && !w_zero) return W4A4_ERR_INVALID_ARG;
  w4a4_status s = check_rank(rank);
  if (s != W4A4_OK) return s;
  if (rank > 0) {
    if (!T || !L2) return W4A4_ERR_INVALID_ARG;
    if (!aligned16(T) || !aligned16(L2)) return W4A4_ERR_MISALIGNED;
  }
  if (M < 1 || N < 8 || N % 8 != 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if ((s = check_k_group(K, group)) != W4A4_OK) return s;
  // the GEMM reads code rows with 32-byte vector loads
  if (!aligned32(Xq) || !aligned16(x_scale) || !aligned32(Wq) || !aligned16(w_scale) || !aligned16(Y) ||
      (bias && !aligned16(bias)) || (acc_debug && !aligned16(acc_debug)))
    return W4A4_ERR_MISALIGNED;
  if ((s = check_device()) != W4A4_OK) return s;
  GemmArgs a;
  a.A = static_cast<const uint8_t*>(Xq);
  a.a_scale = x_scale;
  a.B = static_cast<const uint8_t*>(Wq);
  a.b_scale = w_scale;
  a.M = M;
  a.N = N;
  a.K = K;
  a.inv_group = group > 0 ? 1.0f / (float)group : 1.0f;  // exact: group is a power of two
  a.T = static_cast<const uint16_t*>(T);
  a.L2 = static_cast<const uint16_t*>(L2);
  a.rank = rank;
  a.bias = static_cast<const uint16_t*>(bias);
  a.Y = static_cast<uint16_t*>(Y);
  a.acc_debug = acc_debug;
  a.w_zero = w_zero;
  a.act = act;
  return cuda_status(launch_gemm(a, mode, reinterpret_cast<cudaStream_t>(stream)));
}

w4a4_status w4a4_gemm(const uint8_t* Xq, const float* x_scale, const uint8_t* Wq, const float* w_scale, int M,
                      int N, int K, int group, const void* T, const void* L2, int rank, const void* bias, void* Y,
                      int32_t* acc_debug, w4a4_stream_t stream) {
  return gemm_common(Xq, x_scale, Wq, w_scale, nullptr, M, N, K, group, T, L2, rank, bias, Y, acc_debug,
                     GemmMode::kW4A4, stream);
}

w4a4_status w4a4_gemm_gelu(const uint8_t* Xq, const float* x_scale, const uint8_t* Wq, const float* w_scale,
                           int M, int N, int K, int group, const void* T, const void* L2, int rank, const void* bias,
                           void* Y, int32_t* acc_debug, w4a4_stream_t stream) {
  return gemm_common(Xq, x_scale, Wq, w_scale, nullptr, M, N, K, group, T, L2, rank, bias, Y, acc_debug,
                     GemmMode::kW4A4, stream, 1);
}

w4a4_status w8a8_gemm(const int8_t* Xq, const float* x_scale, const int8_t* Wq, const float* w_scale, int M,
                      int N, int K, int group, const void* bias, void* Y, int32_t* acc_debug,
                      w4a4_stream_t stream) {
  return gemm_common(Xq, x_scale, Wq, w_scale, nullptr, M, N, K, group, nullptr, nullptr, 0, bias, Y, acc_debug,
                     GemmMode::kW8A8, stream);
}

w4a4_status w4a8_gemm(const int8_t* Xq, const float* x_scale, const uint8_t* Wq, const float* w_scale,
                      const uint8_t* w_zero, int M, int N, int K, int group, const void* bias, void* Y,
                      int32_t* acc_debug, w4a4_stream_t stream) {
  return gemm_common(Xq, x_scale, Wq, w_scale, w_zero, M, N, K, group, nullptr, nullptr, 0, bias, Y, acc_debug,
                     GemmMode::kW4A8, stream);
}

// ------------------------------------------------------------------ whole layer
size_t w4a4_workspace_bytes(int M, int K, int rank) {
  if (M < 1 || K < 2 || rank < 0) return 0;
  return round256((size_t)M * (size_t)(K / 2)) + round256((size_t)M * 4u) + round256((size_t)M * rank * 2u);
}

size_t w8a8_workspace_bytes(int M, int K) {
  if (M < 1 || K < 1) return 0;
  return round256((size_t)M * (size_t)K) + round256((size_t)M * 4u);
}

size_t w4a8_workspace_bytes(int M, int K) { return w8a8_workspace_bytes(M, K); }

w4a4_status w4a4_linear(const void* X, const uint8_t* Wq, const float* w_scale, int M, int N, int K, int group,
                        const void* L1, const void* L2, int rank, const void* bias, void* Y, void* workspace,
                        size_t workspace_bytes, w4a4_stream_t stream) {
  if (!X || !Wq || !w_scale || !Y) return W4A4_ERR_INVALID_ARG;
  w4a4_status s = check_rank(rank);
  if (s != W4A4_OK) return s;
  if (rank > 0 && (!L1 || !L2)) return W4A4_ERR_INVALID_ARG;
  if (M < 1 || N < 8 || N % 8 != 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if ((s = check_k_group(K, group)) != W4A4_OK) return s;
  const size_t need = w4a4_workspace_bytes(M, K, rank);
  if (!workspace || workspace_bytes < need || !aligned256(workspace)) return W4A4_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* Xq = ws;
  float* xs = reinterpret_cast<float*>(ws + round256((size_t)M * (size_t)(K / 2)));
  void* T = rank > 0 ? static_cast<void*>(ws + round256((size_t)M * (size_t)(K / 2)) + round256((size_t)M * 4u))
                     : nullptr;
  s = w4a4_rotate_quantize_act(X, M, K, group, Xq, xs, L1, rank, T, stream);
  if (s != W4A4_OK) return s;
  return w4a4_gemm(Xq, xs, Wq, w_scale, M, N, K, group, T, L2, rank, bias, Y, nullptr, stream);
}

w4a4_status w4a4_linear_gelu(const void* X, const uint8_t* Wq, const float* w_scale, int M, int N, int K,
                             int group, const void* L1, const void* L2, int rank, const void* bias, void* Y,
                             void* workspace, size_t workspace_bytes, w4a4_stream_t stream) {
  if (!X || !Wq || !w_scale || !Y) return W4A4_ERR_INVALID_ARG;
  w4a4_status s = check_rank(rank);
  if (s != W4A4_OK) return s;
  if (rank > 0 && (!L1 || !L2)) return W4A4_ERR_INVALID_ARG;
  if (M < 1 || N < 8 || N % 8 != 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if ((s = check_k_group(K, group)) != W4A4_OK) return s;
  const size_t need = w4a4_workspace_bytes(M, K, rank);
  if (!workspace || workspace_bytes < need || !aligned256(workspace)) return W4A4_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* Xq = ws;
  float* xs = reinterpret_cast<float*>(ws + round256((size_t)M * (size_t)(K / 2)));
  void* T = rank > 0 ? static_cast<void*>(ws + round256((size_t)M * (size_t)(K / 2)) + round256((size_t)M * 4u))
                     : nullptr;
  s = w4a4_rotate_quantize_act(X, M, K, group, Xq, xs, L1, rank, T, stream);
  if (s != W4A4_OK) return s;
  return w4a4_gemm_gelu(Xq, xs, Wq, w_scale, M, N, K, group, T, L2, rank, bias, Y, nullptr, stream);
}

size_t w4a4_mlp_workspace_bytes(int M, int D, int H, int rank_up, int rank_down) {
  if (M < 1 || D < 2 || H < 2 || rank_up < 0 || rank_down < 0) return 0;
  return round256(w4a4_workspace_bytes(M, D, rank_up)) + round256((size_t)M * (size_t)H * 2u) +
         round256(w4a4_workspace_bytes(M, H, rank_down));
}

w4a4_status w4a4_mlp(const void* X, int M, int D, int H, int group, const uint8_t* Wq_up, const float* w_scale_up,
                     const void* L1_up, const void* L2_up, int rank_up, const void* bias_up, const uint8_t* Wq_down,
                     const float* w_scale_down, const void* L1_down, const void* L2_down, int rank_down,
                     const void* bias_down, void* Y, void* workspace, size_t workspace_bytes,
                     w4a4_stream_t stream) {
  if (!X || !Wq_up || !w_scale_up || !Wq_down || !w_scale_down || !Y) return W4A4_ERR_INVALID_ARG;
  const size_t need = w4a4_mlp_workspace_bytes(M, D, H, rank_up, rank_down);
  if (need == 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || workspace_bytes < need || !aligned256(workspace)) return W4A4_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t up_bytes = round256(w4a4_workspace_bytes(M, D, rank_up));
  void* h = ws + up_bytes;
  uint8_t* ws_down = ws + up_bytes + round256((size_t)M * (size_t)H * 2u);
  w4a4_status s = w4a4_linear_gelu(X, Wq_up, w_scale_up, M, H, D, group, L1_up, L2_up, rank_up, bias_up, h, ws,
                                   up_bytes, stream);
  if (s != W4A4_OK) return s;
  return w4a4_linear(h, Wq_down, w_scale_down, M, D, H, group, L1_down, L2_down, rank_down, bias_down, Y, ws_down,
                     round256(w4a4_workspace_bytes(M, H, rank_down)), stream);
}

w4a4_status w8a8_linear(const void* X, const int8_t* Wq, const float* w_scale, int M, int N, int K, int group,
                        const void* bias, void* Y, void* workspace, size_t workspace_bytes,
                        w4a4_stream_t stream) {
  if (!X || !Wq || !w_scale || !Y) return W4A4_ERR_INVALID_ARG;
  if (M < 1 || N < 8 || N % 8 != 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  w4a4_status s = check_k_group(K, group);
  if (s != W4A4_OK) return s;
  const size_t need = w8a8_workspace_bytes(M, K);
  if (!workspace || workspace_bytes < need || !aligned256(workspace)) return W4A4_ERR_WORKSPACE;
  int8_t* Xq = static_cast<int8_t*>(workspace);
  float* xs = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + round256((size_t)M * (size_t)K));
  s = w8a8_rotate_quantize_act(X, M, K, group, Xq, xs, stream);
  if (s != W4A4_OK) return s;
  return w8a8_gemm(Xq, xs, Wq, w_scale, M, N, K, group, bias, Y, nullptr, stream);
}

w4a4_status w4a8_linear(const void* X, const uint8_t* Wq, const float* w_scale, const uint8_t* w_zero, int M,
                        int N, int K, int group, const void* bias, void* Y, void* workspace, size_t workspace_bytes,
                        w4a4_stream_t stream) {
  if (!X || !Wq || !w_scale || !w_zero || !Y) return W4A4_ERR_INVALID_ARG;
  if (M < 1 || N < 8 || N % 8 != 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  w4a4_status s = check_k_group(K, group);
  if (s != W4A4_OK) return s;
  const size_t need = w4a8_workspace_bytes(M, K);
  if (!workspace || workspace_bytes < need || !aligned256(workspace)) return W4A4_ERR_WORKSPACE;
  int8_t* Xq = static_cast<int8_t*>(workspace);
  float* xs = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + round256((size_t)M * (size_t)K));
  s = w8a8_rotate_quantize_act(X, M, K, group, Xq, xs, stream);
  if (s != W4A4_OK) return s;
  return w4a8_gemm(Xq, xs, Wq, w_scale, w_zero, M, N, K, group, bias, Y, nullptr, stream);
}

// ------------------------------------------------------------------ runtime LoRA
w4a4_status w4a4_lora_merge(const void* L1, const void* L2, int rank, const void* A, const void* B, int lora_rank,
                            float lora_scale, int K, int N, void* L1_out, void* L2_out, w4a4_stream_t stream) {
  if (!A || !B || !L1_out || !L2_out) return W4A4_ERR_INVALID_ARG;
  if (rank > 0 && (!L1 || !L2)) return W4A4_ERR_INVALID_ARG;
  if (rank < 0 || rank % 16 != 0 || lora_rank < 16 || lora_rank % 16 != 0 || rank + lora_rank > 256)
    return W4A4_ERR_UNSUPPORTED_SHAPE;
  if (K < 1 || N < 8 || N % 8 != 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if ((rank > 0 && (!aligned16(L1) || !aligned16(L2))) || !aligned16(A) || !aligned16(B) || !aligned16(L1_out) ||
      !aligned16(L2_out))
    return W4A4_ERR_MISALIGNED;
  w4a4_status s = check_device();
  if (s != W4A4_OK) return s;
  return cuda_status(launch_lora_merge(static_cast<const uint16_t*>(L1), static_cast<const uint16_t*>(L2), rank,
                                       static_cast<const uint16_t*>(A), static_cast<const uint16_t*>(B), lora_rank,
                                       lora_scale, K, N, static_cast<uint16_t*>(L1_out),
                                       static_cast<uint16_t*>(L2_out), reinterpret_cast<cudaStream_t>(stream)));
}

w4a4_status w4a4_bake_lora_sr(const void* W, const void* A, const void* B, int lora_rank, float lora_scale, int N,
                              int K, int group, unsigned long long seed, void* W_baked, uint8_t* Wq, float* w_scale,
                              w4a4_stream_t stream) {
  if (!W || !A || !B || !W_baked || !Wq || !w_scale) return W4A4_ERR_INVALID_ARG;
  if (lora_rank < 1 || lora_rank > 256 || N < 1) return W4A4_ERR_UNSUPPORTED_SHAPE;
  w4a4_status s = check_k_group(K, group);
  if (s != W4A4_OK) return s;
  if (!aligned16(W) || !aligned16(A) || !aligned16(B) || !aligned16(W_baked) || !aligned16(Wq) ||
      !aligned16(w_scale))
    return W4A4_ERR_MISALIGNED;
  if ((s = check_device()) != W4A4_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_lora_bake(static_cast<const uint16_t*>(W), static_cast<const uint16_t*>(A),
                                   static_cast<const uint16_t*>(B), N, K, lora_rank, lora_scale,
                                   static_cast<uint16_t*>(W_baked), st);
  if (e != cudaSuccess) return W4A4_ERR_CUDA;
  return cuda_status(launch_rotate_quantize_sr(static_cast<const uint16_t*>(W_baked), N, K, group, Wq, w_scale,
                                               seed, st));
}

// ------------------------------------------------------------------ planning
w4a4_status w4a4_plan_rotate_quantize(int M, int K, int group, int sms, int resident_per_sm, int cached,
                                      int* shape) {
  if (!shape) return W4A4_ERR_INVALID_ARG;
  if (M < 1 || sms < 1 || resident_per_sm < 1) return W4A4_ERR_UNSUPPORTED_SHAPE;
  const w4a4_status s = check_k_group(K, group);
  if (s != W4A4_OK) return s;
  return plan_rotate_quantize_shape(M, K, group, sms, resident_per_sm, cached != 0, shape) ? W4A4_OK
                                                                                           : W4A4_ERR_UNSUPPORTED_SHAPE;
}

w4a4_status w4a4_plan_gemm_split(int M, int N, int K, int rank, int sms, int clusters_of_8, int clusters_of_4,
                                  int* split) {
  if (!split) return W4A4_ERR_INVALID_ARG;
  if (M < 1 || N < 8 || N % 8 != 0 || sms < 2 || clusters_of_8 < 0 || clusters_of_4 < 0)
    return W4A4_ERR_UNSUPPORTED_SHAPE;
  w4a4_status s = check_rank(rank);
  if (s != W4A4_OK) return s;
  if ((s = check_k_group(K, 128)) != W4A4_OK) return s;
  return plan_gemm_split(M, N, K, rank, sms, clusters_of_8, clusters_of_4, split) ? W4A4_OK
                                                                                  : W4A4_ERR_UNSUPPORTED_SHAPE;
}

// ------------------------------------------------------------------ failures
w4a4_status w4a4_selftest_wait_timeout(const void* X, const void* L1, int M, int K, int rank, void* T,
                                       unsigned int timeout_us, w4a4_stream_t stream) {
  if (!X || !L1 || !T) return W4A4_ERR_INVALID_ARG;
  if (timeout_us < 1 || timeout_us > 1000000) return W4A4_ERR_INVALID_ARG;
  w4a4_status s = check_rank(rank);
  if (s != W4A4_OK) return s;
  if (rank == 0 || M < 1) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if ((s = check_k_group(K, 128)) != W4A4_OK) return s;
  if (!aligned16(X) || !aligned16(L1) || !aligned16(T)) return W4A4_ERR_MISALIGNED;
  if ((s = check_device()) != W4A4_OK) return s;
  return cuda_status(launch_lowrank_down_ex(static_cast<const uint16_t*>(X), static_cast<const uint16_t*>(L1), M, K,
                                            rank, static_cast<uint16_t*>(T), 1000ull * timeout_us, 1,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

w4a4_status w4a4_get_device_error(w4a4_stream_t stream, unsigned int* code) {
  w4a4_status s = check_device();
  if (s != W4A4_OK) return s;
  unsigned int* p = device_error_word();
  if (!p) return W4A4_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int host = 0;
  if (cudaMemcpyAsync(&host, p, sizeof host, cudaMemcpyDeviceToHost, st) != cudaSuccess) return W4A4_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return W4A4_ERR_CUDA;
  if (host != 0u) {
    if (cudaMemsetAsync(p, 0, sizeof(unsigned int), st) != cudaSuccess) return W4A4_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return W4A4_ERR_CUDA;
  }
  if (code) *code = host;
  return host ? W4A4_ERR_DEVICE_TIMEOUT : W4A4_OK;
}

}  // extern "C"
