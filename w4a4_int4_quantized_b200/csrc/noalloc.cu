// w4a4_linear_noalloc: the whole W4A4 layer without any device allocation.
//
// w4a4_linear needs scratch memory (the packed activation codes, their
// scales and the low-rank activations) and takes it from the caller.  Some
// callers cannot provide it: a host program that has handed all device
// memory to its own fixed pool, or a plugin running inside a runtime that
// forbids cudaMalloc after start-up.  For them this entry point uses a
// fixed scratch buffer that lives in the library itself (a file-scope
// __device__ array, present on every GPU that loads the library until the
// process exits) and otherwise runs exactly the w4a4_linear path.
#include <atomic>
#include <cstdint>

#include "plan_cache.h"
#include "w4a4.h"

namespace w4a4 {
namespace {

constexpr size_t kScratchBytes = W4A4_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch size");

// The scratch itself.  Host code must not use this name as an address: the
// device address comes from cudaGetSymbolAddress below.
__device__ __align__(256) uint8_t g_linear_scratch[kScratchBytes];

// Device address of the scratch in the current context, looked up with
// cudaGetSymbolAddress (with that device current) the first time a context
// asks and cached per context, so a context recreated after cudaDeviceReset
// looks the address up again.
w4a4_status scratch_for_current_device(uint8_t** out) {
  void* addr = nullptr;
  if (symbol_address_cached(reinterpret_cast<const void*>(&g_linear_scratch), &addr) != cudaSuccess ||
      addr == nullptr) {
    cudaGetLastError();
    return W4A4_ERR_CUDA;
  }
  *out = static_cast<uint8_t*>(addr);
  return W4A4_OK;
}

}  // namespace
}  // namespace w4a4

extern "C" w4a4_status w4a4_linear_noalloc(const void* X, const uint8_t* Wq, const float* w_scale, int M, int N,
                                           int K, int group, const void* L1, const void* L2, int rank,
                                           const void* bias, void* Y, w4a4_stream_t stream) {
  if (!X || !Wq || !w_scale || !Y) return W4A4_ERR_INVALID_ARG;
  const size_t need = w4a4_workspace_bytes(M, K, rank);
  if (need == 0) return W4A4_ERR_UNSUPPORTED_SHAPE;
  if (need > w4a4::kScratchBytes) return W4A4_ERR_WORKSPACE;  // layer too large for the built-in scratch
  uint8_t* scratch = nullptr;
  const w4a4_status s = w4a4::scratch_for_current_device(&scratch);
  if (s != W4A4_OK) return s;
  // Every part of the scratch the layer reads is written first in the same
  // call (codes, scales, low-rank activations), so nothing is cleared.
  return w4a4_linear(X, Wq, w_scale, M, N, K, group, L1, L2, rank, bias, Y, scratch, w4a4::kScratchBytes, stream);
}
