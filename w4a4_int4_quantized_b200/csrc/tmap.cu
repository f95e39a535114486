// Encoded TMA descriptors (CUtensorMap) for the kernels of libw4a4, cached
// by everything that goes into them: base pointer, element type, shape,
// row stride, box and swizzle.  A descriptor only describes an address
// range, so a cached one stays valid for any later buffer placed at the same
// address with the same shape; no ownership is implied.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include <utility>

#include "plan_cache.h"
#include "tmap.h"

namespace w4a4 {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  return fn;
}

struct TmapKey {
  int64_t v[12];
};

struct TmapVal {
  CUtensorMap map;
};

}  // namespace

bool make_tmap_nd(CUtensorMap* out, CUtensorMapDataType dt, int esize, const void* base, int rank,
                  const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz) {
  static PlanCache<TmapKey, TmapVal, 128> cache;
  if (rank < 1 || rank > 3) return false;
  TmapKey key;
  memset(&key, 0, sizeof key);
  key.v[0] = (int64_t)reinterpret_cast<uintptr_t>(base);
  key.v[1] = (int64_t)dt | ((int64_t)esize << 8) | ((int64_t)swz << 16) | ((int64_t)rank << 24);
  for (int d = 0; d < rank; ++d) {
    key.v[2 + d] = (int64_t)dims[d];
    key.v[5 + d] = (int64_t)box[d];
    if (d > 0) key.v[8 + d - 1] = (int64_t)strides_bytes[d - 1];
  }
  TmapVal val;
  const bool ok = cache.get(key, val, [&](TmapVal& v) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gd[3], gs[2];
    cuuint32_t bx[3], es[3] = {1, 1, 1};
    for (int d = 0; d < rank; ++d) {
      gd[d] = dims[d];
      bx[d] = box[d];
      if (d > 0) gs[d - 1] = strides_bytes[d - 1];
    }
    return fn(&v.map, dt, (cuuint32_t)rank, const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  });
  if (ok) *out = val.map;
  return ok;
}

bool make_tmap(CUtensorMap* out, CUtensorMapDataType dt, int esize, const void* base, uint64_t rows, uint64_t cols,
               uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * (uint64_t)esize};
  const uint32_t box[2] = {box_cols, box_rows};
  return make_tmap_nd(out, dt, esize, base, 2, dims, strides, box, swz);
}

unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static const std::pair<GetCurrent, GetId> fns = [] {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess)
      f1 = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess)
      f2 = nullptr;
    return std::make_pair(reinterpret_cast<GetCurrent>(f1), reinterpret_cast<GetId>(f2));
  }();
  if (!fns.first || !fns.second) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (fns.first(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (fns.second(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

cudaError_t symbol_address_cached(const void* symbol, void** out) {
  struct Key {
    int64_t v[2];
  };
  struct Val {
    void* p;
  };
  static PlanCache<Key, Val, 64> cache;
  unsigned long long ctx = current_context_id();
  Val v{nullptr};
  if (ctx != 0) {
    const Key key = {{(int64_t)ctx, (int64_t)reinterpret_cast<uintptr_t>(symbol)}};
    if (cache.find(key, v)) {
      *out = v.p;
      return cudaSuccess;
    }
  }
  // the lookup also makes the device's primary context current if the
  // calling thread had none yet; the id is taken again afterwards
  const cudaError_t e = cudaGetSymbolAddress(&v.p, symbol);
  if (e != cudaSuccess) return e;
  ctx = current_context_id();
  if (ctx != 0) cache.insert(Key{{(int64_t)ctx, (int64_t)reinterpret_cast<uintptr_t>(symbol)}}, v);
  *out = v.p;
  return cudaSuccess;
}

}  // namespace w4a4
