// Low-rank down-projection T = X L1 of the SVDQuant branch (A4).
//
// Method: "Krea 2 Turbo - SVDQuant" (sweettea.co), "What's included" -- a
// low-rank correction branch runs in parallel with the 4-bit matmul; reading:
// the branch takes the unrotated bf16 activations, T = X L1 accumulates in
// fp32 and is stored as bf16 for the up-projection folded into the GEMM.
//
// A thin product (N = rank <= 256), so the kernel splits K over a cluster of
// S CTAs (2 <= S <= 16, any size; above 8 a non-portable cluster size) to
// put enough SMs on the activations: each CTA streams a 128-row tile of X
// (K-major, 128-byte swizzle) and the matching rows of L1 (N-major, 128-byte
// swizzle) through a 4- to 8-deep TMA ring and accumulates its K
// slice with tcgen05.mma kind::f16 into TMEM.  The fp32 partials are drained
// into each CTA's shared memory and reduced through distributed shared memory
// in a fixed CTA order (deterministic, no global scratch); CTA c writes rows
// [c*128/S, (c+1)*128/S) of the tile of T.
#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "plan_cache.h"
#include "tmap.h"

namespace w4a4 {

namespace {

constexpr int BM = 128;        // rows of X per tile
constexpr int NSTMAX = 8;      // TMA stages (as many as fit: 4 to 8)
constexpr int kMaxSplit = 16;  // K split (cluster size): 16 needs the non-portable cluster size
constexpr int kThreads = 128;

struct LrBarriers {
  uint64_t full[NSTMAX];
  uint64_t empty[NSTMAX];
  uint64_t acc_full;
  uint32_t tmem_base;
};

struct LrParams {
  uint16_t* T;
  int M, K, r, S, nst;
  unsigned int* err;
  unsigned long long wait_ns;   // limit of the operand and free-slot waits
  int withhold;                 // self-test: the producer issues no operand load
};

// BKL: K per stage, 64 (one 128-byte swizzle atom of X per row) or 128 (two
// atoms side by side: each row's 256 bytes are requested together, which
// streams X faster where the ring still holds four stages, i.e. r <= 64).
// MAXS: the largest split S this instantiation reduces (8 or 16; the
// reduction loop is unrolled to it).
template <int MAXS, int BKL>
__global__ void __launch_bounds__(kThreads, 1)
    lowrank_down_kernel(const LrParams p, const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmL1) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const int rb = (p.r + 63) / 64;                       // 64-rank blocks of L1
  const int kAB = BM * BKL * 2;                         // X stage: BKL / 64 atoms of 16 KB
  const int kBB = rb * BKL * 128;                       // L1 stage: rb boxes of 64 K-rows x 128 bytes
  const int kStage = kAB + kBB;
  const int part_pitch = p.r * 4 + 16;                  // fp32 partial row pitch (padded)
  const int NST = p.nst;
  const int data = max(NST * kStage, BM * part_pitch);
  LrBarriers* bar = reinterpret_cast<LrBarriers*>(smem_raw + (sbase - raw) + data);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const int S = p.S;
  const int m0 = (blockIdx.x / S) * BM;
  const int nkb = p.K / BKL;
  const int kb0 = (int)crank * nkb / S;
  const int kb1 = ((int)crank + 1) * nkb / S;
  uint32_t ncols = 32;
  while ((int)ncols < p.r) ncols <<= 1;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmL1);
      for (int s = 0; s < NST; ++s) {
        mbar_init(&bar->full[s], 1);
        mbar_init(&bar->empty[s], 1);
      }
      mbar_init(&bar->acc_full, 1);
      fence_mbar_init();
    }
  } else if (warp == 2) {
    tmem_alloc(&bar->tmem_base, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  // X may come from the previous kernel of the stream, and the previous
  // layer may still read this T
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------- TMA
    // (self-test: with `withhold` set nothing is issued, so the MMA thread's
    // first operand wait runs out; no copy or MMA is then in flight)
    int s = 0;
    uint32_t ph = 0;
    for (int kb = kb0; kb < (p.withhold ? kb0 : kb1); ++kb) {
      if (!mbar_wait(&bar->empty[s], ph ^ 1u, p.wait_ns)) {
        set_device_error(p.err, kDevErrTimeoutEmpty);
        break;
      }
      const uint32_t st = sbase + (uint32_t)(s * kStage);
      mbar_arrive_expect_tx(&bar->full[s], (uint32_t)kStage);
      for (int a = 0; a < BKL / 64; ++a) tma_load_2d(st + a * (BM * 128), &tmX, kb * BKL + 64 * a, m0, &bar->full[s]);
      for (int b = 0; b < rb; ++b)
        tma_load_2d(st + kAB + b * (BKL * 128), &tmL1, b * 64, kb * BKL, &bar->full[s]);
      if (++s == NST) { s = 0; ph ^= 1u; }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------- MMA
    const uint32_t idesc = idesc_bf16(BM, p.r, false, true);
    int s = 0;
    uint32_t ph = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait(&bar->full[s], ph, p.wait_ns)) {
        set_device_error(p.err, kDevErrTimeoutFull);
        break;
      }
      tc_fence_after();
      const uint32_t st = sbase + (uint32_t)(s * kStage);
#pragma unroll
      for (int ks = 0; ks < BKL / 16; ++ks)
        mma_bf16_ss(tmem, smem_desc_kmajor_sw128(st + (uint32_t)((ks >> 2) * (BM * 128) + (ks & 3) * 32)),
                    smem_desc_mnmajor_sw128(st + (uint32_t)(kAB + ks * 2048), BKL * 128, 1024), idesc,
                    (kb > kb0 || ks > 0) ? 1u : 0u);
      tc_commit(&bar->empty[s]);
      if (++s == NST) { s = 0; ph ^= 1u; }
    }
    tc_commit(&bar->acc_full);
  }

  // --------------------------------------------- drain partials to smem
  __syncwarp();   // lanes 0 of warps 0 and 1 rejoin before the warp-wide TMEM loads
  // (always the full limit: the commit that completes this barrier must be
  // observed before the CTA exits, also after a shortened operand wait)
  if (!mbar_wait(&bar->acc_full, 0)) set_device_error(p.err, kDevErrTimeoutAcc);
  tc_fence_after();
  const int row = warp * 32 + lane;
  const uint32_t part = sbase + (uint32_t)(row * part_pitch);
  for (int c0 = 0; c0 < p.r; c0 += 32) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
    tmem_wait_ld();
    if (kb1 == kb0) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0u;   // an empty K slice contributes zero
    }
    const int nv = min(32, p.r - c0);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (4 * q < nv)
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(part + (uint32_t)((c0 + 4 * q) * 4)),
                     "r"(v[4 * q]), "r"(v[4 * q + 1]), "r"(v[4 * q + 2]), "r"(v[4 * q + 3])
                     : "memory");
  }
  tc_fence_before();
  cluster_sync();

  // --------------------------------------------- reduce across the cluster
  // All S remote loads of an item are issued before any is used (a load
  // from another CTA's shared memory takes hundreds of cycles); the sum then
  // runs in CTA order 0 .. S-1, so T does not depend on timing.
  const int row0 = (int)crank * BM / S, row1 = ((int)crank + 1) * BM / S;   // this CTA's rows of T
  const int vec_per_row = p.r / 4;
  for (int item = threadIdx.x; item < (row1 - row0) * vec_per_row; item += kThreads) {
    const int rr = row0 + item / vec_per_row;
    const int c = (item % vec_per_row) * 4;
    const uint32_t local = sbase + (uint32_t)(rr * part_pitch + c * 4);
    uint4 w[MAXS];
#pragma unroll
    for (int s = 0; s < MAXS; ++s)
      if (s < S) w[s] = ld_cluster_v4(map_to_rank(local, (uint32_t)s));
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < MAXS; ++s) {
      if (s < S) {
        acc[0] = __fadd_rn(acc[0], __uint_as_float(w[s].x));
        acc[1] = __fadd_rn(acc[1], __uint_as_float(w[s].y));
        acc[2] = __fadd_rn(acc[2], __uint_as_float(w[s].z));
        acc[3] = __fadd_rn(acc[3], __uint_as_float(w[s].w));
      }
    }
    const long m = (long)m0 + rr;
    if (m < p.M) {
      __nv_bfloat162 a = __floats2bfloat162_rn(acc[0], acc[1]);
      __nv_bfloat162 b = __floats2bfloat162_rn(acc[2], acc[3]);
      uint2 o = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
      *reinterpret_cast<uint2*>(p.T + m * p.r + c) = o;
    }
  }
  cluster_sync();   // partials stay readable until every CTA has reduced
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

}  // namespace

unsigned int* device_error_word();

namespace {
// the instantiation for a split S (clusters above 8 need the 16-wide
// reduction) and a stage width of 128 (wide) or 64
using LrKernel = void (*)(const LrParams, const CUtensorMap, const CUtensorMap);
LrKernel kernel_for(int S, bool wide) {
  if (wide) return S > 8 ? lowrank_down_kernel<kMaxSplit, 128> : lowrank_down_kernel<8, 128>;
  return S > 8 ? lowrank_down_kernel<kMaxSplit, 64> : lowrank_down_kernel<8, 64>;
}
}  // namespace

cudaError_t launch_lowrank_down_ex(const uint16_t* X, const uint16_t* L1, int M, int K, int r, uint16_t* T,
                                   unsigned long long wait_ns, int withhold, cudaStream_t st) {
  unsigned int* err = device_error_word();
  if (!err) return cudaErrorInvalidDevicePointer;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if ((e = device_sm_count(dev, &sms)) != cudaSuccess) return e;
  const int m_tiles = (M + BM - 1) / BM;
  // 128-wide K stages where K allows and the ring keeps four of them
  const bool wide = K % 128 == 0 && r <= 64;
  const int BKL = wide ? 128 : 64;
  const int nkb = K / BKL;
  const int rb = (r + 63) / 64;
  const int stage = BM * BKL * 2 + rb * BKL * 128;
  // as deep a ring as fits beside the barriers (X streams from HBM once)
  const int nst = std::max(4, std::min(NSTMAX, (232448 - 2048) / stage));
  const int data = std::max(nst * stage, BM * (r * 4 + 16));
  const int smem = data + (int)sizeof(LrBarriers) + 1024;
  static DeviceFlags attr_set;
  if (!attr_set.done(dev)) {
    for (auto k : {lowrank_down_kernel<8, 64>, lowrank_down_kernel<kMaxSplit, 64>, lowrank_down_kernel<8, 128>,
                   lowrank_down_kernel<kMaxSplit, 128>}) {
      if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448)) != cudaSuccess ||
          (e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess)
        return e;
    }
    attr_set.set(dev);
  }
  // K split S (cluster size): the largest S <= 16 for which every cluster of
  // the grid is resident at once.  Clusters must fit inside one GPC, so the
  // count that fits is below sms / S for the larger S; a grid past it runs a
  // second wave and doubles the time.
  struct SKey {
    int64_t v[4];
  };
  static PlanCache<SKey, int, 32> split_cache;
  SKey key = {{dev, m_tiles, nkb, smem + ((int64_t)wide << 32)}};
  int S = 1;
  const bool ok = split_cache.get(key, S, [&](int& out) {
    out = 1;
    for (int sc = std::min(kMaxSplit, nkb); sc >= 2 && out == 1; --sc) {
      if (m_tiles * sc > sms) continue;
      cudaLaunchConfig_t qc = {};
      qc.gridDim = dim3(m_tiles * sc, 1, 1);
      qc.blockDim = dim3(kThreads, 1, 1);
      qc.dynamicSmemBytes = smem;
      cudaLaunchAttribute qa;
      qa.id = cudaLaunchAttributeClusterDimension;
      qa.val.clusterDim.x = sc;
      qa.val.clusterDim.y = 1;
      qa.val.clusterDim.z = 1;
      qc.attrs = &qa;
      qc.numAttrs = 1;
      int max_clusters = 0;
      if ((e = cudaOccupancyMaxActiveClusters(&max_clusters, kernel_for(sc, wide), &qc)) != cudaSuccess)
        return false;
      if (m_tiles <= max_clusters) out = sc;
    }
    return true;
  });
  if (!ok) return e;
  CUtensorMap tX, tL1;
  if (!make_tmap(&tX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, (uint64_t)M, (uint64_t)K, 64, BM,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&tL1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L1, (uint64_t)K, (uint64_t)r, 64, BKL,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(m_tiles * S, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  LrParams prm{T, M, K, r, S, nst, err, wait_ns, withhold};
  e = cudaLaunchKernelEx(&cfg, kernel_for(S, wide), prm, tX, tL1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_lowrank_down(const uint16_t* X, const uint16_t* L1, int M, int K, int r, uint16_t* T,
                                cudaStream_t st) {
  return launch_lowrank_down_ex(X, L1, M, K, r, T, kWaitTimeoutNs, 0, st);
}

}  // namespace w4a4
