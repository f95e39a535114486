// INT4 x INT4 (and INT8 x INT8) GEMM with the fused dequant + low-rank + bias
// epilogue (K2 / K3), hand-written for sm_100a tensor cores.
//
// Method: "Load Diffusion Model INT4 (W4A4)" (comfy.icu), intro -- the matmuls
// of the rotated, 4-bit layers run on tensor cores at 4-bit speed; "Krea 2
// Turbo - SVDQuant" (sweettea.co), "What's included" -- a low-rank branch
// (X L1) L2 is added to the quantized product; "ComfyUI-INT4-Fast"
// (kongchang.com), "Per-Layer Dynamic Routing" -- sensitive layers take the
// INT8 path.  Epilogue reading: y = ((acc * s_a) * s_w) / g + T L2 + b.
//
// sm_100 has no 4-bit integer MMA kind, so codes are widened to 8 bit and fed
// to tcgen05.mma kind::i8 (int32 accumulation in tensor memory).  Widening a
// packed word w (codes q0..q7, q0 in the low nibble) is three ALU operations:
//   (w << 4) & 0xF0F0F0F0  -> bytes 16*q0, 16*q2, 16*q4, 16*q6
//    w       & 0xF0F0F0F0  -> bytes 16*q1, 16*q3, 16*q5, 16*q7
// Both operands are widened the same way, so the K order inside each 8-code
// word is permuted identically on both sides (the dot product is unchanged)
// and every product carries a factor 256, removed exactly by an arithmetic
// shift of the int32 accumulator (|acc| <= 64 K << 2^23 for K <= 32768).
//
// CTA tile 128 x 256, k-block 128 codes, one CTA per SM:
//   warps 0-3   A producers: load packed rows (256-bit loads, two k-blocks of
//               register prefetch), widen, tcgen05.st into a TMEM ring
//               (A is read by the MMA from tensor memory, not shared memory);
//   warps 4-11  B producers: same for the 256 weight rows, written into a
//               shared-memory ring in the 128-byte-swizzled K-major layout;
//   warp 12     one elected thread issues tcgen05.mma and commits stages;
//   warps 0-7   epilogue: tcgen05.ld of the int32 accumulator, dequant,
//               low-rank add, bias, bf16 store (and the optional int32 copy).
// Every mbarrier wait is bounded; on timeout the kernel records an error in
// the device error word and exits without trapping.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace w4a4 {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;                 // 8-bit elements per k-block
constexpr int kStages = 6;
constexpr int kNumAWarps = 4;
constexpr int kNumBWarps = 8;
constexpr int kMmaWarp = kNumAWarps + kNumBWarps;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr int kBStageBytes = BN * BK;   // 32 KB of widened codes
constexpr uint32_t kAccCol = 0;         // int32 accumulator: columns [0, 256)
constexpr uint32_t kACol0 = 256;        // A ring: 32 columns (128 codes) per stage
constexpr uint32_t kTmemCols = 512;
constexpr int kSmemBytes = kStages * kBStageBytes + 1024 /*alignment slack*/ + 256 /*barriers*/;

static_assert(kACol0 + kStages * (BK / 4) <= kTmemCols, "TMEM budget");

struct Params {
  GemmArgs a;
  unsigned int* err;
};

__device__ __forceinline__ void ld_nc_256(const void* p, uint4& lo, uint4& hi) {
  asm volatile("ld.global.nc.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
               : "l"(p));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// 16 packed bytes (32 codes) -> 32 widened bytes (two 16-byte chunks).
__device__ __forceinline__ void widen16(const uint4 p, uint4& c0, uint4& c1) {
  c0.x = (p.x << 4) & 0xF0F0F0F0u;
  c0.y = p.x & 0xF0F0F0F0u;
  c0.z = (p.y << 4) & 0xF0F0F0F0u;
  c0.w = p.y & 0xF0F0F0F0u;
  c1.x = (p.z << 4) & 0xF0F0F0F0u;
  c1.y = p.z & 0xF0F0F0F0u;
  c1.z = (p.w << 4) & 0xF0F0F0F0u;
  c1.w = p.w & 0xF0F0F0F0u;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

template <bool PACKED>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const Params prm) {
  const GemmArgs& p = prm.a;
  constexpr int V = PACKED ? 4 : 8;               // 16-byte vectors per row per k-block
  constexpr int kShift = PACKED ? 8 : 0;          // widened products carry 2^8
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kBStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int m0 = blockIdx.y * BM;
  const int nk = p.K / BK;
  const long row_bytes = PACKED ? p.K / 2 : p.K;

  if (warp == kMmaWarp) {
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&full[s], (kNumAWarps + kNumBWarps) * 32);
        mbar_init(&empty[s], 1);
      }
      mbar_init(acc_full, 1);
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < kMmaWarp) {
    // ------------------------------------------------------------ producers
    const bool is_a = warp < kNumAWarps;
    const int r = is_a ? warp * 32 + lane : (warp - kNumAWarps) * 32 + lane;
    const long g_row = is_a ? (long)m0 + r : (long)n0 + r;
    const bool ok = g_row < (is_a ? p.M : p.N);
    const uint8_t* src = (is_a ? p.A : p.B) + (ok ? g_row : 0) * row_bytes;
    const uint32_t a_taddr = tmem + ((uint32_t)(warp * 32) << 16) + kACol0;
    const uint32_t b_row = sbase + (uint32_t)((r >> 3) * 1024 + (r & 7) * 128);
    const uint32_t sw = (uint32_t)(r & 7);

    auto load = [&](uint4 (&buf)[V], int kb) {
      if (ok && kb < nk) {
        const uint8_t* q = src + (long)kb * (V * 16);
#pragma unroll
        for (int v = 0; v < V; v += 2) ld_nc_256(q + v * 16, buf[v], buf[v + 1]);
      } else {
#pragma unroll
        for (int v = 0; v < V; ++v) buf[v] = make_uint4(0u, 0u, 0u, 0u);
      }
    };
    auto produce = [&](int kb, const uint4 (&cur)[V]) -> bool {
      const int s = kb % kStages;
      const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
      if (!mbar_wait(&empty[s], ph ^ 1u)) {
        set_device_error(prm.err, kDevErrTimeoutEmpty);
        return false;
      }
      tc_fence_after();
      if (is_a) {
        uint32_t regs[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 c0, c1;
          if (PACKED) {
            widen16(cur[c], c0, c1);
          } else {
            c0 = cur[2 * c];
            c1 = cur[2 * c + 1];
          }
          regs[8 * c + 0] = c0.x; regs[8 * c + 1] = c0.y; regs[8 * c + 2] = c0.z; regs[8 * c + 3] = c0.w;
          regs[8 * c + 4] = c1.x; regs[8 * c + 5] = c1.y; regs[8 * c + 6] = c1.z; regs[8 * c + 7] = c1.w;
        }
        tmem_st_32x32b_x32(a_taddr + (uint32_t)(s * (BK / 4)), regs);
        tmem_wait_st();
        tc_fence_before();
      } else {
        const uint32_t row = b_row + (uint32_t)(s * kBStageBytes);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 c0, c1;
          if (PACKED) {
            widen16(cur[c], c0, c1);
          } else {
            c0 = cur[2 * c];
            c1 = cur[2 * c + 1];
          }
          st_shared_v4(row + (((uint32_t)(2 * c) ^ sw) << 4), c0);
          st_shared_v4(row + (((uint32_t)(2 * c + 1) ^ sw) << 4), c1);
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(&full[s]);
      return true;
    };

    uint4 b0[V], b1[V], b2[V];
    load(b0, 0);
    load(b1, 1);
    for (int kb = 0; kb < nk; kb += 3) {
      load(b2, kb + 2);
      if (!produce(kb, b0)) break;
      if (kb + 1 >= nk) break;
      load(b0, kb + 3);
      if (!produce(kb + 1, b1)) break;
      if (kb + 2 >= nk) break;
      load(b1, kb + 4);
      if (!produce(kb + 2, b2)) break;
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_i8(BM, BN);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kStages;
      const uint32_t ph = (uint32_t)(kb / kStages) & 1u;
      if (!mbar_wait(&full[s], ph)) {
        set_device_error(prm.err, kDevErrTimeoutFull);
        break;
      }
      tc_fence_after();
      const uint32_t b_stage = sbase + (uint32_t)(s * kBStageBytes);
#pragma unroll
      for (int ks = 0; ks < BK / 32; ++ks) {
        const uint64_t bdesc = smem_desc_kmajor_sw128(b_stage + (uint32_t)(ks * 32));
        mma_i8_ts(tmem + kAccCol, tmem + kACol0 + (uint32_t)(s * (BK / 4) + ks * 8), bdesc, idesc,
                  (kb | ks) != 0 ? 1u : 0u);
      }
      tc_commit(&empty[s]);
    }
    tc_commit(acc_full);
    if (!mbar_wait(acc_full, 0)) set_device_error(prm.err, kDevErrTimeoutDrain);
  }

  // ------------------------------------------------------------ epilogue
  if (warp < 8) {
    const int quad = warp & 3;
    const int half = warp >> 2;
    if (!mbar_wait(acc_full, 0)) set_device_error(prm.err, kDevErrTimeoutAcc);
    tc_fence_after();
    const long m = (long)m0 + quad * 32 + lane;
    const bool mok = m < p.M;
    const float sa = mok ? __ldg(p.a_scale + m) : 0.0f;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      const int c0 = half * 128 + ch * 32;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(quad * 32) << 16) + kAccCol + (uint32_t)c0, v);
      tmem_wait_ld();
      const int n = n0 + c0;
      const int nv = min(32, p.N - n);
      if (nv <= 0 || !mok) continue;
      float y[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int acc = static_cast<int>(v[j]) >> kShift;
        v[j] = static_cast<uint32_t>(acc);
        const float sw = j < nv ? __ldg(p.b_scale + n + j) : 0.0f;
        y[j] = __fmul_rn(__fmul_rn(__fmul_rn(__int2float_rn(acc), sa), sw), p.inv_group);
      }
      if (p.rank > 0) {
        const uint16_t* trow = p.T + m * p.rank;
#pragma unroll 1
        for (int jj = 0; jj < p.rank; ++jj) {
          const float t = bf16_bits_to_float(trow[jj]);
          const uint16_t* l2 = p.L2 + (long)jj * p.N + n;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nv) y[j] = __fmaf_rn(t, bf16_bits_to_float(__ldg(l2 + j)), y[j]);
        }
      }
      if (p.bias) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nv) y[j] = __fadd_rn(y[j], bf16_bits_to_float(__ldg(p.bias + n + j)));
      }
      uint32_t o[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * j], y[2 * j + 1]);
        o[j] = *reinterpret_cast<uint32_t*>(&h);
      }
      uint4* dst = reinterpret_cast<uint4*>(p.Y + m * p.N + n);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (8 * c < nv) dst[c] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
      if (p.acc_debug) {
        uint4* dd = reinterpret_cast<uint4*>(p.acc_debug + m * p.N + n);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (4 * c < nv) dd[c] = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <bool PACKED>
cudaError_t launch_impl(const GemmArgs& a, unsigned int* err, cudaStream_t st) {
  static int configured[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !configured[dev]) {
    e = cudaFuncSetAttribute(gemm_kernel<PACKED>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  dim3 grid((a.N + BN - 1) / BN, (a.M + BM - 1) / BM);
  Params prm{a, err};
  gemm_kernel<PACKED><<<grid, kThreads, kSmemBytes, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace

unsigned int* device_error_word();

cudaError_t launch_gemm(const GemmArgs& a, bool packed_int4, cudaStream_t st) {
  unsigned int* err = device_error_word();
  if (!err) return cudaErrorInvalidDevicePointer;
  return packed_int4 ? launch_impl<true>(a, err, st) : launch_impl<false>(a, err, st);
}

}  // namespace w4a4
