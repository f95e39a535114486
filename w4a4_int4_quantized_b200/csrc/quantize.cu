// Rotate + absmax + quantize + pack (K1, activations) and the same routine on
// weights (K4).
//
// Method: "Load Diffusion Model INT4 (W4A4)" (comfy.icu), intro -- a Hadamard
// rotation (ConvRot) is applied before 4-bit quantization; "W4A4 and W4A8: The
// New Quantization Toolkit" (renderbob.io), "Decoding the notation" --
// activations are quantized on the fly, weights once.  Readings: unnormalised
// Sylvester H per group of g along K, fp32 butterflies in the order h = 1, 2,
// 4, ... (bit-identical to a pairwise tree sum over the explicit matrix),
// s = fl32(amax / qmax) per row, q = rint_even(fl32(y / s)) with IEEE division.
//
// Design (sm_100a, HBM-bound): one thread owns one whole rotation group of a
// row (64 or 128 elements held as float2 pairs (y_i, y_{i+g/2})), so the
// transform needs no shuffles: g/2 - 1 stages run on packed f32x2 adds, the
// last stage on scalar adds.  The row absmax meets in shared memory.  Codes
// come from a bracketed reciprocal: rint(y * inv_lo) == rint(y * inv_hi)
// (each a single fused multiply-add onto 1.5 * 2^23) proves that the IEEE
// quotient rounds to the same integer; otherwise the thread redoes its group
// with exact division.  Each thread writes its codes as 16-byte stores.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace w4a4 {

namespace {

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Nibbles of eight rounded values (bits of v + 1.5*2^23, integer in the low
// mantissa bits) packed into one word: value j in bits 4j..4j+3.
__device__ __forceinline__ uint32_t pack_nibbles8(const uint32_t (&t)[8]) {
  uint32_t a = __byte_perm(t[0], t[2], 0x5410);
  uint32_t b = __byte_perm(t[1], t[3], 0x5410);
  uint32_t c = (a & 0x000F000Fu) | ((b << 4) & 0x00F000F0u);
  uint32_t d = __byte_perm(t[4], t[6], 0x5410);
  uint32_t e = __byte_perm(t[5], t[7], 0x5410);
  uint32_t f = (d & 0x000F000Fu) | ((e << 4) & 0x00F000F0u);
  return __byte_perm(c, f, 0x6420);
}

// Low bytes of four rounded values packed into one word.
__device__ __forceinline__ uint32_t pack_bytes4(uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3) {
  return __byte_perm(__byte_perm(t0, t1, 0x0040), __byte_perm(t2, t3, 0x0040), 0x5410);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int kStages = 3;

// Shared-memory stride of one staged group: g bf16 plus 16 bytes of padding,
// so that the 16-byte reads of eight consecutive threads (eight consecutive
// groups) fall in eight different bank groups.
template <int G>
constexpr int group_stride() { return G * 2 + 16; }

// Persistent CTAs walk blocks of R consecutive rows.  Blocks are staged in a
// 3-deep shared-memory ring with cp.async (coalesced 16-byte copies, no
// registers held while in flight), so the loads of the next blocks overlap
// the rotation and quantization of the current one.
template <int G, bool ROT, int QMAX>
__global__ void __launch_bounds__(256) rotate_quantize_kernel(const uint16_t* __restrict__ X, int M, int K,
                                                              int rows_per_blk, uint8_t* __restrict__ out,
                                                              float* __restrict__ scale) {
  constexpr int HALF = G / 2;
  constexpr bool INT4 = (QMAX == 7);
  constexpr int GS = group_stride<G>();
  extern __shared__ __align__(16) uint8_t stage_mem[];
  __shared__ unsigned int rowmax[2][256];

  const int gpr = K / G;
  const int tid = threadIdx.x;
  const int lr = tid / gpr;
  const int grp = tid - lr * gpr;
  const int groups_per_blk = rows_per_blk * gpr;
  const int stage_bytes = groups_per_blk * GS;
  const int nblk = (M + rows_per_blk - 1) / rows_per_blk;
  const uint32_t stage0 = smem_u32(stage_mem);
  constexpr int CPG = G / 8;  // 16-byte chunks per group

  auto issue = [&](int it) {
    const int blk = blockIdx.x + it * gridDim.x;
    if (blk < nblk) {
      const long row0 = (long)blk * rows_per_blk;
      const int rows = min(rows_per_blk, (int)(M - row0));
      const int nchunks = rows * gpr * CPG;
      const uint8_t* src = reinterpret_cast<const uint8_t*>(X + row0 * K);
      const uint32_t dst = stage0 + (uint32_t)((it % kStages) * stage_bytes);
      for (int c = tid; c < nchunks; c += blockDim.x)
        cp_async16(dst + (uint32_t)((c / CPG) * GS + (c % CPG) * 16), src + (long)c * 16);
    }
    cp_async_commit();
  };

  if (tid < 256) rowmax[0][tid] = 0u;
#pragma unroll
  for (int it = 0; it < kStages - 1; ++it) issue(it);

  for (int it = 0;; ++it) {
    const int blk = blockIdx.x + it * gridDim.x;
    if (blk >= nblk) break;
    cp_async_wait<kStages - 2>();
    __syncthreads();
    issue(it + kStages - 1);
    if (tid < rows_per_blk) rowmax[(it + 1) & 1][tid] = 0u;
    unsigned int* rmax = rowmax[it & 1];

    const long row = (long)blk * rows_per_blk + lr;
    const bool active = (lr < rows_per_blk) && (row < M);
    float2 P[HALF];  // P[i] = (y_i, y_{i+HALF})
    if (active) {
      const uint32_t gsrc = stage0 + (uint32_t)((it % kStages) * stage_bytes + tid * GS);
      uint32_t w[G / 2];
#pragma unroll
      for (int i = 0; i < G / 8; ++i) {
        uint4 t;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(t.x), "=r"(t.y), "=r"(t.z), "=r"(t.w)
                     : "r"(gsrc + i * 16));
        w[4 * i + 0] = t.x;
        w[4 * i + 1] = t.y;
        w[4 * i + 2] = t.z;
        w[4 * i + 3] = t.w;
      }
#pragma unroll
      for (int i = 0; i < HALF; ++i) {
        const uint32_t a = w[i / 2], b = w[(i + HALF) / 2];
        P[i].x = (i & 1) ? bf16hi(a) : bf16lo(a);
        P[i].y = (i & 1) ? bf16hi(b) : bf16lo(b);
      }
      if (ROT) {
        // stages h = 1 .. HALF/2: pairs (i, i+h) sit in different float2s
#pragma unroll
        for (int h = 1; h < HALF; h <<= 1) {
#pragma unroll
          for (int i = 0; i < HALF; ++i) {
            if ((i & h) == 0) {
              const float2 a = P[i], b = P[i + h];
              P[i] = __fadd2_rn(a, b);
              P[i + h] = __fadd2_rn(a, make_float2(-b.x, -b.y));
            }
          }
        }
        // last stage h = HALF: the two halves of each float2
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
          const float a = P[i].x, b = P[i].y;
          P[i].x = __fadd_rn(a, b);
          P[i].y = __fsub_rn(a, b);
        }
      }
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < HALF; ++i) amax = fmaxf(amax, fmaxf(fabsf(P[i].x), fabsf(P[i].y)));
      atomicMax(&rmax[lr], __float_as_uint(amax));
    }
    __syncthreads();
    if (!active) continue;

    const float amax = __uint_as_float(rmax[lr]);
    const float s = __fdiv_rn(amax, (float)QMAX);
    if (grp == 0) scale[row] = s;
    float inv_hi = 0.0f, inv_lo = 0.0f;
    if (s != 0.0f) {
      const float inv = __frcp_rn(s);
      inv_hi = __fmul_rn(inv, 1.0f + 0x1p-20f);
      inv_lo = __fmul_rn(inv, 1.0f - 0x1p-20f);
    }
    const float2 ih = make_float2(inv_hi, inv_hi), il = make_float2(inv_lo, inv_lo);
    const float2 mg = make_float2(kMagic, kMagic);

    constexpr int NW = INT4 ? G / 8 : G / 4;  // output words
    uint32_t outw[NW];
    uint32_t bad = 0u;
#pragma unroll
    for (int blk8 = 0; blk8 < HALF / 8; ++blk8) {
      uint32_t tx[8], ty[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float2 th = __ffma2_rn(P[8 * blk8 + j], ih, mg);
        const float2 tl = __ffma2_rn(P[8 * blk8 + j], il, mg);
        tx[j] = __float_as_uint(th.x);
        ty[j] = __float_as_uint(th.y);
        bad |= (tx[j] ^ __float_as_uint(tl.x)) | (ty[j] ^ __float_as_uint(tl.y));
      }
      if (INT4) {
        outw[blk8] = pack_nibbles8(tx);
        outw[HALF / 8 + blk8] = pack_nibbles8(ty);
      } else {
        outw[2 * blk8] = pack_bytes4(tx[0], tx[1], tx[2], tx[3]);
        outw[2 * blk8 + 1] = pack_bytes4(tx[4], tx[5], tx[6], tx[7]);
        outw[HALF / 4 + 2 * blk8] = pack_bytes4(ty[0], ty[1], ty[2], ty[3]);
        outw[HALF / 4 + 2 * blk8 + 1] = pack_bytes4(ty[4], ty[5], ty[6], ty[7]);
      }
    }
    if (bad) {
      // A quotient sits within 2^-20 (relative) of a rounding boundary: redo
      // this group with the IEEE quotient the codes are defined by.
#pragma unroll
      for (int blk8 = 0; blk8 < HALF / 8; ++blk8) {
        uint32_t tx[8], ty[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          tx[j] = __float_as_uint(__fadd_rn(rintf(__fdiv_rn(P[8 * blk8 + j].x, s)), kMagic));
          ty[j] = __float_as_uint(__fadd_rn(rintf(__fdiv_rn(P[8 * blk8 + j].y, s)), kMagic));
        }
        if (INT4) {
          outw[blk8] = pack_nibbles8(tx);
          outw[HALF / 8 + blk8] = pack_nibbles8(ty);
        } else {
          outw[2 * blk8] = pack_bytes4(tx[0], tx[1], tx[2], tx[3]);
          outw[2 * blk8 + 1] = pack_bytes4(tx[4], tx[5], tx[6], tx[7]);
          outw[HALF / 4 + 2 * blk8] = pack_bytes4(ty[0], ty[1], ty[2], ty[3]);
          outw[HALF / 4 + 2 * blk8 + 1] = pack_bytes4(ty[4], ty[5], ty[6], ty[7]);
        }
      }
    }
    const long row_bytes = INT4 ? K / 2 : K;
    uint4* dst = reinterpret_cast<uint4*>(out + row * row_bytes + (long)grp * (INT4 ? G / 2 : G));
#pragma unroll
    for (int i = 0; i < NW / 4; ++i)
      dst[i] = make_uint4(outw[4 * i], outw[4 * i + 1], outw[4 * i + 2], outw[4 * i + 3]);
  }
  cp_async_wait<0>();
}

template <int G, bool ROT, int QMAX>
cudaError_t launch_rq(const uint16_t* X, int M, int K, uint8_t* out, float* scale, cudaStream_t st) {
  const int gpr = K / G;
  const int rows_per_blk = gpr >= 128 ? 1 : 128 / gpr;
  const int threads = ((rows_per_blk * gpr + 31) / 32) * 32;
  const int smem = kStages * rows_per_blk * gpr * group_stride<G>();
  auto kern = rotate_quantize_kernel<G, ROT, QMAX>;
  static int attr_set[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int sms = 148, per_sm = 1;
  if (dev < 64 && attr_set[dev] != smem) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem > 48 * 1024 ? smem : 48 * 1024);
    if (e != cudaSuccess) return e;
    attr_set[dev] = smem;
  }
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem)) != cudaSuccess) return e;
  const int nblk = (M + rows_per_blk - 1) / rows_per_blk;
  const int grid = min(nblk, sms * max(per_sm, 1));
  kern<<<grid, threads, smem, st>>>(X, M, K, rows_per_blk, out, scale);
  return cudaGetLastError();
}

}  // namespace

// Rows of X [rows, K] bf16 -> codes (packed nibbles [rows, K/2] when qmax == 7,
// int8 [rows, K] when qmax == 127) and one fp32 scale per row.  group 0 turns
// the rotation off.  Shapes are validated by the caller.
cudaError_t launch_rotate_quantize(const uint16_t* X, int rows, int K, int group, int qmax, uint8_t* out,
                                   float* scale, cudaStream_t st) {
  if (qmax == 7) {
    if (group == 64) return launch_rq<64, true, 7>(X, rows, K, out, scale, st);
    if (group == 128) return launch_rq<128, true, 7>(X, rows, K, out, scale, st);
    return launch_rq<128, false, 7>(X, rows, K, out, scale, st);
  }
  if (group == 64) return launch_rq<64, true, 127>(X, rows, K, out, scale, st);
  if (group == 128) return launch_rq<128, true, 127>(X, rows, K, out, scale, st);
  return launch_rq<128, false, 127>(X, rows, K, out, scale, st);
}

}  // namespace w4a4
