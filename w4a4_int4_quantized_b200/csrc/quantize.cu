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

#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "plan_cache.h"
#include "tmap.h"

namespace w4a4 {

unsigned int* device_error_word();

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

constexpr int kStages = 2;  // stages (blocks of rows) per CTA, both requested up front

struct RqShape {
  int rows_per_blk, threads, smem, grid;
};

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Codes of 16 elements (8 float2 pairs) -> bw: INT4 {.x word, .y word}
// (value j of a word in bits 4j..4j+3), INT8 {.x lo, .x hi, .y lo, .y hi}.
// The fast form brackets each quotient between two fused multiply-adds and
// ORs any disagreement into `bad`; the exact form uses IEEE division.
template <bool INT4, bool EXACT, bool ASYM = false>
__device__ __forceinline__ void quantize_block8(const float2* P8, float2 ih, float2 il, float s, uint32_t* bw,
                                                uint32_t& bad, int zoff = 0) {
  const float2 mg = make_float2(kMagic, kMagic);
  uint32_t tx[8], ty[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (EXACT) {
      tx[j] = __float_as_uint(__fadd_rn(rintf(__fdiv_rn(P8[j].x, s)), kMagic));
      ty[j] = __float_as_uint(__fadd_rn(rintf(__fdiv_rn(P8[j].y, s)), kMagic));
    } else {
      const float2 th = __ffma2_rn(P8[j], ih, mg);
      const float2 tl = __ffma2_rn(P8[j], il, mg);
      tx[j] = __float_as_uint(th.x);
      ty[j] = __float_as_uint(th.y);
      bad |= (tx[j] ^ __float_as_uint(tl.x)) | (ty[j] ^ __float_as_uint(tl.y));
    }
  }
  if (ASYM) {
    // unsigned codes clamp(rint + z, 0, 15); zoff = z - bits(1.5 * 2^23)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      tx[j] = (uint32_t)min(max((int)tx[j] + zoff, 0), 15);
      ty[j] = (uint32_t)min(max((int)ty[j] + zoff, 0), 15);
    }
  }
  if (INT4) {
    bw[0] = pack_nibbles8(tx);
    bw[1] = pack_nibbles8(ty);
  } else {
    bw[0] = pack_bytes4(tx[0], tx[1], tx[2], tx[3]);
    bw[1] = pack_bytes4(tx[4], tx[5], tx[6], tx[7]);
    bw[2] = pack_bytes4(ty[0], ty[1], ty[2], ty[3]);
    bw[3] = pack_bytes4(ty[4], ty[5], ty[6], ty[7]);
  }
}

// Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC 2011): 10 rounds of two 64 x 64 -> 128-bit products
// on a 4-word counter with a Weyl-sequence key schedule.
__device__ __forceinline__ void philox4x64_10(uint64_t c[4], uint64_t k0, uint64_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t m0 = 0xD2E7470EE14C6C93ull, m1 = 0xCA5A826395121157ull;
    const uint64_t hi0 = __umul64hi(m0, c[0]), lo0 = m0 * c[0];
    const uint64_t hi1 = __umul64hi(m1, c[2]), lo1 = m1 * c[2];
    const uint64_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0;
    c[1] = lo1;
    c[2] = n2;
    c[3] = lo0;
    k0 += 0x9E3779B97F4A7C15ull;
    k1 += 0xBB67AE8584CAA73Bull;
  }
}

// u in [0, 1) of elements e0 .. e0 + 7 (e0 a multiple of 4): element e takes
// word e % 4 of Philox(counter = (e / 4, 0, 0, 0), key = (seed, 0)), top 24 bits.
__device__ __forceinline__ void sr_uniform8(uint64_t e0, uint64_t seed, float (&u)[8]) {
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    uint64_t c[4] = {(e0 >> 2) + (uint64_t)b, 0ull, 0ull, 0ull};
    philox4x64_10(c, seed, 0ull);
#pragma unroll
    for (int l = 0; l < 4; ++l) u[4 * b + l] = (float)(uint32_t)(c[l] >> 40) * 0x1p-24f;
  }
}

// Stochastic rounding of 16 elements (8 float2 pairs; .x lanes are elements
// ex0 .. ex0 + 7, .y lanes ey0 .. ey0 + 7 of the row-major array) to INT4
// codes q = clamp(floor(fl32(fl32(y / s) + u)), -8, 7), packed as in the
// round-to-nearest form.
__device__ __forceinline__ void quantize_block8_sr(const float2* P8, float s, uint64_t ex0, uint64_t ey0,
                                                   uint64_t seed, uint32_t* bw) {
  float ux[8], uy[8];
  sr_uniform8(ex0, seed, ux);
  sr_uniform8(ey0, seed, uy);
  uint32_t tx[8], ty[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    int qx = 0, qy = 0;
    if (s != 0.0f) {
      qx = min(max(__float2int_rd(__fadd_rn(__fdiv_rn(P8[j].x, s), ux[j])), -8), 7);
      qy = min(max(__float2int_rd(__fadd_rn(__fdiv_rn(P8[j].y, s), uy[j])), -8), 7);
    }
    tx[j] = (uint32_t)qx;   // pack_nibbles8 keeps the low nibble
    ty[j] = (uint32_t)qy;
  }
  bw[0] = pack_nibbles8(tx);
  bw[1] = pack_nibbles8(ty);
}

// Order-preserving unsigned key of a float (for shared-memory atomic min/max).
__device__ __forceinline__ uint32_t fkey(float v) {
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float fkey_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Persistent CTAs walk blocks of R consecutive rows.  Each block arrives in
// a shared-memory stage by TMA: X viewed as [rows * K/g groups][g/64 halves]
// [64 elements], one box per half covering the block's R * K/g groups, with
// the 128-byte swizzle, so the 16-byte reads of eight consecutive threads
// (eight consecutive groups) hit eight different bank groups.  Both stages
// are requested at once when the kernel starts and each is refilled as soon
// as every thread has taken its group out of it, so the HBM stream runs
// while the rows already delivered are rotated and quantized.  One thread
// owns one group; its g values go from shared memory straight into float2
// registers.
//
// QMAX: 7 = symmetric INT4 (packed), 127 = symmetric INT8, 15 = asymmetric
// 4-bit with a zero point (W4A8 weights, packed unsigned codes): per row
// s = fl32(fl32(max - min) / 15), z = clamp(rint(fl32(-min / s)), 0, 15),
// q = clamp(rint(fl32(y / s)) + z, 0, 15), zero point written to `zero`.
// SR (QMAX 7 only): stochastic rounding with Philox4x64-10 under `seed`
// instead of round-to-nearest (re-quantizing weights with a baked LoRA).
template <int G, bool ROT, int QMAX, int MAXT, bool SR = false>
__global__ void __launch_bounds__(MAXT, MAXT == 128 ? 3 : 1)
    rotate_quantize_kernel(const __grid_constant__ CUtensorMap tmX, int M, int K, int rows_per_blk,
                           uint8_t* __restrict__ out, float* __restrict__ scale, uint8_t* __restrict__ zero,
                           unsigned long long seed, unsigned int* err) {
  constexpr int HALF = G / 2;
  constexpr int NH = G / 64;   // 64-element halves of a group, one TMA box each
  constexpr bool ASYM = (QMAX == 15);
  constexpr bool INT4 = (QMAX == 7) || ASYM;
  extern __shared__ uint8_t stage_raw[];
  // row maxima, three buffers: iteration it uses buffer it % 3 and clears
  // buffer (it + 1) % 3, last read in iteration it - 2, which every thread
  // has left once it passed the row barrier of iteration it - 1
  __shared__ unsigned int rowmax[3][MAXT];
  __shared__ unsigned int rowmin[ASYM ? 3 : 1][ASYM ? MAXT : 1];   // order-preserving keys (ASYM)
  __shared__ __align__(8) uint64_t full[kStages];

  const int gpr = K / G;
  const int tid = threadIdx.x;
  const int lr = tid / gpr;
  const int grp = tid - lr * gpr;
  const int blk_groups = rows_per_blk * gpr;
  // every box starts on a 1024-byte boundary (the 128-byte swizzle repeats
  // every 8 lines), so line j of a box has its chunks permuted by j % 8
  const uint32_t half_bytes = ((uint32_t)blk_groups * 128u + 1023u) & ~1023u;
  const uint32_t stage_bytes = half_bytes * NH;
  const int nblk = (M + rows_per_blk - 1) / rows_per_blk;
  const uint32_t stage0 = (smem_u32(stage_raw) + 1023u) & ~1023u;   // swizzled boxes: 1024-byte aligned

  // block it of this CTA into its stage (thread 0)
  auto issue = [&](int it) {
    const int blk = blockIdx.x + it * gridDim.x;
    if (blk >= nblk) return;
    const int s = it % kStages;
    const uint32_t dst = stage0 + (uint32_t)s * stage_bytes;
    const int g0 = blk * blk_groups;
    mbar_arrive_expect_tx(&full[s], (uint32_t)(NH * blk_groups * 128));   // the boxes' bytes, not the padding
    if (NH == 1) {
      tma_load_2d(dst, &tmX, 0, g0, &full[s]);
    } else {
      tma_load_3d(dst, &tmX, 0, 0, g0, &full[s]);
      tma_load_3d(dst + half_bytes, &tmX, 0, 1, g0, &full[s]);
    }
  };

  rowmax[0][tid] = 0u;
  if (ASYM) rowmin[0][tid] = 0xFFFFFFFFu;
  if (tid == 0) {
    prefetch_tmap(&tmX);
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // launched with programmatic stream serialization: wait for the previous
  // kernel of the stream (it may produce X, or still read this output)
  grid_dependency_wait();
  grid_launch_dependents();
  if (tid == 0)
    for (int it = 0; it < kStages; ++it) issue(it);

  for (int it = 0;; ++it) {
    const int blk = blockIdx.x + it * gridDim.x;
    if (blk >= nblk) break;
    const int stg = it % kStages;
    if (tid < rows_per_blk) {
      rowmax[(it + 1) % 3][tid] = 0u;
      if (ASYM) rowmin[(it + 1) % 3][tid] = 0xFFFFFFFFu;
    }
    unsigned int* rmax = rowmax[it % 3];
    unsigned int* rmin = rowmin[ASYM ? (it % 3) : 0];

    const long row = (long)blk * rows_per_blk + lr;
    const bool active = (lr < rows_per_blk) && (row < M);
    float2 P[HALF];  // P[i] = (y_i, y_{i+HALF})
    if (active) {
      if (!mbar_wait(&full[stg], (uint32_t)(it / kStages) & 1u)) set_device_error(err, kDevErrTimeoutFull);
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const uint32_t line = stage0 + (uint32_t)stg * stage_bytes + (uint32_t)h * half_bytes + (uint32_t)tid * 128u;
        const uint32_t sw = (uint32_t)tid & 7u;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 t;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(t.x), "=r"(t.y), "=r"(t.z), "=r"(t.w)
                       : "r"(line | ((((uint32_t)c) ^ sw) << 4)));
          // elements 64h + 8c .. 64h + 8c + 7 of the group
          const uint32_t wv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int e = 64 * h + 8 * c + q;
            const float f = (q & 1) ? bf16hi(wv[q / 2]) : bf16lo(wv[q / 2]);
            if (e < HALF) P[e].x = f;
            else P[e - HALF].y = f;
          }
        }
      }
      if (ROT) {
        // stages h = 1 .. HALF/2: pairs (i, i+h) sit in different float2s.
        // a - b is formed as fma(b, -1, a): the product is exact, so this is
        // the single IEEE subtraction, without a separate negation.
        const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
        for (int h = 1; h < HALF; h <<= 1) {
#pragma unroll
          for (int i = 0; i < HALF; ++i) {
            if ((i & h) == 0) {
              const float2 a = P[i], b = P[i + h];
              P[i] = __fadd2_rn(a, b);
              P[i + h] = __ffma2_rn(b, m1, a);
            }
          }
        }
      }
      float amax = 0.0f;
      if (ROT) {
        // last stage h = HALF on the two halves of each float2.  Its outputs
        // a + b and a - b have max(|a + b|, |a - b|) = fl(|a| + |b|) exactly
        // (rounding is monotone and sign-symmetric), which gives the absmax.
#pragma unroll
        for (int i = 0; i < HALF; i += 2) {
          const float a0 = P[i].x, b0 = P[i].y, a1 = P[i + 1].x, b1 = P[i + 1].y;
          amax = max3(amax, __fadd_rn(fabsf(a0), fabsf(b0)), __fadd_rn(fabsf(a1), fabsf(b1)));
          P[i].x = __fadd_rn(a0, b0);
          P[i].y = __fsub_rn(a0, b0);
          P[i + 1].x = __fadd_rn(a1, b1);
          P[i + 1].y = __fsub_rn(a1, b1);
        }
      } else {
#pragma unroll
        for (int i = 0; i < HALF; ++i) amax = max3(amax, fabsf(P[i].x), fabsf(P[i].y));
      }
      if (ASYM) {
        // the last stage above already wrote the outputs back into P
        float mn = P[0].x, mx = P[0].x;
#pragma unroll
        for (int i = 0; i < HALF; ++i) {
          mn = fminf(mn, fminf(P[i].x, P[i].y));
          mx = fmaxf(mx, fmaxf(P[i].x, P[i].y));
        }
        atomicMax(&rmax[lr], fkey(mx));
        atomicMin(&rmin[lr], fkey(mn));
      } else {
        atomicMax(&rmax[lr], __float_as_uint(amax));
      }
    }
    __syncthreads();
    // every thread has its group in registers (its row maximum above depends
    // on all of them): the stage takes the block after next
    if (tid == 0) {
      fence_proxy_async_smem();
      issue(it + kStages);
    }
    if (!active) continue;

    float s;
    int zoff = 0;
    if (ASYM) {
      const float mx = fkey_value(rmax[lr]), mn = fkey_value(rmin[lr]);
      s = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
      int z = 0;
      if (s != 0.0f) z = min(max(__float2int_rn(__fdiv_rn(-mn, s)), 0), 15);
      zoff = z - (int)__float_as_uint(kMagic);
      if (grp == 0) zero[row] = (uint8_t)z;
    } else {
      s = __fdiv_rn(__uint_as_float(rmax[lr]), (float)QMAX);
    }
    if (grp == 0) scale[row] = s;
    float inv_hi = 0.0f, inv_lo = 0.0f;
    if (s != 0.0f) {
      const float inv = __frcp_rn(s);
      inv_hi = __fmul_rn(inv, 1.0f + 0x1p-20f);
      inv_lo = __fmul_rn(inv, 1.0f - 0x1p-20f);
    }
    const float2 ih = make_float2(inv_hi, inv_hi), il = make_float2(inv_lo, inv_lo);

    // Codes leave in 16-byte chunks as soon as they are complete: SB blocks of
    // 8 pairs fill one chunk of .x-lane codes and one of .y-lane codes.  A
    // block whose quotients come within 2^-20 (relative) of a rounding
    // boundary is redone at once with the IEEE quotient the codes are
    // defined by.
    constexpr int SB = INT4 ? 4 : 2;
    constexpr int YCH = INT4 ? HALF / 32 : HALF / 16;  // first chunk of .y codes
    const long row_bytes = INT4 ? K / 2 : K;
    uint4* dst = reinterpret_cast<uint4*>(out + row * row_bytes + (long)grp * (INT4 ? G / 2 : G));
#pragma unroll
    for (int c = 0; c < HALF / (8 * SB); ++c) {
      uint32_t w[2 * SB * (INT4 ? 1 : 2)];  // .x words then .y words
#pragma unroll
      for (int b = 0; b < SB; ++b) {
        const int blk8 = c * SB + b;
        uint32_t bw[INT4 ? 2 : 4];
        if constexpr (SR) {
          const uint64_t e0 = (uint64_t)row * (uint64_t)K + (uint64_t)(grp * G + 8 * blk8);
          quantize_block8_sr(P + 8 * blk8, s, e0, e0 + HALF, seed, bw);
        } else {
          uint32_t bad = 0u;
          quantize_block8<INT4, false, ASYM>(P + 8 * blk8, ih, il, s, bw, bad, zoff);
          if (bad) quantize_block8<INT4, true, ASYM>(P + 8 * blk8, ih, il, s, bw, bad, zoff);
        }
        if (INT4) {
          w[b] = bw[0];
          w[SB + b] = bw[1];
        } else {
          w[2 * b] = bw[0];
          w[2 * b + 1] = bw[1];
          w[2 * SB + 2 * b] = bw[2];
          w[2 * SB + 2 * b + 1] = bw[3];
        }
      }
      dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[YCH + c] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  }
}

// Launch shape: rows per block R (R * K/g threads, at most MAXT) and the
// number of resident CTAs decide how many waves the persistent grid walks.
// Every R is tried and the one with the least modelled time kept: a wave
// costs the larger of a fixed memory latency and its bytes at HBM rate, and
// the last wave costs as much as a full one.  (M = 4608, K = 3072, g = 128:
// R = 5 gives 922 blocks on 444 CTAs -- three waves, the last 8% full;
// R = 4 gives 1152 blocks on 592 CTAs -- two waves.)  A pure host function:
// `per_sm(threads, smem)` gives the resident CTAs per SM of a candidate.
template <class Occ>
bool plan_rq_shape(int M, int K, int G, int maxt, int sms, Occ&& per_sm_of, RqShape& out) {
  const int gpr = K / G;
  const int max_r = gpr >= maxt ? 1 : maxt / gpr;
  double best = 1e30;
  bool found = false;
  for (int r = max_r; r >= 1; --r) {
    const int threads = ((r * gpr + 31) / 32) * 32;
    if (threads > maxt) continue;
    const int smem = kStages * (G / 64) * ((r * gpr * 128 + 1023) / 1024) * 1024 + 1024;   // stages + alignment slack
    int per_sm = 0;
    if (!per_sm_of(threads, smem, per_sm)) return false;
    per_sm = per_sm < 1 ? 1 : per_sm;
    const long nblk = (M + r - 1) / r;
    const long resident = (long)sms * per_sm;
    const long grid = nblk < resident ? nblk : resident;
    const long waves = (nblk + grid - 1) / grid;
    const double wave_bytes = (double)grid * r * K * 2.0;
    const double cost = (double)waves * (wave_bytes / 6.5e12 > 1.2e-6 ? wave_bytes / 6.5e12 : 1.2e-6);
    if (cost < best * 0.999) {
      best = cost;
      out = RqShape{r, threads, smem, (int)grid};
      found = true;
    }
  }
  return found;
}

// Shapes already planned, keyed by (device, M, K, kernel instantiation).
struct RqKey {
  int64_t v[4];
};
PlanCache<RqKey, RqShape, 64>& rq_cache() {
  static PlanCache<RqKey, RqShape, 64> c;
  return c;
}

template <int G, bool ROT, int QMAX, int MAXT, bool SR>
int64_t rq_kernel_id() {
  return (int64_t)G | ((int64_t)ROT << 10) | ((int64_t)QMAX << 11) | ((int64_t)MAXT << 19) | ((int64_t)SR << 30);
}

template <int G, bool ROT, int QMAX, int MAXT, bool SR = false>
cudaError_t launch_rq_t(const uint16_t* X, int M, int K, uint8_t* out, float* scale, uint8_t* zero,
                        unsigned long long seed, cudaStream_t st) {
  auto kern = rotate_quantize_kernel<G, ROT, QMAX, MAXT, SR>;
  unsigned int* err = device_error_word();
  if (!err) return cudaErrorInvalidDevicePointer;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static DeviceFlags attr_set;   // one per instantiation
  if (!attr_set.done(dev)) {
    // the largest ring any shape uses (MAXT threads' groups, kStages deep)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kStages * (G / 64) * ((MAXT * 128 + 1023) / 1024) * 1024 + 1024);
    if (e != cudaSuccess) return e;
    attr_set.set(dev);
  }
  RqShape sh;
  const RqKey key = {{dev, M, K, rq_kernel_id<G, ROT, QMAX, MAXT, SR>()}};
  const bool ok = rq_cache().get(key, sh, [&](RqShape& v) {
    int sms = 0;
    if ((e = device_sm_count(dev, &sms)) != cudaSuccess) return false;
    return plan_rq_shape(M, K, G, MAXT, sms, [&](int threads, int smem, int& per_sm) {
      return (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem)) == cudaSuccess;
    }, v);
  });
  if (!ok) return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
  // X as [M * K/G groups][G/64 halves][64 elements] bf16; one box per half
  // holds the groups of one block of rows
  CUtensorMap tm;
  const uint64_t groups = (uint64_t)M * (uint64_t)(K / G);
  const uint32_t blk_groups = (uint32_t)(sh.rows_per_blk * (K / G));
  bool enc;
  if (G == 64) {
    const uint64_t dims[2] = {64, groups};
    const uint64_t strides[1] = {128};
    const uint32_t box[2] = {64, blk_groups};
    enc = make_tmap_nd(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    const uint64_t dims[3] = {64, 2, groups};
    const uint64_t strides[2] = {128, 256};
    const uint32_t box[3] = {64, 1, blk_groups};
    enc = make_tmap_nd(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!enc) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sh.grid, 1, 1);
  cfg.blockDim = dim3(sh.threads, 1, 1);
  cfg.dynamicSmemBytes = sh.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tm, M, K, sh.rows_per_blk, out, scale, zero, seed, err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Rows of up to 128 groups run in 128-thread CTAs (three per SM); wider rows
// (K / g > 128) in 256-thread CTAs, one group per thread either way.
template <int G, bool ROT, int QMAX, bool SR = false>
cudaError_t launch_rq(const uint16_t* X, int M, int K, uint8_t* out, float* scale, uint8_t* zero,
                      unsigned long long seed, cudaStream_t st) {
  if (K / G <= 128) return launch_rq_t<G, ROT, QMAX, 128, SR>(X, M, K, out, scale, zero, seed, st);
  return launch_rq_t<G, ROT, QMAX, 256, SR>(X, M, K, out, scale, zero, seed, st);
}

template <int QMAX, bool SR = false>
cudaError_t launch_rq_group(const uint16_t* X, int rows, int K, int group, uint8_t* out, float* scale, uint8_t* zero,
                            unsigned long long seed, cudaStream_t st) {
  if (group == 64) return launch_rq<64, true, QMAX, SR>(X, rows, K, out, scale, zero, seed, st);
  if (group == 128) return launch_rq<128, true, QMAX, SR>(X, rows, K, out, scale, zero, seed, st);
  return launch_rq<128, false, QMAX, SR>(X, rows, K, out, scale, zero, seed, st);
}

}  // namespace

// Launch-free planning of the rotate + quantize kernel's shape, for the
// host-side thread-safety test: the same planner and cache type the launcher
// uses, fed a fixed occupancy instead of a CUDA query.  `cached` selects a
// shared eight-entry cache (constantly evicted when many shapes are asked
// for) or a direct computation.
bool plan_rotate_quantize_shape(int M, int K, int group, int sms, int resident_per_sm, bool cached, int out[4]) {
  static PlanCache<RqKey, RqShape, 8> test_cache;
  const int G = group == 64 ? 64 : 128;
  const int maxt = K / G <= 128 ? 128 : 256;
  auto make = [&](RqShape& v) {
    return plan_rq_shape(M, K, G, maxt, sms, [&](int, int, int& per_sm) {
      per_sm = resident_per_sm;
      return true;
    }, v);
  };
  RqShape sh;
  const RqKey key = {{sms + 1000 * resident_per_sm, M, K, group}};
  if (!(cached ? test_cache.get(key, sh, make) : make(sh))) return false;
  out[0] = sh.rows_per_blk;
  out[1] = sh.threads;
  out[2] = sh.smem;
  out[3] = sh.grid;
  return true;
}

// Rows of X [rows, K] bf16 -> codes and one fp32 scale per row: packed
// nibbles [rows, K/2] when qmax == 7 (symmetric) or qmax == 15 (asymmetric,
// zero point per row written to `zero`), int8 [rows, K] when qmax == 127.
// group 0 turns the rotation off.  Shapes are validated by the caller.
cudaError_t launch_rotate_quantize(const uint16_t* X, int rows, int K, int group, int qmax, uint8_t* out,
                                   float* scale, uint8_t* zero, cudaStream_t st) {
  if (qmax == 7) return launch_rq_group<7>(X, rows, K, group, out, scale, nullptr, 0ull, st);
  if (qmax == 15) return launch_rq_group<15>(X, rows, K, group, out, scale, zero, 0ull, st);
  return launch_rq_group<127>(X, rows, K, group, out, scale, nullptr, 0ull, st);
}

// Symmetric INT4 with stochastic rounding (Philox4x64-10 under `seed`).
cudaError_t launch_rotate_quantize_sr(const uint16_t* X, int rows, int K, int group, uint8_t* out, float* scale,
                                      unsigned long long seed, cudaStream_t st) {
  return launch_rq_group<7, true>(X, rows, K, group, out, scale, nullptr, seed, st);
}

}  // namespace w4a4
