/*
 * Plain CPU oracle for the W4A4 ConvRot linear layer and its W8A8 and W4A8
 * twins.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA kernels.
 *
 * What it follows (the pages are prose; each step restates them):
 *   - "Load Diffusion Model INT4 (W4A4)" (comfy.icu, intro): every layer is
 *     squeezed to 4 bit with a Hadamard rotation (ConvRot) applied first, then
 *     the matmuls run on integer tensor cores.
 *   - "W4A4 and W4A8: The New Quantization Toolkit" (renderbob.io, "Decoding
 *     the notation"): weights are quantized once, activations on the fly.
 *   - "Krea 2 Turbo - SVDQuant" (sweettea.co, "Why activation-aware INT4" and
 *     "What's included"): the rotation handles outliers; a low-rank branch
 *     runs in parallel with the 4-bit matmul and needs no calibration.
 *   - "ComfyUI-INT4-Fast" (kongchang.com, "Per-Layer Dynamic Routing") and the
 *     toolkit page ("How the toolkit tells you to choose"): sensitive layers
 *     run as W8A8.
 * The pages fix no formula.  Readings used here (listed in the design notes):
 *   H_g[i][j] = (-1)^popcount(i & j) (Sylvester order, entries +-1, no 1/sqrt(g));
 *   rotated y_i = sum_j H_ij x_j in fp32, summed as a balanced binary tree over
 *   j in index order; s = fl32(amax / qmax); q = clamp(rint_even(fl32(y / s)));
 *   one scale per token (activations) and per output channel (weights) over
 *   all of K; the epilogue multiplies by 1/g because H H^T = g I.
 *
 * Build: gcc -std=c11 -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 * No FMA contraction and no fast-math: every fp32 operation is one IEEE
 * round-to-nearest-even operation on SSE registers.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- bf16 <-> fp32 ----------------------------------------------------- */

/* bf16 is the upper half of an IEEE binary32: widening is exact. */
static float bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round-to-nearest-even narrowing of binary32 to bf16 (NaN kept quiet). */
static uint16_t f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

void oracle_f32_to_bf16(const float *x, long n, uint16_t *out) {
    for (long i = 0; i < n; ++i) out[i] = f32_to_bf16(x[i]);
}

void oracle_f64_to_bf16(const double *x, long n, uint16_t *out) {
    /* double -> float (RN) -> bf16 (RN) can double-round; do it in one step:
       round the double directly to 8 significant bits, ties to even. */
    for (long i = 0; i < n; ++i) {
        double v = x[i];
        if (v != v) { out[i] = 0x7fc0u; continue; }
        if (v == 0.0) { out[i] = signbit(v) ? 0x8000u : 0; continue; }
        int e;
        double m = frexp(fabs(v), &e);          /* |v| = m * 2^e, m in [0.5,1) */
        int emin = -125;                        /* smallest normal exponent (frexp form) */
        int prec = 8;                           /* bf16 significand bits */
        int shift = (e < emin) ? prec - (emin - e) : prec;  /* subnormals keep fewer bits */
        double scaled = ldexp(m, shift);
        double r = nearbyint(scaled);           /* default mode: ties to even */
        double mag = ldexp(r, e - shift);
        float f = (float)(v < 0 ? -mag : mag);  /* exact: mag has <= 8 bits */
        if (isinf(f) || fabs(mag) > 3.3895313892515355e38) {
            out[i] = v < 0 ? 0xff80u : 0x7f80u;
            continue;
        }
        uint32_t u;
        memcpy(&u, &f, sizeof u);
        out[i] = (uint16_t)(u >> 16);
    }
}

/* ---- Hadamard matrix ---------------------------------------------------- */

/* Sylvester-ordered Hadamard matrix of order g (a power of two):
   H[i][j] = (-1)^popcount(i & j).  Entries +-1, H H^T = g I. */
void oracle_hadamard(int g, int8_t *H) {
    for (int i = 0; i < g; ++i)
        for (int j = 0; j < g; ++j)
            H[(long)i * g + j] = (__builtin_popcount((unsigned)(i & j)) & 1) ? -1 : 1;
}

/* ---- ConvRot: block-diagonal Hadamard rotation of each row ---------------- */

/* Balanced pairwise sum of H[i][j] * x[j] for j in [lo, lo + len), len a power
   of two: the two halves are summed first, left half on the left.  Each term
   H_ij * x_j is exact (a sign flip). */
static float tree_sum(const int8_t *Hrow, const float *x, int lo, int len) {
    if (len == 1) return Hrow[lo] > 0 ? x[lo] : -x[lo];
    int half = len / 2;
    float a = tree_sum(Hrow, x, lo, half);
    float b = tree_sum(Hrow, x, lo + half, half);
    return a + b;
}

/* Y[row][k] for every row: each group of g consecutive entries along K is
   replaced by H_g times that group (explicit matrix, tree-order fp32 sums).
   g == 0 turns the rotation off (Y = X widened to fp32).
   Returns 0, or -1 when g is not a power of two dividing K. */
int oracle_rotate(const uint16_t *X, long rows, int K, int g, float *Y) {
    if (g == 0) {
        for (long i = 0; i < rows * (long)K; ++i) Y[i] = bf16_to_f32(X[i]);
        return 0;
    }
    if (g < 1 || (g & (g - 1)) || K % g) return -1;
    int8_t *H = (int8_t *)malloc((size_t)g * g);
    if (!H) return -2;
    oracle_hadamard(g, H);
    #pragma omp parallel
    {
        float *x = (float *)malloc(sizeof(float) * g);
        #pragma omp for schedule(static)
        for (long r = 0; r < rows; ++r) {
            for (int k0 = 0; k0 < K; k0 += g) {
                const uint16_t *src = X + r * K + k0;
                for (int j = 0; j < g; ++j) x[j] = bf16_to_f32(src[j]);
                for (int i = 0; i < g; ++i)
                    Y[r * K + k0 + i] = tree_sum(H + (long)i * g, x, 0, g);
            }
        }
        free(x);
    }
    free(H);
    return 0;
}

/* ---- symmetric absmax quantization, one scale per row ---------------------- */

/* s = fl32(max_k |Y[row][k]| / qmax); q = clamp(rint_even(fl32(y / s)), lo, qmax)
   with lo = -8 for qmax == 7 (two's-complement INT4) and lo = -127 for
   qmax == 127 (symmetric INT8).  A row with amax == 0 gets s = 0 and all codes
   0.  Division and rounding are single IEEE fp32 operations. */
void oracle_quantize(const float *Y, long rows, int K, int qmax, int8_t *q, float *scale) {
    const float qmax_f = (float)qmax;
    const int lo = (qmax == 7) ? -8 : -qmax;
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        const float *y = Y + r * K;
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(y[k]);
            if (a > amax) amax = a;
        }
        float s = amax / qmax_f;
        scale[r] = s;
        for (int k = 0; k < K; ++k) {
            int v = 0;
            if (s != 0.0f) {
                float t = y[k] / s;
                float rt = nearbyintf(t);          /* ties to even */
                v = (int)rt;
                if (v < lo) v = lo;
                if (v > qmax) v = qmax;
            }
            q[r * K + k] = (int8_t)v;
        }
    }
}

/* ---- asymmetric 4-bit quantization with a zero point, one pair per row ---- */

/* W4A8 weights ("W4A4 and W4A8: The New Quantization Toolkit", "How the
   toolkit tells you to choose": the W4A8 mode keeps 4-bit weights with a zero
   point).  Per row of the rotated weights: mn = min y, mx = max y,
   s = fl32(fl32(mx - mn) / 15), z = clamp(rint_even(fl32(-mn / s)), 0, 15),
   q = clamp(rint_even(fl32(y / s)) + z, 0, 15) (unsigned codes; the weight
   they stand for is (q - z) * s).  A row with mx == mn gets s = 0, z = 0 and
   all codes 0.  Every division and rounding is a single IEEE fp32 operation. */
void oracle_quantize_asym4(const float *Y, long rows, int K, uint8_t *q, float *scale, uint8_t *zero) {
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        const float *y = Y + r * K;
        float mn = y[0], mx = y[0];
        for (int k = 1; k < K; ++k) {
            if (y[k] < mn) mn = y[k];
            if (y[k] > mx) mx = y[k];
        }
        const float range = mx - mn;
        const float s = range / 15.0f;
        int z = 0;
        if (s != 0.0f) {
            const float t = (-mn) / s;
            z = (int)nearbyintf(t);
            if (z < 0) z = 0;
            if (z > 15) z = 15;
        }
        scale[r] = s;
        zero[r] = (uint8_t)z;
        for (int k = 0; k < K; ++k) {
            int v = 0;
            if (s != 0.0f) {
                v = (int)nearbyintf(y[k] / s) + z;
                if (v < 0) v = 0;
                if (v > 15) v = 15;
            }
            q[r * K + k] = (uint8_t)v;
        }
    }
}

/* ---- INT4 nibble packing ------------------------------------------------- */

/* Row-major [rows, K/2] bytes: byte j of a row holds code 2j in bits 0..3 and
   code 2j+1 in bits 4..7, both as 4-bit two's complement. */
void oracle_pack_int4(const int8_t *q, long rows, int K, uint8_t *packed) {
    for (long r = 0; r < rows; ++r)
        for (int j = 0; j < K / 2; ++j) {
            unsigned lo = (unsigned)q[r * K + 2 * j] & 0xFu;
            unsigned hi = (unsigned)q[r * K + 2 * j + 1] & 0xFu;
            packed[r * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
        }
}

void oracle_unpack_int4(const uint8_t *packed, long rows, int K, int8_t *q) {
    for (long r = 0; r < rows; ++r)
        for (int j = 0; j < K / 2; ++j) {
            uint8_t b = packed[r * (K / 2) + j];
            int lo = b & 0xF, hi = b >> 4;
            q[r * K + 2 * j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
            q[r * K + 2 * j + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
        }
}

/* ---- integer GEMM --------------------------------------------------------- */

/* acc[m][n] = sum_k qa[m][k] * qw[n][k], accumulated in int64 and stored as
   int32.  Returns the number of entries that did not fit int32 (0 expected:
   |acc| <= 64 K for INT4 codes). */
long oracle_int_gemm(const int8_t *qa, const int8_t *qw, long M, long N, int K, int32_t *acc) {
    long overflow = 0;
    #pragma omp parallel for schedule(static) reduction(+ : overflow)
    for (long m = 0; m < M; ++m) {
        const int8_t *a = qa + m * K;
        for (long n = 0; n < N; ++n) {
            const int8_t *w = qw + n * K;
            int64_t s = 0;
            for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)w[k];
            if (s > INT32_MAX || s < INT32_MIN) ++overflow;
            acc[m * N + n] = (int32_t)s;
        }
    }
    return overflow;
}

/* ---- low-rank branch and epilogue -------------------------------------------- */

/* T[m][j] = sum_k X[m][k] * L1[k][j] in fp64 (unrotated bf16 X). */
void oracle_lowrank_down(const uint16_t *X, const uint16_t *L1, long M, int K, int r, double *T) {
    #pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m)
        for (int j = 0; j < r; ++j) {
            double s = 0.0;
            for (int k = 0; k < K; ++k)
                s += (double)bf16_to_f32(X[m * K + k]) * (double)bf16_to_f32(L1[(long)k * r + j]);
            T[m * r + j] = s;
        }
}

/* ---- baking a LoRA into the weights, stochastic-rounding re-quantization ---- */

/* "ComfyUI-INT4-Fast" ("INT4 Quantized Inference Comes to ComfyUI") and the
   toolkit page ("How the toolkit tells you to choose") let a LoRA be baked
   into the 4-bit weights; re-quantizing W + dW rounds stochastically so the
   small LoRA update survives 4-bit rounding in expectation.  Readings:
     Wb[n][k] = bf16(fl32(W[n][k] + fl32(scale * sum_j A[k][j] B[j][n]))),
   the sum as fp32 fused multiply-adds in index order j = 0, 1, ...;
   codes after the usual rotation and absmax scale s = fl32(amax / 7):
     q = clamp(floor(fl32(fl32(y / s) + u)), -8, 7),  u in [0, 1),
   u drawn from Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
   numbers: as easy as 1, 2, 3", SC 2011): element e of the row-major [N, K]
   array takes word e % 4 of Philox(counter = (e / 4, 0, 0, 0),
   key = (seed, 0)), and u = (word >> 40) * 2^-24 (24 random bits, exact in
   fp32). */
void oracle_philox4x64(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4]) {
    const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
    const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
    uint64_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3], k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        const unsigned __int128 p0 = (unsigned __int128)M0 * c0;
        const unsigned __int128 p1 = (unsigned __int128)M1 * c2;
        const uint64_t hi0 = (uint64_t)(p0 >> 64), lo0 = (uint64_t)p0;
        const uint64_t hi1 = (uint64_t)(p1 >> 64), lo1 = (uint64_t)p1;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
        if (r < 9) {
            k0 += W0;
            k1 += W1;
        }
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

void oracle_sr_uniform(long n, uint64_t seed, float *u) {
    #pragma omp parallel for schedule(static)
    for (long b = 0; b < (n + 3) / 4; ++b) {
        const uint64_t ctr[4] = {(uint64_t)b, 0, 0, 0}, key[2] = {seed, 0};
        uint64_t w[4];
        oracle_philox4x64(ctr, key, w);
        for (int l = 0; l < 4 && 4 * b + l < n; ++l) u[4 * b + l] = (float)(w[l] >> 40) * 0x1p-24f;
    }
}

void oracle_lora_bake(const uint16_t *W, const uint16_t *A, const uint16_t *B, int N, int K, int rl, float scale,
                      uint16_t *Wb) {
    #pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            float acc = 0.0f;
            for (int j = 0; j < rl; ++j)
                acc = fmaf(bf16_to_f32(A[(long)k * rl + j]), bf16_to_f32(B[(long)j * N + n]), acc);
            const float d = scale * acc;
            Wb[n * K + k] = f32_to_bf16(bf16_to_f32(W[n * K + k]) + d);
        }
}

/* s = fl32(amax / 7) per row, q = clamp(floor(fl32(fl32(y / s) + u)), -8, 7);
   a row with amax == 0 gets s = 0 and codes 0. */
void oracle_quantize_sr(const float *Y, long rows, int K, const float *U, int8_t *q, float *scale) {
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        const float *y = Y + r * K;
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(y[k]);
            if (a > amax) amax = a;
        }
        const float s = amax / 7.0f;
        scale[r] = s;
        for (int k = 0; k < K; ++k) {
            int v = 0;
            if (s != 0.0f) {
                const float t = y[k] / s;
                const float w = t + U[r * K + k];
                v = (int)floorf(w);
                if (v < -8) v = -8;
                if (v > 7) v = 7;
            }
            q[r * K + k] = (int8_t)v;
        }
    }
}

/* GELU with the tanh approximation, in fp64 (the MLP between the up and down
   projections of the pages' diffusion transformer blocks, "Load Diffusion
   Model INT4 (W4A4)": every linear layer of the model runs in 4 bit, the
   activation between them in high precision):
   gelu(x) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))). */
void oracle_gelu_tanh(const double *x, long n, double *y) {
    const double c = sqrt(2.0 / 3.14159265358979323846);
    #pragma omp parallel for schedule(static)
    for (long i = 0; i < n; ++i) {
        const double v = x[i];
        y[i] = 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)));
    }
}

/* Runtime LoRA merged into the low-rank branch ("ComfyUI-INT4-Fast",
   "INT4 Quantized Inference Comes to ComfyUI": LoRAs apply on top of the 4-bit
   layer; "Krea 2 Turbo - SVDQuant", "What's included": the low-rank branch
   runs beside the 4-bit product).  L1o = [L1 | A] ([K, r + rl]),
   L2o = [L2 ; bf16(fl32(scale * B))] ([r + rl, N]): the LoRA's scale is folded
   into its up matrix with one fp32 multiply and one round-to-nearest-even
   narrowing per element. */
void oracle_lora_merge(const uint16_t *L1, const uint16_t *L2, int r, const uint16_t *A, const uint16_t *B, int rl,
                       float scale, int K, int N, uint16_t *L1o, uint16_t *L2o) {
    const int rt = r + rl;
    for (int k = 0; k < K; ++k)
        for (int j = 0; j < rt; ++j)
            L1o[(long)k * rt + j] = j < r ? L1[(long)k * r + j] : A[(long)k * rl + (j - r)];
    for (int j = 0; j < rt; ++j)
        for (int n = 0; n < N; ++n)
            L2o[(long)j * N + n] = j < r ? L2[(long)j * N + n]
                                         : f32_to_bf16(scale * bf16_to_f32(B[(long)(j - r) * N + n]));
}

/* Y[m][n] = ((acc * sa[m]) * sw[n]) * (1/g) + sum_j T[m][j] * L2[j][n] + bias[n]
   in fp64.  g == 0 means no rotation (factor 1).  T/L2 are ignored when r == 0;
   bias may be NULL. */
/* Y[m][n] += scale * sum_j T[m][j] * U[j][n] in fp64, j in index order: the
 * up-projection of a low-rank branch applied on its own (the runtime LoRA
 * beside the SVDQuant branch, unmerged).  T fp64 [M, r], U bf16 [r, N]. */
void oracle_lowrank_up(const double *T, const uint16_t *U, long M, long N, int r, double scale, double *Y) {
    #pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m)
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int j = 0; j < r; ++j) acc += T[m * r + j] * (double)bf16_to_f32(U[(long)j * N + n]);
            Y[m * N + n] += scale * acc;
        }
}

void oracle_epilogue(const int32_t *acc, const float *sa, const float *sw, long M, long N, int g,
                     const double *T, const uint16_t *L2, int r, const uint16_t *bias, double *Y) {
    const double inv_g = (g > 0) ? 1.0 / (double)g : 1.0;
    #pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m)
        for (long n = 0; n < N; ++n) {
            double y = (double)acc[m * N + n] * (double)sa[m] * (double)sw[n] * inv_g;
            double lr = 0.0;
            for (int j = 0; j < r; ++j) lr += T[m * r + j] * (double)bf16_to_f32(L2[(long)j * N + n]);
            y += lr;
            if (bias) y += (double)bf16_to_f32(bias[n]);
            Y[m * N + n] = y;
        }
}
