/*
 * libw4a4 -- W4A4 ConvRot INT4 linear layer (and its W8A8 twin) for NVIDIA
 * B200 (sm_100a).  C ABI: plain pointers, sizes and a CUDA stream.
 *
 * The method, in the words of the pages it comes from (restated):
 *   - "Load Diffusion Model INT4 (W4A4)" (comfy.icu), intro: every layer is
 *     quantized to 4-bit weights and 4-bit activations, with a Hadamard
 *     rotation (ConvRot) applied first so that the quantization error does not
 *     concentrate in outlier channels; the matmuls then run on integer tensor
 *     cores.  "The inputs you'll actually touch": enable_convrot (on by
 *     default), groupsize, on-the-fly quantization from BF16/FP16 only.
 *   - "W4A4 and W4A8: The New Quantization Toolkit" (renderbob.io), "Decoding
 *     the notation": weights are quantized once, activations on the fly;
 *     "How the toolkit tells you to choose": W8A8 covers layers that do not
 *     tolerate 4 bit, and a caller falls back to it on incompatible shapes.
 *   - "Krea 2 Turbo - SVDQuant" (sweettea.co), "What's included": an optional
 *     low-rank branch (X L1) L2 corrects the quantized product.
 *   - "Save Int4 Model" (comfy.icu), "How it works": one weight_scale per
 *     quantized tensor, a convrot group size recorded per layer.
 *
 * Arithmetic (readings of the pages, identical in the CPU oracle):
 *   H_g[i][j] = (-1)^popcount(i & j), g in {64, 128}; group 0 = no rotation.
 *   Rotation: each group of g consecutive entries along K is multiplied by the
 *     unnormalised H_g in fp32 (butterflies in the order h = 1, 2, 4, ...).
 *   Scale: s = fl32(max_k |y_k| / qmax), one per row (token or output channel);
 *     qmax = 7 (INT4) or 127 (INT8); s = 0 for an all-zero row.
 *   Codes: q = rint_half_even(fl32(y / s)) (IEEE division), |q| <= qmax.
 *   INT4 packing: row-major [rows, K/2] bytes; byte j holds code 2j in bits
 *     0..3 and code 2j+1 in bits 4..7, 4-bit two's complement.
 *   GEMM: acc[m][n] = sum_k qx[m][k] * qw[n][k], exact int32.
 *   Epilogue: Y = bf16_rn( ((acc * s_x[m]) * s_w[n]) * (1/g)
 *                          + sum_j T[m][j] L2[j][n] + bias[n] ),
 *     T = X L1 from the unrotated activations (fp32 sums, stored as bf16).
 *
 * Conventions for every entry point:
 *   - Tensors are caller-owned CUDA device memory, row-major and contiguous,
 *     with 16-byte-aligned base addresses (32-byte for the code tensors Xq and
 *     Wq given to the GEMMs).  bf16 tensors are passed as void*.
 *     The library never allocates on these paths and keeps no state besides
 *     per-device launch attributes and the device error word.
 *   - Calls are asynchronous and ordered on `stream` (NULL = legacy default
 *     stream).  W4A4_OK means "validated and enqueued"; launch failures return
 *     W4A4_ERR_CUDA; faults inside a kernel surface at the caller's next
 *     synchronisation.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check launches nothing and returns the status named below.
 *   - Shape rules: M >= 1; K a multiple of 128 with K / max(g, 128) <= 256
 *     (K <= 32768; K <= 16384 for g = 64); N a multiple of 8 (GEMM and linear);
 *     group in {0, 64, 128}; rank r in [0, 256] and a multiple of 16.
 *   - Only sm_100 devices are supported (W4A4_ERR_UNSUPPORTED_DEVICE
 *     otherwise); there is no CPU fallback.
 *   - The functions are thread-safe and may be called on different streams.
 */
#ifndef W4A4_H_
#define W4A4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* w4a4_stream_t; /* same object as cudaStream_t */

typedef enum {
  W4A4_OK = 0,
  W4A4_ERR_INVALID_ARG = 1,        /* null pointer where one is required, bad enum value */
  W4A4_ERR_UNSUPPORTED_SHAPE = 2,  /* a shape rule above is violated */
  W4A4_ERR_MISALIGNED = 3,         /* a tensor base address is not 16-byte aligned */
  W4A4_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
  W4A4_ERR_DEVICE_TIMEOUT = 5,     /* a kernel gave up a bounded wait (see w4a4_get_device_error) */
  W4A4_ERR_UNSUPPORTED_DEVICE = 6, /* current device is not sm_100 */
  W4A4_ERR_WORKSPACE = 7           /* workspace missing or smaller than *_workspace_bytes() */
} w4a4_status;

/* Version as major * 10000 + minor * 100 + patch. */
int w4a4_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* w4a4_status_string(w4a4_status status);

/* ---------------------------------------------------------------- W4A4 */

/* Offline weight preparation (rotate + per-output-channel INT4 quantize +
 * pack).  Source: "Load Diffusion Model INT4 (W4A4)" (comfy.icu), intro and
 * "on_the_fly_quantization" (quantize BF16/FP16 weights on load).
 *   W        bf16 [N, K] (nn.Linear layout; FP8 checkpoints must be
 *            dequantized by the caller first)
 *   Wq       out: uint8 [N, K/2] packed codes
 *   w_scale  out: fp32 [N]
 */
w4a4_status w4a4_quantize_weights(const void* W, int N, int K, int group, uint8_t* Wq, float* w_scale,
                                  w4a4_stream_t stream);

/* On-the-fly activation path: rotate + per-token INT4 quantize + pack, and
 * the low-rank down-projection T = X L1 when rank > 0.  Source: "W4A4 and
 * W4A8: The New Quantization Toolkit" (renderbob.io), "Decoding the notation";
 * "Krea 2 Turbo - SVDQuant" (sweettea.co), "What's included".
 *   X        bf16 [M, K]
 *   Xq       out: uint8 [M, K/2] packed codes
 *   x_scale  out: fp32 [M]
 *   L1       bf16 [K, rank] or NULL when rank == 0
 *   T        out: bf16 [M, rank] or NULL when rank == 0
 */
w4a4_status w4a4_rotate_quantize_act(const void* X, int M, int K, int group, uint8_t* Xq, float* x_scale,
                                     const void* L1, int rank, void* T, w4a4_stream_t stream);

/* INT4 GEMM with the fused dequant + low-rank + bias epilogue.  Source:
 * "Load Diffusion Model INT4 (W4A4)" (comfy.icu), intro (tensor-core matmul
 * at 4 bit); "Krea 2 Turbo - SVDQuant" (sweettea.co), "What's included"
 * (parallel low-rank branch).
 *   Xq, x_scale  as produced by w4a4_rotate_quantize_act
 *   Wq, w_scale  as produced by w4a4_quantize_weights (same group)
 *   T            bf16 [M, rank] or NULL when rank == 0
 *   L2           bf16 [rank, N] or NULL when rank == 0
 *   bias         bf16 [N] or NULL
 *   Y            out: bf16 [M, N]
 *   acc_debug    out: int32 [M, N] exact integer accumulators, or NULL
 * Layers with too few 256 x 256 output tiles to occupy the GPU run a split-K
 * form (w4a4_plan_gemm_split gives the decision); its int32 sums are exact,
 * so Y is bit-identical to the persistent form's.
 */
w4a4_status w4a4_gemm(const uint8_t* Xq, const float* x_scale, const uint8_t* Wq, const float* w_scale, int M,
                      int N, int K, int group, const void* T, const void* L2, int rank, const void* bias, void* Y,
                      int32_t* acc_debug, w4a4_stream_t stream);

/* Bytes of device workspace w4a4_linear needs: packed codes [M, K/2], scales
 * [M] and T [M, rank], each 256-byte aligned.  Returns 0 for invalid sizes. */
size_t w4a4_workspace_bytes(int M, int K, int rank);

/* The whole layer: w4a4_rotate_quantize_act into `workspace`, then w4a4_gemm.
 *   X bf16 [M, K]; Wq, w_scale from w4a4_quantize_weights; L1 [K, rank],
 *   L2 [rank, N] (NULL when rank == 0); bias [N] or NULL; Y out bf16 [M, N];
 *   workspace: device memory of at least w4a4_workspace_bytes(M, K, rank)
 *   bytes, 256-byte aligned, owned by the caller; it must not be used by
 *   another call that may run concurrently on the GPU.
 */
w4a4_status w4a4_linear(const void* X, const uint8_t* Wq, const float* w_scale, int M, int N, int K, int group,
                        const void* L1, const void* L2, int rank, const void* bias, void* Y, void* workspace,
                        size_t workspace_bytes, w4a4_stream_t stream);

/* Allocation-free form of w4a4_linear.  The pages have no counterpart: this
 * serves callers that cannot allocate device memory -- for instance a host
 * program that has given all device memory to its own fixed pool, or a plugin
 * running inside a runtime that forbids cudaMalloc after start-up -- and so
 * cannot pass the workspace w4a4_linear needs.
 *   Scratch: a fixed array of W4A4_NOALLOC_SCRATCH_BYTES inside the library,
 *     one per GPU that loads the library, held by that GPU's CUDA context for
 *     as long as the context lives (normally until the process exits).  The
 *     call allocates nothing (no cudaMalloc, cudaFree or allocating library
 *     routine).  Layers whose w4a4_workspace_bytes(M, K, rank) exceeds the
 *     scratch are rejected with W4A4_ERR_WORKSPACE; use w4a4_linear for them.
 *   The first call in a context looks up the scratch address on that device
 *     (with it current) and caches it per context, so a context recreated
 *     after cudaDeviceReset looks it up again; make that first call before any
 *     stream capture.
 *   All calls share the scratch.  Calls that may overlap on the GPU (other
 *     streams, other host threads) race on it and must be serialised by the
 *     caller.  The scratch keeps the last call's contents; every byte a call
 *     reads is written earlier in the same call, so nothing is cleared.
 *   Arguments, results and errors are otherwise those of w4a4_linear. */
#define W4A4_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
w4a4_status w4a4_linear_noalloc(const void* X, const uint8_t* Wq, const float* w_scale, int M, int N, int K,
                                int group, const void* L1, const void* L2, int rank, const void* bias, void* Y,
                                w4a4_stream_t stream);

/* ---------------------------------------------------------------- W8A8 */
/* The INT8 path for sensitive layers ("ComfyUI-INT4-Fast" (kongchang.com),
 * "Per-Layer Dynamic Routing"; "W4A4 and W4A8" (renderbob.io), "How the
 * toolkit tells you to choose": int8 is the W8A8 path).  Same rotation and
 * scaling with qmax = 127, codes stored unpacked as int8 [rows, K], no
 * low-rank branch. */
w4a4_status w8a8_quantize_weights(const void* W, int N, int K, int group, int8_t* Wq, float* w_scale,
                                  w4a4_stream_t stream);
w4a4_status w8a8_rotate_quantize_act(const void* X, int M, int K, int group, int8_t* Xq, float* x_scale,
                                     w4a4_stream_t stream);
w4a4_status w8a8_gemm(const int8_t* Xq, const float* x_scale, const int8_t* Wq, const float* w_scale, int M,
                      int N, int K, int group, const void* bias, void* Y, int32_t* acc_debug,
                      w4a4_stream_t stream);
size_t w8a8_workspace_bytes(int M, int K);
w4a4_status w8a8_linear(const void* X, const int8_t* Wq, const float* w_scale, int M, int N, int K, int group,
                        const void* bias, void* Y, void* workspace, size_t workspace_bytes,
                        w4a4_stream_t stream);

/* ---------------------------------------------------------------- W4A8 twin */
/* 4-bit weights with a zero point and 8-bit activations ("W4A4 and W4A8: The
 * New Quantization Toolkit" (renderbob.io), "Decoding the notation" and "How
 * the toolkit tells you to choose": the W4A8 mode keeps 4-bit weights and
 * 8-bit activations, with a zero point on the weights).  Weights are rotated
 * like W4A4, then quantized per output channel asymmetrically:
 *   s = fl32(fl32(max - min) / 15), z = clamp(rint_even(fl32(-min / s)), 0, 15),
 *   q = clamp(rint_even(fl32(y / s)) + z, 0, 15)
 * (a row with max == min gets s = 0, z = 0 and codes 0).  Codes are stored as
 * unsigned nibbles [N, K/2] (code 2j in the low nibble of byte j), the zero
 * point as one byte per row.  Activations are those of the W8A8 path
 * (w8a8_rotate_quantize_act: rotated, symmetric int8 per token).  The GEMM
 * forms acc = sum_k xq * (wq - z) exactly in int32 and applies the W8A8
 * epilogue ((acc * s_x) * s_w) / g + bias -> bf16.  No low-rank branch.
 *
 * Shapes and alignment: as w4a4_quantize_weights (weights) and w8a8_gemm
 * (activations); w_zero needs no alignment.  w4a8_linear takes the
 * workspace of w8a8_linear (w4a8_workspace_bytes). */
w4a4_status w4a8_quantize_weights(const void* W, int N, int K, int group, uint8_t* Wq, float* w_scale,
                                  uint8_t* w_zero, w4a4_stream_t stream);
w4a4_status w4a8_gemm(const int8_t* Xq, const float* x_scale, const uint8_t* Wq, const float* w_scale,
                      const uint8_t* w_zero, int M, int N, int K, int group, const void* bias, void* Y,
                      int32_t* acc_debug, w4a4_stream_t stream);
size_t w4a8_workspace_bytes(int M, int K);
w4a4_status w4a8_linear(const void* X, const uint8_t* Wq, const float* w_scale, const uint8_t* w_zero, int M,
                        int N, int K, int group, const void* bias, void* Y, void* workspace,
                        size_t workspace_bytes, w4a4_stream_t stream);

/* ---------------------------------------------------------------- fused MLP */
/* The MLP of the pages' transformer blocks runs both projections in 4 bit
 * ("Load Diffusion Model INT4 (W4A4)", intro and "The part that actually
 * matters: mixed precision": every linear layer goes to 4 bit, the
 * activation between them stays in high precision).  GELU with the tanh
 * approximation is applied in the up-projection's epilogue, on the fp32
 * result after the bias and before the bf16 store:
 *   gelu(y) = 0.5 y (1 + tanhf(sqrt(2/pi) (y + 0.044715 y^3))),
 * so the down-projection's rotate + quantize reads the activated tensor
 * directly (no separate activation pass over [M, H]).
 * w4a4_gemm_gelu / w4a4_linear_gelu: as w4a4_gemm / w4a4_linear with the
 * fused activation.  w4a4_mlp: Y [M, D] = linear_down(gelu(linear_up(X))) for
 * X [M, D] bf16, up weights Wq_up [H, D/2] (+ scales, low-rank rank_up), down
 * weights Wq_down [D, H/2] (rank_down), one rotation group for both layers;
 * the workspace (w4a4_mlp_workspace_bytes, 256-byte aligned) holds both
 * layers' codes and scales, their low-rank T and the activated [M, H] bf16
 * tensor.  Shape and alignment rules are those of w4a4_linear for each
 * layer (D and H in the K and N roles); the first failing check's status is
 * returned. */
w4a4_status w4a4_gemm_gelu(const uint8_t* Xq, const float* x_scale, const uint8_t* Wq, const float* w_scale,
                           int M, int N, int K, int group, const void* T, const void* L2, int rank, const void* bias,
                           void* Y, int32_t* acc_debug, w4a4_stream_t stream);
w4a4_status w4a4_linear_gelu(const void* X, const uint8_t* Wq, const float* w_scale, int M, int N, int K,
                             int group, const void* L1, const void* L2, int rank, const void* bias, void* Y,
                             void* workspace, size_t workspace_bytes, w4a4_stream_t stream);
size_t w4a4_mlp_workspace_bytes(int M, int D, int H, int rank_up, int rank_down);
w4a4_status w4a4_mlp(const void* X, int M, int D, int H, int group, const uint8_t* Wq_up, const float* w_scale_up,
                     const void* L1_up, const void* L2_up, int rank_up, const void* bias_up, const uint8_t* Wq_down,
                     const float* w_scale_down, const void* L1_down, const void* L2_down, int rank_down,
                     const void* bias_down, void* Y, void* workspace, size_t workspace_bytes,
                     w4a4_stream_t stream);

/* ---------------------------------------------------------------- runtime LoRA */
/* A LoRA applied at run time beside the SVDQuant low-rank branch ("ComfyUI-
 * INT4-Fast", "INT4 Quantized Inference Comes to ComfyUI": LoRAs on top of
 * the 4-bit layers; "Krea 2 Turbo - SVDQuant", "What's included": the
 * low-rank branch beside the 4-bit product).  Writes the operands of one
 * combined branch of rank r + lora_rank:
 *   L1_out [K, r + lora_rank] = [L1 | A]            (bf16, row-major)
 *   L2_out [r + lora_rank, N] = [L2 ; bf16(fl32(lora_scale * B))]
 * so that w4a4_rotate_quantize_act / w4a4_gemm / w4a4_linear with these
 * operands and rank r + lora_rank compute
 *   dequant(acc) + (X L1) L2 + lora_scale (X A) B + bias
 * with a single epilogue low-rank MMA.  L1 [K, r], L2 [r, N] (may be NULL
 * when r == 0), A [K, lora_rank], B [lora_rank, N]: bf16, caller-owned
 * device memory, 16-byte aligned.  Shapes: r % 16 == 0, lora_rank >= 16 and
 * lora_rank % 16 == 0, r + lora_rank <= 256, N % 8 == 0.  Asynchronous on
 * `stream`; the outputs must not alias the inputs.  The pages give no
 * formula for the merge; this is the plainest reading (the scale folded into
 * the up matrix). */
w4a4_status w4a4_lora_merge(const void* L1, const void* L2, int rank, const void* A, const void* B, int lora_rank,
                            float lora_scale, int K, int N, void* L1_out, void* L2_out, w4a4_stream_t stream);

/* ---------------------------------------------------------------- LoRA baking */
/* Bakes a LoRA into the weights and re-quantizes them with stochastic
 * rounding ("ComfyUI-INT4-Fast", "INT4 Quantized Inference Comes to
 * ComfyUI", and "W4A4 and W4A8: The New Quantization Toolkit", "How the
 * toolkit tells you to choose": a LoRA can be merged into the 4-bit
 * weights; rounding stochastically keeps the small update in expectation).
 *   W_baked [N, K] = bf16(fl32(W + fl32(lora_scale * sum_j A[k][j] B[j][n])))
 * (fp32 fused multiply-adds over j in index order), then the W4A4 weight
 * routine (rotation, s = fl32(amax / 7) per row) with
 *   q = clamp(floor(fl32(fl32(y / s) + u)), -8, 7),
 * u in [0, 1) from Philox4x64-10 (Salmon et al., SC 2011): element e of the
 * row-major [N, K] codes uses word e % 4 of Philox(counter = (e / 4, 0, 0, 0),
 * key = (seed, 0)), top 24 bits times 2^-24.  W [N, K], A [K, lora_rank],
 * B [lora_rank, N]: bf16; W_baked (output, [N, K] bf16), Wq [N, K/2] and
 * w_scale [N] as w4a4_quantize_weights; 16-byte aligned device memory.
 * 1 <= lora_rank <= 256; K and group as w4a4_quantize_weights.  The result
 * is deterministic for a given seed. */
w4a4_status w4a4_bake_lora_sr(const void* W, const void* A, const void* B, int lora_rank, float lora_scale, int N,
                              int K, int group, unsigned long long seed, void* W_baked, uint8_t* Wq, float* w_scale,
                              w4a4_stream_t stream);

/* ---------------------------------------------------------------- planning */
/* Host-only view of how the rotate + quantize kernel is launched, for tools
 * and for testing the launch-plan caches from many host threads: no CUDA
 * call is made and nothing is launched.  Given M, K and group (rules as
 * w4a4_rotate_quantize_act), a device with `sms` SMs on which
 * `resident_per_sm` CTAs fit, writes shape[4] = {rows per block, threads per
 * CTA, dynamic shared memory bytes, grid size}.  cached != 0 goes through a
 * small shared plan cache (the same cache type the launchers use, guarded by
 * a mutex), cached == 0 computes the plan directly; both give the same
 * answer.  The pages have no counterpart. */
w4a4_status w4a4_plan_rotate_quantize(int M, int K, int group, int sms, int resident_per_sm, int cached,
                                      int* shape);

/* Host-only view of the GEMM's split-K decision (w4a4_gemm, w4a4_gemm_gelu
 * and w4a8_gemm, and the layers built on them): no CUDA call.  A layer whose
 * 256 x 256 output tiles are too few to give every pair of SMs one runs with
 * its K range split over a cluster of 2 x *split CTAs per tile, the int32
 * partials summed exactly through distributed shared memory.  Given M, N, K
 * (shape rules as w4a4_gemm with group 128), the low-rank rank (0 .. 256, a
 * multiple of 16), a device with `sms` SMs on which `clusters_of_8` clusters
 * of 8 CTAs and `clusters_of_4` of 4 (one CTA per SM) fit at once, writes
 * *split = 4, 2, or 1 for the persistent form.  The launchers make the same
 * decision with the device's own occupancy figures.  The pages have no
 * counterpart. */
w4a4_status w4a4_plan_gemm_split(int M, int N, int K, int rank, int sms, int clusters_of_8, int clusters_of_4,
                                 int* split);

/* ---------------------------------------------------------------- failures */
/* Kernels never trap: a wait on another part of the kernel that runs past its
 * time limit (2 s) records a code in a per-device error word and lets the
 * kernel finish.  This call synchronises `stream`, reads the word of the
 * current device into *code (may be NULL), clears it, and returns
 * W4A4_ERR_DEVICE_TIMEOUT when it was non-zero, W4A4_OK otherwise.  The code
 * is an OR of the W4A4_DEVERR_* bits below.  The pages describe no failure
 * handling for the kernels; this is the library's own. */
#define W4A4_DEVERR_WAIT_OPERANDS 1u /* a tensor-core issuer gave up waiting for its operands */
#define W4A4_DEVERR_WAIT_SLOT 2u     /* a producer gave up waiting for a free pipeline stage */
#define W4A4_DEVERR_WAIT_ACCUM 4u    /* an epilogue gave up waiting for its accumulator */
#define W4A4_DEVERR_WAIT_DRAIN 8u    /* the final drain of in-flight tensor-core work ran out */
w4a4_status w4a4_get_device_error(w4a4_stream_t stream, unsigned int* code);

/* Self-test of the bounded waits, for callers that want to see the failure
 * path work on their device without faulting it.  Launches the low-rank
 * down-projection of w4a4_rotate_quantize_act (X bf16 [M, K], L1 bf16
 * [K, rank], T out bf16 [M, rank]; shape and alignment rules as there, rank
 * > 0) with its operand producer withholding every load and the operand wait
 * limited to timeout_us microseconds (1 .. 1000000).  The tensor-core issuer's
 * first wait then runs out: no copy or MMA is in flight when it gives up, the
 * kernel finishes normally, T is left undefined, and the device error word
 * afterwards holds W4A4_DEVERR_WAIT_OPERANDS (w4a4_get_device_error returns
 * W4A4_ERR_DEVICE_TIMEOUT and clears it).  Later calls are unaffected. */
w4a4_status w4a4_selftest_wait_timeout(const void* X, const void* L1, int M, int K, int rank, void* T,
                                       unsigned int timeout_us, w4a4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* W4A4_H_ */
