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
// Work decomposition: a cluster of two CTAs (one per SM of a TPC) owns a
// 256 x 256 output tile and issues the pair form of the MMA (cta_group::2):
// each CTA holds 128 rows of A, 128 rows (N) of B and its 128 x 256 int32
// accumulator.  Per CTA (k-block = 128 codes):
//   warp 16     TMA: packed A and B tiles (64-byte rows, 64-byte swizzle)
//               into a shared-memory ring (no multicast), and per tile the
//               low-rank operand tiles T and L2;
//   warps 0-15  four sets of four warps; set s widens the k-blocks
//               g = s (mod 4).  Each thread takes one A row and one B row
//               (conflict-free 16-byte reads): A is tcgen05.st into a TMEM
//               ring (the MMA reads A from tensor memory), B is stored into
//               a ring in the 128-byte-swizzled K-major layout the MMA reads
//               from shared memory.  Each widen is a chain of shared-memory
//               round trips (stage barrier, loads, release, free-slot
//               barrier, stores, hand-off), so four chains in flight per CTA
//               keep pace with the MMAs where two did not;
//   warp 17     (even CTA) one thread issues the pair MMAs and commits each
//               stage to the barriers of both CTAs; (odd CTA) relays the
//               arrival of TMA-only operands to the even CTA.
//   warp 18     (even CTA) polls the stage barriers and releases each stage
//               to warp 17 through a named barrier: the issuing warp never
//               reads shared memory, which would stall it behind its own
//               queued MMAs and leave the tensor pipe idle between stages.
//   warps 0-15  epilogue: tcgen05.ld, dequant, low-rank, bias, bf16 TMA
//               stores.
// The kernel is persistent: one pair per TPC walks its output tiles, and the
// TMA and widen stages run ahead into the next tile while the epilogue of the
// current one drains the accumulator (layers with too few tiles use the
// split-K form described at the kernel instead).  With a low-rank branch the tile stays
// 256 x 256 and TMEM holds no second accumulator: the epilogue rewrites the
// int32 accumulator in place as fp32 (acc s_a) s_w', bf16 MMAs accumulate
// T L2 onto it (operand chunks of 128 ranks staged by TMA), and a second read
// adds the bias; bf16 tiles leave via TMA stores staged in the operand buffer.
// The INT8 path skips the widening: TMA writes both operands straight into
// the 128-byte-swizzled layout and the MMA reads both from shared memory.
// Every mbarrier wait is bounded; on timeout the kernel records an error in
// the device error word and runs to completion without trapping.
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

constexpr int BM = 128;          // A rows per CTA; the pair covers 256
constexpr int BK = 128;          // codes per k-block
constexpr int kThreads = 608;    // 19 warps
constexpr int kTmaWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kWaitWarp = 18;
constexpr int kIssueBar = 2;     // named barrier: MMA warp + waiter warp
constexpr int kSets = 4;         // widen sets; set s widens the k-blocks g = s (mod kSets)
constexpr int kSetWarps = 4;     // warps per set: one A row and one B row per thread
constexpr int S8 = 5;            // INT8 TMA stages
constexpr int LRC = 128;         // low-rank rank chunk per MMA round
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;  // int32 accumulator
constexpr uint32_t kACol0 = 256; // A ring: 32 columns per stage
constexpr int kStageTile = 32 * 32 * 2;            // epilogue staging tile: 32 x 32 bf16
constexpr int kOutStageBytes = 16 * kStageTile;    // one per epilogue warp
constexpr int kBarBytes = 512;
constexpr int kPartPitch = 256 * 4 + 16;           // split-K: int32 partial row pitch (bank-spread)
constexpr int kL2fOff = 128 * kPartPitch;          // split-K: fp32 L2 slice after the partials (ring area)
constexpr int kSplitMaxRank = 32;                  // split-K: largest low-rank term (CUDA cores, reduction)
constexpr int kSplitTOff = 8192;                   // split-K: T rows after the bf16 L2 slice (staging area)
constexpr int kSplitSwOff = BM * 4;                // split-K vector area: row scales, column scales, bias
constexpr int kSplitBiasOff = kSplitSwOff + 128 * 4;

// MODE 0: W8A8 (int8 x int8, TMA straight into the MMA layout); 1: W4A4
// (packed INT4 x packed INT4, both widened, A into TMEM); 2: W4A8 (the int8
// activation tile is read by the MMA straight from its own TMA ring, freed by
// the MMA commit; packed unsigned 4-bit weights are widened with their zero
// point subtracted and their packed stages are freed by the widen warps).
template <int MODE, bool LR>
struct Cfg {
  static constexpr bool PACKED = MODE != 0;          // the widen pipeline runs
  static constexpr int PS = 4;                      // packed TMA stages (W4A4: A + B; W4A8: B), kSets apart
  static constexpr int US = MODE == 2 ? 4 : (LR ? 5 : 7);  // widened stages (W4A8: B only)
  static constexpr int AS = MODE == 2 ? 5 : 0;       // W4A8: int8 A stages, read by the MMA in place
  static constexpr int kLead = US - 2;               // k-blocks widened ahead of an epilogue
  static constexpr int BN = 256;                     // N per pair tile
  static constexpr int BNH = BN / 2;                 // B rows staged per CTA
  static constexpr int kARow = MODE == 2 ? BK : BK / 2;  // bytes of an A row per k-block
  static constexpr int kPkA = MODE == 1 ? BM * kARow : 0;  // packed A in the packed stage (W4A4 only)
  static constexpr int kPkB = BNH * BK / 2;
  static constexpr int kPkStage = kPkA + kPkB;
  static constexpr int kWideB = BNH * BK;            // widened B stage
  static constexpr int kI8A = BM * BK;               // INT8 stages
  static constexpr int kI8B = BNH * BK;
  static constexpr int kI8Stage = kI8A + kI8B;
  static constexpr int kRing = PACKED ? PS * kPkStage + US * kWideB + AS * kI8A : S8 * kI8Stage;
  static constexpr int kWOff = PS * kPkStage;        // widened B ring
  static constexpr int kAOff = kWOff + US * kWideB;  // W4A8 int8 A ring
  static constexpr int kLrT = BM * LRC * 2;          // T chunk: 128 rows x 128 ranks, two 64-wide boxes
  static constexpr int kLrL2 = BNH * LRC * 2;        // L2 chunk: 128 ranks x BNH columns, two 64-wide boxes
  static constexpr int kLrBytes = LR ? kLrT + kLrL2 : 0;
  static constexpr int kVecBytes = 2 * 2 * BN * 4;   // scales + bias, two tiles
  static constexpr int kLrOff = kRing;
  static constexpr int kOutOff = kLrOff + kLrBytes;
  // the low-rank form stages its bf16 tiles in the operand buffer, free once
  // the tile's low-rank MMAs have completed
  static constexpr int kOutBytes = LR ? 0 : kOutStageBytes;
  static constexpr int kStageOff = LR ? kLrOff : kOutOff;
  static constexpr int kVecOff = kOutOff + kOutBytes;
  static constexpr int kDataBytes = kVecOff + kVecBytes;
  static constexpr int kSmemBytes = kDataBytes + kBarBytes + 1024;
  static constexpr int kColsPerWarp = BN / 4;        // epilogue: 4 warps per TMEM lane quadrant
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kACol0 + US * (BK / 4) <= kTmemCols, "TMEM budget");
  static_assert(PS <= 8 && US <= 8, "barrier arrays");
  // set s waits on every fill of its own packed stages (g = s mod kSets), in
  // order, so a phase-parity wait can never match a fill two phases old
  static_assert(PS % kSets == 0, "each widen set owns its packed stages");
  static_assert(US >= kSets && kLead >= 1, "widened ring");
  // W4A8: the kLead k-blocks widened ahead of an epilogue also need their
  // int8 A tiles; slot g + kLead - 1 frees only once the MMAs have read
  // k-block g + kLead - 1 - AS, which must belong to the finished tile (else
  // the epilogue, the MMAs and the A loads wait on one another)
  static_assert(MODE != 2 || kLead <= AS, "W4A8: A ring deeper than the k-blocks widened ahead");
  static_assert(kWOff % 1024 == 0 && kAOff % 1024 == 0, "128-byte swizzle atoms");
  static_assert(kWOff + US * kWideB <= kRing && (MODE != 2 || kAOff + AS * kI8A <= kRing), "rings inside the ring area");
  static_assert(!LR || MODE == 1, "low-rank branch: W4A4 only");
  static_assert(!LR || kOutStageBytes <= kLrBytes, "epilogue staging inside the low-rank buffer");
};

struct Params {
  GemmArgs a;
  unsigned int* err;
  int split;   // split-K form: K slices (pairs per cluster), else 1
};

struct Barriers {
  uint64_t tma_full[8];
  uint64_t tma_empty[8];
  uint64_t full[8];      // even CTA: a stage is complete in both CTAs
  uint64_t empty[8];
  uint64_t conv;         // even CTA: both CTAs' epilogues turned the accumulator into fp32
  uint64_t lr_done;      // the low-rank MMAs of the tile completed
  uint64_t lr_full;      // this CTA's low-rank chunk landed (TMA)
  uint64_t lr_ready;     // even CTA: the odd CTA's low-rank chunk landed (relay)
  uint64_t lr_empty;     // the low-rank MMAs of a chunk (not the tile's last) completed
  uint64_t lr_free;      // the epilogue's stores staged in the low-rank buffer have been read
  uint64_t acc_full;
  uint64_t acc_empty;    // even CTA: both CTAs' epilogues have read the accumulators
  uint64_t a_full[8];    // W4A8: this CTA's int8 A stage landed (TMA)
  uint64_t a_empty[8];   // W4A8: the MMAs reading an A stage completed
  uint64_t drain;
  uint32_t tmem_base;
};
static_assert(sizeof(Barriers) <= kBarBytes, "barrier block");

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ uint2 ld_shared_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
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

// 16 packed bytes (32 unsigned codes u, u_0 in the low nibble) -> 32 bytes
// u_k - z in natural k order, as int8.  zk = 0x80808080 - z * 0x01010101:
// each byte u + 128 - z lies in [113, 143], so the 32-bit add carries no byte
// into the next, and flipping bit 7 turns u - z + 128 into u - z in two's
// complement.
__device__ __forceinline__ uint32_t sub_zero4(uint32_t x, uint32_t zk) { return (x + zk) ^ 0x80808080u; }
__device__ __forceinline__ void widen_word_zp(uint32_t w, uint32_t zk, uint32_t& o0, uint32_t& o1) {
  const uint32_t ev = w & 0x0F0F0F0Fu;          // u0 u2 u4 u6
  const uint32_t od = (w >> 4) & 0x0F0F0F0Fu;   // u1 u3 u5 u7
  o0 = sub_zero4(__byte_perm(ev, od, 0x5140), zk);  // u0 u1 u2 u3
  o1 = sub_zero4(__byte_perm(ev, od, 0x7362), zk);  // u4 u5 u6 u7
}
__device__ __forceinline__ void widen16_zero_point(const uint4 p, uint32_t zk, uint4& c0, uint4& c1) {
  widen_word_zp(p.x, zk, c0.x, c0.y);
  widen_word_zp(p.y, zk, c0.z, c0.w);
  widen_word_zp(p.z, zk, c1.x, c1.y);
  widen_word_zp(p.w, zk, c1.z, c1.w);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// int32 accumulator -> float.  W4A4 products carry a factor 2^8; after the
// shift |t| <= 64 K <= 2^21, so t is recovered exactly from the mantissa of
// 1.5 * 2^23 + t (two full-rate ALU operations instead of a conversion-unit
// I2F).  W8A8 and W4A8 accumulators can exceed 2^22 and are rounded by I2F.
template <bool SHIFTED>
__device__ __forceinline__ float acc_to_float(uint32_t v) {
  if constexpr (SHIFTED) {
    const int t = static_cast<int>(v) >> 8;
    return __fsub_rn(__int_as_float(t + 0x4B400000), 12582912.0f);
  } else {
    return __int2float_rn(static_cast<int>(v));
  }
}

// GELU with the tanh approximation (fused MLP up-projection), fp32.
__device__ __forceinline__ float gelu_tanh(float x) {
  const float c = 0.7978845608028654f;   // sqrt(2 / pi)
  const float u = c * (x + 0.044715f * (x * x * x));
  return 0.5f * x * (1.0f + tanhf(u));
}

// SPLIT 1 (W4A4 or W4A8) or 2 (W4A4 with a small low-rank branch, its term
// added in the reduction): a cluster of prm.split pairs shares one 256 x 256
// tile; pair q accumulates the k-blocks [q nk / split, (q + 1) nk / split),
// every CTA leaves its int32 partial in shared memory, and after a cluster
// barrier CTA (q, half) sums column slice q of its half over all pairs
// (exact integer sums, in pair order) and runs the epilogue on it.  For
// layers with too few tiles to occupy the GPU.
template <int MODE, bool LR, bool ACT, int SPLIT = 0>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const Params prm, const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmT,
                const __grid_constant__ CUtensorMap tmL2) {
  using C = Cfg<MODE, LR>;
  constexpr bool PACKED = C::PACKED;
  constexpr int PS = C::PS;
  constexpr int US = C::US;
  constexpr int BN = C::BN;
  constexpr int BNH = C::BNH;
  const GemmArgs& p = prm.a;
  constexpr int kShift = MODE == 1 ? 8 : 0;  // W4A4 widened products carry 2^8
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  Barriers* bar = reinterpret_cast<Barriers*>(smem_raw + (sbase - raw) + C::kDataBytes);

  static_assert(!SPLIT || (MODE != 0 && !LR && (SPLIT == 1 || MODE == 1)),
                "split-K form: W4A4 (with the low-rank term in the reduction) or W4A8");
  static_assert(!SPLIT || BM * kPartPitch <= C::kRing, "split-K partial inside the ring area");
  // split-K operands of the reduction: the fp32 L2 slice (<= 32 ranks x 128
  // columns) after the partials; the bf16 slice and T rows in the epilogue
  // staging area, idle in this form; scales and bias in the vector area
  static_assert(!SPLIT || kL2fOff + kSplitMaxRank * 128 * 4 <= C::kRing, "split-K fp32 L2 slice in the ring area");
  static_assert(!SPLIT || (kSplitMaxRank * 128 * 2 <= kSplitTOff &&
                           kSplitTOff + BM * (2 * kSplitMaxRank + 16) <= C::kOutBytes),
                "split-K bf16 L2 slice and T rows in the staging area");
  static_assert(!SPLIT || kSplitBiasOff + 128 * 2 <= C::kVecBytes, "split-K scales and bias in the vector area");
  static_assert(!SPLIT || BM / 4 + 128 / 4 + 128 / 8 <= 16 * 32, "split-K: one vector copy per epilogue thread");
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t rank = SPLIT ? (crank & 1u) : crank;      // CTA within its pair
  const uint32_t pbase = SPLIT ? (crank & ~1u) : 0u;       // the pair's even CTA in the cluster
  const uint16_t pmask = (uint16_t)(0x3u << pbase);        // both CTAs of the pair
  const bool leader = rank == 0;
  const int n_tiles = (p.N + BN - 1) / BN;
  const int total_tiles = ((p.M + 2 * BM - 1) / (2 * BM)) * n_tiles;
  const int pair0 = SPLIT ? (int)(blockIdx.x / (2 * prm.split)) : (int)(blockIdx.x >> 1);
  const int pair_stride = SPLIT ? total_tiles : (int)(gridDim.x >> 1);
  const int my_tiles = pair0 < total_tiles ? (total_tiles - pair0 + pair_stride - 1) / pair_stride : 0;
  // k-blocks of this pair: all of them, or its slice in the split-K form
  const int kb0 = SPLIT ? (int)(crank >> 1) * (p.K / BK) / prm.split : 0;
  const int nk = SPLIT ? ((int)(crank >> 1) + 1) * (p.K / BK) / prm.split - kb0 : p.K / BK;
  const int lr_chunks = LR ? (p.rank + LRC - 1) / LRC : 0;
  // tile i of this pair (i < my_tiles): this CTA's rows, the pair's columns
  auto tile_m = [&](int i) { return ((pair0 + i * pair_stride) / n_tiles) * (2 * BM) + (int)rank * BM; };
  auto tile_n = [&](int i) { return ((pair0 + i * pair_stride) % n_tiles) * BN; };

  if (warp == kTmaWarp) {
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      if constexpr (SPLIT != 0 || MODE == 2) {
        // the weight tiles of this CTA's first k-blocks into L2 while the
        // previous kernel finishes (a hint only: the loads after the
        // dependency wait read the weights as that kernel left them).  Not in
        // the persistent W4A4 forms, where the extra code costs spills.
        if (my_tiles > 0) {
          const int row_b = tile_n(0) + (int)rank * BNH;
          for (int kb = 0; kb < min(PS, nk); ++kb) prefetch_tile_l2(&tmB, (kb0 + kb) * (PACKED ? BK / 2 : BK), row_b);
        }
      }
      prefetch_tmap(&tmY);
      if (LR) {
        prefetch_tmap(&tmT);
        prefetch_tmap(&tmL2);
      }
      for (int s = 0; s < 8; ++s) {
        mbar_init(&bar->tma_full[s], 1);
        // packed modes: the 4 widen warps of a set read the stage; W8A8: the
        // MMA commit
        mbar_init(&bar->tma_empty[s], PACKED ? kSetWarps : 1);
        mbar_init(&bar->a_full[s], 1);
        mbar_init(&bar->a_empty[s], 1);
        mbar_init(&bar->full[s], PACKED ? 2 * kSetWarps : 1);  // a set's warps in both CTAs, or 1 relay
        mbar_init(&bar->empty[s], 1);
      }
      mbar_init(&bar->conv, 32);       // 16 epilogue warps per CTA
      mbar_init(&bar->lr_done, 1);
      mbar_init(&bar->lr_full, 1);
      mbar_init(&bar->lr_ready, 1);
      mbar_init(&bar->lr_empty, 1);
      mbar_init(&bar->lr_free, 16);     // 16 epilogue warps of this CTA
      mbar_init(&bar->acc_full, 1);
      mbar_init(&bar->acc_empty, 32);  // 16 epilogue warps per CTA
      mbar_init(&bar->drain, 1);
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc_pair(&bar->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const int total_kb = my_tiles * nk;
  // everything above overlaps the tail of the kernel producing the codes
  grid_dependency_wait();

  if (warp == kTmaWarp) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      constexpr int NS = PACKED ? PS : S8;
      constexpr int kStageBytes = PACKED ? C::kPkStage : C::kI8Stage;
      constexpr int kABytes = PACKED ? C::kPkA : C::kI8A;
      int as = 0;            // W4A8: A ring slot and phase
      uint32_t a_ph = 0;
      constexpr int kColA = PACKED ? C::kARow : BK;   // bytes per k-block of an A / B row
      constexpr int kColB = PACKED ? BK / 2 : BK;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      // Low-rank operand chunks (T rows: K-major, two 64-rank boxes; L2
      // columns: N-major, two 64-column boxes) go through one buffer, in
      // order: load q = tile * lr_chunks + chunk.  A load becomes eligible
      // once its tile's k-blocks are half issued and goes out as soon as the
      // buffer is free; this thread never blocks on the buffer while k-block
      // loads remain, since freeing it can depend (through the epilogue) on
      // widening k-blocks still to be loaded.
      const int lr_total = my_tiles * lr_chunks;
      int lr_n = 0, lr_eligible = 0;
      auto issue_lr = [&]() {
        const int per_tile = max(lr_chunks, 1);
        const int ti = lr_n / per_tile, c = lr_n - ti * per_tile;
        const uint32_t lr = sbase + (uint32_t)C::kLrOff;
        const int ra = tile_m(ti), rb = tile_n(ti) + (int)rank * BNH;
        const bool second = p.rank - c * LRC > 64;   // ranks past 64 in this chunk
        mbar_arrive_expect_tx(&bar->lr_full, (uint32_t)((second ? C::kLrT : C::kLrT / 2) + C::kLrL2));
        tma_load_2d(lr, &tmT, c * LRC, ra, &bar->lr_full);
        if (second) tma_load_2d(lr + C::kLrT / 2, &tmT, c * LRC + 64, ra, &bar->lr_full);
        tma_load_2d(lr + C::kLrT, &tmL2, rb, c * LRC, &bar->lr_full);
        tma_load_2d(lr + C::kLrT + C::kLrL2 / 2, &tmL2, rb + 64, c * LRC, &bar->lr_full);
        ++lr_n;
      };
      // the buffer is free for load q: after the previous chunk's MMAs (same
      // tile) or after the previous tile's epilogue stores read their staging
      auto lr_buffer_free = [&](bool block) -> bool {
        const int per_tile = max(lr_chunks, 1);
        const int ti = lr_n / per_tile, c = lr_n - ti * per_tile;
        if (c == 0 && ti == 0) return true;
        uint64_t* b = c == 0 ? &bar->lr_free : &bar->lr_empty;
        const uint32_t parity = (uint32_t)(c == 0 ? ti - 1 : ti * (per_tile - 1) + c - 1) & 1u;
        return block ? mbar_wait(b, parity) : mbar_try_wait(b, parity);
      };
      auto lr_ready_now = [&]() { return LR && lr_n < lr_eligible && lr_buffer_free(false); };
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int row_a = tile_m(i);
        const int row_b = tile_n(i) + (int)rank * BNH;
        for (int kb = 0; kb < nk; ++kb) {
          // wait for the stage, issuing any low-rank load that is due
          bool got = false;
          const unsigned long long t0 = globaltimer_ns();
          for (uint32_t it = 0;; ++it) {
            if (lr_ready_now()) issue_lr();
            if (mbar_try_wait(&bar->tma_empty[s], ph ^ 1u)) {
              got = true;
              break;
            }
            if ((it & 255u) == 255u && globaltimer_ns() - t0 > kWaitTimeoutNs) break;
          }
          if (!got) {
            set_device_error(prm.err, kDevErrTimeoutEmpty);
            ok = false;
            break;
          }
          const uint32_t dst = sbase + (uint32_t)(s * kStageBytes);
          mbar_arrive_expect_tx(&bar->tma_full[s], (uint32_t)kStageBytes);
          if (MODE != 2) tma_load_2d(dst, &tmA, (kb0 + kb) * kColA, row_a, &bar->tma_full[s]);
          tma_load_2d(dst + kABytes, &tmB, (kb0 + kb) * kColB, row_b, &bar->tma_full[s]);
          if (++s == NS) { s = 0; ph ^= 1u; }
          if constexpr (MODE == 2) {
            // the int8 A tile into its own ring, once the MMAs have freed the slot
            if (!mbar_wait(&bar->a_empty[as], a_ph ^ 1u)) {
              set_device_error(prm.err, kDevErrTimeoutEmpty);
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bar->a_full[as], (uint32_t)C::kI8A);
            tma_load_2d(sbase + (uint32_t)(C::kAOff + as * C::kI8A), &tmA, (kb0 + kb) * BK, row_a,
                        &bar->a_full[as]);
            if (++as == C::AS) { as = 0; a_ph ^= 1u; }
          }
          if (LR && kb == nk / 2) lr_eligible = (i + 1) * lr_chunks;
        }
      }
      // the remaining low-rank loads (no k-block load is left to wait for)
      while (LR && ok && lr_n < lr_total) {
        if (!lr_buffer_free(true)) {
          set_device_error(prm.err, kDevErrTimeoutEmpty);
          break;
        }
        issue_lr();
      }
    }
  } else if (warp == kMmaWarp) {
    if (!leader && lane == 0) {
      // relay: tell the even CTA when this CTA's TMA-only operands have landed
      int s = 0, lr_n = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        if (!PACKED) {
          for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait(&bar->tma_full[s], ph)) {
              set_device_error(prm.err, kDevErrTimeoutFull);
              ok = false;
              break;
            }
            mbar_arrive_remote(&bar->full[s], pbase);
            if (++s == S8) { s = 0; ph ^= 1u; }
          }
        }
        for (int c = 0; c < lr_chunks && ok; ++c, ++lr_n) {
          if (!mbar_wait(&bar->lr_full, (uint32_t)lr_n & 1u)) {
            set_device_error(prm.err, kDevErrTimeoutFull);
            ok = false;
            break;
          }
          mbar_arrive_remote(&bar->lr_ready, pbase);
        }
      }
    }
    if (leader) {
      // ---------------------------------------------------------------- MMA
      // The whole warp walks the stages; lane 0 issues.  This warp never
      // polls an mbarrier: a shared-memory read here would queue behind the
      // MMAs already issued and leave the tensor pipe idle between stages.
      // The waiter warp polls the barriers and releases each stage through
      // a named barrier (bar.red also carries its timeout flag).
      constexpr uint32_t idesc = idesc_i8(2 * BM, BN);
      constexpr uint32_t idesc_lr = idesc_bf16(2 * BM, BN, false, true);
      constexpr int NS = PACKED ? US : S8;
      int s = 0, ps = 0;   // widened stage / TMA stage of the k-block (W4A8: A ring slot)
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        for (int kb = 0; kb < nk; ++kb) {
          if (named_barrier_or(kIssueBar, 64, false)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            if (MODE == 1) {
              const uint32_t b_stage = sbase + (uint32_t)(C::kWOff + s * C::kWideB);
#pragma unroll
              for (int ks = 0; ks < BK / 32; ++ks)
                mma_i8_ts_pair(tmem + kAccCol, tmem + kACol0 + (uint32_t)(s * (BK / 4) + ks * 8),
                               smem_desc_kmajor_sw128(b_stage + (uint32_t)(ks * 32)), idesc,
                               (kb | ks) != 0 ? 1u : 0u);
              tc_commit_pair_mc(&bar->empty[s], pmask);
            } else if (MODE == 2) {
              const uint32_t a_stage = sbase + (uint32_t)(C::kAOff + ps * C::kI8A);
              const uint32_t b_stage = sbase + (uint32_t)(C::kWOff + s * C::kWideB);
#pragma unroll
              for (int ks = 0; ks < BK / 32; ++ks)
                mma_i8_ss_pair(tmem + kAccCol, smem_desc_kmajor_sw128(a_stage + (uint32_t)(ks * 32)),
                               smem_desc_kmajor_sw128(b_stage + (uint32_t)(ks * 32)), idesc,
                               (kb | ks) != 0 ? 1u : 0u);
              tc_commit_pair_mc(&bar->empty[s], pmask);
              tc_commit_pair_mc(&bar->a_empty[ps], pmask);
            } else {
              const uint32_t a_stage = sbase + (uint32_t)(s * C::kI8Stage);
#pragma unroll
              for (int ks = 0; ks < BK / 32; ++ks)
                mma_i8_ss_pair(tmem + kAccCol, smem_desc_kmajor_sw128(a_stage + (uint32_t)(ks * 32)),
                               smem_desc_kmajor_sw128(a_stage + C::kI8A + (uint32_t)(ks * 32)), idesc,
                               (kb | ks) != 0 ? 1u : 0u);
              tc_commit_pair_mc(&bar->tma_empty[s], pmask);
            }
          }
          __syncwarp();
          if (++s == NS) s = 0;
          if (++ps == (MODE == 2 ? C::AS : PS)) ps = 0;
        }
        // the integer product of the tile is complete
        if (ok && lane == 0) tc_commit_pair_mc(&bar->acc_full, pmask);
        __syncwarp();
        if (LR) {
          // Once both epilogues have rewritten the accumulator as fp32
          // ((acc s_a) s_w' in place), T L2 accumulates onto it: A = T
          // (K-major, 128-byte swizzle, k-step 16 ranks = 32 bytes), B = L2
          // (N-major, 128-byte swizzle, two 64-column atoms 16 KB apart,
          // k-step 16 ranks = two 8-row groups)
          for (int c = 0; c < lr_chunks && ok; ++c) {
            if (named_barrier_or(kIssueBar, 64, false)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (lane == 0) {
              const uint32_t lr = sbase + (uint32_t)C::kLrOff;
              const int ksteps = min(LRC, p.rank - c * LRC) / 16;
              for (int ks = 0; ks < ksteps; ++ks) {
                const uint32_t a_addr = lr + (uint32_t)((ks >> 2) * (C::kLrT / 2) + (ks & 3) * 32);
                const uint32_t b_addr = lr + (uint32_t)(C::kLrT + ks * 2048);
                mma_bf16_ss_pair(tmem + kAccCol, smem_desc_kmajor_sw128(a_addr),
                                 smem_desc_mnmajor_sw128(b_addr, (uint32_t)(C::kLrL2 / 2), 1024), idesc_lr, 1u);
              }
              if (c + 1 < lr_chunks) tc_commit_pair_mc(&bar->lr_empty, pmask);
            }
            __syncwarp();
          }
          if (ok && lane == 0) tc_commit_pair_mc(&bar->lr_done, pmask);
        }
        __syncwarp();
      }
      // drain: every MMA issued so far has completed before teardown
      if (lane == 0) {
        tc_commit_pair_mc(&bar->drain, (uint16_t)(0x1u << pbase));
        if (!mbar_wait(&bar->drain, 0)) set_device_error(prm.err, kDevErrTimeoutDrain);
      }
      __syncwarp();
    }
  } else if (warp == kWaitWarp) {
    if (leader) {
      // ------------------------------------------------------------- waiter
      // Polls, in the issuer's order, every barrier an MMA stage depends on
      // and releases the stage to the issuer warp through the named barrier.
      constexpr int NS = PACKED ? US : S8;
      int s = 0, lr_n = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        for (int kb = 0; kb < nk; ++kb) {
          // the accumulators are free once both CTAs' epilogues have read tile i-1
          bool late = kb == 0 && i > 0 && !mbar_wait(&bar->acc_empty, (uint32_t)(i - 1) & 1u);
          if (late) {
            if (lane == 0) set_device_error(prm.err, kDevErrTimeoutAcc);
          } else if (PACKED ? !mbar_wait(&bar->full[s], ph)
                            : (!mbar_wait(&bar->tma_full[s], ph) || !mbar_wait(&bar->full[s], ph))) {
            late = true;
            if (lane == 0) set_device_error(prm.err, kDevErrTimeoutFull);
          }
          if (named_barrier_or(kIssueBar, 64, late)) {
            ok = false;
            break;
          }
          if (++s == NS) { s = 0; ph ^= 1u; }
        }
        for (int c = 0; c < lr_chunks && ok; ++c, ++lr_n) {
          // before the first chunk: both epilogues have converted the accumulator
          const bool late = (c == 0 && !mbar_wait(&bar->conv, (uint32_t)i & 1u)) ||
                            !mbar_wait(&bar->lr_full, (uint32_t)lr_n & 1u) ||
                            !mbar_wait(&bar->lr_ready, (uint32_t)lr_n & 1u);
          if (late && lane == 0) set_device_error(prm.err, kDevErrTimeoutFull);
          if (named_barrier_or(kIssueBar, 64, late)) {
            ok = false;
            break;
          }
        }
      }
    }
  } else if (warp < 16) {
    // ------------------------------------------------ widen (INT4) + epilogue
    // four sets of four warps; set s widens the k-blocks g = s (mod 4), so
    // that each warp has four MMA k-blocks of time per widen.  All 16 run
    // the epilogue.
    const int set = warp >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;                   // A row and B row within this CTA's tile
    const bool has_b = r < BNH;                       // warp-uniform
    constexpr bool kWidenA = MODE == 1;               // W4A8 reads int8 A straight from the stage

    // widen k-block g: this thread's A row into TMEM and its B row into the
    // widened shared-memory ring
    auto widen = [&](int g) -> bool {
      const int ps = g % PS;
      const int u = g % US;
      if (!mbar_wait(&bar->tma_full[ps], (uint32_t)(g / PS) & 1u)) {
        set_device_error(prm.err, kDevErrTimeoutFull);
        return false;
      }
      const uint32_t stage = sbase + (uint32_t)(ps * C::kPkStage) + (uint32_t)(r * (BK / 2));
      const uint32_t rsw = (uint32_t)((r >> 1) & 3);
      uint4 pa[4], pb[4];
      uint32_t seen = 0;
      if (kWidenA) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          pa[c] = ld_shared_v4(stage + ((((uint32_t)c) ^ rsw) << 4));
          seen ^= pa[c].x ^ pa[c].y ^ pa[c].z ^ pa[c].w;
        }
      }
      if (has_b) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          pb[c] = ld_shared_v4(stage + (uint32_t)C::kPkA + ((((uint32_t)c) ^ rsw) << 4));
          seen ^= pb[c].x ^ pb[c].y ^ pb[c].z ^ pb[c].w;
        }
      }
      // Hand the packed stage back to TMA only once every lane's loads have
      // returned: the arrive is made data-dependent on all loaded words (an
      // mbarrier arrive by itself does not wait for this warp's outstanding
      // shared-memory loads, and the next bulk copy into the stage would
      // overwrite data not yet read).  Exactly one lane arrives whatever the
      // value.
      seen = __reduce_or_sync(0xffffffffu, seen);
      if (lane == (seen == 0x9E3779B9u ? 1 : 0)) mbar_arrive(&bar->tma_empty[ps]);
      if (!mbar_wait(&bar->empty[u], ((uint32_t)(g / US) & 1u) ^ 1u)) {
        set_device_error(prm.err, kDevErrTimeoutEmpty);
        return false;
      }
      tc_fence_after();
      if (kWidenA) {
        uint32_t regs[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 c0, c1;
          widen16(pa[c], c0, c1);
          regs[8 * c + 0] = c0.x; regs[8 * c + 1] = c0.y; regs[8 * c + 2] = c0.z; regs[8 * c + 3] = c0.w;
          regs[8 * c + 4] = c1.x; regs[8 * c + 5] = c1.y; regs[8 * c + 6] = c1.z; regs[8 * c + 7] = c1.w;
        }
        tmem_st_32x32b_x32(tmem + ((uint32_t)(quad * 32) << 16) + kACol0 + (uint32_t)(u * (BK / 4)), regs);
      }
      if (has_b) {
        const uint32_t row =
            sbase + (uint32_t)(C::kWOff + u * C::kWideB + (r >> 3) * 1024 + (r & 7) * 128);
        const uint32_t rsw128 = (uint32_t)(r & 7);
        uint32_t zk = 0;
        if constexpr (MODE == 2) {
          // zero point of this weight row, as the per-byte bias 128 - z
          const int n = tile_n(g / nk) + (int)rank * BNH + r;
          const uint32_t z = n < p.N ? (uint32_t)__ldg(p.w_zero + n) : 0u;
          zk = 0x80808080u - z * 0x01010101u;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 c0, c1;
          if constexpr (MODE == 2)
            widen16_zero_point(pb[c], zk, c0, c1);
          else
            widen16(pb[c], c0, c1);
          st_shared_v4(row + ((((uint32_t)(2 * c)) ^ rsw128) << 4), c0);
          st_shared_v4(row + ((((uint32_t)(2 * c + 1)) ^ rsw128) << 4), c1);
        }
        fence_proxy_async_smem();
      }
      if (kWidenA) {
        tmem_wait_st();
        tc_fence_before();
      }
      if constexpr (MODE == 2) {
        // the k-block also needs this CTA's int8 A tile: the hand-off below
        // then tells the issuer that A and B have landed in this CTA
        if (!mbar_wait(&bar->a_full[g % C::AS], (uint32_t)(g / C::AS) & 1u)) {
          set_device_error(prm.err, kDevErrTimeoutFull);
          return false;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(&bar->full[u], pbase);
      return true;
    };

    // epilogue of tile i: each of the 16 warps drains its TMEM lane quadrant's
    // share of the accumulator columns (64) into registers, releases the
    // accumulator to the next tile's MMAs, then dequantizes, adds the bias and
    // writes bf16 through TMA stores.  With a low-rank branch it first writes
    // (acc s_a) s_w' back in place as fp32 and waits for the low-rank MMAs to
    // add T L2 onto it before the final read.
    const int cq = warp >> 2;                         // column quarter
    const uint32_t stage_out = sbase + (uint32_t)(C::kStageOff + warp * kStageTile);
    float* vec_base = reinterpret_cast<float*>(smem_raw + (sbase - raw) + C::kVecOff);
    const uint32_t sw64 = (uint32_t)((lane >> 1) & 3);
    auto epilogue = [&](int i) {
      const int m_row0 = tile_m(i) + quad * 32;
      const int n_pair = tile_n(i);
      float* s_sw = vec_base + (i & 1) * 2 * BN;   // double-buffered by tile parity
      float* s_bias = s_sw + BN;
      if (threadIdx.x < BN) {
        const int j = threadIdx.x;
        const int n = n_pair + j;
        // 1/g is a power of two: folding it into the column scale is exact
        // (s_w / g stays a normal float for any scale above 2^-119)
        s_sw[j] = n < p.N ? __ldg(p.b_scale + n) * p.inv_group : 0.0f;
        s_bias[j] = (p.bias && n < p.N) ? bf16_bits_to_float(__ldg(p.bias + n)) : 0.0f;
      }
      named_barrier_sync(1, 512);
      const long m = (long)m_row0 + lane;
      const bool mok = m < p.M;
      const float sa = mok ? __ldg(p.a_scale + m) : 0.0f;
      if (!mbar_wait(&bar->acc_full, (uint32_t)i & 1u)) set_device_error(prm.err, kDevErrTimeoutAcc);
      tc_fence_after();
      uint32_t v[2][32];
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(cq * C::kColsPerWarp) + kAccCol;
      // optional copy of the int32 accumulator (parity checks)
      auto write_debug = [&](const uint32_t(&vv)[32], int ch) {
        const int n = n_pair + cq * C::kColsPerWarp + ch * 32;
        if (!p.acc_debug || !mok || n >= p.N) return;
        const int nv = min(32, p.N - n);
        uint4* dd = reinterpret_cast<uint4*>(p.acc_debug + m * p.N + n);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (4 * c < nv)
            dd[c] = make_uint4((uint32_t)((int)vv[4 * c] >> kShift), (uint32_t)((int)vv[4 * c + 1] >> kShift),
                               (uint32_t)((int)vv[4 * c + 2] >> kShift), (uint32_t)((int)vv[4 * c + 3] >> kShift));
      };
      if constexpr (LR) {
        // Rewrite the accumulator in place as fp32 (acc s_a) s_w', one
        // 32-column chunk at a time, let the low-rank MMAs add T L2 onto it,
        // then read the sum back below.
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const int c0 = cq * C::kColsPerWarp + ch * 32;
          tmem_ld_32x32b_x32(taddr + (uint32_t)(ch * 32), v[ch]);
          tmem_wait_ld();
          write_debug(v[ch], ch);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 w4 = *reinterpret_cast<const float4*>(s_sw + c0 + 4 * q);
            const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int h = 0; h < 4; ++h)
              v[ch][4 * q + h] =
                  __float_as_uint(__fmul_rn(__fmul_rn(acc_to_float<true>(v[ch][4 * q + h]), sa), wv[h]));
          }
          tmem_st_32x32b_x32(taddr + (uint32_t)(ch * 32), v[ch]);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(&bar->conv, pbase);
        if (!mbar_wait(&bar->lr_done, (uint32_t)i & 1u)) set_device_error(prm.err, kDevErrTimeoutAcc);
        tc_fence_after();
      }
      tmem_ld_32x32b_x32(taddr, v[0]);
      tmem_ld_32x32b_x32(taddr + 32, v[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(&bar->acc_empty, pbase);
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const int c0 = cq * C::kColsPerWarp + ch * 32;
        const int n = n_pair + c0;
        if (n >= p.N) continue;  // warp-uniform
        if constexpr (!LR) write_debug(v[ch], ch);
        uint32_t* vv = v[ch];
        uint32_t o[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 w4 = *reinterpret_cast<const float4*>(s_sw + c0 + 4 * q);
          const float4 b4 = *reinterpret_cast<const float4*>(s_bias + c0 + 4 * q);
          const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
          const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
          float y[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int jj = 4 * q + h;
            const float t = LR ? __uint_as_float(vv[jj])
                               : __fmul_rn(__fmul_rn(acc_to_float<MODE == 1>(vv[jj]), sa), wv[h]);
            y[h] = __fadd_rn(t, bv[h]);
            if constexpr (ACT) y[h] = gelu_tanh(y[h]);
          }
          __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]);
          __nv_bfloat162 h1 = __floats2bfloat162_rn(y[2], y[3]);
          o[2 * q] = *reinterpret_cast<uint32_t*>(&h0);
          o[2 * q + 1] = *reinterpret_cast<uint32_t*>(&h1);
        }
        // stage the warp's 32 x 32 tile and let TMA write it (rows past M and
        // columns past N are dropped by the tensor map bounds)
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4(stage_out + (uint32_t)(lane * 64) + ((((uint32_t)c) ^ sw64) << 4),
                       make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmY, stage_out, n, m_row0);
          bulk_commit();
        }
      }
      if constexpr (LR) {
        // hand the low-rank buffer back to TMA once the stores have read it
        if (lane == 0) {
          bulk_wait_read<0>();
          mbar_arrive(&bar->lr_free);
        }
        __syncwarp();
      }
    };

    if constexpr (SPLIT) {
      // The reduction's operands go to shared memory by cp.async while the
      // k-blocks run (one 16-byte copy per thread, two for the low-rank
      // operands; zero fill past M or N), so that none of its global loads
      // waits after the cluster barrier: this CTA's row scales, its column
      // slice's scales and bias, and with a low-rank term the slice's L2
      // columns (bf16) and this CTA's T rows.
      if (my_tiles > 0) {
        const int t = threadIdx.x;                      // 0 .. 511
        const int cw = BN / prm.split;
        const int m0 = tile_m(0);
        const int n_lo = tile_n(0) + (int)(crank >> 1) * cw;
        const uint32_t vs = sbase + (uint32_t)C::kVecOff;
        if (t < BM / 4) {
          const int m = m0 + 4 * t;
          const int nv = min(max(p.M - m, 0), 4);
          cp_async_16(vs + (uint32_t)(16 * t), nv > 0 ? p.a_scale + m : p.a_scale, (uint32_t)(4 * nv));
        } else if (t < BM / 4 + cw / 4) {
          const int c = t - BM / 4, n = n_lo + 4 * c;    // N % 8 == 0: a chunk is wholly in or out
          cp_async_16(vs + (uint32_t)(kSplitSwOff + 16 * c), n < p.N ? p.b_scale + n : p.b_scale, n < p.N ? 16u : 0u);
        } else if (t < BM / 4 + cw / 4 + cw / 8) {
          const int c = t - BM / 4 - cw / 4, n = n_lo + 8 * c;
          const bool in = p.bias && n < p.N;
          cp_async_16(vs + (uint32_t)(kSplitBiasOff + 16 * c), in ? (const void*)(p.bias + n) : (const void*)p.b_scale,
                      in ? 16u : 0u);
        }
        if (SPLIT == 2 && p.rank > 0) {
          const int r = p.rank;
          const int tv = r / 8;                           // 16-byte chunks of a T row
          const uint32_t ts = sbase + (uint32_t)(C::kOutOff + kSplitTOff);
          for (int i = t; i < BM * tv; i += 16 * 32) {
            const int row = i / tv, v = i - row * tv;
            const long m = (long)m0 + row;
            const bool in = m < p.M;
            cp_async_16(ts + (uint32_t)(row * (2 * r + 16) + 16 * v), in ? p.T + m * r + 8 * v : p.T, in ? 16u : 0u);
          }
          const int lv = cw / 8;                          // 16-byte chunks of an L2 slice row
          const uint32_t l2b = sbase + (uint32_t)C::kOutOff;
          for (int i = t; i < r * lv; i += 16 * 32) {
            const int k = i / lv, v = i - k * lv;
            const int n = n_lo + 8 * v;
            const bool in = n < p.N;
            cp_async_16(l2b + (uint32_t)((k * cw + 8 * v) * 2), in ? p.L2 + (long)k * p.N + n : p.L2, in ? 16u : 0u);
          }
        }
      }
      // one tile: widen this pair's k-blocks, then leave this warp's share
      // of the int32 partial (32 rows x 64 columns) in the ring area, idle
      // once the accumulator is final (every MMA has read its stages)
      for (int g = set; g < total_kb; g += kSets)
        if (!widen(g)) break;
      if (my_tiles > 0) {
        if (!mbar_wait(&bar->acc_full, 0u)) set_device_error(prm.err, kDevErrTimeoutAcc);
        tc_fence_after();
        uint32_t v[2][32];
        const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(cq * C::kColsPerWarp) + kAccCol;
        tmem_ld_32x32b_x32(taddr, v[0]);
        tmem_ld_32x32b_x32(taddr + 32, v[1]);
        tmem_wait_ld();
        const uint32_t prow = sbase + (uint32_t)(r * kPartPitch + cq * C::kColsPerWarp * 4);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            st_shared_v4(prow + (uint32_t)((ch * 32 + 4 * q) * 4),
                         make_uint4(v[ch][4 * q], v[ch][4 * q + 1], v[ch][4 * q + 2], v[ch][4 * q + 3]));
      }
      cp_async_wait_all();   // published to the other threads by the cluster barrier below
    } else if (!PACKED) {
      for (int i = 0; i < my_tiles; ++i) epilogue(i);
    } else {
      // The epilogue of tile i-1 runs before this warp widens any k-block
      // kb >= min(kLead, nk) of tile i: the first k-blocks of tile i are then
      // ready the moment the accumulator is released.  kLead < US keeps those
      // early k-blocks clear of the stages that tile i-1's last MMAs free, so
      // every warp reaches the epilogue as soon as the accumulator is final.
      const int lead = min(C::kLead, nk);
      int next_epi = 0;
      int i = 0, kb = set;
      while (kb >= nk) { kb -= nk; ++i; }
      for (int g = set; g < total_kb; g += kSets) {
        while (next_epi < i - 1 || (next_epi == i - 1 && kb >= lead)) epilogue(next_epi++);
        if (!widen(g)) break;
        kb += kSets;
        while (kb >= nk) { kb -= nk; ++i; }
      }
      while (next_epi < my_tiles) epilogue(next_epi++);
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncwarp();   // single-lane roles rejoin their warps before the aligned cluster barrier
  cluster_sync();
  if constexpr (SPLIT) {
    if (warp < 16 && my_tiles > 0) {
      // column slice q of this CTA's 128 rows: the pairs' partials summed in
      // pair order (exact int32), then the epilogue of the unsplit form.  A
      // thread keeps one group of four columns (their scales and bias in
      // registers) and walks rows `step` apart, two rows' loads in flight.
      // With a low-rank branch (rank r = p.rank > 0) the slice's columns of
      // L2 are widened to fp32 after the partials, its rows of T wait in the
      // idle epilogue staging area, and each output adds sum_t T[m][t]
      // L2[t][n] (fp32 fused multiply-adds, even and odd t in two chains)
      // before the bias, like the persistent form's low-rank MMA does.
      const int S = prm.split;
      const int cw = BN / S;                             // columns in the slice
      const int per_row = cw / 4;                        // column groups in the slice
      const int step = 16 * 32 / per_row;                // rows per pass
      const int cs = (threadIdx.x % per_row) * 4;        // this thread's columns within the slice
      const int c = (int)(crank >> 1) * cw + cs;
      const int n = tile_n(0) + c;
      const int row0 = threadIdx.x / per_row;
      const int lr_rank = SPLIT == 2 ? p.rank : 0;
      const uint32_t l2s = sbase + (uint32_t)kL2fOff;                 // fp32 L2 slice [r][cw]
      const uint32_t ts = sbase + (uint32_t)(C::kOutOff + kSplitTOff);  // bf16 T rows [128][r], pitch 2r + 16
      const int t_pitch = 2 * lr_rank + 16;
      const uint8_t* vec_b = smem_raw + (sbase - raw) + C::kVecOff;
      const float* vec = reinterpret_cast<const float*>(vec_b);                        // row scales
      const float* vec_sw = reinterpret_cast<const float*>(vec_b + kSplitSwOff);       // column scales
      const uint16_t* vec_bias = reinterpret_cast<const uint16_t*>(vec_b + kSplitBiasOff);
      if (lr_rank > 0) {
        // the bf16 slice (loaded during the k-blocks) widened to fp32 once
        const uint32_t l2b = sbase + (uint32_t)C::kOutOff;
        for (int i = threadIdx.x; i < lr_rank * per_row; i += 16 * 32) {
          const uint2 h = ld_shared_v2(l2b + (uint32_t)(i * 8));
          st_shared_v4(l2s + (uint32_t)(i * 16), make_uint4(h.x << 16, h.x & 0xFFFF0000u, h.y << 16, h.y & 0xFFFF0000u));
        }
        named_barrier_sync(1, 16 * 32);
      }
      if (n < p.N) {
        float sw[4], bv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          sw[j] = vec_sw[cs + j] * p.inv_group;
          bv[j] = p.bias ? bf16_bits_to_float(vec_bias[cs + j]) : 0.0f;
        }
        for (int rb = row0; rb < BM; rb += 2 * step) {
          uint4 w[2][4];
          float sa[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int row = rb + k * step;
            const long m = (long)tile_m(0) + row;
            sa[k] = (row < BM && m < p.M) ? vec[row] : 0.0f;
            const uint32_t local = sbase + (uint32_t)(row * kPartPitch + c * 4);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (q < S && row < BM) w[k][q] = ld_cluster_v4(map_to_rank(local, (uint32_t)(2 * q) + rank));
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int row = rb + k * step;
            const long m = (long)tile_m(0) + row;
            if (row >= BM || m >= p.M) continue;
            uint32_t acc[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (q < S) {
                acc[0] += w[k][q].x;
                acc[1] += w[k][q].y;
                acc[2] += w[k][q].z;
                acc[3] += w[k][q].w;
              }
            }
            if (p.acc_debug)
              *reinterpret_cast<uint4*>(p.acc_debug + m * p.N + n) =
                  make_uint4((uint32_t)((int)acc[0] >> kShift), (uint32_t)((int)acc[1] >> kShift),
                             (uint32_t)((int)acc[2] >> kShift), (uint32_t)((int)acc[3] >> kShift));
            float y[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) y[j] = __fmul_rn(__fmul_rn(acc_to_float<MODE == 1>(acc[j]), sa[k]), sw[j]);
            if (lr_rank > 0) {
              // plain shared-memory reads, so that the compiler batches the
              // eight L2 rows of a step ahead of the multiply-adds; even and
              // odd ranks accumulate separately and meet at the end
              const float4* l2p = reinterpret_cast<const float4*>(smem_raw + (l2s - raw)) + cs / 4;
              const uint4* tp = reinterpret_cast<const uint4*>(smem_raw + (ts - raw) + row * t_pitch);
              float2 e01 = make_float2(0.0f, 0.0f), e23 = e01, o01 = e01, o23 = e01;
              for (int t0 = 0; t0 < lr_rank; t0 += 8) {
                const uint4 tv = tp[t0 / 8];
                float4 lv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) lv[u] = l2p[(t0 + u) * (cw / 4)];
                const uint32_t tw[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
                for (int u = 0; u < 8; u += 2) {
                  const float te = __uint_as_float(tw[u / 2] << 16);
                  const float to = __uint_as_float(tw[u / 2] & 0xFFFF0000u);
                  e01 = __ffma2_rn(make_float2(te, te), make_float2(lv[u].x, lv[u].y), e01);
                  e23 = __ffma2_rn(make_float2(te, te), make_float2(lv[u].z, lv[u].w), e23);
                  o01 = __ffma2_rn(make_float2(to, to), make_float2(lv[u + 1].x, lv[u + 1].y), o01);
                  o23 = __ffma2_rn(make_float2(to, to), make_float2(lv[u + 1].z, lv[u + 1].w), o23);
                }
              }
              const float2 l01 = __fadd2_rn(e01, o01), l23 = __fadd2_rn(e23, o23);
              y[0] = __fadd_rn(y[0], l01.x);
              y[1] = __fadd_rn(y[1], l01.y);
              y[2] = __fadd_rn(y[2], l23.x);
              y[3] = __fadd_rn(y[3], l23.y);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              y[j] = __fadd_rn(y[j], bv[j]);
              if constexpr (ACT) y[j] = gelu_tanh(y[j]);
            }
            __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(y[2], y[3]);
            *reinterpret_cast<uint2*>(p.Y + m * p.N + n) =
                make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
          }
        }
      }
    }
    __syncwarp();
    cluster_sync();   // the partials stay readable until every CTA has summed its slice
  }
  if (warp == kTmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
// split > 1 (SPLIT): one cluster of `split` pairs per tile, all resident at once.
template <int MODE, bool LR, bool ACT = false, int SPLIT = 0>
cudaError_t launch_impl(const GemmArgs& a, unsigned int* err, cudaStream_t st, int split = 1) {
  using C = Cfg<MODE, LR>;
  auto kern = gemm_kernel<MODE, LR, ACT, SPLIT>;
  static DeviceFlags configured;   // one per instantiation
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (!configured.done(dev)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured.set(dev);
  }
  CUtensorMap tA, tB, tY, tT, tL2;
  // packed 4-bit rows: 64-byte boxes, 64-byte swizzle; int8 rows: 128-byte
  // boxes, 128-byte swizzle
  const bool a_packed = MODE == 1, b_packed = MODE != 0;
  const CUtensorMapSwizzle swz64 = CU_TENSOR_MAP_SWIZZLE_64B, swz128 = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tmap(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.A, (uint64_t)a.M, a_packed ? a.K / 2 : a.K,
                 a_packed ? BK / 2 : BK, BM, a_packed ? swz64 : swz128) ||
      !make_tmap(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.B, (uint64_t)a.N, b_packed ? a.K / 2 : a.K,
                 b_packed ? BK / 2 : BK, C::BNH, b_packed ? swz64 : swz128) ||
      !make_tmap(&tY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.Y, (uint64_t)a.M, (uint64_t)a.N, 32, 32,
                 CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  if (LR) {
    // T [M, r]: 64-rank x 128-row boxes; L2 [r, N]: 64-column x 128-rank boxes
    if (!make_tmap(&tT, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.T, (uint64_t)a.M, (uint64_t)a.rank, 64, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap(&tL2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.L2, (uint64_t)a.rank, (uint64_t)a.N, 64, LRC,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    tT = tY;
    tL2 = tY;
  }
  const int pairs = ((a.M + 2 * BM - 1) / (2 * BM)) * ((a.N + C::BN - 1) / C::BN);
  int sms = 0;
  if ((e = device_sm_count(dev, &sms)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  // persistent: one pair per TPC; split-K: one cluster of `split` pairs per tile
  cfg.gridDim = dim3(SPLIT ? 2 * split * pairs : 2 * std::min(pairs, sms / 2), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = SPLIT ? 2 * split : 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  Params prm{a, err, SPLIT ? split : 1};
  e = cudaLaunchKernelEx(&cfg, kern, prm, tA, tB, tY, tT, tL2);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

unsigned int* device_error_word();

namespace {

// K slices for the split-K form of a W4A4 or W4A8 layer: 4 or 2 when it has
// too few 256 x 256 tiles to give every TPC one (tiles x slices <= SMs / 2),
// each slice keeps at least two k-blocks, a low-rank branch is small (rank
// <= 32) on a long K range (>= 48 k-blocks) with its fp32 slice of L2 within
// the 32 KB epilogue staging area, and every cluster of 2 x slices CTAs fits
// on the GPU at once; else 1 (the persistent form).
struct SplitKey {
  int64_t v[4];
};

// The decision itself, a pure host function: `resident(s, clusters)` gives
// how many clusters of 2 s CTAs (one per SM) fit on the GPU at once.
template <class Resident>
bool choose_split(int tiles, int nkb, int rank, int sms, Resident&& resident, int& out) {
  out = 1;
  for (int s : {4, 2}) {
    if (tiles * s > sms / 2 || nkb < 2 * s) continue;
    // the low-rank term runs on CUDA cores here (M N r fused multiply-adds,
    // ~0.13 us per unit of rank at M = 256, N = 3072): worth it only for a
    // small rank on a long K range
    if (rank > kSplitMaxRank || (rank > 0 && nkb < 48)) continue;
    int clusters = 0;
    if (!resident(s, clusters)) return false;
    if (clusters >= tiles) {
      out = s;
      break;
    }
  }
  return true;
}
template <int MODE, bool ACT>
cudaError_t plan_split(const GemmArgs& a, int* split) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int sms = 0;
  if ((e = device_sm_count(dev, &sms)) != cudaSuccess) return e;
  const int tiles = ((a.M + 2 * BM - 1) / (2 * BM)) * ((a.N + 255) / 256);
  const int nkb = a.K / BK;
  static PlanCache<SplitKey, int, 32> cache;
  const SplitKey key = {{dev, tiles, nkb, sms + ((int64_t)a.rank << 32)}};
  const bool ok = cache.get(key, *split, [&](int& out) {
    using C = Cfg<MODE, false>;
    auto kern = gemm_kernel<MODE, false, ACT, 1>;
    return choose_split(tiles, nkb, a.rank, sms, [&](int s, int& clusters) {
      if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes)) !=
          cudaSuccess)
        return false;
      cudaLaunchConfig_t qc = {};
      qc.gridDim = dim3(2 * s * tiles, 1, 1);
      qc.blockDim = dim3(kThreads, 1, 1);
      qc.dynamicSmemBytes = C::kSmemBytes;
      cudaLaunchAttribute qa;
      qa.id = cudaLaunchAttributeClusterDimension;
      qa.val.clusterDim.x = 2 * s;
      qa.val.clusterDim.y = 1;
      qa.val.clusterDim.z = 1;
      qc.attrs = &qa;
      qc.numAttrs = 1;
      return (e = cudaOccupancyMaxActiveClusters(&clusters, kern, &qc)) == cudaSuccess;
    }, out);
  });
  return ok ? cudaSuccess : e;
}

}  // namespace

bool plan_gemm_split(int M, int N, int K, int rank, int sms, int clusters_of_8, int clusters_of_4, int* split) {
  const int tiles = ((M + 2 * BM - 1) / (2 * BM)) * ((N + 255) / 256);
  return choose_split(tiles, K / BK, rank, sms, [&](int s, int& clusters) {
    clusters = s == 4 ? clusters_of_8 : clusters_of_4;
    return true;
  }, *split);
}

cudaError_t launch_gemm(const GemmArgs& a, GemmMode mode, cudaStream_t st) {
  unsigned int* err = device_error_word();
  if (!err) return cudaErrorInvalidDevicePointer;
  if (mode == GemmMode::kW8A8) return launch_impl<0, false>(a, err, st);
  if (mode == GemmMode::kW4A8) {
    int split = 1;
    cudaError_t e = plan_split<2, false>(a, &split);
    if (e != cudaSuccess) return e;
    return split > 1 ? launch_impl<2, false, false, 1>(a, err, st, split) : launch_impl<2, false>(a, err, st);
  }
  {
    int split = 1;
    cudaError_t e = a.act == 1 ? plan_split<1, true>(a, &split) : plan_split<1, false>(a, &split);
    if (e != cudaSuccess) return e;
    if (split > 1 && a.rank > 0)
      return a.act == 1 ? launch_impl<1, false, true, 2>(a, err, st, split)
                        : launch_impl<1, false, false, 2>(a, err, st, split);
    if (split > 1)
      return a.act == 1 ? launch_impl<1, false, true, 1>(a, err, st, split)
                        : launch_impl<1, false, false, 1>(a, err, st, split);
  }
  if (a.act == 1)
    return a.rank > 0 ? launch_impl<1, true, true>(a, err, st) : launch_impl<1, false, true>(a, err, st);
  return a.rank > 0 ? launch_impl<1, true>(a, err, st) : launch_impl<1, false>(a, err, st);
}

}  // namespace w4a4
