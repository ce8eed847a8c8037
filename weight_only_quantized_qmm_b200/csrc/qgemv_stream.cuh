// Streaming quantized GEMV for few tokens per weight row: the bandwidth-bound
// half of the weight-only quantized matmul ("Quantized matmul", affine mode
// w = q * scale + bias per group), for dense calls y = x . dequant(W)^T and
// for the indirect (MoE) form out[i] = a[off(i)] . dequant(W[ids[i]])^T,
// optionally fused as SiLU(gate) * up over two expert stacks.
//
// Work list.  Every CTA sorts the call's pairs by expert in shared memory
// (dense: one expert holding the M tokens) and cuts each expert's pairs into
// segments of up to CH pairs.  A segment covers all 16-row tiles of its
// expert's matrix; the (segment, tile) list is split into contiguous ranges,
// one per CTA (persistent grid, one CTA per SM).
//
// Each tile streams through shared memory as units of GPU groups (all 16
// rows).  A unit arrives with TMA copies counted on the slot's `full`
// mbarrier: per matrix, the packed codes as one 3-D box (16 rows x Z slices of
// 128 bytes, 128-byte swizzle; few large copies keep the copy engine off the
// critical path) and the unit's scales and biases (16 rows x GPU 16-bit
// values, swizzled at their row width).  Warp roles:
//   * producer (1 warp, one lane) issues the copies, slot by slot;
//   * consumers (KC warps) all read every unit, consumer w taking groups
//     [w * GPW, (w + 1) * GPW).  Per group a consumer turns codes into f16
//     pairs with one lop3 (or prmt) each -- a code q sitting at bit p of a
//     16-bit half becomes 1024 + q * 2^p exactly -- takes the partial dot with
//     x on the tensor cores (mma.m16n8k16 f16; rows of W as m, the segment's
//     pairs as n) and folds it into fp32 accumulators.  x is staged per
//     (group, pair) in f16 as x * 2^(e - p), with 2^e a power of two that puts
//     the group's largest |x| in [2^14, 2^15) (exact for 16-bit activations
//     but for values below 2^-24 of the group maximum) and 2^-p undoing the
//     code's bit offset, so the mma yields
//       D = 2^e * (sum_k q_k x_k) + 1024 * sum_k x''_k   (x'' the staged values)
//     and per row
//       y += s * (2^-e * D - 1024 * 2^-e * sum x'') + b * sum_k x_k,
//     which is sum_k x_k (q_k s + b) rewritten per group.  The slot is free
//     again once all KC consumers arrived on its `empty` mbarrier.  At a new
//     segment the consumers stage its x rows (tensor-core k order, with the
//     per-group records {2^-e, -1024 * 2^-e * sum x'', sum x});
//   * epilogue (1 warp): when every consumer posted its partial for a tile
//     (mbarrier `pfull`), sums them in consumer order (the result does not
//     depend on timing), applies SiLU(gate) * up for the fused form and
//     stores the tile's outputs.
// Every wait is bounded: a timeout sets QMM_ERR_TIMEOUT, skips the remaining
// arithmetic and still drains the copies in flight before the CTA exits.
//
// Launched with programmatic stream serialization: the CTA's set-up (barrier
// initialisation, shared-memory carve-up and, for dense calls, L2 prefetches
// of its first weight units) overlaps the previous kernel's tail; every read
// into shared memory or registers (weights, ids, x) comes after
// griddepcontrol.wait, so whatever the previous kernel in the stream wrote --
// weights included -- is visible.
#pragma once

#include <cuda.h>

#include "qgemv_tma.cuh"

namespace qmm {
namespace stream {

constexpr int kMaxStages = 8;

struct Params {
  QgemvParams q;        // the call: pairs, experts, activations, output
  int upt;              // units per tile (ceil(G / GPU))
  int ntiles_e;         // 16-row tiles per expert matrix
  int CH;               // pairs per segment
  int tok_stride;       // bytes between staged rows of x
  int stages;           // ring depth
  uint32_t tx;          // bytes that land per unit (all matrices)
  int off_code, off_sb, off_bar, off_part, off_xs, off_xsum, off_plan;
};

// Layout of one thread's quarter of a group for the f16 lane arithmetic:
// kCodes codes in kRegs packed words, word k of quarter t being word
// t + 4k of the group's row (so that one ldmatrix.x4 hands each thread its
// words of rows g and g + 8); each word yields kOPW f16 pairs, pair j
// holding codes j and j + kOPW of the word, both at bit offset pos(j) inside
// their 16-bit half (a code at bit p reads as 1024 + q * 2^p).
//   8-bit: pairs (0,2) (1,3), offset 0 (byte permutes, no mask);
//   4-bit: pairs (0,4) (1,5) (2,6) (3,7), offsets 0, 4, 0, 4 (the last two
//          from the word shifted right by 8);
//   2-bit: pairs (j, j+8), offsets 0, 2, 4, 6, 8 for j < 5 and 0, 2, 4 for
//          j = 5..7 (from the word shifted right by 10).
// 3- and 6-bit codes straddle words, so quarter t is the contiguous run of
// codes [kCodes t, kCodes (t + 1)) of the group's row, taken 16 codes (48 or
// 96 bits) at a time:
//   3-bit: three byte permutes place 16-bit windows of the run under the two
//          halves of a register; per window up to three codes sit at bit
//          offsets <= 7, and one lop3 per pair keeps one of them per half
//          (3 prmt + 8 lop3 per 16 codes);
//   6-bit: one funnel shift per pair puts code 4k (or 4k + 1) at bit 4 of the
//          low half and code 4k + 2 (4k + 3) at bit 0 of the high half
//          (8 shf + 8 lop3 per 16 codes).
template <int BITS, int GS>
struct Lanes {
  static constexpr bool kWhole = BITS == 2 || BITS == 4 || BITS == 8;  // lanes never straddle words
  static constexpr int kLPW = kWhole ? 32 / BITS : 1;  // codes per packed word
  static constexpr int kOPW = kWhole ? kLPW / 2 : 1;   // f16 pairs per word
  static constexpr int kCodes = GS / 4;                // codes of a thread's quarter
  static constexpr int kQBits = kCodes * BITS;         // bits of a quarter
  // a 16-bit quarter (2-bit codes, group 32): half of word t / 2, spread over
  // both halves of a register before the masks (see quarter_pairs)
  static constexpr bool kHalf = kWhole && kQBits == 16;
  // packed words a thread reads per row: the quarter's own words, or (a
  // 48-bit quarter) the two words that hold it
  static constexpr int kRegs = kQBits == 24 ? 2 : (kQBits + 31) / 32;  // (3-bit group 32: 3 bytes, may straddle)
  static constexpr int kOuts = kCodes / 2;             // f16 pairs of a quarter
  static constexpr int kSteps = kCodes / 4;            // m16n8k16 steps per group
  static constexpr int kWordsPerGroup = GS * BITS / 32;
  static constexpr bool kOk = kWhole ? (kQBits % 32 == 0 || kHalf) : (BITS == 3 || BITS == 6);
  static constexpr uint32_t kMagic = 0x64006400u;      // f16 1024.0 in both halves
  static constexpr float kOff = 1024.0f;
  __host__ __device__ static constexpr int pos(int j) {
    return BITS == 8 ? 0 : BITS == 4 ? (j & 1) * 4 : (j < 5 ? 2 * j : 2 * (j - 5));
  }
  // pair o of the quarter -> code index (within the quarter) and bit offset
  // of its low and high half
  // (a 3-bit quarter of 8 codes, group 32: pair 3 is codes 6 and 7 of byte
  // 2, at bits 2 and 5 of the two halves)
  static constexpr bool k3g32 = BITS == 3 && kCodes == 8;
  __host__ __device__ static constexpr int lo_code(int o) {
    return kHalf ? o : kWhole ? (o / kOPW) * kLPW + o % kOPW
                  : k3g32 ? "\x00\x01\x02\x06"[o]
                  : 16 * (o / 8) + (BITS == 3 ? "\x00\x01\x02\x08\x09\x0a\x06\x07"[o % 8]
                                              : "\x00\x01\x04\x05\x08\x09\x0c\x0d"[o % 8]);
  }
  __host__ __device__ static constexpr int hi_code(int o) {
    return kHalf ? o + 4 : kWhole ? lo_code(o) + kOPW
                  : k3g32 ? "\x03\x04\x05\x07"[o]
                  : 16 * (o / 8) + (BITS == 3 ? "\x03\x04\x05\x0b\x0c\x0d\x0e\x0f"[o % 8]
                                              : "\x02\x03\x06\x07\x0a\x0b\x0e\x0f"[o % 8]);
  }
  __host__ __device__ static constexpr int lo_pos(int o) {
    return kWhole ? pos(o % kOPW)
                  : k3g32 ? "\x00\x03\x06\x02"[o] : (BITS == 3 ? "\x00\x03\x06\x00\x03\x06\x02\x05"[o % 8] : 4);
  }
  __host__ __device__ static constexpr int hi_pos(int o) {
    return kWhole ? pos(o % kOPW)
                  : k3g32 ? "\x01\x04\x07\x05"[o] : (BITS == 3 ? "\x01\x04\x07\x01\x04\x07\x02\x05"[o % 8] : 0);
  }
  // code of the group held as code i of quarter t
  __host__ __device__ static constexpr int gcode(int t, int i) {
    return (kWhole && !kHalf) ? (t + 4 * (i / kLPW)) * kLPW + i % kLPW : kCodes * t + i;
  }
  // first packed word (within the group's row) that thread t reads
  __host__ __device__ static constexpr int first_word(int t) { return (t * kQBits) >> 5; }
};

// Four 8x8 16-bit matrices from shared memory in the mma fragment layout
// (lanes 8m .. 8m + 7 give the row addresses of matrix m).
__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}

// MODE 0: one pair per segment; 1: up to 8; 2: up to 16.  UG: groups per unit
// (32, or 64 when the row length allows; 16 for 32-word groups).  NS: weight
// matrices per pair (2: gate and up).  SB1: rows of G <= UG groups whose
// scale/bias rows are not 16-byte strided (G % 8 != 0, e.g. K = 768 at group
// 64): a unit is TR = 8 whole row tiles (128 rows, one per consumer warp),
// its 128 scale (bias) rows arrive as one contiguous 1-D bulk copy of 256 G
// bytes, unswizzled; groups >= G are skipped.
template <int BITS, int GS, typename T, int MODE, int UG, int NS, bool MOE, bool SB1 = false>
struct Cfg {
  using L = Lanes<BITS, GS>;
  static constexpr int MT = MODE == 2 ? 2 : 1;
  static constexpr bool ONE = MODE == 0;
  // consumer warps: 16 for dense one-token-tile calls (many units per CTA:
  // the steady state wants the warps); 8 for MoE calls, whose few units per
  // CTA favour more groups per warp (measured: T = 1 gate+up -8%, T = 16 -12%)
  static constexpr int KC = (MT == 1 && !MOE) ? 16 : 8;
  static constexpr int THREADS = (KC + 2) * 32;
  static constexpr int PRODUCER = KC, EPILOGUE = KC + 1;          // warp indices
  static constexpr int WPG = L::kWordsPerGroup;                   // words per group per row
  static constexpr int GPU = UG;                                  // groups per unit
  static constexpr int TR = SB1 ? 8 : 1;                          // 16-row tiles per unit (measured: 8 beats 2 and 4)
  static constexpr int ROWS = 16 * TR;                            // weight rows per unit
  static constexpr int WPT = KC / TR;                             // consumers per row tile
  static constexpr int GPW = GPU / WPT;                           // groups per consumer per unit
  static constexpr int Z = GPU * WPG / 32;                        // 128-byte slices per unit row
  static constexpr int SLICE = ROWS * 128;                        // bytes of one slice (all rows)
  static constexpr int CODE_BYTES = Z * SLICE;                    // one matrix
  static constexpr int SB_BYTES = ROWS * GPU * 2;                 // scales (or biases) of one matrix
  static constexpr int TOKP = 8 * MT;
  static constexpr int CH = ONE ? 1 : TOKP;                       // pairs per segment
  static constexpr int XG = 4 * L::kCodes * 2;                    // staged f16 x bytes per group
  static_assert(L::kOk, "a supported (bits, group size)");
  static_assert(GPW >= 1 && GPW * WPT == GPU && WPT * TR == KC, "whole groups per consumer");
  static_assert(Z >= 1 && Z <= 16, "unit of at most 16 slices (32 KB)");
  static_assert(GPU * WPG % 32 == 0, "units of whole 128-byte slices");
  static_assert(GPU * 2 == 32 || GPU * 2 == 64 || GPU * 2 == 128, "scale rows of one swizzle span");
  // partial-sum ring entries (tiles): one token's partials are small, so
  // that ring is deeper; the multi-token fragments would crowd the stages
  static constexpr int RB = ONE ? 4 : 2;
  static_assert((RB & (RB - 1)) == 0, "partial ring is a power of two");
};

__device__ __forceinline__ void sts128(uint32_t a, float4 v) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ float ldsf(uint32_t a) { return __uint_as_float(lds32(a)); }
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// Contiguous global -> shared copy of `bytes` (a multiple of 16, both
// addresses 16-byte aligned), counted on the mbarrier's transaction bytes.
__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// L2 prefetches of one box of a tensor map (no shared memory, no barrier)
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(map), "r"(x), "r"(y),
               "r"(z)
               : "memory");
}
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
               : "memory");
}

// d = A . B for one m16n8k16 f16 step, starting from a zero accumulator.
__device__ __forceinline__ void mma_f16_first(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  const float z = 0.0f;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}

// (w & MASK) | 1024.0 in both f16 halves: one lop3
template <uint32_t MASK>
__device__ __forceinline__ uint32_t mask_magic(uint32_t w) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w), "n"(MASK), "n"(0x64006400u));
  return d;
}
// bytes (a.SEL0, 0x64, a.SEL2, 0x64): two 8-bit codes as 1024 + q in f16
template <uint32_t SEL>
__device__ __forceinline__ uint32_t byte_magic(uint32_t w) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(w), "r"(0x64646464u), "n"(SEL));
  return d;
}

// The kOPW f16 pairs of one packed word (pair j = codes j, j + kOPW; see Lanes).
template <int BITS>
__device__ __forceinline__ void word_pairs16(uint32_t w, uint32_t* o) {
  if constexpr (BITS == 8) {
    o[0] = byte_magic<0x4240u>(w);
    o[1] = byte_magic<0x4341u>(w);
  } else if constexpr (BITS == 4) {
    o[0] = mask_magic<0x000F000Fu>(w);
    o[1] = mask_magic<0x00F000F0u>(w);
    const uint32_t t = w >> 8;
    o[2] = mask_magic<0x000F000Fu>(t);
    o[3] = mask_magic<0x00F000F0u>(t);
  } else {
    o[0] = mask_magic<0x00030003u>(w);
    o[1] = mask_magic<0x000C000Cu>(w);
    o[2] = mask_magic<0x00300030u>(w);
    o[3] = mask_magic<0x00C000C0u>(w);
    o[4] = mask_magic<0x03000300u>(w);
    const uint32_t t = w >> 10;
    o[5] = mask_magic<0x00030003u>(t);
    o[6] = mask_magic<0x000C000Cu>(t);
    o[7] = mask_magic<0x00300030u>(t);
  }
}

__device__ __forceinline__ uint32_t prmt_rt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// The kOuts f16 pairs of thread t's quarter (see Lanes).
template <class L>
__device__ __forceinline__ void quarter_pairs(const uint32_t (&r)[L::kRegs], int t, uint32_t* o) {
  if constexpr (L::kHalf) {
    // the quarter's two bytes, (b0, b1), into the low bytes of the two halves:
    // pair j = codes j and j + 4, at bit 2j of each half
    const uint32_t v = prmt_rt((t & 1) ? (r[0] >> 16) : r[0], 0u, 0x4140u);
    uint32_t tmp[8];
    word_pairs16<2>(v, tmp);
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = tmp[j];
  } else if constexpr (L::kWhole) {
#pragma unroll
    for (int k = 0; k < L::kRegs; ++k) word_pairs16<32 / L::kLPW>(r[k], o + k * L::kOPW);
  } else if constexpr (L::k3g32) {
    // 8 codes = bytes B0..B2 of the word pair (lo, hi) from byte 3t mod 4
    const uint32_t add = (uint32_t)((3 * t) & 3) * 0x1111u;
    const uint32_t r0 = prmt_rt(r[0], r[1], 0x2110u + add);  // (B0, B1 | B1, B2)
    const uint32_t r2 = prmt_rt(r[0], r[1], 0x2222u + add);  // (B2, B2 | B2, B2)
    o[0] = mask_magic<0x000E0007u>(r0);
    o[1] = mask_magic<0x00700038u>(r0);
    o[2] = mask_magic<0x038001C0u>(r0);
    o[3] = mask_magic<0x00E0001Cu>(r2);
  } else if constexpr (L::kQBits / L::kCodes == 3) {
#pragma unroll
    for (int c = 0; c < L::kCodes / 16; ++c) {
      // 16 codes = bytes B0..B5 of the word pair (lo, hi) from byte `off`
      const uint32_t lo = L::kRegs == 2 ? r[0] : r[c], hi = L::kRegs == 2 ? r[1] : r[c + 1];
      const uint32_t add = (L::kRegs == 2 ? (uint32_t)(t & 1) * 2u : (uint32_t)c * 2u) * 0x1111u;
      const uint32_t r0 = prmt_rt(lo, hi, 0x2110u + add);  // (B0, B1 | B1, B2)
      const uint32_t r1 = prmt_rt(lo, hi, 0x5443u + add);  // (B3, B4 | B4, B5)
      const uint32_t r2 = prmt_rt(lo, hi, 0x5532u + add);  // (B2, B3 | B5, B5)
      o[8 * c + 0] = mask_magic<0x000E0007u>(r0);
      o[8 * c + 1] = mask_magic<0x00700038u>(r0);
      o[8 * c + 2] = mask_magic<0x038001C0u>(r0);
      o[8 * c + 3] = mask_magic<0x000E0007u>(r1);
      o[8 * c + 4] = mask_magic<0x00700038u>(r1);
      o[8 * c + 5] = mask_magic<0x038001C0u>(r1);
      o[8 * c + 6] = mask_magic<0x001C001Cu>(r2);
      o[8 * c + 7] = mask_magic<0x00E000E0u>(r2);
    }
  } else if constexpr (L::kCodes == 8) {
    // 6-bit, group 32: 8 codes = 48 bits of the word pair (lo, hi) from bit
    // 16 (t odd) or 0; the windows start at quarter bits -4, 2, 20, 26
    const uint32_t lo = r[0], hi = r[1];
    const bool b = (t & 1) != 0;
    o[0] = mask_magic<0x003F03F0u>(__funnelshift_r(b ? lo : 0u, b ? hi : lo, b ? 12 : 28));
    o[1] = mask_magic<0x003F03F0u>(__funnelshift_r(lo, hi, b ? 18 : 2));
    o[2] = mask_magic<0x003F03F0u>(__funnelshift_r(b ? hi : lo, b ? 0u : hi, b ? 4 : 20));
    o[3] = mask_magic<0x003F03F0u>(__funnelshift_r(b ? hi : lo, b ? 0u : hi, b ? 10 : 26));
  } else {
#pragma unroll
    for (int c = 0; c < L::kCodes / 16; ++c) {
      // 16 codes = words w0..w2; the windows start at stream bits 24k - 4
      // (codes 4k, 4k + 2) and 24k + 2 (codes 4k + 1, 4k + 3)
      const uint32_t w0 = r[3 * c], w1 = r[3 * c + 1], w2 = r[3 * c + 2];
      o[8 * c + 0] = mask_magic<0x003F03F0u>(__funnelshift_r(0u, w0, 28));
      o[8 * c + 1] = mask_magic<0x003F03F0u>(__funnelshift_r(w0, w1, 2));
      o[8 * c + 2] = mask_magic<0x003F03F0u>(__funnelshift_r(w0, w1, 20));
      o[8 * c + 3] = mask_magic<0x003F03F0u>(__funnelshift_r(w0, w1, 26));
      o[8 * c + 4] = mask_magic<0x003F03F0u>(__funnelshift_r(w1, w2, 12));
      o[8 * c + 5] = mask_magic<0x003F03F0u>(__funnelshift_r(w1, w2, 18));
      o[8 * c + 6] = mask_magic<0x003F03F0u>(__funnelshift_r(w2, 0u, 4));
      o[8 * c + 7] = mask_magic<0x003F03F0u>(__funnelshift_r(w2, 0u, 10));
    }
  }
}

// Tensor-core partial dot of one group for 16 rows x 8 (per token tile)
// columns: d = sum over the group's k16 steps of (1024 + q 2^p) * x''.
template <class L, int MT>
__device__ __forceinline__ void group_dot1(const uint32_t (&rawA)[L::kRegs], const uint32_t (&rawB)[L::kRegs],
                                           int t, const uint32_t (&xb)[MT], uint32_t xo, float (&d)[MT][4]) {
  uint32_t pA[L::kOuts], pB[L::kOuts];
  quarter_pairs<L>(rawA, t, pA);
  quarter_pairs<L>(rawB, t, pB);
#pragma unroll
  for (int q2 = 0; q2 < L::kSteps / 2; ++q2) {
    uint4 bf[MT];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) bf[mt] = lds128(xb[mt] + xo + q2 * 16);
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int q = 2 * q2 + h2;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const uint32_t b0 = h2 ? bf[mt].z : bf[mt].x, b1 = h2 ? bf[mt].w : bf[mt].y;
        if (q == 0)
          mma_f16_first(d[mt], pA[2 * q], pB[2 * q], pA[2 * q + 1], pB[2 * q + 1], b0, b1);
        else
          mma16816<__half>(d[mt], pA[2 * q], pB[2 * q], pA[2 * q + 1], pB[2 * q + 1], b0, b1);
      }
    }
  }
}

// As group_dot1 for one token column, with the x fragments in registers.
template <class L>
__device__ __forceinline__ void group_dot_rx(const uint32_t (&rawA)[L::kRegs], const uint32_t (&rawB)[L::kRegs],
                                             int t, const uint4 (&bf)[L::kSteps / 2], float (&d)[4]) {
  uint32_t pA[L::kOuts], pB[L::kOuts];
  quarter_pairs<L>(rawA, t, pA);
  quarter_pairs<L>(rawB, t, pB);
  // one dependent chain of k16 steps (measured: fewer instructions beat two
  // shorter chains merged at the end); only column 0 (rows g, g + 8: d[0],
  // d[2]) is used, the other columns repeat it
#pragma unroll
  for (int q = 0; q < L::kSteps; ++q) {
    const uint32_t b0 = (q & 1) ? bf[q >> 1].z : bf[q >> 1].x, b1 = (q & 1) ? bf[q >> 1].w : bf[q >> 1].y;
    if (q == 0)
      mma_f16_first(d, pA[0], pB[0], pA[1], pB[1], b0, b1);
    else
      mma16816<__half>(d, pA[2 * q], pB[2 * q], pA[2 * q + 1], pB[2 * q + 1], b0, b1);
  }
}

// both 16-bit halves of a word as floats
template <typename T>
__device__ __forceinline__ float2 halves_to_f32(uint32_t v) {
  if constexpr (std::is_same<T, __half>::value) {
    __half2 h;
    memcpy(&h, &v, 4);
    return __half22float2(h);
  } else {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
  }
}
template <typename T>
__device__ __forceinline__ float half_to_f32(uint32_t v, int hi) {
  if constexpr (std::is_same<T, __half>::value) {
    const float2 f = halves_to_f32<T>(v);
    return hi ? f.y : f.x;
  } else {
    return __uint_as_float(hi ? (v & 0xffff0000u) : (v << 16));
  }
}


// Walk over the CTA's (segment, tile) range; segment sg belongs to the j-th
// distinct expert when seg[j] <= sg < seg[j + 1].
struct Walk {
  int sg, rt, j;
  __device__ __forceinline__ void start(int t, int ntiles_e, const int* seg, int nd) {
    sg = t / ntiles_e;
    rt = t - sg * ntiles_e;
    j = 0;
    while (j < nd - 1 && seg[j + 1] <= sg) ++j;
  }
  __device__ __forceinline__ void next(int ntiles_e, const int* seg, int nd) {
    if (++rt == ntiles_e) {
      rt = 0;
      ++sg;
      while (j < nd - 1 && seg[j + 1] <= sg) ++j;
    }
  }
};

// 2^e as a float for e in [-126, 127]
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((e + 127) << 23); }

// Stage the x rows of a segment's pairs [0, np) for groups [0, Gpad): per
// (pair, group, quarter t) the quarter's kCodes values as f16 pairs in the
// order of the code pairs (Lanes), each x_k * 2^(e - p_k), with 2^e chosen per
// (pair, group) so that the group's largest |x| lands in [2^14, 2^15); per
// (group, pair) the record {2^-e, -1024 * 2^-e * sum of the staged values (as
// rounded), sum of x, 0}.  Groups past G stage zeros; records of pairs
// [np, TOKP) read as zero.
template <class L, typename T, int TOKP, int NTHR>
__device__ __forceinline__ void stage_x(const QgemvParams& q, const int* pairs, int np, int Gpad,
                                        int tok_stride, int sid, uint8_t* xs, float4* rec) {
  constexpr int GS = L::kCodes * 4;
  const int ntask = np * Gpad * 4;
  for (int base = 0; base < ntask; base += NTHR) {
    const int idx = base + sid;
    const bool act = idx < ntask;
    const int tt = idx & 3, gq = idx >> 2;
    const int m = act ? gq / Gpad : 0, gl = act ? gq - m * Gpad : 0;
    __align__(16) T xv[L::kCodes];
    if (act && gl < q.G) {
      const T* xg = reinterpret_cast<const T*>(q.a) + pair_offset(q, pairs[m]) + (int64_t)gl * GS;
      if constexpr (L::kWhole && !L::kHalf) {
        constexpr int WB = L::kLPW * (int)sizeof(T);  // bytes of x under one packed word
#pragma unroll
        for (int k = 0; k < L::kRegs; ++k) {
          const T* xa = xg + L::gcode(tt, k * L::kLPW);
          T* dst = xv + k * L::kLPW;
          if (WB % 16 == 0 && (reinterpret_cast<uintptr_t>(xa) & 15) == 0) {
#pragma unroll
            for (int c = 0; c < WB / 16; ++c)
              reinterpret_cast<uint4*>(dst)[c] = __ldg(reinterpret_cast<const uint4*>(xa) + c);
          } else if (WB == 8 && (reinterpret_cast<uintptr_t>(xa) & 7) == 0) {
            *reinterpret_cast<uint2*>(dst) = __ldg(reinterpret_cast<const uint2*>(xa));
          } else {
#pragma unroll
            for (int c = 0; c < L::kLPW; ++c) dst[c] = xa[c];
          }
        }
      } else {  // the quarter's codes are one contiguous run
        const T* xa = xg + L::gcode(tt, 0);
        if ((reinterpret_cast<uintptr_t>(xa) & 15) == 0) {
#pragma unroll
          for (int c = 0; c < L::kCodes * (int)sizeof(T) / 16; ++c)
            reinterpret_cast<uint4*>(xv)[c] = __ldg(reinterpret_cast<const uint4*>(xa) + c);
        } else {
#pragma unroll
          for (int c = 0; c < L::kCodes; ++c) xv[c] = xa[c];
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < L::kCodes * (int)sizeof(T) / 16; ++c)
        reinterpret_cast<uint4*>(xv)[c] = make_uint4(0u, 0u, 0u, 0u);
    }
    // the group's largest magnitude (the four quarters sit in one quad)
    float mx = 0.0f;
#pragma unroll
    for (int c = 0; c < L::kCodes; ++c) mx = fmaxf(mx, fabsf(to_f32(xv[c])));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    // e = 14 - floor(log2(mx)), kept inside the normal fp32 range
    int e = 0;
    if (mx > 0.0f) {
      const int E = ((__float_as_int(mx) >> 23) & 0xFF) - 127;
      e = min(max(14 - E, -100), 126);
    }
    float sx = 0.0f, ss = 0.0f;
    __align__(16) uint32_t outv[L::kOuts];
#pragma unroll
    for (int o = 0; o < L::kOuts; ++o) {
      const float xl = to_f32(xv[L::lo_code(o)]), xh = to_f32(xv[L::hi_code(o)]);
      const __half hl = __float2half_rn(xl * exp2i(e - L::lo_pos(o))), hh = __float2half_rn(xh * exp2i(e - L::hi_pos(o)));
      ss += __half2float(hl) + __half2float(hh);
      sx += xl + xh;
      outv[o] = (uint32_t)__half_as_ushort(hl) | ((uint32_t)__half_as_ushort(hh) << 16);
    }
    if (act) {
      uint4* dst = reinterpret_cast<uint4*>(xs + (int64_t)m * tok_stride + (size_t)(gl * 4 + tt) * L::kCodes * 2);
#pragma unroll
      for (int c = 0; c < L::kOuts / 4; ++c) dst[c] = reinterpret_cast<const uint4*>(outv)[c];
    }
    sx += __shfl_xor_sync(0xffffffffu, sx, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    sx += __shfl_xor_sync(0xffffffffu, sx, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    if (act && tt == 0) {
      const float c = exp2i(-e);
      rec[gl * TOKP + m] = make_float4(c, -L::kOff * c * ss, sx, 0.0f);
    }
  }
  for (int idx = sid; idx < Gpad * TOKP; idx += NTHR)
    if (idx % TOKP >= np) rec[idx] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
}

// PT (8-bit codes only): per-tensor dynamic-range int8 ("mlex 0.1.3
// src/quant.rs"): the codes are int8 q, u = q + 128 is the code the lanes
// decode, and one scale fl((out_max - out_min) / 255) with bias out_min
// serves every group (scales[0] points to the four float params; no
// scale/bias copies).
template <int BITS, int GS, typename T, int MODE, int UG, int NS, bool MOE, bool SB1, bool PT>
__global__ void __launch_bounds__(Cfg<BITS, GS, T, MODE, UG, NS, MOE, SB1>::THREADS, 1)
qgemv_stream_kernel(const Params p, const __grid_constant__ CUtensorMap tmc0, const __grid_constant__ CUtensorMap tms0,
                    const __grid_constant__ CUtensorMap tmb0, const __grid_constant__ CUtensorMap tmc1,
                    const __grid_constant__ CUtensorMap tms1, const __grid_constant__ CUtensorMap tmb1) {
  using C = Cfg<BITS, GS, T, MODE, UG, NS, MOE, SB1>;
  using L = typename C::L;
  constexpr int GPU = C::GPU, GPW = C::GPW, TOKP = C::TOKP, WPG = C::WPG, MT = C::MT, KC = C::KC, CH = C::CH;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const QgemvParams& q = p.q;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int STAGES = p.stages;
  const uint32_t code_ring = smem_u32(smem + p.off_code);
  const uint32_t sb_ring = smem_u32(smem + p.off_sb);
  const uint32_t bar_full = smem_u32(smem + p.off_bar);
  const uint32_t bar_pfull = bar_full + 16 * kMaxStages;  // after full[] and empty[]
  const uint32_t bar_pempty = bar_pfull + 8 * C::RB;
  const uint32_t part_sa = smem_u32(smem + p.off_part);
  uint8_t* xs = smem + p.off_xs;
  float4* xrec = reinterpret_cast<float4*>(smem + p.off_xsum);  // [Gpad][TOKP] group records
  const int E = q.num_experts;
  int* s_cnt = reinterpret_cast<int*>(smem + p.off_plan);
  int* s_start = s_cnt + E;
  int* s_fill = s_start + E;
  int* s_dist = s_fill + E;
  int* s_seg = s_dist + E;  // E + 1 entries
  int* s_list = s_seg + E + 1;
  // expert (weight block) of distinct entry j; shares the placement counters,
  // which are dead once the plan is built
  int* s_wexp = s_fill;
  __shared__ int s_nd, s_direct;
  __shared__ int64_t s_xoff[16];  // activation row offsets of the staged x rows

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_full + 8 * kMaxStages + 8 * s, KC * 32);  // every consumer lane arrives
    }
    for (int e = 0; e < C::RB; ++e) {
      mbar_init(bar_pfull + 8 * e, KC * 32);
      mbar_init(bar_pempty + 8 * e, 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Dense calls know their tiles without reading memory: before waiting for
  // the previous kernel, the producer asks L2 for the first units of its
  // range.  A prefetch only chooses which lines sit in L2 (the point of
  // coherence), never their contents, so it is safe even when the previous
  // kernel writes these weights; the copies into shared memory come after the
  // wait.
  if (!q.ids && warp == C::PRODUCER && lane == 0) {
    const int TTd = ((q.n_pairs + CH - 1) / CH) * p.ntiles_e;
    const int tb0 = (int)((int64_t)TTd * blockIdx.x / gridDim.x);
    const int te0 = (int)((int64_t)TTd * (blockIdx.x + 1) / gridDim.x);
    const int nun = min((te0 - tb0) * p.upt, STAGES);
    for (int i = 0; i < nun; ++i) {
      const int t = tb0 + i / p.upt, ku = i % p.upt;
      const int y = (t % p.ntiles_e) * C::ROWS;
      tma_prefetch_3d(&tmc0, 0, y, ku * C::Z);
      if constexpr (!PT) {
        tma_prefetch_2d(&tms0, ku * GPU, y);
        tma_prefetch_2d(&tmb0, ku * GPU, y);
      }
    }
  }
  // weights, ids and x may all come from the previous kernel in the stream
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float pt_s = 0.0f, pt_b = 0.0f;  // PT: the per-tensor scale fl((out_max - out_min) / 255) and out_min
  if constexpr (PT) {
    const float* pp = reinterpret_cast<const float*>(q.scales[0]);
    pt_s = __fdiv_rn(__fsub_rn(__ldg(pp + 3), __ldg(pp + 2)), 255.0f);
    pt_b = __ldg(pp + 2);
  }
  if (q.ids) {
    bool direct = false;
    if constexpr (C::ONE) {
      // One pair per segment: a segment's position in the list does not change
      // what it computes, so when every id is in range segment j is simply
      // pair j (one warp reads the ids; no sort, one barrier).
      if (q.n_pairs <= 32 && q.n_pairs <= E) {
        if (warp == 0) {
          const int e = lane < q.n_pairs ? q.ids[lane] : 0;
          const bool all_ok = __all_sync(0xffffffffu, e >= 0 && e < E);
          if (all_ok && lane < q.n_pairs) {
            s_cnt[lane] = 1;
            s_start[lane] = lane;
            s_list[lane] = lane;
            s_dist[lane] = lane;
            s_wexp[lane] = e;
            s_seg[lane] = lane;
          }
          if (lane == 0) {
            s_direct = all_ok;
            if (all_ok) {
              s_seg[q.n_pairs] = q.n_pairs;
              s_nd = q.n_pairs;
            }
          }
        }
        __syncthreads();
        direct = s_direct;
      }
    }
    if (!direct) {  // pairs sorted by expert; out-of-range ids reported and zero-filled
      build_plan(q, s_cnt, s_start, s_fill, s_dist, s_list, s_list + q.n_pairs, &s_nd);
      if (tid == 0) {
        int run = 0;
        s_seg[0] = 0;
        for (int j = 0; j < s_nd; ++j) {
          run += (s_cnt[s_dist[j]] + CH - 1) / CH;
          s_seg[j + 1] = run;
          s_wexp[j] = s_dist[j];
        }
      }
    }
  } else {
    // dense: one expert holding the M tokens, nothing to sort
    if (tid < q.n_pairs) s_list[tid] = tid;
    if (tid == 0) {
      s_cnt[0] = q.n_pairs;
      s_start[0] = 0;
      s_dist[0] = 0;
      s_wexp[0] = 0;
      s_nd = 1;
      s_seg[0] = 0;
      s_seg[1] = (q.n_pairs + CH - 1) / CH;
    }
  }
  __syncthreads();
  // the next kernel in the stream may launch now; it waits for this grid's
  // completion before it reads anything this grid writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int nd = s_nd;
  const int TT = s_seg[nd] * p.ntiles_e;
  const int tb = (int)((int64_t)TT * blockIdx.x / gridDim.x);
  const int te = (int)((int64_t)TT * (blockIdx.x + 1) / gridDim.x);
  const int nt = te - tb;
  const int nunits = nt * p.upt;
  const int Gpad = p.upt * GPU;

  // ---------------------------------------------------------------- producer
  if (warp == C::PRODUCER) {
    if (lane == 0 && nt > 0) {
      int ku = 0, issued = 0;
      Walk w;
      w.start(tb, p.ntiles_e, s_seg, nd);
      for (int i = 0; i < nunits; ++i) {
        const int slot = i % STAGES;
        if (i >= STAGES &&
            !mbar_wait(bar_full + 8 * kMaxStages + 8 * slot, (uint32_t)((i / STAGES) - 1) & 1u, false)) {
          set_status(q.d_status, QMM_ERR_TIMEOUT);
          break;
        }
        const int y = s_wexp[w.j] * (int)q.n_rows + w.rt * C::ROWS;  // first row in the expert stack
        const uint32_t fb = bar_full + 8 * slot;
        mbar_arrive_expect_tx(fb, p.tx);
        const uint32_t cd = code_ring + (uint32_t)(slot * NS * C::CODE_BYTES);
        const uint32_t sd = sb_ring + (uint32_t)(slot * NS * 2 * C::SB_BYTES);
        tma_load_3d(cd, &tmc0, 0, y, ku * C::Z, fb);
        if constexpr (PT) {
        } else if constexpr (SB1) {  // rows y .. y + ROWS - 1 of the [rows, G] arrays, contiguous
          const uint32_t nb = (uint32_t)(2 * C::ROWS * q.G);
          bulk_load_1d(sd, reinterpret_cast<const uint8_t*>(q.scales[0]) + (int64_t)y * q.G * 2, nb, fb);
          bulk_load_1d(sd + C::SB_BYTES, reinterpret_cast<const uint8_t*>(q.biases[0]) + (int64_t)y * q.G * 2, nb, fb);
        } else {
          tma_load_2d(sd, &tms0, ku * GPU, y, fb);
          tma_load_2d(sd + C::SB_BYTES, &tmb0, ku * GPU, y, fb);
        }
        if constexpr (NS == 2) {
          tma_load_3d(cd + C::CODE_BYTES, &tmc1, 0, y, ku * C::Z, fb);
          tma_load_2d(sd + 2 * C::SB_BYTES, &tms1, ku * GPU, y, fb);
          tma_load_2d(sd + 3 * C::SB_BYTES, &tmb1, ku * GPU, y, fb);
        }
        issued = i + 1;
        if (++ku == p.upt) {
          ku = 0;
          if (i + 1 < nunits) w.next(p.ntiles_e, s_seg, nd);
        }
      }
      // no copy may still be landing when the CTA exits: wait (full bound,
      // even after a failure) for the last copies of every slot
      for (int i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
        mbar_wait_n(bar_full + 8 * (i % STAGES), (uint32_t)(i / STAGES) & 1u, kMbarSpins);
    }
    return;
  }

  // ---------------------------------------------------------------- epilogue
  if (warp == C::EPILOGUE) {
    bool failed = false;
    Walk w;
    if (nt > 0) w.start(tb, p.ntiles_e, s_seg, nd);
    for (int jt = 0; jt < nt; ++jt) {
      const int e = jt & (C::RB - 1);
      const bool ok = mbar_wait(bar_pfull + 8 * e, (uint32_t)(jt / C::RB) & 1u, failed);
      if (__any_sync(0xffffffffu, !ok)) {
        if (!failed && lane == 0) set_status(q.d_status, QMM_ERR_TIMEOUT);
        failed = true;
      }
      if (!failed) {
        const int ex = s_dist[w.j], chunk = w.sg - s_seg[w.j];
        const int* pairs = s_list + s_start[ex] + chunk * CH;
        const int np = min(CH, s_cnt[ex] - chunk * CH);
        if constexpr (C::ONE) {
          // partials: [entry][consumer][matrix][16 rows] floats; row tile rt of
          // the unit sums its consumers rt * WPT .. rt * WPT + WPT - 1
          for (int idx = lane; idx < 16 * C::TR; idx += 32) {
            const int rr = idx & 15, rt = idx >> 4;
            float y[NS];
#pragma unroll
            for (int ns = 0; ns < NS; ++ns) {
              y[ns] = 0.0f;
#pragma unroll
              for (int wc = 0; wc < C::WPT; ++wc)
                y[ns] += ldsf(part_sa + (uint32_t)((((e * KC + rt * C::WPT + wc) * NS + ns) * 16 + rr) * 4));
            }
            const float v = NS == 2 ? y[0] / (1.0f + expf(-y[0])) * y[NS - 1] : y[0];
            const int64_t row = (int64_t)w.rt * C::ROWS + rt * 16 + rr;
            if (row < q.n_rows) store_as(q.out, q.out_dtype, (int64_t)pairs[0] * q.out_ld + row, v);
          }
        } else {
          // partials: [entry][consumer][matrix][token tile][lane] float4 (the mma C fragment)
#pragma unroll
          for (int rt = 0; rt < C::TR; ++rt)
          for (int idx = lane; idx < 16 * np; idx += 32) {
            const int r = idx & 15, m = idx >> 4;
            const int mt = m >> 3, col = m & 7;
            const int src = ((r & 7) << 2) | (col >> 1);
            const int ci = ((r >> 3) << 1) | (col & 1);
            float y[NS];
#pragma unroll
            for (int ns = 0; ns < NS; ++ns) {
              const uint32_t a0 =
                  part_sa + (uint32_t)(((((e * KC + rt * C::WPT) * NS + ns) * MT + mt) * 32 + src) * 16 + ci * 4);
              y[ns] = 0.0f;
#pragma unroll
              for (int wc = 0; wc < C::WPT; ++wc) y[ns] += ldsf(a0 + (uint32_t)(wc * NS * MT * 32 * 16));
            }
            const float v = NS == 2 ? y[0] / (1.0f + expf(-y[0])) * y[NS - 1] : y[0];
            const int64_t row = (int64_t)w.rt * C::ROWS + rt * 16 + r;
            if (row < q.n_rows) store_as(q.out, q.out_dtype, (int64_t)pairs[m] * q.out_ld + row, v);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pempty + 8 * e);
      if (jt + 1 < nt) w.next(p.ntiles_e, s_seg, nd);
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  const int g = lane >> 2, t = lane & 3;
  const uint32_t xs_sa = smem_u32(xs), xrec_sa = smem_u32(xrec);
  // row tile (within the unit) and group slot of this consumer
  const int rtl = warp / C::WPT, gw = warp % C::WPT;
  // per-group records of pairs 2t, 2t + 1 (pair 0 only for one pair per segment)
  const uint32_t xrec_lane = xrec_sa + (uint32_t)((gw * GPW * TOKP + (C::ONE ? 0 : 2 * t)) * 16);
  // Code words of group u.  kRegs == 1: the lane's word t of rows g and
  // g + 8 (two 32-bit loads).  kRegs >= 2: ldmatrix.x4 per pair of words
  // (t + 4k, t + 4k + 4): lane l gives the row address of matrix l / 8 =
  // {row l%8, row l%8 + 8} x {chunk c, chunk c + 1}; the 128-byte swizzle puts
  // chunk c of row r at c ^ (r & 7).
  const int lr = lane & 7, lm = lane >> 3;
  // (3- and 6-bit codes: the lane's words first_word(t) + k, one load each)
  auto code_addr = [&](int u, int k2) -> uint32_t {
    const int w0 = (gw * GPW + u) * WPG;  // first word of the group in the unit row
    if constexpr (L::kRegs == 1 || !L::kWhole) {
      const int wr = w0 + ((L::kWhole && !L::kHalf) ? t : L::first_word(t) + k2);  // word in the unit row
      const int wb = wr & 31;
      return (uint32_t)((wr >> 5) * C::SLICE + (rtl * 16 + g) * 128 + (((wb >> 2) ^ g) << 4) + ((wb & 3) << 2));
    } else {
      const int ch = ((w0 & 31) >> 2) + 2 * k2 + (lm >> 1);  // 16-byte chunk within the 128-byte row
      return (uint32_t)((w0 >> 5) * C::SLICE + (rtl * 16 + lr + 8 * (lm & 1)) * 128 + ((ch ^ lr) << 4));
    }
  };
  // scale / bias offsets (within a slot) of rows g and g + 8 for this warp's
  // groups (row g's chunk c sits at chunk c ^ f(g); f is the same for row g + 8)
  // (SB1: plain [16][G] rows, pitch 2 G bytes)
  const int PITCH = SB1 ? 2 * q.G : GPU * 2;
  const int sfx = PITCH == 128 ? (g & 7) : PITCH == 64 ? ((g >> 1) & 3) : ((g >> 2) & 1);
  const int sbyte = gw * GPW * 2;
  const uint32_t soff = SB1 ? (uint32_t)((rtl * 16 + g) * PITCH + sbyte)
                            : (uint32_t)(g * PITCH + ((((sbyte >> 4) ^ sfx)) << 4) + (sbyte & 15));
  // SB1: this warp's groups past the row (>= G) take no part in the sums
  const int live = SB1 ? min(GPW, max(0, q.G - gw * GPW)) : GPW;

  float acc[NS][MT][4];
#pragma unroll
  for (int ns = 0; ns < NS; ++ns)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[ns][mt][i] = 0.0f;
  bool failed = false;
  const int gw_end = q.G - gw * GPW;  // this consumer's groups of unit ku start at ku GPU + gw GPW

  // unit i: slot i % STAGES with phase (i / STAGES) & 1, k-unit ku of tile jt
  int slot = 0, ku = 0, jt = 0, cur_sg = -1, cur_np = -1;
  uint32_t phase = 0;
  uint32_t cslot = code_ring, sslot = sb_ring + soff, bfull = bar_full;
  uint32_t xb[MT], xbu[MT];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) { xb[mt] = xs_sa; xbu[mt] = xs_sa; }
  uint32_t su = xrec_lane;
  Walk w;  // the work-list walk of MoE calls (a dense call is one segment)
  if constexpr (MOE) {
    if (nt > 0) w.start(tb, p.ntiles_e, s_seg, nd);
  }
  for (int i = 0; i < nunits; ++i) {
    if (MOE ? (ku == 0 && w.sg != cur_sg) : i == 0) {
      // a new segment: stage the x rows of its pairs, unless they are the rows
      // already staged (one token routed to several experts)
      int ex = 0, chunk = 0;
      if constexpr (MOE) {
        cur_sg = w.sg;
        ex = s_dist[w.j];
        chunk = w.sg - s_seg[w.j];
      }
      const int np = min(CH, s_cnt[ex] - chunk * CH);
      const int* pn = s_list + s_start[ex] + chunk * CH;
      bool same = MOE && np == cur_np;
      for (int m = 0; m < np && same; ++m) same = pair_offset(q, pn[m]) == s_xoff[m];
      if (!same) {
        asm volatile("bar.sync 1, %0;" ::"n"(KC * 32) : "memory");
        stage_x<L, T, TOKP, KC * 32>(q, pn, np, Gpad, p.tok_stride, tid, xs, xrec);
        if (tid < np) s_xoff[tid] = pair_offset(q, pn[tid]);
        cur_np = np;
        asm volatile("bar.sync 1, %0;" ::"n"(KC * 32) : "memory");
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int tr = (mt * 8 + g) < np ? mt * 8 + g : 0;  // idle columns reread pair 0
          xb[mt] = xs_sa + (uint32_t)(tr * p.tok_stride) + (uint32_t)(t * L::kCodes * 2) +
                   (uint32_t)(gw * GPW * C::XG);
          xbu[mt] = xb[mt];
        }
        su = xrec_lane;
      }
    }
    // (one poll by every lane is the usual case; the vote keeps the branch
    // warp-uniform)
    if (!__all_sync(0xffffffffu, mbar_try_wait(bfull, phase))) {
      const bool ok = mbar_wait(bfull, phase, failed);
      if (__any_sync(0xffffffffu, !ok)) {
        if (!failed && lane == 0) set_status(q.d_status, QMM_ERR_TIMEOUT);
        failed = true;
      }
    }
    // (a consumer whose groups of this unit all lie past the row skips it:
    // they would add exact zeros)
    if (!failed && (SB1 || ku * GPU < gw_end)) {
#pragma unroll
      for (int ns = 0; ns < NS; ++ns) {
        const uint32_t csl = cslot + (uint32_t)(ns * C::CODE_BYTES);
        const uint32_t ssl = sslot + (uint32_t)(ns * 2 * C::SB_BYTES);
        // GPW 16-bit scales (biases) of rows g and g + 8
        uint32_t sv[2][(GPW + 1) / 2], bv[2][(GPW + 1) / 2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t ra = ssl + (uint32_t)(h * 8 * PITCH);
          if constexpr (PT) {  // (the per-tensor scale and bias: no copies)
          } else if constexpr (SB1) {  // 2-byte aligned only: one value at a time
#pragma unroll
            for (int c = 0; c < (GPW + 1) / 2; ++c) {
              sv[h][c] = lds16(ra + 4 * c) | (2 * c + 1 < GPW ? lds16(ra + 4 * c + 2) << 16 : 0u);
              bv[h][c] = lds16(ra + C::SB_BYTES + 4 * c) |
                         (2 * c + 1 < GPW ? lds16(ra + C::SB_BYTES + 4 * c + 2) << 16 : 0u);
            }
          } else if constexpr (GPW == 1) {
            sv[h][0] = lds16(ra);
            bv[h][0] = lds16(ra + C::SB_BYTES);
          } else if constexpr (GPW == 2) {
            sv[h][0] = lds32(ra);
            bv[h][0] = lds32(ra + C::SB_BYTES);
          } else {
#pragma unroll
            for (int c = 0; c < GPW / 4; ++c) {
              const uint2 s2 = lds64(ra + 8 * c), b2 = lds64(ra + C::SB_BYTES + 8 * c);
              sv[h][2 * c] = s2.x; sv[h][2 * c + 1] = s2.y;
              bv[h][2 * c] = b2.x; bv[h][2 * c + 1] = b2.y;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < GPW; ++u) {
          if (SB1 && u >= live) break;  // warp-uniform
          uint32_t rA[L::kRegs], rB[L::kRegs];
          if constexpr (!L::kWhole) {
#pragma unroll
            for (int k = 0; k < L::kRegs; ++k) {
              const uint32_t ca = csl + code_addr(u, k);
              rA[k] = lds32(ca);
              rB[k] = lds32(ca + 1024);
            }
          } else if constexpr (L::kRegs == 1) {
            const uint32_t ca = csl + code_addr(u, 0);
            rA[0] = lds32(ca);
            rB[0] = lds32(ca + 1024);
          } else {
#pragma unroll
            for (int k2 = 0; k2 < L::kRegs / 2; ++k2)
              ldsm_x4(csl + code_addr(u, k2), rA[2 * k2], rB[2 * k2], rA[2 * k2 + 1], rB[2 * k2 + 1]);
          }
          if constexpr (PT) {  // int8 q -> u = q + 128: the top bit of each byte flipped
#pragma unroll
            for (int k = 0; k < L::kRegs; ++k) {
              rA[k] ^= 0x80808080u;
              rB[k] ^= 0x80808080u;
            }
          }
          float d[MT][4];
          if constexpr (C::ONE) {
            // this group's x fragments (staged in the mma's k order); measured:
            // reading them per group beats holding every group's in registers
            uint4 bf[L::kSteps / 2];
#pragma unroll
            for (int q2 = 0; q2 < L::kSteps / 2; ++q2) bf[q2] = lds128(xbu[0] + (uint32_t)(u * C::XG + q2 * 16));
            group_dot_rx<L>(rA, rB, t, bf, d[0]);
          } else
            group_dot1<L, MT>(rA, rB, t, xbu, (uint32_t)(u * C::XG), d);
          const int hw = u & 1;
          const float sa = PT ? pt_s : half_to_f32<T>(sv[0][u >> 1], hw);
          const float sb_ = PT ? pt_s : half_to_f32<T>(sv[1][u >> 1], hw);
          const float ba = PT ? pt_b : half_to_f32<T>(bv[0][u >> 1], hw);
          const float bb = PT ? pt_b : half_to_f32<T>(bv[1][u >> 1], hw);
          // y += s * (2^-e * D - 1024 * 2^-e * sum x'') + b * sum x, per (row, pair)
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            float(&a_)[4] = acc[ns][mt];
            if constexpr (C::ONE) {
              const uint4 rq = lds128(su + (uint32_t)(u * TOKP * 16));
              const float4 r = make_float4(__uint_as_float(rq.x), __uint_as_float(rq.y), __uint_as_float(rq.z), 0.0f);
              a_[0] = fmaf(ba, r.z, fmaf(sa, fmaf(d[0][0], r.x, r.y), a_[0]));
              a_[2] = fmaf(bb, r.z, fmaf(sb_, fmaf(d[0][2], r.x, r.y), a_[2]));
            } else {
              const uint4 q0 = lds128(su + (uint32_t)((u * TOKP + mt * 8) * 16));
              const uint4 q1 = lds128(su + (uint32_t)((u * TOKP + mt * 8) * 16 + 16));
              const float c0 = __uint_as_float(q0.x), n0 = __uint_as_float(q0.y), X0 = __uint_as_float(q0.z);
              const float c1 = __uint_as_float(q1.x), n1 = __uint_as_float(q1.y), X1 = __uint_as_float(q1.z);
              a_[0] = fmaf(ba, X0, fmaf(sa, fmaf(d[mt][0], c0, n0), a_[0]));
              a_[1] = fmaf(ba, X1, fmaf(sa, fmaf(d[mt][1], c1, n1), a_[1]));
              a_[2] = fmaf(bb, X0, fmaf(sb_, fmaf(d[mt][2], c0, n0), a_[2]));
              a_[3] = fmaf(bb, X1, fmaf(sb_, fmaf(d[mt][3], c1, n1), a_[3]));
            }
          }
        }
      }
    }
    mbar_arrive(bfull + 8 * kMaxStages);  // the slot's `empty` barrier: each lane after its own reads

    if (++ku == p.upt) {  // tile done: post this warp's partial
      const int e = jt & (C::RB - 1);
      if (jt >= C::RB) {
        const uint32_t pe = bar_pempty + 8 * e, pp = (uint32_t)((jt / C::RB) - 1) & 1u;
        if (!__all_sync(0xffffffffu, mbar_try_wait(pe, pp))) {
          const bool okp = mbar_wait(pe, pp, failed);
          if (__any_sync(0xffffffffu, !okp)) {
            if (!failed && lane == 0) set_status(q.d_status, QMM_ERR_TIMEOUT);
            failed = true;
          }
        }
      }
#pragma unroll
      for (int ns = 0; ns < NS; ++ns) {
        if constexpr (C::ONE) {
          // lane t = 0 of each quad stores rows g and g + 8 (a predicated
          // store, no divergent region)
          float* pr = reinterpret_cast<float*>(smem + p.off_part) + ((e * KC + warp) * NS + ns) * 16 + g;
          if (t == 0) {
            pr[0] = acc[ns][0][0];
            pr[8] = acc[ns][0][2];
          }
        } else {
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
            sts128(part_sa + (uint32_t)(((((e * KC + warp) * NS + ns) * MT + mt) * 32 + lane) * 16),
                   make_float4(acc[ns][mt][0], acc[ns][mt][1], acc[ns][mt][2], acc[ns][mt][3]));
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[ns][mt][k] = 0.0f;
      }
      mbar_arrive(bar_pfull + 8 * e);  // each lane after its own stores
      ku = 0;
      ++jt;
      if constexpr (MOE) {
        if (i + 1 < nunits) w.next(p.ntiles_e, s_seg, nd);
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) xbu[mt] = xb[mt];
      su = xrec_lane;
    } else {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) xbu[mt] += (uint32_t)(GPU * C::XG);
      su += (uint32_t)(GPU * TOKP * 16);
    }
    if (++slot == STAGES) {
      slot = 0;
      phase ^= 1u;
      cslot = code_ring;
      sslot = sb_ring + soff;
      bfull = bar_full;
    } else {
      cslot += (uint32_t)(NS * C::CODE_BYTES);
      sslot += (uint32_t)(NS * 2 * C::SB_BYTES);
      bfull += 8;
    }
  }
}

// ------------------------------------------------------------------ host side
// 3-D map over packed words [rows, wpr] seen as (word in slice, row, slice of
// 32 words): a box is box_rows rows x z slices, each slice box_rows x 128 bytes,
// swizzled.
inline bool make_code_map3(CUtensorMap* map, const uint32_t* packed, int64_t rows, int64_t wpr, int z,
                           int box_rows) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {32, (cuuint64_t)rows, (cuuint64_t)(wpr / 32)};
  const cuuint64_t strides[2] = {(cuuint64_t)(wpr * 4), 128};
  const cuuint32_t box[3] = {32, (cuuint32_t)box_rows, (cuuint32_t)z};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(packed), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a [rows, G] array of 16-bit scales or biases: 16-row x gpu boxes,
// swizzled at the box row width (32, 64 or 128 bytes) so that the eight rows a
// warp reads at one column fall in different banks.
inline bool make_sb_map(CUtensorMap* map, const void* base, int64_t rows, int G, int gpu) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)G, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)G * 2};
  const cuuint32_t box[2] = {(cuuint32_t)gpu, 16};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz = gpu * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : gpu * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_32B;
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// cudaErrorNotSupported sends the caller to the general kernels.
template <int BITS, int GS, typename T, int MODE, int UG, int NS, bool MOE, bool SB1 = false, bool PT = false>
cudaError_t launch_stream(const QgemvParams& q, cudaStream_t st) {
  static_assert(!PT || (BITS == 8 && NS == 1 && !MOE && !SB1), "per-tensor int8: dense 8-bit lanes");
  using C = Cfg<BITS, GS, T, MODE, UG, NS, MOE, SB1>;
  if (MOE != (q.ids != nullptr)) return cudaErrorNotSupported;
  const int64_t rows_total = q.n_rows * q.num_experts;
  if (q.n_pairs < 1 || q.wpr % 32 != 0 || rows_total < 16) return cudaErrorNotSupported;
  if (SB1) {
    // one unit per row tile; 16-row tiles of every expert start on 16-byte
    // aligned scale/bias rows and never run past the arrays
    if (q.G > C::GPU || q.n_rows % C::ROWS != 0 || NS != 1) return cudaErrorNotSupported;
  } else if (q.G % 8 != 0 || q.G < C::GPU) {
    return cudaErrorNotSupported;
  }
  if (rows_total + 16 >= ((int64_t)1 << 31) || (int64_t)q.n_pairs * q.K >= ((int64_t)1 << 31)) return cudaErrorNotSupported;
  for (int ns = 0; ns < NS; ++ns)
    if (((uintptr_t)q.packed[ns] | (PT ? 0 : ((uintptr_t)q.scales[ns] | (uintptr_t)q.biases[ns]))) & 15)
      return cudaErrorNotSupported;

  Params p{};
  p.q = q;
  p.upt = (q.G + C::GPU - 1) / C::GPU;
  p.ntiles_e = (int)((q.n_rows + C::ROWS - 1) / C::ROWS);
  p.CH = C::CH;
  p.tx = (uint32_t)(NS * C::CODE_BYTES + (PT ? 0 : NS * (SB1 ? 4 * C::ROWS * q.G : 2 * C::SB_BYTES)));
  const int Gpad = p.upt * C::GPU;
  p.tok_stride = Gpad * C::XG + 16;

  // [codes (1024-aligned) | scales+biases | mbarriers | partials | x | sums | plan]
  const size_t part = C::ONE ? (size_t)C::RB * C::KC * NS * 16 * 4 : (size_t)C::RB * C::KC * NS * C::MT * 32 * 16;
  // staged x rows: a segment's pairs (a dense call stages only its own
  // tokens, leaving the rest of shared memory to the weight ring)
  const size_t xs = align128((size_t)(MOE ? C::CH : std::min(C::CH, q.n_pairs)) * p.tok_stride);
  const size_t xsum = align128((size_t)Gpad * C::TOKP * 16);  // float4 records
  const size_t bars = 8 * (2 * kMaxStages + 2 * C::RB);
  const size_t plan = align128((size_t)(5 * q.num_experts + 1 + 2 * q.n_pairs) * sizeof(int));
  if (plan > 32 * 1024) return cudaErrorNotSupported;
  auto total = [&](int stages) {
    return 1024 + (size_t)stages * NS * C::CODE_BYTES + align128((size_t)stages * NS * 2 * C::SB_BYTES) +
           align128(bars) + part + xs + xsum + plan;
  };
  // about 144 KB of the weight stream in flight per SM (measured: deeper rings
  // and an L2 prefetch window ahead of the ring were not faster)
  int stages = (int)((144 * 1024) / p.tx);
  stages = stages < 2 ? 2 : (stages > kMaxStages ? kMaxStages : stages);
  while (stages > 2 && total(stages) > (size_t)kSmemMax) --stages;
  if (total(stages) > (size_t)kSmemMax) return cudaErrorNotSupported;
  p.stages = stages;
  p.off_code = 0;
  p.off_sb = stages * NS * C::CODE_BYTES;
  p.off_bar = p.off_sb + (int)align128((size_t)stages * NS * 2 * C::SB_BYTES);
  p.off_part = p.off_bar + (int)align128(bars);
  p.off_xs = p.off_part + (int)part;
  p.off_xsum = p.off_xs + (int)xs;
  p.off_plan = p.off_xsum + (int)xsum;
  const size_t smem = total(stages);

  CUtensorMap tm[6];
  for (int ns = 0; ns < NS; ++ns) {
    if (!make_code_map3(&tm[3 * ns], q.packed[ns], rows_total, q.wpr, C::Z, C::ROWS)) return cudaErrorNotSupported;
    if (SB1 || PT) {  // no scale/bias maps: 1-D bulk copies, or none
      tm[3 * ns + 1] = tm[3 * ns];
      tm[3 * ns + 2] = tm[3 * ns];
    } else if (!make_sb_map(&tm[3 * ns + 1], q.scales[ns], rows_total, q.G, C::GPU) ||
               !make_sb_map(&tm[3 * ns + 2], q.biases[ns], rows_total, q.G, C::GPU)) {
      return cudaErrorNotSupported;
    }
  }
  if (NS == 1) { tm[3] = tm[0]; tm[4] = tm[1]; tm[5] = tm[2]; }

  auto k = qgemv_stream_kernel<BITS, GS, T, MODE, UG, NS, MOE, SB1, PT>;
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  // dense calls have ceil(N / 16) tiles; the MoE work list is only known on
  // the device, so those calls take one CTA per SM
  const int grid = q.ids ? qmm_host::num_sms() : std::min(qmm_host::num_sms(), p.ntiles_e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, p, tm[0], tm[1], tm[2], tm[3], tm[4], tm[5]);
}

// Instantiation for one (bits, group size, dtype): the unit width and mode.
// Dense calls: one token -> mode 0, up to 8 -> 1, up to 16 -> 2.  MoE calls:
// one activation row per expert is the common case for a single token, so
// mode 0 when n_pairs <= 8, otherwise segments of up to 8 pairs (mode 1).
template <int BITS, int GS, typename T>
cudaError_t try_stream_t(const QgemvParams& q, int mt, bool dual, cudaStream_t st) {
  using L = Lanes<BITS, GS>;
  if constexpr (L::kOk) {
    constexpr int WPG = L::kWordsPerGroup;
    constexpr int UB = WPG > 16 ? 16 : 32;   // base unit (at most 16 slices)
    constexpr int UW = WPG <= 8 ? 64 : UB;   // wide unit: 4 groups per consumer
    if (dual) {
      if (q.n_pairs <= 8) return launch_stream<BITS, GS, T, 0, UB, 2, true>(q, st);
      return launch_stream<BITS, GS, T, 1, UB, 2, true>(q, st);
    }
    if (q.ids) {
      if (q.G % 8 != 0 || q.G < UB) {  // short or odd rows (e.g. the MoE down projection)
        if constexpr (WPG % 2 == 0) {  // 16-group units of whole 128-byte slices
          if (q.G <= 16) {
            if (q.n_pairs <= 8) return launch_stream<BITS, GS, T, 0, 16, 1, true, true>(q, st);
            return launch_stream<BITS, GS, T, 1, 16, 1, true, true>(q, st);
          }
        }
        if constexpr (WPG <= 16) {  // a 32-group unit of at most 16 slices
          if (q.n_pairs <= 8) return launch_stream<BITS, GS, T, 0, 32, 1, true, true>(q, st);
          return launch_stream<BITS, GS, T, 1, 32, 1, true, true>(q, st);
        }
        return cudaErrorNotSupported;
      }
      if (q.n_pairs <= 8) return launch_stream<BITS, GS, T, 0, UB, 1, true>(q, st);
      return launch_stream<BITS, GS, T, 1, UB, 1, true>(q, st);
    }
    // wide units also for rows of whole base units past one wide unit (e.g.
    // K = 14336 at g64: 224 groups, 3.5 wide units): the last unit's groups
    // past the row read zeros and the consumers holding only those skip it,
    // which beats twice the units with half the groups per consumer
    const bool wide = (q.G % UW) == 0 || (q.G > UW && q.G % UB == 0);
    if (q.n_pairs == 1)
      return wide ? launch_stream<BITS, GS, T, 0, UW, 1, false>(q, st) : launch_stream<BITS, GS, T, 0, UB, 1, false>(q, st);
    if (mt == 1)
      return wide ? launch_stream<BITS, GS, T, 1, UW, 1, false>(q, st) : launch_stream<BITS, GS, T, 1, UB, 1, false>(q, st);
    const cudaError_t e2 = launch_stream<BITS, GS, T, 2, UB, 1, false>(q, st);
    if (e2 != cudaErrorNotSupported || q.n_pairs <= 8 || q.amode != 0) return e2;
    // sixteen tokens' x rows do not fit beside the ring: two passes of up to
    // eight tokens each (tokens 8.. read x and write y eight rows further on)
    QgemvParams lo = q, hi = q;
    lo.n_pairs = 8;
    hi.n_pairs = q.n_pairs - 8;
    hi.a = reinterpret_cast<const T*>(q.a) + 8 * q.K;
    hi.out = reinterpret_cast<uint8_t*>(q.out) + 8 * q.out_ld * (q.out_dtype == QMM_F32 ? 4 : 2);
    const cudaError_t e = wide ? launch_stream<BITS, GS, T, 1, UW, 1, false>(lo, st)
                               : launch_stream<BITS, GS, T, 1, UB, 1, false>(lo, st);
    if (e != cudaSuccess) return e;
    return wide ? launch_stream<BITS, GS, T, 1, UW, 1, false>(hi, st) : launch_stream<BITS, GS, T, 1, UB, 1, false>(hi, st);
  } else {
    return cudaErrorNotSupported;
  }
}

// Entry from the per-bit-width files; cudaErrorNotSupported for shapes the
// streaming kernel does not take.
template <int BITS>
cudaError_t try_stream(const QgemvParams& q, int gs, int dtype, int mt, bool dual, cudaStream_t st) {
  if (dtype == QMM_BF16) {
    if (gs == 32) return try_stream_t<BITS, 32, __nv_bfloat16>(q, mt, dual, st);
    if (gs == 64) return try_stream_t<BITS, 64, __nv_bfloat16>(q, mt, dual, st);
    return try_stream_t<BITS, 128, __nv_bfloat16>(q, mt, dual, st);
  }
  if (gs == 32) return try_stream_t<BITS, 32, __half>(q, mt, dual, st);
  if (gs == 64) return try_stream_t<BITS, 64, __half>(q, mt, dual, st);
  return try_stream_t<BITS, 128, __half>(q, mt, dual, st);
}

}  // namespace stream
}  // namespace qmm
