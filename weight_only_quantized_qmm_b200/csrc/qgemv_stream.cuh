// Streaming decode GEMV for the dense case y = x . dequant(W)^T with a few
// tokens (M <= 16): the bandwidth-bound half of the weight-only quantized
// matmul ("Quantized matmul" / affine mode, w = q * scale + bias per group).
//
// One persistent CTA per SM owns a contiguous range of 16-row tiles of W and
// streams each tile through shared memory as units of GPU groups (all 16
// rows).  A unit arrives with three TMA copies counted on the slot's `full`
// mbarrier: the packed codes as one 3-D box (16 rows x Z slices of 128 bytes,
// 128-byte swizzle; few large copies keep the copy engine off the critical
// path), the unit's scales and its biases (16 rows x GPU 16-bit values each).
// Warp roles:
//   * producer (1 warp, one lane) issues the copies, slot by slot;
//   * consumers (kC warps) all read every unit, consumer w taking groups
//     [w * GPW, (w + 1) * GPW).  Per group a consumer turns codes into 16-bit
//     floats (OFF + q, exact), takes the partial dot with x on the tensor
//     cores (mma.m16n8k16; rows of W as m, tokens as n), and folds it into
//     fp32 accumulators as
//       y += s * d + (b - OFF * s) * X,   X = sum of x over the group,
//     which is sum_k x_k (q_k s + b) rewritten per group.  The slot is free
//     again once all kC consumers arrived on its `empty` mbarrier;
//   * epilogue (1 warp): when every consumer posted its partial for a tile
//     (mbarrier `pfull`), sums them in consumer order (the result does not
//     depend on timing) and stores the tile's outputs.
// x is staged once per CTA in the tensor-core k order with its per-group sums.
// Every wait is bounded: a timeout sets QMM_ERR_TIMEOUT, skips the remaining
// arithmetic and still drains the copies in flight before the CTA exits.
//
// Launched with programmatic stream serialization: the producer streams
// weights (which no earlier kernel writes) before griddepcontrol.wait, so a
// call's weight traffic can start while the previous kernel drains; x and y
// are only touched after the wait.
#pragma once

#include <cuda.h>

#include "qgemv_tma.cuh"

namespace qmm {
namespace stream {

constexpr int kRB = 2;          // partial-sum ring entries (tiles)
constexpr int kMaxStages = 8;

struct Params {
  const void* x;        // [M, K] activations (row stride K)
  int M;                // tokens, 1..16
  int64_t K;
  int G;                // groups per row
  int upt;              // units per tile (ceil(G / GPU))
  int64_t N;            // rows of W
  int ntiles;           // ceil(N / 16)
  void* out;            // [M, N]
  int out_dtype;
  int64_t out_ld;
  int32_t* d_status;
  int tok_stride;       // bytes between staged token rows of x
  int stages;           // ring depth
  int pf;               // units prefetched into L2 ahead of the shared-memory loads
  uint32_t magic;       // two 16-bit floats whose low bits take a code (128 + q / 1024 + q)
  int off_code, off_sb, off_bar, off_part, off_xs, off_xsum;
};

// MODE 0: one token; 1: up to 8 tokens; 2: up to 16 tokens.  UG: groups per
// unit (32, or 64 when the row length allows; 16 for 32-word groups).
template <int BITS, int GS, typename T, int MODE, int UG>
struct Cfg {
  using S = Share<BITS, GS, T>;
  static constexpr int MT = MODE == 2 ? 2 : 1;
  static constexpr bool ONE = MODE == 0;
  static constexpr int KC = MT == 1 ? 16 : 8;                     // consumer warps
  static constexpr int THREADS = (KC + 2) * 32;
  static constexpr int STAGERS = (KC + 1) * 32;                   // consumers + epilogue
  static constexpr int PRODUCER = KC, EPILOGUE = KC + 1;          // warp indices
  static constexpr int WPG = S::kWordsPerGroup;                   // words per group per row
  static constexpr int GPU = UG;                                  // groups per unit
  static constexpr int GPW = GPU / KC;                            // groups per consumer per unit
  static constexpr int Z = GPU * WPG / 32;                        // 128-byte slices per unit row
  static constexpr int CODE_BYTES = Z * 16 * 128;
  static constexpr int SB_BYTES = 16 * GPU * 2;                   // scales (or biases) of a unit
  static constexpr uint32_t TX = CODE_BYTES + 2 * SB_BYTES;
  static constexpr int TOKP = 8 * MT;
  static constexpr int XG = 4 * S::kVirt * (int)sizeof(T);        // staged x bytes per group
  static constexpr int NX = S::kSplit ? 2 : 1;                    // per-group sums kept
  static_assert(S::kFast, "integral-lane codes only");
  static_assert(GPW >= 1 && GPW * KC == GPU, "whole groups per consumer");
  static_assert(Z >= 1 && Z <= 16, "unit of at most 16 slices (32 KB)");
  static_assert(GPU * 2 == 32 || GPU * 2 == 64 || GPU * 2 == 128, "scale rows of one swizzle span");
  static_assert((kRB & (kRB - 1)) == 0, "partial ring is a power of two");
};

__device__ __forceinline__ void sts32(uint32_t a, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, float4 v) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}
__device__ __forceinline__ float ldsf(uint32_t a) { return __uint_as_float(lds32(a)); }
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int x, int y, int z) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(map), "r"(x), "r"(y),
               "r"(z)
               : "memory");
}
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// d = sum over the k16 steps of (OFF + v) * x' for 16 rows x 8 columns; the
// first step starts from a zero accumulator.
template <typename T>
__device__ __forceinline__ void mma_first(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  const float z = 0.0f;
  if constexpr (std::is_same<T, __half>::value) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
  }
}

// Codes j and j + LPW/2 of a word of LW-bit lanes as a pair of 16-bit floats
// (MAGIC + code, exact): one shift and one lop3 ((a & b) | c).
template <int LW, int SH>
__device__ __forceinline__ uint32_t lane_pair(uint32_t w, uint32_t magic) {
  constexpr uint32_t MASK = ((1u << LW) - 1u) * 0x00010001u;
  uint32_t d;
  if constexpr (SH == 0) {
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w), "n"(MASK), "r"(magic));
  } else {
    asm("{\n\t.reg .b32 t;\n\tshr.u32 t, %1, %4;\n\tlop3.b32 %0, t, %2, %3, 0xEA;\n\t}"
        : "=r"(d)
        : "r"(w), "n"(MASK), "r"(magic), "n"(SH));
  }
  return d;
}
// All LPW/2 pairs of one word, pair j = codes (j, j + LPW/2).
template <class S>
__device__ __forceinline__ void word_pairs(uint32_t w, uint32_t magic, uint32_t* out) {
  constexpr int LW = S::kLW;
  constexpr int NP = S::kLPW / 2;
  out[0] = lane_pair<LW, 0>(w, magic);
  out[1] = lane_pair<LW, LW>(w, magic);
  if constexpr (NP >= 4) {
    out[2] = lane_pair<LW, 2 * LW>(w, magic);
    out[3] = lane_pair<LW, 3 * LW>(w, magic);
  }
  if constexpr (NP >= 8) {
    out[4] = lane_pair<LW, 4 * LW>(w, magic);
    out[5] = lane_pair<LW, 5 * LW>(w, magic);
    out[6] = lane_pair<LW, 6 * LW>(w, magic);
    out[7] = lane_pair<LW, 7 * LW>(w, magic);
  }
}

template <int BITS, class S, typename T, int MT>
__device__ __forceinline__ void group_dot1(const uint32_t (&rawA)[S::kRegs], const uint32_t (&rawB)[S::kRegs],
                                           const uint32_t (&xb)[MT], uint32_t xo, float (&d)[MT][4],
                                           uint32_t magic) {
  constexpr int NP = S::kLPW / 2;  // pairs per word
  uint32_t pA[S::kRegs * NP], pB[S::kRegs * NP];
#pragma unroll
  for (int k = 0; k < S::kRegs; ++k) {
    word_pairs<S>(rawA[k], magic, pA + k * NP);
    word_pairs<S>(rawB[k], magic, pB + k * NP);
  }
#pragma unroll
  for (int q2 = 0; q2 < S::kSteps / 2; ++q2) {
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
          mma_first<T>(d[mt], pA[2 * q], pB[2 * q], pA[2 * q + 1], pB[2 * q + 1], b0, b1);
        else
          mma16816<T>(d[mt], pA[2 * q], pB[2 * q], pA[2 * q + 1], pB[2 * q + 1], b0, b1);
      }
    }
  }
}

// As group_dot1 for one token column, with the x fragments in registers.
template <int BITS, class S, typename T>
__device__ __forceinline__ void group_dot_rx(const uint32_t (&rawA)[S::kRegs], const uint32_t (&rawB)[S::kRegs],
                                             const uint4 (&bf)[S::kSteps / 2], float (&d)[4], uint32_t magic) {
  constexpr int NP = S::kLPW / 2;
  uint32_t pA[S::kRegs * NP], pB[S::kRegs * NP];
#pragma unroll
  for (int k = 0; k < S::kRegs; ++k) {
    word_pairs<S>(rawA[k], magic, pA + k * NP);
    word_pairs<S>(rawB[k], magic, pB + k * NP);
  }
#pragma unroll
  for (int q = 0; q < S::kSteps; ++q) {
    const uint32_t b0 = (q & 1) ? bf[q >> 1].z : bf[q >> 1].x, b1 = (q & 1) ? bf[q >> 1].w : bf[q >> 1].y;
    if (q == 0)
      mma_first<T>(d, pA[0], pB[0], pA[1], pB[1], b0, b1);
    else
      mma16816<T>(d, pA[2 * q], pB[2 * q], pA[2 * q + 1], pB[2 * q + 1], b0, b1);
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

// Stage x for tokens [0, M) and groups [0, Gpad): per (token, group, quarter t)
// the kVirt values of quarter t in slot order (the codes' mma k order), zero
// past G; per (group, token) the fp32 sum of x over the group (and, for the
// two-nibble 8-bit form, the sum of the slot values x').
template <class S, typename T, int TOKP, int NX, int NTHR>
__device__ __forceinline__ void stage_x(const Params& p, int Gpad, int sid, uint8_t* xs, float* xsum) {
  constexpr int GS = S::kCodes * 4;
  const int ntask = p.M * Gpad * 4;
  for (int base = 0; base < ntask; base += NTHR) {
    const int idx = base + sid;
    const bool act = idx < ntask;
    const int tt = idx & 3, gq = idx >> 2;
    const int m = act ? gq / Gpad : 0, gl = act ? gq - m * Gpad : 0;
    float sb = 0.0f, so = 0.0f;
    if (act) {
      __align__(16) T xv[S::kCodes];
      if (gl < p.G) {
        const T* xa = reinterpret_cast<const T*>(p.x) + (int64_t)m * p.K + (int64_t)gl * GS + tt * S::kCodes;
        if ((reinterpret_cast<uintptr_t>(xa) & 15) == 0) {
#pragma unroll
          for (int c = 0; c < S::kCodes * (int)sizeof(T) / 16; ++c)
            reinterpret_cast<uint4*>(xv)[c] = __ldg(reinterpret_cast<const uint4*>(xa) + c);
        } else {
#pragma unroll
          for (int c = 0; c < S::kCodes; ++c) xv[c] = xa[c];
        }
      } else {
#pragma unroll
        for (int c = 0; c < S::kCodes * (int)sizeof(T) / 16; ++c)
          reinterpret_cast<uint4*>(xv)[c] = make_uint4(0u, 0u, 0u, 0u);
      }
      __align__(16) T outv[S::kVirt];
#pragma unroll
      for (int q = 0; q < S::kVirt; ++q) {
        const int vv = S::slot_virtual(q);
        const float mult = S::virt_mult(vv);
        const float xf = to_f32(xv[S::virt_code(vv)]) * mult;
        outv[q] = from_f32<T>(xf);
        so += xf;
        if (mult == 1.0f) sb += xf;
      }
      uint4* dst = reinterpret_cast<uint4*>(xs + (int64_t)m * p.tok_stride +
                                            (size_t)(gl * 4 + tt) * S::kVirt * sizeof(T));
#pragma unroll
      for (int q = 0; q < (int)(S::kVirt * sizeof(T) / 16); ++q)
        dst[q] = reinterpret_cast<const uint4*>(outv)[q];
    }
    sb += __shfl_xor_sync(0xffffffffu, sb, 1);
    so += __shfl_xor_sync(0xffffffffu, so, 1);
    sb += __shfl_xor_sync(0xffffffffu, sb, 2);
    so += __shfl_xor_sync(0xffffffffu, so, 2);
    if (act && tt == 0) {
      xsum[gl * TOKP + m] = sb;
      if constexpr (NX == 2) xsum[(Gpad + gl) * TOKP + m] = so;
    }
  }
  // padding tokens [M, TOKP) of the sums read as zero
  for (int idx = sid; idx < Gpad * TOKP * NX; idx += NTHR)
    if (idx % TOKP >= p.M) xsum[idx] = 0.0f;
}

template <int BITS, int GS, typename T, int MODE, int UG>
__global__ void __launch_bounds__(Cfg<BITS, GS, T, MODE, UG>::THREADS, 1)
qgemv_stream_kernel(const Params p, const __grid_constant__ CUtensorMap tmc,
                    const __grid_constant__ CUtensorMap tms, const __grid_constant__ CUtensorMap tmb) {
  using C = Cfg<BITS, GS, T, MODE, UG>;
  using S = typename C::S;
  constexpr int GPU = C::GPU, GPW = C::GPW, TOKP = C::TOKP, WPG = C::WPG, MT = C::MT, KC = C::KC;
  constexpr float OFF = S::kOff;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int STAGES = p.stages;
  const uint32_t code_ring = smem_u32(smem + p.off_code);
  const uint32_t sb_ring = smem_u32(smem + p.off_sb);
  const uint32_t bar_full = smem_u32(smem + p.off_bar);
  const uint32_t bar_empty = bar_full + 8 * kMaxStages;
  const uint32_t bar_pfull = bar_empty + 8 * kMaxStages;
  const uint32_t bar_pempty = bar_pfull + 8 * kRB;
  const uint32_t part_sa = smem_u32(smem + p.off_part);
  uint8_t* xs = smem + p.off_xs;
  float* xsum = reinterpret_cast<float*>(smem + p.off_xsum);

  const int tb = (int)((int64_t)p.ntiles * blockIdx.x / gridDim.x);
  const int te = (int)((int64_t)p.ntiles * (blockIdx.x + 1) / gridDim.x);
  const int nt = te - tb;
  const int nunits = nt * p.upt;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, KC);
    }
    for (int e = 0; e < kRB; ++e) {
      mbar_init(bar_pfull + 8 * e, KC);
      mbar_init(bar_pempty + 8 * e, 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // the next kernel in the stream may launch now; it waits for this grid's
  // completion before it reads anything this grid writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---------------------------------------------------------------- producer
  if (warp == C::PRODUCER) {
    if (lane == 0) {
      bool failed = false;
      int tile = tb, ku = 0, issued = 0;
      // L2 prefetch cursor: DRAM streams into L2 ahead of the ring, so the
      // copies into shared memory see L2 latency
      int pt = tb, pk = 0, pi = 0;
      auto prefetch_next = [&]() {
        if (pi < nunits) {
          tma_prefetch_3d(&tmc, 0, pt * 16, pk * C::Z);
          tma_prefetch_2d(&tms, pk * GPU, pt * 16);
          tma_prefetch_2d(&tmb, pk * GPU, pt * 16);
          ++pi;
          if (++pk == p.upt) { pk = 0; ++pt; }
        }
      };
      for (int i = 0; i < p.pf; ++i) prefetch_next();
      for (int i = 0; i < nunits; ++i) {
        if (p.pf > 0) prefetch_next();
        const int slot = i % STAGES;
        if (i >= STAGES && !mbar_wait(bar_empty + 8 * slot, (uint32_t)((i / STAGES) - 1) & 1u, false)) {
          failed = true;
          set_status(p.d_status, QMM_ERR_TIMEOUT);
          break;
        }
        const uint32_t fb = bar_full + 8 * slot;
        mbar_arrive_expect_tx(fb, C::TX);
        tma_load_3d(code_ring + (uint32_t)(slot * C::CODE_BYTES), &tmc, 0, tile * 16, ku * C::Z, fb);
        const uint32_t sd = sb_ring + (uint32_t)(slot * 2 * C::SB_BYTES);
        tma_load_2d(sd, &tms, ku * GPU, tile * 16, fb);
        tma_load_2d(sd + C::SB_BYTES, &tmb, ku * GPU, tile * 16, fb);
        issued = i + 1;
        if (++ku == p.upt) { ku = 0; ++tile; }
      }
      // no copy may still be landing when the CTA exits
      for (int i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
        if (!mbar_wait(bar_full + 8 * (i % STAGES), (uint32_t)(i / STAGES) & 1u, failed)) failed = true;
    }
    return;
  }

  // --------------------------------------------------- x staging (after the wait)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int Gpad = p.upt * GPU;
  stage_x<S, T, TOKP, C::NX, C::STAGERS>(p, Gpad, warp < KC ? tid : tid - 32, xs, xsum);
  asm volatile("bar.sync 1, %0;" ::"n"(C::STAGERS) : "memory");

  // ---------------------------------------------------------------- epilogue
  if (warp == C::EPILOGUE) {
    bool failed = false;
    for (int jt = 0; jt < nt; ++jt) {
      const int e = jt % kRB;
      const bool ok = mbar_wait(bar_pfull + 8 * e, (uint32_t)(jt / kRB) & 1u, failed);
      if (__any_sync(0xffffffffu, !ok)) {
        if (!failed && lane == 0) set_status(p.d_status, QMM_ERR_TIMEOUT);
        failed = true;
      }
      if (!failed) {
        if constexpr (C::ONE) {
          // partials: [entry][consumer][16 rows] floats
          if (lane < 16) {
            float y = 0.0f;
#pragma unroll
            for (int w = 0; w < KC; ++w) y += ldsf(part_sa + (uint32_t)(((e * KC + w) * 16 + lane) * 4));
            const int64_t row = (int64_t)(tb + jt) * 16 + lane;
            if (row < p.N) store_as(p.out, p.out_dtype, row, y);
          }
        } else {
          // partials: [entry][consumer][token tile][lane] float4 (the mma C fragment)
          for (int idx = lane; idx < 16 * p.M; idx += 32) {
            const int r = idx & 15, m = idx >> 4;
            const int mt = m >> 3, col = m & 7;
            const int src = ((r & 7) << 2) | (col >> 1);
            const int ci = ((r >> 3) << 1) | (col & 1);
            const uint32_t a0 = part_sa + (uint32_t)((((e * KC) * MT + mt) * 32 + src) * 16 + ci * 4);
            float y = 0.0f;
#pragma unroll
            for (int w = 0; w < KC; ++w) y += ldsf(a0 + (uint32_t)(w * MT * 32 * 16));
            const int64_t row = (int64_t)(tb + jt) * 16 + r;
            if (row < p.N) store_as(p.out, p.out_dtype, (int64_t)m * p.out_ld + row, y);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pempty + 8 * e);
    }
    return;
  }

  // --------------------------------------------------------------- consumers
  const int g = lane >> 2, t = lane & 3;
  const uint32_t xs_sa = smem_u32(xs), xsum_sa = smem_u32(xsum);
  // this warp's groups of a unit: ug = warp * GPW + u
  uint32_t xb[MT];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int tr = (mt * 8 + g) < p.M ? mt * 8 + g : 0;  // idle columns reread token 0
    xb[mt] = xs_sa + (uint32_t)(tr * p.tok_stride) + (uint32_t)(t * S::kVirt * (int)sizeof(T)) +
             (uint32_t)(warp * GPW * C::XG);
  }
  // per-group sums: tokens 2t, 2t + 1 (token 0 only for a single token)
  const uint32_t xsum_lane = xsum_sa + (uint32_t)((warp * GPW * TOKP + (C::ONE ? 0 : 2 * t)) * 4);
  // shared offsets (within a slot) of this lane's code words, row g, per group u
  uint32_t coff[GPW];
#pragma unroll
  for (int u = 0; u < GPW; ++u) {
    const int ug = warp * GPW + u;
    const int w0 = ug * WPG + t * S::kRegs;  // first word in the unit row
    const int wb = w0 & 31;
    coff[u] = (uint32_t)((w0 >> 5) * 2048 + g * 128 + (((wb >> 2) ^ g) << 4) + ((wb & 3) << 2));
  }
  const uint32_t magic = p.magic;
  // scale / bias offsets (within a slot) of rows g and g + 8 for this warp's groups
  // (row g's chunk c sits at chunk c ^ f(g); f is the same for row g + 8)
  constexpr int PITCH = GPU * 2;
  const int sfx = PITCH == 128 ? (g & 7) : PITCH == 64 ? ((g >> 1) & 3) : ((g >> 2) & 1);
  const int sbyte = warp * GPW * 2;
  const uint32_t soff = (uint32_t)(g * PITCH + ((((sbyte >> 4) ^ sfx)) << 4) + (sbyte & 15));

  float acc[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[mt][i] = 0.0f;
  bool failed = false;

  // unit i: slot i % STAGES with phase (i / STAGES) & 1, k-unit ku of tile jt
  int slot = 0, ku = 0, jt = 0;
  uint32_t phase = 0;
  uint32_t cslot = code_ring, sslot = sb_ring + soff, bfull = bar_full;
  uint32_t xbu[MT];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) xbu[mt] = xb[mt];
  uint32_t su = xsum_lane;
  // one token: this warp's x fragments and group sums of the current k-unit,
  // in registers (reloaded only when the k-unit changes)
  uint4 xr[C::ONE ? GPW : 1][S::kSteps / 2];
  float xsr[C::ONE ? GPW : 1][C::NX];
  int xku = -1;
  for (int i = 0; i < nunits; ++i) {
    bool ok = mbar_try_wait(bfull, phase);
    if (!ok) ok = mbar_wait(bfull, phase, failed);
    if (__any_sync(0xffffffffu, !ok)) {
      if (!failed && lane == 0) set_status(p.d_status, QMM_ERR_TIMEOUT);
      failed = true;
    }
    if constexpr (C::ONE) {
      if (ku != xku) {
        xku = ku;
#pragma unroll
        for (int u = 0; u < GPW; ++u) {
#pragma unroll
          for (int q2 = 0; q2 < S::kSteps / 2; ++q2) xr[u][q2] = lds128(xbu[0] + (uint32_t)(u * C::XG + q2 * 16));
          xsr[u][0] = ldsf(su + (uint32_t)(u * TOKP * 4));
          if constexpr (C::NX == 2) xsr[u][C::NX - 1] = ldsf(su + (uint32_t)((Gpad + u) * TOKP * 4));
        }
      }
    }
    if (!failed) {
      // GPW 16-bit scales (biases) of rows g and g + 8
      uint32_t sv[2][(GPW + 1) / 2], bv[2][(GPW + 1) / 2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t ra = sslot + (uint32_t)(h * 8 * GPU * 2);
        if constexpr (GPW == 1) {
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
        uint32_t rA[S::kRegs], rB[S::kRegs];
        const uint32_t ca = cslot + coff[u];
        if constexpr (S::kRegs >= 4) {
          const uint32_t cbase = ca & ~(uint32_t)127, c0 = (ca >> 4) & 7;  // row base, first chunk
#pragma unroll
          for (int k = 0; k < S::kRegs / 4; ++k) {
            const uint32_t ch = (uint32_t)(((c0 ^ (uint32_t)g) + k) ^ (uint32_t)g);
            const uint4 va = lds128(cbase + (ch << 4)), vb = lds128(cbase + 1024 + (ch << 4));
            rA[4 * k] = va.x; rA[4 * k + 1] = va.y; rA[4 * k + 2] = va.z; rA[4 * k + 3] = va.w;
            rB[4 * k] = vb.x; rB[4 * k + 1] = vb.y; rB[4 * k + 2] = vb.z; rB[4 * k + 3] = vb.w;
          }
        } else if constexpr (S::kRegs == 2) {
          const uint2 va = lds64(ca), vb = lds64(ca + 1024);
          rA[0] = va.x; rA[1] = va.y; rB[0] = vb.x; rB[1] = vb.y;
        } else {
          rA[0] = lds32(ca);
          rB[0] = lds32(ca + 1024);
        }
        float d[MT][4];
        if constexpr (C::ONE)
          group_dot_rx<BITS, S, T>(rA, rB, xr[u], d[0], magic);
        else
          group_dot1<BITS, S, T, MT>(rA, rB, xbu, (uint32_t)(u * C::XG), d, magic);
        const int hw = u & 1;
        const float sa = half_to_f32<T>(sv[0][u >> 1], hw), sb_ = half_to_f32<T>(sv[1][u >> 1], hw);
        const float ba = half_to_f32<T>(bv[0][u >> 1], hw), bb = half_to_f32<T>(bv[1][u >> 1], hw);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          if constexpr (C::ONE) {
            const float X0 = xsr[u][0];
            if constexpr (C::NX == 1) {
              acc[0][0] = fmaf(fmaf(-OFF, sa, ba), X0, fmaf(sa, d[0][0], acc[0][0]));
              acc[0][2] = fmaf(fmaf(-OFF, sb_, bb), X0, fmaf(sb_, d[0][2], acc[0][2]));
            } else {
              const float O0 = xsr[u][C::NX - 1];
              acc[0][0] = fmaf(ba, X0, fmaf(-OFF * sa, O0, fmaf(sa, d[0][0], acc[0][0])));
              acc[0][2] = fmaf(bb, X0, fmaf(-OFF * sb_, O0, fmaf(sb_, d[0][2], acc[0][2])));
            }
          } else {
            const uint2 xr = lds64(su + (uint32_t)((u * TOKP + mt * 8) * 4));
            const float X0 = __uint_as_float(xr.x), X1 = __uint_as_float(xr.y);
            if constexpr (C::NX == 1) {
              const float ca_ = fmaf(-OFF, sa, ba), cb_ = fmaf(-OFF, sb_, bb);
              acc[mt][0] = fmaf(ca_, X0, fmaf(sa, d[mt][0], acc[mt][0]));
              acc[mt][1] = fmaf(ca_, X1, fmaf(sa, d[mt][1], acc[mt][1]));
              acc[mt][2] = fmaf(cb_, X0, fmaf(sb_, d[mt][2], acc[mt][2]));
              acc[mt][3] = fmaf(cb_, X1, fmaf(sb_, d[mt][3], acc[mt][3]));
            } else {
              // bias term on sum(x), offset term on sum(x') (x' = x and 16 x)
              const uint2 xo = lds64(su + (uint32_t)(((Gpad + u) * TOKP + mt * 8) * 4));
              const float O0 = __uint_as_float(xo.x), O1 = __uint_as_float(xo.y);
              const float oa = -OFF * sa, ob = -OFF * sb_;
              acc[mt][0] = fmaf(ba, X0, fmaf(oa, O0, fmaf(sa, d[mt][0], acc[mt][0])));
              acc[mt][1] = fmaf(ba, X1, fmaf(oa, O1, fmaf(sa, d[mt][1], acc[mt][1])));
              acc[mt][2] = fmaf(bb, X0, fmaf(ob, O0, fmaf(sb_, d[mt][2], acc[mt][2])));
              acc[mt][3] = fmaf(bb, X1, fmaf(ob, O1, fmaf(sb_, d[mt][3], acc[mt][3])));
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bfull + 8 * kMaxStages);  // the slot's `empty` barrier

    if (++ku == p.upt) {  // tile done: post this warp's partial
      const int e = jt & (kRB - 1);
      if (jt >= kRB) {
        const bool okp = mbar_wait(bar_pempty + 8 * e, (uint32_t)((jt / kRB) - 1) & 1u, failed);
        if (__any_sync(0xffffffffu, !okp)) {
          if (!failed && lane == 0) set_status(p.d_status, QMM_ERR_TIMEOUT);
          failed = true;
        }
      }
      if constexpr (C::ONE) {
        if (t == 0) {
          sts32(part_sa + (uint32_t)(((e * KC + warp) * 16 + g) * 4), acc[0][0]);
          sts32(part_sa + (uint32_t)(((e * KC + warp) * 16 + g + 8) * 4), acc[0][2]);
        }
      } else {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
          sts128(part_sa + (uint32_t)((((e * KC + warp) * MT + mt) * 32 + lane) * 16),
                 make_float4(acc[mt][0], acc[mt][1], acc[mt][2], acc[mt][3]));
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[mt][k] = 0.0f;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_pfull + 8 * e);
      ku = 0;
      ++jt;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) xbu[mt] = xb[mt];
      su = xsum_lane;
    } else {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) xbu[mt] += (uint32_t)(GPU * C::XG);
      su += (uint32_t)(GPU * TOKP * 4);
    }
    if (++slot == STAGES) {
      slot = 0;
      phase ^= 1u;
      cslot = code_ring;
      sslot = sb_ring + soff;
      bfull = bar_full;
    } else {
      cslot += (uint32_t)C::CODE_BYTES;
      sslot += (uint32_t)(2 * C::SB_BYTES);
      bfull += 8;
    }
  }
}

// ------------------------------------------------------------------ host side
// 3-D map over packed words [rows, wpr] seen as (word in slice, row, slice of
// 32 words): a box is 16 rows x z slices, each slice 16 x 128 bytes, swizzled.
inline bool make_code_map3(CUtensorMap* map, const uint32_t* packed, int64_t rows, int64_t wpr, int z) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {32, (cuuint64_t)rows, (cuuint64_t)(wpr / 32)};
  const cuuint64_t strides[2] = {(cuuint64_t)(wpr * 4), 128};
  const cuuint32_t box[3] = {32, 16, (cuuint32_t)z};
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
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dense calls only (no ids, one matrix); cudaErrorNotSupported sends the caller
// to the general kernels.
template <int BITS, int GS, typename T, int MODE, int UG>
cudaError_t launch_stream(const QgemvParams& q, cudaStream_t st) {
  using C = Cfg<BITS, GS, T, MODE, UG>;
  if (q.ids || q.amode != 0 || q.n_pairs < 1 || q.n_pairs > C::TOKP) return cudaErrorNotSupported;
  if (q.G % 8 != 0 || q.wpr % 32 != 0 || q.n_rows < 16 || q.G < C::GPU) return cudaErrorNotSupported;
  if (((uintptr_t)q.packed[0] | (uintptr_t)q.scales[0] | (uintptr_t)q.biases[0]) & 15) return cudaErrorNotSupported;

  Params p{};
  p.x = q.a;
  p.M = q.n_pairs;
  p.K = q.K;
  p.G = q.G;
  p.upt = (q.G + C::GPU - 1) / C::GPU;
  p.N = q.n_rows;
  p.ntiles = (int)((q.n_rows + 15) / 16);
  p.out = q.out;
  p.out_dtype = q.out_dtype;
  p.out_ld = q.out_ld;
  p.d_status = q.d_status;
  p.magic = C::S::kMagic;
  const int Gpad = p.upt * C::GPU;
  p.tok_stride = Gpad * C::XG + 16;

  // [codes (1024-aligned) | scales+biases | mbarriers | partials | x | sums]
  const size_t part = C::ONE ? (size_t)kRB * C::KC * 16 * 4 : (size_t)kRB * C::KC * C::MT * 32 * 16;
  const size_t xs = align128((size_t)p.M * p.tok_stride);
  const size_t xsum = align128((size_t)Gpad * C::TOKP * 4 * C::NX);
  const size_t bars = 8 * (2 * kMaxStages + 2 * kRB);
  auto total = [&](int stages) {
    return 1024 + (size_t)stages * C::CODE_BYTES + align128((size_t)stages * 2 * C::SB_BYTES) + align128(bars) +
           part + xs + xsum;
  };
  // about 144 KB of the weight stream in flight per SM (measured: deeper rings
  // and an L2 prefetch window ahead of the ring were not faster)
  int stages = (int)((144 * 1024) / C::TX);
  stages = stages < 2 ? 2 : (stages > kMaxStages ? kMaxStages : stages);
  while (stages > 2 && total(stages) > (size_t)kSmemMax) --stages;
  if (total(stages) > (size_t)kSmemMax) return cudaErrorNotSupported;
  p.stages = stages;
  p.pf = 0;  // L2 prefetch window (units); off: measured no faster than the ring alone
  p.off_code = 0;
  p.off_sb = stages * C::CODE_BYTES;
  p.off_bar = p.off_sb + (int)align128((size_t)stages * 2 * C::SB_BYTES);
  p.off_part = p.off_bar + (int)align128(bars);
  p.off_xs = p.off_part + (int)part;
  p.off_xsum = p.off_xs + (int)xs;
  const size_t smem = total(stages);

  CUtensorMap tmc, tms, tmb;
  if (!make_code_map3(&tmc, q.packed[0], q.n_rows, q.wpr, C::Z) ||
      !make_sb_map(&tms, q.scales[0], q.n_rows, q.G, C::GPU) || !make_sb_map(&tmb, q.biases[0], q.n_rows, q.G, C::GPU))
    return cudaErrorNotSupported;

  auto k = qgemv_stream_kernel<BITS, GS, T, MODE, UG>;
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  const int grid = std::min(qmm_host::num_sms(), p.ntiles);
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
  return cudaLaunchKernelEx(&cfg, k, p, tmc, tms, tmb);
}

template <int BITS, int GS, typename T>
cudaError_t try_stream_mt(const QgemvParams& q, int mt, cudaStream_t st) {
  using S = Share<BITS, GS, T>;
  if constexpr (S::kFast) {
    constexpr int WPG = S::kWordsPerGroup;
    constexpr int UB = WPG >= 32 ? 16 : 32;           // base unit
    constexpr int UW = WPG <= 8 ? 64 : UB;            // wide unit: 4 groups per consumer
    const bool wide = (q.G % UW) == 0;
    if (q.n_pairs == 1)
      return wide ? launch_stream<BITS, GS, T, 0, UW>(q, st) : launch_stream<BITS, GS, T, 0, UB>(q, st);
    if (mt == 1)
      return wide ? launch_stream<BITS, GS, T, 1, UW>(q, st) : launch_stream<BITS, GS, T, 1, UB>(q, st);
    return launch_stream<BITS, GS, T, 2, UB>(q, st);
  } else {
    return cudaErrorNotSupported;
  }
}

// Entry from the per-bit-width files: the streaming kernel for dense calls of
// one matrix, cudaErrorNotSupported for everything else.
template <int BITS>
cudaError_t try_stream(const QgemvParams& q, int gs, int dtype, int mt, bool dual, cudaStream_t st) {
  if (dual || q.ids) return cudaErrorNotSupported;
  if (dtype == QMM_BF16) {
    if (gs == 32) return try_stream_mt<BITS, 32, __nv_bfloat16>(q, mt, st);
    if (gs == 64) return try_stream_mt<BITS, 64, __nv_bfloat16>(q, mt, st);
    return try_stream_mt<BITS, 128, __nv_bfloat16>(q, mt, st);
  }
  if (gs == 32) return try_stream_mt<BITS, 32, __half>(q, mt, st);
  if (gs == 64) return try_stream_mt<BITS, 64, __half>(q, mt, st);
  return try_stream_mt<BITS, 128, __half>(q, mt, st);
}

}  // namespace stream
}  // namespace qmm
