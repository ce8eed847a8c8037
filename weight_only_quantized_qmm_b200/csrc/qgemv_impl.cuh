// Decode-shaped quantized matmul (M <= 16) and the MoE indirect-dispatch GEMV,
// dense and fused gate+up+SiLU, in one kernel family: the shared pieces (the
// share layout, conversions, x staging, the expert plan) and the cp.async
// kernel that serves every shape the streaming and TMA kernels decline
// (3- and 6-bit codes, half-word shares, short rows).
//
// What is computed:
//   dense   y[m, n]   = sum_k x[m, k] * w_hat[n, k]
//           ("emily 0.5.1 lib/emily/quantization.ex", quantized_matmul/2)
//   MoE     out[p, n] = sum_k a_p[k] * w_hat_{ids[p]}[n, k]
//   fused   out[p, n] = SiLU(sum_k a_p[k] gate[n, k]) * sum_k a_p[k] up[n, k]
//           ("ferrum-kernels 0.7.7 src/stacked_expert.rs", gemv_moe_id*,
//            gemv_moe_id_gate_up_silu*)
//   with w_hat = q * s_g + b_g (affine groups of GS columns).
//
// How (sm_100a):
//   * The affine factor of each group is pulled out of the reduction:
//       sum_{k in g} x_k (q_k s_g + b_g) = s_g * sum q_k x_k + b_g * sum x_k.
//     The integer part runs on the tensor cores with mma.sync.m16n8k16
//     (bf16 or f16 operands, fp32 accumulate): 16 weight rows form the A
//     operand, up to 8 tokens the B operand.  A pair of codes becomes two
//     exact 16-bit floats with one LOP3 ((lanes & mask) | 0x4300 for bf16 =
//     128 + q, 0x6400 for f16 = 1024 + q).  8-bit codes in bf16 are split into
//     two nibble slots (x and 16 x) because 128 + q > 255 is not exact in bf16.
//   * Each mma's 16 k-slots belong to one quantization group (the 4 threads of
//     a quad each hold one quarter of the group of their two rows), so the
//     fp32 result d_g is scaled by s_g in one FFMA.  The k order inside a
//     thread's quarter is free; x is staged in shared memory in that order.
//   * The terms that do not depend on the codes, b_g * sum x and
//     -OFF * s_g * sum x', are contractions over groups; they run as one extra
//     mma pair per 8 groups with A = (b_g or s_g, exact as stored) and B = the
//     per-group sums split into hi + lo 16-bit parts.
//   * Packed codes and the scale/bias words stream global -> shared with
//     cp.async through a 4-stage ring per warp (no registers in flight, no
//     spin-waits), 16 warps per CTA, one CTA per SM.  The rows are split evenly
//     over the CTAs at row granularity, so every SM streams the same number of
//     bytes.
//   * MoE: every CTA builds the expert -> pairs lists of the call in shared
//     memory (counting by expert), takes its slice of the rows of the
//     distinct experts, and each expert's packed rows are read once however
//     many pairs use it.
#pragma once

#include <algorithm>

#include "qgemv.cuh"

namespace qmm {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxTok = 16;
constexpr int kSmemMax = 226 * 1024;  // dynamic shared memory opt-in per CTA (static use is tiny)

// Layout of one thread's quarter ("share") of one group of one row.
template <int BITS, int GS, typename T>
struct Share {
  static constexpr bool kF16 = std::is_same<T, __half>::value;
  static constexpr bool kSplit = (BITS == 8) && !kF16;       // bf16: 8-bit code -> 2 nibble slots
  static constexpr int kCodes = GS / 4;                       // real codes in the share
  static constexpr int kVirt = kSplit ? 2 * kCodes : kCodes;  // mma k-slots in the share
  static constexpr int kSteps = kVirt / 4;                    // m16n8k16 steps per group
  static constexpr int kBitsShare = kCodes * BITS;
  static constexpr bool kAligned = (kBitsShare % 32) == 0;
  static constexpr int kRegs = (kBitsShare + 31) / 32;
  static constexpr int kWordsPerGroup = GS * BITS / 32;
  // integral-lane fast path (whole words of 2-, 4- or 8-bit lanes)
  static constexpr bool kFast = kAligned && (BITS == 2 || BITS == 4 || BITS == 8);
  static constexpr int kLW = kSplit ? 4 : BITS;  // lane width in the fast path
  static constexpr int kLPW = 32 / kLW;          // lanes per word
  static constexpr uint32_t kLaneMask = (1u << kLW) - 1u;
  static constexpr uint32_t kMask2 = kLaneMask | (kLaneMask << 16);
  static constexpr uint32_t kMagic = kF16 ? 0x64006400u : 0x43004300u;
  static constexpr float kOff = kF16 ? 1024.0f : 128.0f;
  static_assert(kVirt % 4 == 0, "share must fill whole mma steps");

  // slot p of the share (mma k order) -> virtual code v
  __host__ __device__ static constexpr int slot_virtual(int p) {
    if (!kFast) return p;
    const int i = p >> 1, h = p & 1;
    const int wi = i / (kLPW / 2), j = i % (kLPW / 2);
    return wi * kLPW + j + h * (kLPW / 2);
  }
  // virtual code -> real code index inside the share, and x multiplier
  __host__ __device__ static constexpr int virt_code(int v) { return kSplit ? (v >> 1) : v; }
  __host__ __device__ static constexpr float virt_mult(int v) { return (kSplit && (v & 1)) ? 16.0f : 1.0f; }
};

// ------------------------------------------------------------------ loads
// cp.async (LDGSTS): global -> shared without registers; src_bytes < bytes
// zero-fills the rest (src_bytes = 0 reads nothing).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N)); }
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
// 16-bit float bits -> fp32 (bf16: the top half of an fp32; f16: exact widening)
template <typename T>
__device__ __forceinline__ float half_bits_to_f32(uint32_t h) {
  if constexpr (std::is_same<T, __half>::value) return __half2float(__ushort_as_half((unsigned short)h));
  else return __uint_as_float(h << 16);
}

// Copy this thread's share of one group of one row into its ring slot
// (kSlot words).  ok = false zero-fills the slot without reading memory.
template <class S>
__device__ __forceinline__ void copy_share(uint32_t dst, const uint32_t* grp, int t, bool ok,
                                           const uint32_t* safe) {
  if constexpr (S::kAligned) {
    const uint32_t* src = grp + t * S::kRegs;
    if constexpr (S::kRegs % 4 == 0) {
#pragma unroll
      for (int i = 0; i < S::kRegs / 4; ++i) cp_async16(dst + 16 * i, ok ? src + 4 * i : safe, ok ? 16u : 0u);
    } else if constexpr (S::kRegs % 2 == 0) {
#pragma unroll
      for (int i = 0; i < S::kRegs / 2; ++i) cp_async8(dst + 8 * i, ok ? src + 2 * i : safe, ok ? 8u : 0u);
    } else {
#pragma unroll
      for (int i = 0; i < S::kRegs; ++i) cp_async4(dst + 4 * i, ok ? src + i : safe, ok ? 4u : 0u);
    }
  } else {
    // share starts inside a word: the one or two words covering it
    const int bit = t * S::kBitsShare;
    const int w = bit >> 5, sh = bit & 31;
    const bool two = ok && (sh + S::kBitsShare > 32);
    cp_async4(dst, ok ? grp + w : safe, ok ? 4u : 0u);
    cp_async4(dst + 4, two ? grp + w + 1 : safe, two ? 4u : 0u);
  }
}

template <class S>
constexpr int slot_words() { return S::kAligned ? S::kRegs : 2; }

// Read a share back from its ring slot (shared address) into registers,
// bit 0 = first code of the share.
template <class S>
__device__ __forceinline__ void read_share(uint32_t slot, int t, uint32_t (&r)[S::kRegs]) {
  if constexpr (S::kAligned) {
    if constexpr (S::kRegs % 4 == 0) {
#pragma unroll
      for (int i = 0; i < S::kRegs / 4; ++i) {
        const uint4 v = lds128(slot + 16 * i);
        r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
      }
    } else if constexpr (S::kRegs % 2 == 0) {
#pragma unroll
      for (int i = 0; i < S::kRegs / 2; ++i) {
        const uint2 v = lds64(slot + 8 * i);
        r[2 * i] = v.x; r[2 * i + 1] = v.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < S::kRegs; ++i) r[i] = lds32(slot + 4 * i);
    }
  } else {
    const int sh = (t * S::kBitsShare) & 31;
    const uint2 v = lds64(slot);
    r[0] = __funnelshift_r(v.x, v.y, sh);
    if constexpr (S::kRegs > 1) r[1] = v.y >> sh;
  }
}

// pair i of a share as packed 16-bit floats: slots (2i, 2i+1) = (OFF + v_lo, OFF + v_hi)
template <int BITS, class S>
__device__ __forceinline__ uint32_t share_pair(const uint32_t (&r)[S::kRegs], int i) {
  if constexpr (S::kFast) {
    const int wi = i / (S::kLPW / 2), j = i % (S::kLPW / 2);
    return ((r[wi] >> (j * S::kLW)) & S::kMask2) | S::kMagic;
  } else {
    const uint32_t c0 = stream_code<BITS>(r, 2 * i);
    const uint32_t c1 = stream_code<BITS>(r, 2 * i + 1);
    return c0 | (c1 << 16) | S::kMagic;
  }
}

template <typename T>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (std::is_same<T, __half>::value) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ int64_t pair_offset(const QgemvParams& p, int pair) {
  switch (p.amode) {
    case 0: return (int64_t)pair * p.K;
    case 1: return (int64_t)pair * p.stride;
    case 2: return (int64_t)(pair / p.top_k) * p.outer + (int64_t)(pair % p.top_k) * p.inner;
    default: return 0;
  }
}

// Every CTA builds, in shared memory, the expert -> pairs lists of the call
// (a counting sort by expert id) and the list of distinct experts; dense calls
// have one "expert" whose pairs are the M tokens.  A pair with an id outside
// [0, E) gets a zero output row (written by CTA 0) and QMM_ERR_BAD_EXPERT_ID.
// s_ids (n_pairs ints) holds the ids read once from global memory.
__device__ __forceinline__ void build_plan(const QgemvParams& p, int* s_cnt, int* s_start,
                                           int* s_fill, int* s_dist, int* s_list, int* s_ids, int* s_nd) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nthr = blockDim.x;
  const int E = p.num_experts;
  if (p.ids == nullptr) {
    for (int i = tid; i < p.n_pairs; i += nthr) s_list[i] = i;
    if (tid == 0) { s_cnt[0] = p.n_pairs; s_start[0] = 0; s_dist[0] = 0; *s_nd = 1; }
    __syncthreads();
  } else {
    for (int e = tid; e < E; e += nthr) { s_cnt[e] = 0; s_fill[e] = 0; }
    __syncthreads();
    for (int i = tid; i < p.n_pairs; i += nthr) {
      const int e = p.ids[i];
      s_ids[i] = e;
      if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scans over experts: pair starts and distinct list
      int run = 0, nd = 0;
      for (int base = 0; base < E; base += 32) {
        const int e = base + lane;
        const int c = e < E ? s_cnt[e] : 0;
        int incl = c, dincl = c > 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          const int dv = __shfl_up_sync(0xffffffffu, dincl, o);
          if (lane >= o) { incl += v; dincl += dv; }
        }
        if (e < E) {
          s_start[e] = run + incl - c;
          if (c > 0) s_dist[nd + dincl - 1] = e;
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
        nd += __shfl_sync(0xffffffffu, dincl, 31);
      }
      if (lane == 0) *s_nd = nd;
    }
    __syncthreads();
    // stable placement (pairs of an expert in increasing pair order), so that
    // every CTA derives the same lists: one warp ranks 32 pairs at a time
    if (warp == 0) {
      for (int base = 0; base < p.n_pairs; base += 32) {
        const int i = base + lane;
        const int e = i < p.n_pairs ? s_ids[i] : -1;
        const bool valid = e >= 0 && e < E;
        const unsigned same = __match_any_sync(0xffffffffu, valid ? e : E + lane);
        if (valid) {
          const int rank = s_fill[e] + __popc(same & ((1u << lane) - 1u));
          s_list[s_start[e] + rank] = i;
        }
        __syncwarp();
        if (valid && lane == 31 - __clz(same)) s_fill[e] += __popc(same);
        __syncwarp();
      }
    }
    if (blockIdx.x == 0) {
      for (int i = tid; i < p.n_pairs; i += nthr) {
        const int e = s_ids[i];
        if (e < 0 || e >= E) {  // bad id: zero row, report
          for (int64_t n = 0; n < p.n_rows; ++n) store_as(p.out, p.out_dtype, (int64_t)i * p.out_ld + n, 0.0f);
          set_status(p.d_status, QMM_ERR_BAD_EXPERT_ID);
        }
      }
    }
    __syncthreads();
  }

}

// Stage x for groups [gc0, gc0 + gcn) of `ntok` pairs in share-slot order
// (one group quarter per thread), and per (group, token) the hi + lo 16-bit
// splits of sum(x) (bias term) and of -OFF * sum(x') (offset term; the plain
// sum(x') when SEP_S) for the correction mma.
template <class S, typename T, int TOKP, bool SEP_S>
__device__ __forceinline__ void stage_x(const QgemvParams& p, const int* pairs, int ntok, int gc0,
                                        int gcn, T* xs, uint2* xrec) {
  constexpr int GS = S::kCodes * 4;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int nblk = ntok * gcn * 4;
  for (int base = 0; base < nblk; base += nthr) {
    const int idx = base + tid;
    const bool act = idx < nblk;
    float sc = 0.0f, sb = 0.0f;
    const int tt = idx & 3, gq = idx >> 2;
    const int tk = act ? gq / gcn : 0, gl = act ? gq - tk * gcn : 0;
    if (act) {
      const T* xa = reinterpret_cast<const T*>(p.a) + pair_offset(p, pairs[tk]) +
                    (int64_t)(gc0 + gl) * GS + tt * S::kCodes;
      __align__(16) T xv[S::kCodes];
      if ((reinterpret_cast<uintptr_t>(xa) & 15) == 0) {
#pragma unroll
        for (int c = 0; c < S::kCodes * (int)sizeof(T) / 16; ++c)
          reinterpret_cast<uint4*>(xv)[c] = __ldg(reinterpret_cast<const uint4*>(xa) + c);
      } else {
#pragma unroll
        for (int c = 0; c < S::kCodes; ++c) xv[c] = xa[c];
      }
      __align__(16) T outv[S::kVirt];
#pragma unroll
      for (int q = 0; q < S::kVirt; ++q) {
        const int vv = S::slot_virtual(q);
        const float m = S::virt_mult(vv);
        const float xf = to_f32(xv[S::virt_code(vv)]) * m;
        outv[q] = from_f32<T>(xf);
        sc += xf;
        if (m == 1.0f) sb += xf;
      }
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(xs) + (int64_t)tk * p.tok_stride +
                                            (size_t)(gl * 4 + tt) * S::kVirt * sizeof(T));
#pragma unroll
      for (int q = 0; q < (int)(S::kVirt * sizeof(T) / 16); ++q)
        dst[q] = reinterpret_cast<const uint4*>(outv)[q];
    }
    sc += __shfl_xor_sync(0xffffffffu, sc, 1);
    sb += __shfl_xor_sync(0xffffffffu, sb, 1);
    sc += __shfl_xor_sync(0xffffffffu, sc, 2);
    sb += __shfl_xor_sync(0xffffffffu, sb, 2);
    if (act && tt == 0) {
      const float so = SEP_S ? sc : -S::kOff * sc;
      const T bh = from_f32<T>(sb), oh = from_f32<T>(so);
      const T bl = from_f32<T>(sb - to_f32(bh)), ol = from_f32<T>(so - to_f32(oh));
      uint2 rec;
      rec.x = (uint32_t)bits16(bh) | ((uint32_t)bits16(bl) << 16);
      rec.y = (uint32_t)bits16(oh) | ((uint32_t)bits16(ol) << 16);
      xrec[gl * TOKP + tk] = rec;
    }
  }
}

// Sum the K-slice partials of a row block (the bias and offset terms are
// already inside them), apply SiLU(gate) * up for the fused form, and store
// one value per (row, pair).
template <int TOKP, int NS, bool DUAL>
__device__ __forceinline__ void reduce_store(const QgemvParams& p, const float* part, int tiles,
                                             int KS, int ntok, int64_t blk_row0, int64_t r1,
                                             const int* pairs) {
  const int nthr = blockDim.x;
  for (int it = threadIdx.x; it < tiles * 16 * ntok; it += nthr) {
    const int tl = it / (16 * ntok);
    const int rr = (it / ntok) % 16;
    const int tk = it % ntok;
    const int64_t row = blk_row0 + 16 * (int64_t)tl + rr;
    if (row >= r1) continue;
    float y0 = 0.0f, y1 = 0.0f;
    for (int s = 0; s < KS; ++s) {
      const float* pp = part + (((tl * KS + s) * 16 + rr) * TOKP + tk) * NS;
      y0 += pp[0];
      if (DUAL) y1 += pp[1];
    }
    float yv = y0;
    if (DUAL) yv = y0 / (1.0f + expf(-y0)) * y1;
    store_as(p.out, p.out_dtype, (int64_t)pairs[tk] * p.out_ld + row, yv);
  }
}

// Tensor-core partial dot of one group for 16 rows x TOKP tokens: d = sum over
// the group's k-slots of (OFF + v) * x'.  Even and odd k16 steps accumulate
// into separate registers so consecutive mmas do not wait on each other.
template <int BITS, class S, typename T, int MT>
__device__ __forceinline__ void group_dot(const uint32_t (&rawA)[S::kRegs],
                                          const uint32_t (&rawB)[S::kRegs],
                                          const uint32_t (&xb)[MT], uint32_t xo,
                                          float (&d)[MT][4]) {
  float e[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) { d[mt][i] = 0.0f; e[mt][i] = 0.0f; }
#pragma unroll
  for (int q2 = 0; q2 < S::kSteps / 2; ++q2) {
    uint4 bf[MT];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) bf[mt] = lds128(xb[mt] + xo + q2 * 16);
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int q = 2 * q2 + h2;
      const uint32_t a0 = share_pair<BITS, S>(rawA, 2 * q);
      const uint32_t a1 = share_pair<BITS, S>(rawB, 2 * q);
      const uint32_t a2 = share_pair<BITS, S>(rawA, 2 * q + 1);
      const uint32_t a3 = share_pair<BITS, S>(rawB, 2 * q + 1);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        if (h2 == 0)
          mma16816<T>(d[mt], a0, a1, a2, a3, bf[mt].x, bf[mt].y);
        else
          mma16816<T>(e[mt], a0, a1, a2, a3, bf[mt].z, bf[mt].w);
      }
    }
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) d[mt][i] += e[mt][i];
}

// ------------------------------------------------------------------ kernel
template <int BITS, int GS, typename T, int MT, bool DUAL>
struct QgemvCfg {
  using S = Share<BITS, GS, T>;
  static constexpr int NS = DUAL ? 2 : 1;
  static constexpr int SLOT = slot_words<S>();                // words per code share slot
  static constexpr int UG0 = 8 / (SLOT * NS);
  static constexpr int UG = UG0 < 1 ? 1 : UG0;                // groups per pipeline stage: 1, 2, 4 or 8
  static constexpr int SBW = UG == 1 ? 1 : UG / 2 + 1;        // scale (or bias) words per row per stage
  static constexpr int QW = NS * 2 * 2 * SBW;                 // scale+bias words per quad per stage
  static constexpr int STAGES = 4;
  static constexpr int CODE_WORDS = UG * NS * 2 * SLOT * 32;  // per warp per stage
  static constexpr int STAGE_WORDS = CODE_WORDS + 8 * QW;     // + the 8 quads' scale/bias words
  static constexpr int RING_BYTES = STAGES * STAGE_WORDS * 4; // per warp
  static constexpr int TOKP = MT * 8;
  static constexpr int CB = (UG + 7) / 8;                     // correction mmas per stage
  // f16 keeps the -OFF * s * sum(x') term in its own accumulator (OFF * sum(x')
  // may not fit f16); bf16 folds it into the main accumulator
  static constexpr bool SEP_S = std::is_same<T, __half>::value;
};

__device__ __forceinline__ uint32_t dup16(uint32_t v) { return __byte_perm(v, 0, 0x1010); }

template <int BITS, int GS, typename T, int MT, bool DUAL>
__global__ void __launch_bounds__(kThreads, 1) qgemv_kernel(const QgemvParams p) {
  using C = QgemvCfg<BITS, GS, T, MT, DUAL>;
  using S = typename C::S;
  constexpr int NS = C::NS, UG = C::UG, STAGES = C::STAGES, TOKP = C::TOKP, SBW = C::SBW;
  extern __shared__ __align__(128) uint8_t smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;

  int* s_cnt = reinterpret_cast<int*>(smem + p.off_plan);
  const int E = p.num_experts;
  int* s_start = s_cnt + E;
  int* s_fill = s_start + E;
  int* s_dist = s_fill + E;
  int* s_list = s_dist + E;
  __shared__ int s_nd;
  T* xs = reinterpret_cast<T*>(smem + p.off_xs);               // [ntok][kchunk][4][kVirt] (+pad)
  uint2* xrec = reinterpret_cast<uint2*>(smem + p.off_xsum);   // [kchunk][TOKP] {sum x hi,lo | sum x' hi,lo}
  float* part = reinterpret_cast<float*>(smem + p.off_part);   // [kWarps][16][TOKP][NS]
  const uint32_t ring_base = smem_u32(smem + p.off_ring + warp * C::RING_BYTES);

  build_plan(p, s_cnt, s_start, s_fill, s_dist, s_list, s_list + p.n_pairs, &s_nd);

  const int64_t V = (int64_t)s_nd * p.n_rows;
  const int64_t v0 = V * blockIdx.x / gridDim.x;
  const int64_t v1 = V * (blockIdx.x + 1) / gridDim.x;
  const int nchunks = (p.G + p.kchunk - 1) / p.kchunk;
  const uint32_t* safe_src = p.packed[0];  // any valid address, for zero-fill copies
  const uint32_t xs_sa = smem_u32(xs);
  const uint32_t xrec_sa = smem_u32(xrec);

  for (int64_t v = v0; v < v1;) {
    const int64_t j = v / p.n_rows;
    const int64_t r0 = v - j * p.n_rows;
    const int64_t r1 = min(v1 - j * p.n_rows, p.n_rows);
    const int e = s_dist[j];
    const int64_t ebase = (int64_t)e * p.n_rows;  // first packed row of the expert
    v = j * p.n_rows + r1;

    const int cnt = s_cnt[e];
    for (int tc = 0; tc < cnt; tc += p.tok_cap) {
      const int ntok = min(p.tok_cap, cnt - tc);
      const int* pairs = s_list + s_start[e] + tc;

      const int RT = (int)((r1 - r0 + 15) / 16);
      for (int rb = 0; rb < RT; rb += kWarps) {
        const int tiles = min(kWarps, RT - rb);
        const int KS = kWarps / tiles;
        const bool active = warp < tiles * KS;
        const int tile = warp / KS, slice = warp % KS;
        const int64_t blk_row0 = r0 + 16 * (int64_t)rb;       // first row of the row block
        const int64_t trow = blk_row0 + 16 * (int64_t)tile;   // first row of the tile
        const int rows_valid = active ? (int)(r1 - trow < 16 ? r1 - trow : 16) : 0;
        const bool vrow[2] = {g < rows_valid, g + 8 < rows_valid};
        const int64_t rowg[2] = {ebase + trow + g, ebase + trow + g + 8};

        float acc[NS][MT][4], accs[NS][MT][4];
#pragma unroll
        for (int s = 0; s < NS; ++s)
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) { acc[s][mt][i] = 0.0f; accs[s][mt][i] = 0.0f; }

        // per-item constants
        const uint32_t* crow[NS][2];  // packed code rows
        const uint32_t* srow[NS][2][2];  // [stack][row][scales|biases] as words (element row*G)
        int64_t rowG[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          rowG[h] = rowg[h] * p.G;
#pragma unroll
          for (int s = 0; s < NS; ++s) {
            crow[s][h] = p.packed[s] + rowg[h] * p.wpr;
            srow[s][h][0] = reinterpret_cast<const uint32_t*>(p.scales[s]);
            srow[s][h][1] = reinterpret_cast<const uint32_t*>(p.biases[s]);
          }
        }
        int tokrow[MT];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) tokrow[mt] = (mt * 8 + g) < ntok ? mt * 8 + g : 0;

        for (int ch = 0; ch < nchunks; ++ch) {
          const int gc0 = ch * p.kchunk;
          const int gcn = min(p.kchunk, p.G - gc0);
          // stages of UG groups, split evenly over the KS slices of the tile
          const int nstg = (gcn + UG - 1) / UG;
          const int st_beg = (nstg * slice) / KS, st_end = (nstg * (slice + 1)) / KS;
          const int gbeg = gc0 + st_beg * UG;
          const int gend = min(gc0 + st_end * UG, gc0 + gcn);
          const int nst = active ? st_end - st_beg : 0;

          // per-thread copy sources of stage 0 of this slice; each stage advances
          // them by UG groups.  Rows past the tile's end copy zeros from a valid row.
          const int g00 = gbeg;
          const uint32_t* csrc[NS][2];
          uint32_t csize[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            csize[h] = vrow[h] ? 1u : 0u;
#pragma unroll
            for (int s = 0; s < NS; ++s)
              csrc[s][h] = (vrow[h] ? crow[s][h] : crow[s][0]) + (int64_t)g00 * S::kWordsPerGroup;
          }
          if (!vrow[0]) {
#pragma unroll
            for (int s = 0; s < NS; ++s) { csrc[s][0] = safe_src; csrc[s][1] = safe_src; }
          }
          constexpr int NSB = (C::QW + 3) / 4;  // scale/bias words this lane copies per stage
          const uint32_t* ssrc[NSB];
          int sjw[NSB], spar[NSB];
          bool sok[NSB];
#pragma unroll
          for (int i = 0; i < NSB; ++i) {
            const int wq = t + 4 * i;  // [stack][row][scales|biases][word]
            const int s_ = wq / (4 * SBW), h = (wq / (2 * SBW)) % 2, arr = (wq / SBW) % 2;
            const int jw = wq % SBW;
            const bool in = wq < C::QW && s_ < NS;
            const int64_t e0 = rowG[h & 1] + g00;
            sjw[i] = jw;
            spar[i] = (int)(e0 & 1);
            sok[i] = in && vrow[h & 1];
            ssrc[i] = sok[i] ? srow[s_ < NS ? s_ : 0][h & 1][arr] + (e0 >> 1) + jw : safe_src;
          }

          // issue the copies (packed codes + scale/bias words) of stage `st`
          auto issue = [&](int st) {
            if (st < nst) {
              const uint32_t slot = ring_base + (uint32_t)((st % STAGES) * C::STAGE_WORDS * 4);
              const int nu = min(UG, gend - (gbeg + st * UG));
              const int64_t cadv = (int64_t)st * UG * S::kWordsPerGroup;
#pragma unroll
              for (int u = 0; u < UG; ++u) {
#pragma unroll
                for (int s = 0; s < NS; ++s) {
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    const uint32_t dst = slot + (uint32_t)((((u * NS + s) * 2 + h) * 32 + lane) * C::SLOT * 4);
                    const bool ok = (u < nu) && csize[h];
                    copy_share<S>(dst, ok ? csrc[s][h] + cadv + u * S::kWordsPerGroup : safe_src, t, ok,
                                  safe_src);
                  }
                }
              }
              const uint32_t sbq = slot + (uint32_t)((C::CODE_WORDS + g * C::QW) * 4);
              // words needed this stage: [e0>>1, (e0+nu-1)>>1] with e0 = row*G + g0
              const int sadv = (UG == 1) ? 0 : st * (UG / 2);
#pragma unroll
              for (int i = 0; i < NSB; ++i) {
                if (t + 4 * i < C::QW) {
                  int par = spar[i], jw = sjw[i];
                  const uint32_t* src = ssrc[i] + sadv;
                  if (UG == 1) {  // odd stage advance: recompute the word from the parity
                    const int e = par + st;
                    src = ssrc[i] + (e >> 1);
                    par = e & 1;
                  }
                  const bool ok = sok[i] && (jw <= ((par + nu - 1) >> 1));
                  cp_async4(sbq + (uint32_t)((t + 4 * i) * 4), ok ? src : safe_src, ok ? 4u : 0u);
                }
              }
            }
            cp_async_commit();
          };

          __syncthreads();  // previous users of xs / xrec / part are done
#pragma unroll
          for (int st = 0; st < STAGES - 1; ++st) issue(st);

          stage_x<S, T, TOKP, C::SEP_S>(p, pairs, ntok, gc0, gcn, xs, xrec);
          __syncthreads();

          // ---- stream codes + scales through the ring: tensor-core partial dots per
          //      group, scaled by s_g; bias and offset terms through one extra mma
          //      pair per 8 groups (A = b or s of the group, B = split sums) ----
          constexpr uint32_t XG = 4 * S::kVirt * sizeof(T);  // staged x bytes per group
          uint32_t xb_sa[MT], rec_sa[MT];
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            xb_sa[mt] = xs_sa + (uint32_t)(tokrow[mt] * p.tok_stride) + (uint32_t)(t * S::kVirt * sizeof(T));
            rec_sa[mt] = xrec_sa + (uint32_t)(tokrow[mt] * 8);
          }
          const uint32_t ring_lane = ring_base + (uint32_t)(lane * C::SLOT * 4);
          for (int st = 0; st < nst; ++st) {
            __syncwarp();  // every lane is done with the slot the next copies overwrite
            issue(st + STAGES - 1);
            cp_async_wait<STAGES - 1>();
            __syncwarp();  // the quad's scale/bias words were copied by 4 lanes
            const uint32_t soff = (uint32_t)((st % STAGES) * C::STAGE_WORDS * 4);
            const uint32_t slot = ring_lane + soff;
            const int g0 = gbeg + st * UG;
            const int gl0 = g0 - gc0;
            const int nu = min(UG, gend - g0);
            const uint32_t sbq = ring_base + soff + (uint32_t)((C::CODE_WORDS + g * C::QW) * 4);
            const int par0 = (int)((rowG[0] + g0) & 1), par1 = (int)((rowG[1] + g0) & 1);  // constant for even UG
#pragma unroll
            for (int u = 0; u < UG; ++u) {
              if (u < nu) {
                const uint32_t xo = (uint32_t)(gl0 + u) * XG;
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                  uint32_t rawA[S::kRegs], rawB[S::kRegs];
                  read_share<S>(slot + (uint32_t)((((u * NS + s) * 2 + 0) * 32) * C::SLOT * 4), t, rawA);
                  read_share<S>(slot + (uint32_t)((((u * NS + s) * 2 + 1) * 32) * C::SLOT * 4), t, rawB);
                  float d[MT][4];
                  group_dot<BITS, S, T, MT>(rawA, rawB, xb_sa, xo, d);
                  // y += s_g * d
                  const uint32_t sq = sbq + (uint32_t)(s * 4 * SBW * 4);
                  const float s0 = half_bits_to_f32<T>(lds16(sq + (uint32_t)((par0 + u) * 2)));
                  const float s1 = half_bits_to_f32<T>(lds16(sq + (uint32_t)(2 * SBW * 4 + (par1 + u) * 2)));
#pragma unroll
                  for (int mt = 0; mt < MT; ++mt) {
                    acc[s][mt][0] = fmaf(s0, d[mt][0], acc[s][mt][0]);
                    acc[s][mt][1] = fmaf(s0, d[mt][1], acc[s][mt][1]);
                    acc[s][mt][2] = fmaf(s1, d[mt][2], acc[s][mt][2]);
                    acc[s][mt][3] = fmaf(s1, d[mt][3], acc[s][mt][3]);
                  }
                }
              }
            }
            // bias and offset terms: thread t takes groups t and t+4 of each 8-group block
#pragma unroll
            for (int cb = 0; cb < C::CB; ++cb) {
              const int ja = cb * 8 + t, jb = ja + 4;
              const bool va = ja < nu, vb = jb < nu;
#pragma unroll
              for (int s = 0; s < NS; ++s) {
                const uint32_t sq = sbq + (uint32_t)(s * 4 * SBW * 4);
                // [row h][scales|biases] words at sq + (h*2 + arr)*SBW*4; element par_h + j
                auto val = [&](int h, int arr, int jj, bool ok) -> uint32_t {
                  const int par = h ? par1 : par0;
                  return ok ? dup16(lds16(sq + (uint32_t)(((h * 2 + arr) * SBW) * 4 + (par + jj) * 2))) : 0u;
                };
                const uint32_t ba0 = val(0, 1, ja, va), ba1 = val(1, 1, ja, va);
                const uint32_t bb0 = val(0, 1, jb, vb), bb1 = val(1, 1, jb, vb);
                const uint32_t sa0 = val(0, 0, ja, va), sa1 = val(1, 0, ja, va);
                const uint32_t sb0 = val(0, 0, jb, vb), sb1 = val(1, 0, jb, vb);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                  uint2 ra = make_uint2(0u, 0u), rb = make_uint2(0u, 0u);
                  if (va) ra = lds64(rec_sa[mt] + (uint32_t)((gl0 + ja) * TOKP * 8));
                  if (vb) rb = lds64(rec_sa[mt] + (uint32_t)((gl0 + jb) * TOKP * 8));
                  mma16816<T>(acc[s][mt], ba0, ba1, bb0, bb1, ra.x, rb.x);
                  if constexpr (C::SEP_S)
                    mma16816<T>(accs[s][mt], sa0, sa1, sb0, sb1, ra.y, rb.y);
                  else
                    mma16816<T>(acc[s][mt], sa0, sa1, sb0, sb1, ra.y, rb.y);
                }
              }
            }
          }
          cp_async_wait<0>();
        }  // K chunks

        // ---- partial sums -> shared, reduce over slices, store ----
        if (active) {
#pragma unroll
          for (int s = 0; s < NS; ++s)
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int rr = g + ((i >> 1) << 3);
                const int tk = mt * 8 + 2 * t + (i & 1);
                const float v_ = C::SEP_S ? fmaf(-S::kOff, accs[s][mt][i], acc[s][mt][i]) : acc[s][mt][i];
                part[((warp * 16 + rr) * TOKP + tk) * NS + s] = v_;
              }
        }
        __syncthreads();
        reduce_store<TOKP, NS, DUAL>(p, part, tiles, KS, ntok, blk_row0, r1, pairs);
      }  // row blocks
    }    // token chunks
  }      // segments
}

// ------------------------------------------------------------------ host side
static inline size_t align128(size_t v) { return (v + 127) / 128 * 128; }

// Plans the shared-memory carve-up and the K chunking for one instantiation,
// then launches one CTA per SM.  cudaErrorInvalidValue: the call exceeds the
// kernel's shared-memory limits.
template <int BITS, int GS, typename T, int MT, bool DUAL>
cudaError_t launch_one(QgemvParams prm, cudaStream_t st) {
  using C = QgemvCfg<BITS, GS, T, MT, DUAL>;
  using S = typename C::S;
  auto k = qgemv_kernel<BITS, GS, T, MT, DUAL>;
  const int grid = qmm_host::num_sms();
  const int tok_cap = prm.ids ? (prm.n_pairs < kMaxTok ? prm.n_pairs : kMaxTok) : prm.n_pairs;
  const int E = prm.ids ? prm.num_experts : 1;
  const int bpg_tok = GS * (S::kSplit ? 2 : 1) * (int)sizeof(T);  // staged x bytes per group per token

  const size_t plan = align128((size_t)(4 * E + 2 * prm.n_pairs) * sizeof(int));
  const size_t ring = (size_t)kWarps * C::RING_BYTES;
  const size_t part = align128((size_t)kWarps * 16 * C::TOKP * C::NS * sizeof(float));
  auto chunk_bytes = [&](int kc) {
    const size_t ts = (size_t)kc * bpg_tok + 16;
    return align128(ts * tok_cap) + align128((size_t)kc * C::TOKP * 8);
  };
  const size_t fixed = plan + ring + part;
  int kchunk = prm.G;
  while (kchunk > 1 && fixed + chunk_bytes(kchunk) > (size_t)kSmemMax) kchunk = (kchunk + 1) / 2;
  if (fixed + chunk_bytes(kchunk) > (size_t)kSmemMax) return cudaErrorInvalidValue;

  prm.tok_cap = tok_cap;
  prm.kchunk = kchunk;
  prm.tok_stride = kchunk * bpg_tok + 16;
  prm.sb_rows = 0;
  prm.sb_words = 0;
  prm.off_plan = 0;
  prm.off_ring = (int)plan;
  prm.off_part = (int)(plan + ring);
  prm.off_corr = 0;
  prm.off_xs = (int)(plan + ring + part);
  prm.off_xsum = prm.off_xs + (int)align128((size_t)prm.tok_stride * tok_cap);
  prm.off_sb = 0;
  const size_t smem = (size_t)prm.off_xsum + align128((size_t)kchunk * C::TOKP * 8);

  // opt in to the full shared-memory carve-out once per device and instantiation
  // (not a stream operation, so launches stay capturable in CUDA graphs)
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  k<<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

template <int BITS, int GS, typename T>
cudaError_t launch_mt(const QgemvParams& prm, int mt, bool dual, cudaStream_t st) {
  if (dual) {
    if (mt == 1) return launch_one<BITS, GS, T, 1, true>(prm, st);
    return launch_one<BITS, GS, T, 2, true>(prm, st);
  }
  if (mt == 1) return launch_one<BITS, GS, T, 1, false>(prm, st);
  return launch_one<BITS, GS, T, 2, false>(prm, st);
}

}  // namespace qmm
