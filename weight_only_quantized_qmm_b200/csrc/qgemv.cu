// Decode-shaped quantized matmul (M <= 16) and the MoE indirect-dispatch GEMV,
// dense and fused gate+up+SiLU, in one kernel family.
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
//   * The per-group affine factor is pulled out of the reduction:
//       sum_{k in g} x_k (q_k s_g + b_g) = s_g * sum q_k x_k + b_g * sum x_k.
//     The integer part sum q_k x_k runs on the tensor cores with
//     mma.sync.m16n8k16 (bf16 or f16 operands, fp32 accumulate): 16 weight
//     rows form the A operand, up to 8 tokens the B operand.  Codes become
//     exact 16-bit floats with one LOP3 each pair ((lane & mask) | 0x4300 for
//     bf16 = 128 + q, 0x6400 for f16 = 1024 + q); the offset is removed in
//     the per-group fold with the precomputed sum of x.  8-bit codes in bf16
//     are split into two nibble slots (x and 16 x) because 128 + q > 255 is
//     not exact in bf16.
//   * Each mma's 16 k-slots belong to one quantization group: the 4 threads
//     of a quad each hold one quarter of the group of their two rows, so the
//     fp32 mma result can be scaled per group.  The k order inside a thread's
//     quarter is free; x is staged in shared memory in the same order.
//   * Weights stream from HBM with 64/128-bit ld.global.nc.L1::no_allocate,
//     U groups in flight per warp, 16 warps per CTA, one CTA per SM.  The
//     rows are split evenly over the CTAs (row granularity, not tile
//     granularity), so every SM streams the same number of bytes.
//   * MoE: every CTA builds the expert -> pairs lists of the call in shared
//     memory (counting by expert), takes its slice of the rows of the
//     distinct experts, and each expert's packed rows are read once however
//     many pairs use it.
#include <algorithm>

#include "qgemv.cuh"

namespace qmm {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxTok = 16;

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
template <class S>
__device__ __forceinline__ void load_share(const uint32_t* grp, int t, bool ok,
                                           uint32_t (&r)[S::kRegs]) {
  if constexpr (S::kAligned) {
    const uint32_t* p = grp + t * S::kRegs;
    if constexpr (S::kRegs == 1) {
      r[0] = ok ? ldg_stream_u32(p) : 0u;
    } else if constexpr (S::kRegs == 2) {
      uint2 v = make_uint2(0u, 0u);
      if (ok) v = ldg_stream_u64(p);
      r[0] = v.x; r[1] = v.y;
    } else if constexpr (S::kRegs % 4 == 0) {
#pragma unroll
      for (int i = 0; i < S::kRegs / 4; ++i) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (ok) v = ldg_stream_u128(p + 4 * i);
        r[4 * i] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < S::kRegs; ++i) r[i] = ok ? ldg_stream_u32(p + i) : 0u;
    }
  } else {
    // share starts inside a word: fetch the one or two words covering it
    const int bit = t * S::kBitsShare;
    const int w = bit >> 5, sh = bit & 31;
    const uint32_t lo = ok ? ldg_stream_u32(grp + w) : 0u;
    const uint32_t hi = (ok && (sh + S::kBitsShare > 32)) ? ldg_stream_u32(grp + w + 1) : 0u;
    r[0] = __funnelshift_r(lo, hi, sh);
    if constexpr (S::kRegs > 1) r[1] = hi >> sh;
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

// ------------------------------------------------------------------ kernel
template <int BITS, int GS, typename T, int MT, bool DUAL>
__global__ void __launch_bounds__(kThreads, 1) qgemv_kernel(const QgemvParams p) {
  using S = Share<BITS, GS, T>;
  constexpr int NS = DUAL ? 2 : 1;
  // groups in flight per warp: about 16 registers of packed words
  constexpr int U0 = 16 / (2 * S::kRegs * NS);
  constexpr int U = U0 < 1 ? 1 : (U0 > 4 ? 4 : U0);
  constexpr int TOKP = MT * 8;
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
  T* xs = reinterpret_cast<T*>(smem + p.off_xs);
  float* xsb = reinterpret_cast<float*>(smem + p.off_xsum);  // [kchunk][16]
  float* xsc = xsb + p.kchunk * kMaxTok;                      // [kchunk][16]
  float* part = reinterpret_cast<float*>(smem + p.off_part);  // [32][16][TOKP][NS]

  // ---- plan: expert -> pair lists (counting sort by expert id) ----
  if (p.ids == nullptr) {
    for (int i = tid; i < p.n_pairs; i += kThreads) s_list[i] = i;
    if (tid == 0) { s_cnt[0] = p.n_pairs; s_start[0] = 0; s_dist[0] = 0; s_nd = 1; }
    __syncthreads();
  } else {
    for (int e = tid; e < E; e += kThreads) { s_cnt[e] = 0; s_fill[e] = 0; }
    __syncthreads();
    for (int i = tid; i < p.n_pairs; i += kThreads) {
      const int e = p.ids[i];
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
      if (lane == 0) s_nd = nd;
    }
    __syncthreads();
    for (int i = tid; i < p.n_pairs; i += kThreads) {
      const int e = p.ids[i];
      if (e >= 0 && e < E) {
        s_list[s_start[e] + atomicAdd(&s_fill[e], 1)] = i;
      } else if (blockIdx.x == 0) {
        // bad id: zero row, report
        for (int64_t n = 0; n < p.n_rows; ++n) store_as(p.out, p.out_dtype, (int64_t)i * p.out_ld + n, 0.0f);
        set_status(p.d_status, QMM_ERR_BAD_EXPERT_ID);
      }
    }
    __syncthreads();
  }

  const int64_t V = (int64_t)s_nd * p.n_rows;
  const int64_t v0 = V * blockIdx.x / gridDim.x;
  const int64_t v1 = V * (blockIdx.x + 1) / gridDim.x;
  const int nchunks = (p.G + p.kchunk - 1) / p.kchunk;

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
        const int64_t trow = r0 + 16 * (int64_t)(rb + tile);  // first row of the tile (in expert)
        const int rows_valid = active ? (int)(r1 - trow < 16 ? r1 - trow : 16) : 0;
        const bool vA = g < rows_valid, vB = g + 8 < rows_valid;
        const int64_t rowA = ebase + trow + g, rowB = rowA + 8;

        float acc[NS][MT][4];
#pragma unroll
        for (int s = 0; s < NS; ++s)
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[s][mt][i] = 0.0f;

        for (int ch = 0; ch < nchunks; ++ch) {
          const int gc0 = ch * p.kchunk;
          const int gcn = min(p.kchunk, p.G - gc0);
          // ---- stage x for this chunk: slot order of the shares, plus group sums ----
          __syncthreads();
          {
            const int per_tok = gcn * 4 * S::kVirt;
            for (int idx = tid; idx < ntok * per_tok; idx += kThreads) {
              const int tk = idx / per_tok;
              const int rem = idx - tk * per_tok;
              const int gl = rem / (4 * S::kVirt);
              const int rem2 = rem - gl * 4 * S::kVirt;
              const int tt = rem2 / S::kVirt, slot = rem2 - tt * S::kVirt;
              const int vv = S::slot_virtual(slot);
              const int64_t k = (int64_t)(gc0 + gl) * GS + tt * S::kCodes + S::virt_code(vv);
              const T* xa = reinterpret_cast<const T*>(p.a) + pair_offset(p, pairs[tk]);
              const float xv = to_f32(xa[k]) * S::virt_mult(vv);
              T* dst = reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(xs) + (int64_t)tk * p.tok_stride);
              dst[(gl * 4 + tt) * S::kVirt + slot] = from_f32<T>(xv);
            }
          }
          __syncthreads();
          // group sums: one warp per (token, group)
          for (int it = warp; it < ntok * gcn; it += kWarps) {
            const int tk = it / gcn, gl = it - tk * gcn;
            const T* src = reinterpret_cast<const T*>(reinterpret_cast<const uint8_t*>(xs) +
                                                      (int64_t)tk * p.tok_stride) + gl * 4 * S::kVirt;
            float sc = 0.0f, sb = 0.0f;
            for (int q = lane; q < 4 * S::kVirt; q += 32) {
              const float xv = to_f32(src[q]);
              sc += xv;
              const int vv = S::slot_virtual(q % S::kVirt);
              if (S::virt_mult(vv) == 1.0f) sb += xv;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              sc += __shfl_xor_sync(0xffffffffu, sc, o);
              sb += __shfl_xor_sync(0xffffffffu, sb, o);
            }
            if (lane == 0) { xsc[gl * kMaxTok + tk] = sc; xsb[gl * kMaxTok + tk] = sb; }
          }
          __syncthreads();

          if (active) {
            const int gbeg = gc0 + (gcn * slice) / KS;
            const int gend = gc0 + (gcn * (slice + 1)) / KS;
            for (int gi = gbeg; gi < gend; gi += U) {
              uint32_t raw[U][NS][2][S::kRegs];
              T sv[U][NS][2], bv[U][NS][2];
#pragma unroll
              for (int u = 0; u < U; ++u) {
                const int grp = gi + u;
                const bool ok = grp < gend;
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                  const uint32_t* base = p.packed[s] + (int64_t)grp * S::kWordsPerGroup;
                  load_share<S>(base + rowA * p.wpr, t, ok && vA, raw[u][s][0]);
                  load_share<S>(base + rowB * p.wpr, t, ok && vB, raw[u][s][1]);
                  const T* sc = reinterpret_cast<const T*>(p.scales[s]);
                  const T* bi = reinterpret_cast<const T*>(p.biases[s]);
                  sv[u][s][0] = (ok && vA) ? sc[rowA * p.G + grp] : from_f32<T>(0.0f);
                  bv[u][s][0] = (ok && vA) ? bi[rowA * p.G + grp] : from_f32<T>(0.0f);
                  sv[u][s][1] = (ok && vB) ? sc[rowB * p.G + grp] : from_f32<T>(0.0f);
                  bv[u][s][1] = (ok && vB) ? bi[rowB * p.G + grp] : from_f32<T>(0.0f);
                }
              }
#pragma unroll
              for (int u = 0; u < U; ++u) {
                const int grp = gi + u;
                if (grp >= gend) break;
                const int gl = grp - gc0;
                // B fragments for this group: slot layout [t][kVirt] of each token row
                const uint8_t* xrow0 = reinterpret_cast<const uint8_t*>(xs) +
                                       (size_t)(gl * 4 + t) * S::kVirt * sizeof(T);
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                  float d[MT][4];
#pragma unroll
                  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) d[mt][i] = 0.0f;
#pragma unroll
                  for (int st = 0; st < S::kSteps; ++st) {
                    const uint32_t a0 = share_pair<BITS, S>(raw[u][s][0], 2 * st);
                    const uint32_t a1 = share_pair<BITS, S>(raw[u][s][1], 2 * st);
                    const uint32_t a2 = share_pair<BITS, S>(raw[u][s][0], 2 * st + 1);
                    const uint32_t a3 = share_pair<BITS, S>(raw[u][s][1], 2 * st + 1);
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                      const int tok = mt * 8 + g;
                      uint2 bfr = make_uint2(0u, 0u);
                      if (tok < ntok)
                        bfr = *reinterpret_cast<const uint2*>(xrow0 + (size_t)tok * p.tok_stride +
                                                              st * 8);
                      mma16816<T>(d[mt], a0, a1, a2, a3, bfr.x, bfr.y);
                    }
                  }
                  // fold: y += s*d + b*sum(x) - OFF*s*sum(x')
#pragma unroll
                  for (int mt = 0; mt < MT; ++mt) {
                    const float2 sb2 = *reinterpret_cast<const float2*>(xsb + gl * kMaxTok + mt * 8 + 2 * t);
                    const float2 sc2 = *reinterpret_cast<const float2*>(xsc + gl * kMaxTok + mt * 8 + 2 * t);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                      const float s_ = to_f32(sv[u][s][h]), b_ = to_f32(bv[u][s][h]);
                      const float ns_ = -S::kOff * s_;
                      float a0 = acc[s][mt][2 * h], a1 = acc[s][mt][2 * h + 1];
                      a0 = fmaf(s_, d[mt][2 * h], a0);
                      a1 = fmaf(s_, d[mt][2 * h + 1], a1);
                      a0 = fmaf(b_, sb2.x, a0);
                      a1 = fmaf(b_, sb2.y, a1);
                      a0 = fmaf(ns_, sc2.x, a0);
                      a1 = fmaf(ns_, sc2.y, a1);
                      acc[s][mt][2 * h] = a0;
                      acc[s][mt][2 * h + 1] = a1;
                    }
                  }
                }
              }
            }
          }
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
                part[((warp * 16 + rr) * TOKP + tk) * NS + s] = acc[s][mt][i];
              }
        }
        __syncthreads();
        for (int it = tid; it < tiles * 16 * ntok; it += kThreads) {
          const int tl = it / (16 * ntok);
          const int rr = (it / ntok) % 16;
          const int tk = it % ntok;
          const int64_t row = r0 + 16 * (int64_t)(rb + tl) + rr;
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
        __syncthreads();
      }  // row blocks
    }    // token chunks
  }      // segments
}

// ------------------------------------------------------------------ host side
struct QgemvShape {
  int bits, gs, dtype;  // dtype: QMM_BF16 / QMM_F16
  bool dual;
};

template <int BITS, int GS, typename T, int MT, bool DUAL>
static cudaError_t launch_one(const QgemvParams& prm, int grid, size_t smem, cudaStream_t st) {
  auto k = qgemv_kernel<BITS, GS, T, MT, DUAL>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

template <int BITS, int GS, typename T>
static cudaError_t launch_mt(const QgemvParams& prm, int mt, bool dual, int grid, size_t smem,
                             cudaStream_t st) {
  if (dual) {
    if (mt == 1) return launch_one<BITS, GS, T, 1, true>(prm, grid, smem, st);
    return launch_one<BITS, GS, T, 2, true>(prm, grid, smem, st);
  }
  if (mt == 1) return launch_one<BITS, GS, T, 1, false>(prm, grid, smem, st);
  return launch_one<BITS, GS, T, 2, false>(prm, grid, smem, st);
}

template <typename T>
static cudaError_t launch_bg(const QgemvParams& prm, int bits, int gs, int mt, bool dual, int grid,
                             size_t smem, cudaStream_t st) {
#define QMM_GS(B)                                                                   \
  if (gs == 32) return launch_mt<B, 32, T>(prm, mt, dual, grid, smem, st);          \
  if (gs == 64) return launch_mt<B, 64, T>(prm, mt, dual, grid, smem, st);          \
  return launch_mt<B, 128, T>(prm, mt, dual, grid, smem, st);
  switch (bits) {
    case 2: { QMM_GS(2) }
    case 3: { QMM_GS(3) }
    case 4: { QMM_GS(4) }
    case 6: { QMM_GS(6) }
    default: { QMM_GS(8) }
  }
#undef QMM_GS
}

// virtual k-slots per real code (nibble split for 8-bit bf16)
static int slot_factor(int bits, int dtype) { return (bits == 8 && dtype == QMM_BF16) ? 2 : 1; }

// Plans the launch (shared memory carve-up, K chunking) and launches.
// Returns cudaErrorInvalidValue when the call exceeds the kernel's limits.
cudaError_t launch_qgemv(QgemvParams prm, int bits, int gs, int dtype, bool dual,
                         cudaStream_t st) {
  const int tok_cap = prm.ids ? std::min(prm.n_pairs, kMaxTok) : prm.n_pairs;
  if (tok_cap <= 0) return cudaSuccess;
  if (tok_cap > kMaxTok) return cudaErrorInvalidValue;
  const int mt = tok_cap > 8 ? 2 : 1;
  const int tokp = mt * 8;
  const int ns = dual ? 2 : 1;
  const int E = prm.ids ? prm.num_experts : 1;
  const size_t plan = (size_t)(4 * E + prm.n_pairs) * sizeof(int);
  const size_t part = (size_t)kWarps * 16 * tokp * ns * sizeof(float);
  const int bytes_per_group_tok = gs * slot_factor(bits, dtype) * 2;
  const size_t budget = 227 * 1024 - 2048;
  const size_t fixed = ((plan + 127) / 128) * 128 + part;
  if (fixed + 4096 > budget) return cudaErrorInvalidValue;
  // largest chunk of groups whose staged x (+ sums) fits
  int kchunk = prm.G;
  auto need = [&](int kc) {
    const size_t ts = (size_t)kc * bytes_per_group_tok + 16;
    return ((ts * tok_cap + 127) / 128) * 128 + (size_t)kc * kMaxTok * 2 * sizeof(float);
  };
  while (kchunk > 1 && fixed + need(kchunk) > budget) kchunk = (kchunk + 1) / 2;
  if (fixed + need(kchunk) > budget) return cudaErrorInvalidValue;
  prm.tok_cap = tok_cap;
  prm.kchunk = kchunk;
  prm.tok_stride = kchunk * bytes_per_group_tok + 16;
  prm.off_plan = 0;
  prm.off_xs = (int)(((plan + 127) / 128) * 128);
  prm.off_xsum = prm.off_xs + (int)((((size_t)prm.tok_stride * tok_cap + 127) / 128) * 128);
  prm.off_part = prm.off_xsum + (int)((size_t)kchunk * kMaxTok * 2 * sizeof(float));
  const size_t smem = (size_t)prm.off_part + part;
  const int grid = qmm_host::num_sms();
  if (dtype == QMM_BF16) return launch_bg<__nv_bfloat16>(prm, bits, gs, mt, dual, grid, smem, st);
  return launch_bg<__half>(prm, bits, gs, mt, dual, grid, smem, st);
}

}  // namespace qmm
