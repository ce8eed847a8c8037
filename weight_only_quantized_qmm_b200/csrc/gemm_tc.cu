// Prefill-shaped quantized matmul on the 5th-generation tensor cores:
//   y[m, n] = sum_k x[m, k] * w_hat[n, k],  w_hat = q * s_g + b_g
// ("emily 0.5.1 lib/emily/quantization.ex", quantized_matmul/2 with
//  transpose = true), for bf16 or f16 activations with matching scales.
//
// One CTA computes a 128 (weight rows) x 256 (tokens) tile of y^T with
// tcgen05.mma (kind::f16, M = 128, N = 256, K = 16 per instruction), fp32
// accumulator in tensor memory (256 columns):
//   warp 0      TMA producer: x tiles [256 tokens x 64 k] bf16, 128-byte
//               swizzle, one mbarrier per pipeline stage (transaction bytes)
//   warp 1      allocates TMEM, one elected thread issues the MMAs and
//               commits each stage back to the producers
//   warps 2..5  dequantize: each thread owns one weight row, reads its packed
//               codes and the group's scale/bias from global memory (prefetched
//               three stages ahead), forms w_hat in bf16x2/f16x2 exactly once
//               ((OFF + q) - OFF is exact, then one fused q*s + b rounding) and
//               writes it into the stage's A tile in the UMMA K-major 128-byte
//               swizzled layout; then the same warps run the epilogue
//               (tcgen05.ld -> shared-memory transpose -> coalesced stores).
// Every mbarrier wait is bounded; on a timeout the tile is written as NaN.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "mbarrier.cuh"

namespace qmm {

namespace gemm {
constexpr int kBM = 128;                 // weight rows per CTA (UMMA M)
constexpr int kBN = 256;                 // tokens per CTA (UMMA N)
constexpr int kBK = 64;                  // k per stage: one 128-byte swizzle row of 16-bit values
constexpr int kThreads = 320;            // 10 warps
constexpr int kXStage = kBN * kBK * 2;   // 32 KB
constexpr int kAStage = kBM * kBK * 2;   // 16 KB
constexpr int kSBChunk = kBM * 8 * 2;    // 8 groups of scales (or biases) of 128 rows: 2 KB
constexpr uint32_t kSpins = 1u << 22;

// Shared-memory plan of one instantiation.  TW: the packed codes (per stage,
// [128 rows x 64 codes]) and the scales/biases (per chunk of 8 groups) arrive
// by TMA; otherwise the dequant warps read them from global memory.
template <int B, bool TW>
struct Plan {
  // four stages where they fit (8-bit codes: three); a fourth measured +6%
  // over three at M = 2048 on 14336 x 4096
  static constexpr int STAGES = TW ? (B == 8 ? 3 : 4) : 4;
  static constexpr int CODE_STAGE = TW ? kBM * 2 * B * 4 : 0;  // 64 codes = 2B words per row
  static constexpr int X0 = 0;
  static constexpr int A0 = STAGES * kXStage;
  static constexpr int C0 = A0 + STAGES * kAStage;
  static constexpr int SB0 = C0 + STAGES * CODE_STAGE;          // [2 chunks][scales | biases]
  static constexpr int BAR0 = SB0 + (TW ? 2 * 2 * kSBChunk : 0);
  static constexpr int SMEM = 1024 + BAR0 + 256;                // + alignment slack, barriers
  static_assert(8 * (4 * STAGES + 9) + 8 <= 256, "barriers, TMEM slot and abort flag fit their region");
  static_assert(SMEM <= 227 * 1024, "shared memory plan");
};
}  // namespace gemm

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// Bounded wait on an mbarrier phase.  Gives up (returns false) after kSpins
// polls, or as soon as another role of the CTA has raised the abort flag.
__device__ __forceinline__ bool bar_wait(uint32_t b, uint32_t parity, const int* abort_flag) {
  return mbar_wait_abortable(b, parity, gemm::kSpins, abort_flag);
}
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* m, int c0, int c1,
                                       uint32_t b) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(m), "r"(c0), "r"(c1), "r"(b)
      : "memory");
}
// UMMA shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;             // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;   // stride byte offset
  d |= (uint64_t)1u << 46;             // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;             // 128-byte swizzle
  return d;
}
// instruction descriptor: fp32 accumulator, A/B = bf16 (1) or f16 (0), both K-major
template <typename T>
__device__ __forceinline__ uint32_t mma_idesc(int n) {  // n: a multiple of 16 in [16, 256]
  constexpr uint32_t fmt = std::is_same<T, __half>::value ? 0u : 1u;
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(gemm::kBM >> 4) << 24);
}
__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16-bit float pair arithmetic on raw 32-bit registers
template <typename T>
__device__ __forceinline__ uint32_t h2_sub(uint32_t a, uint32_t b) {
  uint32_t r;
  if constexpr (std::is_same<T, __half>::value)
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  else
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
template <typename T>
__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  if constexpr (std::is_same<T, __half>::value)
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  else
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

struct GemmParams {
  const uint32_t* packed;
  const void* scales;
  const void* biases;
  void* y;
  int64_t ldy;  // elements between output rows
  int y_dtype;
  int M, N, K, G, wpr;
  // MoE prefill form (MOE instantiation): the schedule that the routing
  // kernel wrote (see moe_gemm.cu); N is the rows of one expert and y is
  // [n_pairs, N]
  const int32_t* ws_off;    // [E + 1] exclusive prefix of pairs per expert; off[E] = valid pairs
  const int32_t* ws_args;   // [3] blocks of <= 256 pairs, largest expert count, experts used
  const int32_t* ws_pairs;  // [n_pairs] pair indices grouped by expert, bad ids last
  const int32_t* ws_blk_e;  // expert of block b
  const int32_t* ws_blk_s;  // first entry (into ws_pairs) of block b
  int E, top_k, ne11, n_pairs;
  // MoE: the activation rows already gathered in pair-list order (row i of
  // the x map is the row of the pair listed at entry i), so a tile's rows
  // are one contiguous box; 0: the producer gathers them 4 at a time
  int xg;
  // dense: tokens per tile, 256, or 128 when 256-token tiles would leave SMs
  // idle (few tokens, few weight rows)
  int tbn;
};

// ------------------------------------------------------------------ dequant helpers
// packed words of 64 consecutive codes of one row (2*B words), zero past the row
template <int B>
__device__ __forceinline__ void load_codes(const uint32_t* row, int w0, int wpr, bool ok,
                                           uint32_t (&w)[2 * B]) {
  if constexpr (B == 4) {
    if (ok && w0 + 8 <= wpr && ((reinterpret_cast<uintptr_t>(row + w0) & 15) == 0)) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(row + w0));
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(row + w0) + 1);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
      return;
    }
  }
#pragma unroll
  for (int i = 0; i < 2 * B; ++i) w[i] = (ok && w0 + i < wpr) ? __ldg(row + w0 + i) : 0u;
}

// 64 codes -> 32 pairs of (OFF + q) as 16-bit floats (pair p = codes 2p, 2p+1)
template <int B, typename T>
__device__ __forceinline__ void codes_to_pairs(const uint32_t (&w)[2 * B], uint32_t (&pr)[32]) {
  constexpr uint32_t M8 = std::is_same<T, __half>::value ? 0x64646464u : 0x43434343u;
  if constexpr (B == 4) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t t0 = w[i] & 0x0F0F0F0Fu;         // codes 0,2,4,6 of the word
      const uint32_t t1 = (w[i] >> 4) & 0x0F0F0F0Fu;  // codes 1,3,5,7
      const uint32_t u = __byte_perm(t0, t1, 0x5140);  // c0 c1 c2 c3
      const uint32_t v = __byte_perm(t0, t1, 0x7362);  // c4 c5 c6 c7
      // f16 magic 0x6400 = 1024 needs the code in the low byte of the mantissa:
      // both magics keep the code in the low byte and the magic in the high byte
      pr[4 * i + 0] = __byte_perm(u, M8, 0x4140);
      pr[4 * i + 1] = __byte_perm(u, M8, 0x4342);
      pr[4 * i + 2] = __byte_perm(v, M8, 0x4140);
      pr[4 * i + 3] = __byte_perm(v, M8, 0x4342);
    }
  } else {
    constexpr uint32_t MG = std::is_same<T, __half>::value ? 0x64006400u : 0x43004300u;
#pragma unroll
    for (int p = 0; p < 32; ++p) {
      const uint32_t c0 = stream_code<B>(w, 2 * p), c1 = stream_code<B>(w, 2 * p + 1);
      pr[p] = c0 | (c1 << 16) | MG;
    }
  }
}

// The CTA's tiles, in order: tile = blockIdx.x + lt * gridDim.x.
//   dense: weight-row tiles vary slowest, so the CTAs running at the same time
//          share their x tiles and weight rows through L2;
//   MoE:   blocks of <= 256 pairs of one expert vary slowest, so the CTAs
//          running at the same time share the gathered activation rows.
// m0 is the first token (dense) or the first entry of the pair list (MoE);
// cnt the tokens (pairs) of the tile; e the expert.
struct TileOf {
  int n0, m0, cnt, e;
};
template <bool MOE>
__device__ __forceinline__ TileOf tile_of(const GemmParams& p, int lt, int m_tiles, int n_tiles) {
  const int t = blockIdx.x + lt * gridDim.x;
  if constexpr (MOE) {
    const int b = t / n_tiles, nt = t - b * n_tiles;
    const int e = __ldg(p.ws_blk_e + b), m0 = __ldg(p.ws_blk_s + b);
    return TileOf{nt * gemm::kBM, m0, min(gemm::kBN, __ldg(p.ws_off + e + 1) - m0), e};
  } else {
    const int nt = t / m_tiles, mt = t - nt * m_tiles;
    return TileOf{nt * gemm::kBM, mt * p.tbn, min(p.tbn, p.M - mt * p.tbn), 0};
  }
}
// row of the activation matrix that token slot j of a MoE tile reads
// (slots past the tile's pairs read the first pair's row; they are never stored)
__device__ __forceinline__ int moe_a_row(const GemmParams& p, const TileOf& tl, int j) {
  const int pr = __ldg(p.ws_pairs + tl.m0 + (j < tl.cnt ? j : 0));
  return p.ne11 == 1 ? pr / p.top_k : pr;
}
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* m, int c0, int r0, int r1, int r2,
                                            int r3, uint32_t b) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(m), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(b)
      : "memory");
}

// Persistent: every CTA walks its tiles (static round robin over the grid).
// Warp roles:
//   warp 0      TMA producer of the x tiles (one stage = 256 tokens x 64 k)
//   warp 1      TMEM owner (512 columns: two 128 x 256 fp32 accumulators)
//               and MMA issuer; the accumulator alternates per tile, so the
//               epilogue of one tile runs under the main loop of the next
//   warps 2..5  dequantize the weight tile of each stage into the A buffer
//   warps 6..9  epilogue: tcgen05.ld of the finished accumulator, release it,
//               store y directly from registers (per instruction, a warp
//               writes 32 consecutive weight rows of one token)
template <int B, int GS, typename T, bool MOE, bool TW>
__global__ void __launch_bounds__(gemm::kThreads, 1)
qgemm_tc_kernel(const GemmParams p, const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmc,
                const __grid_constant__ CUtensorMap tms, const __grid_constant__ CUtensorMap tmb) {
  using namespace gemm;
  using PL = Plan<B, TW>;
  constexpr int kStages = PL::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
  uint8_t* xs = smem + PL::X0;                        // [kStages][256 x 128 B]
  uint8_t* as = smem + PL::A0;                        // [kStages][128 x 128 B]
  uint8_t* cs = smem + PL::C0;                        // [kStages][128 rows x 2B words] (TW)
  uint8_t* sbs = smem + PL::SB0;                      // [2][scales 2 KB | biases 2 KB] (TW)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PL::BAR0);
  const uint32_t full0 = su32(bars), afull0 = full0 + 8 * kStages, empty0 = afull0 + 8 * kStages;
  const uint32_t accf0 = empty0 + 8 * kStages;      // [2] accumulator complete
  const uint32_t tfree0 = accf0 + 16;               // [2] accumulator read out by the epilogue
  const uint32_t drain = tfree0 + 16;               // every issued MMA complete
  const uint32_t sbfull0 = drain + 8;               // [2] scale/bias chunk landed (TW)
  const uint32_t sbempty0 = sbfull0 + 16;           // [2] scale/bias chunk consumed (TW)
  const uint32_t cfull0 = sbempty0 + 16;            // [kStages] the stage's codes landed (TW)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * kStages + 9);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  // stages per scale/bias chunk (8 groups): a chunk starts at k-stage i when
  // i % SPC == 0 and ends at the chunk's last stage or the row's last stage
  constexpr int SPC = (8 * GS) / kBK;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (p.K + kBK - 1) / kBK;
  const int m_tiles = (p.M + p.tbn - 1) / p.tbn;
  const int n_tiles = (p.N + kBM - 1) / kBM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(afull0 + 8 * s, 4);
      mbar_init(empty0 + 8 * s, 1);
      mbar_init(cfull0 + 8 * s, 1);
    }
    mbar_init(accf0, 1);
    mbar_init(accf0 + 8, 1);
    mbar_init(tfree0, 4);
    mbar_init(tfree0 + 8, 4);
    mbar_init(drain, 1);
    mbar_init(sbfull0, 1);
    mbar_init(sbfull0 + 8, 1);
    mbar_init(sbempty0, 4);
    mbar_init(sbempty0 + 8, 4);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // 512 TMEM columns: accumulators at columns 0 and 256
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(su32(tmem_slot)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // x, the weights and the MoE schedule may come from the previous kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int T_all = (MOE ? __ldg(p.ws_args) : m_tiles) * n_tiles;
  const int my_tiles = (int)blockIdx.x < T_all ? (T_all - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    // dense: lane 0 loads each stage's [256 x 64] x tile; MoE: lane 0 posts
    // the stage's bytes and every lane gathers the activation rows of 8 token
    // slots (two 4-row gathers, one row per slot)
    int j = 0, issued = 0, cc = 0, cissued = 0;
    bool stop = false;
    for (int lt = 0; lt < my_tiles && !stop; ++lt) {
      const TileOf tl = tile_of<MOE>(p, lt, m_tiles, n_tiles);
      const int wrow0 = tl.e * p.N + tl.n0;  // first row of the (stacked) weight matrix
      int rw[8];
      if (MOE && !p.xg) {
#pragma unroll
        for (int q = 0; q < 8; ++q) rw[q] = moe_a_row(p, tl, 8 * lane + q);
      }
      // gathered rows: only the tile's (a MoE block often holds far fewer than
      // 256 pairs), 8 per lane
      const int ngl = (tl.cnt + 7) / 8;
      for (int i = 0; i < nk; ++i, ++j) {
        const int s = j % kStages, u = j / kStages;
        bool ok = true;
        if constexpr (TW) {
          // a new chunk of 8 groups of scales/biases: its ring slot is free once
          // the dequant warps released the chunk two before it
          if (i % SPC == 0) {
            const int cs_ = cc & 1;
            if (lane == 0 && cc >= 2) ok = bar_wait(sbempty0 + 8 * cs_, ((cc >> 1) - 1) & 1, abort_flag);
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
              if (lane == 0) *abort_flag = 1;
              stop = true;
              break;
            }
            if (lane == 0) {
              const uint32_t sb = su32(sbs + cs_ * 2 * kSBChunk), bar = sbfull0 + 8 * cs_;
              mbar_arrive_expect_tx(bar, 2 * kSBChunk);
              tma_2d(sb, &tms, (i * kBK / GS) & ~7, wrow0, bar);
              tma_2d(sb + kSBChunk, &tmb, (i * kBK / GS) & ~7, wrow0, bar);
            }
            cissued = ++cc;
          }
        }
        if (lane == 0 && j >= kStages) ok = bar_wait(empty0 + 8 * s, (u - 1) & 1, abort_flag);
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
          if (lane == 0) *abort_flag = 1;
          stop = true;
          break;
        }
        // the codes (TW) land on their own cfull[s], requested first, so that
        // the dequant warps can start before the larger x tile (full[s]) is in
        if constexpr (TW) {
          if (lane == 0) {
            mbar_arrive_expect_tx(cfull0 + 8 * s, PL::CODE_STAGE);
            tma_2d(su32(cs + s * PL::CODE_STAGE), &tmc, i * 2 * B, wrow0, cfull0 + 8 * s);
          }
        }
        if (MOE && !p.xg) {
          if (lane == 0) mbar_arrive_expect_tx(full0 + 8 * s, (uint32_t)(ngl * 8 * 128));
          __syncwarp();
          if (lane < ngl) {
            const uint32_t d = su32(xs + s * kXStage) + (uint32_t)(lane * 8 * 128);
            tma_gather4(d, &tmx, i * kBK, rw[0], rw[1], rw[2], rw[3], full0 + 8 * s);
            tma_gather4(d + 512, &tmx, i * kBK, rw[4], rw[5], rw[6], rw[7], full0 + 8 * s);
          }
        } else if (lane == 0) {
          // one box of the tile's token rows (256, or 128 for a dense call of
          // 128-token tiles; measured: eight 32-row boxes per stage cost a
          // third of the dense GEMM's throughput)
          mbar_arrive_expect_tx(full0 + 8 * s, MOE ? (uint32_t)kXStage : (uint32_t)(p.tbn * kBK * 2));
          tma_2d(su32(xs + s * kXStage), &tmx, i * kBK, tl.m0, full0 + 8 * s);
        }
        issued = j + 1;
      }
    }
    // no copy may still be landing when the CTA exits: the last copy of every
    // slot is waited for with the full bound, also after an abort
    if (lane == 0) {
      for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i) {
        mbar_wait_n(full0 + 8 * (i % kStages), (uint32_t)(i / kStages) & 1u, gemm::kSpins);
        if (TW) mbar_wait_n(cfull0 + 8 * (i % kStages), (uint32_t)(i / kStages) & 1u, gemm::kSpins);
      }
      for (int c = cissued > 2 ? cissued - 2 : 0; c < cissued; ++c)
        mbar_wait_n(sbfull0 + 8 * (c & 1), (uint32_t)(c >> 1) & 1u, gemm::kSpins);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int j = 0;
      bool stop = false;
      for (int lt = 0; lt < my_tiles && !stop; ++lt) {
        const int b = lt & 1;
        // N of the tile's MMAs: its token count rounded up to 16 (columns past
        // the count read rows that are never stored)
        const uint32_t idesc = mma_idesc<T>(min(kBN, (tile_of<MOE>(p, lt, m_tiles, n_tiles).cnt + 15) & ~15));
        // accumulator b is free once the epilogue has read out tile lt - 2
        if (lt >= 2 && !bar_wait(tfree0 + 8 * b, ((lt >> 1) - 1) & 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(b * kBN);
        for (int i = 0; i < nk; ++i, ++j) {
          const int s = j % kStages, u = j / kStages;
          if (!bar_wait(full0 + 8 * s, u & 1, abort_flag) || !bar_wait(afull0 + 8 * s, u & 1, abort_flag)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = su32(as + s * kAStage), b0 = su32(xs + s * kXStage);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_f16(acc, sw128_desc(a0 + 32 * kk), sw128_desc(b0 + 32 * kk), idesc, (i | kk) != 0 ? 1u : 0u);
          mma_commit(empty0 + 8 * s);  // frees the stage once these MMAs have read it
        }
        mma_commit(accf0 + 8 * b);  // accumulator b complete (also after an abort)
      }
      // TMEM is released only once every issued MMA has completed
      mma_commit(drain);
      mbar_wait_n(drain, 0, gemm::kSpins);
    }
  } else if (warp < 6) {
    // ---------------- dequant (warps 2..5) ----------------
    const int r = (warp & 3) * 32 + lane;  // weight row of the tile owned by this thread
    constexpr int NGS = (kBK + GS - 1) / GS;  // groups touched by a stage (1 or 2)
    constexpr uint32_t OFF2 = std::is_same<T, __half>::value ? 0x64006400u : 0x43004300u;
    constexpr bool kF32Path = (B == 8) && !std::is_same<T, __half>::value;
    const int total = my_tiles * nk;

    // w_hat of this thread's row for stage s (64 codes cw, the stage's NGS
    // scales/biases) written into the stage's A tile, then handed to the MMA
    auto emit = [&](int s, const uint32_t (&cw)[2 * B], const T (&cs_)[NGS], const T (&cb_)[NGS]) {
      uint32_t pr[32];
      float sf0 = 0.f, bf0 = 0.f, sf1 = 0.f, bf1 = 0.f;
      if constexpr (kF32Path) {
        sf0 = to_f32(cs_[0]); bf0 = to_f32(cb_[0]);
        sf1 = to_f32(cs_[NGS - 1]); bf1 = to_f32(cb_[NGS - 1]);
      } else {
        codes_to_pairs<B, T>(cw, pr);
      }
      const uint32_t s2a = (uint32_t)bits16(cs_[0]) * 0x00010001u;
      const uint32_t b2a = (uint32_t)bits16(cb_[0]) * 0x00010001u;
      const uint32_t s2b = (uint32_t)bits16(cs_[NGS - 1]) * 0x00010001u;
      const uint32_t b2b = (uint32_t)bits16(cb_[NGS - 1]) * 0x00010001u;
      uint8_t* arow = as + s * kAStage + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // 16-byte chunk c = pairs 4c..4c+3 = codes 8c..8c+7
        uint4 v;
        uint32_t* vv = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int pi = 4 * c + e;
          const bool second = NGS > 1 && (2 * pi) >= GS;
          if constexpr (kF32Path) {
            // 8-bit codes do not fit the bf16 magic: q exact in fp32, fmaf, one bf16 rounding
            const float q0 = __uint_as_float(0x4B000000u | stream_code<B>(cw, 2 * pi)) - 8388608.0f;
            const float q1 = __uint_as_float(0x4B000000u | stream_code<B>(cw, 2 * pi + 1)) - 8388608.0f;
            const float sv = second ? sf1 : sf0, bv = second ? bf1 : bf0;
            const __nv_bfloat162 h = __floats2bfloat162_rn(fmaf(q0, sv, bv), fmaf(q1, sv, bv));
            vv[e] = *reinterpret_cast<const uint32_t*>(&h);
          } else {
            const uint32_t qv = h2_sub<T>(pr[pi], OFF2);  // exact q
            vv[e] = h2_fma<T>(qv, second ? s2b : s2a, second ? b2b : b2a);
          }
        }
        *reinterpret_cast<uint4*>(arow + ((c ^ (r & 7)) << 4)) = v;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(afull0 + 8 * s);
    };

    if constexpr (TW) {
      // codes and scales/biases were staged by TMA: stage j is k-stage j % nk
      // of the CTA's tile j / nk; its codes land on cfull[s]
      int cc = 0;  // scale/bias chunks entered
      for (int j = 0; j < total; ++j) {
        const int lt = j / nk, i = j - lt * nk;
        const int s = j % kStages, u = j / kStages;
        if (i % SPC == 0) {
          if (!bar_wait(sbfull0 + 8 * (cc & 1), (uint32_t)(cc >> 1) & 1u, abort_flag)) *abort_flag = 1;
          ++cc;
        }
        const int slot = (cc - 1) & 1;
        if (!bar_wait(cfull0 + 8 * s, u & 1, abort_flag)) *abort_flag = 1;
        // (the A buffer of stage s is free: the producer waited for its MMAs
        // before this stage's copies, whose landing the wait above saw)
        uint32_t cw[2 * B];
        const uint32_t crow = su32(cs + s * PL::CODE_STAGE) + (uint32_t)(r * 8 * B);
        // 16-byte chunk q of the row sits at q ^ f(r) under the map's swizzle
        // (32-byte rows: f = bit 2 of r; 64-byte rows: f = bits 1..2 of r)
        const int cf = B == 4 ? (r >> 2) & 1 : B == 8 ? (r >> 1) & 3 : 0;
#pragma unroll
        for (int q = 0; q < B / 2; ++q) {
          const uint4 v = lds128(crow + 16 * (q ^ cf));
          cw[4 * q] = v.x; cw[4 * q + 1] = v.y; cw[4 * q + 2] = v.z; cw[4 * q + 3] = v.w;
        }
        T cs_[NGS], cb_[NGS];
        const uint32_t srow = su32(sbs + slot * 2 * kSBChunk) + (uint32_t)(r * 16);
#pragma unroll
        for (int q = 0; q < NGS; ++q) {
          const int gi = ((i * kBK) / GS + q) & 7;
          const unsigned short sv = (unsigned short)lds16(srow + 2 * gi);
          const unsigned short bv = (unsigned short)lds16(srow + kSBChunk + 2 * gi);
          memcpy(&cs_[q], &sv, 2);
          memcpy(&cb_[q], &bv, 2);
        }
        emit(s, cw, cs_, cb_);
        if (i % SPC == SPC - 1 || i == nk - 1) {  // last stage of the chunk: release it
          if (lane == 0) mbar_arrive(sbempty0 + 8 * slot);
        }
      }
    } else {
      // codes and scales/biases are prefetched kAhead stages ahead into a
      // register ring (compile-time indices: the stage loop is unrolled by
      // kAhead); stage j is k-stage j % nk of the CTA's tile j / nk
      constexpr int kAhead = 3;
      uint32_t rw[kAhead][2 * B];
      T rs[kAhead][NGS], rb[kAhead][NGS];
      auto load = [&](int j, uint32_t (&w)[2 * B], T (&sv)[NGS], T (&bv)[NGS]) {
        const bool in = j < total;
        const int lt = in ? j / nk : 0, i = in ? j - lt * nk : 0;
        const TileOf tl = tile_of<MOE>(p, in ? lt : 0, m_tiles, n_tiles);
        const int n = tl.n0 + r;
        const bool nval = in && n < p.N;
        // row of the (stacked) weight matrix: expert e's rows start at e * N
        const int64_t wr = nval ? (int64_t)tl.e * p.N + n : 0;
        const uint32_t* row = p.packed + wr * p.wpr;
        const T* srow = reinterpret_cast<const T*>(p.scales) + wr * p.G;
        const T* brow = reinterpret_cast<const T*>(p.biases) + wr * p.G;
        const int k0 = i * kBK;
        load_codes<B>(row, k0 * B / 32, p.wpr, nval, w);
#pragma unroll
        for (int jj = 0; jj < NGS; ++jj) {
          const int gidx = (k0 + jj * GS) / GS;
          const bool ok = nval && gidx < p.G;
          sv[jj] = ok ? srow[gidx] : from_f32<T>(0.0f);
          bv[jj] = ok ? brow[gidx] : from_f32<T>(0.0f);
        }
      };
#pragma unroll
      for (int a = 0; a < kAhead; ++a) load(a, rw[a], rs[a], rb[a]);
      for (int j0 = 0; j0 < total; j0 += kAhead) {
#pragma unroll
        for (int a = 0; a < kAhead; ++a) {
          const int j = j0 + a;
          if (j >= total) break;
          const int s = j % kStages, u = j / kStages;
          uint32_t cw[2 * B];
          T cs_[NGS], cb_[NGS];
#pragma unroll
          for (int q = 0; q < 2 * B; ++q) cw[q] = rw[a][q];
#pragma unroll
          for (int q = 0; q < NGS; ++q) { cs_[q] = rs[a][q]; cb_[q] = rb[a][q]; }
          load(j + kAhead, rw[a], rs[a], rb[a]);  // refill this ring slot kAhead stages ahead
          // the A buffer of this stage is free once the MMAs of stage j - kStages are done
          if (u > 0 && !bar_wait(empty0 + 8 * s, (u - 1) & 1, abort_flag)) *abort_flag = 1;
          emit(s, cw, cs_, cb_);
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 6..9): TMEM -> registers -> y ----------------
    const int qq = warp & 3;          // TMEM lane quarter this warp may access
    const int r = qq * 32 + lane;     // weight row of the tile
    const bool f32out = p.y_dtype == QMM_F32;
    auto put = [&](int64_t idx, float f) {
      if (f32out)
        reinterpret_cast<float*>(p.y)[idx] = f;
      else
        reinterpret_cast<T*>(p.y)[idx] = from_f32<T>(f);
    };
    if constexpr (MOE) {
      // pairs whose id was out of range (listed last) get zero rows
      const int bad0 = __ldg(p.ws_off + p.E);
      const int64_t nz = (int64_t)(p.n_pairs - bad0) * p.N;
      const int et = (warp - 6) * 32 + lane;
      for (int64_t z = (int64_t)blockIdx.x * 128 + et; z < nz; z += (int64_t)gridDim.x * 128) {
        const int pr = __ldg(p.ws_pairs + bad0 + (int)(z / p.N));
        put((int64_t)pr * p.N + z % p.N, 0.0f);
      }
    }
    bool failed = false;
    for (int lt = 0; lt < my_tiles; ++lt) {
      const TileOf tl = tile_of<MOE>(p, lt, m_tiles, n_tiles);
      const int b = lt & 1;
      const int n = tl.n0 + r;
      if (!failed) {
        // the MMA warp commits accf on every path it takes; a raised abort flag
        // ends the wait early, and the tile (and all later ones) is written as NaN
        failed = !bar_wait(accf0 + 8 * b, (lt >> 1) & 1, abort_flag) ||
                 *reinterpret_cast<volatile int*>(abort_flag);
        failed = __any_sync(0xffffffffu, failed);
      }
      tc_fence_after();
      for (int c = 0; c < (tl.cnt + 31) / 32; ++c) {  // the TMEM columns the tile's tokens use
        uint32_t v[32];
        if (!failed) tmem_ld32(tmem + ((uint32_t)(qq * 32) << 16) + (uint32_t)(b * kBN + c * 32), v);
        if (n < p.N) {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const int slot = c * 32 + jj;
            if (slot < tl.cnt) {
              const float f = failed ? __int_as_float(0x7fc00000) : __uint_as_float(v[jj]);
              // dense: token m0 + slot; MoE: the pair listed at m0 + slot
              const int64_t orow = MOE ? (int64_t)__ldg(p.ws_pairs + tl.m0 + slot) : (int64_t)(tl.m0 + slot);
              put(orow * p.ldy + n, f);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !failed) mbar_arrive(tfree0 + 8 * b);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
  }
}

// ------------------------------------------------------------------ host
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

template <int B, int GS, typename T, bool MOE, bool TW>
static cudaError_t launch_gemm_t(const GemmParams& prm, const CUtensorMap (&tm)[4], int grid, cudaStream_t st) {
  auto k = qgemm_tc_kernel<B, GS, T, MOE, TW>;
  constexpr int SMEM = gemm::Plan<B, TW>::SMEM;
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(gemm::kThreads);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, prm, tm[0], tm[1], tm[2], tm[3]);
}

template <int B, int GS, typename T, bool MOE>
static cudaError_t launch_gemm_w(bool tw, const GemmParams& prm, const CUtensorMap (&tm)[4], int grid,
                                 cudaStream_t st) {
  if constexpr (B != 3) {  // 64 3-bit codes are 24 bytes: not a TMA box width
    if (tw) return launch_gemm_t<B, GS, T, MOE, true>(prm, tm, grid, st);
  }
  return launch_gemm_t<B, GS, T, MOE, false>(prm, tm, grid, st);
}

template <typename T, bool MOE>
static cudaError_t launch_gemm_b(int bits, int gs, bool tw, const GemmParams& prm, const CUtensorMap (&tm)[4],
                                 int grid, cudaStream_t st) {
#define QMM_G(BB)                                                                  \
  if (gs == 32) return launch_gemm_w<BB, 32, T, MOE>(tw, prm, tm, grid, st);       \
  if (gs == 64) return launch_gemm_w<BB, 64, T, MOE>(tw, prm, tm, grid, st);       \
  return launch_gemm_w<BB, 128, T, MOE>(tw, prm, tm, grid, st);
  switch (bits) {
    case 2: { QMM_G(2) }
    case 3: { QMM_G(3) }
    case 4: { QMM_G(4) }
    case 6: { QMM_G(6) }
    default: { QMM_G(8) }
  }
#undef QMM_G
}

// Maps of the weight side for the TMA-staged dequant: packed codes [rows, wpr]
// u32 in [2 * bits words x 128 rows] boxes (one stage), scales and biases
// [rows, G] 16-bit in [8 groups x 128 rows] boxes (one chunk).  False (the
// caller reads the weights from global memory instead) when the rows are not
// 16-byte strided or a stage's codes are not a whole number of 16 bytes.
static bool make_w_maps(CUtensorMap* tc, CUtensorMap* ts, CUtensorMap* tb, const uint32_t* packed,
                        const void* scales, const void* biases, int64_t rows, int64_t wpr, int64_t G, int bits) {
  if (bits == 3 || wpr % 4 != 0 || G % 8 != 0) return false;
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint32_t estr[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {(cuuint64_t)wpr, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(wpr * 4)};
    const cuuint32_t box[2] = {(cuuint32_t)(2 * bits), (cuuint32_t)gemm::kBM};
    // rows of 32 or 64 bytes are swizzled at their width, so that the eight
    // rows a quarter warp reads at one chunk fall in different banks
    const CUtensorMapSwizzle swz = bits == 4 ? CU_TENSOR_MAP_SWIZZLE_32B
                                   : bits == 8 ? CU_TENSOR_MAP_SWIZZLE_64B
                                               : CU_TENSOR_MAP_SWIZZLE_NONE;
    if (enc(tc, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(packed), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  const cuuint64_t dims[2] = {(cuuint64_t)G, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(G * 2)};
  const cuuint32_t box[2] = {8, (cuuint32_t)gemm::kBM};
  for (int a = 0; a < 2; ++a)
    if (enc(a ? tb : ts, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(a ? biases : scales), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  return true;
}

// 2-D map over x [rows, K] (16-bit): boxes of 64 k x box_rows rows, 128-byte swizzle
static bool make_x_map(CUtensorMap* m, const void* x, int x_dtype, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(K * 2)};
  const cuuint32_t box[2] = {gemm::kBK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      x_dtype == QMM_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return enc(m, dt, 2, const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// cudaErrorNotSupported: the call does not fit this kernel (the caller falls back)
cudaError_t launch_qgemm_tc(const void* x, int x_dtype, int64_t M, int64_t K, const qmm_qweight* w,
                            void* y, int64_t ldy, int y_dtype, cudaStream_t st) {
  if (M > (int64_t)INT32_MAX || K > (int64_t)INT32_MAX || w->rows > (int64_t)INT32_MAX)
    return cudaErrorNotSupported;
  if ((K * 2) % 16 != 0) return cudaErrorNotSupported;
  // 128-token tiles when 256-token tiles would not give every SM one
  const int64_t n_tiles = (w->rows + gemm::kBM - 1) / gemm::kBM;
  const int tbn = (n_tiles * ((M + gemm::kBN - 1) / gemm::kBN) < qmm_host::num_sms() && M > 128) ? 128 : gemm::kBN;
  CUtensorMap tm[4];
  if (!make_x_map(&tm[0], x, x_dtype, M, K, tbn)) return cudaErrorNotSupported;
  const bool tw = make_w_maps(&tm[1], &tm[2], &tm[3], w->packed, w->scales, w->biases, w->rows,
                              K * w->bits / 32, K / w->group_size, w->bits);
  if (!tw) tm[1] = tm[2] = tm[3] = tm[0];
  GemmParams prm{};
  prm.packed = w->packed;
  prm.scales = w->scales;
  prm.biases = w->biases;
  prm.y = y;
  prm.ldy = ldy;
  prm.y_dtype = y_dtype;
  prm.M = (int)M;
  prm.N = (int)w->rows;
  prm.K = (int)K;
  prm.G = (int)(K / w->group_size);
  prm.wpr = (int)(K * w->bits / 32);
  prm.tbn = tbn;
  // persistent: one CTA per SM (or per tile when there are fewer tiles)
  const int64_t tiles = n_tiles * (int64_t)((prm.M + tbn - 1) / tbn);
  const int grid = (int)std::min<int64_t>(tiles, qmm_host::num_sms());
  if (x_dtype == QMM_BF16) return launch_gemm_b<__nv_bfloat16, false>(w->bits, w->group_size, tw, prm, tm, grid, st);
  return launch_gemm_b<__half, false>(w->bits, w->group_size, tw, prm, tm, grid, st);
}

// MoE prefill GEMM over the schedule that moe_route_kernel wrote into `ws`
// (see moe_gemm.cu for the layout): a is [a_rows, K], out is [n_pairs, n_rows].
cudaError_t launch_qgemm_moe(const void* a, int a_dtype, int64_t a_rows, const qmm_expert_stack* w,
                             const int32_t* ws_off, const int32_t* ws_args, const int32_t* ws_pairs,
                             const int32_t* ws_blk_e, const int32_t* ws_blk_s, int top_k, int ne11,
                             int n_pairs, const void* xg, void* out, int out_dtype, cudaStream_t st) {
  const int64_t K = w->n_cols;
  if (a_rows > (int64_t)INT32_MAX || K > (int64_t)INT32_MAX || w->n_rows * w->num_experts > (int64_t)INT32_MAX)
    return cudaErrorNotSupported;
  if ((K * 2) % 16 != 0) return cudaErrorNotSupported;
  // x: 256-row boxes over the gathered rows, or one-row boxes over `a` (the
  // producer gathers 4 rows per copy)
  CUtensorMap tm[4];
  if (xg ? !make_x_map(&tm[0], xg, a_dtype, n_pairs, K, gemm::kBN) : !make_x_map(&tm[0], a, a_dtype, a_rows, K, 1))
    return cudaErrorNotSupported;
  const bool tw = make_w_maps(&tm[1], &tm[2], &tm[3], w->packed, w->scales, w->biases,
                              w->n_rows * w->num_experts, K * w->bits / 32, K / w->group_size, w->bits);
  if (!tw) tm[1] = tm[2] = tm[3] = tm[0];
  GemmParams prm{};
  prm.packed = w->packed;
  prm.scales = w->scales;
  prm.biases = w->biases;
  prm.y = out;
  prm.ldy = w->n_rows;
  prm.y_dtype = out_dtype;
  prm.M = 0;
  prm.N = (int)w->n_rows;
  prm.K = (int)K;
  prm.G = (int)(K / w->group_size);
  prm.wpr = (int)(K * w->bits / 32);
  prm.ws_off = ws_off;
  prm.ws_args = ws_args;
  prm.ws_pairs = ws_pairs;
  prm.ws_blk_e = ws_blk_e;
  prm.ws_blk_s = ws_blk_s;
  prm.tbn = gemm::kBN;  // (blocks of up to 256 pairs)
  prm.E = (int)w->num_experts;
  prm.top_k = top_k;
  prm.ne11 = ne11;
  prm.n_pairs = n_pairs;
  prm.xg = xg != nullptr;
  // the work list is known only on the device: one CTA per SM
  const int grid = qmm_host::num_sms();
  if (a_dtype == QMM_BF16) return launch_gemm_b<__nv_bfloat16, true>(w->bits, w->group_size, tw, prm, tm, grid, st);
  return launch_gemm_b<__half, true>(w->bits, w->group_size, tw, prm, tm, grid, st);
}

}  // namespace qmm
