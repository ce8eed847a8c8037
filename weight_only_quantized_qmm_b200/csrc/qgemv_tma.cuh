// TMA variant of the decode GEMV / MoE kernel family (qgemv_impl.cuh): the
// packed codes of each warp's row tile arrive in shared memory as 16-row x
// 128-byte boxes by the Tensor Memory Accelerator (cp.async.bulk.tensor.2d,
// 128-byte swizzle, mbarrier transaction counting), instead of per-thread
// cp.async.  Only the copy mechanism differs: the arithmetic (tensor-core
// partial dots per group, s_g fold, bias/offset correction mma) is the same.
//
// Used for the shapes the streaming kernel (qgemv_stream.cuh) declines, when
// the rows of the packed matrix start on 16-byte boundaries
// (K * bits / 8 % 16 == 0) and codes are 2, 4 or 8 bits wide with whole-word
// shares (a group is then a power-of-two number of words, so one box row
// holds whole groups) -- e.g. the MoE down projection at K / gs = 12.
#pragma once

#include <cuda.h>

#include "mbarrier.cuh"
#include "qgemv_impl.cuh"

namespace qmm {

// ------------------------------------------------------------------ mbarrier / TMA
// In a pipeline loop, after a first failure the warp only polls briefly
// (`failed`), so a broken copy cannot stretch the kernel by one full timeout
// per remaining stage; draining copies already issued uses the full bound.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, bool failed) {
  return mbar_wait_n(bar, parity, failed ? 1024u : kMbarSpins);
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

template <int BITS, int GS, typename T, int MT, bool DUAL>
struct TmaCfg {
  using S = Share<BITS, GS, T>;
  static constexpr int NS = DUAL ? 2 : 1;
  static constexpr int WPG = S::kWordsPerGroup;          // power of two, 2..32
  static constexpr int SG = 32 / WPG;                    // groups per stage: one 128-byte box row
  static constexpr int SBW = SG == 1 ? 1 : SG / 2 + 1;   // scale (or bias) words per row per stage
  static constexpr int QW = NS * 2 * 2 * SBW;            // scale+bias words per quad per stage
  static constexpr int STAGES = DUAL ? 2 : 4;
  static constexpr int BOX = 16 * 128;                   // bytes of one code box (16 rows)
  static constexpr int CODE_STAGE = NS * BOX;            // code bytes per warp per stage
  static constexpr int SB_STAGE = 8 * QW * 4;            // scale/bias bytes per warp per stage
  static constexpr int TOKP = MT * 8;
  static constexpr int CB = (SG + 7) / 8;                // correction mmas per stage
  static constexpr bool SEP_S = std::is_same<T, __half>::value;
  static_assert(WPG * SG == 32, "a stage is one 128-byte row of packed words");
};

// Read this thread's share of group u (stage-local) of box row r (= g or g + 8)
// from a 128-byte-swizzled box: 16-byte chunk c of row r sits at chunk c ^ (r % 8).
template <class S, int WPG>
__device__ __forceinline__ void read_share_swz(uint32_t box, int r, int g, int t, int u,
                                               uint32_t (&out)[S::kRegs]) {
  const int w = u * WPG + t * S::kRegs;  // first word of the share in the box row
  const uint32_t row = box + (uint32_t)(r * 128);
  if constexpr (S::kRegs >= 4) {
#pragma unroll
    for (int i = 0; i < S::kRegs / 4; ++i) {
      const uint4 v = lds128(row + (uint32_t)((((w >> 2) + i) ^ g) << 4));
      out[4 * i] = v.x; out[4 * i + 1] = v.y; out[4 * i + 2] = v.z; out[4 * i + 3] = v.w;
    }
  } else if constexpr (S::kRegs == 2) {
    const uint2 v = lds64(row + (uint32_t)((((w >> 2) ^ g) << 4) + ((w & 3) << 2)));
    out[0] = v.x; out[1] = v.y;
  } else {
    out[0] = lds32(row + (uint32_t)((((w >> 2) ^ g) << 4) + ((w & 3) << 2)));
  }
}

template <int BITS, int GS, typename T, int MT, bool DUAL>
__global__ void __launch_bounds__(kThreads, 1)
qgemv_tma_kernel(const QgemvParams p, const __grid_constant__ CUtensorMap tm0,
                 const __grid_constant__ CUtensorMap tm1) {
  using C = TmaCfg<BITS, GS, T, MT, DUAL>;
  using S = typename C::S;
  constexpr int NS = C::NS, SG = C::SG, STAGES = C::STAGES, TOKP = C::TOKP, SBW = C::SBW;
  constexpr int WPG = C::WPG;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the swizzled boxes need 1024-byte-aligned destinations
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

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
  uint2* xrec = reinterpret_cast<uint2*>(smem + p.off_xsum);
  float* part = reinterpret_cast<float*>(smem + p.off_part);
  // per warp: STAGES code stages (1024-byte aligned boxes), STAGES scale/bias
  // stages, STAGES mbarriers
  const uint32_t code_base = smem_u32(smem + p.off_ring) + (uint32_t)(warp * STAGES * C::CODE_STAGE);
  const uint32_t sb_base = smem_u32(smem + p.off_sb) + (uint32_t)(warp * STAGES * C::SB_STAGE);
  const uint32_t bar_base = smem_u32(smem + p.off_corr) + (uint32_t)(warp * STAGES * 8);

  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < STAGES; ++i) mbar_init(bar_base + 8 * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();

  build_plan(p, s_cnt, s_start, s_fill, s_dist, s_list, s_list + p.n_pairs, &s_nd);

  const int64_t V = (int64_t)s_nd * p.n_rows;
  const int64_t v0 = V * blockIdx.x / gridDim.x;
  const int64_t v1 = V * (blockIdx.x + 1) / gridDim.x;
  const int nchunks = (p.G + p.kchunk - 1) / p.kchunk;
  const uint32_t* safe_src = p.packed[0];
  const uint32_t xs_sa = smem_u32(xs);
  const uint32_t xrec_sa = smem_u32(xrec);
  uint32_t used = 0;     // stages this warp has consumed (all lanes agree)
  bool failed = false;   // a bounded wait gave up: skip the arithmetic from here on

  for (int64_t v = v0; v < v1;) {
    const int64_t j = v / p.n_rows;
    const int64_t r0 = v - j * p.n_rows;
    const int64_t r1 = min(v1 - j * p.n_rows, p.n_rows);
    const int e = s_dist[j];
    const int64_t ebase = (int64_t)e * p.n_rows;
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
        const int64_t blk_row0 = r0 + 16 * (int64_t)rb;
        const int64_t trow = blk_row0 + 16 * (int64_t)tile;
        const int rows_valid = active ? (int)(r1 - trow < 16 ? r1 - trow : 16) : 0;
        const bool vrow[2] = {g < rows_valid, g + 8 < rows_valid};
        const int64_t rowg[2] = {ebase + trow + g, ebase + trow + g + 8};
        const int box_y = (int)(ebase + trow);

        float acc[NS][MT][4], accs[NS][MT][4];
#pragma unroll
        for (int s = 0; s < NS; ++s)
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) { acc[s][mt][i] = 0.0f; accs[s][mt][i] = 0.0f; }

        const int64_t rowG[2] = {rowg[0] * p.G, rowg[1] * p.G};
        int tokrow[MT];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) tokrow[mt] = (mt * 8 + g) < ntok ? mt * 8 + g : 0;

        for (int ch = 0; ch < nchunks; ++ch) {
          const int gc0 = ch * p.kchunk;
          const int gcn = min(p.kchunk, p.G - gc0);
          const int nstg = (gcn + SG - 1) / SG;
          const int st_beg = (nstg * slice) / KS, st_end = (nstg * (slice + 1)) / KS;
          const int gbeg = gc0 + st_beg * SG;
          const int gend = min(gc0 + st_end * SG, gc0 + gcn);
          const int nst = active ? st_end - st_beg : 0;

          // scale/bias word sources of stage 0 (this lane copies words t, t+4, ...)
          constexpr int NSB = (C::QW + 3) / 4;
          const uint32_t* ssrc[NSB];
          int sjw[NSB], spar[NSB];
          bool sok[NSB];
#pragma unroll
          for (int i = 0; i < NSB; ++i) {
            const int wq = t + 4 * i;  // [stack][row][scales|biases][word]
            const int s_ = wq / (4 * SBW), h = (wq / (2 * SBW)) % 2, arr = (wq / SBW) % 2;
            const int jw = wq % SBW;
            const bool in = wq < C::QW;
            const int64_t e0 = rowG[h] + gbeg;
            sjw[i] = jw;
            spar[i] = (int)(e0 & 1);
            sok[i] = in && vrow[h];
            const void* arrp = in ? (arr ? p.biases[s_] : p.scales[s_]) : nullptr;
            ssrc[i] = sok[i] ? reinterpret_cast<const uint32_t*>(arrp) + (e0 >> 1) + jw : safe_src;
          }

          // stages of this chunk whose copies were issued; none after a failure
          int n_issued = 0;
          auto issue = [&](int st) {
            if (st < nst && !failed) {
              n_issued = st + 1;
              const uint32_t k = (used + (uint32_t)st) % STAGES;
              const int g0 = gbeg + st * SG;
              const int nu = min(SG, gend - g0);
              if (lane == 0) {
                const uint32_t bar = bar_base + 8 * k;
                mbar_arrive_expect_tx(bar, (uint32_t)C::CODE_STAGE);
                tma_load_2d(code_base + k * C::CODE_STAGE, &tm0, g0 * WPG, box_y, bar);
                if constexpr (NS > 1)
                  tma_load_2d(code_base + k * C::CODE_STAGE + C::BOX, &tm1, g0 * WPG, box_y, bar);
              }
              const uint32_t sbq = sb_base + k * C::SB_STAGE + (uint32_t)(g * C::QW * 4);
              const int sadv = (SG == 1) ? 0 : st * (SG / 2);
#pragma unroll
              for (int i = 0; i < NSB; ++i) {
                if (t + 4 * i < C::QW) {
                  int par = spar[i];
                  const uint32_t* src = ssrc[i] + sadv;
                  if (SG == 1) {
                    const int e2 = par + st;
                    src = ssrc[i] + (e2 >> 1);
                    par = e2 & 1;
                  }
                  const bool ok = sok[i] && (sjw[i] <= ((par + nu - 1) >> 1));
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

          constexpr uint32_t XG = 4 * S::kVirt * sizeof(T);
          uint32_t xb_sa[MT], rec_sa[MT];
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            xb_sa[mt] = xs_sa + (uint32_t)(tokrow[mt] * p.tok_stride) + (uint32_t)(t * S::kVirt * sizeof(T));
            rec_sa[mt] = xrec_sa + (uint32_t)(tokrow[mt] * 8);
          }
          for (int st = 0; st < nst; ++st) {
            __syncwarp();  // every lane is done with the stage the next copies overwrite
            issue(st + STAGES - 1);
            const uint32_t k = (used + (uint32_t)st) % STAGES;
            const uint32_t parity = ((used + (uint32_t)st) / STAGES) & 1u;
            // every issued stage is waited on with the full bound (also after a
            // failure), so no copy is in flight at exit; `failed` is warp-uniform
            if (st < n_issued) {
              const bool ok = mbar_wait(bar_base + 8 * k, parity, false);
              if (__any_sync(0xffffffffu, !ok)) {
                if (!failed && lane == 0) set_status(p.d_status, QMM_ERR_TIMEOUT);
                failed = true;
              }
            }
            cp_async_wait<STAGES - 1>();
            __syncwarp();
            if (failed) continue;
            const uint32_t box = code_base + k * C::CODE_STAGE;
            const int g0 = gbeg + st * SG;
            const int gl0 = g0 - gc0;
            const int nu = min(SG, gend - g0);
            const uint32_t sbq = sb_base + k * C::SB_STAGE + (uint32_t)(g * C::QW * 4);
            const int par0 = (int)((rowG[0] + g0) & 1), par1 = (int)((rowG[1] + g0) & 1);
#pragma unroll
            for (int u = 0; u < SG; ++u) {
              if (u < nu) {
                const uint32_t xo = (uint32_t)(gl0 + u) * XG;
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                  uint32_t rawA[S::kRegs], rawB[S::kRegs];
                  read_share_swz<S, WPG>(box + s * C::BOX, g, g, t, u, rawA);
                  read_share_swz<S, WPG>(box + s * C::BOX, g + 8, g, t, u, rawB);
                  float d[MT][4];
#pragma unroll
                  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) d[mt][i] = 0.0f;
#pragma unroll
                  for (int q2 = 0; q2 < S::kSteps / 2; ++q2) {
                    uint4 bf[MT];
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) bf[mt] = lds128(xb_sa[mt] + xo + q2 * 16);
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                      const int q = 2 * q2 + h2;
                      const uint32_t a0 = share_pair<BITS, S>(rawA, 2 * q);
                      const uint32_t a1 = share_pair<BITS, S>(rawB, 2 * q);
                      const uint32_t a2 = share_pair<BITS, S>(rawA, 2 * q + 1);
                      const uint32_t a3 = share_pair<BITS, S>(rawB, 2 * q + 1);
#pragma unroll
                      for (int mt = 0; mt < MT; ++mt)
                        mma16816<T>(d[mt], a0, a1, a2, a3, h2 ? bf[mt].z : bf[mt].x,
                                    h2 ? bf[mt].w : bf[mt].y);
                    }
                  }
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
          used += (uint32_t)nst;
          cp_async_wait<0>();
        }  // K chunks

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
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();  // qgemv.cu: driver entry point, resolved once

// 2-D map over packed words [rows, wpr]: 16-row x 32-word boxes, 128-byte swizzle.
inline bool make_code_map(CUtensorMap* map, const uint32_t* packed, int64_t rows, int64_t wpr) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)wpr, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(wpr * 4)};
  const cuuint32_t box[2] = {32, 16};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t*>(packed), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BITS, int GS, typename T, int MT, bool DUAL>
cudaError_t launch_tma_impl(QgemvParams prm, int64_t rows_total, cudaStream_t st) {
  using C = TmaCfg<BITS, GS, T, MT, DUAL>;
  using S = typename C::S;
  CUtensorMap tm[2];
  for (int s = 0; s < C::NS; ++s)
    if (!make_code_map(&tm[s], prm.packed[s], rows_total, prm.wpr)) return cudaErrorNotSupported;
  if (C::NS == 1) tm[1] = tm[0];
  auto k = qgemv_tma_kernel<BITS, GS, T, MT, DUAL>;
  const int grid = qmm_host::num_sms();
  const int tok_cap = prm.ids ? (prm.n_pairs < kMaxTok ? prm.n_pairs : kMaxTok) : prm.n_pairs;
  const int E = prm.ids ? prm.num_experts : 1;
  const int bpg_tok = GS * (S::kSplit ? 2 : 1) * (int)sizeof(T);

  // [codes (1024-aligned) | scale/bias | mbarriers | plan | part | x | sums]
  const size_t codes = (size_t)kWarps * C::STAGES * C::CODE_STAGE;
  const size_t sb = align128((size_t)kWarps * C::STAGES * C::SB_STAGE);
  const size_t bars = align128((size_t)kWarps * C::STAGES * 8);
  const size_t plan = align128((size_t)(4 * E + 2 * prm.n_pairs) * sizeof(int));
  const size_t part = align128((size_t)kWarps * 16 * C::TOKP * C::NS * sizeof(float));
  auto chunk_bytes = [&](int kc) {
    const size_t ts = (size_t)kc * bpg_tok + 16;
    return align128(ts * tok_cap) + align128((size_t)kc * C::TOKP * 8);
  };
  const size_t fixed = 1024 + codes + sb + bars + plan + part;  // + alignment slack
  // K chunks hold whole stages (the boxes start on 32-word boundaries)
  int kchunk = prm.G;
  while (kchunk > C::SG && fixed + chunk_bytes(kchunk) > (size_t)kSmemMax)
    kchunk = std::max(C::SG, ((kchunk + 1) / 2) / C::SG * C::SG);
  // does not fit: the caller falls back to the cp.async path
  if (fixed + chunk_bytes(kchunk) > (size_t)kSmemMax) return cudaErrorNotSupported;

  prm.tok_cap = tok_cap;
  prm.kchunk = kchunk;
  prm.tok_stride = kchunk * bpg_tok + 16;
  prm.off_ring = 0;
  prm.off_sb = (int)codes;
  prm.off_corr = (int)(codes + sb);  // mbarriers
  prm.off_plan = (int)(codes + sb + bars);
  prm.off_part = prm.off_plan + (int)plan;
  prm.off_xs = prm.off_part + (int)part;
  prm.off_xsum = prm.off_xs + (int)align128((size_t)prm.tok_stride * tok_cap);
  const size_t smem = (size_t)prm.off_xsum + align128((size_t)kchunk * C::TOKP * 8) + 1024;

  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  k<<<grid, kThreads, smem, st>>>(prm, tm[0], tm[1]);
  return cudaGetLastError();
}

// The swizzled box reader takes whole-word shares only (2-bit g32 shares are
// half a word): other layouts go to the cp.async kernel.
template <int BITS, int GS, typename T, int MT, bool DUAL>
cudaError_t launch_tma_one(QgemvParams prm, int64_t rows_total, cudaStream_t st) {
  if constexpr (!Share<BITS, GS, T>::kAligned) {
    return cudaErrorNotSupported;
  } else {
    return launch_tma_impl<BITS, GS, T, MT, DUAL>(prm, rows_total, st);
  }
}

}  // namespace qmm
