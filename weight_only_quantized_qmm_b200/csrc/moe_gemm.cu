// MoE prefill (many tokens): routing on the device and the expert-grouped
// tensor-core GEMM ("ferrum-kernels 0.7.7 src/stacked_expert.rs",
// StackedExpertGgufLinear: gemm_moe_id, gemm_moe_id_indirect, and the
// compute_ids_tpe_gpu routing step they read).
//
//   out[p, :] = a[row(p), :] . dequant(W[ids[p]])^T,   p = token * top_k + slot,
//   row(p) = token (ne11 == 1: every slot of a token reads the token's row) or
//            p     (ne11 == top_k: one row per slot),
//
// computed in two launches on one stream, with no host round trip:
//   1. moe_route_kernel (one CTA) counts the pairs of every expert (tokens
//      per expert), lays out the pair indices grouped by expert, cuts each
//      expert's list into blocks of at most 256 pairs, and writes the block
//      count, the largest expert count and the number of experts used (the
//      12-byte triple that sizes the GEMM's work) -- all into the caller's
//      workspace;
//   2. the persistent tcgen05 GEMM (gemm_tc.cu, MoE instantiation) reads the
//      block list from the workspace: each work item is one block of pairs x
//      128 rows of the block's expert; the producer gathers the pairs'
//      activation rows by TMA (4 rows per copy), the dequant warps expand the
//      expert's codes, and the epilogue scatters each pair's outputs to its
//      row of `out`.
// A pair whose id is outside [0, E) is listed after all experts' pairs,
// reported as QMM_ERR_BAD_EXPERT_ID in *d_status, and gets a zero row.
#include <algorithm>

#include "common.cuh"

namespace qmm {

cudaError_t launch_qgemm_moe(const void* a, int a_dtype, int64_t a_rows, const qmm_expert_stack* w,
                             const int32_t* ws_off, const int32_t* ws_args, const int32_t* ws_pairs,
                             const int32_t* ws_blk_e, const int32_t* ws_blk_s, int top_k, int ne11,
                             int n_pairs, const void* xg, void* out, int out_dtype, cudaStream_t st);

constexpr int kMoeBlock = 256;         // pairs per GEMM block (the tile's token columns)
constexpr int kRouteThreads = 1024;
constexpr int64_t kMaxRouteExperts = 8192;

// Workspace layout, in int32 elements (documented in include/qmm.h).
struct MoeWs {
  int64_t tpe, off, args, pairs, blk_e, blk_s, total;
};
constexpr MoeWs moe_ws_layout(int64_t n_pairs, int64_t E) {
  const int64_t nb = (n_pairs + kMoeBlock - 1) / kMoeBlock + E;  // blocks, at most
  const int64_t pairs = (2 * E + 4 + 3) / 4 * 4;
  const int64_t blk_e = pairs + (n_pairs + 3) / 4 * 4;
  const int64_t blk_s = blk_e + (nb + 3) / 4 * 4;
  return MoeWs{0, E, 2 * E + 1, pairs, blk_e, blk_s, blk_s + (nb + 3) / 4 * 4};
}

// One CTA.  Shared memory: per-expert counts, running fill positions and
// block offsets, each E + 1 ints (index E collects the out-of-range ids).
__global__ void __launch_bounds__(kRouteThreads, 1)
moe_route_kernel(const int32_t* __restrict__ ids, int n_pairs, int E, int32_t* __restrict__ ws, MoeWs L,
                 int32_t* d_status) {
  extern __shared__ int sm[];
  int* cnt = sm;              // [E + 1]
  int* start = cnt + E + 1;   // [E + 1] exclusive prefix of cnt
  int* fill = start + E + 1;  // [E + 1]
  __shared__ int s_bad, s_nb, s_max, s_used;
  const int tid = threadIdx.x, nthr = blockDim.x, warp = tid >> 5, lane = tid & 31;
  // ids may come from the previous kernel in the stream
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int e = tid; e <= E; e += nthr) { cnt[e] = 0; fill[e] = 0; }
  if (tid == 0) s_bad = 0;
  __syncthreads();
  // 1. tokens per expert
  for (int p = tid; p < n_pairs; p += nthr) {
    const int e = ids[p];
    const bool ok = e >= 0 && e < E;
    atomicAdd(&cnt[ok ? e : E], 1);
    if (!ok) s_bad = 1;
  }
  __syncthreads();
  // 2. exclusive prefix over the E + 1 counts (one warp), and the block
  //    offsets of every expert (blocks of at most kMoeBlock pairs)
  if (warp == 0) {
    int run = 0, brun = 0, mx = 0, used = 0;
    for (int base = 0; base <= E; base += 32) {
      const int e = base + lane;
      const int c = e <= E ? cnt[e] : 0;
      const int nb = (e < E) ? (c + kMoeBlock - 1) / kMoeBlock : 0;
      int incl = c, bincl = nb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        const int bv = __shfl_up_sync(0xffffffffu, bincl, o);
        if (lane >= o) { incl += v; bincl += bv; }
      }
      if (e <= E) {
        start[e] = run + incl - c;
        fill[e] = brun + bincl - nb;  // block offset of expert e (fill is reset below)
      }
      int m = (e < E) ? c : 0, u = (e < E && c > 0) ? 1 : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        u += __shfl_xor_sync(0xffffffffu, u, o);
      }
      mx = max(mx, m);
      used += u;
      run += __shfl_sync(0xffffffffu, incl, 31);
      brun += __shfl_sync(0xffffffffu, bincl, 31);
    }
    if (lane == 0) { s_nb = brun; s_max = mx; s_used = used; }
  }
  __syncthreads();
  // 3. per-expert tables: tpe, offsets, and the block list
  for (int e = tid; e <= E; e += nthr) {
    ws[L.off + e] = start[e];
    if (e < E) {
      ws[L.tpe + e] = cnt[e];
      const int nb = (cnt[e] + kMoeBlock - 1) / kMoeBlock;
      for (int k = 0; k < nb; ++k) {
        ws[L.blk_e + fill[e] + k] = e;
        ws[L.blk_s + fill[e] + k] = start[e] + k * kMoeBlock;
      }
    }
  }
  if (tid == 0) {
    ws[L.args + 0] = s_nb;
    ws[L.args + 1] = s_max;
    ws[L.args + 2] = s_used;
    if (s_bad) set_status(d_status, QMM_ERR_BAD_EXPERT_ID);
  }
  __syncthreads();
  for (int e = tid; e <= E; e += nthr) fill[e] = 0;
  __syncthreads();
  // 4. pair indices grouped by expert (the order inside a group is free: every
  //    output row is computed on its own, whatever shares its tile)
  for (int p = tid; p < n_pairs; p += nthr) {
    const int e = ids[p];
    const int ee = (e >= 0 && e < E) ? e : E;
    ws[L.pairs + start[ee] + atomicAdd(&fill[ee], 1)] = p;
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Byte offset (from the workspace start) of the gathered activation rows,
// and the workspace bytes with them: 256-byte aligned rows region after the
// schedule.
constexpr int64_t moe_xg_offset(int64_t n_pairs, int64_t E) { return (moe_ws_layout(n_pairs, E).total * 4 + 255) / 256 * 256; }
constexpr int64_t moe_xg_bytes(int64_t n_pairs, int64_t E, int64_t K) {
  return moe_xg_offset(n_pairs, E) + n_pairs * K * 2;
}

// xg[i, :] = a[row(pairs[i]), :] for every entry i of the pair list (the
// schedule's order), one warp per row, 16-byte copies (K * 2 % 16 == 0).
__global__ void __launch_bounds__(256)
moe_gather_kernel(const uint4* __restrict__ a, const int32_t* __restrict__ pairs, int n_pairs, int top_k, int ne11,
                  int K, uint4* __restrict__ xg) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int vpr = K * 2 / 16;  // 16-byte vectors per row
  for (int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < n_pairs; i += gridDim.x * (blockDim.x >> 5)) {
    const int pr = __ldg(pairs + i);
    const int64_t row = ne11 == 1 ? pr / top_k : pr;
    const uint4* src = a + row * vpr;
    uint4* dst = xg + (int64_t)i * vpr;
    for (int v = lane; v < vpr; v += 32) dst[v] = __ldg(src + v);
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace qmm

using qmm::MoeWs;

namespace {

bool dtype_ok16(int d) { return d == QMM_BF16 || d == QMM_F16; }

qmm_status route(const int32_t* ids, int64_t n_pairs, int64_t E, void* workspace, int64_t workspace_bytes,
                 int32_t* d_status, cudaStream_t st) {
  const MoeWs L = qmm::moe_ws_layout(n_pairs, E);
  if (workspace_bytes < L.total * 4) return QMM_ERR_INVALID_ARG;
  const size_t smem = (size_t)(3 * (E + 1)) * sizeof(int);
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return QMM_ERR_CUDA;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(qmm::moe_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 99 * 1024) !=
        cudaSuccess)
      return QMM_ERR_CUDA;
    configured[dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(qmm::kRouteThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, qmm::moe_route_kernel, ids, (int)n_pairs, (int)E,
                                           static_cast<int32_t*>(workspace), L, d_status);
  return e == cudaSuccess ? QMM_OK : QMM_ERR_CUDA;
}

qmm_status check_moe_gemm_stack(const qmm_expert_stack* w) {
  if (!w) return QMM_ERR_INVALID_ARG;
  if (!qmm_host::dtype_ok(w->sdtype)) return QMM_ERR_DTYPE;
  if (w->num_experts < 1 || w->num_experts > qmm::kMaxRouteExperts || w->n_rows < 1 ||
      qmm_packed_words_per_row(w->n_cols, w->bits) < 0 || qmm_groups_per_row(w->n_cols, w->group_size) < 0)
    return QMM_ERR_INVALID_ARG;
  if (!qmm_host::aligned16(w->packed) || !qmm_host::aligned16(w->scales) || !qmm_host::aligned16(w->biases))
    return QMM_ERR_ALIGNMENT;
  return QMM_OK;
}

bool aligned4(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" {

int64_t qmm_moe_gemm_workspace_bytes(int64_t n_pairs, int64_t num_experts) {
  if (n_pairs < 0 || n_pairs > INT32_MAX / 2 || num_experts < 1 || num_experts > qmm::kMaxRouteExperts) return -1;
  return qmm::moe_ws_layout(n_pairs, num_experts).total * 4;
}

qmm_status qmm_moe_compute_ids_tpe(const int32_t* ids, int64_t n_pairs, int64_t num_experts, void* workspace,
                                   int64_t workspace_bytes, int32_t* d_status, void* stream) {
  if (n_pairs < 0 || n_pairs > INT32_MAX / 2 || num_experts < 1 || num_experts > qmm::kMaxRouteExperts)
    return QMM_ERR_INVALID_ARG;
  if (!aligned4(workspace) || (n_pairs > 0 && !aligned4(ids))) return QMM_ERR_ALIGNMENT;
  if (d_status && !aligned4(d_status)) return QMM_ERR_ALIGNMENT;
  const qmm_status s = qmm_device_check();
  if (s != QMM_OK) return s;
  return route(ids, n_pairs, num_experts, workspace, workspace_bytes, d_status, (cudaStream_t)stream);
}

int64_t qmm_moe_gemm_workspace_bytes_gathered(int64_t n_pairs, int64_t num_experts, int64_t n_cols) {
  if (qmm_moe_gemm_workspace_bytes(n_pairs, num_experts) < 0 || n_cols < 1 || n_cols > (int64_t)1 << 24) return -1;
  return qmm::moe_xg_bytes(n_pairs, num_experts, n_cols);
}

qmm_status qmm_moe_gemm_id(const void* a, qmm_dtype a_dtype, int64_t batch, int64_t top_k, int64_t ne11,
                           void* workspace, int64_t workspace_bytes, const qmm_expert_stack* w, void* out,
                           qmm_dtype out_dtype, void* stream) {
  qmm_status s = check_moe_gemm_stack(w);
  if (s != QMM_OK) return s;
  if (!qmm_host::dtype_ok(a_dtype) || !qmm_host::dtype_ok(out_dtype)) return QMM_ERR_DTYPE;
  if (a_dtype != w->sdtype) return QMM_ERR_DTYPE;
  if (out_dtype != a_dtype && out_dtype != QMM_F32) return QMM_ERR_DTYPE;
  if (!dtype_ok16(a_dtype)) return QMM_ERR_UNSUPPORTED;  // tensor-core path only
  if (batch < 0 || top_k < 1 || (ne11 != 1 && ne11 != top_k)) return QMM_ERR_INVALID_ARG;
  if (batch > INT32_MAX / 2 / top_k) return QMM_ERR_INVALID_ARG;
  const int64_t n_pairs = batch * top_k;
  if (n_pairs == 0) return QMM_OK;
  const MoeWs L = qmm::moe_ws_layout(n_pairs, w->num_experts);
  if (workspace_bytes < L.total * 4) return QMM_ERR_INVALID_ARG;
  if (!qmm_host::aligned16(a) || !qmm_host::aligned16(out) || !aligned4(workspace)) return QMM_ERR_ALIGNMENT;
  if ((w->n_cols * 2) % 16 != 0) return QMM_ERR_UNSUPPORTED;
  s = qmm_device_check();
  if (s != QMM_OK) return s;
  const int32_t* ws = static_cast<const int32_t*>(workspace);
  cudaStream_t st = (cudaStream_t)stream;
  // a workspace with room for the gathered rows: copy them once in the
  // schedule's order, so that the GEMM loads each tile's rows as one box
  void* xg = nullptr;
  if (workspace_bytes >= qmm::moe_xg_bytes(n_pairs, w->num_experts, w->n_cols)) {
    xg = static_cast<char*>(workspace) + qmm::moe_xg_offset(n_pairs, w->num_experts);
    if ((reinterpret_cast<uintptr_t>(xg) & 15) != 0) return QMM_ERR_ALIGNMENT;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min<int64_t>((n_pairs + 7) / 8, (int64_t)qmm_host::num_sms() * 8));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, qmm::moe_gather_kernel, static_cast<const uint4*>(a), ws + L.pairs, (int)n_pairs,
                           (int)top_k, (int)ne11, (int)w->n_cols, static_cast<uint4*>(xg)) != cudaSuccess)
      return QMM_ERR_CUDA;
  }
  const cudaError_t e =
      qmm::launch_qgemm_moe(a, a_dtype, batch * ne11, w, ws + L.off, ws + L.args, ws + L.pairs, ws + L.blk_e,
                            ws + L.blk_s, (int)top_k, (int)ne11, (int)n_pairs, xg, out, out_dtype, st);
  if (e == cudaErrorNotSupported) return QMM_ERR_UNSUPPORTED;
  return e == cudaSuccess ? QMM_OK : QMM_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free form of the MoE prefill GEMM.  Some callers cannot hand
// this library a workspace: an operator or plugin interface that gives the op
// only its input and output tensors, or a latency-critical path on which
// cudaMalloc (which may synchronize the device) is not allowed.  For them the
// routing schedule lives in a fixed array in this library's own device
// memory, sized for the largest call below; every GPU that loads the library
// holds it (70 KB) until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr int64_t kNoAllocMaxPairs = 16384;   // batch * top_k
constexpr int64_t kNoAllocMaxExperts = 256;
constexpr int64_t kNoAllocWords = qmm::moe_ws_layout(kNoAllocMaxPairs, kNoAllocMaxExperts).total;

// The scratch.  Host code must not pass this name to a kernel (on the host it
// is only a stand-in for the device symbol): the device address comes from
// cudaGetSymbolAddress, once per device.
static __device__ __align__(256) int32_t g_moe_scratch[kNoAllocWords];

// Device address of the scratch on the current device (looked up on the first
// call per device, with that device current).
qmm_status scratch_address(int32_t** out) {
  static int32_t* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QMM_ERR_CUDA;
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_moe_scratch) != cudaSuccess || p == nullptr) return QMM_ERR_CUDA;
    cache[dev] = static_cast<int32_t*>(p);
  }
  *out = cache[dev];
  return QMM_OK;
}

}  // namespace

extern "C" qmm_status qmm_moe_gemm_id_noalloc(const void* a, qmm_dtype a_dtype, const int32_t* ids, int64_t batch,
                                              int64_t top_k, int64_t ne11, const qmm_expert_stack* w, void* out,
                                              qmm_dtype out_dtype, int32_t* d_status, void* stream) {
  qmm_status s = check_moe_gemm_stack(w);
  if (s != QMM_OK) return s;
  if (!qmm_host::dtype_ok(a_dtype) || !qmm_host::dtype_ok(out_dtype)) return QMM_ERR_DTYPE;
  if (a_dtype != w->sdtype) return QMM_ERR_DTYPE;
  if (out_dtype != a_dtype && out_dtype != QMM_F32) return QMM_ERR_DTYPE;
  if (!dtype_ok16(a_dtype)) return QMM_ERR_UNSUPPORTED;
  if (batch < 0 || top_k < 1 || (ne11 != 1 && ne11 != top_k)) return QMM_ERR_INVALID_ARG;
  // the built-in scratch serves at most kNoAllocMaxPairs pairs and
  // kNoAllocMaxExperts experts
  if (batch > kNoAllocMaxPairs / top_k || w->num_experts > kNoAllocMaxExperts) return QMM_ERR_UNSUPPORTED;
  const int64_t n_pairs = batch * top_k;
  if (n_pairs == 0) return QMM_OK;
  if (!qmm_host::aligned16(a) || !qmm_host::aligned16(out) || !aligned4(ids)) return QMM_ERR_ALIGNMENT;
  if (d_status && !aligned4(d_status)) return QMM_ERR_ALIGNMENT;
  if ((w->n_cols * 2) % 16 != 0) return QMM_ERR_UNSUPPORTED;
  s = qmm_device_check();
  if (s != QMM_OK) return s;
  int32_t* ws = nullptr;
  s = scratch_address(&ws);
  if (s != QMM_OK) return s;
  // the routing step rewrites every field of the scratch that the GEMM reads
  cudaStream_t st = (cudaStream_t)stream;
  s = route(ids, n_pairs, w->num_experts, ws, kNoAllocWords * 4, d_status, st);
  if (s != QMM_OK) return s;
  const MoeWs L = qmm::moe_ws_layout(n_pairs, w->num_experts);
  const cudaError_t e =
      qmm::launch_qgemm_moe(a, a_dtype, batch * ne11, w, ws + L.off, ws + L.args, ws + L.pairs, ws + L.blk_e,
                            ws + L.blk_s, (int)top_k, (int)ne11, (int)n_pairs, nullptr, out, out_dtype, st);
  if (e == cudaErrorNotSupported) return QMM_ERR_UNSUPPORTED;
  return e == cudaSuccess ? QMM_OK : QMM_ERR_CUDA;
}
