// sdpa_api.cu -- host side of the C ABI declared in include/sdpa.h:
// argument validation (before anything is queued), TMA tensor maps,
// T5 bucket thresholds, workspace plans, kernel launches, and the device
// status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "sdpa.h"
#include "attn_common.cuh"
#include "bias_grad.cuh"
#include "fire.cuh"
#include "bwd_kernels.cuh"
#include "fwd_kernel.cuh"

using namespace sdpa;

namespace {

uint64_t g_wait_limit_ns = 2000000000ull;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shapes of one call: B sequences of Lq query and Lk key rows (padded), or
// B packed sequences along one axis of total_q / total_k rows whose
// lengths are at most Lq / Lk.
struct Geometry {
  int64_t B, Lq, Lk, Hq, Hkv, d;
  bool packed;
  int64_t total_q, total_k;
  const int32_t* cu_q;
  const int32_t* cu_k;
  int64_t sq_b, sq_l, sq_h, skv_b, skv_l, skv_h;
  // positions along the query / key sequence axis (per head)
  int64_t axis_q() const { return packed ? total_q : B * Lq; }
  // rows of LSE, D and the dQ accumulator
  int64_t rows() const { return Hq * axis_q(); }
};

sdpa_status_t make_geometry(const sdpa_shape* s, const sdpa_varlen* vl, Geometry& g) {
  if (!s) return SDPA_ERR_INVALID_ARG;
  g = Geometry{};
  g.B = s->B;
  g.Hq = s->Hq;
  g.Hkv = s->Hkv;
  g.d = s->d;
  if (g.B < 1 || g.Hq < 1 || g.Hkv < 1) return SDPA_ERR_INVALID_ARG;
  if (g.Hq % g.Hkv != 0) return SDPA_ERR_INVALID_ARG;
  if (g.d != 64 && g.d != 128) return SDPA_ERR_UNSUPPORTED;
  if (g.B > 65535 || g.Hq > 65535) return SDPA_ERR_UNSUPPORTED;
  g.sq_l = s->sq_l;
  g.sq_h = s->sq_h;
  g.skv_l = s->skv_l;
  g.skv_h = s->skv_h;
  if (vl) {
    if (!vl->cu_seqlens_q || !vl->cu_seqlens_k) return SDPA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(vl->cu_seqlens_q) & 3u) ||
        (reinterpret_cast<uintptr_t>(vl->cu_seqlens_k) & 3u))
      return SDPA_ERR_INVALID_ARG;
    g.packed = true;
    g.cu_q = vl->cu_seqlens_q;
    g.cu_k = vl->cu_seqlens_k;
    g.Lq = vl->max_seqlen_q;
    g.Lk = vl->max_seqlen_k;
    g.total_q = vl->total_q;
    g.total_k = vl->total_k;
    if (g.Lq < 1 || g.Lk < 1 || g.total_q < 1 || g.total_k < 1) return SDPA_ERR_INVALID_ARG;
    if (g.total_q >= (1ll << 30) || g.total_k >= (1ll << 30)) return SDPA_ERR_UNSUPPORTED;
    g.sq_b = 0;
    g.skv_b = 0;
  } else {
    g.Lq = s->L;
    g.Lk = s->Lk > 0 ? s->Lk : s->L;
    if (g.Lq < 1 || s->Lk < 0) return SDPA_ERR_INVALID_ARG;
    g.sq_b = s->sq_b;
    g.skv_b = s->skv_b;
    if (g.sq_b <= 0 || (g.sq_b % 8) != 0 || g.sq_b >= (1ll << 38)) return SDPA_ERR_INVALID_ARG;
    if (g.skv_b <= 0 || (g.skv_b % 8) != 0 || g.skv_b >= (1ll << 38)) return SDPA_ERR_INVALID_ARG;
  }
  if (g.Lq >= (1ll << 30) || g.Lk >= (1ll << 30)) return SDPA_ERR_UNSUPPORTED;
  if ((g.Lq + 127) / 128 * g.Hq * g.B >= (1ll << 31)) return SDPA_ERR_UNSUPPORTED;
  if ((g.Lk + 127) / 128 * g.Hkv * g.B >= (1ll << 31)) return SDPA_ERR_UNSUPPORTED;
  const int64_t st[4] = {g.sq_l, g.sq_h, g.skv_l, g.skv_h};
  for (int64_t v : st)
    if (v <= 0 || (v % 8) != 0 || v >= (1ll << 38)) return SDPA_ERR_INVALID_ARG;
  return SDPA_OK;
}

// 4-D map over a bf16 tensor along (head_dim, sequence axis, head, batch),
// box = 64 head-dim elements x 128 rows of one head, 128-byte swizzle.  Rows
// past the axis end read as zero.  Packed sequences: one batch entry over
// the whole packed axis.
bool make_axis_map(CUtensorMap* m, const void* base, const Geometry& g, bool query) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int64_t axis = g.packed ? (query ? g.total_q : g.total_k) : (query ? g.Lq : g.Lk);
  const int64_t H = query ? g.Hq : g.Hkv;
  const int64_t sl = query ? g.sq_l : g.skv_l, sh = query ? g.sq_h : g.skv_h;
  const int64_t sbt = g.packed ? sl * axis : (query ? g.sq_b : g.skv_b);
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(g.d), static_cast<cuuint64_t>(axis),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(g.packed ? 1 : g.B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(sl) * 2, static_cast<cuuint64_t>(sh) * 2,
                           static_cast<cuuint64_t>(sbt) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(kTile), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Dense fp32 bias [B|1, Hq|1, Lq, Lk] as a 4-D map (j, i, head, batch) with
// boxes of 32 keys x 128 queries (128-byte swizzle); a broadcast index has
// extent 1 and is always addressed at 0.
bool make_bias_map(CUtensorMap* m, const AttnParams& p) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(p.sb_i) * 4;
  const cuuint64_t head = p.sb_h ? static_cast<cuuint64_t>(p.sb_h) * 4 : row * p.Lq;
  const cuuint64_t batch = p.sb_b ? static_cast<cuuint64_t>(p.sb_b) * 4 : head * (p.sb_h ? p.Hq : 1);
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(p.Lk), static_cast<cuuint64_t>(p.Lq),
                        static_cast<cuuint64_t>(p.sb_h ? p.Hq : 1),
                        static_cast<cuuint64_t>(p.sb_b ? p.B : 1)};
  cuuint64_t strides[3] = {row, head, batch};
  cuuint32_t box[4] = {32, static_cast<cuuint32_t>(kTile), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float*>(p.bias), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Integer thresholds of the T5 log buckets, evaluated in float64 exactly as
// the closed form reads: large(n) = max_exact + trunc(ln(n / max_exact) /
// ln(max_distance / max_exact) * (half - max_exact)).
bool fill_t5(T5Spec& t, int nb, int md, int bidir) {
  const int half = bidir ? nb / 2 : nb;
  const int me = half / 2;
  if (me < 1 || md <= me) return false;
  const int K = half - me;
  if (K > kMaxT5Thresholds) return false;
  t.half = half;
  t.max_exact = me;
  t.bidirectional = bidir ? 1 : 0;
  t.nthr = K;
  const double denom = std::log(static_cast<double>(md) / static_cast<double>(me));
  auto large = [&](int64_t n) -> int64_t {
    const double v = std::log(static_cast<double>(n) / static_cast<double>(me)) / denom *
                     static_cast<double>(half - me);
    return me + static_cast<int64_t>(v);
  };
  const int64_t limit = 4 * static_cast<int64_t>(md) + 1024;
  int64_t n = me;
  for (int k = 0; k < K; ++k) {
    while (n < limit && large(n) < me + k) ++n;
    t.thr[k] = (n < limit) ? static_cast<int>(n) : INT_MAX;
  }
  for (int k = K; k < kMaxT5Thresholds; ++k) t.thr[k] = INT_MAX;
  // the capped bucket (half - 1) holds every n >= thr[K - 1]
  const int sat = t.thr[K - 1];
  t.one_lo_max = sat == INT_MAX ? INT_MIN : -sat;
  t.one_hi_min = bidir ? sat : 0;
  t.log_scale = static_cast<float>(static_cast<double>(half - me) / std::log2(static_cast<double>(md) / me));
  t.inv_max_exact = static_cast<float>(1.0 / me);
  return true;
}

int clamp_window(int64_t w, int64_t L) {
  if (w < 0) return -1;
  return static_cast<int>(w > L ? L : w);
}

// Validation of mask / bias and the common fields of p for geometry g.
sdpa_status_t prepare(const Geometry& g, const sdpa_bias_desc* bias, const sdpa_mask_spec* mask,
                      float scale, AttnParams& p) {
  if (!mask) return SDPA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return SDPA_ERR_INVALID_ARG;
  std::memset(&p, 0, sizeof(p));
  p.B = static_cast<int>(g.B);
  p.Lq = static_cast<int>(g.Lq);
  p.Lk = static_cast<int>(g.Lk);
  p.Hq = static_cast<int>(g.Hq);
  p.Hkv = static_cast<int>(g.Hkv);
  p.G = p.Hq / p.Hkv;
  const int64_t span = std::max(g.Lq, g.Lk);
  p.causal = mask->causal ? 1 : 0;
  p.wl = clamp_window(mask->window_left, span);
  p.wr = clamp_window(mask->window_right, span);
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.sq_b = g.sq_b;
  p.sq_l = g.sq_l;
  p.sq_h = g.sq_h;
  p.skv_b = g.skv_b;
  p.skv_l = g.skv_l;
  p.skv_h = g.skv_h;
  if (g.packed) {
    p.cu_q = g.cu_q;
    p.cu_k = g.cu_k;
    p.total_q = static_cast<int>(g.total_q);
    p.total_k = static_cast<int>(g.total_k);
    p.lse_sb = 0;
    p.lse_sh = g.total_q;
  } else {
    p.lse_sb = g.Hq * g.Lq;
    p.lse_sh = g.Lq;
  }
  p.wait_limit_ns = g_wait_limit_ns;
  p.bias_kind = kBiasNone;
  if (bias && bias->kind != SDPA_BIAS_NONE) {
    if (bias->kind == SDPA_BIAS_DENSE) {
      if (g.packed) return SDPA_ERR_UNSUPPORTED;  // a [B, H, L, L] tensor has no packed form
      if (!bias->ptr || !aligned16(bias->ptr)) return SDPA_ERR_INVALID_ARG;
      if (bias->stride_b < 0 || bias->stride_h < 0 || bias->stride_i < 0) return SDPA_ERR_INVALID_ARG;
      if (bias->stride_b % 4 != 0 || bias->stride_h % 4 != 0 || bias->stride_i % 4 != 0)
        return SDPA_ERR_INVALID_ARG;
      // a bias broadcast over query rows has no 2-D tile layout for the
      // tensor-memory copies that stage bias blocks
      if (bias->stride_i == 0) return SDPA_ERR_UNSUPPORTED;
      p.bias_kind = kBiasDense;
      p.bias = bias->ptr;
      p.sb_b = bias->stride_b;
      p.sb_h = bias->stride_h;
      p.sb_i = bias->stride_i;
    } else if (bias->kind == SDPA_BIAS_T5) {
      if (!bias->ptr) return SDPA_ERR_INVALID_ARG;
      const int nb = bias->num_buckets;
      if (nb < 2 || nb > 128) return SDPA_ERR_INVALID_ARG;
      if (bias->bidirectional && (nb % 2) != 0) return SDPA_ERR_INVALID_ARG;
      if (!fill_t5(p.t5, nb, bias->max_distance, bias->bidirectional)) return SDPA_ERR_INVALID_ARG;
      p.bias_kind = kBiasT5;
      p.t5_table = bias->ptr;
    } else if (bias->kind == SDPA_BIAS_ALIBI) {
      if (!bias->ptr) return SDPA_ERR_INVALID_ARG;
      p.bias_kind = kBiasT5;  // the relative-position kernels, with the ALiBi table
      p.alibi = 1;
      p.alibi_slopes = bias->ptr;
    } else if (bias->kind == SDPA_BIAS_REL) {
      if (!bias->ptr) return SDPA_ERR_INVALID_ARG;
      p.bias_kind = kBiasT5;  // the relative-position kernels, with the caller's table
      p.rel_table = bias->ptr;
      p.rel_off = p.Lq - 1;
      p.rel_rows = p.Lq + p.Lk - 1;
    } else {
      return SDPA_ERR_INVALID_ARG;
    }
  }
  return SDPA_OK;
}

// ------------------------------------------------------------- forward
template <int D, int BIAS>
cudaError_t launch_fwd(const AttnParams& p, const CUtensorMap& q, const CUtensorMap& k,
                       const CUtensorMap& v, const CUtensorMap& bmap, cudaStream_t st) {
  using Lay = FwdLayout<D, BIAS>;
  auto kern = fwd_kernel<D, BIAS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Lay::kSmemAlloc);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM (or per work item, if fewer)
  const int64_t items = static_cast<int64_t>((p.Lq + kTile - 1) / kTile) * p.Hq * p.B;
  const int sms = sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int grid = static_cast<int>(items < sms ? items : sms);
  kern<<<grid, Lay::kThreads, Lay::kSmemAlloc, st>>>(p, q, k, v, bmap);
  return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_fwd_bias(const AttnParams& p, const CUtensorMap& q, const CUtensorMap& k,
                              const CUtensorMap& v, const CUtensorMap& bmap, cudaStream_t st) {
  switch (p.bias_kind) {
    case kBiasDense: return launch_fwd<D, kBiasDense>(p, q, k, v, bmap, st);
    case kBiasT5: return launch_fwd<D, kBiasT5>(p, q, k, v, bmap, st);
    default: return launch_fwd<D, kBiasNone>(p, q, k, v, bmap, st);
  }
}

sdpa_status_t run_fwd(const Geometry& g, const void* q, const void* k, const void* v,
                      const sdpa_bias_desc* bias, const sdpa_mask_spec* mask, float scale,
                      void* o, float* lse, void* stream) {
  AttnParams p;
  sdpa_status_t st = prepare(g, bias, mask, scale, p);
  if (st != SDPA_OK) return st;
  if (!q || !k || !v || !o || !lse) return SDPA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return SDPA_ERR_INVALID_ARG;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  CUtensorMap mq, mk, mv, mb;
  if (!make_axis_map(&mq, q, g, true) || !make_axis_map(&mk, k, g, false) ||
      !make_axis_map(&mv, v, g, false))
    return SDPA_ERR_CUDA;
  std::memset(&mb, 0, sizeof(mb));  // read only by the dense-bias kernels
  if (p.bias_kind == kBiasDense && !make_bias_map(&mb, p)) return SDPA_ERR_CUDA;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e = (g.d == 128) ? dispatch_fwd_bias<128>(p, mq, mk, mv, mb, cs)
                               : dispatch_fwd_bias<64>(p, mq, mk, mv, mb, cs);
  return e == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

// ------------------------------------------------------------ backward
BwdWorkspace plan_of(const Geometry& g) { return bwd_workspace_plan(g.rows()); }

// The backward's pointers, with its workspace (laid out by plan_of) at ws.
sdpa_status_t bind_bwd(AttnParams& p, const Geometry& g, const void* o, const void* dout,
                       const float* lse, void* dq, void* dk, void* dv, void* ws) {
  const BwdWorkspace pl = plan_of(g);
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.o = const_cast<__nv_bfloat16*>(static_cast<const __nv_bfloat16*>(o));
  p.lse = const_cast<float*>(lse);
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.dvec = reinterpret_cast<float*>(w + pl.d_off);
  return SDPA_OK;
}

// Tensor maps, then the launches selected by `phases`.
sdpa_status_t run_bwd(uint32_t phases, const AttnParams& p, const Geometry& g, const void* q,
                      const void* k, const void* v, const void* dout, cudaStream_t stream) {
  CUtensorMap mq, mk, mv, mdo, mb;
  if (!make_axis_map(&mq, q, g, true) || !make_axis_map(&mdo, dout, g, true) ||
      !make_axis_map(&mk, k, g, false) || !make_axis_map(&mv, v, g, false))
    return SDPA_ERR_CUDA;
  std::memset(&mb, 0, sizeof(mb));  // read only by the dense-bias kernels at d = 64
  if (p.bias_kind == kBiasDense && !make_bias_map(&mb, p)) return SDPA_ERR_CUDA;
  cudaError_t e = g.d == 128 ? launch_bwd_d<128>(p, mq, mk, mv, mdo, mb, phases, g.axis_q(), stream)
                             : launch_bwd_d<64>(p, mq, mk, mv, mdo, mb, phases, g.axis_q(), stream);
  return e == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

sdpa_status_t core_bwd(uint32_t phases, const Geometry& g, const void* q, const void* k,
                       const void* v, const void* o, const void* dout, const float* lse,
                       const sdpa_bias_desc* bias, const sdpa_mask_spec* mask, float scale,
                       void* dq, void* dk, void* dv, int32_t deterministic, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (phases == 0 || (phases & ~static_cast<uint32_t>(SDPA_BWD_ALL)) != 0)
    return SDPA_ERR_INVALID_ARG;
  AttnParams p;
  sdpa_status_t st = prepare(g, bias, mask, scale, p);
  if (st != SDPA_OK) return st;
  if (deterministic != 1) return SDPA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, o, dout, lse, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return SDPA_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < plan_of(g).total)
    return SDPA_ERR_WORKSPACE;
  bind_bwd(p, g, o, dout, lse, dq, dk, dv, workspace);
  return run_bwd(phases, p, g, q, k, v, dout, static_cast<cudaStream_t>(stream));
}

// ----- bias gradients: workspace plan (sdpa_bwd_bias_grad) -----
size_t round256(size_t x) { return (x + 255) / 256 * 256; }

struct BiasGradPlan {
  size_t bwd_bytes = 0;   // the backward's own workspace
  bool ds_ws = false;     // dS staged in the workspace (else written into dbias)
  int64_t lp = 0;         // row stride of the staged dS
  size_t ds_bytes = 0;
  int chunks = 1;         // pieces of the reduced index
  int64_t per_chunk = 0;  // reduced indices per piece
  size_t part_bytes = 0;  // partial sums of the pieces
  // relative-position table: the dQ kernel's per-warp diagonal sums, then
  // per-tile and per-head diagonal sums (no dS)
  bool diag = false;
  // T5 table: the dQ kernel's per-bucket sums per (batch, head, query tile, warp)
  bool buckets = false;
  size_t warp_bytes = 0, tile_bytes = 0, band_bytes = 0, diag_bytes = 0;
  // ALiBi: the dQ kernel's per-warp sums of |j - i| dS
  bool moment = false;
  size_t total = 0;
};

// Splits n_red reduced indices into pieces so that `blocks` output blocks per
// piece give about kReduceTargetBlocks blocks in all (at most 65535 pieces).
void split_reduction(int64_t n_red, int64_t blocks, int& chunks, int64_t& per_chunk) {
  int64_t c = (kReduceTargetBlocks + blocks - 1) / blocks;
  c = c < 1 ? 1 : c;
  c = c > n_red ? n_red : c;
  c = c > 65535 ? 65535 : c;
  per_chunk = (n_red + c - 1) / c;
  chunks = static_cast<int>((n_red + per_chunk - 1) / per_chunk);
}

// The bias gradient is built for self-attention of one padded length.
sdpa_status_t plan_bias_grad(const Geometry& g, const sdpa_bias_desc* bias, BiasGradPlan& pl) {
  if (!bias) return SDPA_ERR_INVALID_ARG;
  if (g.packed || g.Lq != g.Lk) return SDPA_ERR_UNSUPPORTED;
  const int64_t B = g.B, Hq = g.Hq, L = g.Lq;
  pl = BiasGradPlan{};
  pl.bwd_bytes = plan_of(g).total;
  pl.lp = (L + 7) / 8 * 8;  // staged dS rows start on 32-byte boundaries
  // B * Hq * L * lp floats must stay far from 2^63 bytes
  const double ds_elems = static_cast<double>(B) * Hq * L * pl.lp;
  if (bias->kind == SDPA_BIAS_DENSE) {
    // the kept indices must nest b > h > i without overlap, so that each
    // gradient entry has exactly one address
    int64_t span = L;
    const int64_t st[3] = {bias->stride_i, bias->stride_h, bias->stride_b};
    const int64_t ex[3] = {L, Hq, B};
    for (int a = 0; a < 3; ++a) {
      if (st[a] < 0) return SDPA_ERR_INVALID_ARG;
      if (st[a] == 0) continue;
      if (st[a] < span) return SDPA_ERR_UNSUPPORTED;
      span = st[a] * ex[a];
    }
    if (bias->stride_i == 0) return SDPA_ERR_UNSUPPORTED;
    pl.ds_ws = bias->stride_b == 0 || bias->stride_h == 0;
    if (pl.ds_ws) {
      if (ds_elems > 1e17) return SDPA_ERR_UNSUPPORTED;
      pl.ds_bytes = round256(static_cast<size_t>(B * Hq * L * pl.lp) * sizeof(float));
      const int64_t n_out = (bias->stride_b ? B : 1) * (bias->stride_h ? Hq : 1) * L;
      const int64_t n_red = (bias->stride_b ? 1 : B) * (bias->stride_h ? 1 : Hq);
      split_reduction(n_red, n_out * ((L + 255) / 256), pl.chunks, pl.per_chunk);
      if (pl.chunks > 1)
        pl.part_bytes = round256(static_cast<size_t>(pl.chunks * n_out * pl.lp) * sizeof(float));
    }
  } else if (bias->kind == SDPA_BIAS_ALIBI) {
    // per (batch, head, query tile, key tile): 8 per-warp sums
    const int64_t nt = (L + kTile - 1) / kTile;
    const double tiles = static_cast<double>(B) * Hq * nt * nt;
    if (tiles * 8.0 > 1e16) return SDPA_ERR_UNSUPPORTED;
    pl.moment = true;
    pl.part_bytes = round256(static_cast<size_t>(B * Hq * nt * nt) * 8 * sizeof(float));
  } else if (bias->kind == SDPA_BIAS_T5) {
    const int64_t nt = (L + kTile - 1) / kTile;
    const int64_t nb = bias->num_buckets;
    if (nb < 1 || nb > 128) return SDPA_ERR_INVALID_ARG;
    if (static_cast<double>(B) * Hq * nt * 8 * nb > 1e15 || B * nt * 8 > (1ll << 30))
      return SDPA_ERR_UNSUPPORTED;
    pl.buckets = true;
    pl.part_bytes = round256(static_cast<size_t>(B * Hq * nt * 8 * nb) * sizeof(float));
  } else if (bias->kind == SDPA_BIAS_REL) {
    // per (batch, head, query tile, key tile): 1024 per-warp sums and 256
    // tile diagonals; per head: 2L - 1 diagonal totals
    const int64_t nt = (L + kTile - 1) / kTile;
    const double tiles = static_cast<double>(B) * Hq * nt * nt;
    if (tiles * 1280.0 > 1e16 || nt > 65535 || B * Hq > 65535) return SDPA_ERR_UNSUPPORTED;
    pl.diag = true;
    const size_t n_tiles = static_cast<size_t>(B * Hq * nt * nt);
    pl.warp_bytes = round256(n_tiles * 1024 * sizeof(float));
    pl.tile_bytes = round256(n_tiles * 256 * sizeof(float));
    pl.band_bytes = round256(static_cast<size_t>(B * Hq * (2 * nt - 1) * 256) * sizeof(float));
    pl.diag_bytes = round256(static_cast<size_t>(Hq * (2 * L - 1)) * sizeof(float));
    pl.part_bytes = pl.warp_bytes + pl.tile_bytes + pl.band_bytes + pl.diag_bytes;
  } else {
    return SDPA_ERR_UNSUPPORTED;  // no bias: nothing to differentiate
  }
  pl.total = pl.bwd_bytes + pl.ds_bytes + pl.part_bytes;
  return SDPA_OK;
}

// The contiguous range [lo, hi] of distances r = j - i in [-(L-1), L-1]
// that fall in each T5 bucket (hi < lo when none does).  False if some
// bucket's distances are not contiguous, which the bucket function rules out.
bool t5_ranges(const T5Spec& t, int L, int num_buckets, T5Ranges& rg) {
  for (int k = 0; k < 128; ++k) {
    rg.lo[k] = 0;
    rg.hi[k] = -1;
  }
  std::vector<char> seen(num_buckets, 0);
  int prev = -1;
  for (int r = -(L - 1); r <= L - 1; ++r) {
    const int k = t5_bucket(r, t);
    if (k < 0 || k >= num_buckets) return false;
    if (k != prev) {
      if (seen[k]) return false;
      seen[k] = 1;
      rg.lo[k] = r;
      prev = k;
    }
    rg.hi[k] = r;
  }
  return true;
}

__global__ void exp2_fma_kernel(const float* x, float* y, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = exp2_fma(x[i]);
}

__global__ void t5_bucket_kernel(const int32_t* rel, int32_t* out, int64_t n, T5Spec spec) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = t5_bucket(rel[i], spec);
}

// One barrier that nothing ever completes, waited on under the wait limit.
__global__ void wait_timeout_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_storage), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{&abort_flag, limit_ns};
    (void)mbar_wait(smem_u32(&bar_storage), 0, ctl);
  }
  __syncthreads();
}

}  // namespace

extern "C" {

const char* sdpa_status_string(sdpa_status_t s) {
  switch (s) {
    case SDPA_OK: return "ok";
    case SDPA_ERR_INVALID_ARG: return "invalid argument";
    case SDPA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SDPA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SDPA_ERR_CUDA: return "CUDA error";
    case SDPA_ERR_TIMEOUT: return "in-kernel wait timed out";
  }
  return "unknown status";
}

void sdpa_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns < 1000 ? 1000 : ns; }

sdpa_status_t sdpa_fwd(const sdpa_shape* shape, const void* q, const void* k, const void* v,
                       const sdpa_bias_desc* bias, const sdpa_mask_spec* mask, float scale,
                       void* o, float* lse, void* stream) {
  Geometry g;
  sdpa_status_t st = make_geometry(shape, nullptr, g);
  if (st != SDPA_OK) return st;
  return run_fwd(g, q, k, v, bias, mask, scale, o, lse, stream);
}

sdpa_status_t sdpa_fwd_varlen(const sdpa_shape* shape, const sdpa_varlen* varlen, const void* q,
                              const void* k, const void* v, const sdpa_bias_desc* bias,
                              const sdpa_mask_spec* mask, float scale, void* o, float* lse,
                              void* stream) {
  if (!varlen) return SDPA_ERR_INVALID_ARG;
  Geometry g;
  sdpa_status_t st = make_geometry(shape, varlen, g);
  if (st != SDPA_OK) return st;
  return run_fwd(g, q, k, v, bias, mask, scale, o, lse, stream);
}

size_t sdpa_bwd_workspace_size(const sdpa_shape* shape, int32_t deterministic) {
  (void)deterministic;
  Geometry g;
  if (make_geometry(shape, nullptr, g) != SDPA_OK) return 0;
  return plan_of(g).total;
}

size_t sdpa_bwd_varlen_workspace_size(const sdpa_shape* shape, const sdpa_varlen* varlen) {
  Geometry g;
  if (!varlen || make_geometry(shape, varlen, g) != SDPA_OK) return 0;
  return plan_of(g).total;
}

sdpa_status_t sdpa_bwd_phases(uint32_t phases, const sdpa_shape* shape, const void* q,
                              const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, const sdpa_bias_desc* bias,
                              const sdpa_mask_spec* mask, float scale, void* dq, void* dk,
                              void* dv, int32_t deterministic, void* workspace,
                              size_t workspace_bytes, void* stream) {
  Geometry g;
  sdpa_status_t st = make_geometry(shape, nullptr, g);
  if (st != SDPA_OK) return st;
  return core_bwd(phases, g, q, k, v, o, dout, lse, bias, mask, scale, dq, dk, dv, deterministic,
                  workspace, workspace_bytes, stream);
}

sdpa_status_t sdpa_bwd(const sdpa_shape* shape, const void* q, const void* k, const void* v,
                       const void* o, const void* dout, const float* lse,
                       const sdpa_bias_desc* bias, const sdpa_mask_spec* mask, float scale,
                       void* dq, void* dk, void* dv, int32_t deterministic, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return sdpa_bwd_phases(SDPA_BWD_ALL, shape, q, k, v, o, dout, lse, bias, mask, scale, dq, dk,
                         dv, deterministic, workspace, workspace_bytes, stream);
}

sdpa_status_t sdpa_bwd_varlen(const sdpa_shape* shape, const sdpa_varlen* varlen, const void* q,
                              const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, const sdpa_bias_desc* bias,
                              const sdpa_mask_spec* mask, float scale, void* dq, void* dk,
                              void* dv, int32_t deterministic, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!varlen) return SDPA_ERR_INVALID_ARG;
  Geometry g;
  sdpa_status_t st = make_geometry(shape, varlen, g);
  if (st != SDPA_OK) return st;
  return core_bwd(SDPA_BWD_ALL, g, q, k, v, o, dout, lse, bias, mask, scale, dq, dk, dv,
                  deterministic, workspace, workspace_bytes, stream);
}

size_t sdpa_bwd_bias_grad_workspace_size(const sdpa_shape* shape, const sdpa_bias_desc* bias) {
  Geometry g;
  if (make_geometry(shape, nullptr, g) != SDPA_OK) return 0;
  BiasGradPlan pl;
  return plan_bias_grad(g, bias, pl) == SDPA_OK ? pl.total : 0;
}

sdpa_status_t sdpa_bwd_bias_grad(const sdpa_shape* shape, const void* q, const void* k,
                                 const void* v, const void* o, const void* dout,
                                 const float* lse, const sdpa_bias_desc* bias,
                                 const sdpa_mask_spec* mask, float scale, void* dq, void* dk,
                                 void* dv, float* dbias, int32_t deterministic, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  Geometry g;
  sdpa_status_t st = make_geometry(shape, nullptr, g);
  if (st != SDPA_OK) return st;
  AttnParams p;
  st = prepare(g, bias, mask, scale, p);
  if (st != SDPA_OK) return st;
  if (p.bias_kind == kBiasNone) return SDPA_ERR_UNSUPPORTED;
  if (deterministic != 1) return SDPA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, k, v, o, dout, lse, dq, dk, dv, dbias};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return SDPA_ERR_INVALID_ARG;
  BiasGradPlan pl;
  st = plan_bias_grad(g, bias, pl);
  if (st != SDPA_OK) return st;
  T5Ranges rg;
  if (p.bias_kind == kBiasT5 && !p.alibi && !p.rel_table &&
      !t5_ranges(p.t5, p.Lq, bias->num_buckets, rg))
    return SDPA_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < pl.total)
    return SDPA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  bind_bwd(p, g, o, dout, lse, dq, dk, dv, ws);
  const int L = p.Lq;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (pl.moment) {
    // ALiBi: per-warp sums of |j - i| dS from the dQ kernel, then per head
    AlibiMoment a;
    a.part = reinterpret_cast<const float*>(ws + pl.bwd_bytes);
    a.out = dbias;
    a.B = p.B;
    a.Hq = p.Hq;
    a.L = L;
    a.nt = (L + kTile - 1) / kTile;
    p.diag_out = reinterpret_cast<float*>(ws + pl.bwd_bytes);
    st = run_bwd(SDPA_BWD_ALL, p, g, q, k, v, dout, cs);
    if (st != SDPA_OK) return st;
    alibi_moment_kernel<<<p.Hq, 1024, 0, cs>>>(a, p);
    return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
  }
  if (pl.buckets) {
    // T5: per-bucket sums per (batch, head, query tile, warp) from the dQ
    // kernel, then per (bucket, head)
    p.t5r = rg;
    p.diag_out = reinterpret_cast<float*>(ws + pl.bwd_bytes);
    st = run_bwd(SDPA_BWD_ALL, p, g, q, k, v, dout, cs);
    if (st != SDPA_OK) return st;
    T5BucketReduce a;
    a.part = p.diag_out;
    a.out = dbias;
    a.B = p.B;
    a.Hq = p.Hq;
    a.nqt = (L + kTile - 1) / kTile;
    a.num_buckets = bias->num_buckets;
    t5_bucket_reduce_kernel<<<dim3(a.num_buckets, p.Hq), 256, 0, cs>>>(a);
    return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
  }
  if (pl.diag) {
    // REL: per-warp diagonal sums from the dQ kernel, folded per tile, per
    // tile offset, then per head, then transposed into the table's layout
    uint8_t* base = ws + pl.bwd_bytes;
    DiagFold f;
    f.warp_part = reinterpret_cast<const float*>(base);
    f.tile_diag = reinterpret_cast<float*>(base + pl.warp_bytes);
    f.band = reinterpret_cast<float*>(base + pl.warp_bytes + pl.tile_bytes);
    f.diag = reinterpret_cast<float*>(base + pl.warp_bytes + pl.tile_bytes + pl.band_bytes);
    f.B = p.B;
    f.Hq = p.Hq;
    f.L = L;
    f.nqt = f.ntk = (L + kTile - 1) / kTile;
    p.diag_out = reinterpret_cast<float*>(base);
    st = run_bwd(SDPA_BWD_ALL, p, g, q, k, v, dout, cs);
    if (st != SDPA_OK) return st;
    diag_tile_fold_kernel<<<dim3(f.nqt, f.ntk, p.B * p.Hq), 256, 0, cs>>>(f, p);
    if (cudaGetLastError() != cudaSuccess) return SDPA_ERR_CUDA;
    diag_band_kernel<<<dim3(2 * f.nqt - 1, p.Hq, p.B), 256, 0, cs>>>(f, p);
    if (cudaGetLastError() != cudaSuccess) return SDPA_ERR_CUDA;
    const unsigned rblocks = static_cast<unsigned>((2 * L - 1 + 127) / 128);
    diag_total_kernel<<<dim3(rblocks, p.Hq), 128, 0, cs>>>(f);
    if (cudaGetLastError() != cudaSuccess) return SDPA_ERR_CUDA;
    T5Reduce a;
    std::memset(&a, 0, sizeof(a));
    a.Hq = p.Hq;
    a.L = L;
    a.partial = f.diag;
    a.out = dbias;
    const int64_t n = static_cast<int64_t>(2 * L - 1) * p.Hq;
    rel_table_grad_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, cs>>>(a);
    return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
  }
  if (pl.ds_ws) {
    p.ds_out = reinterpret_cast<float*>(ws + pl.bwd_bytes);
    p.sd_i = pl.lp;
    p.sd_h = pl.lp * L;
    p.sd_b = p.sd_h * p.Hq;
  } else {
    p.ds_out = dbias;
    p.sd_b = p.sb_b;
    p.sd_h = p.sb_h;
    p.sd_i = p.sb_i;
  }
  const int sms = sm_count();
  if (sms <= 0) return SDPA_ERR_CUDA;
  if (p.causal || p.wl >= 0 || p.wr >= 0) {
    const int64_t rows = static_cast<int64_t>(p.B) * p.Hq * L;
    const int64_t grid = rows < 8ll * sms ? rows : 8ll * sms;
    ds_zero_outside_band_kernel<<<static_cast<unsigned>(grid), 256, 0, cs>>>(p);
    if (cudaGetLastError() != cudaSuccess) return SDPA_ERR_CUDA;
  }
  st = run_bwd(SDPA_BWD_ALL, p, g, q, k, v, dout, cs);
  if (st != SDPA_OK || !pl.ds_ws) return st;
  float* part = reinterpret_cast<float*>(ws + pl.bwd_bytes + pl.ds_bytes);
  if (p.bias_kind == kBiasDense) {
    DenseReduce a;
    a.ds = p.ds_out;
    a.ds_b = p.sd_b;
    a.ds_h = p.sd_h;
    a.ds_i = p.sd_i;
    a.out = dbias;
    a.o_b = p.sb_b;
    a.o_h = p.sb_h;
    a.o_i = p.sb_i;
    a.L = L;
    a.eb = p.sb_b ? p.B : 1;
    a.eh = p.sb_h ? p.Hq : 1;
    a.ei = L;
    a.rb = p.sb_b ? 1 : p.B;
    a.rh = p.sb_h ? 1 : p.Hq;
    a.ri = 1;
    a.n_out = static_cast<int64_t>(a.eb) * a.eh * a.ei;
    a.n_red = static_cast<int64_t>(a.rb) * a.rh * a.ri;
    a.jblocks = (L + 255) / 256;
    a.chunks = pl.chunks;
    a.rchunk = pl.per_chunk;
    a.partial = part;
    a.lp = pl.lp;
    const int64_t work = a.n_out * a.jblocks;
    const int64_t g1 = work < kReduceTargetBlocks ? work : kReduceTargetBlocks;
    dense_bias_reduce_kernel<<<dim3(static_cast<unsigned>(g1), a.chunks), 256, 0, cs>>>(a);
    if (cudaGetLastError() != cudaSuccess) return SDPA_ERR_CUDA;
    if (a.chunks > 1) {
      dense_bias_combine_kernel<<<static_cast<unsigned>(g1), 256, 0, cs>>>(a);
      if (cudaGetLastError() != cudaSuccess) return SDPA_ERR_CUDA;
    }
  }
  return SDPA_OK;
}

// ---------------------------------------------------------------------
// sdpa_bwd_noalloc: the backward's workspace in a fixed device array
// instead of caller memory, for callers that cannot allocate device memory
// (see include/sdpa.h).  In host code `g_noalloc_scratch` names a host-side
// stand-in, not device memory, so the kernels are given the device address
// looked up with cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[SDPA_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, or nullptr.
void* noalloc_scratch_ptr() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = ptr;
  }
  return g_noalloc_ptr[dev];
}
}  // namespace

sdpa_status_t sdpa_bwd_noalloc(const sdpa_shape* shape, const void* q, const void* k,
                               const void* v, const void* o, const void* dout, const float* lse,
                               const sdpa_bias_desc* bias, const sdpa_mask_spec* mask,
                               float scale, void* dq, void* dk, void* dv, int32_t deterministic,
                               void* stream) {
  Geometry g;
  sdpa_status_t st = make_geometry(shape, nullptr, g);
  if (st != SDPA_OK) return st;
  if (plan_of(g).total > sizeof(g_noalloc_scratch)) return SDPA_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_ptr();
  if (!scratch) return SDPA_ERR_CUDA;
  return core_bwd(SDPA_BWD_ALL, g, q, k, v, o, dout, lse, bias, mask, scale, dq, dk, dv,
                  deterministic, scratch, sizeof(g_noalloc_scratch), stream);
}

sdpa_status_t sdpa_t5_bucket(const int32_t* rel, int32_t* out, int64_t n, int32_t num_buckets,
                             int32_t max_distance, int32_t bidirectional, void* stream) {
  if (n < 0 || (n > 0 && (!rel || !out))) return SDPA_ERR_INVALID_ARG;
  if (num_buckets < 2 || num_buckets > 128 || (bidirectional && (num_buckets % 2) != 0))
    return SDPA_ERR_INVALID_ARG;
  T5Spec spec;
  if (!fill_t5(spec, num_buckets, max_distance, bidirectional)) return SDPA_ERR_INVALID_ARG;
  if (n == 0) return SDPA_OK;
  const int64_t blocks = (n + 255) / 256;
  t5_bucket_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0,
                     static_cast<cudaStream_t>(stream)>>>(rel, out, n, spec);
  return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

sdpa_status_t sdpa_exp2_fma(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return SDPA_ERR_INVALID_ARG;
  if (n == 0) return SDPA_OK;
  const int64_t blocks = (n + 255) / 256;
  exp2_fma_kernel<<<static_cast<unsigned>(blocks < 4096 ? blocks : 4096), 256, 0,
                    static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

sdpa_status_t sdpa_read_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SDPA_ERR_CUDA;
  unsigned int h = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&h, g_device_status, sizeof(h)) != cudaSuccess) return SDPA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return SDPA_ERR_CUDA;
  if (h & kStatusTimeout) return SDPA_ERR_TIMEOUT;
  if (h & (kStatusMisaligned | kStatusBadSeqlens)) return SDPA_ERR_UNSUPPORTED;
  return SDPA_OK;
}

sdpa_status_t sdpa_debug_wait_timeout(void* stream) {
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(g_wait_limit_ns);
  return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

// ------------------------------------------------------------------ FIRE
namespace {
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

sdpa_status_t fire_check(const sdpa_fire* f, int64_t Lq, int64_t Lk, FireArgs& a) {
  if (!f || !f->w1 || !f->b1 || !f->w2 || !f->b2) return SDPA_ERR_INVALID_ARG;
  if (!aligned4(f->w1) || !aligned4(f->b1) || !aligned4(f->w2) || !aligned4(f->b2))
    return SDPA_ERR_INVALID_ARG;
  if (f->width < 1 || f->width > 1024 || f->heads < 1 || f->heads > 65535)
    return SDPA_ERR_INVALID_ARG;
  if (!std::isfinite(f->c) || !(f->c > 0.f) || !std::isfinite(f->threshold))
    return SDPA_ERR_INVALID_ARG;
  if (Lq < 1 || Lk < 1 || Lq >= (1ll << 30) || Lk >= (1ll << 30)) return SDPA_ERR_INVALID_ARG;
  if (static_cast<double>(f->threshold) < static_cast<double>(Lq - 1)) return SDPA_ERR_UNSUPPORTED;
  a.w1 = f->w1;
  a.b1 = f->b1;
  a.w2 = f->w2;
  a.b2 = f->b2;
  a.c = f->c;
  a.thr = f->threshold;
  a.W = f->width;
  a.H = f->heads;
  a.Lq = static_cast<int>(Lq);
  a.Lk = static_cast<int>(Lk);
  return SDPA_OK;
}

struct FirePlan {
  size_t hid, dpre, x, dxc, dxt, total;
};

FirePlan fire_plan(int64_t R, int W) {
  FirePlan pl;
  pl.hid = 0;
  pl.dpre = round256(static_cast<size_t>(R) * W * sizeof(float));
  pl.x = pl.dpre + pl.dpre;
  pl.dxc = pl.x + round256(static_cast<size_t>(R) * sizeof(float));
  pl.dxt = pl.dxc + round256(static_cast<size_t>(R) * sizeof(float));
  pl.total = pl.dxt + round256(static_cast<size_t>(R) * sizeof(float));
  return pl;
}
}  // namespace

sdpa_status_t sdpa_fire_table(const sdpa_fire* fire, int64_t Lq, int64_t Lk, float* table,
                              void* stream) {
  FireArgs a;
  sdpa_status_t st = fire_check(fire, Lq, Lk, a);
  if (st != SDPA_OK) return st;
  if (!table || !aligned4(table)) return SDPA_ERR_INVALID_ARG;
  const int64_t n = (Lq + Lk - 1) * static_cast<int64_t>(a.H);
  fire_table_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0,
                      static_cast<cudaStream_t>(stream)>>>(a, table);
  return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

size_t sdpa_fire_backward_workspace_size(const sdpa_fire* fire, int64_t Lq, int64_t Lk) {
  FireArgs a;
  if (fire_check(fire, Lq, Lk, a) != SDPA_OK) return 0;
  return fire_plan(Lq + Lk - 1, a.W).total;
}

sdpa_status_t sdpa_fire_backward(const sdpa_fire* fire, int64_t Lq, int64_t Lk,
                                 const float* d_table, float* d_w1, float* d_b1, float* d_w2,
                                 float* d_b2, float* d_c_threshold, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  FireArgs a;
  sdpa_status_t st = fire_check(fire, Lq, Lk, a);
  if (st != SDPA_OK) return st;
  const void* ptrs[] = {d_table, d_w1, d_b1, d_w2, d_b2, d_c_threshold};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned4(ptr)) return SDPA_ERR_INVALID_ARG;
  const int64_t R = Lq + Lk - 1;
  const FirePlan pl = fire_plan(R, a.W);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < pl.total)
    return SDPA_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  FireWork ws;
  ws.hid = reinterpret_cast<float*>(w + pl.hid);
  ws.dpre = reinterpret_cast<float*>(w + pl.dpre);
  ws.x = reinterpret_cast<float*>(w + pl.x);
  ws.dxc = reinterpret_cast<float*>(w + pl.dxc);
  ws.dxt = reinterpret_cast<float*>(w + pl.dxt);
  FireOut out{d_w1, d_b1, d_w2, d_b2, d_c_threshold};
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  fire_rows_kernel<<<static_cast<unsigned>((R + 127) / 128), 128, 0, cs>>>(a, d_table, ws);
  if (cudaGetLastError() != cudaSuccess) return SDPA_ERR_CUDA;
  const int64_t n_out = static_cast<int64_t>(a.H) * a.W + a.H + 2 * a.W + 2;
  fire_reduce_kernel<<<static_cast<unsigned>(n_out), 256, 0, cs>>>(a, d_table, ws, out);
  return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

}  // extern "C"
