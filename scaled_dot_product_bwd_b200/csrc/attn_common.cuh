// attn_common.cuh -- kernel parameters, mask-band arithmetic and the T5
// relative-position bucket function shared by the forward and backward
// kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "exp2_poly.cuh"
#include "sm100.cuh"

namespace sdpa {

constexpr int kTile = 128;             // query rows and keys per tile
constexpr int kBlk = 64;               // columns per compute warpgroup in a tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxT5Thresholds = 64;

enum BiasKind : int { kBiasNone = 0, kBiasDense = 1, kBiasT5 = 2 };

// T5 bucketing with the log boundaries precomputed on the host (in float64,
// the precision the closed form is evaluated in) as integer thresholds:
// distance n >= max_exact falls in bucket max_exact - 1 + #{k : n >= thr[k]},
// capped at half - 1.  `half` is num_buckets / 2 when bidirectional (then
// keys after the query, rel > 0, are offset by `half`), else num_buckets.
struct T5Spec {
  int half;
  int max_exact;
  int nthr;
  int bidirectional;
  int thr[kMaxT5Thresholds];
  // Every rel <= one_lo_max lies in the capped bucket of keys before the
  // query, every rel >= one_hi_min in one bucket too (the capped bucket of
  // keys after it, or bucket 0 of a unidirectional table); INT_MIN /
  // INT_MAX when no distance in range is capped.
  int one_lo_max, one_hi_min;
  // the closed form in float32 for the device's first guess:
  // (half - max_exact) / log2(max_distance / max_exact) and 1 / max_exact
  float log_scale, inv_max_exact;
};

// The contiguous range [lo, hi] of distances r = j - i (within the
// sequences) that falls in each T5 bucket; hi < lo: bucket unused.
struct T5Ranges {
  int lo[128];
  int hi[128];
};

__host__ __device__ __forceinline__ int t5_bucket(int rel, const T5Spec& s) {
  int n, off = 0;
  if (s.bidirectional) {
    n = rel < 0 ? -rel : rel;
    off = rel > 0 ? s.half : 0;
  } else {
    n = rel < 0 ? -rel : 0;
  }
  int b;
  if (n < s.max_exact) {
    b = n;
  } else {
#ifdef __CUDA_ARCH__
    // The closed form max_exact + trunc(log2(n / max_exact) * log_scale) in
    // float32 is within one of its float64 value; the integer thresholds
    // then decide exactly: thr[k] <= n < thr[k + 1] is bucket max_exact + k,
    // n >= thr[nthr - 1] the capped one.  (A loop over the thresholds reads
    // them one after another and cost ~400 cycles per distance.)
    const int K = s.nthr;
    if (n >= s.thr[K - 1]) {
      b = s.half - 1;
    } else {
      int k = static_cast<int>(__log2f(static_cast<float>(n) * s.inv_max_exact) * s.log_scale);
      k = min(max(k, 0), K - 1);
      if (k + 1 < K && n >= s.thr[k + 1]) ++k;
      if (n < s.thr[k]) --k;
      b = s.max_exact + k;
    }
#else
    b = s.max_exact - 1;
    for (int k = 0; k < s.nthr; ++k) b += (n >= s.thr[k]) ? 1 : 0;
    b = b < s.half - 1 ? b : s.half - 1;
#endif
  }
  return b + off;
}

struct AttnParams {
  // Batch entries, query / key sequence lengths (the longest, for packed
  // sequences), heads (G = Hq / Hkv query heads per KV head).
  int B, Lq, Lk, Hq, Hkv, G;
  int causal, wl, wr;          // wl / wr < 0: unbounded
  float scale;                 // softmax scale
  float scale_log2;            // scale * log2(e)
  int64_t sq_b, sq_l, sq_h;    // element strides: Q, O, dO, dQ
  int64_t skv_b, skv_l, skv_h; // element strides: K, V, dK, dV
  // Packed variable-length sequences: batch entry b holds query rows
  // [cu_q[b], cu_q[b + 1]) and key rows [cu_k[b], cu_k[b + 1]) of one
  // sequence axis (sq_b = skv_b = 0).  nullptr: every entry has Lq / Lk rows.
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;        // rows of the packed sequence axes (cu_q != nullptr)
  // element strides of the per-row float arrays LSE and D: entry (b, h, row)
  // is at b * lse_sb + h * lse_sh + row, row counted along the (packed) query
  // sequence axis
  int64_t lse_sb, lse_sh;
  // forward outputs / backward inputs
  __nv_bfloat16* o;
  float* lse;
  // backward
  const __nv_bfloat16* dout;
  float* dvec;                 // D = rowsum(dO * O), laid out as LSE
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  // optional fp32 dS (the gradient of the logits, = of an additive bias),
  // element strides sd_b, sd_h, sd_i (multiples of 4), j contiguous
  float* ds_out;
  int64_t sd_b, sd_h, sd_i;
  // optional per-warp sums of dS along the diagonals j - i, per T5 bucket
  // or weighted by |j - i| (relative-position bias gradients); layouts in
  // bwd_dq_kernel's diagonal, bucket and moment modes
  float* diag_out;
  // bias
  int bias_kind;
  const float* bias;           // dense
  int64_t sb_b, sb_h, sb_i;
  const float* t5_table;       // [num_buckets, Hq]
  T5Spec t5;
  T5Ranges t5r;                // the T5 table gradient only
  // ALiBi runs in the kBiasT5 kernels: both biases are functions of j - i
  // that the kernels tabulate per tile
  int alibi;                   // 1: bias = -alibi_slopes[h] |j - i| instead of T5
  const float* alibi_slopes;   // [Hq]
  // a relative-position table instead of T5 (when not null): bias =
  // rel_table[(j - i + rel_off) * Hq + h], rows 0 .. rel_rows - 1
  const float* rel_table;
  int rel_off, rel_rows;
  uint64_t wait_limit_ns;
};

// One batch entry's sequences: row offsets along the (packed) sequence axes,
// lengths, and the batch coordinate of the tensor maps (0 when packed).
struct SeqView {
  int q0, k0, Lq, Lk, bc;
};

// Offsets that are not non-decreasing, leave the packed axis, or give a
// sequence longer than the stated maximum record kStatusBadSeqlens and make
// the entry empty, so no kernel addresses memory outside its tensors.
__device__ __forceinline__ SeqView seq_view(const AttnParams& p, int b) {
  SeqView s;
  if (p.cu_q != nullptr) {
    s.q0 = p.cu_q[b];
    s.Lq = p.cu_q[b + 1] - s.q0;
    s.k0 = p.cu_k[b];
    s.Lk = p.cu_k[b + 1] - s.k0;
    s.bc = 0;
    const bool bad = s.q0 < 0 || s.Lq < 0 || s.Lq > p.Lq || s.q0 > p.total_q - s.Lq ||
                     s.k0 < 0 || s.Lk < 0 || s.Lk > p.Lk || s.k0 > p.total_k - s.Lk;
    if (bad) {
      atomicOr(&g_device_status, kStatusBadSeqlens);
      s.q0 = s.k0 = s.Lq = s.Lk = 0;
    }
  } else {
    s.q0 = 0;
    s.k0 = 0;
    s.Lq = p.Lq;
    s.Lk = p.Lk;
    s.bc = b;
  }
  return s;
}

// Index of (b, h, query row i of b's sequence) in LSE and D.
__device__ __forceinline__ int64_t row_index(const AttnParams& p, const SeqView& s, int b, int h,
                                             int i) {
  return static_cast<int64_t>(b) * p.lse_sb + static_cast<int64_t>(h) * p.lse_sh + s.q0 + i;
}

// Relative-position bias of distance rel = j - i for query head hq, in log2
// units (times log2 e), as the kBiasT5 kernels tabulate it per tile: the
// T5 table entry of rel's bucket (catie-aq/flashT5 README, "T5-like relative
// position encoding biases"), ALiBi's -m_h |rel| (Press et al. 2022; named
// by the same README among the supported positional schemes), or a
// caller's table entry for rel (the general form; FIRE's table).
__device__ __forceinline__ float rel_bias_log2(const AttnParams& p, int rel, int hq) {
  if (p.rel_table) {
    // tables cover the in-range distances; the tile-wide lookup rows also
    // span positions past the sequences, which the mask hides: clamp those
    const int r = min(max(rel + p.rel_off, 0), p.rel_rows - 1);
    return p.rel_table[static_cast<int64_t>(r) * p.Hq + hq] * kLog2e;
  }
  if (p.alibi) return -(p.alibi_slopes[hq] * kLog2e) * fabsf(static_cast<float>(rel));
  return p.t5_table[t5_bucket(rel, p.t5) * p.Hq + hq] * kLog2e;
}

// Whether column c of a fully visible tile takes the FMA-pipe exponential:
// never with a dense bias, whose entries may be -inf (masked) even inside a
// visible tile and must give exactly 0; otherwise columns c (mod 8) >=
// MUFU_PER8 do -- a fixed split per kernel, so results stay bit-reproducible.
// MUFU_PER8 = 8 keeps every exponential on the MUFU unit.
template <int BIAS, int MUFU_PER8>
__device__ __forceinline__ constexpr bool emu_exp2(int c) {
  return BIAS != kBiasDense && (c & 7) >= MUFU_PER8;
}

// Compile-time flag for loops written once in two forms (a generic lambda
// called with Flag<true>{} or Flag<false>{}).
template <bool B>
struct Flag {
  static constexpr bool value = B;
};

// T5 table bias of a piece of a tile whose distances j - i are base ..
// base + span: true, with the bias in log2 units in `bias`, when they all
// lie in one capped bucket (or at j >= i of a unidirectional table), so the
// bias is one constant over the piece.
__device__ __forceinline__ bool t5_one_bucket(const AttnParams& p, int base, int span, int hq,
                                              float& bias) {
  if (p.rel_table != nullptr || p.alibi) return false;
  if (base + span > p.t5.one_lo_max && base < p.t5.one_hi_min) return false;
  bias = rel_bias_log2(p, base, hq);
  return true;
}

// 2^x of columns c and c + 1, each on the unit emu_exp2 gives it; a pair
// that both go to the FMA pipe takes the packed form (identical results).
template <int BIAS, int MUFU_PER8>
__device__ __forceinline__ void exp2_pair(int c, float x0, float x1, float& y0, float& y1) {
  const bool f0 = emu_exp2<BIAS, MUFU_PER8>(c), f1 = emu_exp2<BIAS, MUFU_PER8>(c + 1);
  if (f0 && f1) {
    exp2_fma2(x0, x1, y0, y1);
  } else {
    y0 = f0 ? exp2_fma(x0) : fast_exp2(x0);
    y1 = f1 ? exp2_fma(x1) : fast_exp2(x1);
  }
}

// Key tiles [nlo, nhi) that hold any key visible from query rows
// [m0, m0 + rows) (clipped to Lq), keys clipped to Lk.  Empty when nhi <= nlo.
// Positions of both sequences count from 0.
__device__ __forceinline__ void key_tile_range(const AttnParams& p, int Lq, int Lk, int m0,
                                               int rows, int& nlo, int& nhi) {
  const int m_last = min(m0 + rows - 1, Lq - 1);
  int jmin = 0;
  if (p.wl >= 0) jmin = max(0, m0 - p.wl);
  int jmax = Lk - 1;
  if (p.causal) jmax = min(jmax, m_last);
  if (p.wr >= 0) jmax = min(jmax, m_last + p.wr);
  nlo = jmin / kTile;
  nhi = (jmax >= jmin && m_last >= m0) ? jmax / kTile + 1 : nlo;
}

// Query tiles [mlo, mhi) holding any query (< Lq) that sees a key in
// [n0, n0 + kTile) (clipped to Lk).
__device__ __forceinline__ void query_tile_range(const AttnParams& p, int Lq, int Lk, int n0,
                                                 int& mlo, int& mhi) {
  const int n_last = min(n0 + kTile - 1, Lk - 1);
  int imin = 0;
  if (p.causal) imin = n0;
  if (p.wr >= 0) imin = max(imin, n0 - p.wr);
  int imax = Lq - 1;
  if (p.wl >= 0) imax = min(imax, n_last + p.wl);
  mlo = imin / kTile;
  mhi = (imax >= imin && n_last >= n0) ? imax / kTile + 1 : mlo;
}

// L2 prefetch of the dense-bias rows [m0, m0 + 128) x keys [n0, n0 + 128) of
// one (batch, query head), clipped to Lq x Lk (rounded up to 16 bytes, which
// stays inside the row: row strides are multiples of 4 floats).  One thread
// issues.
__device__ __forceinline__ void prefetch_bias_tile(const AttnParams& p, int b, int hq, int m0,
                                                   int n0) {
  const int cols = min(kTile, p.Lk - n0);
  if (cols <= 0) return;
  const uint32_t bytes = static_cast<uint32_t>((cols + 3) & ~3) * 4u;
  const float* base = p.bias + static_cast<int64_t>(b) * p.sb_b + static_cast<int64_t>(hq) * p.sb_h + n0;
  const int rows = min(kTile, p.Lq - m0);
  for (int r = 0; r < rows; ++r) prefetch_l2(base + static_cast<int64_t>(m0 + r) * p.sb_i, bytes);
}

// Byte offset of the 16-element K step kk inside a K-major SW128 tile of
// `rows` rows: a d = 128 tile is two 64-column halves of rows x 128 bytes.
__device__ __forceinline__ uint32_t kmajor_koff(int kk, int rows) {
  return static_cast<uint32_t>((kk >> 2) * rows * 128 + (kk & 3) * 32);
}

// TMEM column of the bf16 A operand for the 16-row K step kk of a 128-wide
// block whose two 64-wide halves were written by the two warpgroups into the
// first 32 columns of their own 64-column regions starting at `base`.
__device__ __forceinline__ uint32_t split_a_col(uint32_t base, int kk) {
  return base + (kk < 4 ? kk * 8 : 64 + (kk - 4) * 8);
}

// Streaming multiprocessors of the current device (persistent grids), cached
// per device.
inline int sm_count() {
  constexpr int kDevs = 64;
  static int cached[kDevs] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kDevs && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kDevs) cached[dev] = n;
  return n;
}

}  // namespace sdpa
