// fwd_kernel.cuh -- fused attention forward for sm_100a.
//
// One CTA owns NQ query tiles of 128 rows of one (batch, query head) and
// streams the key/value tiles of the mask band through shared memory:
//
//   producer warp   TMA: the NQ Q tiles once, then K_j and V_j into a ring of
//                   kStages stages (fully masked key tiles are never loaded --
//                   the point of HF transformers issue #30461: a mask handed
//                   over as a dense tensor forfeits this skipping).
//   MMA warp        one thread issues tcgen05.mma: S_t = Q_t K_j^T into tensor
//                   memory, then O_t += P_t V_j with P_t read from tensor memory.
//   softmax warps   one warpgroup per Q tile, one thread per query row (its
//                   TMEM lane): scale (log2e folded in), bias, mask at band
//                   edges, running max / sum, exp2, P_t back to tensor memory as
//                   bf16; O_t is rescaled in tensor memory only when the row
//                   max grows by more than 2^8 (exact: O and the sum always
//                   share the same reference max).  Epilogue: O = acc / sum ->
//                   bf16, LSE = (max + log2 sum) ln 2.
//
// Definition: codelab "jax-gpu-05-attention-gpu", sections 1 and 4 (score,
// scale, softmax, weighted sum); section 7 (causal masking); transformers
// issue #30461 (causal sliding window); catie-aq/flashT5 README (full and T5
// relative-position biases); codelab section 9 (KV heads shared by groups).
#pragma once

#include "attn_common.cuh"
#include "exp2_poly.cuh"
#include "sm100.cuh"
#include "tmem_sync.cuh"

namespace sdpa {

constexpr float kRescaleThreshold = 8.0f;
// Share of a full tile's exponentials on MUFU (per 8 columns; 8 = all): the
// forward measured fastest with every exponential on MUFU.
constexpr int kFwdMufuPer8 = 8;
// Full tiles without a bias take the lean path: the row max is taken on the
// raw scores (scale > 0 preserves the order), the scale folds into the one
// fused multiply-add that forms each exponent, and pairs of columns go
// through the packed fp32x2 FMA / add of sm_100.
constexpr bool kFwdLeanSoftmax = true;  // log2 units: rescale O when max grows > 2^8

template <int D, int NQ>
struct FwdLayout {
  static constexpr int kTileBytes = kTile * D * 2;  // one 128 x D bf16 tile
  static constexpr int kStages = (D == 128) ? 2 : 3;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + NQ * kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kLutOff = kVOff + kStages * kTileBytes;  // NQ x 2 x 256 floats
  static constexpr int kBarOff = kLutOff + NQ * 2 * 256 * 4;
  // q_full, k_full[S], k_empty[S], v_full[S], v_empty[S], s_full[NQ], p_full[NQ], o_done[NQ],
  // drain
  static constexpr int kNumBars = 2 + 4 * kStages + 3 * NQ;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static constexpr int kThreads = NQ * 128 + 64;
  static constexpr int kTmemCols = (NQ * (128 + D) <= 256) ? 256 : 512;
  static constexpr int kOCol = NQ * 128;            // O_t at kOCol + t * D, S_t at t * 128
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

// Bias term of one score row, in log2 units, for the 128 columns of a tile.
template <int BIAS>
__device__ __forceinline__ float bias_log2(const float* lut_row, const float* brow, int c) {
  if constexpr (BIAS == kBiasT5) return lut_row[c];
  if constexpr (BIAS == kBiasDense) return brow[c] * kLog2e;
  return 0.f;
}

template <int D, int NQ, int BIAS>
__global__ void __launch_bounds__(FwdLayout<D, NQ>::kThreads, 1)
    fwd_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmQ,
               const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
  using Lay = FwdLayout<D, NQ>;
  constexpr int S = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- tile coordinates: heaviest causal query blocks first
  const int rows_cta = kTile * NQ;
  const int nqb = (p.L + rows_cta - 1) / rows_cta;
  const int qb = p.causal ? (nqb - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
  const int hq = blockIdx.y;
  const int b = blockIdx.z;
  const int g = hq / p.G;
  const int m0 = qb * rows_cta;
  int nlo, nhi;
  key_tile_range(p, m0, rows_cta, nlo, nhi);
  int tlo[NQ], thi[NQ];  // key-tile range of each Q tile (a sub-range of [nlo, nhi))
#pragma unroll
  for (int t = 0; t < NQ; ++t) {
    if (m0 + t * kTile < p.L) {
      key_tile_range(p, m0 + t * kTile, kTile, tlo[t], thi[t]);
    } else {
      tlo[t] = nlo;
      thi[t] = nlo;  // entirely past L: nothing to compute
    }
  }
  const int nt = nhi - nlo;

  // ---- barriers
  auto bar = [&](int idx) -> uint32_t { return sb + Lay::kBarOff + 8 * idx; };
  const uint32_t q_full = bar(0);
  auto k_full = [&](int s) { return bar(1 + s); };
  auto k_empty = [&](int s) { return bar(1 + S + s); };
  auto v_full = [&](int s) { return bar(1 + 2 * S + s); };
  auto v_empty = [&](int s) { return bar(1 + 3 * S + s); };
  auto s_full = [&](int t) { return bar(1 + 4 * S + t); };
  auto p_full = [&](int t) { return bar(1 + 4 * S + NQ + t); };
  auto o_done = [&](int t) { return bar(1 + 4 * S + 2 * NQ + t); };
  const uint32_t drain = bar(1 + 4 * S + 3 * NQ);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), kTile);
      mbar_init(o_done(t), 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), Lay::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.wait_limit_ns};

  if (warp == 4 * NQ) {
    // =========================== producer (TMA) ===========================
    if (lane == 0 && nt > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(q_full, NQ * Lay::kTileBytes);
      for (int t = 0; t < NQ; ++t)
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(sb + Lay::kQOff + t * Lay::kTileBytes + h * 16384, &tmQ, q_full, h * 64,
                      m0 + t * kTile, hq, b);
      int issued_k[S], issued_v[S];
      for (int s = 0; s < S; ++s) issued_k[s] = issued_v[s] = -1;
      bool ok = true;
      for (int it = 0; it < nt && ok; ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const int n0 = (nlo + it) * kTile;
        if (!(ok = mbar_wait(k_empty(s), ph ^ 1, ctl))) break;
        mbar_expect_tx(k_full(s), Lay::kTileBytes);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(sb + Lay::kKOff + s * Lay::kTileBytes + h * 16384, &tmK, k_full(s), h * 64,
                      n0, g, b);
        issued_k[s] = ph;
        if (!(ok = mbar_wait(v_empty(s), ph ^ 1, ctl))) break;
        mbar_expect_tx(v_full(s), Lay::kTileBytes);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(sb + Lay::kVOff + s * Lay::kTileBytes + h * 16384, &tmV, v_full(s), h * 64,
                      n0, g, b);
        issued_v[s] = ph;
      }
      if (!ok) {
        // Aborted: let every copy already issued land before the CTA exits.
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mbar_wait(q_full, 0, ign);
        for (int s = 0; s < S; ++s) {
          if (issued_k[s] >= 0) mbar_wait(k_full(s), issued_k[s], ign);
          if (issued_v[s] >= 0) mbar_wait(v_full(s), issued_v[s], ign);
        }
      }
    }
  } else if (warp == 4 * NQ + 1) {
    // ============================ MMA issuer =============================
    if (lane == 0 && nt > 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTile, kTile, 0, 0);  // Q, K both K-major
      constexpr uint32_t kIdO = idesc_bf16_f32(kTile, D, 0, 1);      // V is N(=d)-major
      int cnt[NQ];
      for (int t = 0; t < NQ; ++t) cnt[t] = 0;
      bool ok = mbar_wait(q_full, 0, ctl);
      for (int it = 0; it < nt && ok; ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const int n = nlo + it;
        if (!(ok = mbar_wait(k_full(s), ph, ctl))) break;
        for (int t = 0; t < NQ && ok; ++t) {
          if (n < tlo[t] || n >= thi[t]) continue;
          // S_t's columns held P_t of the previous tile: wait until P_t V was done.
          if (cnt[t] > 0 && !(ok = mbar_wait(o_done(t), (cnt[t] - 1) & 1, ctl))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qa = sb + Lay::kQOff + t * Lay::kTileBytes + (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t ka = sb + Lay::kKOff + s * Lay::kTileBytes + (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_ss(tmem + t * kTile, smem_desc_sw128(qa, 16, 1024), smem_desc_sw128(ka, 16, 1024),
                   kIdS, kk > 0 ? 1u : 0u);
          }
          mma_commit(s_full(t));
        }
        if (!ok) break;
        mma_commit(k_empty(s));
        if (!(ok = mbar_wait(v_full(s), ph, ctl))) break;
        for (int t = 0; t < NQ && ok; ++t) {
          if (n < tlo[t] || n >= thi[t]) continue;
          if (!(ok = mbar_wait(p_full(t), cnt[t] & 1, ctl))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint32_t va = sb + Lay::kVOff + s * Lay::kTileBytes + kk * 2048;
            mma_ts(tmem + Lay::kOCol + t * D, tmem + t * kTile + kk * 8,
                   smem_desc_sw128(va, 16384, 1024), kIdO, (cnt[t] > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(o_done(t));
          ++cnt[t];
        }
        if (!ok) break;
        mma_commit(v_empty(s));
      }
      if (!ok) {
        // Aborted: wait until every MMA already issued has finished with
        // tensor memory before the CTA frees it.
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mma_commit(drain);
        mbar_wait(drain, 0, ign);
      }
    }
  } else {
    // ===================== softmax warpgroup t (rows) =====================
    const int t = warp >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int m0t = m0 + t * kTile;
    const int i = m0t + row;  // query row
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_bits + t * kTile;
    const uint32_t tO = tmem + lane_bits + Lay::kOCol + t * D;
    float* lut = reinterpret_cast<float*>(smem + Lay::kLutOff) + t * 512;
    const float* brow = nullptr;
    if constexpr (BIAS == kBiasDense) {
      // rows past L read row L-1 (in bounds); their outputs are never stored
      brow = p.bias + static_cast<int64_t>(b) * p.sb_b + static_cast<int64_t>(hq) * p.sb_h +
             static_cast<int64_t>(min(i, p.L - 1)) * p.sb_i;
    }
    float m_run = -INFINITY;  // running max, log2 units
    float l_run = 0.f;        // running sum relative to m_run
    // `ok` is kept warp-uniform; after an abort the loop still runs to the
    // end (every wait then returns at once) so that no thread of the
    // warpgroup is left waiting at a named barrier.
    bool ok = true;
    int cnt = 0;
    for (int n = tlo[t]; n < thi[t]; ++n, ++cnt) {
      const int n0 = n * kTile;
      const bool full = tile_is_full(p, m0t, n0, false);
      int lo = 0, hi = kTile - 1;
      if (!full) row_visible_cols(p, i, n0, lo, hi);
      const float* lut_row = nullptr;
      if constexpr (BIAS == kBiasT5) {
        // bias of every distance this tile spans: j - i = (n0 - m0t) + (c - row)
        float* lt = lut + (cnt & 1) * 256;
        const int base = n0 - m0t - (kTile - 1);
        lt[row] = p.t5_table[t5_bucket(base + row, p.t5) * p.Hq + hq] * kLog2e;
        if (row < kTile - 1)
          lt[row + kTile] = p.t5_table[t5_bucket(base + row + kTile, p.t5) * p.Hq + hq] * kLog2e;
        named_barrier(1 + t, kTile);
        lut_row = lt + (kTile - 1) - row;
      }
      if (ok) ok = mbar_wait(s_full(t), cnt & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
      // x: scores in log2 units, in place over the raw accumulator bits
      uint32_t x[128];
      tmem_ld128_sync(tS, x);
      float sum, alpha, m_use;
      bool grow;
      if (kFwdLeanSoftmax && BIAS == kBiasNone && full && p.scale_log2 > 0.f) {
        // ---- lean path: raw max (3-input), exponent = fma(s, c, -m)
        float ma = -INFINITY, mb = -INFINITY;
#pragma unroll
        for (int c = 0; c < kTile; c += 4) {
          ma = fmax3(ma, __uint_as_float(x[c]), __uint_as_float(x[c + 1]));
          mb = fmax3(mb, __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
        }
        const float tmax = fmaxf(ma, mb) * p.scale_log2;
        const float m_new = fmaxf(m_run, tmax);
        grow = m_new > m_run + kRescaleThreshold;
        m_use = grow ? m_new : m_run;
        alpha = grow ? fast_exp2(m_run - m_use) : 1.f;
        const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = f2_pack(-m_use, -m_use);  // m_use is finite in a full tile
        uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int c0 = 0; c0 < kTile; c0 += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const uint64_t arg = f2_fma(f2_pack(__uint_as_float(x[c0 + c]), __uint_as_float(x[c0 + c + 1])),
                                        c2, nm2);
            float v0, v1;
            f2_unpack(arg, v0, v1);
            const float e0 = emu_exp2<BIAS, kFwdMufuPer8>(c0 + c) ? exp2_fma(v0) : fast_exp2(v0);
            const float e1 = emu_exp2<BIAS, kFwdMufuPer8>(c0 + c + 1) ? exp2_fma(v1) : fast_exp2(v1);
            const uint64_t e2 = f2_pack(e0, e1);
            acc[(c >> 1) & 3] = f2_add(acc[(c >> 1) & 3], e2);
            pk[c >> 1] = pack_bf16x2(e0, e1);
          }
          tmem_st16(tS + (c0 >> 1), pk);  // P_t (bf16 pairs) over the first 64 columns of S_t
        }
        float s0, s1, s2, s3, s4, s5, s6, s7;
        f2_unpack(acc[0], s0, s1);
        f2_unpack(acc[1], s2, s3);
        f2_unpack(acc[2], s4, s5);
        f2_unpack(acc[3], s6, s7);
        sum = ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
      } else {
        // four independent max / sum chains instead of one 128 long
        float tm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        const float* bcol = brow ? brow + n0 : nullptr;
        if (full) {
  #pragma unroll
          for (int c = 0; c < kTile; ++c) {
            float v = __uint_as_float(x[c]) * p.scale_log2;
            if constexpr (BIAS != kBiasNone) v += bias_log2<BIAS>(lut_row, bcol, c);
            x[c] = __float_as_uint(v);
            tm[c & 3] = fmaxf(tm[c & 3], v);
          }
        } else {
  #pragma unroll
          for (int c = 0; c < kTile; ++c) {
            const bool vis = (c >= lo) && (c <= hi);
            float v = __uint_as_float(x[c]) * p.scale_log2;
            if constexpr (BIAS == kBiasT5) v += lut_row[c];
            if constexpr (BIAS == kBiasDense) v += vis ? bcol[c] * kLog2e : 0.f;
            v = vis ? v : -INFINITY;
            x[c] = __float_as_uint(v);
            tm[c & 3] = fmaxf(tm[c & 3], v);
          }
        }
        const float tmax = fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3]));
        const float m_new = fmaxf(m_run, tmax);
        const bool grow_g = m_new > m_run + kRescaleThreshold;
        const float m_use_g = grow_g ? m_new : m_run;
        const float alpha_g = grow_g ? fast_exp2(m_run - m_use_g) : 1.f;
        const float m_sub = (m_use_g == -INFINITY) ? 0.f : m_use_g;
        float sm[4] = {0.f, 0.f, 0.f, 0.f};
        if (full) {
          // every entry is finite: a fixed share of the exponentials on the FMA pipe
  #pragma unroll
          for (int c0 = 0; c0 < kTile; c0 += 32) {
            uint32_t pk[16];
  #pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float v0 = __uint_as_float(x[c0 + c]) - m_sub;
              const float v1 = __uint_as_float(x[c0 + c + 1]) - m_sub;
              const float e0 = emu_exp2<BIAS, kFwdMufuPer8>(c0 + c) ? exp2_fma(v0) : fast_exp2(v0);
              const float e1 = emu_exp2<BIAS, kFwdMufuPer8>(c0 + c + 1) ? exp2_fma(v1) : fast_exp2(v1);
              sm[(c >> 1) & 3] += e0 + e1;
              pk[c >> 1] = pack_bf16x2(e0, e1);
            }
            tmem_st16(tS + (c0 >> 1), pk);  // P_t (bf16 pairs) over the first 64 columns of S_t
          }
        } else {
  #pragma unroll
          for (int c0 = 0; c0 < kTile; c0 += 32) {
            uint32_t pk[16];
  #pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float e0 = fast_exp2(__uint_as_float(x[c0 + c]) - m_sub);
              const float e1 = fast_exp2(__uint_as_float(x[c0 + c + 1]) - m_sub);
              sm[(c >> 1) & 3] += e0 + e1;
              pk[c >> 1] = pack_bf16x2(e0, e1);
            }
            tmem_st16(tS + (c0 >> 1), pk);
          }
        }
        sum = (sm[0] + sm[1]) + (sm[2] + sm[3]);
        grow = grow_g;
        alpha = alpha_g;
        m_use = m_use_g;
      }
      l_run = l_run * alpha + sum;
      m_run = m_use;
      tmem_st_wait();
      if (cnt > 0 && __any_sync(0xffffffffu, grow)) {
        // O_t holds earlier tiles: rescale it once P_t V of the previous tile landed.
        ok = mbar_wait(o_done(t), (cnt - 1) & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) continue;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t r[32];
          tmem_ld32_sync(tO + c, r);
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32_sync(tO + c, r);
        }
      }
      tc_fence_before();
      mbar_arrive(p_full(t));
    }
    // ------------------------------ epilogue ------------------------------
    if (ok && cnt > 0) ok = mbar_wait(o_done(t), (cnt - 1) & 1, ctl);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      __nv_bfloat16* orow = p.o + static_cast<int64_t>(b) * p.sq_b +
                            static_cast<int64_t>(i) * p.sq_l + static_cast<int64_t>(hq) * p.sq_h;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        if (cnt > 0) {
          tmem_ld32_sync(tO + c, r);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv, __uint_as_float(r[2 * e + 1]) * inv);
        if (i < p.L) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (i < p.L) {
        p.lse[(static_cast<int64_t>(b) * p.Hq + hq) * p.L + i] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      }
    }
  }

  // ------------------------------- teardown -------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

}  // namespace sdpa
