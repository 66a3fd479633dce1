// bwd_kernels.cuh -- fused attention backward for sm_100a.
//
// The pages print no gradient formulas; these kernels apply the chain rule
// to the forward (codelab "jax-gpu-05-attention-gpu", sections 1 and 4):
//   P = exp(S - LSE)  (S recomputed with the forward's mask and bias)
//   dV = P^T dO,  dP = dO V^T,  D_i = rowsum(dO_i * O_i),  dS = P (dP - D)
//   dK = scale dS^T Q,  dQ = scale dS K
// Three launches, each reducing in a fixed order with no atomics, so the
// result is bit-identical run to run (HF transformers issue #31787,
// "Transformer models are not deterministic when using Flash Attention 2"):
//   1. preprocess: D = rowsum(dO * O) into the workspace.
//   2. dK/dV: one CTA per (key tile, KV head, batch); it walks the query
//      tiles of the band for every query head of the group in a fixed order
//      and accumulates dK, dV in tensor memory (S^T = K Q^T, dP^T = V dO^T,
//      dV += P^T dO, dK += dS^T Q; P^T and dS^T go back to tensor memory as
//      bf16 and feed the last two MMAs directly).
//   3. dQ: one CTA per (query tile, query head, batch); it walks the key
//      tiles of the band in order (S = Q K^T, dP = dO V^T, dQ += dS K).
#pragma once

#include "attn_common.cuh"
#include "sm100.cuh"
#include "tmem_sync.cuh"

namespace sdpa {

struct BwdMaps {
  CUtensorMap q, k, v, dout;
};

// ------------------------------------------------------------ preprocess
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const AttnParams p) {
  constexpr int kTpr = D / 8;  // threads per row, 8 bf16 (16 bytes) each
  const int64_t nrows = static_cast<int64_t>(p.B) * p.L * p.Hq;
  const int64_t gt = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t r = gt / kTpr;
  const int part = static_cast<int>(gt % kTpr);
  float acc = 0.f;
  int h = 0, i = 0, b = 0;
  if (r < nrows) {
    h = static_cast<int>(r % p.Hq);
    i = static_cast<int>((r / p.Hq) % p.L);
    b = static_cast<int>(r / (static_cast<int64_t>(p.Hq) * p.L));
    const int64_t off = b * p.sq_b + i * p.sq_l + h * p.sq_h + part * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(p.o + off);
    const uint4 c = *reinterpret_cast<const uint4*>(p.dout + off);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(a2[e]);
      const float2 y = __bfloat1622float2(c2[e]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (part == 0 && r < nrows) p.dvec[(static_cast<int64_t>(b) * p.Hq + h) * p.L + i] = acc;
}

// ------------------------------------------------------------------ dK / dV
template <int D>
struct DkdvLayout {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kStages = 2;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kQOff = 2 * kTileBytes;
  static constexpr int kDOOff = kQOff + kStages * kTileBytes;
  static constexpr int kVecOff = kDOOff + kStages * kTileBytes;  // 2 x (lse2[128], D[128])
  static constexpr int kLutOff = kVecOff + 2 * 256 * 4;          // 2 x 256 floats
  static constexpr int kBarOff = kLutOff + 2 * 256 * 4;
  // kv_full, q_full[S], q_empty[S], s_full, dp_full, p_full, ds_full, o_done, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 6;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static constexpr int kThreads = 192;
  static constexpr int kTmemCols = 512;
  static constexpr int kSCol = 0, kDPCol = 128, kDVCol = 256, kDKCol = 256 + D;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

template <int D, int BIAS>
__global__ void __launch_bounds__(192, 1)
    bwd_dkdv_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmDO) {
  using Lay = DkdvLayout<D>;
  constexpr int S = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int nkt = (p.L + kTile - 1) / kTile;
  // causal: the first key tiles see the most query tiles; run them first
  const int ntile = static_cast<int>(blockIdx.x);
  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int n0 = ntile * kTile;
  (void)nkt;
  int mlo, mhi;
  query_tile_range(p, n0, mlo, mhi);
  const int nm = mhi > mlo ? mhi - mlo : 0;
  const int total = nm * p.G;  // iterations: query head (outer) x query tile (inner)

  auto bar = [&](int idx) -> uint32_t { return sb + Lay::kBarOff + 8 * idx; };
  const uint32_t kv_full = bar(0);
  auto q_full = [&](int s) { return bar(1 + s); };
  auto q_empty = [&](int s) { return bar(1 + S + s); };
  const uint32_t s_full = bar(1 + 2 * S);
  const uint32_t dp_full = bar(2 + 2 * S);
  const uint32_t p_full = bar(3 + 2 * S);
  const uint32_t ds_full = bar(4 + 2 * S);
  const uint32_t o_done = bar(5 + 2 * S);
  const uint32_t drain = bar(6 + 2 * S);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, kTile);
    mbar_init(ds_full, kTile);
    mbar_init(o_done, 1);
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

  if (warp == 4) {
    // =========================== producer (TMA) ===========================
    if (lane == 0 && total > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_expect_tx(kv_full, 2 * Lay::kTileBytes);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_4d(sb + Lay::kKOff + h * 16384, &tmK, kv_full, h * 64, n0, g, b);
        tma_load_4d(sb + Lay::kVOff + h * 16384, &tmV, kv_full, h * 64, n0, g, b);
      }
      int issued[S];
      for (int s = 0; s < S; ++s) issued[s] = -1;
      bool ok = true;
      for (int it = 0; it < total; ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const int hq = g * p.G + it / nm;
        const int m0 = (mlo + it % nm) * kTile;
        if (!(ok = mbar_wait(q_empty(s), ph ^ 1, ctl))) break;
        mbar_expect_tx(q_full(s), 2 * Lay::kTileBytes);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_4d(sb + Lay::kQOff + s * Lay::kTileBytes + h * 16384, &tmQ, q_full(s), h * 64,
                      m0, hq, b);
          tma_load_4d(sb + Lay::kDOOff + s * Lay::kTileBytes + h * 16384, &tmDO, q_full(s),
                      h * 64, m0, hq, b);
        }
        issued[s] = ph;
      }
      if (!ok) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mbar_wait(kv_full, 0, ign);
        for (int s = 0; s < S; ++s)
          if (issued[s] >= 0) mbar_wait(q_full(s), issued[s], ign);
      }
    }
  } else if (warp == 5) {
    // ============================ MMA issuer =============================
    if (lane == 0 && total > 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTile, kTile, 0, 0);
      constexpr uint32_t kIdO = idesc_bf16_f32(kTile, D, 0, 1);
      bool ok = mbar_wait(kv_full, 0, ctl);
      for (int it = 0; it < total && ok; ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const uint32_t qs = sb + Lay::kQOff + s * Lay::kTileBytes;
        const uint32_t dos = sb + Lay::kDOOff + s * Lay::kTileBytes;
        if (!(ok = mbar_wait(q_full(s), ph, ctl))) break;
        // S^T and dP^T columns held P^T / dS^T of the previous tile.
        if (it > 0 && !(ok = mbar_wait(o_done, (it - 1) & 1, ctl))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + Lay::kSCol, smem_desc_sw128(sb + Lay::kKOff + ko, 16, 1024),
                 smem_desc_sw128(qs + ko, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + Lay::kDPCol, smem_desc_sw128(sb + Lay::kVOff + ko, 16, 1024),
                 smem_desc_sw128(dos + ko, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
        }
        mma_commit(dp_full);
        if (!(ok = mbar_wait(p_full, it & 1, ctl))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts(tmem + Lay::kDVCol, tmem + Lay::kSCol + kk * 8,
                 smem_desc_sw128(dos + kk * 2048, 16384, 1024), kIdO, (it > 0 || kk > 0) ? 1u : 0u);
        if (!(ok = mbar_wait(ds_full, it & 1, ctl))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts(tmem + Lay::kDKCol, tmem + Lay::kDPCol + kk * 8,
                 smem_desc_sw128(qs + kk * 2048, 16384, 1024), kIdO, (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(o_done);
        mma_commit(q_empty(s));
      }
      if (!ok) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mma_commit(drain);
        mbar_wait(drain, 0, ign);
      }
    }
  } else {
    // ================ compute warpgroup: one thread per key ================
    const int row = warp * 32 + lane;
    const int j = n0 + row;
    const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_bits + Lay::kSCol;
    const uint32_t tDP = tmem + lane_bits + Lay::kDPCol;
    float* vec = reinterpret_cast<float*>(smem + Lay::kVecOff);
    float* lut = reinterpret_cast<float*>(smem + Lay::kLutOff);
    auto load_vec = [&](int it, float& l2, float& dd) {
      l2 = INFINITY;
      dd = 0.f;
      if (it < total) {
        const int hq = g * p.G + it / nm;
        const int i = (mlo + it % nm) * kTile + row;
        if (i < p.L) {
          const int64_t idx = (static_cast<int64_t>(b) * p.Hq + hq) * p.L + i;
          l2 = p.lse[idx] * kLog2e;
          dd = p.dvec[idx];
          if (l2 == -INFINITY) l2 = INFINITY;  // row with no visible key: P = 0
        }
      }
    };
    float pf_l2, pf_d;
    load_vec(0, pf_l2, pf_d);
    bool ok = true;
    for (int it = 0; it < total; ++it) {
      const int hq = g * p.G + it / nm;
      const int m0 = (mlo + it % nm) * kTile;
      float* lse2 = vec + (it & 1) * 256;
      float* dvv = lse2 + 128;
      lse2[row] = pf_l2;
      dvv[row] = pf_d;
      const float* lut_row = nullptr;
      if constexpr (BIAS == kBiasT5) {
        // j - i = (n0 - m0) + (row - c): entry r = row - c + 127
        float* lt = lut + (it & 1) * 256;
        const int base = n0 - m0 - (kTile - 1);
        lt[row] = p.t5_table[t5_bucket(base + row, p.t5) * p.Hq + hq] * kLog2e;
        if (row < kTile - 1)
          lt[row + kTile] = p.t5_table[t5_bucket(base + row + kTile, p.t5) * p.Hq + hq] * kLog2e;
        lut_row = lt + row + (kTile - 1);
      }
      named_barrier(1, kTile);
      load_vec(it + 1, pf_l2, pf_d);
      const bool full = tile_is_full(p, m0, n0, true);
      int lo = 0, hi = kTile - 1;
      if (!full) key_visible_rows(p, j, m0, lo, hi);
      const float* bcol = nullptr;
      if constexpr (BIAS == kBiasDense) {
        bcol = p.bias + static_cast<int64_t>(b) * p.sb_b + static_cast<int64_t>(hq) * p.sb_h +
               static_cast<int64_t>(m0) * p.sb_i + min(j, p.L - 1);
      }
      if (ok) ok = mbar_wait(s_full, it & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
      uint32_t pr[128];  // S^T row, then P^T (fp32 bits) in place
      tmem_ld128_sync(tS, pr);
#pragma unroll
      for (int c = 0; c < kTile; ++c) {
        float x = __uint_as_float(pr[c]) * p.scale_log2 - lse2[c];
        const bool vis = full || (c >= lo && c <= hi);
        if constexpr (BIAS == kBiasT5) x += lut_row[-c];
        if constexpr (BIAS == kBiasDense) x += vis ? bcol[static_cast<int64_t>(c) * p.sb_i] * kLog2e : 0.f;
        pr[c] = __float_as_uint(vis ? fast_exp2(x) : 0.f);
      }
#pragma unroll
      for (int c0 = 0; c0 < kTile; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2)
          pk[c >> 1] = pack_bf16x2(__uint_as_float(pr[c0 + c]), __uint_as_float(pr[c0 + c + 1]));
        tmem_st16(tS + (c0 >> 1), pk);  // P^T over the first 64 columns of S^T
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
      if (ok) ok = mbar_wait(dp_full, it & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < kTile; c0 += 32) {
        uint32_t dr[32];
        tmem_ld32_sync(tDP + c0, dr);
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float d0 = __uint_as_float(pr[c0 + c]) * (__uint_as_float(dr[c]) - dvv[c0 + c]);
          const float d1 =
              __uint_as_float(pr[c0 + c + 1]) * (__uint_as_float(dr[c + 1]) - dvv[c0 + c + 1]);
          pk[c >> 1] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tDP + (c0 >> 1), pk);  // dS^T over the first 64 columns of dP^T
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    // ------------------------------ epilogue ------------------------------
    if (ok && total > 0) ok = mbar_wait(o_done, (total - 1) & 1, ctl);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const int64_t off = static_cast<int64_t>(b) * p.skv_b + static_cast<int64_t>(j) * p.skv_l +
                          static_cast<int64_t>(g) * p.skv_h;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* dst = (which == 0 ? p.dv : p.dk) + off;
        const float mul = which == 0 ? 1.f : p.scale;
        const uint32_t tcol = tmem + lane_bits + (which == 0 ? Lay::kDVCol : Lay::kDKCol);
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t r[32];
          if (total > 0) {
            tmem_ld32_sync(tcol + c, r);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
          if (j < p.L) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

// --------------------------------------------------------------------- dQ
template <int D>
struct DqLayout {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kStages = 2;
  static constexpr int kQOff = 0;
  static constexpr int kDOOff = kTileBytes;
  static constexpr int kKOff = 2 * kTileBytes;                  // stages of K
  static constexpr int kVOff = kKOff + kStages * kTileBytes;    // stages of V
  static constexpr int kLutOff = kVOff + kStages * kTileBytes;  // 2 x 256 floats
  static constexpr int kBarOff = kLutOff + 2 * 256 * 4;
  // q_full, kv_full[S], kv_empty[S], s_full, dp_full, ds_full, o_done, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 5;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static constexpr int kThreads = 192;
  static constexpr int kTmemCols = 512;
  static constexpr int kSCol = 0, kDPCol = 128, kDQCol = 256;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

template <int D, int BIAS>
__global__ void __launch_bounds__(192, 1)
    bwd_dq_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmDO) {
  using Lay = DqLayout<D>;
  constexpr int S = Lay::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int nqt = (p.L + kTile - 1) / kTile;
  const int qt = p.causal ? (nqt - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x);
  const int hq = blockIdx.y;
  const int b = blockIdx.z;
  const int g = hq / p.G;
  const int m0 = qt * kTile;
  int nlo, nhi;
  key_tile_range(p, m0, kTile, nlo, nhi);
  const int nt = nhi > nlo ? nhi - nlo : 0;

  auto bar = [&](int idx) -> uint32_t { return sb + Lay::kBarOff + 8 * idx; };
  const uint32_t q_full = bar(0);
  auto kv_full = [&](int s) { return bar(1 + s); };
  auto kv_empty = [&](int s) { return bar(1 + S + s); };
  const uint32_t s_full = bar(1 + 2 * S);
  const uint32_t dp_full = bar(2 + 2 * S);
  const uint32_t ds_full = bar(3 + 2 * S);
  const uint32_t o_done = bar(4 + 2 * S);
  const uint32_t drain = bar(5 + 2 * S);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, kTile);
    mbar_init(o_done, 1);
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

  if (warp == 4) {
    if (lane == 0 && nt > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_expect_tx(q_full, 2 * Lay::kTileBytes);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_4d(sb + Lay::kQOff + h * 16384, &tmQ, q_full, h * 64, m0, hq, b);
        tma_load_4d(sb + Lay::kDOOff + h * 16384, &tmDO, q_full, h * 64, m0, hq, b);
      }
      int issued[S];
      for (int s = 0; s < S; ++s) issued[s] = -1;
      bool ok = true;
      for (int it = 0; it < nt; ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const int n0 = (nlo + it) * kTile;
        if (!(ok = mbar_wait(kv_empty(s), ph ^ 1, ctl))) break;
        mbar_expect_tx(kv_full(s), 2 * Lay::kTileBytes);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_4d(sb + Lay::kKOff + s * Lay::kTileBytes + h * 16384, &tmK, kv_full(s), h * 64,
                      n0, g, b);
          tma_load_4d(sb + Lay::kVOff + s * Lay::kTileBytes + h * 16384, &tmV, kv_full(s), h * 64,
                      n0, g, b);
        }
        issued[s] = ph;
      }
      if (!ok) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mbar_wait(q_full, 0, ign);
        for (int s = 0; s < S; ++s)
          if (issued[s] >= 0) mbar_wait(kv_full(s), issued[s], ign);
      }
    }
  } else if (warp == 5) {
    if (lane == 0 && nt > 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTile, kTile, 0, 0);
      constexpr uint32_t kIdO = idesc_bf16_f32(kTile, D, 0, 1);
      bool ok = mbar_wait(q_full, 0, ctl);
      for (int it = 0; it < nt && ok; ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const uint32_t ks = sb + Lay::kKOff + s * Lay::kTileBytes;
        const uint32_t vs = sb + Lay::kVOff + s * Lay::kTileBytes;
        if (!(ok = mbar_wait(kv_full(s), ph, ctl))) break;
        if (it > 0 && !(ok = mbar_wait(o_done, (it - 1) & 1, ctl))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + Lay::kSCol, smem_desc_sw128(sb + Lay::kQOff + ko, 16, 1024),
                 smem_desc_sw128(ks + ko, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + Lay::kDPCol, smem_desc_sw128(sb + Lay::kDOOff + ko, 16, 1024),
                 smem_desc_sw128(vs + ko, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
        }
        mma_commit(dp_full);
        if (!(ok = mbar_wait(ds_full, it & 1, ctl))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts(tmem + Lay::kDQCol, tmem + Lay::kSCol + kk * 8,
                 smem_desc_sw128(ks + kk * 2048, 16384, 1024), kIdO, (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(o_done);
        mma_commit(kv_empty(s));
      }
      if (!ok) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mma_commit(drain);
        mbar_wait(drain, 0, ign);
      }
    }
  } else {
    // =============== compute warpgroup: one thread per query row ===============
    const int row = warp * 32 + lane;
    const int i = m0 + row;
    const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_bits + Lay::kSCol;
    const uint32_t tDP = tmem + lane_bits + Lay::kDPCol;
    float* lut = reinterpret_cast<float*>(smem + Lay::kLutOff);
    float l2 = INFINITY, dd = 0.f;
    if (i < p.L) {
      const int64_t idx = (static_cast<int64_t>(b) * p.Hq + hq) * p.L + i;
      l2 = p.lse[idx] * kLog2e;
      dd = p.dvec[idx];
      if (l2 == -INFINITY) l2 = INFINITY;
    }
    const float* brow = nullptr;
    if constexpr (BIAS == kBiasDense) {
      brow = p.bias + static_cast<int64_t>(b) * p.sb_b + static_cast<int64_t>(hq) * p.sb_h +
             static_cast<int64_t>(min(i, p.L - 1)) * p.sb_i;
    }
    bool ok = true;
    for (int it = 0; it < nt; ++it) {
      const int n0 = (nlo + it) * kTile;
      const bool full = tile_is_full(p, m0, n0, false);
      int lo = 0, hi = kTile - 1;
      if (!full) row_visible_cols(p, i, n0, lo, hi);
      const float* lut_row = nullptr;
      if constexpr (BIAS == kBiasT5) {
        float* lt = lut + (it & 1) * 256;
        const int base = n0 - m0 - (kTile - 1);
        lt[row] = p.t5_table[t5_bucket(base + row, p.t5) * p.Hq + hq] * kLog2e;
        if (row < kTile - 1)
          lt[row + kTile] = p.t5_table[t5_bucket(base + row + kTile, p.t5) * p.Hq + hq] * kLog2e;
        named_barrier(1, kTile);
        lut_row = lt + (kTile - 1) - row;
      }
      if (ok) ok = mbar_wait(s_full, it & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
      uint32_t pr[128];  // S row, then P (fp32 bits) in place
      tmem_ld128_sync(tS, pr);
#pragma unroll
      for (int c = 0; c < kTile; ++c) {
        float x = __uint_as_float(pr[c]) * p.scale_log2 - l2;
        const bool vis = full || (c >= lo && c <= hi);
        if constexpr (BIAS == kBiasT5) x += lut_row[c];
        if constexpr (BIAS == kBiasDense) x += vis ? brow[n0 + c] * kLog2e : 0.f;
        pr[c] = __float_as_uint(vis ? fast_exp2(x) : 0.f);
      }
      if (ok) ok = mbar_wait(dp_full, it & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < kTile; c0 += 32) {
        uint32_t dr[32];
        tmem_ld32_sync(tDP + c0, dr);
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float d0 = __uint_as_float(pr[c0 + c]) * (__uint_as_float(dr[c]) - dd);
          const float d1 = __uint_as_float(pr[c0 + c + 1]) * (__uint_as_float(dr[c + 1]) - dd);
          pk[c >> 1] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tS + (c0 >> 1), pk);  // dS over the first 64 columns of S
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    if (ok && nt > 0) ok = mbar_wait(o_done, (nt - 1) & 1, ctl);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* dst = p.dq + static_cast<int64_t>(b) * p.sq_b + static_cast<int64_t>(i) * p.sq_l +
                           static_cast<int64_t>(hq) * p.sq_h;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        if (nt > 0) {
          tmem_ld32_sync(tmem + lane_bits + Lay::kDQCol + c, r);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * p.scale,
                              __uint_as_float(r[2 * e + 1]) * p.scale);
        if (i < p.L) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            d4[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

// ------------------------------------------------------------- launchers
constexpr uint32_t kPhasePre = 1u, kPhaseDq = 2u, kPhaseDkdv = 4u;

template <int D, int BIAS>
cudaError_t launch_bwd_t(const AttnParams& p, const BwdMaps& m, uint32_t phases,
                         cudaStream_t st) {
  if (phases & kPhasePre) {
    const int64_t threads = static_cast<int64_t>(p.B) * p.L * p.Hq * (D / 8);
    const int64_t blocks = (threads + 255) / 256;
    bwd_preprocess_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int ntiles = (p.L + kTile - 1) / kTile;
  if (phases & kPhaseDq) {
    auto kern = bwd_dq_kernel<D, BIAS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DqLayout<D>::kSmemAlloc);
    if (e != cudaSuccess) return e;
    kern<<<dim3(ntiles, p.Hq, p.B), DqLayout<D>::kThreads, DqLayout<D>::kSmemAlloc, st>>>(
        p, m.q, m.k, m.v, m.dout);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (phases & kPhaseDkdv) {
    auto kern = bwd_dkdv_kernel<D, BIAS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DkdvLayout<D>::kSmemAlloc);
    if (e != cudaSuccess) return e;
    kern<<<dim3(ntiles, p.Hkv, p.B), DkdvLayout<D>::kThreads, DkdvLayout<D>::kSmemAlloc, st>>>(
        p, m.q, m.k, m.v, m.dout);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int D>
cudaError_t launch_bwd_d(const AttnParams& p, const BwdMaps& m, uint32_t phases,
                         cudaStream_t st) {
  switch (p.bias_kind) {
    case kBiasDense: return launch_bwd_t<D, kBiasDense>(p, m, phases, st);
    case kBiasT5: return launch_bwd_t<D, kBiasT5>(p, m, phases, st);
    default: return launch_bwd_t<D, kBiasNone>(p, m, phases, st);
  }
}

inline cudaError_t launch_bwd(const AttnParams& p, const BwdMaps& m, int d, uint32_t phases,
                              cudaStream_t st) {
  return d == 128 ? launch_bwd_d<128>(p, m, phases, st) : launch_bwd_d<64>(p, m, phases, st);
}

}  // namespace sdpa
