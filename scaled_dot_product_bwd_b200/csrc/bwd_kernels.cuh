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
//   2. dK/dV: one CTA per (128 keys, KV head, batch).  It walks 64-query
//      blocks of the band, for every query head of the group, in a fixed
//      order and accumulates dV and dK in tensor memory:
//        S^T = K Q^T, dP^T = V dO^T           (SS MMAs, 128 x 64)
//        P^T, dS^T -> tensor memory as bf16    (compute warpgroups)
//        dV += P^T dO, dK += dS^T Q            (TS MMAs, 128 x d)
//   3. dQ: one CTA per (128 queries, query head, batch), walking 64-key
//      blocks of the band in order: S = Q K^T, dP = dO V^T, dQ += dS K.
// In both, S and dP are double-buffered in tensor memory and the MMA warp
// issues the scores of block i before the gradient MMAs of block i-1, so the
// exponentials of one block overlap the tensor-core work of its neighbours.
// Two compute warpgroups take alternate blocks.
#pragma once

#include "attn_common.cuh"
#include "sm100.cuh"
#include "tmem_sync.cuh"

namespace sdpa {

constexpr int kBlk = 64;  // inner block: queries (dK/dV kernel) or keys (dQ kernel)

struct BwdMaps {
  CUtensorMap q128, dout128, k128, v128;  // 128-row boxes (resident tiles)
  CUtensorMap q64, dout64, k64, v64;      // 64-row boxes (streamed blocks)
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

// Byte offset of the 16-element K step kk inside a K-major SW128 tile of
// `rows` rows: a d = 128 tile is two 64-column halves of rows x 128 bytes.
__device__ __forceinline__ uint32_t kmajor_koff(int kk, int rows) {
  return static_cast<uint32_t>((kk >> 2) * rows * 128 + (kk & 3) * 32);
}

// ------------------------------------------------------------------ dK / dV
template <int D>
struct DkdvLayout {
  static constexpr int kKVBytes = kTile * D * 2;  // resident K or V tile (128 keys)
  static constexpr int kBlkBytes = kBlk * D * 2;  // one 64-query block of Q or dO
  static constexpr int kStages = 3;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKVBytes;
  static constexpr int kQOff = 2 * kKVBytes;
  static constexpr int kDOOff = kQOff + kStages * kBlkBytes;
  static constexpr int kVecOff = kDOOff + kStages * kBlkBytes;  // stages x (lse2[64], D[64])
  static constexpr int kLutOff = kVecOff + kStages * 2 * kBlk * 4;  // 2 WG x 2 x 256 floats
  static constexpr int kBarOff = kLutOff + 4 * 256 * 4;
  // kv_full, q_full[S], q_empty[S], s_full[2], dp_full[2], p_full[2], ds_full[2],
  // buf_free[2], acc_done, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 10 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static constexpr int kThreads = 320;  // 2 compute warpgroups, producer, MMA
  static constexpr int kTmemCols = 512;
  // S^T[x] at 64 x, dP^T[x] at 128 + 64 x, dV at 256, dK at 256 + D
  static constexpr int kDVCol = 256, kDKCol = 256 + D;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

template <int D, int BIAS>
__global__ void __launch_bounds__(320, 1)
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

  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int n0 = static_cast<int>(blockIdx.x) * kTile;  // causal: low key tiles are heaviest
  int mlo, mhi;
  {
    // 64-query blocks that hold any query seeing a key of this tile
    const int n_last = min(n0 + kTile - 1, p.L - 1);
    int imin = 0;
    if (p.causal) imin = n0;
    if (p.wr >= 0) imin = max(imin, n0 - p.wr);
    int imax = p.L - 1;
    if (p.wl >= 0) imax = min(imax, n_last + p.wl);
    mlo = imin / kBlk;
    mhi = (imax >= imin) ? imax / kBlk + 1 : mlo;
  }
  const int nm = mhi - mlo;
  const int total = nm * p.G;  // blocks: query head (outer) x query block (inner)

  auto bar = [&](int idx) -> uint32_t { return sb + Lay::kBarOff + 8 * idx; };
  const uint32_t kv_full = bar(0);
  auto q_full = [&](int s) { return bar(1 + s); };
  auto q_empty = [&](int s) { return bar(1 + S + s); };
  auto s_full = [&](int x) { return bar(1 + 2 * S + x); };
  auto dp_full = [&](int x) { return bar(3 + 2 * S + x); };
  auto p_full = [&](int x) { return bar(5 + 2 * S + x); };
  auto ds_full = [&](int x) { return bar(7 + 2 * S + x); };
  auto buf_free = [&](int x) { return bar(9 + 2 * S + x); };
  const uint32_t acc_done = bar(11 + 2 * S);
  const uint32_t drain = bar(12 + 2 * S);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(q_full(s), 32);  // the producer warp's lanes (lane 0 with the tx count)
      mbar_init(q_empty(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(dp_full(x), 1);
      mbar_init(p_full(x), kTile);
      mbar_init(ds_full(x), kTile);
      mbar_init(buf_free(x), 1);
    }
    mbar_init(acc_done, 1);
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
  float* vec = reinterpret_cast<float*>(smem + Lay::kVecOff);

  if (warp == 8) {
    // ============================ producer ============================
    if (total > 0) {
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmDO);
        mbar_expect_tx(kv_full, 2 * Lay::kKVBytes);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_4d(sb + Lay::kKOff + h * kTile * 128, &tmK, kv_full, h * 64, n0, g, b);
          tma_load_4d(sb + Lay::kVOff + h * kTile * 128, &tmV, kv_full, h * 64, n0, g, b);
        }
      }
      int issued[S];
      for (int s = 0; s < S; ++s) issued[s] = -1;
      bool ok = true;
      for (int it = 0; it < total; ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const int hq = g * p.G + it / nm;
        const int m0 = (mlo + it % nm) * kBlk;
        if (ok) ok = mbar_wait(q_empty(s), ph ^ 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        // LSE (log2 units) and D of the block's 64 queries, two per lane
        float* lse2 = vec + s * 2 * kBlk;
        float* dvv = lse2 + kBlk;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = lane + 32 * e;
          const int i = m0 + c;
          float l2 = INFINITY, dd = 0.f;  // queries past L: P = 0
          if (i < p.L) {
            const int64_t idx = (static_cast<int64_t>(b) * p.Hq + hq) * p.L + i;
            l2 = p.lse[idx] * kLog2e;
            dd = p.dvec[idx];
            if (l2 == -INFINITY) l2 = INFINITY;  // row with no visible key
          }
          lse2[c] = l2;
          dvv[c] = dd;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_expect_tx(q_full(s), 2 * Lay::kBlkBytes);
          for (int h = 0; h < D / 64; ++h) {
            tma_load_4d(sb + Lay::kQOff + s * Lay::kBlkBytes + h * kBlk * 128, &tmQ, q_full(s),
                        h * 64, m0, hq, b);
            tma_load_4d(sb + Lay::kDOOff + s * Lay::kBlkBytes + h * kBlk * 128, &tmDO, q_full(s),
                        h * 64, m0, hq, b);
          }
        } else {
          mbar_arrive(q_full(s));
        }
        issued[s] = ph;
      }
      if (!ok && lane == 0) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mbar_wait(kv_full, 0, ign);
        for (int s = 0; s < S; ++s)
          if (issued[s] >= 0) mbar_wait(q_full(s), issued[s], ign);
      }
    }
  } else if (warp == 9) {
    // ============================ MMA issuer ============================
    if (lane == 0 && total > 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTile, kBlk, 0, 0);  // 128 keys x 64 queries
      constexpr uint32_t kIdG = idesc_bf16_f32(kTile, D, 0, 1);     // 128 keys x d
      auto grads = [&](int jb) -> bool {
        const int x = jb & 1;
        const int s = jb % S;
        const uint32_t ph = (jb >> 1) & 1;
        const uint32_t qs = sb + Lay::kQOff + s * Lay::kBlkBytes;
        const uint32_t dos = sb + Lay::kDOOff + s * Lay::kBlkBytes;
        if (!mbar_wait(p_full(x), ph, ctl)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          mma_ts(tmem + Lay::kDVCol, tmem + 64 * x + kk * 8,
                 smem_desc_sw128(dos + kk * 2048, kBlk * 128, 1024), kIdG,
                 (jb > 0 || kk > 0) ? 1u : 0u);
        if (!mbar_wait(ds_full(x), ph, ctl)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          mma_ts(tmem + Lay::kDKCol, tmem + 128 + 64 * x + kk * 8,
                 smem_desc_sw128(qs + kk * 2048, kBlk * 128, 1024), kIdG,
                 (jb > 0 || kk > 0) ? 1u : 0u);
        mma_commit(buf_free(x));
        mma_commit(q_empty(s));
        return true;
      };
      bool ok = mbar_wait(kv_full, 0, ctl);
      for (int it = 0; it < total && ok; ++it) {
        const int x = it & 1;
        const int s = it % S;
        const uint32_t qs = sb + Lay::kQOff + s * Lay::kBlkBytes;
        const uint32_t dos = sb + Lay::kDOOff + s * Lay::kBlkBytes;
        if (!(ok = mbar_wait(q_full(s), (it / S) & 1, ctl))) break;
        // buffer x last held block it-2: its P^T / dS^T must have been consumed
        if (it >= 2 && !(ok = mbar_wait(buf_free(x), ((it >> 1) - 1) & 1, ctl))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + 64 * x, smem_desc_sw128(sb + Lay::kKOff + kmajor_koff(kk, kTile), 16, 1024),
                 smem_desc_sw128(qs + kmajor_koff(kk, kBlk), 16, 1024), kIdS, kk > 0 ? 1u : 0u);
        mma_commit(s_full(x));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + 128 + 64 * x,
                 smem_desc_sw128(sb + Lay::kVOff + kmajor_koff(kk, kTile), 16, 1024),
                 smem_desc_sw128(dos + kmajor_koff(kk, kBlk), 16, 1024), kIdS, kk > 0 ? 1u : 0u);
        mma_commit(dp_full(x));
        if (it >= 1 && !(ok = grads(it - 1))) break;
      }
      if (ok) ok = grads(total - 1);
      if (ok) mma_commit(acc_done);
      if (!ok) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mma_commit(drain);
        mbar_wait(drain, 0, ign);
      }
    }
  } else {
    // ======= compute warpgroup wg: blocks it = wg, wg + 2, ...; thread = key =======
    const int wg = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const int j = n0 + row;
    const uint32_t lane_bits = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_bits + 64 * wg;
    const uint32_t tDP = tmem + lane_bits + 128 + 64 * wg;
    float* lut = reinterpret_cast<float*>(smem + Lay::kLutOff) + wg * 512;
    bool ok = true;
    for (int it = wg; it < total; it += 2) {
      const int k = it >> 1;
      const int s = it % S;
      const int hq = g * p.G + it / nm;
      const int m0 = (mlo + it % nm) * kBlk;
      const float* lut_row = nullptr;
      if constexpr (BIAS == kBiasT5) {
        // j - i = (n0 - m0) + (row - c): entry r = row - c + 63, r in [0, 190]
        float* lt = lut + (k & 1) * 256;
        const int base = n0 - m0 - (kBlk - 1);
        for (int r = row; r < kTile + kBlk - 1; r += kTile)
          lt[r] = p.t5_table[t5_bucket(base + r, p.t5) * p.Hq + hq] * kLog2e;
        named_barrier(1 + wg, kTile);
        lut_row = lt + row + (kBlk - 1);
      }
      // visible queries of this key inside the block: [lo, hi]
      int lo = 0, hi = kBlk - 1;
      bool full = (m0 + kBlk <= p.L) && (n0 + kTile <= p.L);
      if (p.causal) full = full && (n0 + kTile - 1 <= m0);
      if (p.wl >= 0) full = full && (m0 + kBlk - 1 <= n0 + p.wl);
      if (p.wr >= 0) full = full && (n0 + kTile - 1 <= m0 + p.wr);
      if (!full) {
        if (p.causal) lo = max(lo, j - m0);
        if (p.wr >= 0) lo = max(lo, j - p.wr - m0);
        hi = min(hi, p.L - 1 - m0);
        if (p.wl >= 0) hi = min(hi, j + p.wl - m0);
      }
      const float* bcol = nullptr;
      if constexpr (BIAS == kBiasDense)
        bcol = p.bias + static_cast<int64_t>(b) * p.sb_b + static_cast<int64_t>(hq) * p.sb_h +
               static_cast<int64_t>(m0) * p.sb_i + min(j, p.L - 1);
      if (ok) ok = mbar_wait(q_full(s), (it / S) & 1, ctl);  // LSE / D staged
      if (ok) ok = mbar_wait(s_full(wg), k & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
      const float* lse2 = vec + s * 2 * kBlk;
      const float* dvv = lse2 + kBlk;
      uint32_t pr[64];  // S^T row, then P^T (fp32 bits)
      tmem_ld64_sync(tS, pr);
#pragma unroll
      for (int c = 0; c < kBlk; ++c) {
        float x = __uint_as_float(pr[c]) * p.scale_log2 - lse2[c];
        const bool vis = full || (c >= lo && c <= hi);
        if constexpr (BIAS == kBiasT5) x += lut_row[-c];
        if constexpr (BIAS == kBiasDense)
          x += vis ? bcol[static_cast<int64_t>(c) * p.sb_i] * kLog2e : 0.f;
        pr[c] = __float_as_uint(vis ? fast_exp2(x) : 0.f);
      }
#pragma unroll
      for (int c0 = 0; c0 < kBlk; c0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2)
          pk[c >> 1] = pack_bf16x2(__uint_as_float(pr[c0 + c]), __uint_as_float(pr[c0 + c + 1]));
        tmem_st16(tS + (c0 >> 1), pk);  // P^T over the first 32 columns of S^T[wg]
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full(wg));
      if (ok) ok = mbar_wait(dp_full(wg), k & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < kBlk; c0 += 32) {
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
        tmem_st16(tDP + (c0 >> 1), pk);  // dS^T over the first 32 columns of dP^T[wg]
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full(wg));
    }
    // ---------------- epilogue: warpgroup 0 stores dV, warpgroup 1 stores dK ----------------
    if (ok && total > 0) ok = mbar_wait(acc_done, 0, ctl);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const int64_t off = static_cast<int64_t>(b) * p.skv_b + static_cast<int64_t>(j) * p.skv_l +
                          static_cast<int64_t>(g) * p.skv_h;
      __nv_bfloat16* dst = (wg == 0 ? p.dv : p.dk) + off;
      const float mul = wg == 0 ? 1.f : p.scale;
      const uint32_t tcol = tmem + lane_bits + (wg == 0 ? Lay::kDVCol : Lay::kDKCol);
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
  static constexpr int kQBytes = kTile * D * 2;   // resident Q or dO tile (128 queries)
  static constexpr int kBlkBytes = kBlk * D * 2;  // one 64-key block of K or V
  static constexpr int kStages = 3;
  static constexpr int kQOff = 0;
  static constexpr int kDOOff = kQBytes;
  static constexpr int kKOff = 2 * kQBytes;
  static constexpr int kVOff = kKOff + kStages * kBlkBytes;
  static constexpr int kLutOff = kVOff + kStages * kBlkBytes;  // 2 WG x 2 x 256 floats
  static constexpr int kBarOff = kLutOff + 4 * 256 * 4;
  // q_full, kv_full[S], kv_empty[S], s_full[2], dp_full[2], ds_full[2], buf_free[2],
  // acc_done, drain
  static constexpr int kNumBars = 1 + 2 * kStages + 8 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static constexpr int kThreads = 320;
  static constexpr int kTmemCols = 512;
  // S[x] at 64 x, dP[x] at 128 + 64 x, dQ at 256
  static constexpr int kDQCol = 256;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

template <int D, int BIAS>
__global__ void __launch_bounds__(320, 1)
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
  {
    // 64-key blocks holding any key visible from rows [m0, m0 + 128)
    const int m_last = min(m0 + kTile - 1, p.L - 1);
    int jmin = 0;
    if (p.wl >= 0) jmin = max(0, m0 - p.wl);
    int jmax = p.L - 1;
    if (p.causal) jmax = min(jmax, m_last);
    if (p.wr >= 0) jmax = min(jmax, m_last + p.wr);
    nlo = jmin / kBlk;
    nhi = (jmax >= jmin) ? jmax / kBlk + 1 : nlo;
  }
  const int nt = nhi - nlo;

  auto bar = [&](int idx) -> uint32_t { return sb + Lay::kBarOff + 8 * idx; };
  const uint32_t q_full = bar(0);
  auto kv_full = [&](int s) { return bar(1 + s); };
  auto kv_empty = [&](int s) { return bar(1 + S + s); };
  auto s_full = [&](int x) { return bar(1 + 2 * S + x); };
  auto dp_full = [&](int x) { return bar(3 + 2 * S + x); };
  auto ds_full = [&](int x) { return bar(5 + 2 * S + x); };
  auto buf_free = [&](int x) { return bar(7 + 2 * S + x); };
  const uint32_t acc_done = bar(9 + 2 * S);
  const uint32_t drain = bar(10 + 2 * S);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(dp_full(x), 1);
      mbar_init(ds_full(x), kTile);
      mbar_init(buf_free(x), 1);
    }
    mbar_init(acc_done, 1);
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

  if (warp == 8) {
    // ============================ producer ============================
    if (lane == 0 && nt > 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(q_full, 2 * Lay::kQBytes);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_4d(sb + Lay::kQOff + h * kTile * 128, &tmQ, q_full, h * 64, m0, hq, b);
        tma_load_4d(sb + Lay::kDOOff + h * kTile * 128, &tmDO, q_full, h * 64, m0, hq, b);
      }
      int issued[S];
      for (int s = 0; s < S; ++s) issued[s] = -1;
      bool ok = true;
      for (int it = 0; it < nt; ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        const int n0 = (nlo + it) * kBlk;
        if (!(ok = mbar_wait(kv_empty(s), ph ^ 1, ctl))) break;
        mbar_expect_tx(kv_full(s), 2 * Lay::kBlkBytes);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_4d(sb + Lay::kKOff + s * Lay::kBlkBytes + h * kBlk * 128, &tmK, kv_full(s),
                      h * 64, n0, g, b);
          tma_load_4d(sb + Lay::kVOff + s * Lay::kBlkBytes + h * kBlk * 128, &tmV, kv_full(s),
                      h * 64, n0, g, b);
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
  } else if (warp == 9) {
    // ============================ MMA issuer ============================
    if (lane == 0 && nt > 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTile, kBlk, 0, 0);  // 128 queries x 64 keys
      constexpr uint32_t kIdQ = idesc_bf16_f32(kTile, D, 0, 1);     // 128 queries x d
      auto grad = [&](int jb) -> bool {
        const int x = jb & 1;
        const int s = jb % S;
        const uint32_t ks = sb + Lay::kKOff + s * Lay::kBlkBytes;
        if (!mbar_wait(ds_full(x), (jb >> 1) & 1, ctl)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          mma_ts(tmem + Lay::kDQCol, tmem + 64 * x + kk * 8,
                 smem_desc_sw128(ks + kk * 2048, kBlk * 128, 1024), kIdQ,
                 (jb > 0 || kk > 0) ? 1u : 0u);
        mma_commit(buf_free(x));
        mma_commit(kv_empty(s));
        return true;
      };
      bool ok = mbar_wait(q_full, 0, ctl);
      for (int it = 0; it < nt && ok; ++it) {
        const int x = it & 1;
        const int s = it % S;
        const uint32_t ks = sb + Lay::kKOff + s * Lay::kBlkBytes;
        const uint32_t vs = sb + Lay::kVOff + s * Lay::kBlkBytes;
        if (!(ok = mbar_wait(kv_full(s), (it / S) & 1, ctl))) break;
        if (it >= 2 && !(ok = mbar_wait(buf_free(x), ((it >> 1) - 1) & 1, ctl))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + 64 * x, smem_desc_sw128(sb + Lay::kQOff + kmajor_koff(kk, kTile), 16, 1024),
                 smem_desc_sw128(ks + kmajor_koff(kk, kBlk), 16, 1024), kIdS, kk > 0 ? 1u : 0u);
        mma_commit(s_full(x));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + 128 + 64 * x,
                 smem_desc_sw128(sb + Lay::kDOOff + kmajor_koff(kk, kTile), 16, 1024),
                 smem_desc_sw128(vs + kmajor_koff(kk, kBlk), 16, 1024), kIdS, kk > 0 ? 1u : 0u);
        mma_commit(dp_full(x));
        if (it >= 1 && !(ok = grad(it - 1))) break;
      }
      if (ok) ok = grad(nt - 1);
      if (ok) mma_commit(acc_done);
      if (!ok) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mma_commit(drain);
        mbar_wait(drain, 0, ign);
      }
    }
  } else {
    // ===== compute warpgroup wg: blocks it = wg, wg + 2, ...; thread = query row =====
    const int wg = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const int i = m0 + row;
    const uint32_t lane_bits = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_bits + 64 * wg;
    const uint32_t tDP = tmem + lane_bits + 128 + 64 * wg;
    float* lut = reinterpret_cast<float*>(smem + Lay::kLutOff) + wg * 512;
    float l2 = INFINITY, dd = 0.f;
    if (i < p.L) {
      const int64_t idx = (static_cast<int64_t>(b) * p.Hq + hq) * p.L + i;
      l2 = p.lse[idx] * kLog2e;
      dd = p.dvec[idx];
      if (l2 == -INFINITY) l2 = INFINITY;
    }
    const float* brow = nullptr;
    if constexpr (BIAS == kBiasDense)
      brow = p.bias + static_cast<int64_t>(b) * p.sb_b + static_cast<int64_t>(hq) * p.sb_h +
             static_cast<int64_t>(min(i, p.L - 1)) * p.sb_i;
    bool ok = true;
    for (int it = wg; it < nt; it += 2) {
      const int k = it >> 1;
      const int n0 = (nlo + it) * kBlk;
      const float* lut_row = nullptr;
      if constexpr (BIAS == kBiasT5) {
        // j - i = (n0 - m0) + (c - row): entry r = c - row + 127, r in [0, 190]
        float* lt = lut + (k & 1) * 256;
        const int base = n0 - m0 - (kTile - 1);
        for (int r = row; r < kTile + kBlk - 1; r += kTile)
          lt[r] = p.t5_table[t5_bucket(base + r, p.t5) * p.Hq + hq] * kLog2e;
        named_barrier(1 + wg, kTile);
        lut_row = lt + (kTile - 1) - row;
      }
      int lo = 0, hi = kBlk - 1;
      bool full = n0 + kBlk <= p.L;
      if (p.causal) full = full && (n0 + kBlk - 1 <= m0);
      if (p.wl >= 0) full = full && (n0 >= m0 + kTile - 1 - p.wl);
      if (p.wr >= 0) full = full && (n0 + kBlk - 1 <= m0 + p.wr);
      if (!full) {
        if (p.wl >= 0) lo = max(lo, i - p.wl - n0);
        hi = min(hi, p.L - 1 - n0);
        if (p.causal) hi = min(hi, i - n0);
        if (p.wr >= 0) hi = min(hi, i + p.wr - n0);
      }
      if (ok) ok = mbar_wait(s_full(wg), k & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
      uint32_t pr[64];  // S row, then P (fp32 bits)
      tmem_ld64_sync(tS, pr);
#pragma unroll
      for (int c = 0; c < kBlk; ++c) {
        float x = __uint_as_float(pr[c]) * p.scale_log2 - l2;
        const bool vis = full || (c >= lo && c <= hi);
        if constexpr (BIAS == kBiasT5) x += lut_row[c];
        if constexpr (BIAS == kBiasDense) x += vis ? brow[n0 + c] * kLog2e : 0.f;
        pr[c] = __float_as_uint(vis ? fast_exp2(x) : 0.f);
      }
      if (ok) ok = mbar_wait(dp_full(wg), k & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < kBlk; c0 += 32) {
        uint32_t dr[32];
        tmem_ld32_sync(tDP + c0, dr);
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float d0 = __uint_as_float(pr[c0 + c]) * (__uint_as_float(dr[c]) - dd);
          const float d1 = __uint_as_float(pr[c0 + c + 1]) * (__uint_as_float(dr[c + 1]) - dd);
          pk[c >> 1] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tS + (c0 >> 1), pk);  // dS over the first 32 columns of S[wg]
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full(wg));
    }
    // ------------- epilogue: warpgroup wg stores dQ columns [wg D/2, (wg+1) D/2) -------------
    if (ok && nt > 0) ok = mbar_wait(acc_done, 0, ctl);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* dst = p.dq + static_cast<int64_t>(b) * p.sq_b + static_cast<int64_t>(i) * p.sq_l +
                           static_cast<int64_t>(hq) * p.sq_h;
#pragma unroll
      for (int c = wg * (D / 2); c < (wg + 1) * (D / 2); c += 32) {
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
        p, m.q128, m.k64, m.v64, m.dout128);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (phases & kPhaseDkdv) {
    auto kern = bwd_dkdv_kernel<D, BIAS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DkdvLayout<D>::kSmemAlloc);
    if (e != cudaSuccess) return e;
    kern<<<dim3(ntiles, p.Hkv, p.B), DkdvLayout<D>::kThreads, DkdvLayout<D>::kSmemAlloc, st>>>(
        p, m.q64, m.k128, m.v128, m.dout64);
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
