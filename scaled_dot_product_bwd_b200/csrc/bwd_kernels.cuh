// bwd_kernels.cuh -- fused attention backward for sm_100a.
//
// The pages print no gradient formulas; these kernels apply the chain rule
// to the forward (codelab "jax-gpu-05-attention-gpu", sections 1 and 4):
//   P = exp(S - LSE)  (S recomputed with the forward's mask and bias)
//   dV = P^T dO,  dP = dO V^T,  D_i = rowsum(dO_i * O_i),  dS = P (dP - D)
//   dK = scale dS^T Q,  dQ = scale dS K
// Two launches:
//   1. preprocess: D = rowsum(dO * O); zeroes the dQ turn counters and the
//      work-item counter of launch 2.
//   2. one persistent kernel for all three gradients.  A work item is 128
//      keys of one (batch, KV head); it walks the 128-query tiles of the
//      mask band, every query head of the group at each tile, and per block
//        S^T = K Q^T, dP^T = V dO^T            (SS MMAs, 128 x 128)
//        P^T -> tensor memory (bf16), dS -> shared memory (bf16)
//        dV += P^T dO (TS), dK += dS^T Q (SS), dQ_part = dS K (SS)
//      dV and dK stay in tensor memory for the whole item.  Each dQ_part is
//      added into an fp32 accumulator in global memory, the contributions to
//      one query tile in descending key-tile order: a turn counter per
//      (query tile, 32-row quarter) holds the number of key tiles already
//      added, the first key tile stores, the last one writes
//      dQ = scale * sum as bf16.  A fixed-order split-K reduction with no
//      floating-point atomics, so the result is bit-identical run to run
//      (HF transformers issue #31787, "Transformer models are not
//      deterministic when using Flash Attention 2").
//
// Work items are handed out by an atomic ticket counter, group by group
// ((batch, KV head) major) and within a group from the last key tile to the
// first, which is also the order of the dQ sums.  A waiting item only waits
// for items with smaller tickets, all of which are held by CTAs that are
// running or done, so the waits always end.  Within an item the query tiles
// run from the first of its band to the last, every head of the group at
// each: under a causal or windowed mask key tile n + 1 then reaches each
// query tile G blocks before key tile n does, so the contributions to a
// tile arrive spaced out and in order, and a turn is usually free when it
// is needed.
#pragma once

#include "attn_common.cuh"
#include "exp2_poly.cuh"
#include "sm100.cuh"
#include "tmem_sync.cuh"

namespace sdpa {

// Share of a full tile's exponentials on MUFU (per 8 columns; 8 = all).
constexpr int kBwdMufuPer8 = 5;

// ------------------------------------------------------------ preprocess
// D = rowsum(dO * O) for every query row along the (padded or packed)
// sequence axis, and zeroes `n_zero` words of turn counters plus the ticket.
// Rows of query tiles that no key tile reaches (a left window that starts
// past the end of a shorter key sequence, an empty packed key sequence)
// get no dQ contribution from the main kernel: their dQ is zeroed here.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const AttnParams p, int64_t n_axis,
                                                             int64_t n_zero) {
  constexpr int kTpr = D / 8;  // threads per row, 8 bf16 (16 bytes) each
  const int64_t gt = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (gt < n_zero) p.turns[gt] = 0u;
  if (gt == 0) *p.tickets = 0u;
  const int64_t nrows = n_axis * p.Hq;
  const int64_t r = gt / kTpr;
  const int part = static_cast<int>(gt % kTpr);
  float acc = 0.f;
  int h = 0;
  int64_t a = 0, b = 0, i = 0;
  if (r < nrows) {
    h = static_cast<int>(r % p.Hq);
    a = r / p.Hq;                         // position along the sequence axis
    b = p.cu_q ? 0 : a / p.Lq;
    i = p.cu_q ? a : a % p.Lq;
    const int64_t off = b * p.sq_b + i * p.sq_l + h * p.sq_h + part * 8;
    const uint4 x4 = *reinterpret_cast<const uint4*>(p.o + off);
    const uint4 y4 = *reinterpret_cast<const uint4*>(p.dout + off);
    const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&x4);
    const __nv_bfloat162* y2 = reinterpret_cast<const __nv_bfloat162*>(&y4);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = __bfloat1622float2(x2[e]);
      const float2 y = __bfloat1622float2(y2[e]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (r < nrows) {
    if (part == 0) p.dvec[b * p.lse_sb + h * p.lse_sh + i] = acc;
    // the sequence of this row: b itself, or (packed) the last entry whose
    // first row is at or before it
    int bb = static_cast<int>(b);
    if (p.cu_q) {
      int lo = 0, hi = p.B;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.cu_q[mid] <= a) lo = mid; else hi = mid;
      }
      bb = lo;
    }
    const SeqView sv = seq_view(p, bb);
    const int il = static_cast<int>(p.cu_q ? a - sv.q0 : i);
    int nlo, nhi;
    key_tile_range(p, sv.Lq, sv.Lk, (il / kTile) * kTile, kTile, nlo, nhi);
    if (nhi <= nlo || il < 0 || il >= sv.Lq)
      *reinterpret_cast<uint4*>(p.dq + b * p.sq_b + i * p.sq_l + h * p.sq_h + part * 8) =
          make_uint4(0u, 0u, 0u, 0u);
  }
}

// ------------------------------------------------------------ turn counters
__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(unsigned int* p, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Whole warp: wait until *ctr == want, for at most ctl.limit_ns.  On expiry
// (or if another wait of the CTA aborted) raises the abort flag and the
// device status and returns false.
__device__ __forceinline__ bool wait_turn(const unsigned int* ctr, unsigned int want,
                                          const WaitCtl& ctl) {
  if (__shfl_sync(0xffffffffu, ld_acquire_u32(ctr), 0) == want) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t k = 1;; ++k) {
    if (k > 32) __nanosleep(64);
    if (__shfl_sync(0xffffffffu, ld_acquire_u32(ctr), 0) == want) return true;
    if ((k & 255u) == 0) {
      const bool stop = *ctl.abort || (globaltimer_ns() - t0 > ctl.limit_ns);
      if (__shfl_sync(0xffffffffu, stop ? 1 : 0, 0)) {
        if ((threadIdx.x & 31) == 0) {
          *ctl.abort = 1;
          atomicOr(&g_device_status, kStatusTimeout);
        }
        return false;
      }
    }
  }
}

// 16 columns of one row, bf16, as two uint4 (columns c..c+7, c+8..c+15)
__device__ __forceinline__ void pack16(const uint32_t* r, float mul, uint4& lo, uint4& hi) {
  lo.x = pack_bf16x2(__uint_as_float(r[0]) * mul, __uint_as_float(r[1]) * mul);
  lo.y = pack_bf16x2(__uint_as_float(r[2]) * mul, __uint_as_float(r[3]) * mul);
  lo.z = pack_bf16x2(__uint_as_float(r[4]) * mul, __uint_as_float(r[5]) * mul);
  lo.w = pack_bf16x2(__uint_as_float(r[6]) * mul, __uint_as_float(r[7]) * mul);
  hi.x = pack_bf16x2(__uint_as_float(r[8]) * mul, __uint_as_float(r[9]) * mul);
  hi.y = pack_bf16x2(__uint_as_float(r[10]) * mul, __uint_as_float(r[11]) * mul);
  hi.z = pack_bf16x2(__uint_as_float(r[12]) * mul, __uint_as_float(r[13]) * mul);
  hi.w = pack_bf16x2(__uint_as_float(r[14]) * mul, __uint_as_float(r[15]) * mul);
}

__device__ __forceinline__ uint4 shfl_xor_u4(uint4 v, int m) {
  v.x = __shfl_xor_sync(0xffffffffu, v.x, m);
  v.y = __shfl_xor_sync(0xffffffffu, v.y, m);
  v.z = __shfl_xor_sync(0xffffffffu, v.z, m);
  v.w = __shfl_xor_sync(0xffffffffu, v.w, m);
  return v;
}

__device__ __forceinline__ float4 shfl_xor_f4(float4 v, int m) {
  v.x = __shfl_xor_sync(0xffffffffu, v.x, m);
  v.y = __shfl_xor_sync(0xffffffffu, v.y, m);
  v.z = __shfl_xor_sync(0xffffffffu, v.z, m);
  v.w = __shfl_xor_sync(0xffffffffu, v.w, m);
  return v;
}

__device__ __forceinline__ float4 f4_add(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// ---------------------------------------------------------------- layout
// Tensor memory (512 columns): S^T 0..127 | dP^T 128..255 | dV 256.. | dK
// 256 + d..  P^T (bf16) overwrites the first half of each compute
// warpgroup's S^T columns and feeds the dV MMA from there.  The dQ partial
// (128 queries x d fp32) goes over the dP^T columns at d = 128 (the compute
// warpgroups have read dP^T by then) and into two buffers of its own at
// 384 and 448 at d = 64.
template <int D, int BIAS>
struct BwdLayout {
  static constexpr int kTileBytes = kTile * D * 2;  // 128 rows x d bf16
  static constexpr int kDSBytes = kTile * kTile * 2;  // dS, 128 keys x 128 queries bf16
  // Q blocks are read by S^T and dK, dO blocks by dP^T and dV.  At d = 128
  // K, V, dS and two stages of each ring fill the 227 KB of shared memory.
  static constexpr int kSQ = (D == 128) ? 2 : 4;
  static constexpr int kSO = (D == 128) ? (BIAS == kBiasT5 ? 1 : 2) : 4;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kDSOff = 2 * kTileBytes;
  static constexpr int kQOff = kDSOff + kDSBytes;
  static constexpr int kDOOff = kQOff + kSQ * kTileBytes;
  static constexpr int kVecOff = kDOOff + kSO * kTileBytes;      // 2 x (lse2[128], D[128])
  static constexpr int kLutOff = kVecOff + 2 * 2 * kTile * 4;    // T5 only: 8 warps x 96 floats
  static constexpr int kLutBytes = (BIAS == kBiasT5) ? 8 * 96 * 4 : 0;
  static constexpr int kBarOff = kLutOff + kLutBytes;
  static constexpr int kNumBars = 2 + 2 * kSQ + 2 * kSO + 22;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;        // tmem slot, abort, item slots
  static constexpr int kSmemAlloc = kMiscOff + 32;
  // warps 0-7: two compute warpgroups; 8-11: dQ reducer; 12 producer,
  // 13 / 14 MMA issuers, 15 spare
  static constexpr int kThreads = 512;
  static constexpr int kTmemCols = 512;
  static constexpr int kSCol = 0, kDPCol = 128, kDVCol = 256, kDKCol = 256 + D;
  static constexpr bool kDQShared = (D == 128);
  static constexpr int kDQCol = kDQShared ? kDPCol : 256 + 2 * D;
  static_assert(kDQShared || kDQCol + 2 * D <= kTmemCols, "tensor memory budget");
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

// Registers per thread after the warpgroups reallocate (launched with 128
// each, 512 threads = 65536): compute warpgroups, reducer, producer/issuers.
// 2 x 152 + 128 + 80 = 512 = 4 x 128.
constexpr uint32_t kRegsCompute = 152, kRegsReducer = 128, kRegsIssue = 80;
static_assert(2 * kRegsCompute + kRegsReducer + kRegsIssue == 4 * 128, "register split");

template <int D, int BIAS, bool DS_OUT>
__global__ void __launch_bounds__(512, 1)
    bwd_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmQ,
               const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmDO) {
  using Lay = BwdLayout<D, BIAS>;
  constexpr int SQ = Lay::kSQ;
  constexpr int SO = Lay::kSO;
  extern __shared__ uint8_t smem[];
  if (!smem_base_ok(smem)) {
    if (threadIdx.x == 0) atomicOr(&g_device_status, kStatusMisaligned);
    return;
  }
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work items: (batch, KV head) groups, key tiles ascending within one
  const int ntk = (p.Lk + kTile - 1) / kTile;
  const int ntq = (p.Lq + kTile - 1) / kTile;
  const int n_items = p.B * p.Hkv * ntk;
  struct Item {
    int b, g, n, mlo, mhi, nb;
    bool rows;  // the key tile holds keys of the sequence
    SeqView s;
  };
  auto item_at = [&](int t) {
    Item w;
    const int grp = t / ntk;
    w.n = ntk - 1 - (t - grp * ntk);  // key tiles of a group from the last to the first
    w.b = grp / p.Hkv;
    w.g = grp - w.b * p.Hkv;
    w.s = seq_view(p, w.b);
    w.mlo = w.mhi = 0;
    w.nb = 0;
    w.rows = w.n * kTile < w.s.Lk;
    if (w.rows) {
      query_tile_range(p, w.s.Lq, w.s.Lk, w.n * kTile, w.mlo, w.mhi);
      if (w.mhi > w.mlo) w.nb = (w.mhi - w.mlo) * p.G;
    }
    return w;
  };

  // ---- barriers
  auto bar = [&](int idx) -> uint32_t { return sb + Lay::kBarOff + 8 * idx; };
  const uint32_t kv_full = bar(0);
  const uint32_t kv_empty = bar(1);
  auto q_full = [&](int s) { return bar(2 + s); };
  auto q_empty = [&](int s) { return bar(2 + SQ + s); };
  auto o_full = [&](int s) { return bar(2 + 2 * SQ + s); };
  auto o_empty = [&](int s) { return bar(2 + 2 * SQ + SO + s); };
  constexpr int kB = 2 + 2 * SQ + 2 * SO;
  auto vec_full = [&](int x) { return bar(kB + x); };
  auto vec_empty = [&](int x) { return bar(kB + 2 + x); };
  const uint32_t s_full = bar(kB + 4);
  const uint32_t p_full = bar(kB + 5);
  const uint32_t s_free = bar(kB + 6);
  const uint32_t dp_full = bar(kB + 7);
  const uint32_t ds_full = bar(kB + 8);
  const uint32_t ds_free = bar(kB + 9);
  auto dq_full = [&](int x) { return bar(kB + 10 + x); };
  auto dq_free = [&](int x) { return bar(kB + 12 + x); };
  const uint32_t acc_done = bar(kB + 14);
  const uint32_t acc_free = bar(kB + 15);
  auto item_full = [&](int x) { return bar(kB + 16 + x); };
  auto item_empty = [&](int x) { return bar(kB + 18 + x); };
  auto drain = [&](int x) { return bar(kB + 20 + x); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 8);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 2);  // both issuers, after their last MMA of the item
    for (int s = 0; s < SQ; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 2);
    }
    for (int s = 0; s < SO; ++s) {
      mbar_init(o_full(s), 1);
      mbar_init(o_empty(s), 2);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(vec_full(x), 32);          // the producer warp's lanes
      mbar_init(vec_empty(x), 2 * kTile);  // both compute warpgroups
      mbar_init(dq_full(x), 1);
      mbar_init(dq_free(x), 4);            // the reducer warps
      mbar_init(item_full(x), 1);
      mbar_init(item_empty(x), 14);        // 2 issuers, 8 compute and 4 reducer warps
      mbar_init(drain(x), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 2 * kTile);
    mbar_init(s_free, 1);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 2 * kTile);
    mbar_init(ds_free, 1);
    mbar_init(acc_done, 2);
    mbar_init(acc_free, 2 * kTile);
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

  // Item ids from the producer's ring of two slots.  Returns false on abort.
  auto next_item = [&](int k, int& t) -> bool {
    bool ok = mbar_wait(item_full(k & 1), (k >> 1) & 1, ctl);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) return false;
    t = item_slot[k & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(item_empty(k & 1));
    return true;
  };

  if (warp >= 12) {
    regs_shrink<kRegsIssue>();
    if (warp == 12) {
      // ============================ producer ============================
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmDO);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      int issued_q[SQ], issued_o[SO];
      for (int s = 0; s < SQ; ++s) issued_q[s] = -1;
      for (int s = 0; s < SO; ++s) issued_o[s] = -1;
      int kv_issued = -1;
      bool ok = true;
      int i = 0, k = 0, u = 0;
      while (ok) {
        int t = -1;
        if (lane == 0) {
          t = static_cast<int>(atomicAdd(p.tickets, 1u));
          if (t >= n_items) t = -1;
        }
        t = __shfl_sync(0xffffffffu, t, 0);
        ok = mbar_wait(item_empty(k & 1), ((k >> 1) & 1) ^ 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (lane == 0) {
          item_slot[k & 1] = t;
          mbar_arrive(item_full(k & 1));
        }
        ++k;
        if (t < 0) break;
        const Item w = item_at(t);
        if (w.nb == 0) continue;
        if (lane == 0) {
          if (u > 0) ok = mbar_wait(kv_empty, (u - 1) & 1, ctl);
          if (ok) {
            mbar_expect_tx(kv_full, 2 * Lay::kTileBytes);
            for (int h = 0; h < D / 64; ++h) {
              tma_load_4d(sb + Lay::kKOff + h * kTile * 128, &tmK, kv_full, h * 64,
                          w.s.k0 + w.n * kTile, w.g, w.s.bc);
              tma_load_4d(sb + Lay::kVOff + h * kTile * 128, &tmV, kv_full, h * 64,
                          w.s.k0 + w.n * kTile, w.g, w.s.bc);
            }
            kv_issued = u & 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        // LSE (log2 units) and D of one block's 128 queries, four per lane,
        // loaded one block ahead of the slot they go to.
        float l2v[4], ddv[4];
        auto load_vec = [&](int blk) {
          const int mi = w.mlo + blk / p.G;
          const int hq = w.g * p.G + blk % p.G;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int iq = mi * kTile + lane + 32 * e;
            l2v[e] = INFINITY;  // queries past the sequence: P = 0
            ddv[e] = 0.f;
            if (iq < w.s.Lq) {
              const int64_t idx = row_index(p, w.s, w.b, hq, iq);
              l2v[e] = p.lse[idx] * kLog2e;
              ddv[e] = p.dvec[idx];
              if (l2v[e] == -INFINITY) l2v[e] = INFINITY;  // row with no visible key
            }
          }
        };
        load_vec(0);
        for (int blk = 0; blk < w.nb; ++blk, ++i) {
          const int mi = w.mlo + blk / p.G;
          const int hq = w.g * p.G + blk % p.G;
          const int x = i & 1;
          if (lane == 0) {
            const int sq = i % SQ, so = i % SO;
            ok = mbar_wait(q_empty(sq), ((i / SQ) & 1) ^ 1, ctl);
            if (ok) {
              mbar_expect_tx(q_full(sq), Lay::kTileBytes);
              for (int h = 0; h < D / 64; ++h)
                tma_load_4d(sb + Lay::kQOff + sq * Lay::kTileBytes + h * kTile * 128, &tmQ,
                            q_full(sq), h * 64, w.s.q0 + mi * kTile, hq, w.s.bc);
              issued_q[sq] = (i / SQ) & 1;
              ok = mbar_wait(o_empty(so), ((i / SO) & 1) ^ 1, ctl);
            }
            if (ok) {
              mbar_expect_tx(o_full(so), Lay::kTileBytes);
              for (int h = 0; h < D / 64; ++h)
                tma_load_4d(sb + Lay::kDOOff + so * Lay::kTileBytes + h * kTile * 128, &tmDO,
                            o_full(so), h * 64, w.s.q0 + mi * kTile, hq, w.s.bc);
              issued_o[so] = (i / SO) & 1;
              if constexpr (BIAS == kBiasDense) prefetch_bias_tile(p, w.b, hq, mi * kTile, w.n * kTile);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (ok) ok = mbar_wait(vec_empty(x), ((i >> 1) & 1) ^ 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          float* lse2 = vec + x * 2 * kTile;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            lse2[lane + 32 * e] = l2v[e];
            lse2[kTile + lane + 32 * e] = ddv[e];
          }
          mbar_arrive(vec_full(x));
          if (blk + 1 < w.nb) load_vec(blk + 1);
        }
        ++u;
      }
      if (!ok && lane == 0) {
        // Aborted: let every copy already issued land before the CTA exits.
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        if (kv_issued >= 0) mbar_wait(kv_full, kv_issued, ign);
        for (int s = 0; s < SQ; ++s)
          if (issued_q[s] >= 0) mbar_wait(q_full(s), issued_q[s], ign);
        for (int s = 0; s < SO; ++s)
          if (issued_o[s] >= 0) mbar_wait(o_full(s), issued_o[s], ign);
      }
    } else if (warp == 13 || warp == 14) {
      // ===================== MMA issuers (one thread each) =====================
      // Warp 13: S^T(i) = K Q^T once dV(i - 1) has read P^T(i - 1) out of the
      // S^T columns, then dV(i) += P^T(i) dO(i) once P^T(i) is written.
      // Warp 14: dP^T(i) = V dO^T into its columns (at d = 128 once the
      // reducer has read dQ(i - 1) from them), then, once dS(i) is in shared
      // memory, dQ(i) = dS(i) K and dK += dS(i)^T Q(i).
      const bool chain_s = (warp == 13);
      bool ok = true;
      int i = 0, k = 0, u = 0;
      constexpr uint32_t kIdS = idesc_bf16_f32(kTile, kTile, 0, 0);  // 128 keys x 128 queries
      constexpr uint32_t kIdG = idesc_bf16_f32(kTile, D, 0, 1);      // dV, dK: 128 keys x d
      constexpr uint32_t kIdQ = idesc_bf16_f32(kTile, D, 1, 1);      // dQ: 128 queries x d
      while (true) {
        int t = -1;
        if (!(ok = next_item(k, t))) break;
        ++k;
        if (t < 0) break;
        const Item w = item_at(t);
        if (w.nb == 0) continue;
        if (lane == 0) {
          ok = issuer_wait(kv_full, u & 1, ctl);
          for (int blk = 0; blk < w.nb && ok; ++blk, ++i) {
            const int sq = i % SQ, so = i % SO;
            const uint32_t qs = sb + Lay::kQOff + sq * Lay::kTileBytes;
            const uint32_t dos = sb + Lay::kDOOff + so * Lay::kTileBytes;
            const uint32_t dss = sb + Lay::kDSOff;
            if (chain_s) {
              if (!(ok = issuer_wait(q_full(sq), (i / SQ) & 1, ctl))) break;
              if (i > 0 && !(ok = issuer_wait(s_free, (i - 1) & 1, ctl))) break;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + Lay::kSCol,
                       smem_desc_sw128(sb + Lay::kKOff + kmajor_koff(kk, kTile), 16, 1024),
                       smem_desc_sw128(qs + kmajor_koff(kk, kTile), 16, 1024), kIdS,
                       kk > 0 ? 1u : 0u);
              mma_commit(s_full);
              mma_commit(q_empty(sq));
              if (!(ok = issuer_wait(o_full(so), (i / SO) & 1, ctl))) break;
              if (!(ok = issuer_wait(p_full, i & 1, ctl))) break;
              // the item's first dV MMA overwrites the accumulator
              if (blk == 0 && u > 0 && !(ok = issuer_wait(acc_free, (u - 1) & 1, ctl))) break;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < kTile / 16; ++kk)
                mma_ts(tmem + Lay::kDVCol, split_a_col(tmem + Lay::kSCol, kk),
                       smem_desc_sw128(dos + kk * 2048, kTile * 128, 1024), kIdG,
                       (blk > 0 || kk > 0) ? 1u : 0u);
              mma_commit(s_free);
              mma_commit(o_empty(so));
            } else {
              if (!(ok = issuer_wait(o_full(so), (i / SO) & 1, ctl))) break;
              if (Lay::kDQShared && i > 0 &&
                  !(ok = issuer_wait(dq_free((i - 1) & 1), ((i - 1) >> 1) & 1, ctl)))
                break;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + Lay::kDPCol,
                       smem_desc_sw128(sb + Lay::kVOff + kmajor_koff(kk, kTile), 16, 1024),
                       smem_desc_sw128(dos + kmajor_koff(kk, kTile), 16, 1024), kIdS,
                       kk > 0 ? 1u : 0u);
              mma_commit(dp_full);
              mma_commit(o_empty(so));
              if (!(ok = issuer_wait(ds_full, i & 1, ctl))) break;
              if (!(ok = issuer_wait(q_full(sq), (i / SQ) & 1, ctl))) break;
              if (!Lay::kDQShared && i >= 2 &&
                  !(ok = issuer_wait(dq_free(i & 1), ((i >> 1) - 1) & 1, ctl)))
                break;
              tc_fence_after();
              // dQ(i) = dS(i) K: A = dS (queries contiguous), B = K (d contiguous)
              const uint32_t dqc = Lay::kDQShared ? Lay::kDPCol : Lay::kDQCol + D * (i & 1);
#pragma unroll
              for (int kk = 0; kk < kTile / 16; ++kk)
                mma_ss(tmem + dqc, smem_desc_sw128(dss + kk * 2048, kTile * 128, 1024),
                       smem_desc_sw128(sb + Lay::kKOff + kk * 2048, kTile * 128, 1024), kIdQ,
                       kk > 0 ? 1u : 0u);
              mma_commit(dq_full(i & 1));
              if (blk == 0 && u > 0 && !(ok = issuer_wait(acc_free, (u - 1) & 1, ctl))) break;
              // dK += dS(i)^T Q(i): A = dS^T (queries contiguous), B = Q (d contiguous)
#pragma unroll
              for (int kk = 0; kk < kTile / 16; ++kk)
                mma_ss(tmem + Lay::kDKCol, smem_desc_sw128(dss + kmajor_koff(kk, kTile), 16, 1024),
                       smem_desc_sw128(qs + kk * 2048, kTile * 128, 1024), kIdG,
                       (blk > 0 || kk > 0) ? 1u : 0u);
              mma_commit(ds_free);
              mma_commit(q_empty(sq));
            }
          }
          if (ok) {
            mma_commit(acc_done);
            mma_commit(kv_empty);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        i = __shfl_sync(0xffffffffu, i, 0);
        if (!ok) break;
        ++u;
      }
      if (!ok && lane == 0) {
        // Aborted: wait until every MMA this thread issued has finished with
        // tensor memory before the CTA frees it.
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mma_commit(drain(chain_s ? 0 : 1));
        mbar_wait(drain(chain_s ? 0 : 1), 0, ign);
      }
    }
  } else if (warp >= 8) {
    regs_grow<kRegsReducer>();
    // ======== dQ reducer: thread = query row 32 (warp - 8) + lane of the tile ========
    // Per block: read the dQ partial out of tensor memory, wait for this
    // (query tile, quarter)'s turn, add it to the fp32 accumulator (or store
    // it, for the first key tile; or write dQ = scale * sum as bf16, for the
    // last), then pass the turn on.  Lanes 2m and 2m + 1 hold rows r and
    // r + 1; for every 8 columns they trade halves, so that each 16-byte
    // access of the pair covers one whole 32-byte sector of one row.
    const int rq = warp - 8;
    const uint32_t lane_bits = static_cast<uint32_t>(rq * 32) << 16;
    const bool odd = (lane & 1) != 0;
    const int co = odd ? 4 : 0;  // this lane's columns in each group of 8
    // One block's share of the reduction: its query tile's place in the key
    // tiles' order (idx, first, last) and which of this lane's two rows exist.
    struct Red {
      unsigned int idx;
      int mi, hq;
      bool first, last, va, vb;
    };
    auto red_at = [&](const Item& w, int blk) {
      Red r;
      r.mi = w.mlo + blk / p.G;
      r.hq = w.g * p.G + blk % p.G;
      int nlo, nhi;
      key_tile_range(p, w.s.Lq, w.s.Lk, r.mi * kTile, kTile, nlo, nhi);
      // key tiles add in descending order: nhi - 1 first, nlo last
      r.idx = static_cast<unsigned int>(nhi - 1 - w.n);
      r.first = r.idx == 0;
      r.last = w.n == nlo;
      const int ra = r.mi * kTile + rq * 32 + (lane & ~1);  // the lane pair's first row
      r.va = ra < w.s.Lq;
      r.vb = ra + 1 < w.s.Lq;
      return r;
    };
    auto ctr_of = [&](const Item& w, const Red& r) {
      return p.turns + ((static_cast<int64_t>(w.b) * p.Hq + r.hq) * ntq + r.mi) * 4 + rq;
    };
    auto acc_of = [&](const Item& w, const Red& r) {
      return p.dq_acc + row_index(p, w.s, w.b, r.hq, r.mi * kTile + rq * 32 + (lane & ~1)) * D + co;
    };
    // This lane's running sums of one 64-column half of the block's two
    // rows: group g (8 columns) of the half at [2g] (row a) and [2g + 1].
    float4 old[16];
    auto load_half = [&](const Item& w, const Red& r, int half) {
      if (r.first) return;
      const float* acc_a = acc_of(w, r) + 64 * half;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        old[2 * g] = r.va ? __ldcg(reinterpret_cast<const float4*>(acc_a + 8 * g))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        old[2 * g + 1] = r.vb ? __ldcg(reinterpret_cast<const float4*>(acc_a + D + 8 * g))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    // wait for the block's turn, then fetch the first half's running sums
    auto fetch = [&](const Item& w, const Red& r) -> bool {
      if (r.first) return true;
      if (!wait_turn(ctr_of(w, r), r.idx, ctl)) return false;
      load_half(w, r, 0);
      return true;
    };
    bool ok = true;
    int i = 0, k = 0;
    while (true) {
      int t = -1;
      if (!(ok = next_item(k, t))) break;
      ++k;
      if (t < 0) break;
      const Item w = item_at(t);
      if (w.nb == 0) continue;
      Red cur = red_at(w, 0);
      if (!(ok = fetch(w, cur))) break;
      for (int blk = 0; blk < w.nb; ++blk, ++i) {
        ok = mbar_wait(dq_full(i & 1), (i >> 1) & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tq =
            tmem + lane_bits + (Lay::kDQShared ? Lay::kDPCol : Lay::kDQCol + D * (i & 1));
        float* acc_a = acc_of(w, cur);
        __nv_bfloat16* dq_a = p.dq + static_cast<int64_t>(w.b) * p.sq_b +
                              static_cast<int64_t>(w.s.q0 + cur.mi * kTile + rq * 32 + (lane & ~1)) * p.sq_l +
                              static_cast<int64_t>(cur.hq) * p.sq_h + co;
#pragma unroll
        for (int half = 0; half < D / 64; ++half) {
          // at d = 128 the second half's running sums come once the first
          // half's are spent (registers), while the partial is still held
          if (half > 0) load_half(w, cur, half);
#pragma unroll
          for (int c = 0; c < 64; c += 16) {
            uint32_t v[16];
            tmem_ld16_sync(tq + 64 * half + c, v);
            if (half + 1 == D / 64 && c + 16 == 64) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(dq_free(i & 1));  // the partial is out of tensor memory
            }
#pragma unroll
            for (int g2 = 0; g2 < 2; ++g2) {
              const int g = c / 8 + g2;        // group of the half
              const int col = 64 * half + 8 * g;
              const float4 lo = make_float4(__uint_as_float(v[8 * g2]), __uint_as_float(v[8 * g2 + 1]),
                                            __uint_as_float(v[8 * g2 + 2]), __uint_as_float(v[8 * g2 + 3]));
              const float4 hi = make_float4(__uint_as_float(v[8 * g2 + 4]), __uint_as_float(v[8 * g2 + 5]),
                                            __uint_as_float(v[8 * g2 + 6]), __uint_as_float(v[8 * g2 + 7]));
              // the even lane sends its columns 4..7, the odd lane its 0..3
              const float4 got = shfl_xor_f4(odd ? lo : hi, 1);
              float4 sa = odd ? got : lo;   // row a, columns col + co ..
              float4 sbv = odd ? hi : got;  // row b
              if (!cur.first) {
                sa = f4_add(old[2 * g], sa);
                sbv = f4_add(old[2 * g + 1], sbv);
              }
              if (cur.last) {
                const float sc = p.scale;
                const uint2 pa = make_uint2(pack_bf16x2(sa.x * sc, sa.y * sc), pack_bf16x2(sa.z * sc, sa.w * sc));
                const uint2 pb = make_uint2(pack_bf16x2(sbv.x * sc, sbv.y * sc), pack_bf16x2(sbv.z * sc, sbv.w * sc));
                if (cur.va) *reinterpret_cast<uint2*>(dq_a + col) = pa;
                if (cur.vb) *reinterpret_cast<uint2*>(dq_a + p.sq_l + col) = pb;
              } else {
                if (cur.va) __stcg(reinterpret_cast<float4*>(acc_a + col), sa);
                if (cur.vb) __stcg(reinterpret_cast<float4*>(acc_a + D + col), sbv);
              }
            }
          }
        }
        // The next block of the item is another query tile (or head), whose
        // turn only ever waits on key tiles handed out earlier: take it and
        // start its loads before passing this block's turn on, so their
        // latencies overlap.
        unsigned int* ctr = ctr_of(w, cur);
        const unsigned int pass = cur.idx + 1u;
        const bool release = !cur.last;
        if (blk + 1 < w.nb) {
          cur = red_at(w, blk + 1);
          if (!(ok = fetch(w, cur))) break;
        }
        if (release) {
          __threadfence();
          __syncwarp();
          if (lane == 0) st_release_u32(ctr, pass);
        }
      }
      if (!ok) break;
    }
  } else {
    if constexpr (kRegsCompute > 128) regs_grow<kRegsCompute>();
    // ===== compute warpgroup wg: query columns [64 wg, 64 wg + 64); thread = key =====
    const int wg = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const int c0w = kBlk * wg;
    const uint32_t lane_bits = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_bits + Lay::kSCol + c0w;
    const uint32_t tDP = tmem + lane_bits + Lay::kDPCol + c0w;
    float* lut = reinterpret_cast<float*>(smem + Lay::kLutOff) + warp * 96;
    uint8_t* ds_row = smem + Lay::kDSOff + wg * (kTile * 128) + row * 128;
    bool ok = true;
    int i = 0, k = 0, u = 0;
    while (true) {
      int t = -1;
      if (!(ok = next_item(k, t))) break;
      ++k;
      if (t < 0) break;
      const Item w = item_at(t);
      if (!w.rows) continue;
      const int Lq = w.s.Lq, Lk = w.s.Lk;
      const int n0 = w.n * kTile;
      const int j = n0 + row;  // this thread's key
      for (int blk = 0; blk < w.nb; ++blk, ++i) {
        const int x = i & 1;
        const int mi = w.mlo + blk / p.G;
        const int hq = w.g * p.G + blk % p.G;
        const int m0 = mi * kTile + c0w;  // first query of this warpgroup's columns
        const float* lut_row = nullptr;
        if constexpr (BIAS == kBiasT5) {
          // this warp's keys jw..jw+31 and queries m0..m0+63: j - i = (jw - m0 - 63) + e,
          // e in [0, 94]; the thread reads entry lane + 63 - c for column c
          const int base = n0 + (warp & 3) * 32 - m0 - (kBlk - 1);
          __syncwarp();
          for (int e = lane; e < 32 + kBlk - 1; e += 32) lut[e] = rel_bias_log2(p, base + e, hq);
          __syncwarp();
          lut_row = lut + lane + (kBlk - 1);
        }
        // visible queries of this key among the warpgroup's 64: [lo, hi]
        int lo = 0, hi = kBlk - 1;
        bool full = (m0 + kBlk <= Lq) && (n0 + kTile <= Lk);
        if (p.causal) full = full && (n0 + kTile - 1 <= m0);
        if (p.wl >= 0) full = full && (m0 + kBlk - 1 <= n0 + p.wl);
        if (p.wr >= 0) full = full && (n0 + kTile - 1 <= m0 + p.wr);
        if (!full) {
          if (p.causal) lo = max(lo, j - m0);
          if (p.wr >= 0) lo = max(lo, j - p.wr - m0);
          hi = min(hi, Lq - 1 - m0);
          if (p.wl >= 0) hi = min(hi, j + p.wl - m0);
          if (j >= Lk) hi = -1;  // past the key sequence: no query sees it
        }
        const float* bcol = nullptr;
        if constexpr (BIAS == kBiasDense)
          bcol = p.bias + static_cast<int64_t>(w.b) * p.sb_b + static_cast<int64_t>(hq) * p.sb_h +
                 static_cast<int64_t>(min(m0, Lq - 1)) * p.sb_i + min(j, Lk - 1);
        if (ok) ok = mbar_wait(vec_full(x), (i >> 1) & 1, ctl);  // LSE / D staged
        if (ok) ok = mbar_wait(s_full, i & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const float* lse2 = vec + x * 2 * kTile + c0w;
        const float* dvv = vec + x * 2 * kTile + kTile + c0w;
        uint32_t pr[64];  // S^T row, then P^T (fp32 bits)
        tmem_ld64_sync(tS, pr);
        const float4* lse4 = reinterpret_cast<const float4*>(lse2);
        if (full) {
#pragma unroll
          for (int c4 = 0; c4 < kBlk / 4; ++c4) {
            const float4 l = lse4[c4];
            const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * c4 + e;
              float xv = fmaf(__uint_as_float(pr[c]), p.scale_log2, -lv[e]);
              if constexpr (BIAS == kBiasT5) xv += lut_row[-c];
              if constexpr (BIAS == kBiasDense)
                xv = fmaf(bcol[static_cast<int64_t>(c) * p.sb_i], kLog2e, xv);
              pr[c] = __float_as_uint(emu_exp2<BIAS, kBwdMufuPer8>(c) ? exp2_fma(xv) : fast_exp2(xv));
            }
          }
        } else {
#pragma unroll
          for (int c4 = 0; c4 < kBlk / 4; ++c4) {
            const float4 l = lse4[c4];
            const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * c4 + e;
              const bool vis = (c >= lo) && (c <= hi);
              float xv = fmaf(__uint_as_float(pr[c]), p.scale_log2, -lv[e]);
              if constexpr (BIAS == kBiasT5) xv += lut_row[-c];
              if constexpr (BIAS == kBiasDense)
                xv = fmaf(bcol[static_cast<int64_t>(vis ? c : 0) * p.sb_i], kLog2e, xv);
              pr[c] = __float_as_uint(fast_exp2(vis ? xv : -INFINITY));
            }
          }
        }
#pragma unroll
        for (int cc = 0; cc < kBlk; cc += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2)
            pk[c >> 1] = pack_bf16x2(__uint_as_float(pr[cc + c]), __uint_as_float(pr[cc + c + 1]));
          tmem_st16(tS + (cc >> 1), pk);  // P^T over the first 32 of this warpgroup's columns
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
        if (ok) ok = mbar_wait(dp_full, i & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        // the dS buffer is free once dQ(i - 1) and dK(i - 1) have read it
        if (i > 0) ok = mbar_wait(ds_free, (i - 1) & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        float* ds_dst = nullptr;  // DS_OUT: fp32 dS of (query m0 + c, key j)
        if constexpr (DS_OUT) {
          if (j < Lk)
            ds_dst = p.ds_out + static_cast<int64_t>(w.b) * p.sd_b +
                     static_cast<int64_t>(hq) * p.sd_h + static_cast<int64_t>(m0) * p.sd_i + j;
        }
#pragma unroll
        for (int cc = 0; cc < kBlk; cc += 16) {
          uint32_t dr[16];
          tmem_ld16_sync(tDP + cc, dr);
          const float4* d4v = reinterpret_cast<const float4*>(dvv + cc);
          uint32_t pk[8];  // dS as bf16 pairs, queries cc..cc+15
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            const float4 dv4 = d4v[c >> 2];
            const float d0 = __uint_as_float(pr[cc + c]) * (__uint_as_float(dr[c]) - dv4.x);
            const float d1 = __uint_as_float(pr[cc + c + 1]) * (__uint_as_float(dr[c + 1]) - dv4.y);
            const float d2 = __uint_as_float(pr[cc + c + 2]) * (__uint_as_float(dr[c + 2]) - dv4.z);
            const float d3 = __uint_as_float(pr[cc + c + 3]) * (__uint_as_float(dr[c + 3]) - dv4.w);
            pk[c >> 1] = pack_bf16x2(d0, d1);
            pk[(c >> 1) + 1] = pack_bf16x2(d2, d3);
            if constexpr (DS_OUT) {
              // neighbouring lanes hold neighbouring keys: each store of the
              // warp writes 128 contiguous bytes of one query row; masked
              // and out-of-range entries are 0 (P = 0); rows past Lq are skipped
              if (ds_dst) {
                const float dd[4] = {d0, d1, d2, d3};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  if (m0 + cc + c + e < Lq)
                    __stcs(ds_dst + static_cast<int64_t>(cc + c + e) * p.sd_i, dd[e]);
              }
            }
          }
          // into this thread's row of the 128-byte swizzled dS tile (64
          // queries = 128 bytes): 16-byte chunk q goes to position q ^ (row % 8)
#pragma unroll
          for (int q2 = 0; q2 < 2; ++q2) {
            const int q = (cc >> 3) + q2;
            *reinterpret_cast<uint4*>(ds_row + ((q ^ (row & 7)) << 4)) =
                make_uint4(pk[4 * q2], pk[4 * q2 + 1], pk[4 * q2 + 2], pk[4 * q2 + 3]);
          }
        }
        // dP^T is read: at d = 128 the dQ MMA writes those columns next
        tc_fence_before();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(ds_full);
        mbar_arrive(vec_empty(x));
      }
      if (!ok) break;
      // ---------- item epilogue: warpgroup 0 stores dV, warpgroup 1 stores dK ----------
      if (w.nb > 0) {
        ok = mbar_wait(acc_done, u & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
      // lanes 2m, 2m + 1 hold keys j, j + 1 and trade halves of every 16
      // columns, so each 16-byte store of the pair fills one 32-byte sector
      const bool odd = (lane & 1) != 0;
      const int ja = j - (odd ? 1 : 0);
      const int64_t off = static_cast<int64_t>(w.b) * p.skv_b + static_cast<int64_t>(w.s.k0 + ja) * p.skv_l +
                          static_cast<int64_t>(w.g) * p.skv_h + (odd ? 8 : 0);
      __nv_bfloat16* dst_a = (wg == 0 ? p.dv : p.dk) + off;
      __nv_bfloat16* dst_b = dst_a + p.skv_l;
      const float mul = wg == 0 ? 1.f : p.scale;
      const uint32_t tcol = tmem + lane_bits + (wg == 0 ? Lay::kDVCol : Lay::kDKCol);
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        if (w.nb > 0) {
          tmem_ld32_sync(tcol + c, r);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0u;
        }
#pragma unroll
        for (int h = 0; h < 32; h += 16) {
          uint4 lo4, hi4;
          pack16(r + h, mul, lo4, hi4);
          const uint4 got = shfl_xor_u4(odd ? lo4 : hi4, 1);
          const uint4 va = odd ? got : lo4;  // key ja
          const uint4 vb = odd ? hi4 : got;  // key ja + 1
          if (ja < Lk) *reinterpret_cast<uint4*>(dst_a + c + h) = va;
          if (ja + 1 < Lk) *reinterpret_cast<uint4*>(dst_b + c + h) = vb;
        }
      }
      if (w.nb > 0) {
        tc_fence_before();
        mbar_arrive(acc_free);  // the next item's first dV / dK MMA may overwrite
        ++u;
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
// Launch selection bits of the backward (sdpa_bwd_phases).
constexpr uint32_t kPhasePre = 1u, kPhaseGrads = 2u;

// Workspace of the backward, in this order, each part 256-byte aligned:
// D [rows] fp32 | turn counters [B * Hq * ceil(Lq / 128) * 4] u32 + the
// ticket counter | dQ accumulator [rows * d] fp32, rows = the LSE rows
// (B * Hq * Lq, or Hq * total rows when packed).
struct BwdWorkspace {
  size_t d_off, turn_off, acc_off, total;
  int64_t n_turns;
};

inline BwdWorkspace bwd_workspace_plan(int64_t rows, int64_t B, int64_t Hq, int64_t Lq, int64_t d) {
  auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
  BwdWorkspace w;
  w.n_turns = B * Hq * ((Lq + kTile - 1) / kTile) * 4;
  w.d_off = 0;
  w.turn_off = r256(static_cast<size_t>(rows) * 4);
  w.acc_off = w.turn_off + r256(static_cast<size_t>(w.n_turns + 1) * 4);
  w.total = w.acc_off + r256(static_cast<size_t>(rows) * static_cast<size_t>(d) * 4);
  return w;
}

template <int D, int BIAS>
cudaError_t launch_bwd_t(const AttnParams& p, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mdo, uint32_t phases,
                         int64_t n_axis, int64_t n_turns, cudaStream_t st) {
  if (phases & kPhasePre) {
    const int64_t threads = std::max(n_axis * p.Hq * (D / 8), n_turns + 1);
    const int64_t blocks = (threads + 255) / 256;
    bwd_preprocess_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, st>>>(p, n_axis, n_turns);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (phases & kPhaseGrads) {
    using Lay = BwdLayout<D, BIAS>;
    auto kern = bwd_kernel<D, BIAS, false>;
    if constexpr (BIAS != kBiasNone) {
      if (p.ds_out) kern = bwd_kernel<D, BIAS, true>;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Lay::kSmemAlloc);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (or per work item, if fewer)
    const int64_t items = static_cast<int64_t>(p.B) * p.Hkv * ((p.Lk + kTile - 1) / kTile);
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    kern<<<static_cast<int>(items < sms ? items : sms), Lay::kThreads, Lay::kSmemAlloc, st>>>(
        p, mq, mk, mv, mdo);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int D>
cudaError_t launch_bwd_d(const AttnParams& p, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mdo, uint32_t phases,
                         int64_t n_axis, int64_t n_turns, cudaStream_t st) {
  switch (p.bias_kind) {
    case kBiasDense: return launch_bwd_t<D, kBiasDense>(p, mq, mk, mv, mdo, phases, n_axis, n_turns, st);
    case kBiasT5: return launch_bwd_t<D, kBiasT5>(p, mq, mk, mv, mdo, phases, n_axis, n_turns, st);
    default: return launch_bwd_t<D, kBiasNone>(p, mq, mk, mv, mdo, phases, n_axis, n_turns, st);
  }
}

}  // namespace sdpa
