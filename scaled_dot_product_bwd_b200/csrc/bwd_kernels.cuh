// bwd_kernels.cuh -- attention backward for sm_100a.
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
//   2. dQ: one CTA per SM walks (128 queries, query head, batch entry) items,
//      each over the 128-key tiles of its mask band in ascending order:
//        S = Q K^T, dP = dO V^T                 (SS MMAs, 128 x 128)
//        dS -> tensor memory (bf16), dQ += dS K (TS MMA, 128 x d)
//      with S double-buffered, so the next tile's scores are ready while
//      this tile's dS is formed.  The split-K sum over key tiles runs inside
//      one CTA's tensor memory, in tile order.
//   3. dK / dV: one CTA per (128 keys, KV head, batch entry) walks the
//      128-query tiles of the band for every query head of the group, in a
//      fixed order, and accumulates dV and dK in tensor memory:
//        S^T = K Q^T, dP^T = V dO^T             (SS MMAs, 128 x 128)
//        P^T, dS^T -> tensor memory (bf16)
//        dV += P^T dO, dK += dS^T Q             (TS MMAs, 128 x d)
// The dQ launch recomputes S and dP, 2 of the 7 MMAs of the pair: the price
// of summing dQ without atomics or a cross-CTA ordering protocol.  All score
// MMAs are 128 x 128 (an N = 64 MMA with both operands in shared memory is
// shared-memory-bandwidth bound on this part); the two compute warpgroups
// split every tile's 128 columns between them.  Rows of both sequences are
// addressed through the batch entry's SeqView, so cross-attention lengths
// and packed sequences take the same kernels.
#pragma once

#include "attn_common.cuh"
#include "exp2_poly.cuh"
#include "sm100.cuh"
#include "tmem_sync.cuh"

namespace sdpa {

// Share of a full tile's exponentials on MUFU (per 8 columns; 8 = all),
// chosen by measurement: at d = 128 without a bias the dK/dV kernel gains
// from moving 3 of 8 to the FMA pipe and the dQ kernel from none; with a
// relative-position bias (whose table adds FMA-pipe work per element) 2 of
// 8 in both (alibi_causal_4k dQ 0.955 -> 0.933 ms, dK/dV 1.244 -> 1.200);
// at d = 64, where the MMAs take half as long for the same exponentials, 2
// of 8 in both (t5rpe dQ 0.176 -> 0.168 ms, dK/dV 0.212 -> 0.208 ms).
template <int D, int BIAS>
constexpr int kDkdvMufuPer8 = (D == 64 || BIAS == kBiasT5) ? 6 : 5;
template <int D, int BIAS>
constexpr int kDqMufuPer8 = (D == 64 || BIAS == kBiasT5) ? 6 : 8;

// ------------------------------------------------------------ preprocess
// D = rowsum(dO * O) for every query row along the (padded or packed)
// sequence axis, D / 8 threads per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const AttnParams p, int64_t n_axis) {
  constexpr int kTpr = D / 8;  // threads per row, 8 bf16 (16 bytes) each
  const int64_t gt = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t nrows = n_axis * p.Hq;
  const int64_t r = gt / kTpr;
  const int part = static_cast<int>(gt % kTpr);
  float acc = 0.f;
  int h = 0;
  int64_t b = 0, i = 0;
  if (r < nrows) {
    h = static_cast<int>(r % p.Hq);
    const int64_t a = r / p.Hq;  // position along the sequence axis
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
  if (r < nrows && part == 0) p.dvec[b * p.lse_sb + h * p.lse_sh + i] = acc;
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

// ------------------------------------------------------------------ dK / dV
// CTA = 128 keys of one (KV head, batch entry).  Blocks of 128 queries
// stream through; both compute warpgroups work on every block, warpgroup w
// on the query columns [64 w, 64 w + 64).  Tensor memory (512 columns):
//   S^T 0..127 | dP^T 128..255 | dV 256.. | dK 256 + d..
// P^T (bf16) overwrites the first half of each warpgroup's S^T columns, dS^T
// the first half of its dP^T columns; the TS MMAs read them from there.
template <int D, int BIAS>
struct DkdvLayout {
  static constexpr int kTileBytes = kTile * D * 2;  // 128 rows x d bf16
  // A dense bias at d = 64 is staged by TMA: each block's 128 x 128 fp32
  // tile (64 KB) in a two-slot ring, loaded one block ahead, in place of
  // 64 scattered global loads per thread that the exponentials wait for.
  static constexpr bool kBiasTma = (BIAS == kBiasDense && D == 64);
  static constexpr int kBiasTileBytes = kTile * kTile * 4;
  static constexpr int kSB = kBiasTma ? 2 : 0;
  // Q blocks are used until the block's dK MMA, dO blocks only until its dV
  // MMA: the Q ring is the deeper one.  At d = 128 without a T5 table this
  // fills the 227 KB of shared memory to the last kilobyte; so does the
  // bias ring with two-slot Q and dO rings at d = 64.
  static constexpr int kSQ = (D == 128) ? (BIAS == kBiasT5 ? 2 : 3) : (kBiasTma ? 2 : 4);
  static constexpr int kSO = (D == 128) ? 2 : (kBiasTma ? 2 : 4);
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kQOff = 2 * kTileBytes;                  // Q ring
  static constexpr int kDOOff = kQOff + kSQ * kTileBytes;       // dO ring
  static constexpr int kBOff = kDOOff + kSO * kTileBytes;       // bias ring (kBiasTma), 1 KB aligned
  static constexpr int kVecOff = kBOff + kSB * kBiasTileBytes;  // 2 x (-lse2[128], D[128])
  static constexpr int kLutOff = kVecOff + 2 * 2 * kTile * 4;   // T5 only: 8 warps x 96 floats
  static constexpr int kLutBytes = (BIAS == kBiasT5) ? 8 * 96 * 4 : 0;
  static constexpr int kBarOff = kLutOff + kLutBytes;
  // kv_full, q_full[SQ], q_empty[SQ], o_full[SO], o_empty[SO], vec_full[2],
  // vec_empty[2], s_full[2], dp_full, p_full[2], ds_full, s_free[2], dp_free,
  // acc_done, drain[2], then with the bias ring b_full[2], b_empty[2]
  static constexpr int kNumBars = 1 + 2 * kSQ + 2 * kSO + 4 + 12 + (kBiasTma ? 4 : 0);
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemAlloc = kMiscOff + 16;
  // 2 compute warpgroups, producer, two MMA issuers
  static constexpr int kThreads = 352;
  static constexpr int kTmemCols = 512;
  static constexpr int kSCol = 0, kDPCol = 128, kDVCol = 256, kDKCol = 256 + D;
  // At d = 64, dV and dK take 128 columns: S^T gets a second buffer at 384,
  // so S^T(i + 1) is computed while the warpgroups work on block i instead
  // of waiting for dV(i) to read P^T(i) out of the one buffer.
  static constexpr bool kSDouble = (D == 64);
  static constexpr int kSCol1 = 384;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(kBOff % 1024 == 0, "128-byte swizzled TMA boxes start on 1 KB");
};


template <int D, int BIAS>
__global__ void __launch_bounds__(352, 1)
    bwd_dkdv_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmB) {
  using Lay = DkdvLayout<D, BIAS>;
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

  const int g = blockIdx.y;
  const int b = blockIdx.z;
  const int n0 = static_cast<int>(blockIdx.x) * kTile;  // causal: low key tiles are heaviest
  const SeqView s = seq_view(p, b);
  if (n0 >= s.Lk) return;  // past this entry's key sequence (packed, or a shorter one)
  const int Lq = s.Lq, Lk = s.Lk;
  int mlo, mhi;
  query_tile_range(p, Lq, Lk, n0, mlo, mhi);
  const int nm = mhi > mlo ? mhi - mlo : 0;
  const int total = nm * p.G;  // blocks: query head (outer) x query tile (inner)

  auto bar = [&](int idx) -> uint32_t { return sb + Lay::kBarOff + 8 * idx; };
  const uint32_t kv_full = bar(0);
  auto q_full = [&](int s) { return bar(1 + s); };
  auto q_empty = [&](int s) { return bar(1 + SQ + s); };
  auto o_full = [&](int s) { return bar(1 + 2 * SQ + s); };
  auto o_empty = [&](int s) { return bar(1 + 2 * SQ + SO + s); };
  constexpr int kB = 1 + 2 * SQ + 2 * SO;
  auto vec_full = [&](int x) { return bar(kB + x); };
  auto vec_empty = [&](int x) { return bar(kB + 2 + x); };
  // S^T ready, P^T ready, S^T buffer free: with two S^T buffers, block i's
  // on barrier i % 2 with parity (i / 2) % 2 (S^T(i + 1) is issued before
  // the wait for P^T(i), so the warpgroups may publish P^T(i + 1) first: one
  // barrier would then complete two phases and lose a wakeup); else one
  // barrier with parity i % 2
  constexpr bool SD = Lay::kSDouble;
  auto sb_of = [&](int i) { return SD ? (i & 1) : 0; };
  auto sb_par = [&](int i) { return static_cast<uint32_t>(SD ? ((i >> 1) & 1) : (i & 1)); };
  auto s_col = [&](int i) { return static_cast<uint32_t>(SD && (i & 1) ? Lay::kSCol1 : Lay::kSCol); };
  auto s_full = [&](int x) { return bar(kB + 4 + x); };
  const uint32_t dp_full = bar(kB + 6);
  auto p_full = [&](int x) { return bar(kB + 7 + x); };
  const uint32_t ds_full = bar(kB + 9);
  auto s_free = [&](int x) { return bar(kB + 10 + x); };
  const uint32_t dp_free = bar(kB + 12);
  const uint32_t acc_done = bar(kB + 13);
  auto drain = [&](int x) { return bar(kB + 14 + x); };
  constexpr bool BT = Lay::kBiasTma;
  auto b_full = [&](int x) { return bar(kB + 16 + x); };
  auto b_empty = [&](int x) { return bar(kB + 18 + x); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    if constexpr (BT) {
      for (int x = 0; x < 2; ++x) {
        mbar_init(b_full(x), 1);
        mbar_init(b_empty(x), 2 * kTile);  // both compute warpgroups
      }
    }
    // Q blocks are read by both issuers (S^T and dK), dO blocks too (dP^T and
    // dV): a slot is free once each issuer's last MMA on it has completed.
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
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(p_full(x), 2 * kTile);
      mbar_init(s_free(x), 1);
    }
    mbar_init(dp_full, 1);
    mbar_init(ds_full, 2 * kTile);
    mbar_init(dp_free, 1);
    mbar_init(acc_done, 2);
    mbar_init(drain(0), 1);
    mbar_init(drain(1), 1);
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
        mbar_expect_tx(kv_full, 2 * Lay::kTileBytes);
        for (int h = 0; h < D / 64; ++h) {
          tma_load_4d(sb + Lay::kKOff + h * kTile * 128, &tmK, kv_full, h * 64, s.k0 + n0, g, s.bc);
          tma_load_4d(sb + Lay::kVOff + h * kTile * 128, &tmV, kv_full, h * 64, s.k0 + n0, g, s.bc);
        }
      }
      // LSE and D of one block's 128 queries, four per lane, loaded one
      // block ahead of the slot they go to.  Nothing here uses the loaded
      // values (a use would hold the warp until they arrive): they are
      // converted where they are written, after the next block's copies
      // have been issued.
      float l2v[4], ddv[4];
      auto load_vec = [&](int it) {
        const int hq = g * p.G + it / nm;
        const int m0 = (mlo + it % nm) * kTile;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = m0 + lane + 32 * e;
          l2v[e] = -INFINITY;  // queries past the sequence: P = 0
          ddv[e] = 0.f;
          if (i < Lq) {
            const int64_t idx = row_index(p, s, b, hq, i);
            l2v[e] = p.lse[idx];
            ddv[e] = p.dvec[idx];
          }
        }
      };
      load_vec(0);
      int issued_q[SQ], issued_o[SO], issued_b[2] = {-1, -1};
      for (int e = 0; e < SQ; ++e) issued_q[e] = -1;
      for (int e = 0; e < SO; ++e) issued_o[e] = -1;
      bool ok = true;
      for (int it = 0; it < total; ++it) {
        const int hq = g * p.G + it / nm;
        const int m0 = (mlo + it % nm) * kTile;
        const int x = it & 1;
        // The copies go first: they wait only for their ring slots, not for
        // the LSE / D slot, so they run as far ahead as the rings allow.
        if (lane == 0) {
          const int sq = it % SQ, so = it % SO;
          if constexpr (BT) {
            // ahead of Q: its slot frees once the warpgroups have formed P of
            // the block two back, before that block's dK MMA frees Q's slot.
            // Rows m0.. (queries) and keys n0.. of (b, hq): 4 boxes of 32
            // keys; past either sequence the box reads zeros (those pairs
            // are masked)
            const uint32_t bph = (it >> 1) & 1;
            ok = mbar_wait(b_empty(x), bph ^ 1, ctl);
            if (ok) {
              mbar_expect_tx(b_full(x), Lay::kBiasTileBytes);
              const int hb = p.sb_h ? hq : 0, bb = p.sb_b ? b : 0;
              for (int q4 = 0; q4 < 4; ++q4)
                tma_load_4d(sb + Lay::kBOff + x * Lay::kBiasTileBytes + q4 * (kTile * 128), &tmB,
                            b_full(x), n0 + 32 * q4, m0, hb, bb);
              issued_b[x] = static_cast<int>(bph);
            }
          }
          if (ok) ok = mbar_wait(q_empty(sq), ((it / SQ) & 1) ^ 1, ctl);
          if (ok) {
            mbar_expect_tx(q_full(sq), Lay::kTileBytes);
            for (int h = 0; h < D / 64; ++h)
              tma_load_4d(sb + Lay::kQOff + sq * Lay::kTileBytes + h * kTile * 128, &tmQ,
                          q_full(sq), h * 64, s.q0 + m0, hq, s.bc);
            issued_q[sq] = (it / SQ) & 1;
            ok = mbar_wait(o_empty(so), ((it / SO) & 1) ^ 1, ctl);
          }
          if (ok) {
            mbar_expect_tx(o_full(so), Lay::kTileBytes);
            for (int h = 0; h < D / 64; ++h)
              tma_load_4d(sb + Lay::kDOOff + so * Lay::kTileBytes + h * kTile * 128, &tmDO,
                          o_full(so), h * 64, s.q0 + m0, hq, s.bc);
            issued_o[so] = (it / SO) & 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (ok) ok = mbar_wait(vec_empty(x), ((it >> 1) & 1) ^ 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        float* lse2 = vec + x * 2 * kTile;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // -LSE in log2 units; -inf (a row with no visible key, or past
          // the sequence) gives P = 0
          lse2[lane + 32 * e] = l2v[e] == -INFINITY ? -INFINITY : -l2v[e] * kLog2e;
          lse2[kTile + lane + 32 * e] = ddv[e];
        }
        mbar_arrive(vec_full(x));
        if (it + 1 < total) load_vec(it + 1);
      }
      if (!ok && lane == 0) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mbar_wait(kv_full, 0, ign);
        for (int e = 0; e < SQ; ++e)
          if (issued_q[e] >= 0) mbar_wait(q_full(e), issued_q[e], ign);
        for (int e = 0; e < SO; ++e)
          if (issued_o[e] >= 0) mbar_wait(o_full(e), issued_o[e], ign);
        for (int e = 0; e < 2; ++e)
          if (issued_b[e] >= 0) mbar_wait(b_full(e), issued_b[e], ign);
      }
    }
  } else if (warp == 9 || warp == 10) {
    // ===================== MMA issuers (one thread each) =====================
    // Warp 9 owns the S^T chain: S^T(i), then dV(i) once P^T(i) is ready, then
    // S^T(i+1) once dV(i) has read P^T(i) out of the S^T columns (at d = 64,
    // with two S^T buffers, S^T(i+1) goes before the wait for P^T(i) and
    // waits only for dV(i-1)).  Warp 10 owns
    // the dP^T chain: dP^T(i), dK(i) once dS^T(i) is ready, dP^T(i+1) once dK(i)
    // is done.  Neither waits on the other's barriers, so a stalled chain does
    // not hold up MMAs that are ready in the other.
    if (lane == 0 && total > 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTile, kTile, 0, 0);  // 128 keys x 128 queries
      constexpr uint32_t kIdG = idesc_bf16_f32(kTile, D, 0, 1);      // 128 keys x d
      const bool chain_s = (warp == 9);
      // Descriptors are built once: one at shared-memory offset 0 per layout,
      // plus the byte offset / 16 of each operand (the start-address field),
      // so an MMA costs the issuing thread two adds.  The issuer shares its
      // sub-partition with busy compute warps, so its instruction count is
      // what its issue rate is spent on.
      const uint64_t dk0 = smem_desc_sw128(sb, 16, 1024);            // K-major
      const uint64_t dmn0 = smem_desc_sw128(sb, kTile * 128, 1024);  // MN-major, 64-wide halves
      bool ok = issuer_wait(kv_full, 0, ctl);
      for (int it = 0; it < total && ok; ++it) {
        const int sq = it % SQ, so = it % SO;
        const uint64_t qm = dmn0 + ((Lay::kQOff + sq * Lay::kTileBytes) >> 4);
        const uint64_t od = dk0 + ((Lay::kDOOff + so * Lay::kTileBytes) >> 4);
        const uint64_t om = dmn0 + ((Lay::kDOOff + so * Lay::kTileBytes) >> 4);
        if (chain_s) {
          // S^T(j) = K Q(j)^T into its buffer, once Q(j) has landed and dV
          // has read P^T of the buffer's previous block
          auto issue_s = [&](int j) -> bool {
            const int sj = j % SQ;
            if (!issuer_wait(q_full(sj), (j / SQ) & 1, ctl)) return false;
            const int nbuf = SD ? 2 : 1;
            if (j >= nbuf && !issuer_wait(s_free(sb_of(j - nbuf)), sb_par(j - nbuf), ctl)) return false;
            tc_fence_after();
            const uint64_t qkj = dk0 + ((Lay::kQOff + sj * Lay::kTileBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + s_col(j), dk0 + ((Lay::kKOff + kmajor_koff(kk, kTile)) >> 4),
                     qkj + (kmajor_koff(kk, kTile) >> 4), kIdS, kk > 0 ? 1u : 0u);
            mma_commit(s_full(sb_of(j)));
            mma_commit(q_empty(sj));
            return true;
          };
          if (SD) {
            // S^T(it + 1) ahead of the wait for P^T(it)
            if (it == 0 && !(ok = issue_s(0))) break;
            if (it + 1 < total && !(ok = issue_s(it + 1))) break;
          } else {
            if (!(ok = issue_s(it))) break;
          }
          if (!(ok = issuer_wait(o_full(so), (it / SO) & 1, ctl))) break;
          if (!(ok = issuer_wait(p_full(sb_of(it)), sb_par(it), ctl))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts(tmem + Lay::kDVCol, split_a_col(tmem + s_col(it), kk), om + kk * (2048 >> 4),
                   kIdG, (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(s_free(sb_of(it)));
          mma_commit(o_empty(so));
        } else {
          if (!(ok = issuer_wait(o_full(so), (it / SO) & 1, ctl))) break;
          if (it > 0 && !(ok = issuer_wait(dp_free, (it - 1) & 1, ctl))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tmem + Lay::kDPCol, dk0 + ((Lay::kVOff + kmajor_koff(kk, kTile)) >> 4),
                   od + (kmajor_koff(kk, kTile) >> 4), kIdS, kk > 0 ? 1u : 0u);
          mma_commit(dp_full);
          mma_commit(o_empty(so));
          if (!(ok = issuer_wait(q_full(sq), (it / SQ) & 1, ctl))) break;
          if (!(ok = issuer_wait(ds_full, it & 1, ctl))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts(tmem + Lay::kDKCol, split_a_col(tmem + Lay::kDPCol, kk), qm + kk * (2048 >> 4),
                   kIdG,
                   (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(dp_free);
          mma_commit(q_empty(sq));
        }
      }
      if (ok) mma_commit(acc_done);
      if (!ok) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mma_commit(drain(chain_s ? 0 : 1));
        mbar_wait(drain(chain_s ? 0 : 1), 0, ign);
      }
    }
  } else {
    // ===== compute warpgroup wg: query columns [64 wg, 64 wg + 64); thread = key =====
    const int wg = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const int j = n0 + row;
    const int c0w = kBlk * wg;  // first query column of this warpgroup
    const uint32_t lane_bits = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS0 = tmem + lane_bits + c0w;  // + the block's S^T buffer column
    const uint32_t tDP = tmem + lane_bits + Lay::kDPCol + c0w;
    float* lut = reinterpret_cast<float*>(smem + Lay::kLutOff) + warp * 96;
    // Staged bias: this warp's keys are box warp % 4 of the block; query
    // column c is the box's row c0w + c, 128 bytes whose 16-byte chunks sit
    // at chunk ^ (row % 8) (128-byte swizzle).  The warp reads one whole row
    // per column: no bank conflicts.
    const uint8_t* bbox = smem + Lay::kBOff + (warp & 3) * (kTile * 128) + c0w * 128;
    uint32_t boff[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) boff[k] = (((lane >> 2) ^ k) << 4) | ((lane & 3) << 2);
    bool ok = true;
    for (int it = 0; it < total; ++it) {
      const int x = it & 1;
      const int hq = g * p.G + it / nm;
      const int m0 = (mlo + it % nm) * kTile + c0w;  // first query of this warpgroup
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
      if constexpr (BIAS == kBiasDense && !BT)
        bcol = p.bias + static_cast<int64_t>(b) * p.sb_b + static_cast<int64_t>(hq) * p.sb_h +
               static_cast<int64_t>(min(m0, Lq - 1)) * p.sb_i + min(j, Lk - 1);
      const uint8_t* bt = bbox + x * Lay::kBiasTileBytes;
      // bias of query column c (every column of the staged box is in range)
      auto bias_at = [&](int c, bool valid) -> float {
        if constexpr (BT) return *reinterpret_cast<const float*>(bt + c * 128 + boff[c & 7]);
        else return bcol[static_cast<int64_t>(valid ? c : 0) * p.sb_i];
      };
      if (ok) ok = mbar_wait(vec_full(x), (it >> 1) & 1, ctl);  // LSE / D staged
      const uint32_t tS = tS0 + s_col(it);
      if (ok) ok = mbar_wait(s_full(sb_of(it)), sb_par(it), ctl);
      if constexpr (BT) {
        if (ok) ok = mbar_wait(b_full(x), (it >> 1) & 1, ctl);
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
      const float* lse2 = vec + x * 2 * kTile + c0w;
      const float* dvv = vec + x * 2 * kTile + kTile + c0w;
      uint32_t pr[64];  // S^T row, then P^T (fp32 bits)
      tmem_ld64_sync(tS, pr);
      // in pairs of columns: packed fp32 pair instructions for the affine
      // step and the FMA-pipe exponentials (rounded as the scalar ones)
      const float4* lse4 = reinterpret_cast<const float4*>(lse2);  // -LSE, log2 units
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
      if (full) {
#pragma unroll
        for (int c4 = 0; c4 < kBlk / 4; ++c4) {
          const float4 l = lse4[c4];
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const int c = 4 * c4 + e;
            uint64_t x2 = f2_fma(f2_pack(__uint_as_float(pr[c]), __uint_as_float(pr[c + 1])), sc2,
                                 e ? f2_pack(l.z, l.w) : f2_pack(l.x, l.y));
            if constexpr (BIAS == kBiasT5) x2 = f2_add(x2, f2_pack(lut_row[-c], lut_row[-c - 1]));
            if constexpr (BIAS == kBiasDense)
              x2 = f2_fma(f2_pack(bias_at(c, true), bias_at(c + 1, true)), f2_pack(kLog2e, kLog2e), x2);
            float x0, x1, y0, y1;
            f2_unpack(x2, x0, x1);
            exp2_pair<BIAS, kDkdvMufuPer8<D, BIAS>>(c, x0, x1, y0, y1);
            pr[c] = __float_as_uint(y0);
            pr[c + 1] = __float_as_uint(y1);
          }
        }
      } else {
#pragma unroll
        for (int c4 = 0; c4 < kBlk / 4; ++c4) {
          const float4 l = lse4[c4];
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const int c = 4 * c4 + e;
            const bool v0 = (c >= lo) && (c <= hi), v1 = (c + 1 >= lo) && (c + 1 <= hi);
            uint64_t x2 = f2_fma(f2_pack(__uint_as_float(pr[c]), __uint_as_float(pr[c + 1])), sc2,
                                 e ? f2_pack(l.z, l.w) : f2_pack(l.x, l.y));
            if constexpr (BIAS == kBiasT5) x2 = f2_add(x2, f2_pack(lut_row[-c], lut_row[-c - 1]));
            if constexpr (BIAS == kBiasDense)
              x2 = f2_fma(f2_pack(bias_at(c, v0), bias_at(c + 1, v1)), f2_pack(kLog2e, kLog2e), x2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            pr[c] = __float_as_uint(fast_exp2(v0 ? x0 : -INFINITY));
            pr[c + 1] = __float_as_uint(fast_exp2(v1 ? x1 : -INFINITY));
          }
        }
      }
      if constexpr (BT) mbar_arrive(b_empty(x));  // the bias block is read
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
      mbar_arrive(p_full(sb_of(it)));
      if (ok) ok = mbar_wait(dp_full, it & 1, ctl);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) continue;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < kBlk; cc += 32) {
        uint32_t dr[32];
        tmem_ld32_sync(tDP + cc, dr);
        uint32_t pk[16];
        const float4* d4v = reinterpret_cast<const float4*>(dvv + cc);
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 dv4 = d4v[c >> 2];
          // dS = P (dP - D), two columns per instruction
          const uint64_t a2 = f2_mul(
              f2_pack(__uint_as_float(pr[cc + c]), __uint_as_float(pr[cc + c + 1])),
              f2_sub(f2_pack(__uint_as_float(dr[c]), __uint_as_float(dr[c + 1])), f2_pack(dv4.x, dv4.y)));
          const uint64_t b2 = f2_mul(
              f2_pack(__uint_as_float(pr[cc + c + 2]), __uint_as_float(pr[cc + c + 3])),
              f2_sub(f2_pack(__uint_as_float(dr[c + 2]), __uint_as_float(dr[c + 3])), f2_pack(dv4.z, dv4.w)));
          float d0, d1, d2, d3;
          f2_unpack(a2, d0, d1);
          f2_unpack(b2, d2, d3);
          pk[c >> 1] = pack_bf16x2(d0, d1);
          pk[(c >> 1) + 1] = pack_bf16x2(d2, d3);
        }
        tmem_st16(tDP + (cc >> 1), pk);  // dS^T over the first 32 of this warpgroup's columns
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ds_full);
      mbar_arrive(vec_empty(x));
    }
    // ---------------- epilogue: warpgroup 0 stores dV, warpgroup 1 stores dK ----------------
    if (ok && total > 0) ok = mbar_wait(acc_done, 0, ctl);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      // lanes 2m, 2m + 1 hold keys j, j + 1 and trade halves of every 16
      // columns, so each 16-byte store of the pair fills one 32-byte sector
      const bool odd = (lane & 1) != 0;
      const int ja = j - (odd ? 1 : 0);
      const int64_t off = static_cast<int64_t>(s.bc) * p.skv_b +
                          static_cast<int64_t>(s.k0 + ja) * p.skv_l +
                          static_cast<int64_t>(g) * p.skv_h + (odd ? 8 : 0);
      __nv_bfloat16* dst_a = (wg == 0 ? p.dv : p.dk) + off;
      __nv_bfloat16* dst_b = dst_a + p.skv_l;
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
// Persistent: one CTA per SM walks a heavy-first list of work items, each 128
// queries of one (query head, batch entry); blocks of 128 keys stream through;
// warpgroup w takes the key columns [64 w, 64 w + 64).  Ring, buffer and
// barrier indices count across items, so the next item's Q / dO load and
// first scores overlap the current item's last blocks and epilogue.  Tensor
// memory: S[0] 0..127 | S[1] 128..255 | dP 256..383 | dQ 384..  The scores
// are double-buffered, so S of block i + 1 is computed while block i's dS is
// formed.  dS (bf16) goes over the first half of each warpgroup's columns of
// its own, already loaded, S buffer: dP of block i + 1 can then be computed
// as soon as block i's dP has been loaded, and S of block i + 2 waits only
// for the dQ MMA of block i.
// DSM (what the kernel does with the fp32 dS besides the dQ MMA): 0 nothing,
// 1 store it (dense-bias gradient), 2 store its per-warp sums along the
// diagonals j - i, staged through shared memory (relative-position table
// gradient), 3 add those sums up per T5 bucket over the work item and store
// one sum per bucket and warp (T5 table gradient), 4 store each warp's sum
// of |j - i| dS (ALiBi slope gradient).
constexpr int kDsNone = 0, kDsStore = 1, kDsDiag = 2, kDsDiagT5 = 3, kDsMoment = 4;

template <int D, int BIAS, int DSM = kDsNone>
struct DqLayout {
  static constexpr int kTileBytes = kTile * D * 2;
  // Dense bias at d = 64: each block's 128 x 128 fp32 bias comes by TMA into
  // a 2-stage ring (4 boxes of 128 rows x 32 columns, 128-byte swizzle).
  static constexpr bool kBiasTma = (BIAS == kBiasDense && D == 64);
  static constexpr int kBiasTileBytes = kTile * kTile * 4;
  static constexpr int kSB = kBiasTma ? 2 : 0;
  // K blocks are used until the block's dQ MMA, V blocks only until its dP
  // MMA: the K ring is the deeper one.
  static constexpr int kSK = (D == 128) ? (BIAS == kBiasT5 ? 2 : 3) : (kBiasTma ? 2 : 4);
  // (at d = 128 the diagonal staging area takes the second V stage)
  static constexpr bool kStage = (DSM == kDsDiag || DSM == kDsDiagT5);
  static constexpr int kSV = (D == 128) ? (kStage ? 1 : 2) : (kBiasTma ? 2 : 3);
  static constexpr int kQOff = 0;
  static constexpr int kDOOff = kTileBytes;
  static constexpr int kKOff = 2 * kTileBytes;                // K ring
  static constexpr int kVOff = kKOff + kSK * kTileBytes;      // V ring
  static constexpr int kBOff = kVOff + kSV * kTileBytes;      // bias ring (kBiasTma)
  static constexpr int kLutOff = kBOff + kSB * kBiasTileBytes;  // T5 only: 8 warps x 96 floats
  static constexpr int kLutBytes = (BIAS == kBiasT5) ? 8 * 96 * 4 : 0;
  // diagonal sums: per warp, 32 rows x 32 keys of fp32 dS, row stride 33 floats
  static constexpr int kDiagOff = kLutOff + kLutBytes;
  static constexpr int kDiagBytes = kStage ? 8 * 32 * 33 * 4 : 0;
  // bucket mode: per warp, 128 per-bucket sums
  static constexpr int kBAccOff = kDiagOff + kDiagBytes;
  static constexpr int kBAccBytes = (DSM == kDsDiagT5) ? 8 * 128 * 4 : 0;
  static constexpr int kBarOff = kBAccOff + kBAccBytes;
  // q_full, k_full[SK], k_empty[SK], v_full[SV], v_empty[SV], s_full[2], dq_done[2],
  // dp_full, dp_used, ds_full[2], acc_done, drain[3], q_empty, o_full, o_empty,
  // b_full[2], b_empty[2]
  static constexpr int kNumBars = 1 + 2 * kSK + 2 * kSV + 19;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemAlloc = kMiscOff + 16;
  // 2 compute warpgroups, producer, MMA issuers: three (scores, dP, dQ),
  // or two (dP and dQ on one) for the diagonal-sum forms, whose warpgroups
  // stage dS in shared memory every block (measured: a third issuer made
  // those slower, every other form faster)
  static constexpr int kIssuers = (DSM == kDsDiag || DSM == kDsDiagT5) ? 2 : 3;
  static constexpr int kThreads = 288 + 32 * kIssuers;
  static constexpr int kTmemCols = 512;
  static constexpr int kDPCol = 256, kDQCol = 384;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

// DSM: see DqLayout (the bias-gradient paths).
template <int D, int BIAS, int DSM = kDsNone>
__global__ void __launch_bounds__(DqLayout<D, BIAS, DSM>::kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmB) {
  using Lay = DqLayout<D, BIAS, DSM>;
  constexpr int SK = Lay::kSK;
  constexpr int SV = Lay::kSV;
  extern __shared__ uint8_t smem[];
  if (!smem_base_ok(smem)) {
    if (threadIdx.x == 0) atomicOr(&g_device_status, kStatusMisaligned);
    return;
  }
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work items: (query tile, head, batch), heaviest causal query tiles
  // first; consecutive items are neighbouring heads, which share K / V in L2.
  const int nqt = (p.Lq + kTile - 1) / kTile;
  const int heads = p.Hq * p.B;
  const int n_items = nqt * heads;
  struct Item {
    int m0, hq, b, g, nlo, nt;
    bool rows;  // the query tile holds queries of the sequence
    SeqView s;
  };
  auto item_at = [&](int id) {
    Item w;
    const int r = id / heads;
    const int rem = id - r * heads;
    const int qt = p.causal ? nqt - 1 - r : r;
    w.m0 = qt * kTile;
    w.hq = rem % p.Hq;
    w.b = rem / p.Hq;
    w.g = w.hq / p.G;
    w.s = seq_view(p, w.b);
    w.rows = w.m0 < w.s.Lq;
    w.nlo = 0;
    w.nt = 0;
    if (w.rows) {
      int nhi;
      key_tile_range(p, w.s.Lq, w.s.Lk, w.m0, kTile, w.nlo, nhi);
      w.nt = nhi > w.nlo ? nhi - w.nlo : 0;
    }
    return w;
  };

  auto bar = [&](int idx) -> uint32_t { return sb + Lay::kBarOff + 8 * idx; };
  const uint32_t q_full = bar(0);
  auto k_full = [&](int s) { return bar(1 + s); };
  auto k_empty = [&](int s) { return bar(1 + SK + s); };
  auto v_full = [&](int s) { return bar(1 + 2 * SK + s); };
  auto v_empty = [&](int s) { return bar(1 + 2 * SK + SV + s); };
  constexpr int kB = 1 + 2 * SK + 2 * SV;
  auto s_full = [&](int x) { return bar(kB + x); };
  auto dq_done = [&](int x) { return bar(kB + 2 + x); };  // dQ MMA of a block in buffer x done
  const uint32_t dp_full = bar(kB + 4);
  const uint32_t dp_used = bar(kB + 5);
  // dS of block i ready, by block parity: the warpgroups can finish dS(i + 1)
  // (dP(i + 1) does not wait for the dQ MMAs) before the dQ issuer looks for
  // dS(i); a single barrier would then have completed two phases and the
  // wait for block i's parity would never succeed.
  auto ds_full = [&](int x) { return x == 0 ? bar(kB + 6) : bar(kB + 13); };
  const uint32_t acc_done = bar(kB + 7);
  auto drain = [&](int x) { return x < 2 ? bar(kB + 8 + x) : bar(kB + 18); };
  // Q is read only by the score issuer, dO only by the dP issuer: each tile is
  // released as soon as its one reader is done with the item
  const uint32_t q_empty = bar(kB + 10);
  const uint32_t o_full = bar(kB + 11);
  const uint32_t o_empty = bar(kB + 12);
  auto b_full = [&](int x) { return bar(kB + 14 + x); };
  auto b_empty = [&](int x) { return bar(kB + 16 + x); };
  constexpr bool BT = Lay::kBiasTma;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(b_full(x), 1);
      mbar_init(b_empty(x), 2 * kTile);
    }
    // K blocks are read by both issuers (S and dQ): a slot is free once each
    // issuer's last MMA on it has completed.
    for (int s = 0; s < SK; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 2);
    }
    for (int s = 0; s < SV; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(dq_done(x), 1);
    }
    mbar_init(dp_full, 1);
    mbar_init(dp_used, 2 * kTile);
    mbar_init(ds_full(0), 2 * kTile);
    mbar_init(ds_full(1), 2 * kTile);
    mbar_init(acc_done, 1);
    mbar_init(drain(0), 1);
    mbar_init(drain(1), 1);
    mbar_init(drain(2), 1);
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
    // Per item: Q and dO once (each after its reader is done with the
    // previous item's), then K and V of every key block into their rings.
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmDO);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued_k[SK], issued_v[SV];
      for (int s = 0; s < SK; ++s) issued_k[s] = -1;
      for (int s = 0; s < SV; ++s) issued_v[s] = -1;
      int q_issued = -1, o_issued = -1;
      int b_issued[2] = {-1, -1};
      int c = 0;  // key blocks so far, over all items
      int u = 0;  // items with a non-empty band so far
      bool ok = true;
      for (int id = blockIdx.x; id < n_items && ok; id += gridDim.x) {
        const Item w = item_at(id);
        if (w.nt == 0) continue;
        if (u > 0 && !(ok = mbar_wait(q_empty, (u - 1) & 1, ctl))) break;
        mbar_expect_tx(q_full, Lay::kTileBytes);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(sb + Lay::kQOff + h * kTile * 128, &tmQ, q_full, h * 64, w.s.q0 + w.m0,
                      w.hq, w.s.bc);
        q_issued = u & 1;
        if (u > 0 && !(ok = mbar_wait(o_empty, (u - 1) & 1, ctl))) break;
        mbar_expect_tx(o_full, Lay::kTileBytes);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(sb + Lay::kDOOff + h * kTile * 128, &tmDO, o_full, h * 64, w.s.q0 + w.m0,
                      w.hq, w.s.bc);
        o_issued = u & 1;
        for (int it = 0; it < w.nt; ++it, ++c) {
          const int sk = c % SK, sv = c % SV;
          const int n0 = (w.nlo + it) * kTile;
          if constexpr (BT) {
            // this block's bias: rows m0.., keys n0.. of (b, hq), 4 boxes.
            // Ahead of K: its slot frees once the warpgroups have formed P
            // of the block two back, K's only after that block's dQ MMA.
            const int x = c & 1;
            const uint32_t bph = (c >> 1) & 1;
            if (!(ok = mbar_wait(b_empty(x), bph ^ 1, ctl))) break;
            mbar_expect_tx(b_full(x), Lay::kBiasTileBytes);
            const int hb = p.sb_h ? w.hq : 0, bb = p.sb_b ? w.b : 0;
            for (int q4 = 0; q4 < 4; ++q4)
              tma_load_4d(sb + Lay::kBOff + x * Lay::kBiasTileBytes + q4 * (kTile * 128), &tmB,
                          b_full(x), n0 + 32 * q4, w.m0, hb, bb);
            b_issued[x] = static_cast<int>(bph);
          }
          if (!(ok = mbar_wait(k_empty(sk), ((c / SK) & 1) ^ 1, ctl))) break;
          mbar_expect_tx(k_full(sk), Lay::kTileBytes);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(sb + Lay::kKOff + sk * Lay::kTileBytes + h * kTile * 128, &tmK,
                        k_full(sk), h * 64, w.s.k0 + n0, w.g, w.s.bc);
          issued_k[sk] = (c / SK) & 1;
          if constexpr (BIAS == kBiasDense && !BT) prefetch_bias_tile(p, w.b, w.hq, w.m0, n0);
          if (!(ok = mbar_wait(v_empty(sv), ((c / SV) & 1) ^ 1, ctl))) break;
          mbar_expect_tx(v_full(sv), Lay::kTileBytes);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(sb + Lay::kVOff + sv * Lay::kTileBytes + h * kTile * 128, &tmV,
                        v_full(sv), h * 64, w.s.k0 + n0, w.g, w.s.bc);
          issued_v[sv] = (c / SV) & 1;
        }
        ++u;
      }
      if (!ok) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        if (q_issued >= 0) mbar_wait(q_full, q_issued, ign);
        if (o_issued >= 0) mbar_wait(o_full, o_issued, ign);
        for (int x = 0; x < 2; ++x)
          if (b_issued[x] >= 0) mbar_wait(b_full(x), b_issued[x], ign);
        for (int s = 0; s < SK; ++s)
          if (issued_k[s] >= 0) mbar_wait(k_full(s), issued_k[s], ign);
        for (int s = 0; s < SV; ++s)
          if (issued_v[s] >= 0) mbar_wait(v_full(s), issued_v[s], ign);
      }
    }
  } else if (Lay::kIssuers == 3 && warp >= 9 && warp <= 11) {
    // ===================== MMA issuers (one thread each) =====================
    // Warp 9 runs the score chain: S(i) into buffer i % 2 once K(i) has landed
    // and the dQ MMA of block i - 2 has read dS out of that buffer.  Warp 10
    // runs the dP chain: dP(i + 1) as soon as both warpgroups have loaded
    // dP(i).  Warp 11 issues dQ(i) += dS(i) K(i) as soon as dS(i) is ready.
    // With dP and dQ on one thread, dQ(i) waited behind the issue of
    // dP(i + 1) (~1300 cycles on the mistral-shaped workload) and S(i + 2)
    // behind dQ(i).  Block indices run on across items.
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTile, kTile, 0, 0);  // 128 queries x 128 keys
      constexpr uint32_t kIdQ = idesc_bf16_f32(kTile, D, 0, 1);      // 128 queries x d
      const int role = warp - 9;  // 0 scores, 1 dP, 2 dQ
      // descriptors built once, plus byte offset / 16 per operand (see the
      // dK/dV kernel's issuers)
      const uint64_t dk0 = smem_desc_sw128(sb, 16, 1024);            // K-major
      const uint64_t dmn0 = smem_desc_sw128(sb, kTile * 128, 1024);  // MN-major, 64-wide halves
      int c = 0;  // key blocks so far, over all items
      int u = 0;  // items with a non-empty band so far
      bool ok = true;
      for (int id = blockIdx.x; id < n_items && ok; id += gridDim.x) {
        const Item w = item_at(id);
        if (w.nt == 0) continue;
        if (role == 0 && !(ok = issuer_wait(q_full, u & 1, ctl))) break;
        if (role == 1 && !(ok = issuer_wait(o_full, u & 1, ctl))) break;
        for (int it = 0; it < w.nt; ++it, ++c) {
          const int x = c & 1;
          const int sk = c % SK;
          if (role == 0) {
            if (!(ok = issuer_wait(k_full(sk), (c / SK) & 1, ctl))) break;
            if (c >= 2 && !(ok = issuer_wait(dq_done(x), ((c >> 1) - 1) & 1, ctl))) break;
            tc_fence_after();
            const uint64_t kd = dk0 + ((Lay::kKOff + sk * Lay::kTileBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + kTile * x, dk0 + ((Lay::kQOff + kmajor_koff(kk, kTile)) >> 4),
                     kd + (kmajor_koff(kk, kTile) >> 4), kIdS,
                     kk > 0 ? 1u : 0u);
            mma_commit(s_full(x));
            mma_commit(k_empty(sk));
          } else if (role == 1) {
            const int sv = c % SV;
            if (!(ok = issuer_wait(v_full(sv), (c / SV) & 1, ctl))) break;
            if (c > 0 && !(ok = issuer_wait(dp_used, (c - 1) & 1, ctl))) break;
            tc_fence_after();
            const uint64_t vd = dk0 + ((Lay::kVOff + sv * Lay::kTileBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + Lay::kDPCol, dk0 + ((Lay::kDOOff + kmajor_koff(kk, kTile)) >> 4),
                     vd + (kmajor_koff(kk, kTile) >> 4), kIdS, kk > 0 ? 1u : 0u);
            mma_commit(dp_full);
            mma_commit(v_empty(sv));
          } else {
            if (!(ok = issuer_wait(k_full(sk), (c / SK) & 1, ctl))) break;
            if (!(ok = issuer_wait(ds_full(c & 1), (c >> 1) & 1, ctl))) break;
            tc_fence_after();
            const uint64_t kmd = dmn0 + ((Lay::kKOff + sk * Lay::kTileBytes) >> 4);
            // the item's first dQ MMA overwrites the accumulator: every
            // warpgroup thread read the previous item's dQ before marking dS ready
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              mma_ts(tmem + Lay::kDQCol, split_a_col(tmem + kTile * x, kk), kmd + kk * (2048 >> 4),
                     kIdQ,
                     (it > 0 || kk > 0) ? 1u : 0u);
            mma_commit(dq_done(x));
            mma_commit(k_empty(sk));
          }
        }
        if (!ok) break;
        if (role == 0) mma_commit(q_empty);   // the item's Q is read
        if (role == 1) mma_commit(o_empty);   // the item's dO is read
        if (role == 2) mma_commit(acc_done);  // the item's dQ is complete
        ++u;
      }
      if (!ok) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mma_commit(drain(role));
        mbar_wait(drain(role), 0, ign);
      }
    }
  } else if (Lay::kIssuers == 2 && (warp == 9 || warp == 10)) {
    // ================ MMA issuers, bias-gradient forms (two threads) ================
    // Warp 9 runs the score chain as above.  Warp 10 runs dP one block ahead
    // of dQ within an item: dP(i + 1) as soon as both warpgroups have loaded
    // dP(i), then dQ(i) once dS(i) is ready.  (A third issuer made these
    // diagonal-sum forms slower: their warpgroups' extra work per block,
    // not the dQ issue, bounds them.)
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTile, kTile, 0, 0);  // 128 queries x 128 keys
      constexpr uint32_t kIdQ = idesc_bf16_f32(kTile, D, 0, 1);      // 128 queries x d
      const bool chain_s = (warp == 9);
      // descriptors built once, plus byte offset / 16 per operand (see the
      // dK/dV kernel's issuers)
      const uint64_t dk0 = smem_desc_sw128(sb, 16, 1024);            // K-major
      const uint64_t dmn0 = smem_desc_sw128(sb, kTile * 128, 1024);  // MN-major, 64-wide halves
      auto issue_dp = [&](int c) -> bool {
        const int sv = c % SV;
        if (!issuer_wait(v_full(sv), (c / SV) & 1, ctl)) return false;
        if (c > 0 && !issuer_wait(dp_used, (c - 1) & 1, ctl)) return false;
        tc_fence_after();
        const uint64_t vd = dk0 + ((Lay::kVOff + sv * Lay::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + Lay::kDPCol, dk0 + ((Lay::kDOOff + kmajor_koff(kk, kTile)) >> 4),
                 vd + (kmajor_koff(kk, kTile) >> 4), kIdS, kk > 0 ? 1u : 0u);
        mma_commit(dp_full);
        mma_commit(v_empty(sv));
        return true;
      };
      int c = 0;  // key blocks so far, over all items
      int u = 0;  // items with a non-empty band so far
      bool ok = true;
      for (int id = blockIdx.x; id < n_items && ok; id += gridDim.x) {
        const Item w = item_at(id);
        if (w.nt == 0) continue;
        if (!(ok = issuer_wait(chain_s ? q_full : o_full, u & 1, ctl))) break;
        if (!chain_s && !(ok = issue_dp(c))) break;
        for (int it = 0; it < w.nt; ++it, ++c) {
          const int x = c & 1;
          const int sk = c % SK;
          const uint64_t kd = dk0 + ((Lay::kKOff + sk * Lay::kTileBytes) >> 4);
          const uint64_t kmd = dmn0 + ((Lay::kKOff + sk * Lay::kTileBytes) >> 4);
          if (chain_s) {
            if (!(ok = issuer_wait(k_full(sk), (c / SK) & 1, ctl))) break;
            if (c >= 2 && !(ok = issuer_wait(dq_done(x), ((c >> 1) - 1) & 1, ctl))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + kTile * x, dk0 + ((Lay::kQOff + kmajor_koff(kk, kTile)) >> 4),
                     kd + (kmajor_koff(kk, kTile) >> 4), kIdS,
                     kk > 0 ? 1u : 0u);
            mma_commit(s_full(x));
            mma_commit(k_empty(sk));
          } else {
            if (it + 1 < w.nt && !(ok = issue_dp(c + 1))) break;
            if (!(ok = issuer_wait(k_full(sk), (c / SK) & 1, ctl))) break;
            if (!(ok = issuer_wait(ds_full(c & 1), (c >> 1) & 1, ctl))) break;
            tc_fence_after();
            // the item's first dQ MMA overwrites the accumulator: every
            // warpgroup thread read the previous item's dQ before marking dS ready
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              mma_ts(tmem + Lay::kDQCol, split_a_col(tmem + kTile * x, kk), kmd + kk * (2048 >> 4),
                     kIdQ,
                     (it > 0 || kk > 0) ? 1u : 0u);
            mma_commit(dq_done(x));
            mma_commit(k_empty(sk));
          }
        }
        if (!ok) break;
        mma_commit(chain_s ? q_empty : o_empty);  // the item's Q / dO is read
        if (!chain_s) mma_commit(acc_done);
        ++u;
      }
      if (!ok) {
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mma_commit(drain(chain_s ? 0 : 1));
        mbar_wait(drain(chain_s ? 0 : 1), 0, ign);
      }
    }
  } else {
    // ===== compute warpgroup wg: key columns [64 wg, 64 wg + 64); thread = query row =====
    const int wg = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const int c0w = kBlk * wg;
    const uint32_t lane_bits = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tDP = tmem + lane_bits + Lay::kDPCol + c0w;
    float* lut = reinterpret_cast<float*>(smem + Lay::kLutOff) + warp * 96;
    // Bucket mode: lane l's buckets l, l + 32, ... and their distance ranges,
    // read from the parameters once (lanes reading different entries of a
    // parameter array are served one address at a time); a bucket past the
    // table's count gets an empty range.
    int rlo[4], rhi[4];
    if constexpr (DSM == kDsDiagT5) {
      // this warp's per-bucket sums; entry k is only ever touched by lane k % 32
      float* bacc = reinterpret_cast<float*>(smem + Lay::kBAccOff) + warp * 128;
      for (int k = lane; k < 128; k += 32) bacc[k] = 0.f;
      const int nbk = p.t5.bidirectional ? 2 * p.t5.half : p.t5.half;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = lane + 32 * q;
        rlo[q] = k < nbk ? p.t5r.lo[k] : (1 << 29);
        rhi[q] = k < nbk ? p.t5r.hi[k] : -(1 << 29);
      }
    }
    bool ok = true;
    int c = 0;  // key blocks so far, over all items
    int u = 0;  // items with a non-empty band so far
    for (int id = blockIdx.x; id < n_items; id += gridDim.x) {
      const Item w = item_at(id);
      if (!w.rows) continue;  // past this entry's query sequence: nothing to write
      const int m0 = w.m0, hq = w.hq, b = w.b, nt = w.nt;
      const int Lq = w.s.Lq, Lk = w.s.Lk;
      // every key of the warpgroup's 64 from n0 is visible from all 128 rows
      auto dq_tile_full = [&](int n0) {
        bool f = n0 + kBlk <= Lk;
        if (p.causal) f = f && (n0 + kBlk - 1 <= m0);
        if (p.wl >= 0) f = f && (n0 >= m0 + kTile - 1 - p.wl);
        if (p.wr >= 0) f = f && (n0 + kBlk - 1 <= m0 + p.wr);
        return f;
      };
      const int i = m0 + row;
      float l2 = INFINITY, dd = 0.f;
      if (i < Lq) {
        const int64_t idx = row_index(p, w.s, b, hq, i);
        l2 = p.lse[idx] * kLog2e;
        dd = p.dvec[idx];
        if (l2 == -INFINITY) l2 = INFINITY;
      }
      const float* brow = nullptr;
      if constexpr (BIAS == kBiasDense)
        brow = p.bias + static_cast<int64_t>(b) * p.sb_b + static_cast<int64_t>(hq) * p.sb_h +
               static_cast<int64_t>(min(i, Lq - 1)) * p.sb_i;
      // bucket mode: this row's sums of the halves inside the capped bucket
      // of keys before / after the query (or bucket 0 of a unidirectional table)
      float one_lo = 0.f, one_hi = 0.f;
      for (int it = 0; it < nt; ++it, ++c) {
        const int x = c & 1;
        const int n0 = (w.nlo + it) * kTile + c0w;  // first key of this warpgroup
        const float* lut_row = nullptr;
        bool one_b = false;  // the warp's piece lies in one T5 bucket: bias ub throughout
        float ub = 0.f;
        if constexpr (BIAS == kBiasT5) {
          // this warp's queries iw..iw+31 and keys n0..n0+63: j - i = (n0 - iw - 31) + e,
          // e in [0, 94]; the thread reads entry 31 - lane + cc for column cc
          const int base = n0 - m0 - (warp & 3) * 32 - 31;
          one_b = dq_tile_full(n0) && t5_one_bucket(p, base, 32 + kBlk - 2, hq, ub);
          if (!one_b) {
            __syncwarp();
            for (int e = lane; e < 32 + kBlk - 1; e += 32) lut[e] = rel_bias_log2(p, base + e, hq);
            __syncwarp();
          }
          lut_row = lut + 31 - lane;
        }
        int lo = 0, hi = kBlk - 1;
        const bool full = dq_tile_full(n0);
        if (!full) {
          if (p.wl >= 0) lo = max(lo, i - p.wl - n0);
          hi = min(hi, Lk - 1 - n0);
          if (p.causal) hi = min(hi, i - n0);
          if (p.wr >= 0) hi = min(hi, i + p.wr - n0);
        }
        if (ok) ok = mbar_wait(s_full(x), (c >> 1) & 1, ctl);
        if constexpr (BT) {
          if (ok) ok = mbar_wait(b_full(c & 1), (c >> 1) & 1, ctl);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) continue;
        tc_fence_after();
        const uint32_t tSx = tmem + lane_bits + kTile * x + c0w;
        uint32_t pr[64];  // S row, then P (fp32 bits)
        tmem_ld64_sync(tSx, pr);
        if constexpr (BT) {
          // this warpgroup's 64 bias columns from the staged block: boxes
          // 2 wg and 2 wg + 1, row `row`, 8 swizzled 16-byte chunks each
          const uint8_t* bt = smem + Lay::kBOff + (c & 1) * Lay::kBiasTileBytes;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint8_t* brw = bt + (2 * wg + h) * (kTile * 128) + row * 128;
#pragma unroll
            for (int k4 = 0; k4 < 8; ++k4) {
              const float4 b4 = *reinterpret_cast<const float4*>(brw + ((k4 ^ (row & 7)) << 4));
              const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int cc = 32 * h + 4 * k4 + e;
                const float xv = fmaf(bv[e], kLog2e, fmaf(__uint_as_float(pr[cc]), p.scale_log2, -l2));
                pr[cc] = __float_as_uint(fast_exp2(full || (cc >= lo && cc <= hi) ? xv : -INFINITY));
              }
            }
          }
          mbar_arrive(b_empty(c & 1));  // the bias block is read
        } else if (full && BIAS == kBiasDense) {
          // the row's 64 bias values as 16-byte loads, 32 at a time
          const float4* b4 = reinterpret_cast<const float4*>(brow + n0);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float4 bb[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) bb[q] = b4[8 * h + q];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float bv[4] = {bb[q].x, bb[q].y, bb[q].z, bb[q].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int cc = 32 * h + 4 * q + e;
                const float xv = fmaf(bv[e], kLog2e, fmaf(__uint_as_float(pr[cc]), p.scale_log2, -l2));
                pr[cc] = __float_as_uint(fast_exp2(xv));
              }
            }
          }
        } else if (full) {
          // in pairs of columns: packed fp32 pair instructions for the
          // affine step and the FMA-pipe exponentials (rounded as the scalar
          // ones); a one-bucket T5 bias is folded into the row constant
          const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
          auto exp_full = [&](auto table) {
            const float nl = one_b ? ub - l2 : -l2;
            const uint64_t nl2 = f2_pack(nl, nl);
#pragma unroll
            for (int cc = 0; cc < kBlk; cc += 2) {
              uint64_t x2 = f2_fma(f2_pack(__uint_as_float(pr[cc]), __uint_as_float(pr[cc + 1])), sc2, nl2);
              if constexpr (decltype(table)::value) x2 = f2_add(x2, f2_pack(lut_row[cc], lut_row[cc + 1]));
              float x0, x1, y0, y1;
              f2_unpack(x2, x0, x1);
              exp2_pair<BIAS, kDqMufuPer8<D, BIAS>>(cc, x0, x1, y0, y1);
              pr[cc] = __float_as_uint(y0);
              pr[cc + 1] = __float_as_uint(y1);
            }
          };
          if (BIAS == kBiasT5 && !one_b)
            exp_full(Flag<true>{});
          else
            exp_full(Flag<false>{});
        } else {
#pragma unroll
          for (int cc = 0; cc < kBlk; ++cc) {
            const bool vis = (cc >= lo) && (cc <= hi);
            float xv = fmaf(__uint_as_float(pr[cc]), p.scale_log2, -l2);
            if constexpr (BIAS == kBiasT5) xv += lut_row[cc];
            if constexpr (BIAS == kBiasDense) xv += vis ? brow[n0 + cc] * kLog2e : 0.f;
            pr[cc] = __float_as_uint(fast_exp2(vis ? xv : -INFINITY));
          }
        }
        if (ok) ok = mbar_wait(dp_full, c & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) continue;
        tc_fence_after();
        uint32_t pk[32];  // dS as bf16 pairs
#pragma unroll
        for (int cc = 0; cc < kBlk; cc += 32) {
          uint32_t dr[32];
          tmem_ld32_sync(tDP + cc, dr);
          if (cc + 32 == kBlk) {
            tc_fence_before();
            mbar_arrive(dp_used);  // the dP columns may now take the next block
          }
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            // dS = P (dP - D), two columns per instruction
            const uint64_t d2 = f2_mul(
                f2_pack(__uint_as_float(pr[cc + e]), __uint_as_float(pr[cc + e + 1])),
                f2_sub(f2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])), f2_pack(dd, dd)));
            float d0, d1;
            f2_unpack(d2, d0, d1);
            pk[(cc + e) >> 1] = pack_bf16x2(d0, d1);
            if constexpr (DSM != kDsNone) {  // P is spent: keep the fp32 dS in its place
              pr[cc + e] = __float_as_uint(d0);
              pr[cc + e + 1] = __float_as_uint(d1);
            }
          }
        }
        // dS over the first 32 of this warpgroup's columns of its S buffer
        tmem_st16(tSx, *reinterpret_cast<const uint32_t(*)[16]>(pk));
        tmem_st16(tSx + 16, *reinterpret_cast<const uint32_t(*)[16]>(pk + 16));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(ds_full(c & 1));
        if constexpr (DSM == kDsMoment) {
          // sum over this warp's 32 rows x 64 keys of |j - i| dS (distances
          // are exact in fp32); one value per (batch, head, query tile, key
          // tile, warp)
          const float t0 = static_cast<float>(n0 - i);
          float m4[4] = {0.f, 0.f, 0.f, 0.f};  // four chains: columns c % 4
#pragma unroll
          for (int cc = 0; cc < kBlk; ++cc)
            m4[cc & 3] = fmaf(fabsf(t0 + static_cast<float>(cc)), __uint_as_float(pr[cc]), m4[cc & 3]);
          float mom = (m4[0] + m4[1]) + (m4[2] + m4[3]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mom += __shfl_xor_sync(0xffffffffu, mom, o);
          const int ntk = (p.Lk + kTile - 1) / kTile;
          if (lane == 0)
            p.diag_out[(((static_cast<int64_t>(b) * p.Hq + hq) * nqt + m0 / kTile) * ntk +
                        (n0 - c0w) / kTile) * 8 + warp] = mom;
        }
        if constexpr (DSM == kDsDiag || DSM == kDsDiagT5) {
          // Sums of this warp's 32 rows x 64 keys of dS along the diagonals,
          // in two halves of 32 keys: each half is staged row by row
          // (stride 33 floats: conflict-free both ways), then lane l adds up
          // the diagonal t = c - r = l - 31 (rows 31 - l..31) and, for
          // l < 31, t = l + 1 (rows 0..30 - l), one element per step, so a
          // step's 32 reads hit 32 banks.  In absolute terms t is the
          // distance j - i = n0 + 32 h - (m0 + 32 (warp % 4)) + t.
          // Diagonal mode: per (batch, head, query tile, key tile), 8 warps
          // x 2 halves x 64 floats (t + 31 at 0..62 for t <= 0, 32 + t - 1
          // for t >= 1).  Bucket mode (T5 table): the 63 sums go to this
          // warp's per-bucket accumulators in shared memory instead, lane k
          // adding those of bucket k (and k + 32, ...), whose distances form
          // one range [t5r.lo[k], t5r.hi[k]], as a difference of two prefix
          // sums over the half's diagonals; a half whose distances all lie
          // in the capped bucket of a side, or all at j >= i of a
          // unidirectional table (bucket 0), skips the staging: each row
          // adds its 32 values to a register sum for that bucket, which the
          // warp reduces once per work item (most halves away from the
          // diagonal are such).
          float* stg = reinterpret_cast<float*>(smem + Lay::kDiagOff) + warp * (32 * 33);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int t0 = n0 + 32 * h - m0 - (warp & 3) * 32;  // distance j - i at t = 0
            bool one_bucket = false;
            if constexpr (DSM == kDsDiagT5)
              one_bucket = t0 + 31 <= p.t5.one_lo_max || t0 - 31 >= p.t5.one_hi_min;
            float s1 = 0.f, s2 = 0.f;
            if (one_bucket) {
              // the row's 32 values as a pairwise tree of packed fp32 pair
              // additions, into the side's register sum (reduced over the
              // warp once per item)
              uint64_t v[8];
#pragma unroll
              for (int q = 0; q < 8; ++q)
                v[q] = f2_add(f2_pack(__uint_as_float(pr[32 * h + 4 * q]), __uint_as_float(pr[32 * h + 4 * q + 1])),
                              f2_pack(__uint_as_float(pr[32 * h + 4 * q + 2]), __uint_as_float(pr[32 * h + 4 * q + 3])));
#pragma unroll
              for (int w2 = 4; w2 > 0; w2 >>= 1)
#pragma unroll
                for (int q = 0; q < w2; ++q) v[q] = f2_add(v[2 * q], v[2 * q + 1]);
              float va, vb;
              f2_unpack(v[0], va, vb);
              if (t0 + 31 <= p.t5.one_lo_max)
                one_lo += va + vb;
              else
                one_hi += va + vb;
              continue;
            } else {
              __syncwarp();
#pragma unroll
              for (int cc = 0; cc < 32; ++cc) stg[lane * 33 + cc] = __uint_as_float(pr[32 * h + cc]);
              __syncwarp();
              // two chains per sum (even and odd steps), added at the end
              float s1b = 0.f, s2b = 0.f;
#pragma unroll
              for (int k = 0; k < 32; k += 2) {
                const bool f0 = k <= lane, f1 = k + 1 <= lane;
                const float v0 = stg[(f0 ? 31 - lane + k : k - lane - 1) * 33 + k];
                const float v1 = stg[(f1 ? 32 - lane + k : k - lane) * 33 + k + 1];
                s1 += f0 ? v0 : 0.f;
                s2 += f0 ? 0.f : v0;
                s1b += f1 ? v1 : 0.f;
                s2b += f1 ? 0.f : v1;
              }
              s1 += s1b;
              s2 += s2b;
            }
            if constexpr (DSM == kDsDiag) {
              const int ntk = (p.Lk + kTile - 1) / kTile;
              float* dst = p.diag_out +
                           ((((static_cast<int64_t>(b) * p.Hq + hq) * nqt + m0 / kTile) * ntk +
                             (n0 - c0w) / kTile) * 8 + warp) * 128;
              dst[h * 64 + lane] = s1;
              if (lane < 31) dst[h * 64 + 32 + lane] = s2;
            } else {
              float* bacc = reinterpret_cast<float*>(smem + Lay::kBAccOff) + warp * 128;
              {
                // prefix sums over t = -31 .. 31 (s1 of lanes 0..31, then s2
                // of lanes 0..30) at index t + 32 (index 0: the empty
                // prefix); a bucket's sum is the difference of two of them
                float a = s1, e = lane < 31 ? s2 : 0.f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                  const float xa = __shfl_up_sync(0xffffffffu, a, o);
                  const float xe = __shfl_up_sync(0xffffffffu, e, o);
                  if (lane >= o) {
                    a += xa;
                    e += xe;
                  }
                }
                e += __shfl_sync(0xffffffffu, a, 31);
                __syncwarp();
                stg[lane + 1] = a;
                if (lane < 31) stg[lane + 33] = e;
                if (lane == 0) stg[0] = 0.f;
                __syncwarp();
                const int nbk = p.t5.bidirectional ? 2 * p.t5.half : p.t5.half;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  if (32 * q >= nbk) break;
                  const int lo = max(rlo[q] - t0, -31);
                  const int hi = min(rhi[q] - t0, 31);
                  if (lo <= hi) bacc[lane + 32 * q] += stg[hi + 32] - stg[lo + 31];
                }
              }
            }
          }
        }
        if constexpr (DSM == kDsStore) {
          // fp32 dS of this row's 64 keys while the dQ MMA runs; masked keys
          // have P = 0 and so dS = 0.  Lanes 2m and 2m + 1 hold neighbouring
          // rows; for every 8 keys they swap four values so that each store
          // writes one whole 32-byte piece of a row from two lanes (the even
          // lane's row first, then the odd lane's), rather than every lane
          // half a piece of its own row.  Streaming stores: dS is not read
          // again here and should not evict the K / V tiles that
          // neighbouring heads reuse from L2.
          const int64_t head_off = static_cast<int64_t>(b) * p.sd_b + static_cast<int64_t>(hq) * p.sd_h;
          if (n0 + kBlk <= Lk) {
            const bool odd = (lane & 1) != 0;
            const int i_a = odd ? i - 1 : i;  // the even lane's row
            const int i_b = odd ? i : i + 1;  // the odd lane's row
            const int c_off = n0 + (odd ? 4 : 0);
            float* row_a = p.ds_out + head_off + static_cast<int64_t>(i_a) * p.sd_i + c_off;
            float* row_b = p.ds_out + head_off + static_cast<int64_t>(i_b) * p.sd_i + c_off;
#pragma unroll
            for (int g = 0; g < kBlk; g += 8) {
              float lo[4], hi[4], got[4];
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                lo[t] = __uint_as_float(pr[g + t]);
                hi[t] = __uint_as_float(pr[g + 4 + t]);
              }
              // the even lane sends its keys g+4..g+7, the odd lane its g..g+3
#pragma unroll
              for (int t = 0; t < 4; ++t) got[t] = __shfl_xor_sync(0xffffffffu, odd ? lo[t] : hi[t], 1);
              const float4 va = odd ? make_float4(got[0], got[1], got[2], got[3])
                                    : make_float4(lo[0], lo[1], lo[2], lo[3]);
              const float4 vb = odd ? make_float4(hi[0], hi[1], hi[2], hi[3])
                                    : make_float4(got[0], got[1], got[2], got[3]);
              if (i_a < Lq) __stcs(reinterpret_cast<float4*>(row_a + g), va);
              if (i_b < Lq) __stcs(reinterpret_cast<float4*>(row_b + g), vb);
            }
          } else if (i < Lq) {
            float* dst = p.ds_out + head_off + static_cast<int64_t>(i) * p.sd_i + n0;
#pragma unroll
            for (int e = 0; e < kBlk; ++e)
              if (n0 + e < Lk) __stcs(dst + e, __uint_as_float(pr[e]));
          }
        }
      }
      if constexpr (DSM == kDsDiagT5) {
        // this warp's per-bucket sums over the item's key tiles, at
        // [b, hq, query tile, warp, bucket]; the accumulators restart at 0
        const int nbk = p.t5.bidirectional ? 2 * p.t5.half : p.t5.half;
        float* bacc = reinterpret_cast<float*>(smem + Lay::kBAccOff) + warp * 128;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          one_lo += __shfl_xor_sync(0xffffffffu, one_lo, o);
          one_hi += __shfl_xor_sync(0xffffffffu, one_hi, o);
        }
        const int k_lo = p.t5.half - 1;
        const int k_hi = p.t5.bidirectional ? 2 * p.t5.half - 1 : 0;
        if (lane == (k_lo & 31)) bacc[k_lo] += one_lo;
        if (lane == (k_hi & 31)) bacc[k_hi] += one_hi;
        float* dstb = p.diag_out +
                      (((static_cast<int64_t>(b) * p.Hq + hq) * nqt + m0 / kTile) * 8 + warp) * nbk;
        for (int k = lane; k < nbk; k += 32) {
          dstb[k] = bacc[k];
          bacc[k] = 0.f;
        }
      }
      // ----------- epilogue: warpgroup wg stores dQ columns [wg D/2, (wg+1) D/2) -----------
      // Items without a visible key (none exist for the masks accepted at the
      // boundary) store zeros without touching tensor memory.
      if (nt > 0) {
        if (ok) ok = mbar_wait(acc_done, u & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        ++u;
      }
      if (ok) {
        uint32_t r[D / 2];
        if (nt > 0) {
          tc_fence_after();
#pragma unroll
          for (int cc = 0; cc < D / 2; cc += 32)
            tmem_ld32_sync(tmem + lane_bits + Lay::kDQCol + wg * (D / 2) + cc,
                           *reinterpret_cast<uint32_t(*)[32]>(r + cc));
        } else {
#pragma unroll
          for (int e = 0; e < D / 2; ++e) r[e] = 0u;
        }
        // lanes 2m, 2m + 1 hold rows i, i + 1 and trade halves of every 16
        // columns, so each 16-byte store of the pair fills one 32-byte sector
        const bool odd = (lane & 1) != 0;
        const int ia = i - (odd ? 1 : 0);
        __nv_bfloat16* dst_a = p.dq + static_cast<int64_t>(w.s.bc) * p.sq_b +
                               static_cast<int64_t>(w.s.q0 + ia) * p.sq_l +
                               static_cast<int64_t>(hq) * p.sq_h + wg * (D / 2) + (odd ? 8 : 0);
        __nv_bfloat16* dst_b = dst_a + p.sq_l;
#pragma unroll
        for (int cc = 0; cc < D / 2; cc += 16) {
          uint4 lo4, hi4;
          pack16(r + cc, p.scale, lo4, hi4);
          const uint4 got = shfl_xor_u4(odd ? lo4 : hi4, 1);
          const uint4 va = odd ? got : lo4;  // row ia
          const uint4 vb = odd ? hi4 : got;  // row ia + 1
          if (ia < Lq) *reinterpret_cast<uint4*>(dst_a + cc) = va;
          if (ia + 1 < Lq) *reinterpret_cast<uint4*>(dst_b + cc) = vb;
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
// Launch selection bits of the backward (sdpa_bwd_phases).
constexpr uint32_t kPhasePre = 1u, kPhaseDq = 2u, kPhaseDkdv = 4u;

// Workspace of the backward: D [rows] fp32, rows = the LSE rows
// (B * Hq * Lq, or Hq * total rows when packed), 256-byte rounded.
struct BwdWorkspace {
  size_t d_off, total;
};

inline BwdWorkspace bwd_workspace_plan(int64_t rows) {
  BwdWorkspace w;
  w.d_off = 0;
  w.total = (static_cast<size_t>(rows) * 4 + 255) / 256 * 256;
  return w;
}

template <int D, int BIAS>
cudaError_t launch_bwd_t(const AttnParams& p, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mdo, const CUtensorMap& mb,
                         uint32_t phases, int64_t n_axis, cudaStream_t st) {
  if (phases & kPhasePre) {
    const int64_t threads = n_axis * p.Hq * (D / 8);
    const int64_t blocks = (threads + 255) / 256;
    bwd_preprocess_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, st>>>(p, n_axis);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (phases & kPhaseDq) {
    auto kern = bwd_dq_kernel<D, BIAS>;
    int smem_bytes = DqLayout<D, BIAS>::kSmemAlloc;
    int threads = DqLayout<D, BIAS>::kThreads;
    if constexpr (BIAS == kBiasDense) {
      if (p.ds_out) {
        kern = bwd_dq_kernel<D, BIAS, kDsStore>;
        smem_bytes = DqLayout<D, BIAS, kDsStore>::kSmemAlloc;
        threads = DqLayout<D, BIAS, kDsStore>::kThreads;
      }
    }
    if constexpr (BIAS == kBiasT5) {
      if (p.diag_out && p.rel_table) {
        kern = bwd_dq_kernel<D, BIAS, kDsDiag>;
        smem_bytes = DqLayout<D, BIAS, kDsDiag>::kSmemAlloc;
        threads = DqLayout<D, BIAS, kDsDiag>::kThreads;
      } else if (p.diag_out && p.alibi) {
        kern = bwd_dq_kernel<D, BIAS, kDsMoment>;
        smem_bytes = DqLayout<D, BIAS, kDsMoment>::kSmemAlloc;
        threads = DqLayout<D, BIAS, kDsMoment>::kThreads;
      } else if (p.diag_out) {
        kern = bwd_dq_kernel<D, BIAS, kDsDiagT5>;
        smem_bytes = DqLayout<D, BIAS, kDsDiagT5>::kSmemAlloc;
        threads = DqLayout<D, BIAS, kDsDiagT5>::kThreads;
      }
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (or per work item, if fewer)
    const int64_t items = static_cast<int64_t>((p.Lq + kTile - 1) / kTile) * p.Hq * p.B;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    kern<<<static_cast<int>(items < sms ? items : sms), threads, smem_bytes, st>>>(
        p, mq, mk, mv, mdo, mb);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (phases & kPhaseDkdv) {
    using Lay = DkdvLayout<D, BIAS>;
    auto kern = bwd_dkdv_kernel<D, BIAS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Lay::kSmemAlloc);
    if (e != cudaSuccess) return e;
    const int ntk = (p.Lk + kTile - 1) / kTile;
    kern<<<dim3(ntk, p.Hkv, p.B), Lay::kThreads, Lay::kSmemAlloc, st>>>(p, mq, mk, mv, mdo, mb);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int D>
cudaError_t launch_bwd_d(const AttnParams& p, const CUtensorMap& mq, const CUtensorMap& mk,
                         const CUtensorMap& mv, const CUtensorMap& mdo, const CUtensorMap& mb,
                         uint32_t phases, int64_t n_axis, cudaStream_t st) {
  switch (p.bias_kind) {
    case kBiasDense: return launch_bwd_t<D, kBiasDense>(p, mq, mk, mv, mdo, mb, phases, n_axis, st);
    case kBiasT5: return launch_bwd_t<D, kBiasT5>(p, mq, mk, mv, mdo, mb, phases, n_axis, st);
    default: return launch_bwd_t<D, kBiasNone>(p, mq, mk, mv, mdo, mb, phases, n_axis, st);
  }
}

}  // namespace sdpa
