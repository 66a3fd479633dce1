// fwd_kernel.cuh -- fused attention forward for sm_100a.
//
// Persistent: one CTA per SM walks a list of work items -- a tile of 128
// query rows of one (batch, query head), heaviest causal tiles first -- and
// for each streams the key/value tiles of the mask band through shared memory.
// Every ring and buffer index below counts across items, so the producers and
// the S issuer run on into the next item while the softmax warps finish the
// current one:
//
//   K producer warp   TMA: the item's Q tile (once the previous item's last S
//                     MMA has read the single Q buffer), then K_j into a ring
//                     of kSK stages
//                     (fully masked key tiles are never loaded -- the point of
//                     HF transformers issue #30461: a mask handed over as a
//                     dense tensor forfeits this skipping).
//   V producer warp   TMA: V_j into a ring of kSV stages.
//   S issuer          one thread: S_j = Q K_j^T into tensor-memory buffer
//                     j mod 3, as soon as K_j has landed and the P V MMA of
//                     tile j - 3 has finished reading that buffer.
//   PV issuer         one thread: O += P_j V_j with P_j read from tensor memory.
//   softmax warps     two warpgroups, thread = query row (its TMEM lane);
//                     warpgroup w owns the key columns [64 w, 64 w + 64) of
//                     every tile.  Per tile: load its half of S_j, take the
//                     partial row max, exchange it with the other warpgroup
//                     through shared memory, then scale (log2 e folded in),
//                     bias, band-edge mask, exp2, P_j back to tensor memory as
//                     bf16 over its own S columns.  O is rescaled in tensor
//                     memory only when the row max grows by more than 2^8
//                     (exact: O and the row sum always share one reference
//                     max); each warpgroup rescales half of O's columns.
//                     Epilogue: O = acc / sum -> bf16, LSE = (max + log2 sum) ln 2.
//
// Tensor memory (512 columns): S buffers at 0, 128, 256; O at 384 (d columns).
// Three S buffers let the tensor core compute S_{j+1} and S_{j+2} while the
// softmax of tile j runs, so neither side waits on the other's latency.
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

constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when max grows > 2^8
// Share of a full tile's exponentials on MUFU (per 8 columns; 8 = all): with
// both warpgroups on one tile, 6 of 8 on MUFU and 2 on the FMA pipe measured
// fastest at d = 128 (5 and 4 were slower); at d = 64, where P V takes half
// as long, 5 of 8 (t5rpe forward 0.175 -> 0.173 ms).
template <int D>
constexpr int kFwdMufuPer8 = (D == 64) ? 5 : 6;
// Full tiles without a bias take the lean path: the row max is taken on the
// raw scores (scale > 0 preserves the order), the scale folds into the one
// fused multiply-add that forms each exponent, and pairs of columns go
// through the packed fp32x2 FMA / add of sm_100.
constexpr bool kFwdLeanSoftmax = true;
// Named barriers: 1, 2 guard each warpgroup's T5 bias table; 3 is the
// row-max / row-sum exchange between the two warpgroups.
constexpr uint32_t kXchgBar = 3;

template <int D, int BIAS>
struct FwdLayout {
  static constexpr int kTileBytes = kTile * D * 2;  // one 128 x D bf16 tile
  static constexpr int kNS = 3;                     // S buffers in tensor memory
  // Dense bias at d = 64: each tile's 128 x 128 fp32 bias block comes by TMA
  // into a 2-stage ring (4 boxes of 128 rows x 32 columns, 128-byte swizzle).
  static constexpr bool kBiasTma = (BIAS == kBiasDense && D == 64);
  static constexpr int kBiasTileBytes = kTile * kTile * 4;
  static constexpr int kSB = kBiasTma ? 2 : 0;
  // K is needed up to three tiles ahead of V (the S buffers run ahead of P V).
  static constexpr int kSK = (D == 128) ? 3 : (kBiasTma ? 2 : 4);
  static constexpr int kSV = (D == 128) ? 2 : (kBiasTma ? 2 : 4);
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kTileBytes;
  static constexpr int kVOff = kKOff + kSK * kTileBytes;
  static constexpr int kBOff = kVOff + kSV * kTileBytes;    // bias ring (kBiasTma)
  static constexpr int kRedOff = kBOff + kSB * kBiasTileBytes;  // max[2][2][128], sum[2][2][128]
  static constexpr int kRedBytes = 8 * kTile * 4;
  static constexpr int kLutOff = kRedOff + kRedBytes;       // T5 only: 2 WG x 2 x 256 floats
  static constexpr int kLutBytes = (BIAS == kBiasT5) ? 4 * 256 * 4 : 0;
  static constexpr int kBarOff = kLutOff + kLutBytes;
  // q_full, q_empty, k_full[SK], k_empty[SK], v_full[SV], v_empty[SV],
  // s_full[NS], p_full[NS], pv_done[NS], acc_done, drain[2], b_full[2], b_empty[2]
  static constexpr int kNumBars = 2 + 2 * kSK + 2 * kSV + 3 * kNS + 3 + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemAlloc = kMiscOff + 16;
  // 2 softmax warpgroups; warp 8 K producer, 9 S issuer, 10 PV issuer, 11 V producer
  static constexpr int kThreads = 384;
  static constexpr int kTmemCols = 512;
  static constexpr int kOCol = kNS * kTile;
  static_assert(kOCol + D <= kTmemCols, "tensor memory budget");
  static_assert(kSK <= 4 && kSV <= 4, "producer bookkeeping");
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

template <int D, int BIAS>
__global__ void __launch_bounds__(384, 1)
    fwd_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmQ,
               const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmB) {
  using Lay = FwdLayout<D, BIAS>;
  constexpr int SK = Lay::kSK;
  constexpr int SV = Lay::kSV;
  constexpr int NS = Lay::kNS;
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
  // Query tiles past a (packed) sequence's end are empty items.
  const int nqt = (p.Lq + kTile - 1) / kTile;
  const int heads = p.Hq * p.B;
  const int n_items = nqt * heads;
  struct Item {
    int m0, hq, b, g, nlo, nt;
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
    int nhi;
    key_tile_range(p, w.s.Lq, w.s.Lk, w.m0, kTile, w.nlo, nhi);
    w.nt = (w.m0 < w.s.Lq && nhi > w.nlo) ? nhi - w.nlo : 0;
    return w;
  };

  // ---- barriers
  auto bar = [&](int idx) -> uint32_t { return sb + Lay::kBarOff + 8 * idx; };
  const uint32_t q_full = bar(0);
  const uint32_t q_empty = bar(1);
  auto k_full = [&](int s) { return bar(2 + s); };
  auto k_empty = [&](int s) { return bar(2 + SK + s); };
  auto v_full = [&](int s) { return bar(2 + 2 * SK + s); };
  auto v_empty = [&](int s) { return bar(2 + 2 * SK + SV + s); };
  constexpr int kB = 2 + 2 * SK + 2 * SV;
  auto s_full = [&](int x) { return bar(kB + x); };
  auto p_full = [&](int x) { return bar(kB + NS + x); };
  auto pv_done = [&](int x) { return bar(kB + 2 * NS + x); };
  const uint32_t acc_done = bar(kB + 3 * NS);
  auto drain = [&](int x) { return bar(kB + 3 * NS + 1 + x); };
  auto b_full = [&](int x) { return bar(kB + 3 * NS + 3 + x); };
  auto b_empty = [&](int x) { return bar(kB + 3 * NS + 5 + x); };
  constexpr bool BT = Lay::kBiasTma;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < SK; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < SV; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int x = 0; x < NS; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(p_full(x), 2 * kTile);
      mbar_init(pv_done(x), 1);
    }
    mbar_init(acc_done, 1);
    mbar_init(drain(0), 1);
    mbar_init(drain(1), 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(b_full(x), 1);
      mbar_init(b_empty(x), 2 * kTile);
    }
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

  if (warp == 8 || warp == 11) {
    // ===================== producers (TMA): K (+Q) and V =====================
    const bool is_k = (warp == 8);
    if (lane == 0) {
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      const int stages = is_k ? SK : SV;
      const uint32_t ring = sb + (is_k ? Lay::kKOff : Lay::kVOff);
      tma_prefetch_desc(map);
      if (is_k) tma_prefetch_desc(&tmQ);
      int issued[4] = {-1, -1, -1, -1};
      int b_issued[2] = {-1, -1};
      int q_issued = -1;
      int c = 0;  // tiles loaded so far, over all items
      int u = 0;  // items with a non-empty band so far
      bool ok = true;
      for (int id = blockIdx.x; id < n_items && ok; id += gridDim.x) {
        const Item w = item_at(id);
        if (w.nt == 0) continue;
        if (is_k) {
          // the single Q buffer is free once the previous item's S MMAs are done
          if (u > 0 && !(ok = mbar_wait(q_empty, (u - 1) & 1, ctl))) break;
          mbar_expect_tx(q_full, Lay::kTileBytes);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(sb + Lay::kQOff + h * kTile * 128, &tmQ, q_full, h * 64, w.s.q0 + w.m0,
                        w.hq, w.s.bc);
          q_issued = u & 1;
        }
        for (int it = 0; it < w.nt; ++it, ++c) {
          const int s = c % stages;
          const uint32_t ph = (c / stages) & 1;
          const uint32_t full = is_k ? k_full(s) : v_full(s);
          const uint32_t empty = is_k ? k_empty(s) : v_empty(s);
          if (!(ok = mbar_wait(empty, ph ^ 1, ctl))) break;
          mbar_expect_tx(full, Lay::kTileBytes);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(ring + s * Lay::kTileBytes + h * kTile * 128, map, full, h * 64,
                        w.s.k0 + (w.nlo + it) * kTile, w.g, w.s.bc);
          issued[s] = static_cast<int>(ph);
          if constexpr (BT) {
            if (is_k) {
              // this tile's bias block: rows m0.., keys n0.. of (b, hq), 4 boxes
              const int x = c & 1;
              const uint32_t bph = (c >> 1) & 1;
              if (!(ok = mbar_wait(b_empty(x), bph ^ 1, ctl))) break;
              mbar_expect_tx(b_full(x), Lay::kBiasTileBytes);
              const int n0 = (w.nlo + it) * kTile;
              const int hb = p.sb_h ? w.hq : 0, bb = p.sb_b ? w.b : 0;
              for (int q4 = 0; q4 < 4; ++q4)
                tma_load_4d(sb + Lay::kBOff + x * Lay::kBiasTileBytes + q4 * (kTile * 128), &tmB,
                            b_full(x), n0 + 32 * q4, w.m0, hb, bb);
              b_issued[x] = static_cast<int>(bph);
            }
          } else if constexpr (BIAS == kBiasDense) {
            if (is_k) prefetch_bias_tile(p, w.b, w.hq, w.m0, (w.nlo + it) * kTile);
          }
        }
        ++u;
      }
      if (!ok) {
        // Aborted: let every copy already issued land before the CTA exits.
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        if (q_issued >= 0) mbar_wait(q_full, q_issued, ign);
        for (int s = 0; s < stages; ++s)
          if (issued[s] >= 0) mbar_wait(is_k ? k_full(s) : v_full(s), issued[s], ign);
        for (int x = 0; x < 2; ++x)
          if (b_issued[x] >= 0) mbar_wait(b_full(x), b_issued[x], ign);
      }
    }
  } else if (warp == 9 || warp == 10) {
    // ===================== MMA issuers (one thread each) =====================
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kTile, kTile, 0, 0);  // Q, K both K-major
      constexpr uint32_t kIdO = idesc_bf16_f32(kTile, D, 0, 1);      // V is N(=d)-major
      const bool chain_s = (warp == 9);
      // Descriptors are built once: one at shared-memory offset 0 per layout,
      // plus the byte offset / 16 of each operand (the start-address field),
      // so an MMA costs the issuing thread two adds; it shares its
      // sub-partition with busy softmax warps.
      const uint64_t dk0 = smem_desc_sw128(sb, 16, 1024);            // K-major
      const uint64_t dmn0 = smem_desc_sw128(sb, kTile * 128, 1024);  // MN-major, 64-wide halves
      int c = 0;  // tiles so far, over all items
      int u = 0;  // items with a non-empty band so far
      bool ok = true;
      for (int id = blockIdx.x; id < n_items && ok; id += gridDim.x) {
        const Item w = item_at(id);
        if (w.nt == 0) continue;
        if (chain_s && !(ok = issuer_wait(q_full, u & 1, ctl))) break;
        for (int it = 0; it < w.nt; ++it, ++c) {
          const int x = c % NS;
          if (chain_s) {
            const int sk = c % SK;
            if (!(ok = issuer_wait(k_full(sk), (c / SK) & 1, ctl))) break;
            // buffer x held P of tile c - NS: wait until its P V MMA is done
            if (c >= NS && !(ok = issuer_wait(pv_done(x), ((c / NS) - 1) & 1, ctl))) break;
            tc_fence_after();
            const uint64_t kd = dk0 + ((Lay::kKOff + sk * Lay::kTileBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + x * kTile, dk0 + ((Lay::kQOff + kmajor_koff(kk, kTile)) >> 4),
                     kd + (kmajor_koff(kk, kTile) >> 4), kIdS, kk > 0 ? 1u : 0u);
            mma_commit(s_full(x));
            mma_commit(k_empty(sk));
          } else {
            // P V of an item's first tile overwrites O: every softmax thread
            // read the previous item's O before it marked this P ready.
            const int sv = c % SV;
            if (!(ok = issuer_wait(v_full(sv), (c / SV) & 1, ctl))) break;
            if (!(ok = issuer_wait(p_full(x), (c / NS) & 1, ctl))) break;
            tc_fence_after();
            const uint64_t vmd = dmn0 + ((Lay::kVOff + sv * Lay::kTileBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              mma_ts(tmem + Lay::kOCol, split_a_col(tmem + x * kTile, kk), vmd + kk * (2048 >> 4), kIdO,
                     (it > 0 || kk > 0) ? 1u : 0u);
            mma_commit(pv_done(x));
            mma_commit(v_empty(sv));
          }
        }
        if (!ok) break;
        mma_commit(chain_s ? q_empty : acc_done);
        ++u;
      }
      if (!ok) {
        // Aborted: wait until every MMA this thread issued has finished with
        // tensor memory before the CTA frees it.
        volatile int never = 0;
        const WaitCtl ign{&never, p.wait_limit_ns};
        mma_commit(drain(chain_s ? 0 : 1));
        mbar_wait(drain(chain_s ? 0 : 1), 0, ign);
      }
    }
  } else {
    // ===== softmax warpgroup wg: key columns [64 wg, 64 wg + 64); thread = query row =====
    const int wg = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const int c0w = kBlk * wg;
    const uint32_t lane_bits = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + lane_bits + Lay::kOCol + wg * (D / 2);
    float* red = reinterpret_cast<float*>(smem + Lay::kRedOff);  // max [parity][wg][row]
    float* rsum = red + 4 * kTile;                               // sum [parity][wg][row]
    float* lut = reinterpret_cast<float*>(smem + Lay::kLutOff) + wg * 512;
    // `ok` is kept warp-uniform.  After an abort every wait returns at once,
    // but every tile of every item still passes the exchange barrier, so no
    // thread of the CTA is left waiting at a named barrier.
    bool ok = true;
    int gc = 0;  // tiles so far, over all items
    int u = 0;   // items with a non-empty band so far
    for (int id = blockIdx.x; id < n_items; id += gridDim.x) {
      const Item w = item_at(id);
      const int m0 = w.m0, hq = w.hq, b = w.b, nt = w.nt;
      const int Lq = w.s.Lq, Lk = w.s.Lk;
      const int i = m0 + row;  // query row
      const float* brow = nullptr;
      if constexpr (BIAS == kBiasDense) {
        // rows past Lq read row Lq-1 (in bounds); their outputs are never stored
        brow = p.bias + static_cast<int64_t>(b) * p.sb_b + static_cast<int64_t>(hq) * p.sb_h +
               static_cast<int64_t>(min(i, Lq - 1)) * p.sb_i;
      }
      float m_run = -INFINITY;  // running row max, log2 units (identical in both warpgroups)
      float l_run = 0.f;        // this warpgroup's share of the row sum, relative to m_run
      for (int it = 0; it < nt; ++it, ++gc) {
        const int x = gc % NS;
        const int n0 = (w.nlo + it) * kTile + c0w;  // first key of this warpgroup's columns
        const uint32_t tS = tmem + lane_bits + x * kTile + c0w;
        bool full = n0 + kBlk <= Lk;
        if (p.causal) full = full && (n0 + kBlk - 1 <= m0);
        if (p.wl >= 0) full = full && (n0 >= m0 + kTile - 1 - p.wl);
        if (p.wr >= 0) full = full && (n0 + kBlk - 1 <= m0 + p.wr);
        const float* lut_row = nullptr;
        // a fully visible piece of the warpgroup inside one T5 bucket: bias
        // ub throughout, taken by the lean path below without a table
        bool one_b = false;
        float ub = 0.f;
        if constexpr (BIAS == kBiasT5) {
          // j - i = (n0 - m0) + (c - row): entry r = c - row + 127, r in [0, 190]
          float* lt = lut + (gc & 1) * 256;
          const int base = n0 - m0 - (kTile - 1);
          // (the same for the whole warpgroup, so all or none of it takes the
          // barrier; the table of tile gc - 2 is no longer read: every
          // thread has passed the maximum exchange of tile gc - 1)
          one_b = kFwdLeanSoftmax && full && p.scale_log2 > 0.f &&
                  t5_one_bucket(p, base, kTile + kBlk - 2, hq, ub);
          if (!one_b) {
            for (int r = row; r < kTile + kBlk - 1; r += kTile)
              lt[r] = rel_bias_log2(p, base + r, hq);
            named_barrier(1 + wg, kTile);
          }
          lut_row = lt + (kTile - 1) - row;
        }
        int lo = 0, hi = kBlk - 1;
        if (!full) {
          if (p.wl >= 0) lo = max(lo, i - p.wl - n0);
          hi = min(hi, Lk - 1 - n0);
          if (p.causal) hi = min(hi, i - n0);
          if (p.wr >= 0) hi = min(hi, i + p.wr - n0);
        }
        // lean: no bias, or a one-bucket T5 bias (a constant ub folded into
        // the maximum and the exponent's offset)
        const bool lean = kFwdLeanSoftmax && (BIAS == kBiasNone || (BIAS == kBiasT5 && one_b)) &&
                          full && p.scale_log2 > 0.f;

        // ---- phase A: this warpgroup's half of S_j and its partial row max
        if (ok) ok = mbar_wait(s_full(x), (gc / NS) & 1, ctl);
        if constexpr (BT) {
          if (ok) ok = mbar_wait(b_full(gc & 1), (gc >> 1) & 1, ctl);
        }
        ok = __all_sync(0xffffffffu, ok);
        const bool live = ok;
        uint32_t xs[kBlk];  // raw accumulator bits (lean) or log2-unit scores
        float pmax = -INFINITY;
        if (live) {
          tc_fence_after();
          tmem_ld64_sync(tS, xs);
          if (lean) {
            float ma = -INFINITY, mb = -INFINITY;
#pragma unroll
            for (int c = 0; c < kBlk; c += 4) {
              ma = fmax3(ma, __uint_as_float(xs[c]), __uint_as_float(xs[c + 1]));
              mb = fmax3(mb, __uint_as_float(xs[c + 2]), __uint_as_float(xs[c + 3]));
            }
            pmax = fmaf(fmaxf(ma, mb), p.scale_log2, ub);
          } else {
            float tm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if constexpr (BT) {
              // this warpgroup's 64 bias columns from the staged block: boxes
              // 2 wg and 2 wg + 1, row `row`, 8 swizzled 16-byte chunks each
              const uint8_t* bt = smem + Lay::kBOff + (gc & 1) * Lay::kBiasTileBytes;
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint8_t* brw = bt + (2 * wg + h) * (kTile * 128) + row * 128;
#pragma unroll
                for (int k4 = 0; k4 < 8; ++k4) {
                  const float4 b4 = *reinterpret_cast<const float4*>(brw + ((k4 ^ (row & 7)) << 4));
                  const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const int c = 32 * h + 4 * k4 + e;
                    float v = fmaf(bv[e], kLog2e, __uint_as_float(xs[c]) * p.scale_log2);
                    if (!full) v = (c >= lo && c <= hi) ? v : -INFINITY;
                    xs[c] = __float_as_uint(v);
                    tm[c & 3] = fmaxf(tm[c & 3], v);
                  }
                }
              }
              mbar_arrive(b_empty(gc & 1));  // the bias block is read
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
                    const int c = 32 * h + 4 * q + e;
                    const float v = fmaf(bv[e], kLog2e, __uint_as_float(xs[c]) * p.scale_log2);
                    xs[c] = __float_as_uint(v);
                    tm[c & 3] = fmaxf(tm[c & 3], v);
                  }
                }
              }
            } else if (full) {
#pragma unroll
              for (int c = 0; c < kBlk; ++c) {
                float v = __uint_as_float(xs[c]) * p.scale_log2;
                if constexpr (BIAS == kBiasT5) v += lut_row[c];
                xs[c] = __float_as_uint(v);
                tm[c & 3] = fmaxf(tm[c & 3], v);
              }
            } else {
#pragma unroll
              for (int c = 0; c < kBlk; ++c) {
                const bool vis = (c >= lo) && (c <= hi);
                float v = __uint_as_float(xs[c]) * p.scale_log2;
                if constexpr (BIAS == kBiasT5) v += lut_row[c];
                if constexpr (BIAS == kBiasDense) v += vis ? brow[n0 + c] * kLog2e : 0.f;
                v = vis ? v : -INFINITY;
                xs[c] = __float_as_uint(v);
                tm[c & 3] = fmaxf(tm[c & 3], v);
              }
            }
            pmax = fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3]));
          }
        }
        // ---- exchange the partial maxima (double-buffered by tile parity)
        red[((gc & 1) * 2 + wg) * kTile + row] = pmax;
        named_barrier(kXchgBar, 2 * kTile);
        if (!live) continue;
        const float tmax = fmaxf(pmax, red[((gc & 1) * 2 + (1 - wg)) * kTile + row]);
        const float m_new = fmaxf(m_run, tmax);
        const bool grow = m_new > m_run + kRescaleThreshold;
        const float m_use = grow ? m_new : m_run;
        const float alpha = grow ? fast_exp2(m_run - m_use) : 1.f;
        const float m_sub = (m_use == -INFINITY) ? 0.f : m_use;  // finite on every lean tile

        // ---- phase B: exponentials, P_j (bf16) over the first 32 of this warpgroup's S columns
        float sum;
        if (lean) {
          const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
          const uint64_t nm2 = f2_pack(ub - m_sub, ub - m_sub);
          uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
          for (int c0 = 0; c0 < kBlk; c0 += 32) {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const uint64_t arg = f2_fma(
                  f2_pack(__uint_as_float(xs[c0 + c]), __uint_as_float(xs[c0 + c + 1])), c2, nm2);
              float v0, v1, e0, e1;
              f2_unpack(arg, v0, v1);
              exp2_pair<BIAS, kFwdMufuPer8<D>>(c0 + c, v0, v1, e0, e1);
              acc[(c >> 1) & 3] = f2_add(acc[(c >> 1) & 3], f2_pack(e0, e1));
              pk[c >> 1] = pack_bf16x2(e0, e1);
            }
            tmem_st16(tS + (c0 >> 1), pk);
          }
          float s0, s1, s2, s3, s4, s5, s6, s7;
          f2_unpack(acc[0], s0, s1);
          f2_unpack(acc[1], s2, s3);
          f2_unpack(acc[2], s4, s5);
          f2_unpack(acc[3], s6, s7);
          sum = ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
        } else {
          float sm[4] = {0.f, 0.f, 0.f, 0.f};
          if (full) {
            // every entry is finite: a fixed share of the exponentials on the FMA pipe
#pragma unroll
            for (int c0 = 0; c0 < kBlk; c0 += 32) {
              uint32_t pk[16];
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                const float v0 = __uint_as_float(xs[c0 + c]) - m_sub;
                const float v1 = __uint_as_float(xs[c0 + c + 1]) - m_sub;
                float e0, e1;
                exp2_pair<BIAS, kFwdMufuPer8<D>>(c0 + c, v0, v1, e0, e1);
                sm[(c >> 1) & 3] += e0 + e1;
                pk[c >> 1] = pack_bf16x2(e0, e1);
              }
              tmem_st16(tS + (c0 >> 1), pk);
            }
          } else {
#pragma unroll
            for (int c0 = 0; c0 < kBlk; c0 += 32) {
              uint32_t pk[16];
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                const float e0 = fast_exp2(__uint_as_float(xs[c0 + c]) - m_sub);
                const float e1 = fast_exp2(__uint_as_float(xs[c0 + c + 1]) - m_sub);
                sm[(c >> 1) & 3] += e0 + e1;
                pk[c >> 1] = pack_bf16x2(e0, e1);
              }
              tmem_st16(tS + (c0 >> 1), pk);
            }
          }
          sum = (sm[0] + sm[1]) + (sm[2] + sm[3]);
        }
        l_run = l_run * alpha + sum;
        m_run = m_use;
        tmem_st_wait();
        if (it > 0 && __any_sync(0xffffffffu, grow)) {
          // O holds earlier tiles: rescale this warpgroup's half of its columns
          // once P V of the previous tile has landed.
          ok = mbar_wait(pv_done((gc - 1) % NS), ((gc - 1) / NS) & 1, ctl);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) continue;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 2; c += 32) {
            uint32_t r[32];
            tmem_ld32_sync(tO + c, r);
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32_sync(tO + c, r);
          }
        }
        tc_fence_before();
        mbar_arrive(p_full(x));
      }

      // ------------------------------ epilogue ------------------------------
      // Rows that see no key (a left window that starts past the end of a
      // shorter key sequence, an empty packed key sequence) get O = 0 and
      // LSE = -inf without touching tensor memory; rows past the end of the
      // query sequence are not written.
      float l_tot = 0.f;
      if (nt > 0) {
        rsum[((u & 1) * 2 + wg) * kTile + row] = l_run;
        named_barrier(kXchgBar, 2 * kTile);
        l_tot = l_run + rsum[((u & 1) * 2 + (1 - wg)) * kTile + row];
        if (ok) ok = mbar_wait(acc_done, u & 1, ctl);
        ok = __all_sync(0xffffffffu, ok);
        ++u;
      }
      if (ok) {
        // this warpgroup's half of the O row; once read, the next item's first
        // P V may overwrite O (this thread marks that P ready only after this)
        uint32_t r[D / 2];
        if (nt > 0) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 2; c += 32)
            tmem_ld32_sync(tO + c, *reinterpret_cast<uint32_t(*)[32]>(r + c));
        } else {
#pragma unroll
          for (int e = 0; e < D / 2; ++e) r[e] = 0u;
        }
        const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
        // O: lanes 2m and 2m + 1 hold rows i and i + 1.  For every 16
        // columns (32 bytes of bf16) they trade halves, so each 16-byte
        // store of the pair writes one whole 32-byte sector of one row: the
        // even lane's row first, then the odd lane's.
        const bool odd = (lane & 1) != 0;
        const int i_a = odd ? i - 1 : i, i_b = odd ? i : i + 1;
        __nv_bfloat16* row_a = p.o + static_cast<int64_t>(b) * p.sq_b +
                               static_cast<int64_t>(w.s.q0 + i_a) * p.sq_l +
                               static_cast<int64_t>(hq) * p.sq_h + wg * (D / 2) + (odd ? 8 : 0);
        __nv_bfloat16* row_b = row_a + p.sq_l;
#pragma unroll
        for (int c = 0; c < D / 2; c += 16) {
          uint4 lo, hi;
          lo.x = pack_bf16x2(__uint_as_float(r[c]) * inv, __uint_as_float(r[c + 1]) * inv);
          lo.y = pack_bf16x2(__uint_as_float(r[c + 2]) * inv, __uint_as_float(r[c + 3]) * inv);
          lo.z = pack_bf16x2(__uint_as_float(r[c + 4]) * inv, __uint_as_float(r[c + 5]) * inv);
          lo.w = pack_bf16x2(__uint_as_float(r[c + 6]) * inv, __uint_as_float(r[c + 7]) * inv);
          hi.x = pack_bf16x2(__uint_as_float(r[c + 8]) * inv, __uint_as_float(r[c + 9]) * inv);
          hi.y = pack_bf16x2(__uint_as_float(r[c + 10]) * inv, __uint_as_float(r[c + 11]) * inv);
          hi.z = pack_bf16x2(__uint_as_float(r[c + 12]) * inv, __uint_as_float(r[c + 13]) * inv);
          hi.w = pack_bf16x2(__uint_as_float(r[c + 14]) * inv, __uint_as_float(r[c + 15]) * inv);
          // the even lane sends its columns c+8.., the odd lane its columns c..
          const uint4 snd = odd ? lo : hi;
          uint4 got;
          got.x = __shfl_xor_sync(0xffffffffu, snd.x, 1);
          got.y = __shfl_xor_sync(0xffffffffu, snd.y, 1);
          got.z = __shfl_xor_sync(0xffffffffu, snd.z, 1);
          got.w = __shfl_xor_sync(0xffffffffu, snd.w, 1);
          const uint4 va = odd ? got : lo;  // row i_a
          const uint4 vb = odd ? hi : got;  // row i_b
          if (i_a < Lq) *reinterpret_cast<uint4*>(row_a + c) = va;
          if (i_b < Lq) *reinterpret_cast<uint4*>(row_b + c) = vb;
        }
        if (wg == 0) {
          // LSE: each group of four lanes gathers its four rows into the first
          // lane, which writes them as one 16-byte store when all four rows
          // exist and the address is 16-byte aligned (scalar stores otherwise).
          const float lse = l_tot > 0.f ? (m_run + __log2f(l_tot)) * kLn2 : -INFINITY;
          float4 l4;
          l4.x = __shfl_sync(0xffffffffu, lse, lane & ~3);
          l4.y = __shfl_sync(0xffffffffu, lse, (lane & ~3) + 1);
          l4.z = __shfl_sync(0xffffffffu, lse, (lane & ~3) + 2);
          l4.w = __shfl_sync(0xffffffffu, lse, (lane & ~3) + 3);
          const int64_t li = row_index(p, w.s, b, hq, i);
          const int i0 = i - (lane & 3);
          const bool vec = (((li - (lane & 3)) & 3) == 0) && (i0 + 3 < Lq);
          if (vec) {
            if ((lane & 3) == 0) *reinterpret_cast<float4*>(p.lse + li) = l4;
          } else if (i < Lq) {
            p.lse[li] = lse;
          }
        }
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
