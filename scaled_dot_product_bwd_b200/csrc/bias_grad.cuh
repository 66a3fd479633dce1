// Bias gradients.  The scores are linear in an additive bias, so a dense
// bias's gradient is dS summed over each index the bias is broadcast along
// (from the fp32 dS the dQ kernel stores in its store mode), a T5 table
// entry's gradient is dS summed over every (b, i, j) whose distance j - i
// falls in its bucket (from the per-bucket sums the dQ kernel writes in its
// bucket mode), a relative-position table row's over its distance (from the
// per-warp diagonal sums of its diagonal mode), and an ALiBi slope's is
// minus the sum of |j - i| dS (from the per-warp sums of its moment mode;
// catie-aq/flashT5 README, "Full attention biases" and
// "T5-like relative position encoding biases": a learnable bias needs these
// to train).
//
// Every kernel here is bandwidth-bound and deterministic: each output is a
// sum taken in one fixed order (fixed chunking of the reduced index, chunks
// added in ascending order, a fixed shared-memory tree), independent of
// timing, so repeated calls give identical bits.
#pragma once

#include "attn_common.cuh"

namespace sdpa {

// Blocks the reduction grids aim for (8 per SM on a 148-SM part); a constant,
// not the device's SM count, so the chunking -- and with it the rounding of
// every sum -- is the same on every device.
constexpr int64_t kReduceTargetBlocks = 1184;

// ---------------------------------------------------------------------
// dS entries the backward never visits: for query row i, the key tiles
// outside [nlo, nhi) of i's query tile (key_tile_range), which hold no key
// visible from any row of the tile.  The dQ kernel writes every column of
// the tiles inside the band (masked keys as 0); this fills the rest with 0.
__device__ __forceinline__ void zero_span(float* row, int j0, int j1) {
  // j0 is 0 or a multiple of the tile width, so row + j0 is 16-byte aligned
  for (int j = j0 + 4 * static_cast<int>(threadIdx.x); j < j1; j += 4 * static_cast<int>(blockDim.x)) {
    if (j + 4 <= j1) {
      *reinterpret_cast<float4*>(row + j) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      for (int t = j; t < j1; ++t) row[t] = 0.f;
    }
  }
}

__global__ void __launch_bounds__(256) ds_zero_outside_band_kernel(const AttnParams p) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.Hq * p.Lq;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int i = static_cast<int>(r % p.Lq);
    const int64_t bh = r / p.Lq;
    const int hq = static_cast<int>(bh % p.Hq);
    const int b = static_cast<int>(bh / p.Hq);
    int nlo, nhi;
    key_tile_range(p, p.Lq, p.Lk, (i / kTile) * kTile, kTile, nlo, nhi);
    float* row = p.ds_out + static_cast<int64_t>(b) * p.sd_b + static_cast<int64_t>(hq) * p.sd_h +
                 static_cast<int64_t>(i) * p.sd_i;
    // [0, nlo * 128) and [nhi * 128, Lk); with an empty band the two cover the row
    zero_span(row, 0, min(nlo * kTile, p.Lk));
    zero_span(row, min(nhi * kTile, p.Lk), p.Lk);
  }
}

// ---------------------------------------------------------------------
// Dense bias broadcast along some of (b, h, i): out[b', h', i', j] = sum of
// dS[b, h, i, j] over the broadcast indices.  Output rows o enumerate the
// kept indices (extents eb, eh, ei: the full extent where kept, else 1);
// the reduced index t enumerates the broadcast ones (extents rb, rh, ri).
struct DenseReduce {
  const float* ds;               // [B, Hq, L, lp] fp32, row stride lp (a multiple of 8)
  int64_t ds_b, ds_h, ds_i;
  float* out;                    // the bias gradient, element strides o_b, o_h, o_i
  int64_t o_b, o_h, o_i;
  int L;
  int eb, eh, ei;                // kept extents
  int rb, rh, ri;                // reduced extents
  int64_t n_out, n_red;          // eb*eh*ei, rb*rh*ri
  int jblocks;                   // ceil(L / 256)
  int chunks;                    // pieces of the reduced index (grid y)
  int64_t rchunk;                // reduced indices per piece
  float* partial;                // [chunks, n_out, lp] when chunks > 1
  int64_t lp;
};

__device__ __forceinline__ void dense_out_index(const DenseReduce& a, int64_t o, int& b, int& h,
                                                int& i) {
  i = static_cast<int>(o % a.ei);
  const int64_t r = o / a.ei;
  h = static_cast<int>(r % a.eh);
  b = static_cast<int>(r / a.eh);
}

__global__ void __launch_bounds__(256) dense_bias_reduce_kernel(const DenseReduce a) {
  const int z = blockIdx.y;
  const int64_t t0 = static_cast<int64_t>(z) * a.rchunk;
  const int64_t t1 = min(a.n_red, t0 + a.rchunk);
  const int64_t work = a.n_out * a.jblocks;
  for (int64_t w = blockIdx.x; w < work; w += gridDim.x) {
    const int64_t o = w / a.jblocks;
    const int j = static_cast<int>(w % a.jblocks) * 256 + static_cast<int>(threadIdx.x);
    if (j >= a.L) continue;
    int ob, oh, oi;
    dense_out_index(a, o, ob, oh, oi);
    float acc = 0.f;
    // reduced index t = (tb, th, ti), ti fastest; exactly one of o's and t's
    // coordinate is non-zero along each axis
    int ti = static_cast<int>(t0 % a.ri);
    int th = static_cast<int>((t0 / a.ri) % a.rh);
    int tb = static_cast<int>(t0 / (static_cast<int64_t>(a.ri) * a.rh));
    for (int64_t t = t0; t < t1; ++t) {
      acc += a.ds[static_cast<int64_t>(ob + tb) * a.ds_b + static_cast<int64_t>(oh + th) * a.ds_h +
                  static_cast<int64_t>(oi + ti) * a.ds_i + j];
      if (++ti == a.ri) {
        ti = 0;
        if (++th == a.rh) {
          th = 0;
          ++tb;
        }
      }
    }
    if (a.chunks == 1)
      a.out[ob * a.o_b + oh * a.o_h + oi * a.o_i + j] = acc;
    else
      a.partial[(static_cast<int64_t>(z) * a.n_out + o) * a.lp + j] = acc;
  }
}

// Second stage when the reduced index was split: add the pieces in order.
__global__ void __launch_bounds__(256) dense_bias_combine_kernel(const DenseReduce a) {
  const int64_t work = a.n_out * a.jblocks;
  for (int64_t w = blockIdx.x; w < work; w += gridDim.x) {
    const int64_t o = w / a.jblocks;
    const int j = static_cast<int>(w % a.jblocks) * 256 + static_cast<int>(threadIdx.x);
    if (j >= a.L) continue;
    float acc = 0.f;
    for (int z = 0; z < a.chunks; ++z) acc += a.partial[(static_cast<int64_t>(z) * a.n_out + o) * a.lp + j];
    int ob, oh, oi;
    dense_out_index(a, o, ob, oh, oi);
    a.out[ob * a.o_b + oh * a.o_h + oi * a.o_i + j] = acc;
  }
}

// ---------------------------------------------------------------------
// Relative-position table gradient.  The bias depends on j - i alone, so
// sum dS along each diagonal r = j - i (r in [-(L-1), L-1]).
struct T5Reduce {
  const float* partial;          // diagonal sums [Hq, 2L - 1]: partial[h, r + L - 1]
  int Hq, L;
  float* out;                    // table gradient [2L - 1, Hq]
};

// ---------------------------------------------------------------------
// The same diagonal sums from the dQ kernel's per-warp partials (its
// diagonal mode), without the L x L dS: first each visited 128 x 128 tile's
// 255 diagonals D = j - i - (n0 - m0) in [-127, 127], then the per-head
// totals.  Both sum in an order fixed by the shape alone.
struct DiagFold {
  const float* warp_part;        // [B, Hq, nqt, ntk, 8 warps, 2 halves, 64]
  float* tile_diag;              // [B, Hq, nqt, ntk, 256]
  float* band;                   // [B, Hq, 2 nqt - 1 tile offsets, 256]
  float* diag;                   // [Hq, 2L - 1]: diag[h, r + L - 1]
  int B, Hq, L, nqt, ntk;
};

// One block per (query tile, key tile, b * Hq + h), thread D + 127: adds
// the warp-half pieces that cover tile diagonal D, warps then halves in
// index order.  Warp w (rows 32 (w % 4).., warpgroup w / 4 holding keys
// 64 (w / 4)..) half h covers D = 64 (w / 4) + 32 h - 32 (w % 4) + t,
// t in [-31, 31].  Tiles outside the mask band are skipped (never read).
__global__ void __launch_bounds__(256) diag_tile_fold_kernel(const DiagFold a, const AttnParams p) {
  const int mi = blockIdx.x, ni = blockIdx.y, bh = blockIdx.z;
  int nlo, nhi;
  key_tile_range(p, a.L, a.L, mi * kTile, kTile, nlo, nhi);
  if (ni < nlo || ni >= nhi) return;
  const int D = static_cast<int>(threadIdx.x) - 127;
  if (D > 127) return;
  const int64_t blk = (static_cast<int64_t>(bh) * a.nqt + mi) * a.ntk + ni;
  const float* src = a.warp_part + blk * 1024;
  float acc = 0.f;
  for (int w = 0; w < 8; ++w) {
    for (int h = 0; h < 2; ++h) {
      const int t = D - 64 * (w >> 2) - 32 * h + 32 * (w & 3);
      if (t < -31 || t > 31) continue;
      acc += src[(w * 2 + h) * 64 + (t <= 0 ? t + 31 : 31 + t)];
    }
  }
  a.tile_diag[blk * 256 + threadIdx.x] = acc;
}

// band[b, h, dt + nt - 1, D + 127] = sum over query tiles mi (four
// interleaved accumulators, mi % 4, added in a fixed tree) of the tile
// diagonal D of tile (mi, mi + dt): one block per (tile offset dt, head,
// batch entry), thread D + 127, so a warp reads 32 consecutive diagonals of
// one tile.
__global__ void __launch_bounds__(256) diag_band_kernel(const DiagFold a, const AttnParams p) {
  const int nb = 2 * a.nqt - 1;
  const int dt = static_cast<int>(blockIdx.x) - (a.nqt - 1);
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int D = static_cast<int>(threadIdx.x);  // D + 127
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (D < 255) {
    const int mi0 = max(0, -dt), mi1 = min(a.nqt, a.ntk - dt);
#pragma unroll 4
    for (int mi = mi0; mi < mi1; ++mi) {
      int nlo, nhi;
      key_tile_range(p, a.L, a.L, mi * kTile, kTile, nlo, nhi);
      const int ni = mi + dt;
      if (ni < nlo || ni >= nhi) continue;
      const int64_t blk = ((static_cast<int64_t>(b) * a.Hq + h) * a.nqt + mi) * a.ntk + ni;
      acc[mi & 3] += a.tile_diag[blk * 256 + D];
    }
  }
  a.band[((static_cast<int64_t>(b) * a.Hq + h) * nb + blockIdx.x) * 256 + D] =
      (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

// diag[h, r + L - 1]: over b, the band sums of the (at most two) tile
// offsets dt with r - 128 dt in [-127, 127], the lower dt first.
__global__ void __launch_bounds__(128) diag_total_kernel(const DiagFold a) {
  const int nd = 2 * a.L - 1;
  const int nb = 2 * a.nqt - 1;
  const int dr = blockIdx.x * 128 + static_cast<int>(threadIdx.x);
  if (dr >= nd) return;
  const int r = dr - (a.L - 1);
  const int h = blockIdx.y;
  // lowest dt with r - 128 dt <= 127: ceil((r - 127) / 128)
  const int dt0 = r - 127 >= 0 ? r / 128 : -((127 - r) / 128);
  float acc = 0.f;
  for (int b = 0; b < a.B; ++b) {
    for (int dt = dt0; dt <= dt0 + 1; ++dt) {
      const int Dv = r - kTile * dt;
      if (Dv < -127 || dt < -(a.nqt - 1) || dt > a.nqt - 1) continue;
      acc += a.band[((static_cast<int64_t>(b) * a.Hq + h) * nb + dt + a.nqt - 1) * 256 + Dv + 127];
    }
  }
  a.diag[static_cast<int64_t>(h) * nd + dr] = acc;
}

// T5: out[k, h] = sum over (b, query tile, warp) of the dQ kernel's per-bucket
// partial sums (its bucket mode: per (b, h, query tile, warp) one sum per
// bucket over every key tile); one block per (k, h), thread t adds the
// entries t, t + 256, ... in order, then a fixed tree over the threads.
struct T5BucketReduce {
  const float* part;             // [B, Hq, nqt, 8, num_buckets]
  float* out;                    // [num_buckets, Hq]
  int B, Hq, nqt, num_buckets;
};

__global__ void __launch_bounds__(256) t5_bucket_reduce_kernel(const T5BucketReduce a) {
  __shared__ float red[256];
  const int k = blockIdx.x;
  const int h = blockIdx.y;
  const int per_b = a.nqt * 8;
  float acc = 0.f;
  for (int e = static_cast<int>(threadIdx.x); e < a.B * per_b; e += 256) {
    const int b = e / per_b;
    const int rem = e - b * per_b;  // query tile * 8 + warp
    acc += a.part[((static_cast<int64_t>(b) * a.Hq + h) * per_b + rem) * a.num_buckets + k];
  }
  red[threadIdx.x] = acc;
  for (int w = 128; w > 0; w >>= 1) {
    __syncthreads();
    if (static_cast<int>(threadIdx.x) < w) red[threadIdx.x] += red[threadIdx.x + w];
  }
  if (threadIdx.x == 0) a.out[static_cast<int64_t>(k) * a.Hq + h] = red[0];
}

// REL: out[(r + L - 1) * Hq + h] = diagonal sum of r (a transpose).
__global__ void __launch_bounds__(256) rel_table_grad_kernel(const T5Reduce a) {
  const int nd = 2 * a.L - 1;
  const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (idx >= static_cast<int64_t>(nd) * a.Hq) return;
  const int row = static_cast<int>(idx / a.Hq);
  const int h = static_cast<int>(idx - static_cast<int64_t>(row) * a.Hq);
  a.out[idx] = a.partial[static_cast<int64_t>(h) * nd + row];
}

// ALiBi: the bias -m_h |j - i| is linear in the slope, so its gradient is
// -sum of |j - i| dS over (b, i, j).  The dQ kernel's moment mode writes
// that sum per (b, h, query tile, key tile, warp) for the tiles in the
// mask band; out[h] adds them up, one block per head: thread t takes the
// entries t, t + 1024, ... in order (entries of tiles outside the band are
// never written and are skipped), then a fixed tree over the threads.
struct AlibiMoment {
  const float* part;             // [B, Hq, nt, nt, 8]
  float* out;                    // [Hq]
  int B, Hq, L, nt;
};

__global__ void __launch_bounds__(1024) alibi_moment_kernel(const AlibiMoment a, const AttnParams p) {
  __shared__ float red[1024];
  const int h = blockIdx.x;
  const int64_t per_b = static_cast<int64_t>(a.nt) * a.nt * 8;
  float acc = 0.f;
  for (int64_t e = threadIdx.x; e < a.B * per_b; e += 1024) {
    const int b = static_cast<int>(e / per_b);
    const int64_t rem = e - b * per_b;
    const int mi = static_cast<int>(rem / (a.nt * 8));
    const int ni = static_cast<int>((rem / 8) % a.nt);
    int nlo, nhi;
    key_tile_range(p, a.L, a.L, mi * kTile, kTile, nlo, nhi);
    if (ni < nlo || ni >= nhi) continue;
    acc += a.part[(static_cast<int64_t>(b) * a.Hq + h) * per_b + rem];
  }
  red[threadIdx.x] = acc;
  for (int w = 512; w > 0; w >>= 1) {
    __syncthreads();
    if (static_cast<int>(threadIdx.x) < w) red[threadIdx.x] += red[threadIdx.x + w];
  }
  if (threadIdx.x == 0) a.out[h] = -red[0];
}

}  // namespace sdpa
