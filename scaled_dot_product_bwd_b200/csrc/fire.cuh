// fire.cuh -- FIRE relative-position bias (Li et al. 2023, "Functional
// Interpolation for Relative Positions Improves Long Context Transformers";
// named by the catie-aq/flashT5 README among the positional schemes it means
// to support) as a table over the distances j - i, and the gradients of its
// parameters from the table's gradient.
//
//   x(r) = psi(|r|) / psi(threshold),  psi(t) = log(c t + 1)
//   table[r + Lq - 1, h] = b2[h] + sum_w w2[h, w] relu(w1[w] x(r) + b1[w])
//
// for r = j - i in [-(Lq - 1), Lk - 1] (threshold >= Lq - 1 makes the
// paper's psi(max(threshold, i)) equal psi(threshold) on every row).
// Float32 arithmetic; every sum over table rows is taken in a fixed order.
#pragma once

#include <stdint.h>

namespace sdpa {

struct FireArgs {
  const float* w1;   // [W]
  const float* b1;   // [W]
  const float* w2;   // [H, W]
  const float* b2;   // [H]
  float c, thr;
  int W, H, Lq, Lk;
};

__device__ __forceinline__ float fire_x(const FireArgs& f, int row, float& num, float& den,
                                        float& dist) {
  dist = fabsf(static_cast<float>(row - (f.Lq - 1)));
  num = log1pf(f.c * dist);
  den = log1pf(f.c * f.thr);
  return num / den;
}

// table[row * H + h], one thread per entry
__global__ void __launch_bounds__(256) fire_table_kernel(const FireArgs f, float* table) {
  const int64_t R = static_cast<int64_t>(f.Lq) + f.Lk - 1;
  const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (idx >= R * f.H) return;
  const int row = static_cast<int>(idx / f.H);
  const int h = static_cast<int>(idx - static_cast<int64_t>(row) * f.H);
  float num, den, dist;
  const float x = fire_x(f, row, num, den, dist);
  const float* w2 = f.w2 + static_cast<int64_t>(h) * f.W;
  float acc = f.b2[h];
  for (int w = 0; w < f.W; ++w) acc = fmaf(w2[w], fmaxf(fmaf(f.w1[w], x, f.b1[w]), 0.f), acc);
  table[idx] = acc;
}

// Backward, stage 1, one thread per table row: the hidden activations, the
// gradient reaching each pre-activation, and the gradient reaching c and the
// threshold through x (workspace, row-major per row).
struct FireWork {
  float* hid;    // [R, W]
  float* dpre;   // [R, W]
  float* x;      // [R]
  float* dxc;    // [R]: d loss / dx * dx / dc
  float* dxt;    // [R]: d loss / dx * dx / dthreshold
};

__global__ void __launch_bounds__(128) fire_rows_kernel(const FireArgs f, const float* g,
                                                        const FireWork ws) {
  const int R = f.Lq + f.Lk - 1;
  const int row = blockIdx.x * 128 + static_cast<int>(threadIdx.x);
  if (row >= R) return;
  float num, den, dist;
  const float x = fire_x(f, row, num, den, dist);
  const float* gr = g + static_cast<int64_t>(row) * f.H;
  float dx = 0.f;
  for (int w = 0; w < f.W; ++w) {
    const float pre = fmaf(f.w1[w], x, f.b1[w]);
    float dh = 0.f;
    for (int h = 0; h < f.H; ++h) dh = fmaf(gr[h], f.w2[static_cast<int64_t>(h) * f.W + w], dh);
    const float dp = pre > 0.f ? dh : 0.f;
    ws.hid[static_cast<int64_t>(row) * f.W + w] = fmaxf(pre, 0.f);
    ws.dpre[static_cast<int64_t>(row) * f.W + w] = dp;
    dx = fmaf(dp, f.w1[w], dx);
  }
  const float ct1 = fmaf(f.c, f.thr, 1.f);
  const float dxdc = (dist / fmaf(f.c, dist, 1.f)) / den - num * (f.thr / ct1) / (den * den);
  const float dxdt = -num * (f.c / ct1) / (den * den);
  ws.x[row] = x;
  ws.dxc[row] = dx * dxdc;
  ws.dxt[row] = dx * dxdt;
}

// Backward, stage 2: one block per output value, in the order d_w2 [H, W],
// d_b2 [H], d_w1 [W], d_b1 [W], d_c, d_threshold.  Thread t adds rows
// t, t + 256, ... in order; the 256 partial sums meet in a fixed tree.
struct FireOut {
  float* w1;
  float* b1;
  float* w2;
  float* b2;
  float* c_thr;  // [2]
};

__global__ void __launch_bounds__(256) fire_reduce_kernel(const FireArgs f, const float* g,
                                                          const FireWork ws, const FireOut out) {
  __shared__ float red[256];
  const int R = f.Lq + f.Lk - 1;
  const int64_t o = blockIdx.x;
  const int64_t n_w2 = static_cast<int64_t>(f.H) * f.W;
  float acc = 0.f;
  for (int row = static_cast<int>(threadIdx.x); row < R; row += 256) {
    float term;
    if (o < n_w2) {
      const int h = static_cast<int>(o / f.W), w = static_cast<int>(o % f.W);
      term = g[static_cast<int64_t>(row) * f.H + h] * ws.hid[static_cast<int64_t>(row) * f.W + w];
    } else if (o < n_w2 + f.H) {
      term = g[static_cast<int64_t>(row) * f.H + (o - n_w2)];
    } else if (o < n_w2 + f.H + f.W) {
      const int w = static_cast<int>(o - n_w2 - f.H);
      term = ws.dpre[static_cast<int64_t>(row) * f.W + w] * ws.x[row];
    } else if (o < n_w2 + f.H + 2 * f.W) {
      term = ws.dpre[static_cast<int64_t>(row) * f.W + (o - n_w2 - f.H - f.W)];
    } else if (o == n_w2 + f.H + 2 * f.W) {
      term = ws.dxc[row];
    } else {
      term = ws.dxt[row];
    }
    acc += term;
  }
  red[threadIdx.x] = acc;
  for (int w = 128; w > 0; w >>= 1) {
    __syncthreads();
    if (static_cast<int>(threadIdx.x) < w) red[threadIdx.x] += red[threadIdx.x + w];
  }
  if (threadIdx.x != 0) return;
  const float v = red[0];
  if (o < n_w2) out.w2[o] = v;
  else if (o < n_w2 + f.H) out.b2[o - n_w2] = v;
  else if (o < n_w2 + f.H + f.W) out.w1[o - n_w2 - f.H] = v;
  else if (o < n_w2 + f.H + 2 * f.W) out.b1[o - n_w2 - f.H - f.W] = v;
  else out.c_thr[o - n_w2 - f.H - 2 * f.W] = v;
}

}  // namespace sdpa
