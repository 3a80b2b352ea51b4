// The fp32 weight stage on given scores (kiattn_weights_from_S): one warp
// per row.  It runs the tensor-core forward's own weight code on the dumped
// scores: the per-row calibration (row_calibration), the grid tables in the
// forward's form (one pair table (G_k, G_{k+1}) per CTA for FWM and the fixed
// step, one table per row for MinMax, both from grid_value), and the element
// function fwd_weights2<V, true> (two scores at a time, as packed fp32
// pairs) that the forward's sweep 2 calls on every unit, compiled for the
// same operator variant V; keys past the row's last visible one go through it
// too and are zeroed afterwards, as the forward's masked keys are.  The bins
// and t written out are the grid positions fwd_weights2 returns, so a
// bit-exact match against the oracle's fp32 definition pins the forward's
// weights, bins and t themselves.
#pragma once
#include "kia_fast.cuh"

namespace kia {

constexpr int kWeightsWarps = 4;

template <class V>
__global__ void __launch_bounds__(32 * kWeightsWarps)
weights_from_S_kernel(const float* __restrict__ S, int rows, int cols,
                      const int* __restrict__ row_len, OpParams p, float* __restrict__ w,
                      int* __restrict__ bin, float* __restrict__ tout, float* __restrict__ row_m,
                      float* __restrict__ row_n) {
  // FWM and the fixed step: the forward's per-CTA pairs (G_k, G_{k+1}) and
  // the tail's zero pair at K
  __shared__ float2 sPair[V::FWM ? KIA_MAX_KCAP + 1 : 1];
  // MinMax: one grid per row, as the forward's per-row table
  __shared__ float sTab[kWeightsWarps][V::MINMAX ? KIA_MAX_K + 1 : 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if constexpr (V::FWM) {
    for (int k = (int)threadIdx.x; k <= p.K; k += (int)blockDim.x)
      sPair[k] = k < p.K ? make_float2(grid_value(k, p.fwm_h), grid_value(k + 1, p.fwm_h))
                         : make_float2(0.0f, 0.0f);
    __syncthreads();
  }
  const int row = blockIdx.x * kWeightsWarps + warp;
  if (row >= rows) return;
  const float* s = S + (size_t)row * cols;
  int L = row_len[row];
  L = L < 1 ? 1 : (L > cols ? cols : L);
  // row extrema (section 3: calibration statistics); max and min are exact
  // in any order
  float m = -INFINITY, n = INFINITY;
  for (int j = lane; j < L; j += 32) {
    const float x = s[j];
    m = fmaxf(m, x);
    n = fminf(n, x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    n = fminf(n, __shfl_xor_sync(0xffffffffu, n, o));
  }
  if (lane == 0) {
    if (row_m) row_m[row] = m;
    if (row_n) row_n[row] = n;
  }
  if constexpr (!V::MINMAX) n = m;   // as the forward: FWM does not use the row minimum
  const RowCal rc = row_calibration(p, m, n);
  if constexpr (V::MINMAX) {
    // the forward's per-row grid: all ones on a degenerate row (rh = 0 then
    // puts every key on node 0, weight 1)
    const bool degen = rc.h == 0.0f;
    for (int k = lane; k <= p.K; k += 32) sTab[warp][k] = degen ? 1.0f : grid_value(k, rc.h);
    __syncwarp();
  }
  const float Kf = p.Kf, Km1f = (float)(p.K - 1);
  // one key's outputs from its grid position and weights
  auto put = [&](int j, const Pos& pos, float wf) {
    const bool vis = j < L;
    const bool tail = V::FWM && pos.u > Kf;
    const bool live = vis && !tail;
    int b = pos.k;
    if constexpr (V::NEAREST) b += pos.t >= 0.5f ? 1 : 0;
    w[(size_t)row * cols + j] = vis ? wf : 0.0f;
    if (bin) bin[(size_t)row * cols + j] = live ? b : -1;
    if (tout) tout[(size_t)row * cols + j] = live ? pos.t : 0.0f;
  };
  // keys j and j + 32 as one packed pair, as the forward's sweep 2 computes
  // its scores
  auto run = [&](const auto& grid) {
    for (int j = lane; j < cols; j += 64) {
      const int j1 = j + 32;
      const float x0 = s[j], x1 = j1 < cols ? s[j1] : x0;
      float2 wf, wl;
      const Pos2 ps = fwd_weights2<V, true>(grid, rc.m, rc.rh, Kf, Km1f, x0, x1, wf, wl);
      put(j, ps.a, wf.x);
      if (j1 < cols) put(j1, ps.b, wf.y);
    }
  };
  if constexpr (V::MINMAX) run(GridF{sTab[warp], 1});
  else run(make_gridz(sPair, p.K));
}

}  // namespace kia
