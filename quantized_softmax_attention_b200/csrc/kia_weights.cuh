// The fp32 weight stage on given scores (kiattn_weights_from_S): one warp
// per row.  It runs exactly the per-row calibration and per-element grid
// arithmetic of the fused kernels (kia_common.cuh), so a bit-exact match
// against the oracle's fp32 definition here pins the fused kernels' weight
// arithmetic too.
#pragma once
#include "kia_common.cuh"

namespace kia {

constexpr int kWeightsWarps = 4;

__global__ void __launch_bounds__(32 * kWeightsWarps)
weights_from_S_kernel(const float* __restrict__ S, int rows, int cols,
                      const int* __restrict__ row_len, OpParams p, float* __restrict__ w,
                      int* __restrict__ bin, float* __restrict__ tout, float* __restrict__ row_m,
                      float* __restrict__ row_n) {
  __shared__ float sG[kWeightsWarps][KIA_MAX_KCAP + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWeightsWarps + warp;
  if (row >= rows) return;
  const float* s = S + (size_t)row * cols;
  int L = row_len[row];
  L = L < 1 ? 1 : (L > cols ? cols : L);
  // row extrema (section 3: calibration statistics)
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
  const RowCal c = row_calibration(p, m, n);
  const bool degen = (p.cal == KIA_CAL_MINMAX) && c.h == 0.0f;
  if (!degen) {
    for (int k = lane; k <= p.K; k += 32) sG[warp][k] = grid_value(k, c.h);
  }
  __syncwarp();
  for (int j = lane; j < cols; j += 32) {
    float wj = 0.0f, tj = 0.0f;
    int bj = -1;
    if (j < L) {
      if (degen) {
        wj = 1.0f;
        bj = 0;
      } else {
        const GridPos g = grid_position(p, c, s[j]);
        if (!g.tail) {
          if (p.rec == KIA_REC_LERP) {
            wj = lerp_weight(g.t, sG[warp][g.k], sG[warp][g.k + 1]);
            bj = g.k;
          } else {
            bj = nearest_node(g);
            wj = sG[warp][bj];
          }
          tj = g.t;
        }
      }
    }
    w[(size_t)row * cols + j] = wj;
    if (bin) bin[(size_t)row * cols + j] = bj;
    if (tout) tout[(size_t)row * cols + j] = tj;
  }
}

}  // namespace kia
