// Backward row passes around the main backward kernels:
//   prep    - (exact-fp32 path) centering D_i = dO_i . O_bar_i (O_bar = O, or
//             O_L for Prob-STE), clears the row accumulators, checks the
//             stats header against the call;
//   calib   - (exact-fp32 path) calibration coefficients per row from A, C
//             and the gradient mode (section 3 Calibration gradients;
//             Appendix B), applied as the 2-sparse update at the argmax /
//             argmin keys;
//   scan    - the zero-sum projection's common-mode shift c_i, which adds
//             c_i to every visible score gradient of row i: dQ_i += c_i sum_J k_j
//             and dK_j += sum_{i sees j} c_i q_i (prefix / suffix sums);
//   decomp  - the fixed-upstream gradient decomposition per row over a dS
//             dump (Appendix F).
// All are bandwidth-bound row passes.
#pragma once
#include "kia_elem.cuh"
#include "kia_stats.cuh"

namespace kia {

constexpr int kRowWarps = 8;  // warps (rows) per block in the row passes

template <int D>
__global__ void __launch_bounds__(32 * kRowWarps)
bwd_prep_kernel(const float* __restrict__ O, const float* __restrict__ dO, StatsView st, WorkView wk,
                float* __restrict__ dQ_zero, OpParams p, int B, int H, int T) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long rows = (long long)B * H * T;
  const long long row = (long long)blockIdx.x * kRowWarps + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    const bool ok = header_matches(st.header, B, H, T, D, p);
    *wk.status = ok ? 0 : 1;
    if (!ok) atomicExch(&g_kia_device_error, KIA_ERR_STATS_MISMATCH);
  }
  if (row >= rows) return;
  const float* ob = (st.OL ? st.OL : O) + row * D;
  const float* g = dO + row * D;
  float acc = 0.0f;
#pragma unroll
  for (int c = lane; c < D; c += 32) acc = fmaf(g[c], ob[c], acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    wk.D[row] = acc;
    wk.A[row] = 0.0f;
    wk.C[row] = 0.0f;
    wk.gm[row] = 0.0f;
    wk.gn[row] = 0.0f;
  }
  if (dQ_zero) {
#pragma unroll
    for (int c = lane; c < D; c += 32) dQ_zero[row * D + c] = 0.0f;
  }
}

// Calibration coefficients (Appendix B):
//   MinMax: g_m = A / h + C / K,  g_n = -C / K;   FWM: g_m = A / h, g_n = 0.
// full: both; detach: none; max-only: g_m; min-only: g_n; projection: the
// shift c = A / (h |J_i|) on every visible key (applied by the scan pass).
template <int D>
__global__ void __launch_bounds__(32 * kRowWarps)
bwd_calib_kernel(const float* __restrict__ Q, const float* __restrict__ Kt, StatsView st,
                 WorkView wk, float* __restrict__ dQ, float* __restrict__ dK,
                 float* __restrict__ dS_dbg, OpParams p, int B, int H, int T) {
  if (*wk.status != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long rows = (long long)B * H * T;
  const long long row = (long long)blockIdx.x * kRowWarps + warp;
  if (row >= rows || p.softmax || p.grad == KIA_GRAD_DETACH) return;
  const int i = (int)(row % T);
  const long long bh = row / T;
  const float rh = st.rh[row];
  if (rh == 0.0f) return;  // degenerate row: no calibration term
  const float A = wk.A[row], C = wk.C[row];
  const int L = p.causal ? i + 1 : T;
  if (p.grad == KIA_GRAD_PROJECT) {
    const float c = A * rh / (float)L;
    if (lane == 0) wk.gm[row] = c;
    if (dS_dbg) {
      float* ds = dS_dbg + row * (long long)T;
      for (int j = lane; j < L; j += 32) ds[j] += c;
    }
    return;
  }
  float gm = 0.0f, gn = 0.0f;
  const float gm_full = (p.cal == KIA_CAL_MINMAX) ? A * rh + C / p.Kf : A * rh;
  const float gn_full = (p.cal == KIA_CAL_MINMAX) ? -C / p.Kf : 0.0f;
  if (p.grad == KIA_GRAD_FULL || p.grad == KIA_GRAD_MAX_ONLY) gm = gm_full;
  if (p.grad == KIA_GRAD_FULL || p.grad == KIA_GRAD_MIN_ONLY) gn = gn_full;
  const int am = wk.am[row], an = wk.an[row];
  if (lane == 0) {
    wk.gm[row] = gm;
    wk.gn[row] = gn;
    if (dS_dbg) {
      float* ds = dS_dbg + row * (long long)T;
      ds[am] += gm;
      ds[an] += gn;
    }
  }
  const size_t base = (size_t)bh * T * D;
  const float* q = Q + row * D;
  const float* ka = Kt + base + (size_t)am * D;
  const float* kn = Kt + base + (size_t)an * D;
#pragma unroll
  for (int c = lane; c < D; c += 32) {
    dQ[row * D + c] += gm * ka[c] + gn * kn[c];
    if (gm != 0.0f) atomicAdd(dK + base + (size_t)am * D + c, gm * q[c]);
    if (gn != 0.0f) atomicAdd(dK + base + (size_t)an * D + c, gn * q[c]);
  }
}

// Zero-sum projection, common-mode part: dQ_i += c_i sum_{j in J_i} k_j and
// (with_dk) dK_j += sum_{i : j in J_i} c_i q_i.  Block = (bh, 32-column chunk,
// 128-row chunk); each of its 8 warps owns 16 consecutive rows.  The sums
// over the rows before (for dQ) and after (for dK) the chunk are re-read by
// the block (from L2 after the first blocks of a head), the in-chunk prefix
// is exclusive across warps; fp64 running sums.
constexpr int kScanRows = 128, kScanWarps = 8;

template <int D>
__global__ void __launch_bounds__(32 * kScanWarps)
bwd_project_scan_kernel(const float* __restrict__ Q, const float* __restrict__ Kt, WorkView wk,
                        float* __restrict__ dQ, float* __restrict__ dK, OpParams p, int T,
                        int with_dk) {
  if (*wk.status != 0) return;
  __shared__ double sK[kScanWarps][32];   // per-warp partial sums of k (rows before / own)
  __shared__ double sQ[kScanWarps][32];   // per-warp partial sums of c q (rows after / own)
  const int bh = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int col = blockIdx.y * 32 + lane;
  const int c0 = blockIdx.z * kScanRows, c1 = min(T, c0 + kScanRows);
  const size_t base = (size_t)bh * T * D;
  const float* cc = wk.gm + (size_t)bh * T;
  const bool causal = p.causal;
  // rows outside the chunk that every row of the chunk sees
  const int kb = causal ? c0 : 0, ke = causal ? c0 : T;    // dQ: keys [0, c0) (or all)
  double ok = 0.0, oq = 0.0;
  if (causal) {
    for (int r = warp; r < kb; r += kScanWarps) ok += (double)Kt[base + (size_t)r * D + col];
    if (with_dk)
      for (int r = c1 + warp; r < T; r += kScanWarps)
        oq += (double)cc[r] * (double)Q[base + (size_t)r * D + col];
  } else {
    for (int r = warp; r < ke; r += kScanWarps) {
      ok += (double)Kt[base + (size_t)r * D + col];
      if (with_dk) oq += (double)cc[r] * (double)Q[base + (size_t)r * D + col];
    }
  }
  sK[warp][lane] = ok;
  sQ[warp][lane] = oq;
  __syncthreads();
  double outK = 0.0, outQ = 0.0;
#pragma unroll
  for (int w = 0; w < kScanWarps; ++w) { outK += sK[w][lane]; outQ += sQ[w][lane]; }
  __syncthreads();
  if (!causal) {
    for (int r = c0 + warp; r < c1; r += kScanWarps) {
      dQ[base + (size_t)r * D + col] += (float)((double)cc[r] * outK);
      if (with_dk) dK[base + (size_t)r * D + col] += (float)outQ;
    }
    return;
  }
  // causal: this warp's 16 rows, with the exclusive in-chunk prefix (keys)
  // and suffix (queries) of the other warps' rows
  const int per = kScanRows / kScanWarps;
  const int r0 = c0 + warp * per, r1 = min(c1, r0 + per);
  double mk = 0.0, mq = 0.0;
  for (int r = r0; r < r1; ++r) {
    mk += (double)Kt[base + (size_t)r * D + col];
    if (with_dk) mq += (double)cc[r] * (double)Q[base + (size_t)r * D + col];
  }
  sK[warp][lane] = mk;
  sQ[warp][lane] = mq;
  __syncthreads();
  double runK = outK, runQ = outQ;
#pragma unroll
  for (int w = 0; w < kScanWarps; ++w) {
    if (w < warp) runK += sK[w][lane];
    if (w > warp) runQ += sQ[w][lane];
  }
  for (int r = r0; r < r1; ++r) {
    runK += (double)Kt[base + (size_t)r * D + col];
    dQ[base + (size_t)r * D + col] += (float)((double)cc[r] * runK);
  }
  if (!with_dk) return;
  for (int r = r1 - 1; r >= r0; --r) {
    runQ += (double)cc[r] * (double)Q[base + (size_t)r * D + col];
    dK[base + (size_t)r * D + col] += (float)runQ;
  }
}

// Fixed-upstream decomposition of the score gradient (Appendix F; Table
// S24): per row, ||dS_i||^2 over the visible keys and the squared norms of
// the maximum- and minimum-side calibration terms the backward applied.  One
// warp per row, fp64 sums.
__global__ void __launch_bounds__(32 * kRowWarps)
grad_decomp_kernel(const float* __restrict__ dS, WorkView wk, long long rows, int T, int causal,
                   int grad, double* __restrict__ out) {
  if (*wk.status != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * kRowWarps + warp;
  if (row >= rows) return;
  const int i = (int)(row % T);
  const int L = causal ? i + 1 : T;
  const float* ds = dS + row * (long long)T;
  double s2 = 0.0;
  if ((T & 3) == 0 && (reinterpret_cast<uintptr_t>(dS) & 15) == 0) {
    // four 128-key chunks in flight per lane; each float4's four squares are
    // summed in fp32 (exact to 2^-22 relative), the rest in fp64
    for (int j0 = 4 * lane; j0 < L; j0 += 512) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = j0 + 128 * u;
        v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j + 3 < L) {
          v[u] = __ldg(reinterpret_cast<const float4*>(ds + j));
        } else if (j < L) {
          v[u].x = ds[j];
          if (j + 1 < L) v[u].y = ds[j + 1];
          if (j + 2 < L) v[u].z = ds[j + 2];
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        s2 += (double)fmaf(v[u].x, v[u].x, fmaf(v[u].y, v[u].y, fmaf(v[u].z, v[u].z, v[u].w * v[u].w)));
    }
  } else {
    for (int j = lane; j < L; j += 32) s2 = fma((double)ds[j], (double)ds[j], s2);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
  if (lane == 0) {
    const double gm = (double)wk.gm[row], gn = (double)wk.gn[row];
    const bool proj = grad == KIA_GRAD_PROJECT;
    out[3 * row + 0] = s2;
    out[3 * row + 1] = proj ? gm * gm * (double)L : gm * gm;
    out[3 * row + 2] = proj ? 0.0 : gn * gn;
  }
}

}  // namespace kia
