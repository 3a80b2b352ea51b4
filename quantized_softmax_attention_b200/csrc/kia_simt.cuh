// Exact-fp32 path (KIA_GEMM_FP32): every contraction is a plain fp32 FMA
// chain on the CUDA cores, one thread per query row (forward, dQ side) or per
// key row (dK/dV side).  It exists to check the operator at fp32 precision
// (no TF32 operand rounding); the tensor-core path is the fast one.
// Dot products always run over the head dimension in ascending order, so a
// score recomputed in any kernel of this path is bit-identical to the one
// the forward saw.
#pragma once
#include "kia_elem.cuh"
#include "kia_stats.cuh"

namespace kia {

constexpr int kSimtRows = 128;  // rows (threads) per block
constexpr int kSimtKeys = 32;   // keys per shared tile

template <int D>
__device__ __forceinline__ float dot_row(const float* a, const float* b) {
  float s = 0.0f;
#pragma unroll 16
  for (int c = 0; c < D; ++c) s = fmaf(a[c], b[c], s);
  return s;
}

// Load rows r0..r0+nr-1 of a [T, D] matrix into smem tile with row stride ld
// (zeros beyond T).
template <int D>
__device__ __forceinline__ void load_rows(float* tile, int ld, const float* src, int r0, int nr,
                                          int T, bool trunc = false) {
  for (int e = threadIdx.x; e < nr * D; e += blockDim.x) {
    const int rr = e / D, c = e % D;
    const int g = r0 + rr;
    const float x = (g < T) ? src[(size_t)g * D + c] : 0.0f;
    tile[rr * ld + c] = trunc ? tf32_trunc(x) : x;
  }
}

// Grid table for one query-tile block: per-row [k][row] (MinMax) or one
// shared table (FWM); row_state for the calling thread's row.
template <int D>
__global__ void __launch_bounds__(kSimtRows)
simt_fwd_kernel(const float* __restrict__ Q, const float* __restrict__ Kt,
                const float* __restrict__ V, float* __restrict__ O, StatsView st, OpParams p,
                int B, int H, int T) {
  extern __shared__ float sm[];
  float* sQ = sm;                                   // [128][D+1]
  float* sK = sQ + kSimtRows * (D + 1);             // [32][D]
  float* sV = sK + kSimtKeys * D;                   // [32][D]
  float* sTab = sV + kSimtKeys * D;                 // [(K+1)][128] or [K+1]
  const int bh = blockIdx.y;
  const int r = threadIdx.x;
  const int i0 = blockIdx.x * kSimtRows;
  const int i = i0 + r;
  const bool live = i < T;
  const size_t base = (size_t)bh * T * D;
  const int L = live ? (p.causal ? i + 1 : T) : 0;
  const int kend = p.causal ? min(T, i0 + kSimtRows) : T;
  if (blockIdx.x == 0 && blockIdx.y == 0 && r == 0) write_header(st.header, B, H, T, D, p);

  load_rows<D>(sQ, D + 1, Q + base, i0, kSimtRows, T);
  // sweep 1: row statistics (section 3: the grid needs the final extrema)
  float m = -INFINITY, n = INFINITY;
  int am = 0, an = 0;
  for (int k0 = 0; k0 < kend; k0 += kSimtKeys) {
    __syncthreads();
    load_rows<D>(sK, D, Kt + base, k0, kSimtKeys, T);
    __syncthreads();
    for (int jj = 0; jj < kSimtKeys; ++jj) {
      const int j = k0 + jj;
      if (j < L) {
        const float s = dot_row<D>(sQ + r * (D + 1), sK + jj * D);
        if (s > m) { m = s; am = j; }
        if (s < n) { n = s; an = j; }
      }
    }
  }
  const RowState rs = make_row_state(p, m, n);
  const int ts = (p.cal == KIA_CAL_MINMAX) ? kSimtRows : 1;
  const float* tab = (p.cal == KIA_CAL_MINMAX) ? sTab + r : sTab;
  if (!p.softmax) {
    if (p.cal == KIA_CAL_MINMAX) {
      if (!rs.degen) {
        for (int k = 0; k <= p.K; ++k) {
          const float G = grid_value(k, rs.cal.h);
          sTab[k * kSimtRows + r] = G;
          if (live) st.table[(size_t)(bh * T + i) * (p.K + 1) + k] = G;
        }
      } else if (live) {
        for (int k = 0; k <= p.K; ++k) st.table[(size_t)(bh * T + i) * (p.K + 1) + k] = 1.0f;
      }
    } else {
      // one grid for every row (the fixed-step grid may outnumber the threads)
      for (int k = r; k <= p.K; k += kSimtRows) {
        const float G = grid_value(k, p.fwm_h);
        sTab[k] = G;
        if (blockIdx.x == 0 && blockIdx.y == 0) st.table[k] = G;
      }
    }
  }
  // sweep 2: weights, normalisers, P V (and P_L V for Prob-STE)
  const bool wantL = needs_OL(p);
  float acc[D], accL[D];
#pragma unroll
  for (int c = 0; c < D; ++c) { acc[c] = 0.0f; accL[c] = 0.0f; }
  float W = 0.0f, WL = 0.0f;
  for (int k0 = 0; k0 < kend; k0 += kSimtKeys) {
    __syncthreads();
    load_rows<D>(sK, D, Kt + base, k0, kSimtKeys, T);
    load_rows<D>(sV, D, V + base, k0, kSimtKeys, T);
    __syncthreads();
    for (int jj = 0; jj < kSimtKeys; ++jj) {
      const int j = k0 + jj;
      if (j < L) {
        const float s = dot_row<D>(sQ + r * (D + 1), sK + jj * D);
        const ElemFwd e = elem_forward(p, rs, tab, ts, s);
        W += e.wf;
        WL += e.wl;
        const float* v = sV + jj * D;
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = fmaf(e.wf, v[c], acc[c]);
        if (wantL) {
#pragma unroll
          for (int c = 0; c < D; ++c) accL[c] = fmaf(e.wl, v[c], accL[c]);
        }
      }
    }
  }
  if (!live) return;
  const size_t row = (size_t)bh * T + i;
  float* o = O + row * D;
#pragma unroll
  for (int c = 0; c < D; ++c) o[c] = __fdiv_rn(acc[c], W);
  if (wantL) {
    float* ol = st.OL + row * D;
#pragma unroll
    for (int c = 0; c < D; ++c) ol[c] = __fdiv_rn(accL[c], WL);
  }
  st.m[row] = m;
  st.n[row] = n;
  st.am[row] = am;
  st.an[row] = an;
  st.rh[row] = rs.degen ? 0.0f : rs.cal.rh;
  st.h[row] = rs.degen ? 0.0f : rs.cal.h;
  st.Wf[row] = W;
  st.Wb[row] = (!p.softmax && lerp_normpoint(p)) ? WL : W;
}

// dQ side: one thread per query row; writes dQ (before calibration
// corrections), the row sums A, C, and the detached score gradient rows.
template <int D>
__global__ void __launch_bounds__(kSimtRows)
simt_bwd_q_kernel(const float* __restrict__ Q, const float* __restrict__ Kt,
                  const float* __restrict__ V, const float* __restrict__ dO, StatsView st,
                  WorkView wk, float* __restrict__ dQ, float* __restrict__ dS_dbg, OpParams p,
                  int T) {
  if (*wk.status != 0) return;
  extern __shared__ float sm[];
  float* sQ = sm;                                   // [128][D+1]
  float* sG = sQ + kSimtRows * (D + 1);             // dO rows [128][D+1]
  float* sK = sG + kSimtRows * (D + 1);             // [32][D]
  float* sV = sK + kSimtKeys * D;                   // [32][D]
  float* sTab = sV + kSimtKeys * D;                 // [(K+1)][128] or [K+1]
  const int bh = blockIdx.y;
  const int r = threadIdx.x;
  const int i0 = blockIdx.x * kSimtRows;
  const int i = i0 + r;
  const bool live = i < T;
  const size_t base = (size_t)bh * T * D;
  const int L = live ? (p.causal ? i + 1 : T) : 0;
  const int kend = p.causal ? min(T, i0 + kSimtRows) : T;
  const size_t row = (size_t)bh * T + (live ? i : 0);
  const bool tr = p.tf32_ops != 0;
  load_rows<D>(sQ, D + 1, Q + base, i0, kSimtRows, T, tr);
  load_rows<D>(sG, D + 1, dO + base, i0, kSimtRows, T, tr);
  RowState rs;
  rs.cal.m = st.m[row];
  rs.cal.rh = st.rh[row];
  rs.cal.h = st.h[row];
  rs.degen = !p.softmax && p.cal == KIA_CAL_MINMAX && rs.cal.h == 0.0f;
  const float rWb = __fdiv_rn(1.0f, st.Wb[row]);
  const float Dc = wk.D[row];
  const int ts = (p.cal == KIA_CAL_MINMAX) ? kSimtRows : 1;
  const float* tab = (p.cal == KIA_CAL_MINMAX) ? sTab + r : sTab;
  if (!p.softmax) {
    if (p.cal == KIA_CAL_MINMAX) {
      for (int k = 0; k <= p.K; ++k) sTab[k * kSimtRows + r] = st.table[row * (p.K + 1) + k];
    } else {
      for (int k = r; k <= p.K; k += kSimtRows) sTab[k] = st.table[k];
    }
  }
  float acc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) acc[c] = 0.0f;
  float A = 0.0f, C = 0.0f;
  for (int k0 = 0; k0 < kend; k0 += kSimtKeys) {
    __syncthreads();
    load_rows<D>(sK, D, Kt + base, k0, kSimtKeys, T, tr);
    load_rows<D>(sV, D, V + base, k0, kSimtKeys, T, tr);
    __syncthreads();
    for (int jj = 0; jj < kSimtKeys; ++jj) {
      const int j = k0 + jj;
      if (j < L) {
        const float s = dot_row<D>(sQ + r * (D + 1), sK + jj * D);
        const float dp = dot_row<D>(sG + r * (D + 1), sV + jj * D);
        const ElemFwd e = elem_forward(p, rs, tab, ts, s);
        // a one-key row has P = 1 whatever its score: zero gradient
        const float dw = (L == 1) ? 0.0f : (dp - Dc) * rWb;
        const float delta = elem_backward(p, rs, tab, ts, s, e.wf, dw, A, C);
        const float dl = tr ? tf32_trunc(delta) : delta;
        const float* k = sK + jj * D;
#pragma unroll
        for (int c = 0; c < D; ++c) acc[c] = fmaf(dl, k[c], acc[c]);
        if (dS_dbg) dS_dbg[((size_t)bh * T + i) * T + j] = delta;
      }
    }
  }
  if (!live) return;
  float* dq = dQ + row * D;
#pragma unroll
  for (int c = 0; c < D; ++c) dq[c] = acc[c];
  wk.A[row] = A;
  wk.C[row] = C;
  wk.am[row] = st.am[row];
  wk.an[row] = st.an[row];
}

// dK / dV side: one thread per key row, queries streamed through shared
// memory with their row statistics and grid tables.
template <int D>
__global__ void __launch_bounds__(kSimtRows)
simt_bwd_kv_kernel(const float* __restrict__ Q, const float* __restrict__ Kt,
                   const float* __restrict__ V, const float* __restrict__ dO, StatsView st,
                   WorkView wk, float* __restrict__ dK, float* __restrict__ dV, OpParams p,
                   int T) {
  if (*wk.status != 0) return;
  extern __shared__ float sm[];
  float* sK = sm;                                   // [128][D+1]
  float* sVv = sK + kSimtRows * (D + 1);            // [128][D+1]
  float* sQ = sVv + kSimtRows * (D + 1);            // [32][D]
  float* sG = sQ + kSimtKeys * D;                   // [32][D]
  float* sRow = sG + kSimtKeys * D;                 // [32][6]: m, rh, h, rWb, rWf, D
  float* sTab = sRow + kSimtKeys * 6;               // [32][K+1] or [K+1]
  const int bh = blockIdx.y;
  const int r = threadIdx.x;
  const int j0 = blockIdx.x * kSimtRows;
  const int j = j0 + r;
  const bool live = j < T;
  const size_t base = (size_t)bh * T * D;
  const bool tr = p.tf32_ops != 0;
  load_rows<D>(sK, D + 1, Kt + base, j0, kSimtRows, T, tr);
  load_rows<D>(sVv, D + 1, V + base, j0, kSimtRows, T, tr);
  const int qstart = p.causal ? j0 : 0;
  const int K1 = p.K + 1;
  float aK[D], aV[D];
#pragma unroll
  for (int c = 0; c < D; ++c) { aK[c] = 0.0f; aV[c] = 0.0f; }
  for (int q0 = qstart; q0 < T; q0 += kSimtKeys) {
    __syncthreads();
    load_rows<D>(sQ, D, Q + base, q0, kSimtKeys, T, tr);
    load_rows<D>(sG, D, dO + base, q0, kSimtKeys, T, tr);
    if (threadIdx.x < kSimtKeys) {
      const int qi = q0 + threadIdx.x;
      const size_t qr = (size_t)bh * T + (qi < T ? qi : 0);
      sRow[threadIdx.x * 6 + 0] = st.m[qr];
      sRow[threadIdx.x * 6 + 1] = st.rh[qr];
      sRow[threadIdx.x * 6 + 2] = st.h[qr];
      sRow[threadIdx.x * 6 + 3] = __fdiv_rn(1.0f, st.Wb[qr]);
      sRow[threadIdx.x * 6 + 4] = __fdiv_rn(1.0f, st.Wf[qr]);
      sRow[threadIdx.x * 6 + 5] = wk.D[qr];
    }
    if (!p.softmax) {
      if (p.cal == KIA_CAL_MINMAX) {
        for (int e = threadIdx.x; e < kSimtKeys * K1; e += blockDim.x) {
          const int qi = q0 + e / K1;
          const size_t qr = (size_t)bh * T + (qi < T ? qi : 0);
          sTab[e] = st.table[qr * K1 + e % K1];
        }
      } else {
        for (int e = threadIdx.x; e < K1; e += blockDim.x) sTab[e] = st.table[e];
      }
    }
    __syncthreads();
    if (!live) continue;
    for (int ii = 0; ii < kSimtKeys; ++ii) {
      const int qi = q0 + ii;
      if (qi >= T) break;
      if (p.causal && j > qi) continue;
      const float* rowp = sRow + ii * 6;
      RowState rs;
      rs.cal.m = rowp[0];
      rs.cal.rh = rowp[1];
      rs.cal.h = rowp[2];
      rs.degen = !p.softmax && p.cal == KIA_CAL_MINMAX && rs.cal.h == 0.0f;
      const float* tab = (p.cal == KIA_CAL_MINMAX) ? sTab + ii * K1 : sTab;
      const float s = dot_row<D>(sQ + ii * D, sK + r * (D + 1));
      const float dp = dot_row<D>(sG + ii * D, sVv + r * (D + 1));
      const ElemFwd e = elem_forward(p, rs, tab, 1, s);
      const int Lq = p.causal ? qi + 1 : T;
      const float dw = (Lq == 1) ? 0.0f : (dp - rowp[5]) * rowp[3];
      float A = 0.0f, C = 0.0f;
      const float delta = elem_backward(p, rs, tab, 1, s, e.wf, dw, A, C);
      const float P = tr ? tf32_trunc(e.wf * rowp[4]) : e.wf * rowp[4];
      const float dl = tr ? tf32_trunc(delta) : delta;
      const float* q = sQ + ii * D;
      const float* g = sG + ii * D;
#pragma unroll
      for (int c = 0; c < D; ++c) {
        aK[c] = fmaf(dl, q[c], aK[c]);
        aV[c] = fmaf(P, g[c], aV[c]);
      }
    }
  }
  if (!live) return;
  const size_t row = (size_t)bh * T + j;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    dK[row * D + c] = aK[c];
    dV[row * D + c] = aV[c];
  }
}

}  // namespace kia
