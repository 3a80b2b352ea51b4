// Geometry probe on given scores (kiattn_geometry): per query row the score
// span, the native interval width h, the query norm, the entropies of the
// softmax and operator probabilities, their total variation, and the
// softmax and operator mass in the top rounding bucket (the keys whose
// nearest grid node is the row maximum's).  Quantities of "Pretraining
// Transformers with Quantized Softmax in Attention", section 4 (geometry
// probe), section 5.4 and Appendix D.6 (Figure S4).
//
// One warp per row, specialised at compile time on calibration and
// reconstruction.  Rows of at most kGeoRowKeys keys are copied from HBM once
// into the warp's shared-memory buffer (asynchronous copies, all in flight
// together); the three sweeps run as rolled loops over it, and the second
// leaves e and w there for the third.  (An earlier form held the row in
// registers, unrolled over eight 128-key chunks: its code overflowed the
// instruction cache.)  Longer rows take three sweeps over global memory, the
// later two served by L1/L2.  The operator
// weights are the fused kernels' paired fp32 weight stage (kia_fast.cuh), so
// the grid decisions are the forward's; a key is in the top bucket iff its
// grid coordinate u = (m - s) / h is below 1/2 (nearest node 0).
#pragma once
#include <cfloat>
#include <type_traits>

#include "kia_common.cuh"
#include "kia_fast.cuh"

namespace kia {

constexpr int kGeoWarps = 8;
constexpr int kGeoRowKeys = 1024;                 // rows up to this length are staged
constexpr size_t kGeoSmemBytes = (size_t)kGeoWarps * 2 * kGeoRowKeys * 4;   // 64 KB

// out fields per row (include/kiattn.h: KIA_GEO_*)
enum { kGeoSpan = 0, kGeoH, kGeoQNorm, kGeoEntSoftmax, kGeoEntOp, kGeoTV, kGeoTopSoftmax,
       kGeoTopOp, kGeoFields };

struct GeoSums {
  float Z, Ex, W, Wlw, Tsm, Top;
};

struct GeoRow {
  GridP g;
  float m, rh, Kf, Km1f;
};

// Two keys: replaces (s0, s1) by their softmax numerators e = e^{s-m} and
// writes the operator numerators (w0, w1); keys not visible (ok = false)
// contribute nothing and come back as zeros.
template <class V, bool PARTIAL>
__device__ __forceinline__ void geo_pair(const GeoRow& r, float& s0, float& s1, float& w0,
                                         float& w1, bool ok0, bool ok1, GeoSums& a) {
  if constexpr (PARTIAL) {
    s0 = ok0 ? s0 : r.m;
    s1 = ok1 ? s1 : r.m;
  }
  float2 wf, wl;
  fwd_weights2<V, false>(r.g, r.m, r.rh, r.Kf, r.Km1f, s0, s1, wf, wl);
  const float2 x = sub2(make_float2(s0, s1), make_float2(r.m, r.m));      // s - m <= 0
  const float2 u = mul2(make_float2(-x.x, -x.y), make_float2(r.rh, r.rh)); // grid coordinate
  float e0 = __expf(x.x), e1 = __expf(x.y);
  if constexpr (PARTIAL) {
    e0 = ok0 ? e0 : 0.0f;
    e1 = ok1 ? e1 : 0.0f;
    wf.x = ok0 ? wf.x : 0.0f;
    wf.y = ok1 ? wf.y : 0.0f;
  }
  a.Z += e0 + e1;
  a.Ex = fmaf(e0, x.x, fmaf(e1, x.y, a.Ex));
  a.W += wf.x + wf.y;
  a.Wlw = fmaf(wf.x, __logf(fmaxf(wf.x, FLT_MIN)), fmaf(wf.y, __logf(fmaxf(wf.y, FLT_MIN)), a.Wlw));
  a.Tsm += (u.x < 0.5f ? e0 : 0.0f) + (u.y < 0.5f ? e1 : 0.0f);
  a.Top += (u.x < 0.5f ? wf.x : 0.0f) + (u.y < 0.5f ? wf.y : 0.0f);
  s0 = e0;
  s1 = e1;
  w0 = wf.x;
  w1 = wf.y;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <class V>
__global__ void __launch_bounds__(32 * kGeoWarps)
geometry_kernel(const float* __restrict__ S, const float* __restrict__ Q, long long rows, int T,
                int d, int causal, OpParams p, float* __restrict__ out) {
  // (G_k, G_{k+1}) pairs: one per warp under MinMax (the grid follows the
  // row), one per block under FWM (the grid is the same for every row)
  __shared__ float2 sPair[V::MINMAX ? kGeoWarps : 1][V::MINMAX ? KIA_MAX_K : KIA_MAX_KCAP];
  // per warp: the row's scores, overwritten by e = e^{s - m}, and the
  // operator's weights w (rows of at most kGeoRowKeys keys)
  extern __shared__ float sRows[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if constexpr (V::FWM) {
    for (int k = threadIdx.x; k < p.K; k += blockDim.x)
      sPair[0][k] = make_float2(grid_value(k, p.fwm_h), grid_value(k + 1, p.fwm_h));
    __syncthreads();
  }
  const long long row = (long long)blockIdx.x * kGeoWarps + warp;
  if (row >= rows) return;
  const int i = (int)(row % T);
  const int L = causal ? i + 1 : T;
  const float* s = S + row * (long long)T;
  const bool staged = L <= kGeoRowKeys;
  float* se = sRows + (size_t)warp * 2 * kGeoRowKeys;   // scores, then e
  float* sw = se + kGeoRowKeys;                          // w
  // the row into shared memory, all copies in flight together: 16 bytes at a
  // time where the row starts on a 16-byte boundary, else 4
  if (staged) {
    if ((reinterpret_cast<uintptr_t>(s) & 15) == 0) {
      const int L4 = L & ~3;
      for (int j = 4 * lane; j < L4; j += 128) cp_async16(se + j, s + j);
      if (lane < L - L4) cp_async4(se + L4 + lane, s + L4 + lane);
    } else {
      for (int j = lane; j < L; j += 32) cp_async4(se + j, s + j);
    }
  }
  // the query's squared norm while the copies land
  float qn = 0.0f;
  if (Q) {
    const float* q = Q + row * (long long)d;
    for (int k = lane; k < d; k += 32) qn = fmaf(q[k], q[k], qn);
  }
  if (staged) {
    cp_async_wait_all();
    __syncwarp();
  }

  // sweep 1: row extrema (section 3, calibration statistics)
  float m = -INFINITY, n = INFINITY;
  if (staged) {
#pragma unroll 4
    for (int j = lane; j < L; j += 32) {
      const float x = se[j];
      m = fmaxf(m, x);
      n = fminf(n, x);
    }
  } else {
    for (int j = lane; j < L; j += 32) {
      const float x = s[j];
      m = fmaxf(m, x);
      n = fminf(n, x);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    n = fminf(n, __shfl_xor_sync(0xffffffffu, n, o));
  }
  const RowCal c = row_calibration(p, m, n);
  GeoRow r;
  r.m = m;
  r.rh = c.rh;   // 0 on a degenerate MinMax row: u = 0, every weight G_0 = 1
  r.Kf = p.Kf;
  r.Km1f = p.Kf - 1.0f;
  if constexpr (V::MINMAX) {
    const bool degen = c.h == 0.0f;
    for (int k = lane; k < p.K; k += 32)
      sPair[warp][k] = degen ? make_float2(1.0f, 1.0f)
                             : make_float2(grid_value(k, c.h), grid_value(k + 1, c.h));
    __syncwarp();
    r.g.q = sPair[warp];
  } else {
    r.g.q = sPair[0];
  }

  // sweep 2: normalisers, entropy sums and top-bucket masses, two keys
  // (j, j + 32) at a time; a staged row keeps e and w for sweep 3
  GeoSums a = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  auto sweep2 = [&](auto* src, auto keep_c) {
    constexpr bool KEEP = decltype(keep_c)::value;
    for (int j = lane; j < L; j += 64) {
      const bool ok1 = j + 32 < L;
      float x0 = src[j], x1 = ok1 ? src[j + 32] : m, w0, w1;
      if (ok1) geo_pair<V, false>(r, x0, x1, w0, w1, true, true, a);
      else geo_pair<V, true>(r, x0, x1, w0, w1, true, false, a);
      if constexpr (KEEP) {
        se[j] = x0;
        sw[j] = w0;
        if (ok1) {
          se[j + 32] = x1;
          sw[j + 32] = w1;
        }
      }
    }
  };
  if (staged) sweep2(se, std::true_type{});
  else sweep2(s, std::false_type{});
  const float Z = warp_sum(a.Z), Ex = warp_sum(a.Ex), W = warp_sum(a.W),
              Wlw = warp_sum(a.Wlw), Tsm = warp_sum(a.Tsm), Top = warp_sum(a.Top);
  const float rZ = 1.0f / Z, rW = 1.0f / W;

  // sweep 3: total variation 1/2 sum_j |P_op,j - P_softmax,j| (a long row
  // recomputes e and w from its scores)
  float tv = 0.0f;
  if (staged) {
#pragma unroll 4
    for (int j = lane; j < L; j += 32) tv += fabsf(fmaf(sw[j], rW, -se[j] * rZ));
  } else {
    GeoSums dummy = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = lane; j < L; j += 32) {
      float x = s[j], y = m, w0, w1;
      geo_pair<V, true>(r, x, y, w0, w1, true, false, dummy);
      tv += fabsf(fmaf(w0, rW, -x * rZ));
    }
  }
  tv = 0.5f * warp_sum(tv);

  if (Q) qn = sqrtf(warp_sum(qn));
  if (lane < kGeoFields) {
    float val;
    switch (lane) {
      case kGeoSpan: val = __fsub_rn(m, n); break;
      case kGeoH: val = c.h; break;
      case kGeoQNorm: val = qn; break;
      case kGeoEntSoftmax: val = __logf(Z) - Ex * rZ; break;
      case kGeoEntOp: val = __logf(W) - Wlw * rW; break;
      case kGeoTV: val = tv; break;
      case kGeoTopSoftmax: val = Tsm * rZ; break;
      default: val = Top * rW; break;
    }
    out[row * kGeoFields + lane] = val;
  }
}

}  // namespace kia
