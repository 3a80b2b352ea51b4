// Element stage of the tensor-core kernels, specialised at compile time on
// the operator variant (section 3: calibration x reconstruction x surrogate,
// or exact softmax).  The fp32 arithmetic of the weights is the sequence
// fixed in kia_common.cuh (and pinned bit for bit by the weight-stage test):
//   u = (m - s) * rh  (MinMax: min(u, K)),  k = min(floor u, K-1),  t = u - k,
//   LERP w = fma(t, G_{k+1} - G_k, G_k),  Nearest w = G_{k + [t >= 1/2]}.
// floor(u) for 0 <= u <= K-1 is taken as (u + 1.5*2^23 rounded down) -
// 1.5*2^23, which is exact and yields the integer index from the same bits.
//
// Degenerate MinMax rows (span < 1e-12) need no branch: their grid is all
// ones and rh = 0, so u = 0, w = 1 (uniform P), a_k = 0, and the backward
// slope becomes the per-row flag dg = 1 (dS = dw = (dP - mean dP)/|J|).
#pragma once
#include "kia_common.cuh"

namespace kia {

template <int CAL_, int REC_, bool PROB_, bool SOFTMAX_>
struct Var {
  static constexpr int CAL = CAL_;
  static constexpr int REC = REC_;
  static constexpr bool PROB = PROB_;        // Nearest + Prob-STE: forward also keeps P_L
  static constexpr bool SOFTMAX = SOFTMAX_;  // exact softmax attention
  static constexpr bool NEAREST = (REC_ == KIA_REC_NEAREST) && !SOFTMAX_;
  static constexpr bool FWM = (CAL_ == KIA_CAL_FWM) && !SOFTMAX_;
  static constexpr bool MINMAX = (CAL_ == KIA_CAL_MINMAX) && !SOFTMAX_;
};

constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;

struct Pos {
  float u;   // grid coordinate (MinMax: clamped to K)
  float t;   // position inside the interval
  float kf;  // interval index as a float
  int k;     // interval index
};

template <class V>
__device__ __forceinline__ Pos grid_pos(float m, float rh, float Kf, float Km1f, float s) {
  Pos p;
  float u = __fmul_rn(__fsub_rn(m, s), rh);
  if constexpr (V::MINMAX) u = fminf(u, Kf);
  p.u = u;
  const float uc = fminf(fmaxf(u, 0.0f), Km1f);
  const float tmp = __fadd_rd(uc, kMagic);
  p.kf = __fsub_rn(tmp, kMagic);
  p.k = __float_as_int(tmp) - kMagicBits;
  p.t = __fsub_rn(u, p.kf);
  return p;
}

// Forward weights: wf (forward probabilities' numerator) and wl (LERP weight,
// kept for Prob-STE).  tab[k * ts] = G_k.
template <class V>
__device__ __forceinline__ void fwd_weights(const float* tab, int ts, float m, float rh, float Kf,
                                            float Km1f, float s, float& wf, float& wl) {
  if constexpr (V::SOFTMAX) {
    wf = __expf(s - m);
    wl = wf;
  } else {
    const Pos p = grid_pos<V>(m, rh, Kf, Km1f, s);
    if constexpr (V::NEAREST) {
      const int r = p.k + (p.t >= 0.5f ? 1 : 0);
      wf = tab[r * ts];
      if constexpr (V::PROB) {
        const float g0 = tab[p.k * ts], g1 = tab[(p.k + 1) * ts];
        wl = __fmaf_rn(p.t, __fsub_rn(g1, g0), g0);
      } else {
        wl = wf;
      }
    } else {
      const float g0 = tab[p.k * ts], g1 = tab[(p.k + 1) * ts];
      wf = __fmaf_rn(p.t, __fsub_rn(g1, g0), g0);
      wl = wf;
    }
    if constexpr (V::FWM) {
      if (p.u > Kf) {
        wf = 0.0f;
        wl = 0.0f;
      }
    }
  }
}

// Backward of one element (normalisation Jacobian already applied: dw =
// (dP - D) / W_bar).  Returns dS; accumulates A += dw a_k and, when NEED_C,
// C += dw (b - a_k u / h) with b = -(1-t) k G_k - t (k+1) G_{k+1}.
// nrh = -rh; dg = 1 on degenerate rows, else 0.
template <class V, bool NEED_C>
__device__ __forceinline__ float bwd_delta(const float* tab, int ts, float m, float rh, float nrh,
                                           float dg, float Kf, float Km1f, float s, float dw,
                                           float& A, float& C) {
  if constexpr (V::SOFTMAX) {
    return __expf(s - m) * dw;
  } else {
    const Pos p = grid_pos<V>(m, rh, Kf, Km1f, s);
    float g0 = tab[p.k * ts], g1 = tab[(p.k + 1) * ts];
    if constexpr (V::FWM) {
      if (p.u > Kf) {
        g0 = 0.0f;
        g1 = 0.0f;
      }
    }
    const float a = __fsub_rn(g1, g0);
    const float da = dw * a;
    A += da;
    float delta;
    if constexpr (V::MINMAX) {
      delta = fmaf(dw, dg, da * nrh);
      if constexpr (NEED_C) {
        const float kg0 = p.kf * g0;
        const float bpos = fmaf(p.t, fmaf(p.kf + 1.0f, g1, -kg0), kg0);  // -b
        C = fmaf(delta, p.u, fmaf(-dw, bpos, C));
      }
    } else {
      delta = da * nrh;
    }
    return delta;
  }
}

// The forward probability numerator in the key pass (thread = key row).
template <class V>
__device__ __forceinline__ float fwd_weight_only(const float* tab, int ts, float m, float rh,
                                                 float Kf, float Km1f, float s) {
  float wf, wl;
  fwd_weights<V>(tab, ts, m, rh, Kf, Km1f, s, wf, wl);
  return wf;
}

// Backward of one element in the key pass: the forward probability P (for
// dV) and dS (for dK), with the grid position computed once.
template <class V>
__device__ __forceinline__ void kv_elem(const float* tab, int ts, float m, float rh, float nrh,
                                        float dg, float rWf, float Kf, float Km1f, float s,
                                        float dw, float& P, float& dS) {
  if constexpr (V::SOFTMAX) {
    const float w = __expf(s - m);
    P = w * rWf;
    dS = w * dw;
  } else {
    const Pos p = grid_pos<V>(m, rh, Kf, Km1f, s);
    float g0 = tab[p.k * ts], g1 = tab[(p.k + 1) * ts];
    float wf;
    if constexpr (V::NEAREST) {
      wf = (p.t >= 0.5f) ? g1 : g0;
    } else {
      wf = __fmaf_rn(p.t, __fsub_rn(g1, g0), g0);
    }
    if constexpr (V::FWM) {
      if (p.u > Kf) {
        g0 = 0.0f;
        g1 = 0.0f;
        wf = 0.0f;
      }
    }
    P = wf * rWf;
    const float da = dw * __fsub_rn(g1, g0);
    if constexpr (V::MINMAX) {
      dS = fmaf(dw, dg, da * nrh);
    } else {
      dS = da * nrh;
    }
  }
}

}  // namespace kia
