// Per-element forward weights and backward score gradient of K-interval
// attention (section 3; Appendices A and B), shared by every kernel so the
// exact-fp32 and tensor-core paths apply identical element arithmetic.
#pragma once
#include "kia_common.cuh"

namespace kia {

// Row-level constants the element stage needs.
struct RowState {
  RowCal cal;
  bool degen;   // MinMax span below 1e-12 (Appendix A degenerate branch)
};

__device__ __forceinline__ RowState make_row_state(const OpParams& p, float m, float n) {
  RowState r;
  r.cal = row_calibration(p, m, n);
  r.degen = !p.softmax && p.cal == KIA_CAL_MINMAX && r.cal.h == 0.0f;
  return r;
}

// Forward weights of one element: wf (the forward probabilities'
// numerator: LERP for LERP, the hard node for Nearest, e^{s-m} for softmax)
// and wl (the LERP weight, used by Prob-STE's normalisation point).
// `tab` points at G_0 of the row's grid, with stride `ts` between entries.
struct ElemFwd {
  float wf;
  float wl;
};

__device__ __forceinline__ ElemFwd elem_forward(const OpParams& p, const RowState& r,
                                                const float* tab, int ts, float s) {
  ElemFwd e;
  if (p.softmax) {
    e.wf = round_exp_rt(expf(s - r.cal.m), p.exp_round);
    e.wl = e.wf;
    return e;
  }
  if (r.degen) {
    e.wf = 1.0f;
    e.wl = 1.0f;
    return e;
  }
  const GridPos g = grid_position(p, r.cal, s);
  if (g.tail) {
    e.wf = 0.0f;
    e.wl = 0.0f;
    return e;
  }
  const float Gk = tab[g.k * ts];
  const float Gk1 = tab[(g.k + 1) * ts];
  e.wl = lerp_weight(g.t, Gk, Gk1);
  e.wf = (p.rec == KIA_REC_LERP) ? e.wl : (g.t >= 0.5f ? Gk1 : Gk);
  return e;
}

// Backward of one element given dw = (dP - D) / W_bar (normalisation
// Jacobian at the surrogate's point, Appendix B).  Returns the detached score
// gradient delta; accumulates the calibration row sums
//   A += dw * a_k,   C += dw * (b - a_k u / h) = dw * b + delta * u,
// with a_k = G_{k+1} - G_k and b = -(1-t) k G_k - t (k+1) G_{k+1} (the
// derivative of the LERP weight with respect to h at fixed u).
__device__ __forceinline__ float elem_backward(const OpParams& p, const RowState& r,
                                               const float* tab, int ts, float s, float wf,
                                               float dw, float& A, float& C) {
  // softmax: e^{s-m} (dP - D) / W; the reduced-precision baselines pass
  // straight through their rounding, so the slope is the unrounded e^{s-m}
  if (p.softmax) return (p.exp_round ? expf(s - r.cal.m) : wf) * dw;
  if (r.degen) return dw;          // uniform P: (dP - mean dP) / |J|
  const GridPos g = grid_position(p, r.cal, s);
  if (g.tail) return 0.0f;         // FWM tail: zero gradient through mask and clamp
  const float Gk = tab[g.k * ts];
  const float Gk1 = tab[(g.k + 1) * ts];
  const float a = __fsub_rn(Gk1, Gk);
  const float delta = -dw * a * r.cal.rh;
  A = fmaf(dw, a, A);
  const float kf = (float)g.k;
  const float b = -(1.0f - g.t) * kf * Gk - g.t * (kf + 1.0f) * Gk1;
  C = fmaf(dw, b, fmaf(delta, g.u, C));
  return delta;
}

}  // namespace kia
