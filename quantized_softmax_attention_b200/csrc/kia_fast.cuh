// Element stage of the tensor-core kernels, specialised at compile time on
// the operator variant (section 3: calibration x reconstruction x surrogate,
// or exact softmax).  The fp32 arithmetic of the weights is the sequence
// fixed in kia_common.cuh (and pinned bit for bit by the weight-stage test):
//   u = (m - s) * rh  (MinMax: min(u, K)),  k = min(floor u, K-1),  t = u - k,
//   LERP w = fma(t, G_{k+1} - G_k, G_k),  Nearest w = G_{k + [t >= 1/2]}.
// floor(u) for 0 <= u <= K-1 is taken as (u + 1.5*2^23 rounded down) -
// 1.5*2^23, which is exact and yields the integer index from the same bits.
// Both weights of a row read the pair (G_k, G_{k+1}); Nearest selects from it.
//
// Degenerate MinMax rows (span < 1e-12) need no branch: their grid is all
// ones and rh = 0, so u = 0, w = 1 (uniform P), a_k = 0, and the backward
// slope becomes the per-row flag dg = 1 (dS = dw = (dP - mean dP)/|J|).
#pragma once
#include "kia_common.cuh"

namespace kia {

template <int CAL_, int REC_, bool PROB_, bool SOFTMAX_, int EXPR_ = 0>
struct Var {
  static constexpr int EXPR = EXPR_;         // softmax numerator rounding (round_exp)
  static constexpr int CAL = CAL_;
  static constexpr int REC = REC_;
  static constexpr bool PROB = PROB_;        // Nearest + Prob-STE: forward also keeps P_L
  static constexpr bool SOFTMAX = SOFTMAX_;  // exact softmax attention
  static constexpr bool NEAREST = (REC_ == KIA_REC_NEAREST) && !SOFTMAX_;
  static constexpr bool FWM = (CAL_ == KIA_CAL_FWM) && !SOFTMAX_;
  static constexpr bool MINMAX = (CAL_ == KIA_CAL_MINMAX) && !SOFTMAX_;
};

// Which of the 16 consecutive queries q0..q0+15 may attend key kj: key and
// query inside [0, T), and kj <= q under the causal mask (bit i for q0 + i).
__device__ __forceinline__ uint32_t visible16(int kj, int q0, int T, bool causal) {
  if (kj >= T) return 0u;
  uint32_t vis = 0xFFFFu;
  const int nq = T - q0;                        // queries left before T
  if (nq < 16) vis = nq <= 0 ? 0u : (1u << nq) - 1u;
  if (causal) {
    const int d = kj - q0;                      // first visible query offset
    if (d >= 16) return 0u;
    if (d > 0) vis &= 0xFFFFu << d;
  }
  return vis;
}

// Calibration terms of a chunk of 16 query columns, added in tensor memory
// once the chunk's score gradients are stored there, column i at TMEM address
// col0 + i for this warp's 32 lanes: bm (bn) marks, the same in every lane,
// the columns whose argmax (argmin) key lies among the warp's 32 keys; cm[i]
// (cn[i]) holds column i's (key offset in the tile, coefficient bits).  Per
// marked column the warp reads the column, the thread holding that key adds
// the coefficient, and the warp writes the column back, argmax terms before
// argmin terms.  A few instructions per term: adding into the registers
// instead needs a jump on a run-time index into the array or a test per
// column, and either cost many times that.
__device__ __forceinline__ void add_calibration_tmem(uint32_t col0, uint32_t bm, uint32_t bn,
                                                     const int2* cm, const int2* cn, int r) {
  if ((bm | bn) == 0u) return;
  tmem_st_wait();   // the chunk's own stores have landed
  while ((bm | bn) != 0u) {
    const bool fm = bm != 0u;
    const int i = __ffs(fm ? bm : bn) - 1;
    if (fm) bm &= bm - 1u;
    else bn &= bn - 1u;
    const int2 c = (fm ? cm : cn)[i];
    const uint32_t ta = col0 + (uint32_t)i;
    const float x = tmem_ld1_sync(ta);
    tmem_st1(ta, c.x == r ? x + __int_as_float(c.y) : x);
    tmem_st_wait();   // before a later term of the same column reads it
  }
}

constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;

// Grid of one row: G_k at p[k * ts] (float table), or the pair
// (G_k, G_{k+1}) at q[k] (pair table, one 8-byte load).
struct GridF {
  const float* p;
  int ts;
  __device__ __forceinline__ float2 pair(int k) const {
    return make_float2(p[k * ts], p[(k + 1) * ts]);
  }
};
struct GridP {
  const float2* q;
  __device__ __forceinline__ float2 pair(int k) const { return q[k]; }
};
// FWM / fixed-step grid in shared memory: pairs (G_k, G_{k+1}) for k = 0..K-1
// followed by a zero pair at index K.  A tail key (u > K) fetches the zero
// pair, which gives it weight 0 and slope 0 with no selects afterwards.
struct GridZ {
  const float2* q;   // pair 0 (shared memory)
  int K;             // index of the zero pair
  __device__ __forceinline__ float2 at(int k, bool tail) const { return q[tail ? K : k]; }
};
__device__ __forceinline__ GridZ make_gridz(const float2* pairs, int K) { return GridZ{pairs, K}; }
template <class G>
inline constexpr bool kZeroTail = false;
template <>
inline constexpr bool kZeroTail<GridZ> = true;

struct Pos {
  float u;   // grid coordinate (MinMax: clamped to K)
  float t;   // position inside the interval
  float kf;  // interval index as a float
  int k;     // interval index
};

// CLAMP0: the score may exceed the row max by an ulp (recomputed by another
// contraction order), so clamp u at 0 before taking the interval index.
template <class V, bool CLAMP0>
__device__ __forceinline__ Pos grid_pos(float m, float rh, float Kf, float Km1f, float s) {
  Pos p;
  float u = __fmul_rn(__fsub_rn(m, s), rh);
  if constexpr (V::MINMAX) u = fminf(u, Kf);
  p.u = u;
  float uc = fminf(u, Km1f);
  if constexpr (CLAMP0) uc = fmaxf(uc, 0.0f);
  const float tmp = __fadd_rd(uc, kMagic);
  p.kf = __fsub_rn(tmp, kMagic);
  p.k = __float_as_int(tmp) - kMagicBits;
  p.t = __fsub_rn(u, p.kf);
  return p;
}

// ------------------------------------------------ packed pairs (f32x2)
// sm_100 issues two fp32 adds / muls / fmas as one instruction; each half is
// an ordinary IEEE round-to-nearest (or round-down) operation, so results are
// bit-identical to the scalar sequence.
__device__ __forceinline__ unsigned long long pk(float2 a) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a.x), "f"(a.y));
  return r;
}
__device__ __forceinline__ float2 upk(unsigned long long r) {
  float2 a;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a.x), "=f"(a.y) : "l"(r));
  return a;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(a)), "l"(pk(b)));
  return upk(r);
}
__device__ __forceinline__ float2 add2_rd(float2 a, float2 b) {
  unsigned long long r;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(a)), "l"(pk(b)));
  return upk(r);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  unsigned long long r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(a)), "l"(pk(b)));
  return upk(r);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(a)), "l"(pk(b)));
  return upk(r);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(pk(a)), "l"(pk(b)), "l"(pk(c)));
  return upk(r);
}

// Forward weights of two scores at once: the same arithmetic as fwd_weights,
// each half of every packed operation an ordinary IEEE operation, so the
// weights, bins and t are bit-identical to fwd_weights' on each score.
// wf2 / wl2 as in fwd_weights; returns both grid positions.
struct Pos2 {
  Pos a, b;
};
template <class V, bool CLAMP0, class G>
__device__ __forceinline__ Pos2 fwd_weights2(const G& grid, float m, float rh, float Kf,
                                             float Km1f, float s0, float s1, float2& wf2,
                                             float2& wl2) {
  Pos2 ps{};
  if constexpr (V::SOFTMAX) {
    wf2 = make_float2(round_exp<V::EXPR>(expf(s0 - m)), round_exp<V::EXPR>(expf(s1 - m)));
    wl2 = wf2;
  } else {
    float2 u = mul2(sub2(make_float2(m, m), make_float2(s0, s1)), make_float2(rh, rh));
    if constexpr (V::MINMAX) u = make_float2(fminf(u.x, Kf), fminf(u.y, Kf));
    float2 uc = make_float2(fminf(u.x, Km1f), fminf(u.y, Km1f));
    if constexpr (CLAMP0) uc = make_float2(fmaxf(uc.x, 0.0f), fmaxf(uc.y, 0.0f));
    const float2 mg = make_float2(kMagic, kMagic);
    const float2 tmp = add2_rd(uc, mg);
    const float2 kf = sub2(tmp, mg);
    const float2 t = sub2(u, kf);
    const int k0 = __float_as_int(tmp.x) - kMagicBits, k1 = __float_as_int(tmp.y) - kMagicBits;
    float2 g0, g1;
    if constexpr (kZeroTail<G>) {
      g0 = grid.at(k0, V::FWM && u.x > Kf);
      g1 = grid.at(k1, V::FWM && u.y > Kf);
    } else {
      g0 = grid.pair(k0);
      g1 = grid.pair(k1);
    }
    const float2 lo = make_float2(g0.x, g1.x), hi = make_float2(g0.y, g1.y);
    const float2 lerp = fma2(t, sub2(hi, lo), lo);
    if constexpr (V::NEAREST) {
      wf2 = make_float2(t.x >= 0.5f ? hi.x : lo.x, t.y >= 0.5f ? hi.y : lo.y);
      wl2 = V::PROB ? lerp : wf2;
    } else {
      wf2 = lerp;
      wl2 = lerp;
    }
    if constexpr (V::FWM && !kZeroTail<G>) {
      const bool t0 = u.x > Kf, t1 = u.y > Kf;
      wf2 = make_float2(t0 ? 0.0f : wf2.x, t1 ? 0.0f : wf2.y);
      wl2 = make_float2(t0 ? 0.0f : wl2.x, t1 ? 0.0f : wl2.y);
    }
    ps.a = Pos{u.x, t.x, kf.x, k0};
    ps.b = Pos{u.y, t.y, kf.y, k1};
  }
  return ps;
}

// Forward weights: wf (forward probabilities' numerator) and wl (LERP
// weight, used by Prob-STE's normalisation point).  Returns the grid
// position the weights came from (zero for softmax), so that the weight-stage
// test entry point reports the bins and t of this very code.  CLAMP0 for
// scores that may lie above the row max (recomputed by another contraction
// order, or masked).
template <class V, bool CLAMP0, class G>
__device__ __forceinline__ Pos fwd_weights(const G& grid, float m, float rh, float Kf,
                                           float Km1f, float s, float& wf, float& wl) {
  if constexpr (V::SOFTMAX) {
    wf = round_exp<V::EXPR>(expf(s - m));
    wl = wf;
    return Pos{0.0f, 0.0f, 0.0f, 0};
  } else {
    const Pos p = grid_pos<V, CLAMP0>(m, rh, Kf, Km1f, s);
    float2 g;
    if constexpr (kZeroTail<G>) g = grid.at(p.k, V::FWM && p.u > Kf);
    else g = grid.pair(p.k);
    const float lerp = __fmaf_rn(p.t, __fsub_rn(g.y, g.x), g.x);
    if constexpr (V::NEAREST) {
      wf = (p.t >= 0.5f) ? g.y : g.x;
      wl = V::PROB ? lerp : wf;
    } else {
      wf = lerp;
      wl = lerp;
    }
    if constexpr (V::FWM && !kZeroTail<G>) {
      const bool tail = p.u > Kf;
      wf = tail ? 0.0f : wf;
      wl = tail ? 0.0f : wl;
    }
    return p;
  }
}

// Backward of one element in the query pass (dw = (dP - D) / W_bar, the
// normalisation Jacobian at the surrogate's point).  Returns the detached
// dS; accumulates A += dw a_k and, when NEED_C, C += dw (b - a_k u / h) with
// b = -(1-t) k G_k - t (k+1) G_{k+1}.  nrh = -rh; dg = 1 on degenerate rows.
// FOLD: degenerate rows come with nrh = 1 and a grid whose first slope is 1
// (the caller's copy patched to G_1 = 2), so dS = dw needs no dg term.
template <class V, bool NEED_C, bool FOLD = false, class G>
__device__ __forceinline__ float bwd_delta(const G& grid, float m, float rh, float nrh, float dg,
                                           float Kf, float Km1f, float s, float dw, float& A,
                                           float& C) {
  if constexpr (V::SOFTMAX) {
    // straight through the rounding of the reduced-precision baselines:
    // the slope is the unrounded e^{s-m}
    return expf(s - m) * dw;
  } else {
    const Pos p = grid_pos<V, true>(m, rh, Kf, Km1f, s);
    float2 g;
    if constexpr (kZeroTail<G>) {
      g = grid.at(p.k, V::FWM && p.u > Kf);
    } else {
      g = grid.pair(p.k);
      if constexpr (V::FWM) {
        const bool tail = p.u > Kf;
        g.x = tail ? 0.0f : g.x;
        g.y = tail ? 0.0f : g.y;
      }
    }
    const float da = dw * __fsub_rn(g.y, g.x);
    A += da;
    float delta;
    if constexpr (V::MINMAX) {
      delta = FOLD ? da * nrh : fmaf(dw, dg, da * nrh);
      if constexpr (NEED_C) {
        const float kg0 = p.kf * g.x;
        const float bpos = fmaf(p.t, fmaf(p.kf + 1.0f, g.y, -kg0), kg0);  // -b
        C = fmaf(delta, p.u, fmaf(-dw, bpos, C));
      }
    } else {
      delta = da * nrh;
    }
    return delta;
  }
}

// Calibration coefficients of one row from its row sums (Appendix B):
//   MinMax: g_m = A / h + C / K,  g_n = -C / K;   FWM: g_m = A / h, g_n = 0,
// filtered by the gradient mode; the zero-sum projection instead returns its
// common-mode shift c = A / (h |J_i|) in gm (gn = 0).  Degenerate and
// softmax rows have none.
__device__ __forceinline__ void calibration_coeffs(const OpParams& p, float A, float C, float rh,
                                                   int L, float& gm, float& gn) {
  gm = 0.0f;
  gn = 0.0f;
  if (p.softmax || rh == 0.0f || p.grad == KIA_GRAD_DETACH) return;
  if (p.grad == KIA_GRAD_PROJECT) {
    gm = A * rh / (float)L;
    return;
  }
  const float gm_full = (p.cal == KIA_CAL_MINMAX) ? A * rh + C / p.Kf : A * rh;
  const float gn_full = (p.cal == KIA_CAL_MINMAX) ? -C / p.Kf : 0.0f;
  if (p.grad == KIA_GRAD_FULL || p.grad == KIA_GRAD_MAX_ONLY) gm = gm_full;
  if (p.grad == KIA_GRAD_FULL || p.grad == KIA_GRAD_MIN_ONLY) gn = gn_full;
}

}  // namespace kia
