/*
 * K-interval attention -- fp64 CPU oracle.  TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this library.  It shares no code, header, table or constant with the
 * CUDA path; it is deliberately plain (loops, fp64, no blocking or fusion) so
 * that a reader can check it against the paper by eye.
 *
 * Source: "Pretraining Transformers with Quantized Softmax in Attention"
 * (Zhu, Hu, Kozlowski), paperlayer.ai abstract page:
 *   - Operator family / Calibration / Reconstruction bullets (section 3):
 *     MinMax takes the interval width from the row span, FWM fixes a window
 *     [m - tau, m] with h = tau/K and gives keys below it zero weight; LERP
 *     interpolates between adjacent exponential grid values, Nearest rounds to
 *     a grid value; all weights are normalised, P = w / W.
 *   - Appendix A (operator definitions and edge cases): causal rows, future
 *     positions get zero weight, scores shifted by the row maximum; separate
 *     branch for spans below eps = 1e-12; FWM at K = 4 uses h = 1.5.
 *   - Appendix B (gradient derivations): normalisation Jacobian evaluated at
 *     the surrogate's point; full calibration gradient through shifted scores,
 *     grid values and h, with zero row sum; detach drops the extremum terms;
 *     zero-sum projection removes only the common mode; under FWM only the
 *     maximum matters and tail keys get zero gradient; Weight-STE and
 *     Prob-STE share the hard forward and the LERP scalar derivatives but use
 *     different normalisation points.
 *
 * Readings of points the pages leave open:
 *   grid nodes m - k h, k = 0..K (G_k = e^{-k h}); Nearest picks the nearer
 *   node, ties (t = 1/2) to the larger u; interval index k = min(floor u,
 *   K-1); FWM window u <= K for LERP and Nearest alike; degenerate MinMax rows
 *   (span < 1e-12) get uniform P and dS = (dP - mean dP)/|J|; arg-extrema take
 *   the lowest index; max-only keeps the live row max (n frozen), min-only
 *   keeps the live row min (m frozen); the projection subtracts the mean over
 *   all keys of the row; the caller pre-scales Q (no 1/sqrt(d) inside); the
 *   untruncated fixed step (Appendix D.4) is FWM's grid with no window, the
 *   node index unbounded; the reduced-precision exponential baselines
 *   (Appendix D.5) round e^{s-m} (as fp32) to bfloat16 or FP8 E4M3,
 *   nearest-even, and pass straight through the rounding with the row
 *   maximum held fixed.
 *
 * Parity pins (tests/test_oracle_pins.py, tests/test_oracle_autograd.py,
 * tests/test_oracle_reduced_exp.py, tests/test_oracle_geometry.py):
 * central finite differences, frozen-statistic finite differences, zero row
 * sums, bitwise-equal forwards across gradient modes, STE coincidence on grid
 * nodes, the softmax limit and the chord bound, the K = 1 closed form, brute
 * force Jacobians on tiny rows, an independent PyTorch fp64 autograd
 * restatement, libm's exp for the grid values of the fp32 weight stage.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define REF_CAL_MINMAX 0
#define REF_CAL_FWM 1
#define REF_CAL_FIXED 2 /* untruncated fixed step (Appendix D.4): h = tau / K, no window */
#define REF_REC_LERP 0
#define REF_REC_NEAREST 1
#define REF_STE_WEIGHT 0
#define REF_STE_PROB 1
#define REF_GRAD_FULL 0
#define REF_GRAD_DETACH 1
#define REF_GRAD_MAX_ONLY 2
#define REF_GRAD_MIN_ONLY 3
#define REF_GRAD_PROJECT 4
/* operand rounding applied before every product (TF32 emulation) */
#define REF_ROUND_NONE 0
#define REF_ROUND_TRUNC 1 /* keep the top 10 mantissa bits, drop the rest */
#define REF_ROUND_RNA 2   /* to nearest, ties away from zero */
#define REF_ROUND_RNE 3   /* to nearest, ties to even */

typedef struct {
  int K;        /* number of intervals, >= 1 */
  int cal;      /* REF_CAL_* */
  double tau;   /* FWM window width */
  int rec;      /* REF_REC_* */
  int ste;      /* REF_STE_* (ignored for LERP) */
  int grad;     /* REF_GRAD_* */
  int causal;   /* 1: key j is visible to query i iff j <= i */
  int softmax;  /* 1: exact softmax attention instead of K-interval */
  int rounding; /* REF_ROUND_* */
  int exp_round; /* softmax only (Appendix D.5): 0 exact, 1 bfloat16, 2 FP8 E4M3 numerator */
} ref_cfg;

/* per-row statistics exported by the oracle, in this order */
enum {
  ST_M = 0, ST_N, ST_AM, ST_AN, ST_H, ST_WFWD, ST_WL, ST_WN, ST_A, ST_C, ST_DEGEN,
  ST_COUNT
};

static const double REF_EPS_SPAN = 1e-12; /* Appendix A: degenerate-span branch */

/* ---------------------------------------------------------------- helpers */

static double round_operand(float x, int mode) {
  if (mode == REF_ROUND_NONE) return (double)x;
  uint32_t b;
  memcpy(&b, &x, 4);
  if ((b & 0x7f800000u) == 0x7f800000u) return (double)x; /* inf / nan */
  if (mode == REF_ROUND_TRUNC) {
    b &= 0xffffe000u;
  } else if (mode == REF_ROUND_RNA) {
    b += 0x1000u;
    b &= 0xffffe000u;
  } else { /* RNE */
    uint32_t lsb = (b >> 13) & 1u;
    b += 0xfffu + lsb;
    b &= 0xffffe000u;
  }
  float y;
  memcpy(&y, &b, 4);
  return (double)y;
}

static double round_operand_d(double x, int mode) {
  if (mode == REF_ROUND_NONE) return x;
  return round_operand((float)x, mode);
}

/* --------------------------------------------------- one row, fp64 method */

typedef struct {
  double m, n, h, WL, WN;
  int am, an, degen;
} rowstat;

/* Forward of one row (Appendix A): scores s[0..L-1], all visible.
 * fm / fn, when given, replace the row max / min (frozen statistics); the
 * interval index is then clamped to 0..K-1 so that the local linear piece
 * extends past the grid ends, which is what "locally fixed interval index"
 * means for a derivative taken at that point.
 * Outputs per key: wL (LERP weight), wN (Nearest weight), k, t, in-window. */
static void row_forward(const double* s, int L, const ref_cfg* c, const double* fm,
                        const double* fn, double* wL, double* wN, int* kk, double* tt,
                        unsigned char* win, rowstat* st) {
  double m = s[0], n = s[0];
  int am = 0, an = 0;
  for (int j = 1; j < L; ++j) {
    if (s[j] > m) { m = s[j]; am = j; }
    if (s[j] < n) { n = s[j]; an = j; }
  }
  st->m = m; st->n = n; st->am = am; st->an = an;
  double mm = fm ? *fm : m;
  double nn = fn ? *fn : n;
  const int K = c->K;
  double h;
  int degen = 0;
  if (c->cal == REF_CAL_MINMAX) {
    double span = mm - nn;
    if (span < REF_EPS_SPAN) degen = 1;
    h = span / K;          /* section 3: width from the row span */
  } else {
    h = c->tau / K;        /* section 3: h = tau / K */
  }
  st->h = h;
  st->degen = degen;
  double WL = 0.0, WN = 0.0;
  for (int j = 0; j < L; ++j) {
    if (degen) {
      wL[j] = 1.0; wN[j] = 1.0; kk[j] = 0; tt[j] = 0.0; win[j] = 1;
    } else {
      double u = (mm - s[j]) / h;
      int inw = (c->cal == REF_CAL_FWM) ? (u <= (double)K) : 1;
      win[j] = (unsigned char)inw;
      if (!inw) {
        wL[j] = 0.0; wN[j] = 0.0; kk[j] = -1; tt[j] = 0.0;
      } else {
        int k = (int)floor(u);
        /* the fixed-step grid continues past node K down to the row minimum */
        if (c->cal != REF_CAL_FIXED && k > K - 1) k = K - 1;
        if (k < 0) k = 0;
        double t = u - k;
        double Gk = exp(-(double)k * h);
        double Gk1 = exp(-(double)(k + 1) * h);
        wL[j] = (1.0 - t) * Gk + t * Gk1;     /* LERP between adjacent nodes */
        wN[j] = (t >= 0.5) ? Gk1 : Gk;        /* nearest node, ties to k+1 */
        kk[j] = k; tt[j] = t;
      }
    }
    WL += wL[j];
    WN += wN[j];
  }
  st->WL = WL; st->WN = WN;
}

/* Forward probabilities: LERP uses P_L, Nearest (either STE) uses P_N. */
static int uses_lerp_forward(const ref_cfg* c) { return c->rec == REF_REC_LERP; }
/* Normalisation point of the backward (Appendix B): LERP and Prob-STE at the
 * LERP point, Weight-STE at the hard point. */
static int uses_lerp_normpoint(const ref_cfg* c) {
  return c->rec == REF_REC_LERP || c->ste == REF_STE_PROB;
}

/* Backward of one row given dP_j = dO_i . v_j and the centering D.
 * Writes dS[0..L-1] and returns A, C (row sums of the calibration terms). */
static void row_backward(const double* s, int L, const ref_cfg* c, const rowstat* st,
                         const double* wL, const double* wN, const int* kk,
                         const double* tt, const unsigned char* win, const double* dP,
                         double D, double* dS, double* Aout, double* Cout) {
  (void)s; (void)wL; (void)wN;
  const int K = c->K;
  if (st->degen) {
    /* uniform P on the row: softmax Jacobian at uniform P, every mode */
    double mean = 0.0;
    for (int j = 0; j < L; ++j) mean += dP[j];
    mean /= L;
    for (int j = 0; j < L; ++j) dS[j] = (dP[j] - mean) / L;
    *Aout = 0.0; *Cout = 0.0;
    return;
  }
  const double h = st->h;
  const double Wbar = uses_lerp_normpoint(c) ? st->WL : st->WN;
  double A = 0.0, C = 0.0;
  for (int j = 0; j < L; ++j) {
    if (!win[j]) { dS[j] = 0.0; continue; }   /* FWM tail: mask and clamp */
    int k = kk[j];
    double t = tt[j];
    double Gk = exp(-(double)k * h);
    double Gk1 = exp(-(double)(k + 1) * h);
    double a = Gk1 - Gk;                       /* dw/du on this interval */
    double u = k + t;
    double dw = (dP[j] - D) / Wbar;            /* normalisation Jacobian */
    dS[j] = -dw * a / h;                       /* du/ds = -1/h */
    A += dw * a;
    /* dw/dh at fixed u: through the grid values G_k = e^{-k h} */
    double b = -(1.0 - t) * k * Gk - t * (k + 1) * Gk1;
    C += dw * (b - a * u / h);                 /* + through u = (m - s)/h */
  }
  double gm, gn;
  if (c->cal == REF_CAL_MINMAX) {
    gm = A / h + C / K;    /* dh/dm = 1/K */
    gn = -C / K;           /* dh/dn = -1/K */
  } else {
    gm = A / h;            /* FWM: h fixed, only the shift by m */
    gn = 0.0;
  }
  switch (c->grad) {
    case REF_GRAD_FULL:
      dS[st->am] += gm;
      dS[st->an] += gn;
      break;
    case REF_GRAD_DETACH:
      break;
    case REF_GRAD_MAX_ONLY:
      dS[st->am] += gm;
      break;
    case REF_GRAD_MIN_ONLY:
      dS[st->an] += gn;
      break;
    case REF_GRAD_PROJECT: {
      double mean = 0.0;
      for (int j = 0; j < L; ++j) mean += dS[j];
      mean /= L;
      for (int j = 0; j < L; ++j) dS[j] -= mean;
      break;
    }
  }
  *Aout = A; *Cout = C;
}

/* Rounding of an fp32 value to bfloat16 (8 significand bits, fp32's
 * exponent range), to nearest, ties to even: keep the top 16 bits. */
static float round_bf16(float x) {
  uint32_t b;
  memcpy(&b, &x, 4);
  if ((b & 0x7f800000u) == 0x7f800000u) return x;
  b += 0x7fffu + ((b >> 16) & 1u);
  b &= 0xffff0000u;
  float y;
  memcpy(&y, &b, 4);
  return y;
}

/* Rounding to FP8 E4M3 (4 exponent bits with bias 7, 3 fraction bits;
 * normal numbers from 2^-6, subnormals in steps of 2^-9, largest finite 448),
 * to nearest, ties to even, saturating at 448. */
static float round_e4m3(float x) {
  const double a = fabs((double)x);
  if (a != a) return x;
  if (a >= 448.0) return x < 0 ? -448.0f : 448.0f;
  int e;
  frexp(a, &e);            /* a in [2^(e-1), 2^e) */
  int E = e - 1;
  if (E < -6) E = -6;      /* subnormal range: fixed step 2^-9 */
  const double q = ldexp(1.0, E - 3);
  const double r = nearbyint(a / q) * q;   /* a / q is exact; nearbyint: ties to even */
  return (float)(x < 0 ? -r : r);
}

/* The numerator of the reduced-precision exponential baselines (Appendix
 * D.5): e^{s-m} as fp32, then rounded to the format. */
static double rounded_exp(double x, int mode) {
  const float e32 = (float)exp(x);
  if (mode == 1) return (double)round_bf16(e32);
  if (mode == 2) return (double)round_e4m3(e32);
  return exp(x);
}

float kiattn_ref_round_exp_format(float x, int mode) {
  return mode == 1 ? round_bf16(x) : (mode == 2 ? round_e4m3(x) : x);
}

/* Softmax row (reference row of the sweep; Appendix G: softmax runs use
 * softmax's own backward), or a reduced-precision exponential baseline:
 * P = R(e^{s-m}) / sum R(e^{s-m}).  E receives the unrounded e^{s-m} (the
 * straight-through slope of the baselines' backward). */
static void softmax_row_r(const double* s, int L, int mode, double* P, double* E, rowstat* st) {
  double m = s[0];
  int am = 0;
  double n = s[0];
  int an = 0;
  for (int j = 1; j < L; ++j) {
    if (s[j] > m) { m = s[j]; am = j; }
    if (s[j] < n) { n = s[j]; an = j; }
  }
  double W = 0.0;
  for (int j = 0; j < L; ++j) {
    E[j] = exp(s[j] - m);
    P[j] = mode ? rounded_exp(s[j] - m, mode) : E[j];
    W += P[j];
  }
  for (int j = 0; j < L; ++j) P[j] /= W;
  st->m = m; st->n = n; st->am = am; st->an = an; st->h = 0.0;
  st->WL = W; st->WN = W; st->degen = 0;
}


/* ------------------------------------------------------------- row API */

/* Rows of scores (fp64, row-major [rows, cols]); row i sees keys
 * 0..row_len[i]-1.  dP is the upstream dL/dP (same shape) or NULL for a
 * forward only.  Outputs (each nullable): P_fwd, dS, P_L, P_N (the LERP and
 * Nearest probabilities), stats [rows, ST_COUNT].  frozen_m / frozen_n
 * (nullable, per row) override the row extrema for finite-difference checks
 * of the partial gradient modes.  Returns 0, or -1 on bad arguments. */
int kiattn_ref_rows(const double* S, const int* row_len, int rows, int cols,
                    const double* dP, const ref_cfg* c, const double* frozen_m,
                    const double* frozen_n, double* P_fwd, double* dS, double* P_L,
                    double* P_N, double* stats) {
  if (!S || !row_len || !c || rows < 0 || cols <= 0 || c->K < 1) return -1;
  int bad = 0;
#pragma omp parallel
  {
    double* wL = (double*)malloc(sizeof(double) * cols);
    double* wN = (double*)malloc(sizeof(double) * cols);
    double* tt = (double*)malloc(sizeof(double) * cols);
    double* Pb = (double*)malloc(sizeof(double) * cols);
    double* ds = (double*)malloc(sizeof(double) * cols);
    int* kk = (int*)malloc(sizeof(int) * cols);
    unsigned char* win = (unsigned char*)malloc(cols);
#pragma omp for schedule(dynamic, 4)
    for (int i = 0; i < rows; ++i) {
      const int L = row_len[i];
      const double* s = S + (size_t)i * cols;
      double* pf = P_fwd ? P_fwd + (size_t)i * cols : NULL;
      if (L < 1 || L > cols) { bad = 1; continue; }
      rowstat st;
      double A = 0.0, C = 0.0;
      if (c->softmax) {
        softmax_row_r(s, L, c->exp_round, Pb, ds, &st);
        if (pf) { for (int j = 0; j < cols; ++j) pf[j] = j < L ? Pb[j] : 0.0; }
        if (P_L) { for (int j = 0; j < cols; ++j) P_L[(size_t)i * cols + j] = j < L ? Pb[j] : 0.0; }
        if (P_N) { for (int j = 0; j < cols; ++j) P_N[(size_t)i * cols + j] = j < L ? Pb[j] : 0.0; }
        if (dP && dS) {
          const double* dp = dP + (size_t)i * cols;
          double D = 0.0;
          for (int j = 0; j < L; ++j) D += Pb[j] * dp[j];
          /* e^{s-m} (dP - D) / W: the softmax Jacobian, taken straight through
           * the rounding of the reduced-precision baselines */
          for (int j = 0; j < cols; ++j)
            dS[(size_t)i * cols + j] = j < L ? ds[j] / st.WL * (dp[j] - D) : 0.0;
        }
      } else {
        row_forward(s, L, c, frozen_m ? frozen_m + i : NULL, frozen_n ? frozen_n + i : NULL,
                    wL, wN, kk, tt, win, &st);
        const int lerp_fwd = uses_lerp_forward(c);
        for (int j = 0; j < cols; ++j) {
          double pl = j < L ? wL[j] / st.WL : 0.0;
          double pn = j < L ? wN[j] / st.WN : 0.0;
          if (pf) pf[j] = lerp_fwd ? pl : pn;
          if (P_L) P_L[(size_t)i * cols + j] = pl;
          if (P_N) P_N[(size_t)i * cols + j] = pn;
        }
        if (dP && dS) {
          const double* dp = dP + (size_t)i * cols;
          const int lerp_np = uses_lerp_normpoint(c);
          double D = 0.0;
          for (int j = 0; j < L; ++j) {
            double pb = lerp_np ? wL[j] / st.WL : wN[j] / st.WN;
            D += pb * dp[j];
          }
          row_backward(s, L, c, &st, wL, wN, kk, tt, win, dp, D, ds, &A, &C);
          for (int j = 0; j < cols; ++j) dS[(size_t)i * cols + j] = j < L ? ds[j] : 0.0;
        }
      }
      if (stats) {
        double* o = stats + (size_t)i * ST_COUNT;
        o[ST_M] = st.m; o[ST_N] = st.n; o[ST_AM] = st.am; o[ST_AN] = st.an;
        o[ST_H] = st.h;
        o[ST_WFWD] = (c->softmax || uses_lerp_forward(c)) ? st.WL : st.WN;
        o[ST_WL] = st.WL; o[ST_WN] = st.WN; o[ST_A] = A; o[ST_C] = C;
        o[ST_DEGEN] = st.degen;
      }
    }
    free(wL); free(wN); free(tt); free(Pb); free(ds); free(kk); free(win);
  }
  return bad ? -1 : 0;
}

/* -------------------------------------------------------- attention API */

/* Full operator on [BH, T, d] fp32 inputs, fp64 arithmetic.
 * O is required; dQ/dK/dV are computed when dO and all three are given.
 * O_bar (nullable) receives the output at the normalisation point (O_L for
 * Prob-STE, else O).  stats (nullable) [BH*T, ST_COUNT].  P_dump / dS_dump
 * (nullable) [BH, T, T].  With c->rounding != NONE every operand of every
 * product (Q, K for S; w, V for PV; dO, V for dP; P, dO for dV; dS, Q for dK;
 * dS, K for dQ) is first rounded to TF32 by the stated rule; row sums,
 * centering and normalisation stay in fp64.  Only (bh) pairs in
 * [bh_begin, bh_end) are computed (bounded samples). */
int kiattn_ref_attention(const float* Q, const float* Kt, const float* V, const float* dO,
                         int BH, int T, int d, const ref_cfg* c, int bh_begin, int bh_end,
                         double* O, double* O_bar, double* dQ, double* dK, double* dV,
                         double* stats, double* P_dump, double* dS_dump) {
  if (!Q || !Kt || !V || !O || !c || BH < 1 || T < 1 || d < 1 || c->K < 1) return -1;
  if (bh_begin < 0 || bh_end > BH || bh_begin >= bh_end) return -1;
  const int want_bwd = dO && dQ && dK && dV;
  const int R = c->rounding;
  int bad = 0;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * T);
    double* wL = (double*)malloc(sizeof(double) * T);
    double* wN = (double*)malloc(sizeof(double) * T);
    double* tt = (double*)malloc(sizeof(double) * T);
    double* P = (double*)malloc(sizeof(double) * T);
    double* dp = (double*)malloc(sizeof(double) * T);
    double* ds = (double*)malloc(sizeof(double) * T);
    double* ob = (double*)malloc(sizeof(double) * d);
    int* kk = (int*)malloc(sizeof(int) * T);
    unsigned char* win = (unsigned char*)malloc(T);
    /* per-(b,h) rounded copies of the operands */
    double* q = (double*)malloc(sizeof(double) * (size_t)T * d);
    double* k = (double*)malloc(sizeof(double) * (size_t)T * d);
    double* v = (double*)malloc(sizeof(double) * (size_t)T * d);
    double* g = (double*)malloc(sizeof(double) * (size_t)T * d);
#pragma omp for schedule(dynamic, 1)
    for (int bh = bh_begin; bh < bh_end; ++bh) {
      const size_t base = (size_t)bh * T * d;
      for (size_t x = 0; x < (size_t)T * d; ++x) {
        q[x] = round_operand(Q[base + x], R);
        k[x] = round_operand(Kt[base + x], R);
        v[x] = round_operand(V[base + x], R);
        g[x] = want_bwd ? round_operand(dO[base + x], R) : 0.0;
      }
      if (want_bwd) {
        for (size_t x = 0; x < (size_t)T * d; ++x) { dQ[base + x] = 0.0; dK[base + x] = 0.0; dV[base + x] = 0.0; }
      }
      for (int i = 0; i < T; ++i) {
        const int L = c->causal ? i + 1 : T;
        for (int j = 0; j < L; ++j) {
          double acc = 0.0;
          for (int x = 0; x < d; ++x) acc += q[(size_t)i * d + x] * k[(size_t)j * d + x];
          s[j] = acc;
        }
        rowstat st;
        double A = 0.0, C = 0.0;
        double Wfwd, Wbar;
        const double *wf, *wb;
        if (c->softmax) {
          softmax_row_r(s, L, c->exp_round, P, wN, &st);   /* wN: unrounded e^{s-m} */
          /* unnormalised weights so that O = sum(w v)/W like the rest */
          for (int j = 0; j < L; ++j) wL[j] = P[j] * st.WL;
          wf = wL; wb = wL; Wfwd = st.WL; Wbar = st.WL;
        } else {
          row_forward(s, L, c, NULL, NULL, wL, wN, kk, tt, win, &st);
          wf = uses_lerp_forward(c) ? wL : wN;
          Wfwd = uses_lerp_forward(c) ? st.WL : st.WN;
          wb = uses_lerp_normpoint(c) ? wL : wN;
          Wbar = uses_lerp_normpoint(c) ? st.WL : st.WN;
        }
        /* O = (sum_j w_j v_j) / W  (Appendix A: P = w / W, O = P V) */
        double* o = O + base + (size_t)i * d;
        for (int x = 0; x < d; ++x) { o[x] = 0.0; ob[x] = 0.0; }
        for (int j = 0; j < L; ++j) {
          const double rf = round_operand_d(wf[j], R);
          const double rb = round_operand_d(wb[j], R);
          for (int x = 0; x < d; ++x) {
            o[x] += rf * v[(size_t)j * d + x];
            ob[x] += rb * v[(size_t)j * d + x];
          }
        }
        for (int x = 0; x < d; ++x) { o[x] /= Wfwd; ob[x] /= Wbar; }
        if (O_bar) for (int x = 0; x < d; ++x) O_bar[base + (size_t)i * d + x] = ob[x];
        if (P_dump) {
          double* pr = P_dump + ((size_t)bh * T + i) * T;
          for (int j = 0; j < T; ++j) pr[j] = j < L ? wf[j] / Wfwd : 0.0;
        }
        if (want_bwd) {
          /* dP_j = dO_i . v_j ; centering D = dO_i . O_bar_i */
          for (int j = 0; j < L; ++j) {
            double acc = 0.0;
            for (int x = 0; x < d; ++x) acc += g[(size_t)i * d + x] * v[(size_t)j * d + x];
            dp[j] = acc;
          }
          double D = 0.0;
          for (int x = 0; x < d; ++x) D += (double)dO[base + (size_t)i * d + x] * ob[x];
          if (c->softmax) {
            /* straight through the baselines' rounding: slope e^{s-m} / W */
            for (int j = 0; j < L; ++j) ds[j] = wN[j] / st.WL * (dp[j] - D);
          } else {
            row_backward(s, L, c, &st, wL, wN, kk, tt, win, dp, D, ds, &A, &C);
          }
          for (int j = 0; j < L; ++j) {
            const double dsr = round_operand_d(ds[j], R);
            const double pr = round_operand_d(wf[j] / Wfwd, R);
            for (int x = 0; x < d; ++x) {
              dQ[base + (size_t)i * d + x] += dsr * k[(size_t)j * d + x];
              dK[base + (size_t)j * d + x] += dsr * q[(size_t)i * d + x];
              dV[base + (size_t)j * d + x] += pr * g[(size_t)i * d + x];
            }
          }
          if (dS_dump) {
            double* dr = dS_dump + ((size_t)bh * T + i) * T;
            for (int j = 0; j < T; ++j) dr[j] = j < L ? ds[j] : 0.0;
          }
        }
        if (stats) {
          double* so = stats + ((size_t)bh * T + i) * ST_COUNT;
          so[ST_M] = st.m; so[ST_N] = st.n; so[ST_AM] = st.am; so[ST_AN] = st.an;
          so[ST_H] = st.h; so[ST_WFWD] = Wfwd; so[ST_WL] = st.WL; so[ST_WN] = st.WN;
          so[ST_A] = A; so[ST_C] = C; so[ST_DEGEN] = st.degen;
        }
      }
    }
    free(s); free(wL); free(wN); free(tt); free(P); free(dp); free(ds); free(ob);
    free(kk); free(win); free(q); free(k); free(v); free(g);
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------- fp32 weight stage (bit-exact) */

/* fp64 exponential for x <= 0 from IEEE operations in a fixed order:
 * Cody & Waite argument reduction (x = n ln2 + r, ln2 split into a head
 * with trailing zero bits so that n * head is exact, and a tail) followed
 * by the Taylor series of e^r through r^13/13! in Horner form, then an exact
 * scaling by 2^n.  |r| <= ln2/2 bounds the truncation term below 1e-17.
 * Results below 2^-150 (x < -104) round to 0 in fp32 and are returned as 0. */
static double own_exp(double x) {
  if (x < -104.5) return 0.0;
  if (x == 0.0) return 1.0;
  const double inv_ln2 = 1.4426950408889634;          /* 1/ln 2 */
  const double ln2_hi = 0.693147180369123816490;       /* 0x1.62e42fee00000p-1 */
  const double ln2_lo = 1.90821492927058770002e-10;    /* ln 2 - ln2_hi */
  double nd = nearbyint(x * inv_ln2);
  double r = (x - nd * ln2_hi) - nd * ln2_lo;
  /* 1/k! for k = 13..2, written out as quotients of exact integers */
  double p = 1.0 / 6227020800.0;           /* 13! */
  p = fma(p, r, 1.0 / 479001600.0);        /* 12! */
  p = fma(p, r, 1.0 / 39916800.0);         /* 11! */
  p = fma(p, r, 1.0 / 3628800.0);          /* 10! */
  p = fma(p, r, 1.0 / 362880.0);           /* 9! */
  p = fma(p, r, 1.0 / 40320.0);            /* 8! */
  p = fma(p, r, 1.0 / 5040.0);             /* 7! */
  p = fma(p, r, 1.0 / 720.0);              /* 6! */
  p = fma(p, r, 1.0 / 120.0);              /* 5! */
  p = fma(p, r, 1.0 / 24.0);               /* 4! */
  p = fma(p, r, 1.0 / 6.0);                /* 3! */
  p = fma(p, r, 0.5);                      /* 2! */
  p = fma(p, r, 1.0);
  p = fma(p, r, 1.0);
  return ldexp(p, (int)nd);
}

double kiattn_ref_own_exp(double x) { return own_exp(x); }

/* The fp32 weight stage, written as the fixed sequence of fp32 operations
 * that the CUDA path must reproduce bit for bit (row extrema, width,
 * reciprocal width, u, interval index, t, grid, LERP/Nearest weight).
 * S is fp32 [rows, cols]; row i sees keys 0..row_len[i]-1.
 * Outputs: w (fp32), bin (k for LERP, r for Nearest, -1 tail or invisible),
 * t (fp32), row_m, row_n (fp32), each nullable except w. */
int kiattn_ref_weights_fp32(const float* S, int rows, int cols, const int* row_len,
                            const ref_cfg* c, float* w, int* bin, float* tout, float* row_m,
                            float* row_n) {
  if (!S || !row_len || !c || !w || rows < 0 || cols <= 0 || c->K < 1 || c->K > 1024) return -1;
  const int K = c->K;
  const float Kf = (float)K;
  const float tau = (float)c->tau;
  int bad = 0;
#pragma omp parallel for schedule(static)
  for (int i = 0; i < rows; ++i) {
    const float* s = S + (size_t)i * cols;
    const int L = row_len[i];
    if (L < 1 || L > cols) { bad = 1; continue; }
    float m = s[0], n = s[0];
    for (int j = 1; j < L; ++j) {
      if (s[j] > m) m = s[j];
      if (s[j] < n) n = s[j];
    }
    if (row_m) row_m[i] = m;
    if (row_n) row_n[i] = n;
    float h, rh;
    int degen = 0;
    if (c->cal == REF_CAL_MINMAX) {
      float span = m - n;
      if (span < 1e-12f) degen = 1;
      h = span / Kf;
      rh = Kf / span;
    } else {
      h = tau / Kf;
      rh = Kf / tau;
    }
    const int fixed = c->cal == REF_CAL_FIXED;
    float G[1024 + 1];
    if (!degen && !fixed) {
      for (int k = 0; k <= K; ++k) G[k] = (float)own_exp(-(double)k * (double)h);
    }
    for (int j = 0; j < cols; ++j) {
      float wj = 0.0f, tj = 0.0f;
      int bj = -1;
      if (j < L) {
        if (degen) {
          wj = 1.0f; bj = 0; tj = 0.0f;
        } else {
          float diff = m - s[j];
          float uu = diff * rh;
          int tail = 0;
          if (c->cal == REF_CAL_MINMAX) {
            if (uu > Kf) uu = Kf;
          } else if (c->cal == REF_CAL_FWM) {
            tail = uu > Kf;
          }
          if (!tail) {
            int k = (int)floorf(uu);
            if (!fixed && k > K - 1) k = K - 1;
            float t = uu - (float)k;
            /* fixed step: grid values on demand, G_k = RN32(E(-k h)) for any k */
            const float Gk = fixed ? (float)own_exp(-(double)k * (double)h) : G[k];
            const float Gk1 = fixed ? (float)own_exp(-(double)(k + 1) * (double)h) : G[k + 1];
            if (c->rec == REF_REC_LERP) {
              float a = Gk1 - Gk;
              wj = fmaf(t, a, Gk);
              bj = k;
            } else {
              int r = k + (t >= 0.5f ? 1 : 0);
              wj = r == k ? Gk : Gk1;
              bj = r;
            }
            tj = t;
          }
        }
      }
      w[(size_t)i * cols + j] = wj;
      if (bin) bin[(size_t)i * cols + j] = bj;
      if (tout) tout[(size_t)i * cols + j] = tj;
    }
  }
  return bad ? -1 : 0;
}

int kiattn_ref_stat_count(void) { return ST_COUNT; }
