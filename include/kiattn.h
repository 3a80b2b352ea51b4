/*
 * kiattn -- K-interval attention (quantized softmax in attention), forward
 * and backward, on NVIDIA B200 (sm_100a).  C ABI.
 *
 * The operator is the one defined in "Pretraining Transformers with
 * Quantized Softmax in Attention" (Zhu, Hu, Kozlowski; arXiv 2609.33591):
 *   section 3 (operator family, calibration, reconstruction, calibration
 *   gradients, surrogate placement), Appendix A (operator definitions and
 *   edge cases) and Appendix B (gradient derivations).
 *
 * For one (batch, head) and query row i with visible keys J_i (j <= i when
 * causal, all keys otherwise):
 *   s_j = q_i . k_j                     (no 1/sqrt(d): the caller scales Q)
 *   m = max s, n = min s                (arg-extrema: lowest index on ties)
 *   h = (m - n)/K  (MinMax)   or   tau/K  (FWM)
 *   u_j = (m - s_j)/h,  k_j = min(floor u_j, K-1),  t_j = u_j - k_j
 *   G_k = e^{-k h}, k = 0..K            (the K+1 grid values)
 *   LERP     w_j = G_k + t_j (G_{k+1} - G_k)
 *   Nearest  w_j = G_{k + [t_j >= 1/2]}
 *   FWM: w_j = 0 when u_j > K (the tail below m - tau)
 *   MinMax rows with span m - n < 1e-12: w_j = 1 (degenerate branch)
 *   P = w / sum(w),  O_i = sum_j P_j v_j
 * Backward, with the normalisation Jacobian at the surrogate's point (LERP
 * and Prob-STE at the LERP weights, Weight-STE at the hard weights), the LERP
 * scalar derivatives, and the calibration derivatives through m (and n)
 * filtered by the gradient mode (full, detach, max-only, min-only, zero-sum
 * projection).
 *
 * Conventions for every entry point:
 *   - Tensors are device pointers to fp32, contiguous [B, H, T, d], 16-byte
 *     aligned.  Keys are stored like Q (not transposed); the argument is
 *     called Kt only to keep it apart from the interval count K.
 *   - The caller owns and allocates every buffer (outputs, stats,
 *     workspace).  The library allocates nothing, never synchronises, and
 *     enqueues all work on `stream` (a cudaStream_t; NULL = legacy default).
 *   - Return 0 on success or a negative KIA_ERR_* code; nothing is launched
 *     when an argument check fails.  kiattn_strerror() names the code.
 *   - Supported: d in {64, 128}; T >= 1 (any T, ragged tails included);
 *     1 <= K <= 64; tau > 0 (FWM); B*H*T <= 2^30.
 */
#ifndef KIATTN_H_
#define KIATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* calibration (section 3, Calibration) */
#define KIA_CAL_MINMAX 0 /* h = row span / K */
#define KIA_CAL_FWM 1    /* window [m - tau, m], h = tau / K, zero tail */
/* untruncated fixed step (Appendix D.4): h = tau / K anchored at the row
 * maximum like FWM, with the grid continued past node K over the whole row
 * span (nodes until e^{-k h} underflows in fp32, k h >= 104.5); calibration
 * gradient as FWM's (the maximum only).  Needs ceil(104.5 K / tau) <= 400,
 * else KIA_ERR_UNSUPPORTED (e.g. tau = 6 allows K <= 22). */
#define KIA_CAL_FIXED 2
/* reconstruction (section 3, Reconstruction) */
#define KIA_REC_LERP 0
#define KIA_REC_NEAREST 1
/* surrogate placement for Nearest (section 3, Surrogate placement; Figure 1) */
#define KIA_STE_WEIGHT 0 /* straight-through before normalisation */
#define KIA_STE_PROB 1   /* straight-through after normalisation */
/* gradient mode (section 3, Calibration gradients; Appendix B; section 5.1) */
#define KIA_GRAD_FULL 0
#define KIA_GRAD_DETACH 1
#define KIA_GRAD_MAX_ONLY 2
#define KIA_GRAD_MIN_ONLY 3
#define KIA_GRAD_PROJECT 4
/* contraction arithmetic (Appendix C.1: TF32 products in training) */
#define KIA_GEMM_TF32 0 /* tcgen05 TF32 tensor-core products, fp32 accumulation */
#define KIA_GEMM_FP32 1 /* exact fp32 products on the CUDA cores (checking mode) */
/* operator */
#define KIA_OP_KINTERVAL 0
#define KIA_OP_SOFTMAX 1 /* exact softmax attention (Appendix G reference row) */
/* reduced-precision exponential baselines (Appendix D.5): softmax whose
 * numerator e^{s-m} (fp32) is rounded to nearest-even bfloat16, or to
 * nearest-even FP8 E4M3; P = R(e) / sum R(e).  The backward passes straight
 * through the rounding (dS_j = e_j (dP_j - D) / W, e unrounded, D the row's
 * dO . O, W the rounded normaliser) with the row maximum held fixed, as
 * softmax's stabilising shift.  The calibration and gradient-mode fields do
 * not apply. */
#define KIA_OP_SOFTMAX_BF16EXP 2
#define KIA_OP_SOFTMAX_FP8EXP 3

/* error codes */
#define KIA_OK 0
#define KIA_ERR_INVALID_ARG -1  /* null pointer, bad size, bad enum, misalignment */
#define KIA_ERR_UNSUPPORTED -2  /* valid but not implemented (e.g. d not 64/128) */
#define KIA_ERR_CUDA -3         /* a CUDA launch or driver call failed */
#define KIA_ERR_TIMEOUT -4      /* a bounded device-side wait gave up */
#define KIA_ERR_STATS_MISMATCH -5 /* stats buffer written by another shape/config */
#define KIA_ERR_CAPACITY -6     /* size beyond a fixed-capacity entry point's limit */

typedef struct {
  int n_intervals; /* K >= 1 */
  int cal;         /* KIA_CAL_* */
  float tau;       /* FWM window width in nats (6 in the paper); fixed-step K h */
  int rec;         /* KIA_REC_* */
  int ste;         /* KIA_STE_* (ignored for LERP) */
  int grad;        /* KIA_GRAD_* (backward only) */
  int causal;      /* 1: key j visible to query i iff j <= i */
  int gemm;        /* KIA_GEMM_* */
  int op;          /* KIA_OP_* */
} kia_config;

/* Bytes of the per-row statistics buffer that kiattn_fwd writes and
 * kiattn_bwd reads: row max/min and their indices, 1/h, the normalisers,
 * the per-row grid (MinMax), and for Prob-STE the LERP-point output O_L.
 * Returns 0 for invalid arguments. */
size_t kiattn_stats_bytes(int B, int H, int T, int d, const kia_config* cfg);

/* Bytes of device scratch kiattn_bwd needs (per-row centering D, the row
 * sums A and C of the calibration terms, the calibration coefficients).
 * Returns 0 for invalid arguments. */
size_t kiattn_workspace_bytes(int B, int H, int T, int d, const kia_config* cfg);

/* Forward (section 3; Appendix A).  Q, Kt, V: inputs [B,H,T,d].  O: output
 * [B,H,T,d].  stats: kiattn_stats_bytes() bytes, written here and read by
 * kiattn_bwd (keep it unchanged between the two calls).  The forward does
 * not depend on cfg->grad, so one forward serves every gradient mode.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
int kiattn_fwd(const float* Q, const float* Kt, const float* V, float* O, void* stats, int B,
               int H, int T, int d, const kia_config* cfg, void* stream);

/* Backward (section 3, Calibration gradients and Surrogate placement;
 * Appendix B).  Inputs Q, Kt, V, O (the forward output), dO [B,H,T,d] and
 * the stats written by kiattn_fwd with the same shape and config (cfg->grad
 * may differ).  Outputs dQ, dK, dV [B,H,T,d] (overwritten).  dS_dbg, when
 * not NULL, receives the score gradient [B,H,T,T] (invisible entries 0) for
 * checking.  workspace: kiattn_workspace_bytes() bytes of device scratch,
 * contents on entry irrelevant.
 * Errors: INVALID_ARG, UNSUPPORTED, STATS_MISMATCH, CUDA. */
int kiattn_bwd(const float* Q, const float* Kt, const float* V, const float* O, const float* dO,
               const void* stats, float* dQ, float* dK, float* dV, float* dS_dbg, int B, int H,
               int T, int d, const kia_config* cfg, void* workspace, void* stream);

/* Backward for callers that cannot allocate device memory.  Some callers
 * can't call cudaMalloc: a plugin inside a host engine that owns all device
 * memory and forbids allocation once it has started, or a latency-bound
 * loop where an allocation would synchronise the device.  This entry point
 * takes the same arguments as kiattn_bwd minus the workspace and uses a
 * scratch array that the library itself declares (no counterpart in the
 * paper: it only changes where the backward's scratch lives).
 *   - Capacity: B*H*T <= KIA_NOALLOC_MAX_ROWS rows; larger calls return
 *     KIA_ERR_CAPACITY and launch nothing.  Every GPU that loads the
 *     library holds the scratch (about 28 MiB) until the process exits.
 *   - The first call in a CUDA context (normally the device's primary
 *     context, made current by cudaSetDevice) looks up the scratch's device
 *     address in that context; make that first call before any stream
 *     capture.  The address is kept per context, so after cudaDeviceReset,
 *     or under another context of the same device, the next call looks it up
 *     again (again outside capture).
 *   - It calls no cudaMalloc / cudaFree.  Each call clears the scratch
 *     fields that must start at zero; the scratch keeps the last call's
 *     contents otherwise.
 *   - All calls share one scratch per device: calls that overlap on the GPU
 *     (several streams, several host threads) race; serialise them.
 *   - The scratch is the library's own, so the caller has no handle to the
 *     per-row calibration coefficients the backward leaves in it:
 *     kiattn_grad_decomposition needs a kiattn_bwd call with a workspace of
 *     the caller's. */
#define KIA_NOALLOC_MAX_ROWS (1 << 20)
int kiattn_bwd_noalloc(const float* Q, const float* Kt, const float* V, const float* O,
                       const float* dO, const void* stats, float* dQ, float* dK, float* dV,
                       float* dS_dbg, int B, int H, int T, int d, const kia_config* cfg,
                       void* stream);

/* The fp32 weight stage alone on given scores (section 3, Reconstruction;
 * Appendix A), for bit-exact checking.  S: device fp32 [rows, cols]; row i
 * sees keys 0..row_len[i]-1 (device int32 [rows], 1..cols).  Outputs
 * (device, [rows, cols]; t, bin, row_m, row_n nullable): w the weight, bin
 * the interval index k (LERP) or node r (Nearest), -1 for FWM tail or
 * invisible keys, t the in-interval position; row_m / row_n [rows] the
 * row extrema.  Degenerate MinMax rows give w = 1, bin = 0, t = 0.
 * Errors: INVALID_ARG, CUDA. */
int kiattn_weights_from_S(const float* S, int rows, int cols, const int* row_len,
                          const kia_config* cfg, float* w, int* bin, float* t, float* row_m,
                          float* row_n, void* stream);

/* The score contraction of the forward alone, S = Q Kt^T per (batch, head),
 * with the same tile path and arithmetic as kiattn_fwd (cfg->gemm).  S:
 * device fp32 [B,H,T,T]; entries outside the visible set are set to 0.
 * For checking the TF32 operand rounding against the oracle.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
int kiattn_scores(const float* Q, const float* Kt, float* S, int B, int H, int T, int d,
                  const kia_config* cfg, void* stream);

/* Fixed-upstream decomposition of the score gradient (Appendix F, "The
 * detached-gradient record and its replication"; Table S24): for each row i,
 * out[3 i + 0] = ||dS_i||^2 (the backward's dS of the mode it ran with),
 * out[3 i + 1] = the squared norm of that mode's maximum-side calibration
 * term (g_m^2 for full and max-only; under the zero-sum projection the
 * common-mode shift c_i on every visible key, c_i^2 |J_i|; 0 otherwise),
 * out[3 i + 2] = that of the minimum-side term (g_n^2 for full and min-only,
 * 0 otherwise), i.e. the norms of (mode - detach) split by extremum.  The
 * maximum- and minimum-dependent norm ratios of the appendix are
 * sqrt(sum out[.,1] / sum out[.,0]) and sqrt(sum out[.,2] / sum out[.,0])
 * over the rows of interest.
 * dS: the dS_dbg [B,H,T,T] written by kiattn_bwd; workspace: the workspace of
 * that same kiattn_bwd call (it holds g_m, g_n per row); cfg as in that call;
 * out: device fp64 [B*H*T*3], caller-owned.  Sums run in fp64 (groups of
 * four squares in fp32 first).  Nothing is written when the kiattn_bwd call
 * rejected its stats (workspace status set).
 * Errors: INVALID_ARG (null pointer, B, H or T < 1), UNSUPPORTED (shape
 * beyond the operator's limits), CUDA (launch failure). */
int kiattn_grad_decomposition(const float* dS, const void* workspace, int B, int H, int T,
                              const kia_config* cfg, double* out, void* stream);

/* Geometry probe (section 4, geometry probe; section 5.4; Appendix D.6,
 * Figure S4): per query row, on given scores, the quantities the paper
 * records to describe learned score geometry.  Fields of out[row * 8 + f]:
 *   KIA_GEO_SPAN         m - n over the row's visible keys
 *   KIA_GEO_H            native interval width h (MinMax span / K, 0 for a
 *                        degenerate row; FWM and fixed step tau / K)
 *   KIA_GEO_QNORM        ||q_i||_2 (0 when Q is NULL)
 *   KIA_GEO_ENT_SOFTMAX  entropy (nats) of softmax(s_i)
 *   KIA_GEO_ENT_OP       entropy of the operator's forward probabilities
 *   KIA_GEO_TV           total variation 1/2 sum_j |P_op - P_softmax|
 *   KIA_GEO_TOP_SOFTMAX  softmax mass on the keys whose nearest grid node is
 *                        node 0 (the top rounding bucket)
 *   KIA_GEO_TOP_OP       the operator's mass on the same keys
 * The operator weights and the grid decisions are the forward's fp32 weight
 * stage (bit-identical to kiattn_weights_from_S); sums run in fp32.
 * S: device fp32 [B,H,T,T] row-major scores (e.g. from kiattn_scores); row i
 * sees keys j <= i when cfg->causal, else all T.  Q: device fp32 [B,H,T,d]
 * or NULL.  cfg: the grid to measure against (cal, K, tau, rec, causal;
 * op must be KIA_OP_KINTERVAL; grad and ste are ignored).  out: device fp32
 * [B*H*T*8], caller-owned.  Runs on `stream`, allocates nothing.
 * Errors: INVALID_ARG (null S or out, B, H or T < 1, d < 1 with Q given, op
 * not K-interval), UNSUPPORTED (shape beyond the operator's limits), CUDA. */
#define KIA_GEO_SPAN 0
#define KIA_GEO_H 1
#define KIA_GEO_QNORM 2
#define KIA_GEO_ENT_SOFTMAX 3
#define KIA_GEO_ENT_OP 4
#define KIA_GEO_TV 5
#define KIA_GEO_TOP_SOFTMAX 6
#define KIA_GEO_TOP_OP 7
#define KIA_GEO_FIELDS 8
int kiattn_geometry(const float* S, const float* Q, int B, int H, int T, int d,
                    const kia_config* cfg, float* out, void* stream);

/* Error word raised by device code since the last reset: KIA_ERR_TIMEOUT
 * when a bounded wait inside a kernel gave up, KIA_ERR_STATS_MISMATCH when
 * kiattn_bwd was handed stats written for another shape or config (the
 * backward kernels then skip their work), 0 otherwise.  Synchronous: it
 * copies the word from the device (and clears it when reset != 0). */
int kiattn_device_error(int reset);

/* Test hook for the bounded device-side waits (failure handling without a
 * GPU fault; no counterpart in the paper).  Every wait inside the tensor-core
 * kernels gives up after a time limit, raises KIA_ERR_TIMEOUT in the error
 * word read by kiattn_device_error(), lets the copies and MMAs already in
 * flight land, frees its tensor memory and returns, so the context stays
 * usable.  what = 1 makes every following kiattn_fwd on the tensor-core
 * path withhold one operand copy -- the first CTA never issues its first Q
 * tile, so nothing is in flight for it and the waits on it run out; the
 * outputs of that call are then undefined.  wait_limit_ns > 0 sets the limit
 * of every wait (default 2 s) so that a test does not sit out the default.
 * kiattn_debug_bounded_wait(0, 0) restores the defaults.  Synchronous (it
 * writes the limit to the device); not thread-safe; meant for tests.
 * Errors: INVALID_ARG (what not 0 or 1), CUDA. */
int kiattn_debug_bounded_wait(int what, unsigned long long wait_limit_ns);

/* Phase timing for profiling.  kiattn_profile_enable(1) makes kiattn_fwd
 * and kiattn_bwd record CUDA events on their stream around each internal
 * kernel (the library creates its events once; no device memory).
 * kiattn_profile_read() synchronises on the last recorded event and writes
 * the milliseconds of the most recent calls' phases into ms[0..n-1] in this
 * order: forward kernel, backward row prep, backward query pass, backward
 * key pass, backward calibration rows; it returns the number written or a
 * negative KIA_ERR_* code.  Not thread-safe; meant for benchmarks. */
int kiattn_profile_enable(int on);
int kiattn_profile_read(float* ms, int n);

/* Human-readable name of a KIA_* return code (static string). */
const char* kiattn_strerror(int code);

/* Library version, major * 10000 + minor * 100 + patch. */
int kiattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KIATTN_H_ */
