// kiattn C ABI: argument checks, launch configuration and the order of the
// kernels for K-interval attention forward and backward on sm_100a.
// One translation unit: the kernels live in the headers included below.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "../../include/kiattn.h"
#include "kia_common.cuh"
#include "kia_elem.cuh"
#include "kia_epilogue.cuh"
#include "kia_geometry.cuh"
#include "kia_simt.cuh"
#include "kia_stats.cuh"
#include "kia_tc.cuh"
#include "kia_weights.cuh"

using namespace kia;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------ phase profiling
// Events: 0 fwd start, 1 fwd end, 2 bwd start, 3 after prep, 4 after the
// query pass, 5 after the key pass, 6 after the calibration rows.
constexpr int kProfEvents = 7;
bool g_prof_on = false;
bool g_prof_created = false;
cudaEvent_t g_prof_ev[kProfEvents];

void prof_mark(int i, cudaStream_t s) {
  if (g_prof_on) cudaEventRecord(g_prof_ev[i], s);
}

// failure-handling test hook (kiattn_debug_bounded_wait)
int g_withhold = 0;

// Extent of the untruncated fixed-step grid (Appendix D.4): the node count
// Kc at which G_Kc = RN32(e^{-Kc h}) is zero (every Kc h >= 104.5 nats, since
// e^{-103.98} is already below half the least fp32 subnormal), so that keys
// past node Kc carry exactly zero weight and may be treated as a tail.
int fixed_step_extent(const kia_config* cfg) {
  const float h = cfg->tau / (float)cfg->n_intervals;
  const double kc = ceil(104.5 / (double)h);
  return kc < 1.0 ? 1 : (kc > 1e9 ? 1000000000 : (int)kc);
}

int check_config(const kia_config* cfg) {
  if (!cfg) return KIA_ERR_INVALID_ARG;
  if (cfg->n_intervals < 1 || cfg->n_intervals > KIA_MAX_K) return KIA_ERR_UNSUPPORTED;
  if (cfg->cal != KIA_CAL_MINMAX && cfg->cal != KIA_CAL_FWM && cfg->cal != KIA_CAL_FIXED)
    return KIA_ERR_INVALID_ARG;
  if (cfg->rec != KIA_REC_LERP && cfg->rec != KIA_REC_NEAREST) return KIA_ERR_INVALID_ARG;
  if (cfg->ste != KIA_STE_WEIGHT && cfg->ste != KIA_STE_PROB) return KIA_ERR_INVALID_ARG;
  if (cfg->grad < KIA_GRAD_FULL || cfg->grad > KIA_GRAD_PROJECT) return KIA_ERR_INVALID_ARG;
  if (cfg->gemm != KIA_GEMM_TF32 && cfg->gemm != KIA_GEMM_FP32) return KIA_ERR_INVALID_ARG;
  if (cfg->op < KIA_OP_KINTERVAL || cfg->op > KIA_OP_SOFTMAX_FP8EXP) return KIA_ERR_INVALID_ARG;
  if (cfg->causal != 0 && cfg->causal != 1) return KIA_ERR_INVALID_ARG;
  if (cfg->cal != KIA_CAL_MINMAX && !(cfg->tau > 0.0f && cfg->tau < 1e30f))
    return KIA_ERR_INVALID_ARG;
  if (cfg->cal == KIA_CAL_FIXED && cfg->op == KIA_OP_KINTERVAL &&
      fixed_step_extent(cfg) > KIA_MAX_KCAP)
    return KIA_ERR_UNSUPPORTED;
  return KIA_OK;
}

int check_shape(int B, int H, int T, int d) {
  if (B < 1 || H < 1 || T < 1) return KIA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return KIA_ERR_UNSUPPORTED;
  const long long rows = (long long)B * H * T;
  if (rows > (1ll << 30) || (long long)B * H > 65535ll * 1024) return KIA_ERR_UNSUPPORTED;
  if (rows * (long long)d > (1ll << 40)) return KIA_ERR_UNSUPPORTED;
  return KIA_OK;
}

OpParams make_params(const kia_config* cfg) {
  OpParams p;
  p.K = cfg->n_intervals;
  p.Kf = (float)p.K;
  p.cal = cfg->cal;
  p.rec = cfg->rec;
  p.ste = (cfg->rec == KIA_REC_LERP) ? KIA_STE_WEIGHT : cfg->ste;
  p.grad = cfg->grad;
  p.causal = cfg->causal;
  p.softmax = cfg->op != KIA_OP_KINTERVAL;
  p.exp_round = cfg->op == KIA_OP_SOFTMAX_BF16EXP ? 1 : (cfg->op == KIA_OP_SOFTMAX_FP8EXP ? 2 : 0);
  p.tau = cfg->tau;
  p.fwm_h = (cfg->cal != KIA_CAL_MINMAX) ? cfg->tau / p.Kf : 0.0f;
  p.fwm_rh = (cfg->cal != KIA_CAL_MINMAX) ? p.Kf / cfg->tau : 0.0f;
  p.tf32_ops = 0;
  p.fixed_step = 0;
  p.withhold = g_withhold;
  if (cfg->cal == KIA_CAL_FIXED) {
    // the fixed-step operator is FWM's grid (h = tau / K, anchored at the row
    // maximum) with its window widened to the grid's full extent
    p.cal = KIA_CAL_FWM;
    p.fixed_step = 1;
    p.K = fixed_step_extent(cfg);
    p.Kf = (float)p.K;
  }
  if (p.softmax) {  // the softmax row has no grid: normalise the unused axes
    p.cal = KIA_CAL_MINMAX;
    p.rec = KIA_REC_LERP;
    p.ste = KIA_STE_WEIGHT;
    p.K = 1;
    p.Kf = 1.0f;
    p.tau = 0.0f;
    p.fwm_h = p.fwm_rh = 0.0f;
    p.fixed_step = 0;
  }
  return p;
}

// With KIATTN_DEBUG set in the environment, a failed CUDA call prints the
// runtime's message to stderr; the return code is KIA_ERR_CUDA either way.
int cuda_fail(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return KIA_OK;
  if (getenv("KIATTN_DEBUG")) fprintf(stderr, "kiattn: %s: %s\n", where, cudaGetErrorString(e));
  return KIA_ERR_CUDA;
}

int launch_status() { return cuda_fail(cudaGetLastError(), "kernel launch"); }

template <typename Kern>
int set_smem(Kern k, size_t bytes) {
  if (bytes > 48 * 1024) {
    if (cuda_fail(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes),
                  "shared memory attribute"))
      return KIA_ERR_CUDA;
  }
  return KIA_OK;
}

size_t simt_tab_floats(const OpParams& p, int rowsPerTab) {
  if (p.softmax) return 0;
  return (p.cal == KIA_CAL_MINMAX) ? (size_t)(p.K + 1) * rowsPerTab : (size_t)(p.K + 1);
}

template <int D>
int simt_forward(const float* Q, const float* Kt, const float* V, float* O, void* stats, int B,
                 int H, int T, const OpParams& p, cudaStream_t s) {
  const long long rows = (long long)B * H * T;
  StatsView st = stats_view(stats, rows, D, p);
  const size_t smem =
      (kSimtRows * (D + 1) + 2 * kSimtKeys * D + simt_tab_floats(p, kSimtRows)) * sizeof(float);
  if (set_smem(simt_fwd_kernel<D>, smem)) return KIA_ERR_CUDA;
  dim3 grid((T + kSimtRows - 1) / kSimtRows, B * H);
  simt_fwd_kernel<D><<<grid, kSimtRows, smem, s>>>(Q, Kt, V, O, st, p, B, H, T);
  return launch_status();
}

template <int D>
int simt_backward(const float* Q, const float* Kt, const float* V, const float* dO,
                  const StatsView& st, const WorkView& wk, float* dQ, float* dK, float* dV,
                  float* dS_dbg, int B, int H, int T, const OpParams& p, cudaStream_t s) {
  dim3 grid((T + kSimtRows - 1) / kSimtRows, B * H);
  const size_t smq = (2 * kSimtRows * (D + 1) + 2 * kSimtKeys * D + simt_tab_floats(p, kSimtRows)) *
                     sizeof(float);
  if (set_smem(simt_bwd_q_kernel<D>, smq)) return KIA_ERR_CUDA;
  simt_bwd_q_kernel<D><<<grid, kSimtRows, smq, s>>>(Q, Kt, V, dO, st, wk, dQ, dS_dbg, p, T);
  if (launch_status()) return KIA_ERR_CUDA;
  const size_t smkv = (2 * kSimtRows * (D + 1) + 2 * kSimtKeys * D + kSimtKeys * 6 +
                       simt_tab_floats(p, kSimtKeys)) *
                      sizeof(float);
  if (set_smem(simt_bwd_kv_kernel<D>, smkv)) return KIA_ERR_CUDA;
  simt_bwd_kv_kernel<D><<<grid, kSimtRows, smkv, s>>>(Q, Kt, V, dO, st, wk, dK, dV, p, T);
  return launch_status();
}

template <int D>
int backward_rows(const float* Q, const float* Kt, const float* O, const float* dO,
                  const StatsView& st, const WorkView& wk, float* dQ, float* dK, float* dS_dbg,
                  int B, int H, int T, const OpParams& p, cudaStream_t s, bool prep,
                  float* dQ_zero) {
  const long long rows = (long long)B * H * T;
  const unsigned nb = (unsigned)((rows + kRowWarps - 1) / kRowWarps);
  if (prep) {
    bwd_prep_kernel<D><<<nb, 32 * kRowWarps, 0, s>>>(O, dO, st, wk, dQ_zero, p, B, H, T);
    return launch_status();
  }
  bwd_calib_kernel<D><<<nb, 32 * kRowWarps, 0, s>>>(Q, Kt, st, wk, dQ, dK, dS_dbg, p, B, H, T);
  if (launch_status()) return KIA_ERR_CUDA;
  if (!p.softmax && p.grad == KIA_GRAD_PROJECT) {
    dim3 g(B * H, D / 32, (T + kScanRows - 1) / kScanRows);
    bwd_project_scan_kernel<D><<<g, 32 * kScanWarps, 0, s>>>(Q, Kt, wk, dQ, dK, p, T, 1);
    if (launch_status()) return KIA_ERR_CUDA;
  }
  return KIA_OK;
}

template <int D>
int backward(const float* Q, const float* Kt, const float* V, const float* O, const float* dO,
             const void* stats, float* dQ, float* dK, float* dV, float* dS_dbg, int B, int H,
             int T, const OpParams& p, int gemm, void* workspace, cudaStream_t s) {
  const long long rows = (long long)B * H * T;
  StatsView st = stats_view(const_cast<void*>(stats), rows, D, p);
  WorkView wk = work_view(workspace, rows);
  if (dS_dbg) {
    if (cudaMemsetAsync(dS_dbg, 0, (size_t)rows * T * sizeof(float), s) != cudaSuccess)
      return KIA_ERR_CUDA;
  }
  const bool tc = gemm == KIA_GEMM_TF32;
  prof_mark(2, s);
  int rc;
  if (tc) {
    // query pass (checks the stats, centering, dQ with its calibration terms),
    // key pass (dK with the calibration terms folded into dS, dV)
    prof_mark(3, s);
    rc = tc_backward<D>(Q, Kt, V, O, dO, st, wk, dQ, dK, dV, dS_dbg, B, H, T, p, s, prof_mark);
    if (rc) return rc;
    if (!p.softmax && p.grad == KIA_GRAD_PROJECT) {
      // the key pass already folded the projection shift into dK
      dim3 g(B * H, D / 32, (T + kScanRows - 1) / kScanRows);
      bwd_project_scan_kernel<D><<<g, 32 * kScanWarps, 0, s>>>(Q, Kt, wk, dQ, dK, p, T, 0);
      if (launch_status()) return KIA_ERR_CUDA;
    }
    prof_mark(6, s);
    return KIA_OK;
  }
  // exact-fp32 kernels
  rc = backward_rows<D>(Q, Kt, O, dO, st, wk, dQ, dK, dS_dbg, B, H, T, p, s, true, nullptr);
  if (rc) return rc;
  prof_mark(3, s);
  OpParams q = p;
  q.tf32_ops = tc ? 1 : 0;
  rc = simt_backward<D>(Q, Kt, V, dO, st, wk, dQ, dK, dV, dS_dbg, B, H, T, q, s);
  if (rc) return rc;
  prof_mark(4, s);
  prof_mark(5, s);
  rc = backward_rows<D>(Q, Kt, O, dO, st, wk, dQ, dK, dS_dbg, B, H, T, p, s, false, nullptr);
  prof_mark(6, s);
  return rc;
}

// Scratch of kiattn_bwd_noalloc: the backward's workspace for up to
// KIA_NOALLOC_MAX_ROWS rows, declared by the library so that the caller
// allocates nothing.  Host code only ever uses its device address.  That
// address belongs to the CUDA context the module was loaded into, so it is
// looked up once per context (keyed by the driver's context id, which is
// never reused within a process): a device reset or a caller's own context
// on the same device gets its own lookup instead of a stale address.
constexpr size_t kNoallocScratchBytes = work_bytes_c(KIA_NOALLOC_MAX_ROWS);
static __device__ __align__(256) unsigned char g_kia_noalloc_scratch[kNoallocScratchBytes];
constexpr int kMaxContexts = 64;
struct NoallocSlot {
  unsigned long long ctx_id;
  void* addr;
};
NoallocSlot g_noalloc[kMaxContexts] = {};
int g_noalloc_used = 0;
int g_noalloc_next = 0;
std::mutex g_noalloc_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the calling thread's current context (the runtime's primary context
// of the current device unless the caller made another one current); 0 on
// error.  The runtime makes the primary context current on its first call
// that needs one, so a thread with none yet gets it from cudaGetSymbolAddress.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_cur || !get_id) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess)
      return 0;
    get_cur = reinterpret_cast<CtxGetCurrentFn>(a);
    get_id = reinterpret_cast<CtxGetIdFn>(b);
  }
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS) return 0;
  if (!ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kia_noalloc_scratch) != cudaSuccess) return 0;
    if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  }
  unsigned long long id = 0;
  return get_id(ctx, &id) == CUDA_SUCCESS ? id : 0;
}

// Device address of the scratch in the calling thread's current context.
void* noalloc_scratch() {
  const unsigned long long id = current_context_id();
  if (id == 0) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  for (int i = 0; i < g_noalloc_used; ++i)
    if (g_noalloc[i].ctx_id == id) return g_noalloc[i].addr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_kia_noalloc_scratch) != cudaSuccess || !p) return nullptr;
  // a process that cycles through more contexts than slots overwrites the
  // oldest slot (its context is the likeliest to be gone)
  g_noalloc[g_noalloc_next] = NoallocSlot{id, p};
  g_noalloc_next = (g_noalloc_next + 1) % kMaxContexts;
  if (g_noalloc_used < kMaxContexts) ++g_noalloc_used;
  return p;
}

}  // namespace

extern "C" {

size_t kiattn_stats_bytes(int B, int H, int T, int d, const kia_config* cfg) {
  if (check_config(cfg) || check_shape(B, H, T, d)) return 0;
  const OpParams p = make_params(cfg);
  return stats_layout((long long)B * H * T, d, p).total;
}

size_t kiattn_workspace_bytes(int B, int H, int T, int d, const kia_config* cfg) {
  if (check_config(cfg) || check_shape(B, H, T, d)) return 0;
  return work_bytes((long long)B * H * T);
}

int kiattn_fwd(const float* Q, const float* Kt, const float* V, float* O, void* stats, int B,
               int H, int T, int d, const kia_config* cfg, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_shape(B, H, T, d))) return rc;
  if (!Q || !Kt || !V || !O || !stats) return KIA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(Kt) || !aligned16(V) || !aligned16(O) || !aligned16(stats))
    return KIA_ERR_INVALID_ARG;
  const OpParams p = make_params(cfg);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  prof_mark(0, s);
  if (cfg->gemm == KIA_GEMM_FP32) {
    rc = d == 64 ? simt_forward<64>(Q, Kt, V, O, stats, B, H, T, p, s)
                 : simt_forward<128>(Q, Kt, V, O, stats, B, H, T, p, s);
  } else {
    rc = d == 64 ? tc_forward<64>(Q, Kt, V, O, stats, B, H, T, p, s)
                 : tc_forward<128>(Q, Kt, V, O, stats, B, H, T, p, s);
  }
  prof_mark(1, s);
  return rc;
}

int kiattn_bwd(const float* Q, const float* Kt, const float* V, const float* O, const float* dO,
               const void* stats, float* dQ, float* dK, float* dV, float* dS_dbg, int B, int H,
               int T, int d, const kia_config* cfg, void* workspace, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_shape(B, H, T, d))) return rc;
  if (!Q || !Kt || !V || !O || !dO || !stats || !dQ || !dK || !dV || !workspace)
    return KIA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(Kt) || !aligned16(V) || !aligned16(O) || !aligned16(dO) ||
      !aligned16(stats) || !aligned16(dQ) || !aligned16(dK) || !aligned16(dV) ||
      !aligned16(workspace) || (dS_dbg && !aligned16(dS_dbg)))
    return KIA_ERR_INVALID_ARG;
  const OpParams p = make_params(cfg);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 64 ? backward<64>(Q, Kt, V, O, dO, stats, dQ, dK, dV, dS_dbg, B, H, T, p, cfg->gemm,
                                workspace, s)
                 : backward<128>(Q, Kt, V, O, dO, stats, dQ, dK, dV, dS_dbg, B, H, T, p,
                                 cfg->gemm, workspace, s);
}

int kiattn_bwd_noalloc(const float* Q, const float* Kt, const float* V, const float* O,
                       const float* dO, const void* stats, float* dQ, float* dK, float* dV,
                       float* dS_dbg, int B, int H, int T, int d, const kia_config* cfg,
                       void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_shape(B, H, T, d))) return rc;
  const long long rows = (long long)B * H * T;
  if (rows > KIA_NOALLOC_MAX_ROWS || work_bytes(rows) > kNoallocScratchBytes)
    return KIA_ERR_CAPACITY;
  void* scratch = noalloc_scratch();
  if (!scratch) return KIA_ERR_CUDA;
  return kiattn_bwd(Q, Kt, V, O, dO, stats, dQ, dK, dV, dS_dbg, B, H, T, d, cfg, scratch,
                    stream);
}

int kiattn_weights_from_S(const float* S, int rows, int cols, const int* row_len,
                          const kia_config* cfg, float* w, int* bin, float* t, float* row_m,
                          float* row_n, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!S || !row_len || !w || rows < 1 || cols < 1) return KIA_ERR_INVALID_ARG;
  if ((long long)rows * cols > (1ll << 40)) return KIA_ERR_UNSUPPORTED;
  if (cfg->op != KIA_OP_KINTERVAL) return KIA_ERR_INVALID_ARG;
  const OpParams p = make_params(cfg);
  const unsigned nb = (unsigned)((rows + kWeightsWarps - 1) / kWeightsWarps);
  // the forward's compile-time variant of this configuration
  return dispatch_variant(p, [&]<class V>() {
    weights_from_S_kernel<V><<<nb, 32 * kWeightsWarps, 0, static_cast<cudaStream_t>(stream)>>>(
        S, rows, cols, row_len, p, w, bin, t, row_m, row_n);
    return launch_status();
  });
}

int kiattn_scores(const float* Q, const float* Kt, float* S, int B, int H, int T, int d,
                  const kia_config* cfg, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_shape(B, H, T, d))) return rc;
  if (!Q || !Kt || !S || !aligned16(Q) || !aligned16(Kt) || !aligned16(S))
    return KIA_ERR_INVALID_ARG;
  const OpParams p = make_params(cfg);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cfg->gemm == KIA_GEMM_FP32) {
    return d == 64 ? simt_scores<64>(Q, Kt, S, B, H, T, p, s)
                   : simt_scores<128>(Q, Kt, S, B, H, T, p, s);
  }
  return d == 64 ? tc_scores<64>(Q, Kt, S, B, H, T, p, s) : tc_scores<128>(Q, Kt, S, B, H, T, p, s);
}

int kiattn_grad_decomposition(const float* dS, const void* workspace, int B, int H, int T,
                              const kia_config* cfg, double* out, void* stream) {
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_shape(B, H, T, 64))) return rc;
  if (!dS || !workspace || !out) return KIA_ERR_INVALID_ARG;
  const long long rows = (long long)B * H * T;
  WorkView wk = work_view(const_cast<void*>(workspace), rows);
  const long long blocks = (rows + kRowWarps - 1) / kRowWarps;
  if (blocks > 0x7fffffffll) return KIA_ERR_UNSUPPORTED;
  grad_decomp_kernel<<<(unsigned)blocks, 32 * kRowWarps, 0, static_cast<cudaStream_t>(stream)>>>(
      dS, wk, rows, T, cfg->causal, cfg->grad, out);
  return launch_status();
}

int kiattn_geometry(const float* S, const float* Q, int B, int H, int T, int d,
                    const kia_config* cfg, float* out, void* stream) {
  static_assert(kGeoFields == KIA_GEO_FIELDS, "geometry field count");
  int rc = check_config(cfg);
  if (rc) return rc;
  if ((rc = check_shape(B, H, T, 64))) return rc;
  if (!S || !out || cfg->op != KIA_OP_KINTERVAL || (Q && (d < 1 || d > 4096)))
    return KIA_ERR_INVALID_ARG;
  const long long rows = (long long)B * H * T;
  const long long blocks = (rows + kGeoWarps - 1) / kGeoWarps;
  if (blocks > 0x7fffffffll) return KIA_ERR_UNSUPPORTED;
  const OpParams p = make_params(cfg);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dq = Q ? d : 0;
  auto launch = [&](auto var) {
    using V = decltype(var);
    if (cudaFuncSetAttribute(geometry_kernel<V>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kGeoSmemBytes) != cudaSuccess)
      return;
    geometry_kernel<V><<<(unsigned)blocks, 32 * kGeoWarps, kGeoSmemBytes, s>>>(
        S, Q, rows, T, dq, cfg->causal, p, out);
  };
  const bool lerp = p.rec == KIA_REC_LERP;
  if (p.cal == KIA_CAL_MINMAX) {
    if (lerp) launch(Var<KIA_CAL_MINMAX, KIA_REC_LERP, false, false>{});
    else launch(Var<KIA_CAL_MINMAX, KIA_REC_NEAREST, false, false>{});
  } else {
    if (lerp) launch(Var<KIA_CAL_FWM, KIA_REC_LERP, false, false>{});
    else launch(Var<KIA_CAL_FWM, KIA_REC_NEAREST, false, false>{});
  }
  return launch_status();
}

const char* kiattn_strerror(int code) {
  switch (code) {
    case KIA_OK: return "ok";
    case KIA_ERR_INVALID_ARG: return "invalid argument";
    case KIA_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case KIA_ERR_CUDA: return "CUDA launch or driver error";
    case KIA_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    case KIA_ERR_STATS_MISMATCH: return "stats buffer was written for another shape or config";
    case KIA_ERR_CAPACITY: return "size exceeds the fixed scratch capacity";
    default: return "unknown error";
  }
}

int kiattn_version(void) { return 10000; }

int kiattn_profile_enable(int on) {
  if (on && !g_prof_created) {
    for (int i = 0; i < kProfEvents; ++i)
      if (cudaEventCreate(&g_prof_ev[i]) != cudaSuccess) return KIA_ERR_CUDA;
    g_prof_created = true;
  }
  g_prof_on = on != 0;
  return KIA_OK;
}

int kiattn_profile_read(float* ms, int n) {
  if (!ms || n < 0) return KIA_ERR_INVALID_ARG;
  if (!g_prof_created) return KIA_ERR_INVALID_ARG;
  if (cudaEventSynchronize(g_prof_ev[kProfEvents - 1]) != cudaSuccess ||
      cudaEventSynchronize(g_prof_ev[1]) != cudaSuccess)
    return KIA_ERR_CUDA;
  const int pairs[5][2] = {{0, 1}, {2, 3}, {3, 4}, {4, 5}, {5, 6}};
  int w = 0;
  for (int i = 0; i < 5 && w < n; ++i, ++w) {
    float t = 0.0f;
    if (cudaEventElapsedTime(&t, g_prof_ev[pairs[i][0]], g_prof_ev[pairs[i][1]]) != cudaSuccess)
      t = -1.0f;
    ms[w] = t;
  }
  return w;
}

int kiattn_debug_bounded_wait(int what, unsigned long long wait_limit_ns) {
  if (what < 0 || what > 1) return KIA_ERR_INVALID_ARG;
  const unsigned long long lim = wait_limit_ns ? wait_limit_ns : (unsigned long long)kWaitLimitNs;
  if (cudaMemcpyToSymbol(g_kia_wait_limit_ns, &lim, sizeof(lim)) != cudaSuccess)
    return KIA_ERR_CUDA;
  g_withhold = what;
  return KIA_OK;
}

int kiattn_device_error(int reset) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_kia_device_error, sizeof(int)) != cudaSuccess) return KIA_ERR_CUDA;
  if (reset) {
    const int z = 0;
    if (cudaMemcpyToSymbol(g_kia_device_error, &z, sizeof(int)) != cudaSuccess) return KIA_ERR_CUDA;
  }
  return v;
}

}  // extern "C"
