// Device-side building blocks shared by the kiattn kernels (sm_100a):
// the fp32 weight stage of K-interval attention, our own fp64 exponential for
// the grid values, and thin inline-PTX wrappers for mbarriers, TMA and the
// tcgen05 tensor-core / tensor-memory instructions.
//
// Operator reference: "Pretraining Transformers with Quantized Softmax in
// Attention", section 3 (Calibration, Reconstruction) and Appendix A.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kiattn.h"

#define KIA_MAX_K 64
// fixed-step grids: at most this many intervals before G_k underflows
#define KIA_MAX_KCAP 400
#define KIA_TILE 128

namespace kia {

// ----------------------------------------------------------------- config

struct OpParams {
  int K;          // number of intervals
  float Kf;       // (float)K
  int cal;        // KIA_CAL_*
  int rec;        // KIA_REC_*
  int ste;        // KIA_STE_*
  int grad;       // KIA_GRAD_*
  int causal;
  int softmax;    // exact softmax attention instead of K-interval
  float tau;
  float fwm_h;    // tau / K  (fp32 division)
  float fwm_rh;   // K / tau  (fp32 division)
  int tf32_ops;   // CUDA-core kernels: truncate product operands to TF32 like tcgen05
  int fixed_step; // untruncated fixed step (Appendix D.4), run as FWM with K = the grid's
                  // extent, the first node count at which G_k underflows to zero in fp32
  int exp_round;  // softmax only: 0 exact e^{s-m}; 1 rounded to bf16; 2 rounded to FP8 E4M3
  int withhold;   // failure-handling test hook (forward only): 1 = the first CTA never
                  // issues the first Q tile, so the waits on it run out; 0 normally
};

// Reduced-precision exponential baselines (Appendix D.5): the softmax
// numerator e^{s-m} (fp32) rounded to bfloat16 (R = 1) or to FP8 E4M3 (R =
// 2), both to nearest, ties to even; R = 0 leaves it exact.
template <int R>
__device__ __forceinline__ float round_exp(float e) {
  if constexpr (R == 1) {
    return __bfloat162float(__float2bfloat16_rn(e));
  } else if constexpr (R == 2) {
    const __nv_fp8_storage_t q = __nv_cvt_float_to_fp8(e, __NV_SATFINITE, __NV_E4M3);
    return __half2float(__half(__nv_cvt_fp8_to_halfraw(q, __NV_E4M3)));
  } else {
    return e;
  }
}
__device__ __forceinline__ float round_exp_rt(float e, int mode) {
  return mode == 1 ? round_exp<1>(e) : (mode == 2 ? round_exp<2>(e) : e);
}

// The tcgen05 kind::tf32 MMA reads fp32 operands and ignores their low 13
// mantissa bits; CUDA-core kernels standing in for it apply the same mask.
__device__ __forceinline__ float tf32_trunc(float x) {
  return __uint_as_float(__float_as_uint(x) & 0xffffe000u);
}

// Forward probabilities are the LERP weights for LERP, the hard weights for
// Nearest (both surrogates).  The backward's normalisation point is the LERP
// point for LERP and Prob-STE and the hard point for Weight-STE (Appendix B).
__host__ __device__ inline bool lerp_forward(const OpParams& p) { return p.rec == KIA_REC_LERP; }
__host__ __device__ inline bool lerp_normpoint(const OpParams& p) {
  return p.rec == KIA_REC_LERP || p.ste == KIA_STE_PROB;
}
__host__ __device__ inline bool needs_OL(const OpParams& p) {
  return !p.softmax && p.rec == KIA_REC_NEAREST && p.ste == KIA_STE_PROB;
}

// ------------------------------------------------- fp64 exponential, x <= 0
// Cody & Waite argument reduction x = n ln2 + r (ln 2 split into a 32-bit
// head, so that n * head is exact for |n| < 2^21, and a tail), Taylor series
// of e^r through r^13/13! in Horner form (truncation below 1e-17 for
// |r| <= ln2/2), exact scaling by 2^n.  Every step is an explicit IEEE
// round-to-nearest operation, so the result is a fixed function of x.
// Values below 2^-150 round to zero in fp32 and are returned as 0.
__device__ __forceinline__ double grid_exp(double x) {
  if (x < -104.5) return 0.0;
  if (x == 0.0) return 1.0;
  const double kInvLn2 = 1.4426950408889634;
  const double kLn2Hi = 0.693147180369123816490;     // 0x1.62e42fee00000p-1
  const double kLn2Lo = 1.90821492927058770002e-10;  // ln 2 - kLn2Hi
  const double n = rint(__dmul_rn(x, kInvLn2));
  const double r = __dsub_rn(__dsub_rn(x, __dmul_rn(n, kLn2Hi)), __dmul_rn(n, kLn2Lo));
  double p = 1.0 / 6227020800.0;
  p = __fma_rn(p, r, 1.0 / 479001600.0);
  p = __fma_rn(p, r, 1.0 / 39916800.0);
  p = __fma_rn(p, r, 1.0 / 3628800.0);
  p = __fma_rn(p, r, 1.0 / 362880.0);
  p = __fma_rn(p, r, 1.0 / 40320.0);
  p = __fma_rn(p, r, 1.0 / 5040.0);
  p = __fma_rn(p, r, 1.0 / 720.0);
  p = __fma_rn(p, r, 1.0 / 120.0);
  p = __fma_rn(p, r, 1.0 / 24.0);
  p = __fma_rn(p, r, 1.0 / 6.0);
  p = __fma_rn(p, r, 0.5);
  p = __fma_rn(p, r, 1.0);
  p = __fma_rn(p, r, 1.0);
  const long long e = (long long)((int)n + 1023) << 52;
  return __dmul_rn(p, __longlong_as_double(e));
}

// G_k = RN32(e^{-k h}) for the fp32 width h.
__device__ __forceinline__ float grid_value(int k, float h) {
  return __double2float_rn(grid_exp(__dmul_rn(-(double)k, (double)h)));
}

// ------------------------------------------------------ row calibration
// Per-row constants of section 3 (Calibration), in the fixed fp32 sequence
// that the bit-exact weight-stage check pins: span = m - n, h = span / K,
// rh = K / span (MinMax), or h = tau / K, rh = K / tau (FWM).  A MinMax row
// whose span is below 1e-12 takes the degenerate branch of Appendix A; it is
// marked by h = 0.
struct RowCal {
  float m;
  float rh;
  float h;
};

__device__ __forceinline__ RowCal row_calibration(const OpParams& p, float m, float n) {
  RowCal c;
  c.m = m;
  if (p.cal == KIA_CAL_MINMAX) {
    const float span = __fsub_rn(m, n);
    if (span < 1e-12f) {
      c.h = 0.0f;
      c.rh = 0.0f;
    } else {
      c.h = __fdiv_rn(span, p.Kf);
      c.rh = __fdiv_rn(p.Kf, span);
    }
  } else {
    c.h = p.fwm_h;
    c.rh = p.fwm_rh;
  }
  return c;
}

// ------------------------------------------------------- element stage
// Position of score s on the grid (section 3, Reconstruction): u = (m - s) *
// rh; MinMax clamps u to K, FWM marks u > K as tail; k = min(floor u, K-1);
// t = u - k (exact in fp32).
struct GridPos {
  float u;
  float t;
  int k;
  bool tail;
};

__device__ __forceinline__ GridPos grid_position(const OpParams& p, const RowCal& c, float s) {
  GridPos g;
  float u = __fmul_rn(__fsub_rn(c.m, s), c.rh);
  g.tail = false;
  if (p.cal == KIA_CAL_MINMAX) {
    u = fminf(u, p.Kf);
  } else {
    g.tail = u > p.Kf;
  }
  int k = (int)floorf(u);
  k = k > p.K - 1 ? p.K - 1 : k;
  // u >= 0 whenever s is the score the row max came from; a score
  // recomputed by a different contraction order can exceed m by an ulp
  k = k < 0 ? 0 : k;
  g.k = k;
  g.u = u;
  g.t = __fsub_rn(u, (float)k);
  return g;
}

// LERP weight w = G_k + t a_k with a_k = G_{k+1} - G_k (one fp32 FMA).
__device__ __forceinline__ float lerp_weight(float t, float Gk, float Gk1) {
  return __fmaf_rn(t, __fsub_rn(Gk1, Gk), Gk);
}
// Nearest node r = k + [t >= 1/2].
__device__ __forceinline__ int nearest_node(const GridPos& g) { return g.k + (g.t >= 0.5f ? 1 : 0); }

// ------------------------------------------------------------- PTX: misc

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .b32 r;\n\t.reg .pred p;\n\t"
      "elect.sync r|p, 0xffffffff;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred;
}

// ------------------------------------------------------------ mbarriers

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of a phase (true once the phase of this parity is over).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait.  Gives up after ~g_kia_wait_limit_ns or as soon as another
// thread of the CTA has raised *abort; on giving up it raises *abort and the
// library-wide error word, and returns false.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Library-wide device error word (the library is a single translation unit).
__device__ int g_kia_device_error;
// Limit of every bounded wait; the failure-handling test hook shortens it.
__device__ unsigned long long g_kia_wait_limit_ns = kWaitLimitNs;

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes (or about hint_ns pass) instead of polling shared memory,
// which would take shared-memory bandwidth from the tensor core's operands.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
constexpr uint32_t kSuspendHintNs = 1000000u;     // 1 ms per sleep, then re-check abort

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait_sleep(bar, parity, kSuspendHintNs)) return true;
    // the abort flag and the time limit (a global load) only every 16th
    // pass, so that nothing slow sits between two probes of the barrier
    if ((n & 15u) == 0u) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > g_kia_wait_limit_ns) {
        *abort = 1;
        atomicExch(&g_kia_device_error, KIA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Bounded wait by a whole warp (an MMA-issuing warp runs its loop converged
// and elects one lane only to issue): every lane waits on the same phase and
// the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

// Watchdog of a polling loop that serves several barriers: call idle() on
// every pass that made no progress and progress() on every pass that did.
// Gives up like mbar_wait: after ~g_kia_wait_limit_ns without progress, or at
// once when *abort is raised.
struct PollGuard {
  uint64_t t0;
  uint32_t idle_passes;
  __device__ __forceinline__ PollGuard() : t0(global_timer_ns()), idle_passes(0) {}
  __device__ __forceinline__ void progress() { idle_passes = 0; }
  __device__ __forceinline__ bool idle(volatile int* abort) {
    if (idle_passes == 0) t0 = global_timer_ns();
    __nanosleep(100);   // back off instead of hammering shared memory
    if ((++idle_passes & 15u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > g_kia_wait_limit_ns) {
        *abort = 1;
        atomicExch(&g_kia_device_error, KIA_ERR_TIMEOUT);
        return false;
      }
    }
    return true;
  }
};

// A persistent CTA's work items: round r of gridDim.x items gives CTA c the
// item r * G + c in even rounds and r * G + (G - 1 - c) in odd ones.  Items
// are numbered heaviest first, so the serpentine order evens out the sums.
struct ItemSeq {
  int r, n;
  __device__ __forceinline__ explicit ItemSeq(int nitems) : r(-1), n(nitems) {}
  // the next item of this CTA, or -1 when there is none
  __device__ __forceinline__ int next() {
    const int G = (int)gridDim.x;
    for (;;) {
      ++r;
      if ((long long)r * G >= n) return -1;
      const int c = (r & 1) ? G - 1 - (int)blockIdx.x : (int)blockIdx.x;
      const int it = r * G + c;
      if (it < n) return it;
    }
  }
};

// After an abort: let copies and MMAs already in flight land before the CTA
// releases its shared and tensor memory (bounded: ~200 us).
__device__ __forceinline__ void drain_in_flight() {
  const uint64_t t0 = global_timer_ns();
  while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 3-D tiled load (no multicast): box at (x, y, z) of the tensor map into
// shared memory, completion counted on bar in bytes.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Four-byte asynchronous copy global -> shared (no register staging); the
// copies of a thread are waited for with cp_async_wait_all().
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
               : "memory");
}
// Sixteen-byte asynchronous copy global -> shared (both addresses 16-byte
// aligned), cached in L2 only.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Bring the 128-byte line holding addr into L2 (no register result).
__device__ __forceinline__ void prefetch_l2(const void* addr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(addr));
}

// 3-D tiled store: the box at (x, y, z) of the tensor map from shared
// memory (rows outside the tensor are not written), as one bulk group.
__device__ __forceinline__ void tma_store_3d(const void* tmap, const void* src, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_store_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every committed bulk store of this thread has completed.
__device__ __forceinline__ void tma_store_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Wait until every committed bulk store of this thread has finished reading
// its shared-memory source (the buffer may then be rewritten).
__device__ __forceinline__ void tma_store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Make this thread's generic-proxy shared-memory writes visible to the
// async proxy (TMA) before a barrier.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// --------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on bar once every tcgen05 op issued so far by this thread is done.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc], kind::tf32.
__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc], kind::tf32.
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor for kind::tf32 with fp32 accumulation (bit layout of
// the tcgen05 instruction descriptor: c_format [4,6), a_format [7,10),
// b_format [10,13), a_major bit 15, b_major bit 16, N>>3 at [17,23),
// M>>4 at [24,29)).
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)a_mn_major << 15) |
         ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory matrix descriptor (sm_100, descriptor version 1, base offset
// 0: tiles are 1024-byte aligned).  Layout type 2 = 128-byte swizzle with
// 16-byte atoms (K-major operands), 1 = 128-byte swizzle with 32-byte atoms
// (the only layout for MN-major 32-bit operands).  lbo / sbo in bytes.
constexpr uint32_t kLayoutSW128 = 2;
constexpr uint32_t kLayoutSW128Atom32 = 1;

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)layout << 61;
  return d;
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane
// (warp quadrant * 32 + i), columns col..col+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Wait for this thread's TMEM loads and tie the destination registers to the
// wait, so that no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_ld_wait_regs(float (&v)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                 "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_ld_wait_regs(float (&v)[16], float (&w)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                 "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), "+f"(w[0]), "+f"(w[1]),
                 "+f"(w[2]), "+f"(w[3]), "+f"(w[4]), "+f"(w[5]), "+f"(w[6]), "+f"(w[7]),
                 "+f"(w[8]), "+f"(w[9]), "+f"(w[10]), "+f"(w[11]), "+f"(w[12]), "+f"(w[13]),
                 "+f"(w[14]), "+f"(w[15])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_ld_wait_regs(float (&v)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                 "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), "+f"(v[16]), "+f"(v[17]),
                 "+f"(v[18]), "+f"(v[19]), "+f"(v[20]), "+f"(v[21]), "+f"(v[22]), "+f"(v[23]),
                 "+f"(v[24]), "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]),
                 "+f"(v[30]), "+f"(v[31])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// One column of the warp's 32 TMEM lanes: read (waiting for it), and write.
__device__ __forceinline__ float tmem_ld1_sync(uint32_t taddr) {
  uint32_t x;
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(x)
      : "r"(taddr)
      : "memory");
  return __uint_as_float(x);
}
__device__ __forceinline__ void tmem_st1(uint32_t taddr, float v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr),
               "r"(__float_as_uint(v))
               : "memory");
}

// Named barrier among `count` threads (multiple of 32), id 1..15.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace kia
