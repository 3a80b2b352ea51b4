// Tensor-core backward of K-interval attention (sm_100a), d = 64, as two
// kernels that both recompute the scores and dP = dO V^T:
//
//  query pass (one CTA per (batch*head, 128-query tile); thread = query row):
//    S = Q_i K_j^T, dP = dO_i V_j^T                (tcgen05 kind::tf32, TMEM)
//    dw = (dP - D) / W_bar                         (normalisation Jacobian at
//                                                   the surrogate's point)
//    dS = dw * ds-slope (LERP -a_k/h; softmax w; degenerate 1; FWM tail 0)
//    row sums A = sum dw a_k, C = sum dw (b - a_k u/h) in registers
//    dQ_i += dS K_j                                (A operand from TMEM)
//  key pass (one CTA per (batch*head, 128-key tile); thread = key row):
//    S^T, dP^T recomputed; P = w_fwd / W_fwd; dS^T as above
//    dV_j += P^T dO_i,  dK_j += dS^T Q_i          (A operands from TMEM)
//
// Each output row is owned by one CTA and written once: no atomics.  The
// calibration terms (section 3, Calibration gradients; Appendix B) are
// added afterwards from A and C by the row passes in kia_epilogue.cuh.
// Warp roles (6 warps): 0 = TMA producer, 1 = MMA issuer and TMEM owner,
// 2..5 = element warps (thread r owns TMEM lane r).
#pragma once
#include "kia_tc.cuh"

namespace kia {

constexpr int kBwdThreads = 192;
constexpr int kBwdSmemTabK = 32;  // key pass: per-query grids up to K = 32 in shared memory

// Per-query constants of one query tile in the key pass, struct of arrays.
enum { QC_M = 0, QC_RH, QC_RWB, QC_RWF, QC_D, QC_L, QC_COUNT };

struct BwdQBars {
  uint64_t qd_full;               // Q_i, dO_i (K-major), once
  uint64_t kv_full, kv_empty;     // K_j, V_j K-major (for S, dP)
  uint64_t kmn_full, kmn_empty;   // K_j MN-major (for dQ)
  uint64_t sp_full;               // S and dP in TMEM
  uint64_t elem_done;             // dS written into the S columns (128 arrivals)
  uint64_t st_free;               // dQ MMA of the step done (S columns free)
  uint64_t dq_full;               // all dQ MMAs done
  uint32_t tmem_base;
  int abort;
};

struct BwdKBars {
  uint64_t kv_full;               // K_j, V_j K-major, once
  uint64_t qd_full, qd_empty;     // Q_i, dO_i K-major (for S^T, dP^T)
  uint64_t mn_full, mn_empty;     // Q_i, dO_i MN-major (for dK, dV)
  uint64_t sp_full;               // S^T and dP^T in TMEM
  uint64_t qc_ready;              // per-query constants of the step loaded (128 arrivals)
  uint64_t elem_done;             // P^T, dS^T written (128 arrivals)
  uint64_t st_free;               // dV, dK MMAs of the step done
  uint64_t acc_full;              // all dV, dK MMAs done
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float* smem_f(uint8_t* base, uint32_t off) {
  return reinterpret_cast<float*>(base + off);
}

// ---------------------------------------------------------------- query pass

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
tc_bwd_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKmn,
                const __grid_constant__ CUtensorMap tmV, StatsView st, WorkView wk,
                float* __restrict__ dQ, float* __restrict__ dS_dbg, OpParams p, int T) {
  static_assert(D == 64, "tensor-core backward tiles are laid out for d = 64");
  constexpr uint32_t kTile = D * KIA_TILE * 4;
  if (*wk.status != 0) return;
  extern __shared__ uint8_t smraw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
  float* sQ = smem_f(base, 0);
  float* sG = smem_f(base, kTile);
  float* sK = smem_f(base, 2 * kTile);
  float* sKmn = smem_f(base, 3 * kTile);
  float* sV = smem_f(base, 4 * kTile);
  float* sTab = smem_f(base, 5 * kTile);
  const bool minmax_tab = !p.softmax && p.cal == KIA_CAL_MINMAX;
  const int tab_floats = p.softmax ? 0 : (minmax_tab ? (p.K + 1) * KIA_TILE : (p.K + 1));
  BwdQBars& bar = *reinterpret_cast<BwdQBars*>(sTab + ((tab_floats + 31) & ~31));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int qt = nt - 1 - blockIdx.y;
  const int nkt = p.causal ? qt + 1 : nt;
  constexpr uint32_t kColS = 0, kColP = 128, kColDQ = 256;

  if (threadIdx.x == 0) {
    mbar_init(&bar.qd_full, 1);
    mbar_init(&bar.kv_full, 1);
    mbar_init(&bar.kv_empty, 1);
    mbar_init(&bar.kmn_full, 1);
    mbar_init(&bar.kmn_empty, 1);
    mbar_init(&bar.sp_full, 1);
    mbar_init(&bar.elem_done, 128);
    mbar_init(&bar.st_free, 1);
    mbar_init(&bar.dq_full, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  volatile int* abort = &bar.abort;
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmG);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmKmn);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar.qd_full, 2 * kTile);
      for (int b = 0; b < D / 32; ++b) {
        tma_load_3d(sQ + b * 32 * KIA_TILE, &tmQ, &bar.qd_full, b * 32, qt * KIA_TILE, bh);
        tma_load_3d(sG + b * 32 * KIA_TILE, &tmG, &bar.qd_full, b * 32, qt * KIA_TILE, bh);
      }
      for (int j = 0; j < nkt; ++j) {
        if (!mbar_wait(&bar.kv_empty, (j & 1) ^ 1, abort)) { failed = true; break; }
        mbar_arrive_expect_tx(&bar.kv_full, 2 * kTile);
        for (int b = 0; b < D / 32; ++b) {
          tma_load_3d(sK + b * 32 * KIA_TILE, &tmK, &bar.kv_full, b * 32, j * KIA_TILE, bh);
          tma_load_3d(sV + b * 32 * KIA_TILE, &tmV, &bar.kv_full, b * 32, j * KIA_TILE, bh);
        }
        if (!mbar_wait(&bar.kmn_empty, (j & 1) ^ 1, abort)) { failed = true; break; }
        mbar_arrive_expect_tx(&bar.kmn_full, kTile);
        for (int b = 0; b < D / 32; ++b)
          tma_load_3d(sKmn + b * 32 * KIA_TILE, &tmKmn, &bar.kmn_full, b * 32, j * KIA_TILE, bh);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_tf32(128, 128, 0, 0);
      const uint32_t id_dq = idesc_tf32(128, D, 0, 1);
      const uint32_t qa = smem_u32(sQ), ga = smem_u32(sG), ka = smem_u32(sK),
                     kma = smem_u32(sKmn), va = smem_u32(sV);
      failed = !mbar_wait(&bar.qd_full, 0, abort);
      for (int j = 0; j < nkt && !failed; ++j) {
        if (!mbar_wait(&bar.kv_full, j & 1, abort)) { failed = true; break; }
        if (j > 0 && !mbar_wait(&bar.st_free, (j - 1) & 1, abort)) { failed = true; break; }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks)
          mma_tf32_ss(tmem + kColS, desc_kmajor(qa, ks), desc_kmajor(ka, ks), id_s, ks > 0);
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks)
          mma_tf32_ss(tmem + kColP, desc_kmajor(ga, ks), desc_kmajor(va, ks), id_s, ks > 0);
        tc_commit(&bar.sp_full);
        tc_commit(&bar.kv_empty);
        if (!mbar_wait(&bar.elem_done, j & 1, abort)) { failed = true; break; }
        if (!mbar_wait(&bar.kmn_full, j & 1, abort)) { failed = true; break; }
        tc_fence_after();
        // dQ_i += dS K_j  (contraction over the 128 keys of the tile)
#pragma unroll
        for (int ks = 0; ks < KIA_TILE / 8; ++ks)
          mma_tf32_ts(tmem + kColDQ, tmem + kColS + 8u * ks, desc_mnmajor(kma, ks), id_dq,
                      (j > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&bar.st_free);
        tc_commit(&bar.kmn_empty);
      }
      if (!failed) tc_commit(&bar.dq_full);
    }
  } else {
    // ------------------------------------------------------ element warps
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int q = qt * KIA_TILE + r;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const long long rowbase = (long long)bh * T;
    const long long qr = rowbase + (q < T ? q : T - 1);
    // this row's calibration and centering (written by the forward and prep)
    RowState rs;
    rs.cal.m = st.m[qr];
    rs.cal.rh = st.rh[qr];
    rs.cal.h = st.h[qr];
    rs.degen = minmax_tab && rs.cal.h == 0.0f;
    const float rWb = __fdiv_rn(1.0f, st.Wb[qr]);
    const float Dc = wk.D[qr];
    const int L = p.causal ? q + 1 : T;
    const int ts = minmax_tab ? KIA_TILE : 1;
    const float* tab = minmax_tab ? sTab + r : sTab;
    if (!p.softmax) {
      if (minmax_tab) {
        for (int k = 0; k <= p.K; ++k) sTab[k * KIA_TILE + r] = st.table[qr * (p.K + 1) + k];
      } else if (r <= p.K) {
        sTab[r] = st.table[r];
      }
    }
    named_bar_sync(1, 128);
    float A = 0.0f, C = 0.0f;
    float v[32], g[32];
    for (int j = 0; j < nkt && !failed; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.sp_full, j & 1, abort))) { failed = true; break; }
      tc_fence_after();
      const bool edge = (p.causal && j == qt) || (j + 1) * KIA_TILE > T;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(tmem + lane_addr + kColS + 32u * c, v);
        tmem_ld32(tmem + lane_addr + kColP + 32u * c, g);
        tmem_ld_wait();
        const int key0 = j * KIA_TILE + c * 32;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int key = key0 + i;
          const bool ok = !edge || (key < T && (!p.causal || key <= q));
          const ElemFwd e = elem_forward(p, rs, tab, ts, v[i]);
          // a one-key row has P = 1 whatever its score: zero gradient
          const float dw = (!ok || L == 1) ? 0.0f : (g[i] - Dc) * rWb;
          const float delta = ok ? elem_backward(p, rs, tab, ts, v[i], e.wf, dw, A, C) : 0.0f;
          v[i] = delta;
        }
        tmem_st32(tmem + lane_addr + kColS + 32u * c, v);
        if (dS_dbg && q < T) {
          float* dst = dS_dbg + (rowbase + q) * T + key0;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (key0 + i < T) dst[i] = v[i];
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar.elem_done);
    }
    if (!failed && __all_sync(0xffffffffu, mbar_wait(&bar.dq_full, 0, abort))) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(tmem + lane_addr + kColDQ + 32u * c, v);
        tmem_ld_wait();
        if (q < T) {
          float4* o4 = reinterpret_cast<float4*>(dQ + (rowbase + q) * D + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            o4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
      if (q < T) {
        wk.A[rowbase + q] = A;
        wk.C[rowbase + q] = C;
      }
    } else {
      failed = true;
    }
  }
  if (failed || *abort) drain_in_flight();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ key pass

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
tc_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQmn,
                 const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmGmn,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 StatsView st, WorkView wk, float* __restrict__ dK, float* __restrict__ dV,
                 OpParams p, int T) {
  static_assert(D == 64, "tensor-core backward tiles are laid out for d = 64");
  constexpr uint32_t kTile = D * KIA_TILE * 4;
  if (*wk.status != 0) return;
  extern __shared__ uint8_t smraw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
  float* sK = smem_f(base, 0);
  float* sV = smem_f(base, kTile);
  float* sQ = smem_f(base, 2 * kTile);
  float* sG = smem_f(base, 3 * kTile);
  float* sQmn = smem_f(base, 4 * kTile);
  float* sGmn = smem_f(base, 5 * kTile);
  float* sC = smem_f(base, 6 * kTile);                  // [QC_COUNT][128]
  float* sTab = sC + QC_COUNT * KIA_TILE;
  const bool minmax_tab = !p.softmax && p.cal == KIA_CAL_MINMAX;
  const bool tab_in_smem = !minmax_tab || p.K <= kBwdSmemTabK;
  const int K1 = p.K + 1;
  const int tab_floats = p.softmax ? 0 : (minmax_tab ? (tab_in_smem ? K1 * KIA_TILE : 0) : K1);
  BwdKBars& bar = *reinterpret_cast<BwdKBars*>(sTab + ((tab_floats + 31) & ~31));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int kt = blockIdx.y;
  const int q0 = p.causal ? kt : 0;
  const int nsteps = nt - q0;
  constexpr uint32_t kColS = 0, kColP = 128, kColDV = 256, kColDK = 256 + D;

  if (threadIdx.x == 0) {
    mbar_init(&bar.kv_full, 1);
    mbar_init(&bar.qd_full, 1);
    mbar_init(&bar.qd_empty, 1);
    mbar_init(&bar.mn_full, 1);
    mbar_init(&bar.mn_empty, 1);
    mbar_init(&bar.sp_full, 1);
    mbar_init(&bar.qc_ready, 128);
    mbar_init(&bar.elem_done, 128);
    mbar_init(&bar.st_free, 1);
    mbar_init(&bar.acc_full, 1);
    bar.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  volatile int* abort = &bar.abort;
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmQmn);
      tma_prefetch_desc(&tmG);
      tma_prefetch_desc(&tmGmn);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar.kv_full, 2 * kTile);
      for (int b = 0; b < D / 32; ++b) {
        tma_load_3d(sK + b * 32 * KIA_TILE, &tmK, &bar.kv_full, b * 32, kt * KIA_TILE, bh);
        tma_load_3d(sV + b * 32 * KIA_TILE, &tmV, &bar.kv_full, b * 32, kt * KIA_TILE, bh);
      }
      for (int s = 0; s < nsteps; ++s) {
        const int qi = q0 + s;
        if (!mbar_wait(&bar.qd_empty, (s & 1) ^ 1, abort)) { failed = true; break; }
        mbar_arrive_expect_tx(&bar.qd_full, 2 * kTile);
        for (int b = 0; b < D / 32; ++b) {
          tma_load_3d(sQ + b * 32 * KIA_TILE, &tmQ, &bar.qd_full, b * 32, qi * KIA_TILE, bh);
          tma_load_3d(sG + b * 32 * KIA_TILE, &tmG, &bar.qd_full, b * 32, qi * KIA_TILE, bh);
        }
        if (!mbar_wait(&bar.mn_empty, (s & 1) ^ 1, abort)) { failed = true; break; }
        mbar_arrive_expect_tx(&bar.mn_full, 2 * kTile);
        for (int b = 0; b < D / 32; ++b) {
          tma_load_3d(sQmn + b * 32 * KIA_TILE, &tmQmn, &bar.mn_full, b * 32, qi * KIA_TILE, bh);
          tma_load_3d(sGmn + b * 32 * KIA_TILE, &tmGmn, &bar.mn_full, b * 32, qi * KIA_TILE, bh);
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_tf32(128, 128, 0, 0);
      const uint32_t id_acc = idesc_tf32(128, D, 0, 1);
      const uint32_t ka = smem_u32(sK), va = smem_u32(sV), qa = smem_u32(sQ), ga = smem_u32(sG),
                     qma = smem_u32(sQmn), gma = smem_u32(sGmn);
      failed = !mbar_wait(&bar.kv_full, 0, abort);
      for (int s = 0; s < nsteps && !failed; ++s) {
        if (!mbar_wait(&bar.qd_full, s & 1, abort)) { failed = true; break; }
        if (s > 0 && !mbar_wait(&bar.st_free, (s - 1) & 1, abort)) { failed = true; break; }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks)
          mma_tf32_ss(tmem + kColS, desc_kmajor(ka, ks), desc_kmajor(qa, ks), id_s, ks > 0);
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks)
          mma_tf32_ss(tmem + kColP, desc_kmajor(va, ks), desc_kmajor(ga, ks), id_s, ks > 0);
        tc_commit(&bar.sp_full);
        tc_commit(&bar.qd_empty);
        if (!mbar_wait(&bar.elem_done, s & 1, abort)) { failed = true; break; }
        if (!mbar_wait(&bar.mn_full, s & 1, abort)) { failed = true; break; }
        tc_fence_after();
        // dV_j += P^T dO_i, dK_j += dS^T Q_i  (contraction over the 128 queries)
#pragma unroll
        for (int ks = 0; ks < KIA_TILE / 8; ++ks)
          mma_tf32_ts(tmem + kColDV, tmem + kColS + 8u * ks, desc_mnmajor(gma, ks), id_acc,
                      (s > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
        for (int ks = 0; ks < KIA_TILE / 8; ++ks)
          mma_tf32_ts(tmem + kColDK, tmem + kColP + 8u * ks, desc_mnmajor(qma, ks), id_acc,
                      (s > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&bar.st_free);
        tc_commit(&bar.mn_empty);
      }
      if (!failed) tc_commit(&bar.acc_full);
    }
  } else {
    // ------------------------------------------------------ element warps
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int kj = kt * KIA_TILE + r;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const long long rowbase = (long long)bh * T;
    if (!p.softmax && !minmax_tab && r < K1) sTab[r] = st.table[r];
    float v[32], g[32];
    for (int s = 0; s < nsteps && !failed; ++s) {
      const int qi = q0 + s;
      // per-query constants of this tile: thread r loads query r (every
      // reader of the previous step's constants is past elem_done, waited
      // at the end of that step)
      {
        const int q = qi * KIA_TILE + r;
        const long long qr = rowbase + (q < T ? q : T - 1);
        sC[QC_M * KIA_TILE + r] = st.m[qr];
        sC[QC_RH * KIA_TILE + r] = st.rh[qr];
        sC[QC_RWB * KIA_TILE + r] = __fdiv_rn(1.0f, st.Wb[qr]);
        sC[QC_RWF * KIA_TILE + r] = __fdiv_rn(1.0f, st.Wf[qr]);
        sC[QC_D * KIA_TILE + r] = wk.D[qr];
        sC[QC_L * KIA_TILE + r] = (float)(p.causal ? q + 1 : T);
        if (minmax_tab && tab_in_smem)
          for (int k = 0; k < K1; ++k) sTab[r * K1 + k] = st.table[qr * K1 + k];
      }
      mbar_arrive(&bar.qc_ready);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.qc_ready, s & 1, abort))) { failed = true; break; }
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.sp_full, s & 1, abort))) { failed = true; break; }
      tc_fence_after();
      const bool edge =
          (p.causal && qi == kt) || (qi + 1) * KIA_TILE > T || (kt + 1) * KIA_TILE > T;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        tmem_ld32(tmem + lane_addr + kColS + 32u * c, v);
        tmem_ld32(tmem + lane_addr + kColP + 32u * c, g);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int ql = c * 32 + i;
          const int q = qi * KIA_TILE + ql;
          const bool ok = !edge || (kj < T && q < T && (!p.causal || kj <= q));
          RowState rs;
          rs.cal.m = sC[QC_M * KIA_TILE + ql];
          rs.cal.rh = sC[QC_RH * KIA_TILE + ql];
          rs.cal.h = 1.0f;
          rs.degen = minmax_tab && rs.cal.rh == 0.0f;
          const float* tab =
              minmax_tab
                  ? (tab_in_smem ? sTab + ql * K1 : st.table + (rowbase + (q < T ? q : 0)) * K1)
                  : sTab;
          const ElemFwd e = elem_forward(p, rs, tab, 1, v[i]);
          const float dw = (!ok || sC[QC_L * KIA_TILE + ql] == 1.0f)
                               ? 0.0f
                               : (g[i] - sC[QC_D * KIA_TILE + ql]) * sC[QC_RWB * KIA_TILE + ql];
          float A = 0.0f, C = 0.0f;
          const float delta = ok ? elem_backward(p, rs, tab, 1, v[i], e.wf, dw, A, C) : 0.0f;
          v[i] = ok ? e.wf * sC[QC_RWF * KIA_TILE + ql] : 0.0f;  // P^T
          g[i] = delta;                                         // dS^T
        }
        tmem_st32(tmem + lane_addr + kColS + 32u * c, v);
        tmem_st32(tmem + lane_addr + kColP + 32u * c, g);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar.elem_done);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.elem_done, s & 1, abort))) { failed = true; break; }
    }
    if (!failed && __all_sync(0xffffffffu, mbar_wait(&bar.acc_full, 0, abort))) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(tmem + lane_addr + kColDV + 32u * c, v);
        tmem_ld32(tmem + lane_addr + kColDK + 32u * c, g);
        tmem_ld_wait();
        if (kj < T) {
          float4* dv4 = reinterpret_cast<float4*>(dV + (rowbase + kj) * D + c * 32);
          float4* dk4 = reinterpret_cast<float4*>(dK + (rowbase + kj) * D + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            dv4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            dk4[i] = make_float4(g[4 * i], g[4 * i + 1], g[4 * i + 2], g[4 * i + 3]);
          }
        }
      }
    } else {
      failed = true;
    }
  }
  if (failed || *abort) drain_in_flight();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D>
size_t tc_bwd_q_smem(const OpParams& p) {
  const bool minmax_tab = !p.softmax && p.cal == KIA_CAL_MINMAX;
  const int tab = p.softmax ? 0 : (minmax_tab ? (p.K + 1) * KIA_TILE : (p.K + 1));
  return 1024 + 5 * (size_t)D * KIA_TILE * 4 + (size_t)((tab + 31) & ~31) * 4 + sizeof(BwdQBars);
}

template <int D>
size_t tc_bwd_kv_smem(const OpParams& p) {
  const bool minmax_tab = !p.softmax && p.cal == KIA_CAL_MINMAX;
  const bool tab_in_smem = !minmax_tab || p.K <= kBwdSmemTabK;
  const int tab =
      p.softmax ? 0 : (minmax_tab ? (tab_in_smem ? (p.K + 1) * KIA_TILE : 0) : (p.K + 1));
  return 1024 + 6 * (size_t)D * KIA_TILE * 4 + QC_COUNT * KIA_TILE * 4 +
         (size_t)((tab + 31) & ~31) * 4 + sizeof(BwdKBars);
}

template <int D>
int tc_backward(const float* Q, const float* Kt, const float* V, const float* dO,
                const StatsView& st, const WorkView& wk, float* dQ, float* dK, float* dV,
                float* dS_dbg, int B, int H, int T, const OpParams& p, cudaStream_t s,
                void (*mark)(int, cudaStream_t)) {
  if constexpr (D != 64) {
    return KIA_ERR_UNSUPPORTED;
  } else {
    const int BH = B * H;
    CUtensorMap tq, tqm, tg, tgm, tk, tkm, tv;
    if (!make_tmap(&tq, Q, BH, T, D) || !make_tmap(&tqm, Q, BH, T, D, true) ||
        !make_tmap(&tg, dO, BH, T, D) || !make_tmap(&tgm, dO, BH, T, D, true) ||
        !make_tmap(&tk, Kt, BH, T, D) || !make_tmap(&tkm, Kt, BH, T, D, true) ||
        !make_tmap(&tv, V, BH, T, D))
      return KIA_ERR_CUDA;
    const size_t smq = tc_bwd_q_smem<D>(p), smk = tc_bwd_kv_smem<D>(p);
    if (smq > 232448 || smk > 232448) return KIA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(tc_bwd_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smq) != cudaSuccess ||
        cudaFuncSetAttribute(tc_bwd_kv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smk) != cudaSuccess)
      return KIA_ERR_CUDA;
    const int nt = (T + KIA_TILE - 1) / KIA_TILE;
    dim3 grid(BH, nt);
    tc_bwd_q_kernel<D><<<grid, kBwdThreads, smq, s>>>(tq, tg, tk, tkm, tv, st, wk, dQ, dS_dbg, p,
                                                      T);
    if (cudaGetLastError() != cudaSuccess) return KIA_ERR_CUDA;
    mark(4, s);
    tc_bwd_kv_kernel<D><<<grid, kBwdThreads, smk, s>>>(tq, tqm, tg, tgm, tk, tv, st, wk, dK, dV,
                                                       p, T);
    mark(5, s);
    return cudaGetLastError() == cudaSuccess ? KIA_OK : KIA_ERR_CUDA;
  }
}

}  // namespace kia
