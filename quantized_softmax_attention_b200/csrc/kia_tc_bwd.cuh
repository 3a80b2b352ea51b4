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
// Both passes stream the other side in half tiles of 64 rows through two
// TMEM buffers, so the MMAs of the next half tile run while the element
// warps work on the current one.  Each output row is owned by one CTA and
// written once: no atomics.  The calibration terms (section 3, Calibration
// gradients; Appendix B) are added afterwards from A and C by the row passes
// in kia_epilogue.cuh.
// Warp roles (10 warps): 0 = TMA producer, 1 = MMA issuer and TMEM owner,
// 2..9 = element warps (warp w reaches TMEM lanes 32*(w%4)..+31; warps w and
// w+4 split each half tile's 64 columns).
#pragma once
#include "kia_fast.cuh"
#include "kia_tc.cuh"

namespace kia {

constexpr int kBwdSmemTabK = 32;  // key pass: per-query grids up to K = 32 in shared memory

struct BwdQBars {
  uint64_t qd_full;               // Q_i, dO_i (K-major), once
  uint64_t kv_full, kv_empty;     // K_j, V_j K-major (for S, dP)
  uint64_t kmn_full, kmn_empty;   // K_j MN-major (for dQ)
  uint64_t sp_full[2];            // S and dP of a half tile in TMEM buffer b
  uint64_t elem_done[2];          // dS written into buffer b (256 arrivals)
  uint64_t st_free[2];            // dQ MMA of buffer b done
  uint64_t dq_full;               // all dQ MMAs done
  uint64_t row_sync;              // element-thread rendezvous (256 arrivals)
  uint32_t tmem_base;
  int abort;
};

struct BwdKBars {
  uint64_t kv_full;               // K_j, V_j K-major, once
  uint64_t qd_full, qd_empty;     // Q_i, dO_i K-major (for S^T, dP^T)
  uint64_t mn_full, mn_empty;     // Q_i, dO_i MN-major (for dK, dV)
  uint64_t sp_full[2];            // S^T and dP^T of a half tile in TMEM buffer b
  uint64_t qc_ready;              // per-query constants of a tile loaded (256 arrivals)
  uint64_t elem_done[2];          // P^T, dS^T written into buffer b (256 arrivals)
  uint64_t st_free[2];            // dV, dK MMAs of buffer b done
  uint64_t acc_full;              // all dV, dK MMAs done
  uint32_t tmem_base;
  int abort;
};

// ---------------------------------------------------------------- query pass

template <int D, class V, bool NEED_C>
__global__ void __launch_bounds__(kTcThreads, 1)
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
  float* sQ = reinterpret_cast<float*>(base);
  float* sG = reinterpret_cast<float*>(base + kTile);
  float* sK = reinterpret_cast<float*>(base + 2 * kTile);
  float* sKmn = reinterpret_cast<float*>(base + 3 * kTile);
  float* sV = reinterpret_cast<float*>(base + 4 * kTile);
  float* sAC = reinterpret_cast<float*>(base + 5 * kTile);   // [2 halves][2][128]
  float* sTab = sAC + 4 * KIA_TILE;
  const int tab_floats = V::SOFTMAX ? 0 : (V::MINMAX ? (p.K + 1) * KIA_TILE : (p.K + 1));
  BwdQBars& bar = *reinterpret_cast<BwdQBars*>(sTab + ((tab_floats + 31) & ~31));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int qt = nt - 1 - blockIdx.y;
  const int nkt = p.causal ? qt + 1 : nt;
  const int nunits = 2 * nkt;          // half key tiles
  constexpr uint32_t kColDQ = 256;

  if (threadIdx.x == 0) {
    mbar_init(&bar.qd_full, 1);
    mbar_init(&bar.kv_full, 1);
    mbar_init(&bar.kv_empty, 1);
    mbar_init(&bar.kmn_full, 1);
    mbar_init(&bar.kmn_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.sp_full[b], 1);
      mbar_init(&bar.elem_done[b], kElemThreads);
      mbar_init(&bar.st_free[b], 1);
    }
    mbar_init(&bar.dq_full, 1);
    mbar_init(&bar.row_sync, kElemThreads);
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
      const uint32_t id_s = idesc_tf32(128, 64, 0, 0);
      const uint32_t id_dq = idesc_tf32(128, D, 0, 1);
      const uint32_t qa = smem_u32(sQ), ga = smem_u32(sG), ka = smem_u32(sK),
                     kma = smem_u32(sKmn), va = smem_u32(sV);
      // dQ of half tile u: A = dS in TMEM buffer u&1, B = rows 64*(u&1).. of K_j (MN-major)
      auto issue_dq = [&](int u) -> bool {
        const int b = u & 1, j = u >> 1;
        if (!mbar_wait(&bar.elem_done[b], (u >> 1) & 1, abort)) return false;
        if (b == 0 && !mbar_wait(&bar.kmn_full, j & 1, abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_tf32_ts(tmem + kColDQ, tmem + 128u * b + 8u * kk, desc_mnmajor(kma, 8 * b + kk),
                      id_dq, (u > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&bar.st_free[b]);
        if (b == 1) tc_commit(&bar.kmn_empty);
        return true;
      };
      failed = !mbar_wait(&bar.qd_full, 0, abort);
      for (int u = 0; u < nunits && !failed; ++u) {
        const int b = u & 1, j = u >> 1;
        if (b == 0 && !mbar_wait(&bar.kv_full, j & 1, abort)) { failed = true; break; }
        if (u >= 2 && !mbar_wait(&bar.st_free[b], ((u >> 1) - 1) & 1, abort)) { failed = true; break; }
        tc_fence_after();
        const uint32_t koff = (uint32_t)b * 64u * 128u;     // rows 64b.. of the key tile
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks)
          mma_tf32_ss(tmem + 128u * b, desc_kmajor(qa, ks), desc_kmajor(ka + koff, ks), id_s,
                      ks > 0);
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks)
          mma_tf32_ss(tmem + 128u * b + 64u, desc_kmajor(ga, ks), desc_kmajor(va + koff, ks),
                      id_s, ks > 0);
        tc_commit(&bar.sp_full[b]);
        if (b == 1) tc_commit(&bar.kv_empty);
        if (u >= 1 && !issue_dq(u - 1)) { failed = true; break; }
      }
      if (!failed && !issue_dq(nunits - 1)) failed = true;
      if (!failed) tc_commit(&bar.dq_full);
    }
  } else {
    // ------------------------------------------------------ element warps
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    const int q = qt * KIA_TILE + r;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const long long rowbase = (long long)bh * T;
    const long long qr = rowbase + (q < T ? q : T - 1);
    // this row's calibration and centering (written by the forward and prep)
    const float m = st.m[qr];
    const float rh = st.rh[qr];
    const float nrh = -rh;
    const float dg = (V::MINMAX && rh == 0.0f) ? 1.0f : 0.0f;
    const int L = p.causal ? q + 1 : T;
    // a one-key row has P = 1 whatever its score: zero gradient
    const float rWb = (L == 1) ? 0.0f : __fdiv_rn(1.0f, st.Wb[qr]);
    const float Dc = wk.D[qr];
    const float Kf = p.Kf, Km1f = (float)(p.K - 1);
    const float* tab = sTab;
    int ts = 1;
    if constexpr (V::MINMAX) {
      for (int k = half; k <= p.K; k += 2) sTab[k * KIA_TILE + r] = st.table[qr * (p.K + 1) + k];
      tab = sTab + r;
      ts = KIA_TILE;
    } else if constexpr (!V::SOFTMAX) {
      const int k = (int)threadIdx.x - 64;
      if (k >= 0 && k <= p.K) sTab[k] = st.table[k];
    }
    mbar_arrive(&bar.row_sync);
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, 0, abort))) failed = true;
    float A = 0.0f, C = 0.0f;
    float v[32], g[32];
    for (int u = 0; u < nunits && !failed; ++u) {
      const int b = u & 1, j = u >> 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.sp_full[b], (u >> 1) & 1, abort))) { failed = true; break; }
      tc_fence_after();
      const uint32_t cs = 128u * b + 32u * half;       // this thread's 32 columns of S
      tmem_ld32(tmem + lane_addr + cs, v);
      tmem_ld32(tmem + lane_addr + cs + 64u, g);
      tmem_ld_wait();
      const int key0 = j * KIA_TILE + 64 * b + 32 * half;
      const bool edge = (p.causal && j == qt) || (j + 1) * KIA_TILE > T;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float dw = (g[i] - Dc) * rWb;
        if (edge) {
          const int key = key0 + i;
          if (!(key < T && (!p.causal || key <= q))) dw = 0.0f;
        }
        v[i] = bwd_delta<V, NEED_C>(tab, ts, m, rh, nrh, dg, Kf, Km1f, v[i], dw, A, C);
      }
      tmem_st32(tmem + lane_addr + cs, v);
      if (dS_dbg && q < T) {
        float* dst = dS_dbg + (rowbase + q) * T + key0;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (key0 + i < T) dst[i] = v[i];
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar.elem_done[b]);
    }
    // row sums of both halves
    sAC[(half * 2 + 0) * KIA_TILE + r] = A;
    sAC[(half * 2 + 1) * KIA_TILE + r] = C;
    mbar_arrive(&bar.row_sync);
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, 1, abort))) failed = true;
    if (!failed && __all_sync(0xffffffffu, mbar_wait(&bar.dq_full, 0, abort))) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        const uint32_t col = (uint32_t)(half * (D / 2) + 32 * c);
        tmem_ld32(tmem + lane_addr + kColDQ + col, v);
        tmem_ld_wait();
        if (q < T) {
          float4* o4 = reinterpret_cast<float4*>(dQ + (rowbase + q) * D + col);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            o4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
      if (q < T && half == 0) {
        wk.A[rowbase + q] = sAC[0 * KIA_TILE + r] + sAC[2 * KIA_TILE + r];
        wk.C[rowbase + q] = sAC[1 * KIA_TILE + r] + sAC[3 * KIA_TILE + r];
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

template <int D, class V>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQmn,
                 const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmGmn,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 StatsView st, WorkView wk, float* __restrict__ dK, float* __restrict__ dV,
                 OpParams p, int T, int tab_in_smem) {
  static_assert(D == 64, "tensor-core backward tiles are laid out for d = 64");
  constexpr uint32_t kTile = D * KIA_TILE * 4;
  if (*wk.status != 0) return;
  extern __shared__ uint8_t smraw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
  float* sK = reinterpret_cast<float*>(base);
  float* sV = reinterpret_cast<float*>(base + kTile);
  float* sQ = reinterpret_cast<float*>(base + 2 * kTile);
  float* sG = reinterpret_cast<float*>(base + 3 * kTile);
  float* sQmn = reinterpret_cast<float*>(base + 4 * kTile);
  float* sGmn = reinterpret_cast<float*>(base + 5 * kTile);
  float4* sC4 = reinterpret_cast<float4*>(base + 6 * kTile);       // (m, rh, D, rWb) per query
  float2* sC2 = reinterpret_cast<float2*>(sC4 + KIA_TILE);         // (rWf, dg) per query
  float* sTab = reinterpret_cast<float*>(sC2 + KIA_TILE);
  const int K1 = p.K + 1;
  const int tab_floats = V::SOFTMAX ? 0 : (V::MINMAX ? (tab_in_smem ? K1 * KIA_TILE : 0) : K1);
  BwdKBars& bar = *reinterpret_cast<BwdKBars*>(sTab + ((tab_floats + 31) & ~31));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int kt = blockIdx.y;
  const int q0 = p.causal ? kt : 0;
  const int ntiles = nt - q0;
  const int nunits = 2 * ntiles;       // half query tiles
  constexpr uint32_t kColDV = 256, kColDK = 256 + D;

  if (threadIdx.x == 0) {
    mbar_init(&bar.kv_full, 1);
    mbar_init(&bar.qd_full, 1);
    mbar_init(&bar.qd_empty, 1);
    mbar_init(&bar.mn_full, 1);
    mbar_init(&bar.mn_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.sp_full[b], 1);
      mbar_init(&bar.elem_done[b], kElemThreads);
      mbar_init(&bar.st_free[b], 1);
    }
    mbar_init(&bar.qc_ready, kElemThreads);
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
      for (int s = 0; s < ntiles; ++s) {
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
      const uint32_t id_s = idesc_tf32(128, 64, 0, 0);
      const uint32_t id_acc = idesc_tf32(128, D, 0, 1);
      const uint32_t ka = smem_u32(sK), va = smem_u32(sV), qa = smem_u32(sQ), ga = smem_u32(sG),
                     qma = smem_u32(sQmn), gma = smem_u32(sGmn);
      // dV += P^T dO, dK += dS^T Q for half tile u (queries 64*(u&1).. of tile u>>1)
      auto issue_acc = [&](int u) -> bool {
        const int b = u & 1, s = u >> 1;
        if (!mbar_wait(&bar.elem_done[b], (u >> 1) & 1, abort)) return false;
        if (b == 0 && !mbar_wait(&bar.mn_full, s & 1, abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_tf32_ts(tmem + kColDV, tmem + 128u * b + 8u * kk, desc_mnmajor(gma, 8 * b + kk),
                      id_acc, (u > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_tf32_ts(tmem + kColDK, tmem + 128u * b + 64u + 8u * kk,
                      desc_mnmajor(qma, 8 * b + kk), id_acc, (u > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&bar.st_free[b]);
        if (b == 1) tc_commit(&bar.mn_empty);
        return true;
      };
      failed = !mbar_wait(&bar.kv_full, 0, abort);
      for (int u = 0; u < nunits && !failed; ++u) {
        const int b = u & 1, s = u >> 1;
        if (b == 0 && !mbar_wait(&bar.qd_full, s & 1, abort)) { failed = true; break; }
        if (u >= 2 && !mbar_wait(&bar.st_free[b], ((u >> 1) - 1) & 1, abort)) { failed = true; break; }
        tc_fence_after();
        const uint32_t qoff = (uint32_t)b * 64u * 128u;     // query rows 64b.. of the tile
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks)
          mma_tf32_ss(tmem + 128u * b, desc_kmajor(ka, ks), desc_kmajor(qa + qoff, ks), id_s,
                      ks > 0);
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks)
          mma_tf32_ss(tmem + 128u * b + 64u, desc_kmajor(va, ks), desc_kmajor(ga + qoff, ks),
                      id_s, ks > 0);
        tc_commit(&bar.sp_full[b]);
        if (b == 1) tc_commit(&bar.qd_empty);
        if (u >= 1 && !issue_acc(u - 1)) { failed = true; break; }
      }
      if (!failed && !issue_acc(nunits - 1)) failed = true;
      if (!failed) tc_commit(&bar.acc_full);
    }
  } else {
    // ------------------------------------------------------ element warps
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quad * 32 + lane;
    const int e = (int)threadIdx.x - 64;          // 0..255
    const int kj = kt * KIA_TILE + r;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const long long rowbase = (long long)bh * T;
    const float Kf = p.Kf, Km1f = (float)(p.K - 1);
    if (!V::SOFTMAX && !V::MINMAX && e < K1) sTab[e] = st.table[e];
    float v[32], g[32];
    for (int u = 0; u < nunits && !failed; ++u) {
      const int b = u & 1, s = u >> 1;
      const int qi = q0 + s;
      if (b == 0) {
        // per-query constants of tile qi: every reader of the previous
        // tile's constants has arrived on that tile's last elem_done
        if (u >= 2 &&
            !__all_sync(0xffffffffu, mbar_wait(&bar.elem_done[1], ((u - 1) >> 1) & 1, abort))) {
          failed = true;
          break;
        }
        if (e < KIA_TILE) {
          const int q = qi * KIA_TILE + e;
          const long long qr = rowbase + (q < T ? q : T - 1);
          const float rhq = st.rh[qr];
          const int Lq = p.causal ? q + 1 : T;
          sC4[e] = make_float4(st.m[qr], rhq, wk.D[qr],
                               Lq == 1 ? 0.0f : __fdiv_rn(1.0f, st.Wb[qr]));
          sC2[e] = make_float2(__fdiv_rn(1.0f, st.Wf[qr]),
                               (V::MINMAX && rhq == 0.0f) ? 1.0f : 0.0f);
          if (V::MINMAX && tab_in_smem)
            for (int k = 0; k < K1; ++k) sTab[e * K1 + k] = st.table[qr * K1 + k];
        }
        mbar_arrive(&bar.qc_ready);
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.qc_ready, s & 1, abort))) { failed = true; break; }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.sp_full[b], (u >> 1) & 1, abort))) { failed = true; break; }
      tc_fence_after();
      const uint32_t cs = 128u * b + 32u * half;
      tmem_ld32(tmem + lane_addr + cs, v);
      tmem_ld32(tmem + lane_addr + cs + 64u, g);
      tmem_ld_wait();
      const int ql0 = 64 * b + 32 * half;              // first query (in the tile) of the chunk
      const bool edge =
          (p.causal && qi == kt) || (qi + 1) * KIA_TILE > T || (kt + 1) * KIA_TILE > T;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int ql = ql0 + i;
        const float4 c4 = sC4[ql];
        const float2 c2 = sC2[ql];
        const float* tab;
        int ts = 1;
        if constexpr (V::MINMAX) {
          tab = tab_in_smem ? sTab + ql * K1
                            : st.table + (rowbase + min(qi * KIA_TILE + ql, T - 1)) * K1;
        } else {
          tab = sTab;
        }
        float dw = (g[i] - c4.z) * c4.w;
        float P, dS;
        kv_elem<V>(tab, ts, c4.x, c4.y, -c4.y, c2.y, c2.x, Kf, Km1f, v[i], dw, P, dS);
        if (edge) {
          const int q = qi * KIA_TILE + ql;
          if (!(kj < T && q < T && (!p.causal || kj <= q))) {
            P = 0.0f;
            dS = 0.0f;
          }
        }
        v[i] = P;
        g[i] = dS;
      }
      tmem_st32(tmem + lane_addr + cs, v);
      tmem_st32(tmem + lane_addr + cs + 64u, g);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar.elem_done[b]);
    }
    if (!failed && __all_sync(0xffffffffu, mbar_wait(&bar.acc_full, 0, abort))) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        const uint32_t col = (uint32_t)(half * (D / 2) + 32 * c);
        tmem_ld32(tmem + lane_addr + kColDV + col, v);
        tmem_ld32(tmem + lane_addr + kColDK + col, g);
        tmem_ld_wait();
        if (kj < T) {
          float4* dv4 = reinterpret_cast<float4*>(dV + (rowbase + kj) * D + col);
          float4* dk4 = reinterpret_cast<float4*>(dK + (rowbase + kj) * D + col);
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
  return 1024 + 5 * (size_t)D * KIA_TILE * 4 + 4 * KIA_TILE * 4 + (size_t)((tab + 31) & ~31) * 4 +
         sizeof(BwdQBars);
}

template <int D>
size_t tc_bwd_kv_smem(const OpParams& p, bool tab_in_smem) {
  const bool minmax_tab = !p.softmax && p.cal == KIA_CAL_MINMAX;
  const int tab =
      p.softmax ? 0 : (minmax_tab ? (tab_in_smem ? (p.K + 1) * KIA_TILE : 0) : (p.K + 1));
  return 1024 + 6 * (size_t)D * KIA_TILE * 4 + KIA_TILE * (16 + 8) +
         (size_t)((tab + 31) & ~31) * 4 + sizeof(BwdKBars);
}

template <int D, class V>
int tc_backward_v(const float* Q, const float* Kt, const float* Vv, const float* dO,
                  const StatsView& st, const WorkView& wk, float* dQ, float* dK, float* dV,
                  float* dS_dbg, int B, int H, int T, const OpParams& p, cudaStream_t s,
                  void (*mark)(int, cudaStream_t)) {
  const int BH = B * H;
  CUtensorMap tq, tqm, tg, tgm, tk, tkm, tv;
  if (!make_tmap(&tq, Q, BH, T, D) || !make_tmap(&tqm, Q, BH, T, D, true) ||
      !make_tmap(&tg, dO, BH, T, D) || !make_tmap(&tgm, dO, BH, T, D, true) ||
      !make_tmap(&tk, Kt, BH, T, D) || !make_tmap(&tkm, Kt, BH, T, D, true) ||
      !make_tmap(&tv, Vv, BH, T, D))
    return KIA_ERR_CUDA;
  const size_t smq = tc_bwd_q_smem<D>(p);
  const bool kv_tab_smem = p.K <= kBwdSmemTabK;
  const size_t smk = tc_bwd_kv_smem<D>(p, kv_tab_smem);
  if (smq > 232448 || smk > 232448) return KIA_ERR_UNSUPPORTED;
  const bool need_c = V::MINMAX && (p.grad == KIA_GRAD_FULL || p.grad == KIA_GRAD_MAX_ONLY ||
                                    p.grad == KIA_GRAD_MIN_ONLY);
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  dim3 grid(BH, nt);
  if (need_c) {
    if (cudaFuncSetAttribute(tc_bwd_q_kernel<D, V, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smq) != cudaSuccess)
      return KIA_ERR_CUDA;
    tc_bwd_q_kernel<D, V, true><<<grid, kTcThreads, smq, s>>>(tq, tg, tk, tkm, tv, st, wk, dQ,
                                                              dS_dbg, p, T);
  } else {
    if (cudaFuncSetAttribute(tc_bwd_q_kernel<D, V, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smq) != cudaSuccess)
      return KIA_ERR_CUDA;
    tc_bwd_q_kernel<D, V, false><<<grid, kTcThreads, smq, s>>>(tq, tg, tk, tkm, tv, st, wk, dQ,
                                                               dS_dbg, p, T);
  }
  if (cudaGetLastError() != cudaSuccess) return KIA_ERR_CUDA;
  mark(4, s);
  if (cudaFuncSetAttribute(tc_bwd_kv_kernel<D, V>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smk) != cudaSuccess)
    return KIA_ERR_CUDA;
  tc_bwd_kv_kernel<D, V><<<grid, kTcThreads, smk, s>>>(tq, tqm, tg, tgm, tk, tv, st, wk, dK, dV, p,
                                                       T, kv_tab_smem ? 1 : 0);
  mark(5, s);
  return cudaGetLastError() == cudaSuccess ? KIA_OK : KIA_ERR_CUDA;
}

template <int D>
int tc_backward(const float* Q, const float* Kt, const float* V, const float* dO,
                const StatsView& st, const WorkView& wk, float* dQ, float* dK, float* dV,
                float* dS_dbg, int B, int H, int T, const OpParams& p, cudaStream_t s,
                void (*mark)(int, cudaStream_t)) {
  if constexpr (D != 64) {
    return KIA_ERR_UNSUPPORTED;
  } else {
    return dispatch_variant(p, [&]<class Vt>() {
      return tc_backward_v<D, Vt>(Q, Kt, V, dO, st, wk, dQ, dK, dV, dS_dbg, B, H, T, p, s, mark);
    });
  }
}

}  // namespace kia
