// Fused tensor-core forward of K-interval attention (sm_100a).
//
// One CTA per (batch*head, 128-query tile), heaviest causal tiles first.
// Two sweeps over the key tiles, because the grid of a row is anchored at
// its final extrema (section 3, Calibration): no weight exists before the
// row max (and min) are known, so there is no online rescaling.
//   sweep 1: S = Q K^T (tcgen05 kind::tf32, accumulator in TMEM) -> row
//            max / min and their lowest indices;
//   calibration: h, 1/h, and the grid G_k = e^{-k h} (per row under MinMax,
//            one shared table under FWM) into shared memory;
//   sweep 2: S recomputed -> weights from the grid (LERP or Nearest, FWM
//            tail) -> written back into the same TMEM columns as the A
//            operand of O += P V (and P_L for Prob-STE, O_L += P_L V);
//   epilogue: O = O_acc / W (and O_L = O_L_acc / W_L), per-row statistics.
//
// Warp roles (18 warps): 0 = TMA producer, 1 = MMA issuer and TMEM owner,
// 2..17 = element warps.  Element warp w reaches TMEM lanes 32*(w%4)..+31
// (query rows); the four warps that share those rows split each 128-column
// tile into 32-column groups, so each query row is served by four threads
// whose row statistics are merged through shared memory.
#pragma once
#include "kia_fast.cuh"
#include "kia_tc.cuh"

namespace kia {

constexpr int kRowSplit = 4;        // element threads per TMEM lane (row)
constexpr int kElemThreads = 128 * kRowSplit;   // 16 element warps
constexpr int kTcThreads = kElemThreads + 64;   // + producer + MMA warp

template <int D>
struct FwdCfg {
  static constexpr int kStages = (D == 64) ? 2 : 1;      // K and V ring depth
  static constexpr uint32_t kTileBytes = D * KIA_TILE * 4;
};

struct FwdBars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2];    // S tile ready in TMEM buffer b (tcgen05.commit)
  uint64_t s_free[2];    // sweep 1: element warps done reading buffer b
  uint64_t p_ready[2];   // sweep 2: P written into buffer b
  uint64_t pv_done[2];   // sweep 2: P V of buffer b finished (tcgen05.commit)
  uint64_t pl_free;      // P_L consumed by O_L += P_L V (tcgen05.commit)
  uint64_t o_full;       // all P V done
  uint64_t row_sync;     // element-thread rendezvous, used 3 times
  uint32_t tmem_base;
  int abort;
};

// Shared-memory scratch of the element warps: per-column-group row statistics.
struct FwdRowX {
  float m[kRowSplit][KIA_TILE];
  float n[kRowSplit][KIA_TILE];
  int am[kRowSplit][KIA_TILE];
  int an[kRowSplit][KIA_TILE];
  float W[kRowSplit][KIA_TILE];
  float WL[kRowSplit][KIA_TILE];
};

template <int D, class V>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, float* __restrict__ O, StatsView st,
              OpParams p, int B, int H, int T, int nsb, int tab_in_smem) {
  using Cfg = FwdCfg<D>;
  constexpr int NS = Cfg::kStages;
  constexpr bool PROB = V::PROB;
  extern __shared__ uint8_t smraw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smraw) + 1023) &
                                             ~uintptr_t(1023));
  float* sQ = reinterpret_cast<float*>(base);
  float* sK = reinterpret_cast<float*>(base + Cfg::kTileBytes);
  float* sV = reinterpret_cast<float*>(base + (1 + NS) * Cfg::kTileBytes);
  FwdRowX& rx = *reinterpret_cast<FwdRowX*>(base + (1 + 2 * NS) * Cfg::kTileBytes);
  float* sTab = reinterpret_cast<float*>(&rx + 1);
  const int tab_floats =
      V::SOFTMAX ? 0 : (V::MINMAX ? (tab_in_smem ? (p.K + 1) * KIA_TILE : 0) : 2 * (p.K + 1));
  FwdBars& bar = *reinterpret_cast<FwdBars*>(sTab + ((tab_floats + 31) & ~31));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int qt = nt - 1 - blockIdx.y;
  const int nkt = p.causal ? qt + 1 : nt;
  // TMEM columns: S buffers [0, 128*nsb), P_L, O, O_L
  const uint32_t col_pl = 128u * nsb;
  const uint32_t col_o = col_pl + (PROB ? 128u : 0u);
  const uint32_t col_ol = col_o + D;

  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], 1);
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.s_free[s], kElemThreads);
      mbar_init(&bar.p_ready[s], kElemThreads);
      mbar_init(&bar.pv_done[s], 1);
    }
    mbar_init(&bar.pl_free, 1);
    mbar_init(&bar.o_full, 1);
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
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar.q_full, Cfg::kTileBytes);
      for (int b = 0; b < D / 32; ++b)
        tma_load_3d(sQ + b * 32 * KIA_TILE, &tmQ, &bar.q_full, b * 32, qt * KIA_TILE, bh);
      int kc = 0, vc = 0;
      for (int sweep = 0; sweep < 2 && !failed; ++sweep) {
        for (int j = 0; j < nkt; ++j) {
          {
            const int s = kc % NS, n = kc / NS;
            if (!mbar_wait(&bar.k_empty[s], (n & 1) ^ 1, abort)) { failed = true; break; }
            mbar_arrive_expect_tx(&bar.k_full[s], Cfg::kTileBytes);
            float* dst = sK + s * (Cfg::kTileBytes / 4);
            for (int b = 0; b < D / 32; ++b)
              tma_load_3d(dst + b * 32 * KIA_TILE, &tmK, &bar.k_full[s], b * 32, j * KIA_TILE, bh);
            ++kc;
          }
          if (sweep == 1) {
            const int s = vc % NS, n = vc / NS;
            if (!mbar_wait(&bar.v_empty[s], (n & 1) ^ 1, abort)) { failed = true; break; }
            mbar_arrive_expect_tx(&bar.v_full[s], Cfg::kTileBytes);
            float* dst = sV + s * (Cfg::kTileBytes / 4);
            for (int b = 0; b < D / 32; ++b)
              tma_load_3d(dst + b * 32 * KIA_TILE, &tmV, &bar.v_full[s], b * 32, j * KIA_TILE, bh);
            ++vc;
          }
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_tf32(128, 128, 0, 0);
      const uint32_t idesc_o = idesc_tf32(128, D, 0, 1);
      const uint32_t qa = smem_u32(sQ);
      int kc = 0, vc = 0;
      int use1[2] = {0, 0};   // sweep-1 uses of each S buffer
      int use2[2] = {0, 0};   // sweep-2 uses of each S buffer
      failed = !mbar_wait(&bar.q_full, 0, abort);
      // issue S = Q K_j^T into buffer j % nsb
      auto issue_s = [&](int sweep, int j) -> bool {
        const int b = j % nsb;
        if (sweep == 0) {
          if (use1[b] > 0 && !mbar_wait(&bar.s_free[b], (use1[b] - 1) & 1, abort)) return false;
          ++use1[b];
        } else {
          if (use2[b] == 0) {
            if (use1[b] > 0 && !mbar_wait(&bar.s_free[b], (use1[b] - 1) & 1, abort)) return false;
          } else if (!mbar_wait(&bar.pv_done[b], (use2[b] - 1) & 1, abort)) {
            return false;
          }
          ++use2[b];
        }
        const int s = kc % NS, n = kc / NS;
        if (!mbar_wait(&bar.k_full[s], n & 1, abort)) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(sK + s * (Cfg::kTileBytes / 4));
#pragma unroll
        for (int ks = 0; ks < D / 8; ++ks)
          mma_tf32_ss(tmem + 128u * b, desc_kmajor(qa, ks), desc_kmajor(ka, ks), idesc_s,
                      ks > 0 ? 1u : 0u);
        tc_commit(&bar.s_full[b]);
        tc_commit(&bar.k_empty[s]);
        ++kc;
        return true;
      };
      if (!failed) {
        for (int j = 0; j < nkt; ++j)
          if (!issue_s(0, j)) { failed = true; break; }
      }
      if (!failed) {
        int pr[2] = {0, 0};
        if (!issue_s(1, 0)) failed = true;
        for (int j = 0; j < nkt && !failed; ++j) {
          // two S buffers: the next S overlaps this tile's weights and P V;
          // one buffer: the next S must wait until P V has read P
          if (nsb == 2 && j + 1 < nkt && !issue_s(1, j + 1)) { failed = true; break; }
          const int b = j % nsb;
          if (!mbar_wait(&bar.p_ready[b], pr[b] & 1, abort)) { failed = true; break; }
          ++pr[b];
          const int s = vc % NS, n = vc / NS;
          if (!mbar_wait(&bar.v_full[s], n & 1, abort)) { failed = true; break; }
          tc_fence_after();
          const uint32_t va = smem_u32(sV + s * (Cfg::kTileBytes / 4));
#pragma unroll
          for (int ks = 0; ks < KIA_TILE / 8; ++ks)
            mma_tf32_ts(tmem + col_o, tmem + 128u * b + 8u * ks, desc_mnmajor(va, ks), idesc_o,
                        (j > 0 || ks > 0) ? 1u : 0u);
          if constexpr (PROB) {
#pragma unroll
            for (int ks = 0; ks < KIA_TILE / 8; ++ks)
              mma_tf32_ts(tmem + col_ol, tmem + col_pl + 8u * ks, desc_mnmajor(va, ks), idesc_o,
                          (j > 0 || ks > 0) ? 1u : 0u);
            tc_commit(&bar.pl_free);
          }
          tc_commit(&bar.v_empty[s]);
          tc_commit(&bar.pv_done[b]);
          ++vc;
          if (nsb == 1 && j + 1 < nkt && !issue_s(1, j + 1)) { failed = true; break; }
        }
        if (!failed) tc_commit(&bar.o_full);
      }
    }
  } else {
    // ------------------------------------------------------ element warps
    const int quad = warp & 3;
    const int part = (warp - 2) >> 2;          // which 32 columns of a tile
    const int r = quad * 32 + lane;            // query row in the tile
    const int qrow = qt * KIA_TILE + r;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t col0 = 32u * part;
    const long long grow = (long long)bh * T + (qrow < T ? qrow : T - 1);
    int sf[2] = {0, 0};  // completed phases of s_full per buffer
    // row extrema and the keys of their first occurrences
    float m = -INFINITY, n = INFINITY;
    int am = 0, an = 0;
    float v[32];
    // sweep 1: statistics of this thread's 32 columns of each tile
    for (int j = 0; j < nkt; ++j) {
      const int b = j % nsb;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.s_full[b], sf[b] & 1, abort))) { failed = true; break; }
      ++sf[b];
      tc_fence_after();
      const bool edge = (p.causal && j == qt) || (j + 1) * KIA_TILE > T;
      tmem_ld32(tmem + lane_addr + 128u * b + col0, v);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bar.s_free[b]);
      const int key0 = j * KIA_TILE + (int)col0;
      if (!edge) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          // strict comparisons keep the lowest index on ties
          if (v[i] > m) am = key0 + i;
          m = fmaxf(m, v[i]);
          if constexpr (V::MINMAX) {
            if (v[i] < n) an = key0 + i;
            n = fminf(n, v[i]);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int key = key0 + i;
          const bool ok = key < T && (!p.causal || key <= qrow);
          const float vx = ok ? v[i] : -INFINITY;
          if (vx > m) am = key;
          m = fmaxf(m, vx);
          if constexpr (V::MINMAX) {
            const float vn = ok ? v[i] : INFINITY;
            if (vn < n) an = key;
            n = fminf(n, vn);
          }
        }
      }
    }
    // merge the four column groups of the row (lowest index on ties)
    rx.m[part][r] = m;
    rx.n[part][r] = n;
    rx.am[part][r] = am;
    rx.an[part][r] = an;
    mbar_arrive(&bar.row_sync);
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, 0, abort))) failed = true;
    m = rx.m[0][r];
    am = rx.am[0][r];
    n = rx.n[0][r];
    an = rx.an[0][r];
#pragma unroll
    for (int h = 1; h < kRowSplit; ++h) {
      const float mh = rx.m[h][r], nh = rx.n[h][r];
      const int ah = rx.am[h][r], bh2 = rx.an[h][r];
      am = (mh > m) ? ah : (mh == m ? min(am, ah) : am);
      m = fmaxf(m, mh);
      an = (nh < n) ? bh2 : (nh == n ? min(an, bh2) : an);
      n = fminf(n, nh);
    }
    if constexpr (!V::MINMAX) {
      n = m;   // FWM and softmax do not use the row minimum
      an = am;
    }
    // calibration (section 3) and the grid
    const RowCal rc = row_calibration(p, m, n);
    const bool degen = V::MINMAX && rc.h == 0.0f;
    float2* sPair = reinterpret_cast<float2*>(sTab);
    if constexpr (V::MINMAX) {
      if (tab_in_smem) {
        for (int k = part; k <= p.K; k += kRowSplit) {
          const float G = degen ? 1.0f : grid_value(k, rc.h);
          sTab[k * KIA_TILE + r] = G;
          if (qrow < T) st.table[grow * (p.K + 1) + k] = G;
        }
      } else {
        for (int k = part; k <= p.K; k += kRowSplit) {
          const float G = degen ? 1.0f : grid_value(k, rc.h);
          if (qrow < T) st.table[grow * (p.K + 1) + k] = G;
        }
        __threadfence_block();
      }
    } else if constexpr (!V::SOFTMAX) {
      // one grid for every row: pairs (G_k, G_{k+1}), k = 0..K-1
      const int k = (int)threadIdx.x - 64;
      if (k >= 0 && k < p.K) {
        const float G0 = grid_value(k, p.fwm_h), G1 = grid_value(k + 1, p.fwm_h);
        sPair[k] = make_float2(G0, G1);
        if (bh == 0 && qt == nt - 1) {
          st.table[k] = G0;
          if (k == p.K - 1) st.table[k + 1] = G1;
        }
      }
    }
    mbar_arrive(&bar.row_sync);
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, 1, abort))) failed = true;
    const float Kf = p.Kf, Km1f = (float)(p.K - 1);
    // sweep 2: weights -> P (and P_L) in TMEM, normalisers
    float W = 0.0f, WL = 0.0f;
    auto sweep2 = [&](auto grid) {
      for (int j = 0; j < nkt && !failed; ++j) {
        const int b = j % nsb;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.s_full[b], sf[b] & 1, abort))) { failed = true; break; }
        ++sf[b];
        if (PROB && j > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(&bar.pl_free, (j - 1) & 1, abort))) {
          failed = true;
          break;
        }
        tc_fence_after();
        const bool edge = (p.causal && j == qt) || (j + 1) * KIA_TILE > T;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          const uint32_t col = col0 + 16u * c;
          float w16[16], vl[16];
          tmem_ld16(tmem + lane_addr + 128u * b + col, w16);
          tmem_ld_wait();
          const int key0 = j * KIA_TILE + (int)col;
          if (!edge) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float wf, wl;
              fwd_weights<V, false>(grid, rc.m, rc.rh, Kf, Km1f, w16[i], wf, wl);
              W += wf;
              w16[i] = wf;
              if constexpr (PROB) {
                WL += wl;
                vl[i] = wl;
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float wf, wl;
              fwd_weights<V, true>(grid, rc.m, rc.rh, Kf, Km1f, w16[i], wf, wl);
              const int key = key0 + i;
              const bool ok = key < T && (!p.causal || key <= qrow);
              wf = ok ? wf : 0.0f;
              wl = ok ? wl : 0.0f;
              W += wf;
              w16[i] = wf;
              if constexpr (PROB) {
                WL += wl;
                vl[i] = wl;
              }
            }
          }
          tmem_st16(tmem + lane_addr + 128u * b + col, w16);
          if constexpr (PROB) tmem_st16(tmem + lane_addr + col_pl + col, vl);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar.p_ready[b]);
      }
    };
    if constexpr (V::MINMAX) {
      if (tab_in_smem) sweep2(GridF{sTab + r, KIA_TILE});
      else sweep2(GridF{st.table + grow * (p.K + 1), 1});
    } else {
      sweep2(GridP{sPair});
    }
    // normalisers of the whole row
    rx.W[part][r] = W;
    rx.WL[part][r] = WL;
    mbar_arrive(&bar.row_sync);
    if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, 0, abort))) failed = true;
    const float Wrow = (rx.W[0][r] + rx.W[1][r]) + (rx.W[2][r] + rx.W[3][r]);
    const float WLrow =
        PROB ? (rx.WL[0][r] + rx.WL[1][r]) + (rx.WL[2][r] + rx.WL[3][r]) : Wrow;
    // epilogue: this thread writes D/4 columns of its row
    if (!failed && __all_sync(0xffffffffu, mbar_wait(&bar.o_full, 0, abort))) {
      tc_fence_after();
      constexpr int kCols = D / kRowSplit;     // 16 or 32
      const uint32_t col = (uint32_t)(part * kCols);
      float o[kCols];
      auto write_row = [&](uint32_t tcol, float* dst, float w) {
        if constexpr (kCols == 16) tmem_ld16(tmem + lane_addr + tcol + col, o);
        else tmem_ld32(tmem + lane_addr + tcol + col, o);
        tmem_ld_wait();
        if (qrow < T) {
          float4* o4 = reinterpret_cast<float4*>(dst + grow * D + col);
#pragma unroll
          for (int i = 0; i < kCols / 4; ++i)
            o4[i] = make_float4(__fdiv_rn(o[4 * i], w), __fdiv_rn(o[4 * i + 1], w),
                                __fdiv_rn(o[4 * i + 2], w), __fdiv_rn(o[4 * i + 3], w));
        }
      };
      write_row(col_o, O, Wrow);
      if constexpr (PROB) write_row(col_ol, st.OL, WLrow);
      if (qrow < T && part == 0) {
        st.m[grow] = m;
        st.n[grow] = n;
        st.am[grow] = am;
        st.an[grow] = an;
        st.rh[grow] = degen ? 0.0f : rc.rh;
        st.h[grow] = degen ? 0.0f : rc.h;
        st.Wf[grow] = Wrow;
        st.Wb[grow] = (!V::SOFTMAX && lerp_normpoint(p)) ? WLrow : Wrow;
      }
      if (bh == 0 && qt == nt - 1 && threadIdx.x == 64) write_header(st.header, B, H, T, D, p);
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
size_t tc_fwd_smem(const OpParams& p, bool tab_in_smem) {
  constexpr int NS = FwdCfg<D>::kStages;
  const bool minmax_tab = !p.softmax && p.cal == KIA_CAL_MINMAX;
  const int tab =
      p.softmax ? 0 : (minmax_tab ? (tab_in_smem ? (p.K + 1) * KIA_TILE : 0) : 2 * (p.K + 1));
  return 1024 + (size_t)(1 + 2 * NS) * FwdCfg<D>::kTileBytes + sizeof(FwdRowX) +
         (size_t)((tab + 31) & ~31) * 4 + sizeof(FwdBars);
}

template <int D, class V>
int tc_forward_v(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, float* O,
                 const StatsView& st, int B, int H, int T, const OpParams& p, cudaStream_t s) {
  bool tab_in_smem = true;
  size_t smem = tc_fwd_smem<D>(p, true);
  if (smem > 232448) {
    tab_in_smem = false;
    smem = tc_fwd_smem<D>(p, false);
  }
  if (smem > 232448) return KIA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(tc_fwd_kernel<D, V>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return KIA_ERR_CUDA;
  // TMEM: S buffers (128 columns each), P_L (128, Prob-STE), O and O_L (D each)
  int nsb = 2;
  if (256 + (V::PROB ? 128 + 2 * D : D) > 512) nsb = 1;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  dim3 grid(B * H, nt);
  tc_fwd_kernel<D, V><<<grid, kTcThreads, smem, s>>>(tq, tk, tv, O, st, p, B, H, T, nsb,
                                                     tab_in_smem ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? KIA_OK : KIA_ERR_CUDA;
}

// Calls f.template operator()<V>() with the compile-time variant of p.
template <class F>
int dispatch_variant(const OpParams& p, F&& f) {
  if (p.softmax) return f.template operator()<Var<KIA_CAL_MINMAX, KIA_REC_LERP, false, true>>();
  const bool prob = p.rec == KIA_REC_NEAREST && p.ste == KIA_STE_PROB;
  if (p.cal == KIA_CAL_MINMAX) {
    if (p.rec == KIA_REC_LERP)
      return f.template operator()<Var<KIA_CAL_MINMAX, KIA_REC_LERP, false, false>>();
    if (prob) return f.template operator()<Var<KIA_CAL_MINMAX, KIA_REC_NEAREST, true, false>>();
    return f.template operator()<Var<KIA_CAL_MINMAX, KIA_REC_NEAREST, false, false>>();
  }
  if (p.rec == KIA_REC_LERP)
    return f.template operator()<Var<KIA_CAL_FWM, KIA_REC_LERP, false, false>>();
  if (prob) return f.template operator()<Var<KIA_CAL_FWM, KIA_REC_NEAREST, true, false>>();
  return f.template operator()<Var<KIA_CAL_FWM, KIA_REC_NEAREST, false, false>>();
}

template <int D>
int tc_forward(const float* Q, const float* Kt, const float* V, float* O, void* stats, int B,
               int H, int T, const OpParams& p, cudaStream_t s) {
  const long long rows = (long long)B * H * T;
  StatsView st = stats_view(stats, rows, D, p);
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, Q, B * H, T, D) || !make_tmap(&tk, Kt, B * H, T, D) ||
      !make_tmap(&tv, V, B * H, T, D, /*mn_major=*/true))
    return KIA_ERR_CUDA;
  return dispatch_variant(p, [&]<class Vt>() {
    return tc_forward_v<D, Vt>(tq, tk, tv, O, st, B, H, T, p, s);
  });
}

}  // namespace kia
