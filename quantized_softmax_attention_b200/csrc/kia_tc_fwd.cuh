// Fused tensor-core forward of K-interval attention (sm_100a).
//
// One CTA per (batch*head, 128-query tile), heaviest causal tiles first.
// Two sweeps over the keys, because the grid of a row is anchored at its
// final extrema (section 3, Calibration): no weight exists before the row
// max (and min) are known, so there is no online rescaling.
//   sweep 1: S = Q K^T (tcgen05 kind::tf32, accumulator in TMEM) -> row
//            max / min and their lowest indices;
//   calibration: h, 1/h, and the grid G_k = e^{-k h} (per row under MinMax,
//            one shared table under FWM) into shared memory;
//   sweep 2: S recomputed -> weights from the grid (LERP or Nearest, FWM
//            tail) -> written back into the same TMEM columns as the A
//            operand of O += P V (and P_L for Prob-STE, O_L += P_L V);
//   epilogue: O = O_acc / W (and O_L = O_L_acc / W_L), per-row statistics.
//
// Sweep 1 walks the keys in whole key tiles (N = 128 MMAs), sweep 2 in
// units of 64 (half key tiles); units are numbered across both sweeps, and
// unit U lives in TMEM region U % R (S / P in its first 64 columns, P_L in
// the next 64; R = 3 regions where the accumulators leave room), so the
// scores of the next units are computed while the current ones are turned
// into weights and multiplied into O.
// Warp roles (20 warps): 0 = TMA producer, 1 = issuer of the accumulating
// MMAs (O += P V, O_L += P_L V) and TMEM owner, 18 = issuer of the score
// MMAs (S = Q K^T) -- two issuing warps, each running its loop converged
// with one elected lane issuing -- 19 = spare, 2..17 = element warps, all
// sixteen on every unit: warp w reaches TMEM lanes 32*(w%4)..+31 (query
// rows), and the four warps that share those rows take a quarter of each
// unit's columns, so each query row is served by four threads whose row
// statistics are merged through shared memory.  O and O_L leave through
// shared memory and TMA stores.
#pragma once
#include <algorithm>

#include "kia_fast.cuh"
#include "kia_tc.cuh"

namespace kia {

constexpr int kRowSplit = 4;        // element threads per TMEM lane (row)
constexpr int kElemThreads = 128 * kRowSplit;   // 16 element warps (warps 2..17)
constexpr int kScoreWarp = 2 + kElemThreads / 32;   // warp 18: issues the score MMAs
// + TMA producer (warp 0), accumulating-MMA issuer (warp 1), score-MMA issuer
// (warp 18) and one spare warp, so that every SM sub-partition holds five
// warps (the register budget is set by the busiest sub-partition anyway)
constexpr int kTcThreads = kElemThreads + 128;

template <int D, bool PROB>
struct FwdCfg {
  static constexpr int kKStages = (D == 64) ? 3 : 1;     // K ring depth
  static constexpr int kVStages = (D == 64) ? 2 : 1;     // V ring depth
  static constexpr uint32_t kTileBytes = D * KIA_TILE * 4;
  // TMEM regions of 128 columns left beside O (and O_L), at most 3
  static constexpr int kAccCols = PROB ? 2 * D : D;
  static constexpr int kRegions = (512 - kAccCols) / 128 < 3 ? (512 - kAccCols) / 128 : 3;
  static_assert(kRegions >= 2, "two TMEM regions at least");
};

struct FwdBars {
  uint64_t q_full, q_empty;       // Q of an item / free once its S MMAs are done
  uint64_t k_full[3], k_empty[3];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[3];    // S of a unit ready in region r (tcgen05.commit)
  uint64_t s_free[3];    // sweep 1: the element warps done reading region r
  uint64_t p_ready[3];   // sweep 2: P (and P_L) written into region r
  uint64_t pv_done[3];   // sweep 2: P V of region r finished (tcgen05.commit)
  uint64_t o_full;       // all P V of an item done
  uint64_t o_free;       // the item's O (and O_L) read out of TMEM
  uint64_t row_sync;     // element-thread rendezvous, two or three times per item
  uint32_t tmem_base;
  int abort;
};

// Shared-memory scratch of the element warps: per-thread row statistics.
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
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
              const __grid_constant__ CUtensorMap tmOL, StatsView st, OpParams p, int B, int H,
              int T, int tab_in_smem, int nsk) {
  constexpr bool PROB = V::PROB;
  using Cfg = FwdCfg<D, PROB>;
  // K ring depth: Cfg::kKStages, one less when a MinMax grid table needs the
  // room (the producer and the score issuer are the only users of the ring)
  const int NSK = V::MINMAX ? nsk : Cfg::kKStages;   // a constant for the other variants
  constexpr int NSV = Cfg::kVStages, R = Cfg::kRegions;
  constexpr uint32_t kTileF = Cfg::kTileBytes / 4;     // floats per operand tile
  extern __shared__ uint8_t smraw[];
  uint8_t* base = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
  float* sQ = reinterpret_cast<float*>(base);
  float* sV = sQ + kTileF;
  FwdRowX& rx = *reinterpret_cast<FwdRowX*>(sV + NSV * kTileF);
  // epilogue: 1 KB per element warp to turn its rows into full-sector stores
  float* sStage = reinterpret_cast<float*>(&rx + 1);      // [16 warps][32][8]
  // the grid table: FWM's pairs, or MinMax's rows [K + 1][128] when
  // tab_in_smem is 1 (after the staging block) or 2 (over it: the table is
  // written after sweep 1 and read in sweep 2, the staging block written in
  // the epilogue, so each warp lets its stores read their staging before the
  // rendezvous that precedes the table's writes)
  constexpr int kStageF = kElemThreads / 32 * 256;
  float* sTab = (V::MINMAX && tab_in_smem == 2) ? sStage : sStage + kStageF;
  const int tab_end =
      V::SOFTMAX ? kStageF
                 : (V::MINMAX ? (tab_in_smem == 1   ? kStageF + (p.K + 1) * KIA_TILE
                                 : tab_in_smem == 2 ? max(kStageF, (p.K + 1) * KIA_TILE)
                                                    : kStageF)
                              : kStageF + 2 * (p.K + 1));
  FwdBars& bar = *reinterpret_cast<FwdBars*>(sStage + ((tab_end + 31) & ~31));
  // the K ring last (1024-aligned), so that its depth moves no other buffer
  float* sK = reinterpret_cast<float*>(
      base + ((reinterpret_cast<uint8_t*>(&bar + 1) - base + 1023) & ~(ptrdiff_t)1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = B * H;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int nitems = BH * nt;
  // item it -> (query tile, batch*head), heaviest causal tiles first; this
  // CTA takes its items in the serpentine order of ItemSeq
  auto item_qt = [&](int it) { return nt - 1 - it / BH; };
  auto item_bh = [&](int it) { return it % BH; };
  auto item_nkt = [&](int it) { return p.causal ? item_qt(it) + 1 : nt; };
  // TMEM columns: region r = [128 r, 128 r + 128); then O and O_L (D each)
  constexpr uint32_t col_o = 128u * R;
  constexpr uint32_t col_ol = col_o + D;

  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 1);
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.s_full[s], 1);
      mbar_init(&bar.s_free[s], kElemThreads);
      mbar_init(&bar.p_ready[s], kElemThreads);
      mbar_init(&bar.pv_done[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    mbar_init(&bar.o_full, 1);
    mbar_init(&bar.o_free, kElemThreads);
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
      int kc = 0, vc = 0, n = 0;
      ItemSeq seq(nitems);
      for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
        const int qt = item_qt(it), bh = item_bh(it), nkt = item_nkt(it);
        // Q of this item once the previous item's S MMAs are done with it
        if (!mbar_wait(&bar.q_empty, (n & 1) ^ 1, abort)) { failed = true; break; }
        // failure-handling test hook: the first CTA withholds its first Q tile
        // (neither the expected-bytes arrival nor the copy is issued, so
        // nothing is in flight for it) and the waits on it run out
        const bool withhold = p.withhold == 1 && blockIdx.x == 0 && n == 0;
        if (!withhold) {
          mbar_arrive_expect_tx(&bar.q_full, Cfg::kTileBytes);
          for (int b = 0; b < D / 32; ++b)
            tma_load_3d(sQ + b * 32 * KIA_TILE, &tmQ, &bar.q_full, b * 32, qt * KIA_TILE, bh);
        }
        for (int sweep = 0; sweep < 2 && !failed; ++sweep) {
          for (int j = 0; j < nkt; ++j) {
            {
              const int s = kc % NSK, nn = kc / NSK;
              if (!mbar_wait(&bar.k_empty[s], (nn & 1) ^ 1, abort)) { failed = true; break; }
              mbar_arrive_expect_tx(&bar.k_full[s], Cfg::kTileBytes);
              float* dst = sK + s * kTileF;
              for (int b = 0; b < D / 32; ++b)
                tma_load_3d(dst + b * 32 * KIA_TILE, &tmK, &bar.k_full[s], b * 32, j * KIA_TILE, bh);
              ++kc;
            }
            if (sweep == 1) {
              const int s = vc % NSV, nn = vc / NSV;
              if (!mbar_wait(&bar.v_empty[s], (nn & 1) ^ 1, abort)) { failed = true; break; }
              mbar_arrive_expect_tx(&bar.v_full[s], Cfg::kTileBytes);
              float* dst = sV + s * kTileF;
              for (int b = 0; b < D / 32; ++b)
                tma_load_3d(dst + b * 32 * KIA_TILE, &tmV, &bar.v_full[s], b * 32, j * KIA_TILE, bh);
              ++vc;
            }
          }
        }
      }
    }
  } else if (warp == kScoreWarp) {
    // ------------------------------------------------- score-MMA issuer
    // The whole warp runs the loop, so that its waits and descriptor
    // arithmetic stay warp-uniform; one elected lane issues each unit's MMAs
    // and their commits (issuing from a lone lane halved the MMA rate).
    {
      const uint32_t idesc_s = idesc_tf32(128, 64, 0, 0);    // sweep 2: half tiles
      const uint32_t idesc_t = idesc_tf32(128, 128, 0, 0);   // sweep 1: whole tiles
      // descriptors built once; each MMA only adds a constant step
      const uint64_t dq0 = desc_kmajor(smem_u32(sQ), 0);
      const uint64_t dk0 = desc_kmajor(smem_u32(sK), 0);
      int kc = 0, n = 0, G = 0;           // K tiles, items, units (numbered across items)
      // per region: phase bits of the s_free / pv_done waits, and whether its
      // last unit was a sweep-2 unit (released by pv_done) or not (s_free)
      uint32_t sf_par = 0, pv_par = 0, last_pv = 0;
      ItemSeq seq(nitems);
      for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
        if (!warp_wait(&bar.q_full, n & 1, abort)) { failed = true; break; }
        const int nkt = item_nkt(it), nunits = 2 * nkt;
        // units of an item: sweep 1 key tiles j (N = 128), then sweep 2 half
        // tiles u (N = 64); unit G goes into region G % R once the unit R
        // before it has released the region
        for (int v = 0; v < nkt + nunits; ++v, ++G) {
          const bool sweep2 = v >= nkt;
          const int r = G % R;
          if (G >= R) {
            if ((last_pv >> r) & 1u) {
              if (!warp_wait(&bar.pv_done[r], (pv_par >> r) & 1u, abort)) { failed = true; break; }
              pv_par ^= 1u << r;
            } else {
              if (!warp_wait(&bar.s_free[r], (sf_par >> r) & 1u, abort)) { failed = true; break; }
              sf_par ^= 1u << r;
            }
          }
          last_pv = sweep2 ? (last_pv | (1u << r)) : (last_pv & ~(1u << r));
          const int h = sweep2 ? ((v - nkt) & 1) : 0;   // half of the key tile (sweep 2)
          const int s = kc % NSK, nn = kc / NSK;
          if (h == 0 && !warp_wait(&bar.k_full[s], nn & 1, abort)) { failed = true; break; }
          const uint64_t dk = dk0 + desc_step((uint32_t)s * Cfg::kTileBytes + (uint32_t)h * 64u * 128u);
          const uint32_t dst = tmem + 128u * r;
          const bool last_half = !sweep2 || h == 1;
          if (elect_one()) {
            tc_fence_after();
            if (!sweep2) {
#pragma unroll
              for (int ks = 0; ks < D / 8; ++ks)
                mma_tf32_ss(dst, dq0 + kstep_kmajor(ks), dk + kstep_kmajor(ks), idesc_t, ks > 0 ? 1u : 0u);
            } else {
#pragma unroll
              for (int ks = 0; ks < D / 8; ++ks)
                mma_tf32_ss(dst, dq0 + kstep_kmajor(ks), dk + kstep_kmajor(ks), idesc_s, ks > 0 ? 1u : 0u);
            }
            tc_commit(&bar.s_full[r]);
            if (last_half) tc_commit(&bar.k_empty[s]);
          }
          __syncwarp();
          if (last_half) ++kc;
        }
        if (!failed) {
          if (elect_one()) tc_commit(&bar.q_empty);    // Q free once these MMAs are done
          __syncwarp();
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------- accumulating-MMA issuer
    // (whole warp, one elected lane issuing; see the score issuer)
    {
      const uint32_t idesc_o = idesc_tf32(128, D, 0, 1);
      const uint64_t dv0 = desc_mnmajor(smem_u32(sV), 0);
      int vc = 0, n = 0, G = 0;
      uint32_t pr_par = 0;                // per-region phase bits of the p_ready waits
      ItemSeq seq(nitems);
      for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
        const int nunits = 2 * item_nkt(it);
        G += item_nkt(it);                // this item's sweep-1 units (whole tiles)
        for (int u = 0; u < nunits; ++u, ++G) {
          const int r = G % R, h = u & 1;
          if (!warp_wait(&bar.p_ready[r], (pr_par >> r) & 1u, abort)) { failed = true; break; }
          pr_par ^= 1u << r;
          const int s = vc % NSV, nn = vc / NSV;
          if (h == 0 && !warp_wait(&bar.v_full[s], nn & 1, abort)) { failed = true; break; }
          // the accumulators restart with this item: the previous item's
          // epilogue must have read them
          if (u == 0 && n > 0 && !warp_wait(&bar.o_free, (n - 1) & 1, abort)) { failed = true; break; }
          const uint64_t dv = dv0 + desc_step((uint32_t)s * Cfg::kTileBytes) + kstep_mnmajor(8 * h);
          const uint32_t pa = tmem + 128u * r;
          const uint32_t acc0 = u > 0 ? 1u : 0u;
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_tf32_ts(tmem + col_o, pa + 8u * kk, dv + kstep_mnmajor(kk), idesc_o,
                          kk > 0 ? 1u : acc0);
            if constexpr (PROB) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_tf32_ts(tmem + col_ol, pa + 64u + 8u * kk, dv + kstep_mnmajor(kk), idesc_o,
                            kk > 0 ? 1u : acc0);
            }
            tc_commit(&bar.pv_done[r]);
            if (h == 1) tc_commit(&bar.v_empty[s]);
          }
          __syncwarp();
          if (h == 1) ++vc;
        }
        if (!failed) {
          if (elect_one()) tc_commit(&bar.o_full);
          __syncwarp();
        }
      }
    }
  } else if (warp < kScoreWarp) {
    // ------------------------------------------------------ element warps
    const int quad = warp & 3;
    const int part = (warp - 2) >> 2;          // 0..3: this warp's quarter of every unit
    const int r = quad * 32 + lane;            // query row in the tile
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const float Kf = p.Kf, Km1f = (float)(p.K - 1);
    int gbase = 0, n = 0, rs = 0;   // rs: row_sync phases passed
    ItemSeq seq(nitems);
    for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
      const int qt = item_qt(it), bh = item_bh(it), nunits = 2 * item_nkt(it);
      const int qrow = qt * KIA_TILE + r;
      const long long grow = (long long)bh * T + (qrow < T ? qrow : T - 1);
      // a unit holds masked keys when it reaches past the first row of the
      // tile (causal) or past the sequence end
      const int edge_from = p.causal ? (qt * KIA_TILE) / 64 : nunits;
      auto is_edge = [&](int u) { return u >= edge_from || (u + 1) * 64 > T; };
      // row extrema and the keys of their first occurrences
      float m = -INFINITY, n_ = INFINITY;
      int am = 0, an = 0;
      // sweep 1: statistics of this thread's 32 columns of every key tile
      const int nkt = nunits / 2;
      for (int j = 0; j < nkt; ++j) {
        const int U = gbase + j, rg = U % R;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.s_full[rg], (U / R) & 1, abort))) { failed = true; break; }
        tc_fence_after();
        {
          float v[32];
          tmem_ld32(tmem + lane_addr + 128u * rg + 32u * part, v);
          tmem_ld_wait_regs(v);
          tc_fence_before();
          mbar_arrive(&bar.s_free[rg]);
          const int key0 = KIA_TILE * j + 32 * part;
          if (!is_edge(2 * j + (part >> 1))) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              // strict comparisons keep the lowest index on ties
              if (v[i] > m) am = key0 + i;
              m = fmaxf(m, v[i]);
              if constexpr (V::MINMAX) {
                if (v[i] < n_) an = key0 + i;
                n_ = fminf(n_, v[i]);
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
                if (vn < n_) an = key;
                n_ = fminf(n_, vn);
              }
            }
          }
        }
      }
      if (failed) break;
      if (V::MINMAX && tab_in_smem == 2) {
        // the table overlays the staging block: this warp's epilogue stores
        // of the previous item have read it before the rendezvous below
        if (elect_one()) tma_store_wait_read();
        __syncwarp();
      }
      // merge the four threads of the row (lowest index on ties)
      rx.m[part][r] = m;
      rx.n[part][r] = n_;
      rx.am[part][r] = am;
      rx.an[part][r] = an;
      mbar_arrive(&bar.row_sync);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, rs++ & 1, abort))) { failed = true; break; }
      m = rx.m[0][r];
      am = rx.am[0][r];
      n_ = rx.n[0][r];
      an = rx.an[0][r];
#pragma unroll
      for (int h = 1; h < kRowSplit; ++h) {
        const float mh = rx.m[h][r], nh = rx.n[h][r];
        const int ah = rx.am[h][r], bh2 = rx.an[h][r];
        am = (mh > m) ? ah : (mh == m ? min(am, ah) : am);
        m = fmaxf(m, mh);
        an = (nh < n_) ? bh2 : (nh == n_ ? min(an, bh2) : an);
        n_ = fminf(n_, nh);
      }
      if constexpr (!V::MINMAX) {
        n_ = m;   // FWM and softmax do not use the row minimum
        an = am;
      }
      // calibration (section 3) and the grid
      const RowCal rc = row_calibration(p, m, n_);
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
        // one grid for every row and item: pairs (G_k, G_{k+1}), k = 0..K-1,
        // and the tail's zero pair at K, computed with the CTA's first item and
        // kept
        if (n == 0 && threadIdx.x == 64) sPair[p.K] = make_float2(0.0f, 0.0f);
        for (int k = (int)threadIdx.x - 64; k < p.K; k += kElemThreads) {
          if (n == 0) {
            const float G0 = grid_value(k, p.fwm_h), G1 = grid_value(k + 1, p.fwm_h);
            sPair[k] = make_float2(G0, G1);
          }
          if (bh == 0 && qt == nt - 1) {
            const float2 G = sPair[k];
            st.table[k] = G.x;
            if (k == p.K - 1) st.table[k + 1] = G.y;
          }
        }
      }
      // the grid in place before sweep 2: per row under MinMax; FWM's shared
      // grid is built with the CTA's first item only (softmax has none)
      if (V::MINMAX || (!V::SOFTMAX && n == 0)) {
        mbar_arrive(&bar.row_sync);
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, rs++ & 1, abort))) { failed = true; break; }
      }
      // sweep 2: weights -> P (and P_L) in TMEM, normalisers (even and odd
      // columns summed separately, as packed pairs)
      float2 W2 = make_float2(0.0f, 0.0f), WL2 = make_float2(0.0f, 0.0f);
      auto sweep2 = [&](auto grid) {
        for (int u = 0; u < nunits && !failed; ++u) {
          const int U = gbase + nkt + u, rg = U % R;
          if (!__all_sync(0xffffffffu, mbar_wait(&bar.s_full[rg], (U / R) & 1, abort))) { failed = true; break; }
          tc_fence_after();
          const bool edge = is_edge(u);
          const uint32_t col_s = 128u * rg + 16u * part;  // this thread's 16 S / P columns
          {
            constexpr int c = 0;
            float w16[16];
            [[maybe_unused]] float vl[16];
            tmem_ld16(tmem + lane_addr + col_s, w16);
            tmem_ld_wait_regs(w16);
            const int key0 = 64 * u + 16 * part;
            if (!edge) {
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                // two scores at a time (packed fp32 pairs); clamped like the
                // edge tiles: these scores come from other MMAs than the ones
                // the row max was taken from, and nothing makes the two
                // bit-identical
                float2 wf, wl;
                fwd_weights2<V, true>(grid, rc.m, rc.rh, Kf, Km1f, w16[i], w16[i + 1], wf, wl);
                W2 = add2(W2, wf);
                w16[i] = wf.x;
                w16[i + 1] = wf.y;
                if constexpr (PROB) {
                  WL2 = add2(WL2, wl);
                  vl[i] = wl.x;
                  vl[i + 1] = wl.y;
                }
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; i += 2) {
                float2 wf, wl;
                fwd_weights2<V, true>(grid, rc.m, rc.rh, Kf, Km1f, w16[i], w16[i + 1], wf, wl);
                const int key = key0 + i;
                const bool ok0 = key < T && (!p.causal || key <= qrow);
                const bool ok1 = key + 1 < T && (!p.causal || key + 1 <= qrow);
                wf = make_float2(ok0 ? wf.x : 0.0f, ok1 ? wf.y : 0.0f);
                wl = make_float2(ok0 ? wl.x : 0.0f, ok1 ? wl.y : 0.0f);
                W2 = add2(W2, wf);
                w16[i] = wf.x;
                w16[i + 1] = wf.y;
                if constexpr (PROB) {
                  WL2 = add2(WL2, wl);
                  vl[i] = wl.x;
                  vl[i + 1] = wl.y;
                }
              }
            }
            tmem_st16(tmem + lane_addr + col_s + 16u * c, w16);
            if constexpr (PROB) tmem_st16(tmem + lane_addr + col_s + 64u + 16u * c, vl);
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&bar.p_ready[rg]);
        }
      };
      if constexpr (V::MINMAX) {
        if (tab_in_smem) sweep2(GridF{sTab + r, KIA_TILE});
        else sweep2(GridF{st.table + grow * (p.K + 1), 1});
      } else {
        sweep2(make_gridz(sPair, p.K));
      }
      if (failed) break;
      gbase += nkt + nunits;
      // normalisers of the whole row
      rx.W[part][r] = W2.x + W2.y;
      rx.WL[part][r] = WL2.x + WL2.y;
      mbar_arrive(&bar.row_sync);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, rs++ & 1, abort))) { failed = true; break; }
      const float Wrow = (rx.W[0][r] + rx.W[1][r]) + (rx.W[2][r] + rx.W[3][r]);
      const float WLrow =
          PROB ? (rx.WL[0][r] + rx.WL[1][r]) + (rx.WL[2][r] + rx.WL[3][r]) : Wrow;
      // epilogue: this thread's D/4 columns of O (and O_L) out of TMEM, the
      // accumulators released, then stores staged per warp into whole sectors
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.o_full, n & 1, abort))) { failed = true; break; }
      tc_fence_after();
      constexpr int kCols = D / kRowSplit;     // 16 or 32
      const uint32_t col = (uint32_t)(part * kCols);
      float o[kCols], ol[PROB ? kCols : 1];
      if constexpr (kCols == 16) tmem_ld16(tmem + lane_addr + col_o + col, o);
      else tmem_ld32(tmem + lane_addr + col_o + col, o);
      tmem_ld_wait_regs(o);
      if constexpr (PROB) {
        if constexpr (kCols == 16) tmem_ld16(tmem + lane_addr + col_ol + col, ol);
        else tmem_ld32(tmem + lane_addr + col_ol + col, ol);
        tmem_ld_wait_regs(ol);
      }
      tc_fence_before();
      mbar_arrive(&bar.o_free);
      {
        // this warp's 32 rows x D/4 columns of O (and O_L), 8 columns per TMA
        // store through its staging block
        float* stg = sStage + (warp - 2) * 256;
        const int row0 = qt * KIA_TILE + quad * 32;
        const float rw = __frcp_rn(Wrow), rwl = __frcp_rn(WLrow);
#pragma unroll
        for (int pass = 0; pass < (PROB ? 2 : 1) * kCols / 8; ++pass) {
          constexpr int kPer = kCols / 8;             // passes per output
          const bool second = PROB && pass >= kPer;
          const int cp = second ? pass - kPer : pass;
          const float* src = ((PROB && second) ? ol : o) + 8 * cp;
          epilogue_store8(stg, second ? &tmOL : &tmO, src, second ? rwl : rw, lane,
                          (int)col + 8 * cp, row0, bh);
        }
      }
      if (qrow < T && part == 0) {
        st.m[grow] = m;
        st.n[grow] = n_;
        st.am[grow] = am;
        st.an[grow] = an;
        st.rh[grow] = degen ? 0.0f : rc.rh;
        st.h[grow] = degen ? 0.0f : rc.h;
        st.Wf[grow] = Wrow;
        st.Wb[grow] = (!V::SOFTMAX && lerp_normpoint(p)) ? WLrow : Wrow;
      }
      if (bh == 0 && qt == nt - 1 && threadIdx.x == 64) write_header(st.header, B, H, T, D, p);
    }
    epilogue_store_drain();
  }
  if (failed || *abort) drain_in_flight();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// tab_in_smem: 0 MinMax grids in global memory, 1 in their own region, 2 over
// the epilogue's staging block
template <int D, bool PROB>
size_t tc_fwd_smem(const OpParams& p, int tab_in_smem, int nsk) {
  using Cfg = FwdCfg<D, PROB>;
  const bool minmax_tab = !p.softmax && p.cal == KIA_CAL_MINMAX;
  const int stage_f = kElemThreads / 32 * 256;
  const int tab_end =
      p.softmax ? stage_f
                : (minmax_tab ? (tab_in_smem == 1   ? stage_f + (p.K + 1) * KIA_TILE
                                 : tab_in_smem == 2 ? std::max(stage_f, (p.K + 1) * KIA_TILE)
                                                    : stage_f)
                              : stage_f + 2 * (p.K + 1));
  const size_t head = (size_t)(1 + Cfg::kVStages) * Cfg::kTileBytes + sizeof(FwdRowX) +
                      (size_t)((tab_end + 31) & ~31) * 4 + sizeof(FwdBars);
  return 1024 + ((head + 1023) & ~(size_t)1023) + (size_t)nsk * Cfg::kTileBytes;
}

template <int D, class V>
int tc_forward_v(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                 const CUtensorMap& to, const CUtensorMap& tol, const StatsView& st, int B, int H,
                 int T, const OpParams& p, cudaStream_t s) {
  // a MinMax grid table in shared memory if it fits, with a K ring one stage
  // shallower if that is what makes it fit; else the grids are read from
  // global memory
  constexpr int kNsk = FwdCfg<D, V::PROB>::kKStages;
  const size_t kMax = dyn_smem_budget(tc_fwd_kernel<D, V>);
  int tab_in_smem = 1;
  int nsk = kNsk;
  size_t smem = tc_fwd_smem<D, V::PROB>(p, 1, nsk);
  if (smem > kMax && kNsk > 2) {
    nsk = kNsk - 1;
    smem = tc_fwd_smem<D, V::PROB>(p, 1, nsk);
  }
  if (smem > kMax && V::MINMAX) {
    // over the staging block, with the full K ring
    tab_in_smem = 2;
    nsk = kNsk;
    smem = tc_fwd_smem<D, V::PROB>(p, 2, nsk);
  }
  if (smem > kMax) {
    tab_in_smem = 0;
    nsk = kNsk;
    smem = tc_fwd_smem<D, V::PROB>(p, 0, nsk);
  }
  if (smem > kMax) return KIA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(tc_fwd_kernel<D, V>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return KIA_ERR_CUDA;
  // persistent: one CTA per SM walks the (query tile, batch*head) items
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int sms = num_sms();
  if (sms <= 0) return KIA_ERR_CUDA;
  const dim3 grid(std::min(sms, B * H * nt));
  tc_fwd_kernel<D, V><<<grid, kTcThreads, smem, s>>>(tq, tk, tv, to, tol, st, p, B, H, T,
                                                     tab_in_smem, nsk);
  return cudaGetLastError() == cudaSuccess ? KIA_OK : KIA_ERR_CUDA;
}

// Calls f.template operator()<V>() with the compile-time variant of p.
template <class F>
int dispatch_variant(const OpParams& p, F&& f) {
  if (p.softmax) {
    if (p.exp_round == 1)
      return f.template operator()<Var<KIA_CAL_MINMAX, KIA_REC_LERP, false, true, 1>>();
    if (p.exp_round == 2)
      return f.template operator()<Var<KIA_CAL_MINMAX, KIA_REC_LERP, false, true, 2>>();
    return f.template operator()<Var<KIA_CAL_MINMAX, KIA_REC_LERP, false, true>>();
  }
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
  CUtensorMap tq, tk, tv, to, tol;
  if (!make_tmap(&tq, Q, B * H, T, D) || !make_tmap(&tk, Kt, B * H, T, D) ||
      !make_tmap(&tv, V, B * H, T, D, /*mn_major=*/true) || !make_tmap_out(&to, O, B * H, T, D) ||
      !make_tmap_out(&tol, st.OL ? st.OL : O, B * H, T, D))
    return KIA_ERR_CUDA;
  return dispatch_variant(p, [&]<class Vt>() {
    return tc_forward_v<D, Vt>(tq, tk, tv, to, tol, st, B, H, T, p, s);
  });
}

}  // namespace kia
