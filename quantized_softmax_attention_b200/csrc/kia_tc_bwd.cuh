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
// Both passes stream the other side in half tiles of 64 rows through three
// rotating TMEM regions, so the MMAs of the next half tiles run while the
// element warps work on the current one.  Each output row is owned by one
// CTA and written once: no atomics.  The query pass also computes the
// centering D of its rows and, once its row sums are complete, the
// calibration terms (section 3, Calibration gradients; Appendix B): g_m at
// the argmax key and g_n at the argmin key (or the zero-sum projection's
// shift), added to dQ there and folded into dS^T by the key pass before its
// dK contraction.
// Warp roles (20 warps): 0 = TMA producer, 1 = issuer of the accumulating
// MMAs (dQ, or dV and dK) and TMEM owner, 18 = issuer of the score MMAs
// (S and dP), 19 = spare (query pass) or the per-query constant producer
// (key pass), 2..17 = element warps, all sixteen on every half tile: warp w
// reaches TMEM lanes 32*(w%4)..+31, and the four warps that share those
// lanes take 16 of the half tile's 64 columns each.  (Two groups taking
// alternate half tiles left one group idle at the end of every item while
// the other finished its last half tile.)
#pragma once
#include <algorithm>
#include <type_traits>

#include "kia_fast.cuh"
#include "kia_tc.cuh"

namespace kia {

// key pass: slots of per-query constants (MinMax keeps two, so that the
// slots' per-query grids fit in shared memory up to K = 22)
template <class V>
__host__ __device__ constexpr int kv_const_slots() { return V::MINMAX ? 2 : 4; }
constexpr int kBwdRegions = 3;    // TMEM regions of 128 columns (S | dP) in rotation
constexpr int kBwdSlots = 3;      // query pass: slots of the K / V half-tile ring
constexpr int kKmnSlots = 2;      // query pass: slots of the K MN-major half-tile ring
constexpr uint32_t kHalfTile = 64 * 64 * 4;       // one operand's half tile (64 rows, d = 64)
constexpr uint32_t kHalfPair = 2 * kHalfTile;     // K half and V half (Q half and dO half)
constexpr int kKvSlots = 2;       // key pass: slots of each half-tile query ring

struct BwdQBars {
  uint64_t qd_full, qd_empty;     // Q_i, dO_i (K-major), per item
  uint64_t d_read;                // the element warps done reading dO_i for the centering D
  uint64_t kv_full[3], kv_empty[3];     // half tiles of K, V K-major (for S, dP)
  uint64_t kmn_full[3], kmn_empty[3];   // half tiles of K MN-major (for dQ)
  uint64_t sp_full[3];            // S and dP of a half tile in TMEM region r
  uint64_t elem_done[3];          // dS written into region r
  uint64_t st_free[3];            // dQ MMA of region r done
  uint64_t dq_full;               // all dQ MMAs of an item done
  uint64_t dq_free;               // the item's dQ read out of TMEM
  uint64_t row_sync;              // element-thread rendezvous
  uint32_t tmem_base;
  int abort;
};

struct BwdKBars {
  uint64_t kv_full, kv_empty;     // K_j, V_j K-major, per item
  uint64_t qd_full[2], qd_empty[2];     // half tiles of Q, dO K-major (for S^T, dP^T)
  uint64_t mn_full[2], mn_empty[2];     // half tiles of Q, dO MN-major (for dK, dV)
  uint64_t sp_full[3];            // S^T and dP^T of a half tile in TMEM region r
  uint64_t qc_ready[4];           // per-query constants of a unit loaded into slot s
  uint64_t qc_free[4];            // the unit's group done with slot s
  uint64_t elem_done[3];          // P^T, dS^T written into region r
  uint64_t st_free[3];            // dV, dK MMAs of region r done
  uint64_t acc_full;              // all dV, dK MMAs of an item done
  uint64_t acc_free;              // the item's dV, dK read out of TMEM
  uint64_t acc_issued;            // the item's last dV, dK MMAs issued
  uint32_t tmem_base;
  int abort;
};

// ---------------------------------------------------------------- query pass

template <int D, class V, bool NEED_C>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_bwd_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKmn,
                const __grid_constant__ CUtensorMap tmV, const float* __restrict__ Kt,
                const float* __restrict__ O,
                const __grid_constant__ CUtensorMap tmdQ, StatsView st, WorkView wk,
                float* __restrict__ dS_dbg, OpParams p, int B, int H, int T, int tab_in_smem,
                int nkv) {
  static_assert(D == 64, "tensor-core backward tiles are laid out for d = 64");
  constexpr uint32_t kTile = D * KIA_TILE * 4;
  // the stats must come from a forward of this shape and configuration
  __shared__ int s_hdr_ok;
  if (threadIdx.x == 0) {
    const bool ok = header_matches(st.header, B, H, T, D, p);
    s_hdr_ok = ok ? 1 : 0;
    if (blockIdx.x == 0) *wk.status = ok ? 0 : 1;
    if (!ok) atomicExch(&g_kia_device_error, KIA_ERR_STATS_MISMATCH);
  }
  __syncthreads();
  if (!s_hdr_ok) return;
  extern __shared__ uint8_t smraw[];
  uint8_t* base = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
  // Q_i and dO_i stay for an item; the keys stream through two rings of half tiles
  // (64 keys): K and V K-major (for S and dP) and K MN-major (for dQ), three
  // slots each, so that a slot refills while the next two are in use.
  float* sQ = reinterpret_cast<float*>(base);
  float* sG = reinterpret_cast<float*>(base + kTile);
  // the K / V ring has kBwdSlots slots, one less when a MinMax grid table
  // needs the room (only the producer and the score issuer use the ring)
  const int NKV = V::MINMAX ? nkv : kBwdSlots;   // a constant for the other variants
  uint8_t* sKmn = base + 2 * kTile;                          // [2][K half, MN-major]
  // epilogue: 1 KB per element warp to turn its rows into full-sector stores
  float* sStage = reinterpret_cast<float*>(sKmn + kKmnSlots * kHalfTile);   // [16 warps][32][8]
  float* sAC = sStage + kElemThreads / 32 * 256;              // [kRowSplit][2][128]
  float* sDc = sAC + 2 * kRowSplit * KIA_TILE;               // [128] centering D
  float* sTab = sDc + KIA_TILE;
  const int tab_floats =
      V::SOFTMAX ? 0 : (V::MINMAX ? (tab_in_smem ? (p.K + 1) * KIA_TILE : 0) : 2 * (p.K + 1));
  BwdQBars& bar = *reinterpret_cast<BwdQBars*>(sTab + ((tab_floats + 31) & ~31));
  // the K / V ring last (1024-aligned), so that its depth moves no other buffer
  uint8_t* sKV =
      base + ((reinterpret_cast<uint8_t*>(&bar + 1) - base + 1023) & ~(ptrdiff_t)1023);  // [NKV][K | V]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = B * H;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int nitems = BH * nt;
  // item it -> (query tile, batch*head), heaviest causal tiles first; this
  // CTA takes its items in the serpentine order of ItemSeq
  auto item_qt = [&](int it) { return nt - 1 - it / BH; };
  auto item_bh = [&](int it) { return it % BH; };
  auto item_units = [&](int it) { return 2 * (p.causal ? item_qt(it) + 1 : nt); };
  constexpr int R = kBwdRegions;
  constexpr uint32_t kColDQ = 128u * R;

  if (threadIdx.x == 0) {
    mbar_init(&bar.qd_full, 1);
    mbar_init(&bar.qd_empty, 1);
    mbar_init(&bar.d_read, kElemThreads);
    for (int sl = 0; sl < kBwdSlots; ++sl) {
      mbar_init(&bar.kv_full[sl], 1);
      mbar_init(&bar.kv_empty[sl], 1);
      mbar_init(&bar.kmn_full[sl], 1);
      mbar_init(&bar.kmn_empty[sl], 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&bar.sp_full[b], 1);
      mbar_init(&bar.elem_done[b], kElemThreads);
      mbar_init(&bar.st_free[b], 1);
    }
    mbar_init(&bar.dq_full, 1);
    mbar_init(&bar.dq_free, kElemThreads);
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
    // Q_i, dO_i of each item once its previous item's MMAs are done with
    // them; the two key rings refill independently, each as soon as its
    // slot is free (half tiles numbered across the CTA's items).
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmG);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmKmn);
      tma_prefetch_desc(&tmV);
      ItemSeq sq(nitems), sk(nitems), sm(nitems);
      int iq = sq.next(), nq = 0;                    // next item for Q / dO
      int ik = sk.next(), uk = 0, gk = 0;             // K / V ring: item, unit, global unit
      int im = sm.next(), um = 0, gm = 0;             // K MN-major ring
      PollGuard guard;
      while ((iq >= 0 || ik >= 0 || im >= 0) && !failed) {
        bool moved = false;
        // Q_i and dO_i replace the previous item's once its S and dP MMAs are
        // done and the element warps have read its dO for D (an item of two
        // half tiles can finish its MMAs before that)
        if (iq >= 0 && mbar_test(&bar.qd_empty, (nq & 1) ^ 1) &&
            (nq == 0 || mbar_test(&bar.d_read, (nq - 1) & 1))) {
          mbar_arrive_expect_tx(&bar.qd_full, 2 * kTile);
          for (int b = 0; b < D / 32; ++b) {
            tma_load_3d(sQ + b * 32 * KIA_TILE, &tmQ, &bar.qd_full, b * 32, item_qt(iq) * KIA_TILE,
                        item_bh(iq));
            tma_load_3d(sG + b * 32 * KIA_TILE, &tmG, &bar.qd_full, b * 32, item_qt(iq) * KIA_TILE,
                        item_bh(iq));
          }
          iq = sq.next();
          ++nq;
          moved = true;
        }
        if (ik >= 0) {
          const int sl = gk % NKV;
          if (mbar_test(&bar.kv_empty[sl], ((gk / NKV) & 1) ^ 1)) {
            uint8_t* dst = sKV + sl * kHalfPair;
            mbar_arrive_expect_tx(&bar.kv_full[sl], kHalfPair);
            for (int b = 0; b < D / 32; ++b) {
              tma_load_3d(dst + b * kHalfBlockBytes, &tmK, &bar.kv_full[sl], b * 32, 64 * uk,
                          item_bh(ik));
              tma_load_3d(dst + kHalfTile + b * kHalfBlockBytes, &tmV, &bar.kv_full[sl], b * 32,
                          64 * uk, item_bh(ik));
            }
            ++gk;
            if (++uk == item_units(ik)) { uk = 0; ik = sk.next(); }
            moved = true;
          }
        }
        if (im >= 0) {
          const int sl = gm % kKmnSlots;
          if (mbar_test(&bar.kmn_empty[sl], ((gm / kKmnSlots) & 1) ^ 1)) {
            uint8_t* dst = sKmn + sl * kHalfTile;
            mbar_arrive_expect_tx(&bar.kmn_full[sl], kHalfTile);
            for (int b = 0; b < D / 32; ++b)
              tma_load_3d(dst + b * kHalfBlockBytes, &tmKmn, &bar.kmn_full[sl], b * 32, 64 * um,
                          item_bh(im));
            ++gm;
            if (++um == item_units(im)) { um = 0; im = sm.next(); }
            moved = true;
          }
        }
        if (moved) guard.progress();
        else if (!guard.idle(abort)) failed = true;
      }
    }
  } else if (warp == kScoreWarp) {
    // ------------------------------------------------- score-MMA issuer
    // The whole warp runs the loop (warp-uniform waits and descriptor
    // arithmetic); one elected lane issues each unit's MMAs and commits.
    {
      const uint32_t id_s = idesc_tf32(128, 64, 0, 0);
      // descriptors built once; each MMA only adds a constant step
      const uint64_t dqa = desc_kmajor(smem_u32(sQ), 0), dga = desc_kmajor(smem_u32(sG), 0),
                     dkv = desc_kmajor_half(smem_u32(sKV));
      uint32_t sf_par = 0;                // per-region phase bits of the st_free waits
      int g = 0, n = 0;                   // global half tile, item count
      ItemSeq seq(nitems);
      for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
        if (!warp_wait(&bar.qd_full, n & 1, abort)) { failed = true; break; }
        // S, dP of half tile u (keys 64 u..) into region g % R, once the dQ
        // MMA of half tile g - R has released the region
        const int nunits = item_units(it);
        for (int u = 0; u < nunits; ++u, ++g) {
          const int r = g % R;
          if (g >= R) {
            if (!warp_wait(&bar.st_free[r], (sf_par >> r) & 1u, abort)) { failed = true; break; }
            sf_par ^= 1u << r;
          }
          const int sl = g % NKV;
          if (!warp_wait(&bar.kv_full[sl], (g / NKV) & 1, abort)) { failed = true; break; }
          const uint64_t dk = dkv + desc_step((uint32_t)sl * kHalfPair);   // K half, V half after it
          const uint64_t dv = dk + desc_step(kHalfTile);
          const uint32_t dst = tmem + 128u * r;
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < D / 8; ++ks)
              mma_tf32_ss(dst, dqa + kstep_kmajor(ks), dk + kstep_kmajor_half(ks), id_s, ks > 0);
#pragma unroll
            for (int ks = 0; ks < D / 8; ++ks)
              mma_tf32_ss(dst + 64u, dga + kstep_kmajor(ks), dv + kstep_kmajor_half(ks), id_s, ks > 0);
            tc_commit(&bar.sp_full[r]);
            tc_commit(&bar.kv_empty[sl]);
          }
          __syncwarp();
        }
        if (!failed) {
          if (elect_one()) tc_commit(&bar.qd_empty);   // Q_i, dO_i free once these MMAs are done
          __syncwarp();
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------- dQ-MMA issuer
    // (whole warp, one elected lane issuing)
    {
      const uint32_t id_dq = idesc_tf32(128, D, 0, 1);
      const uint64_t dkm = desc_mnmajor_half(smem_u32(sKmn));
      uint32_t ed_par = 0;                // per-region phase bits of the elem_done waits
      int g = 0, n = 0;
      ItemSeq seq(nitems);
      for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
        const int nunits = item_units(it);
        // dQ of half tile u: A = dS in region g % R, B = K half (MN-major)
        for (int u = 0; u < nunits; ++u, ++g) {
          const int r = g % R, sl = g % kKmnSlots;
          if (!warp_wait(&bar.elem_done[r], (ed_par >> r) & 1u, abort)) { failed = true; break; }
          ed_par ^= 1u << r;
          if (!warp_wait(&bar.kmn_full[sl], (g / kKmnSlots) & 1, abort)) { failed = true; break; }
          // the accumulator restarts with this item: the previous item's
          // epilogue must have read it
          if (u == 0 && n > 0 && !warp_wait(&bar.dq_free, (n - 1) & 1, abort)) { failed = true; break; }
          const uint64_t db = dkm + desc_step((uint32_t)sl * kHalfTile);
          const uint32_t pa = tmem + 128u * r;
          const uint32_t acc0 = u > 0 ? 1u : 0u;
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_tf32_ts(tmem + kColDQ, pa + 8u * kk, db + kstep_mnmajor(kk), id_dq,
                          kk > 0 ? 1u : acc0);
            tc_commit(&bar.st_free[r]);
            tc_commit(&bar.kmn_empty[sl]);
          }
          __syncwarp();
        }
        if (!failed) {
          if (elect_one()) tc_commit(&bar.dq_full);
          __syncwarp();
        }
      }
    }
  } else if (warp < kScoreWarp) {
    // ------------------------------------------------------ element warps
    const int quad = warp & 3;
    const int part = (warp - 2) >> 2;       // 0..3: columns 16 part .. +15 of every unit
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const float Kf = p.Kf, Km1f = (float)(p.K - 1);
    float2* sPair = reinterpret_cast<float2*>(sTab);
    if constexpr (!V::MINMAX && !V::SOFTMAX) {
      // pairs k = 0..K-1 and the tail's zero pair at K
      for (int k = (int)threadIdx.x - 64; k <= p.K; k += kElemThreads)
        sPair[k] = k < p.K ? make_float2(st.table[k], st.table[k + 1]) : make_float2(0.0f, 0.0f);
    }
    // An item's prologue operands from global memory: this row's
    // calibration (written by the forward), and a quarter of a row of O_bar
    // (O, or O_L for Prob-STE) for the centering D = dO . O_bar, which four
    // consecutive element threads form for one row, with dO from the item's
    // tile in shared memory, and add by shuffles.  They are loaded during the
    // previous item's epilogue, so that their DRAM latency passes during its
    // stores.
    const int e = (int)threadIdx.x - 64;
    const int rr = e >> 2, cc = e & 3;         // row of the tile, quarter of the row
    struct Pro {
      float m, rh, Wb;
      int am, an;
      float4 ob[D / 16];
    };
    auto load_pro = [&](int it, Pro& x) {
      const long long rb = (long long)item_bh(it) * T;
      const int q = item_qt(it) * KIA_TILE + r, qq = item_qt(it) * KIA_TILE + rr;
      const long long qr = rb + (q < T ? q : T - 1), qrr = rb + (qq < T ? qq : T - 1);
      x.m = st.m[qr];
      x.am = st.am[qr];
      x.an = V::MINMAX ? st.an[qr] : x.am;
      x.rh = st.rh[qr];
      x.Wb = st.Wb[qr];
      const float4* o4 =
          reinterpret_cast<const float4*>((V::PROB ? st.OL : O) + qrr * D) + cc * (D / 16);
#pragma unroll
      for (int c = 0; c < D / 16; ++c) x.ob[c] = o4[c];
    };
    Pro pro;
    int gbase = 0, n = 0;
    ItemSeq seq(nitems);
    int it0 = seq.next();
    if (it0 >= 0) load_pro(it0, pro);
    for (int it = it0; it >= 0 && !failed; it = seq.next(), ++n) {
      const int qt = item_qt(it), bh = item_bh(it), nunits = item_units(it);
      const int q = qt * KIA_TILE + r;
      const long long rowbase = (long long)bh * T;
      const long long qr = rowbase + (q < T ? q : T - 1);
      const float m = pro.m;
      const int am = pro.am, an = pro.an;
      const float rh = pro.rh;
      const float Wb = pro.Wb;
      const int qq = qt * KIA_TILE + rr;
      const long long qrr = rowbase + (qq < T ? qq : T - 1);
      // a degenerate MinMax row (1/h = 0) has dS = dw: with its grid in shared
      // memory through the copy patched to G_1 = 2 (below) and the factor 1,
      // else through dg
      const bool fold = V::MINMAX && tab_in_smem && rh == 0.0f;
      const float nrh = fold ? 1.0f : -rh;
      const float dg = (V::MINMAX && !tab_in_smem && rh == 0.0f) ? 1.0f : 0.0f;
      const int L = p.causal ? q + 1 : T;
      // a one-key row has P = 1 whatever its score: zero gradient
      const float rWb = (L == 1) ? 0.0f : __fdiv_rn(1.0f, Wb);
      // the key rows this row's epilogue gathers (argmax, argmin) into L2 now
      prefetch_l2(Kt + (rowbase + am) * D + part * (D / kRowSplit));
      if constexpr (V::MINMAX) prefetch_l2(Kt + (rowbase + an) * D + part * (D / kRowSplit));
      {
        // dO_i's row rr, columns 16 cc .. 16 cc + 15: column block cc / 2 of
        // the tile, 16-byte chunks (cc % 2) 4 + c, stored at chunk position
        // chunk ^ (row % 8) of the row's 128 bytes (the 128-byte swizzle)
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.qd_full, n & 1, abort))) { failed = true; break; }
        const uint8_t* grow = reinterpret_cast<const uint8_t*>(sG) + (cc >> 1) * (KIA_TILE * 128) + rr * 128;
        float acc = 0.0f;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          const float4 ga = *reinterpret_cast<const float4*>(grow + ((((cc & 1) * 4 + c) ^ (rr & 7)) * 16));
          acc = fmaf(ga.x, pro.ob[c].x, acc);
          acc = fmaf(ga.y, pro.ob[c].y, acc);
          acc = fmaf(ga.z, pro.ob[c].z, acc);
          acc = fmaf(ga.w, pro.ob[c].w, acc);
        }
        mbar_arrive(&bar.d_read);
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (cc == 0) {
          sDc[rr] = acc;
          if (qq < T) wk.D[qrr] = acc;
        }
      }
      if constexpr (V::MINMAX) {
        if (tab_in_smem)
          for (int k = part; k <= p.K; k += kRowSplit)
            sTab[k * KIA_TILE + r] = (fold && k == 1) ? 2.0f : st.table[qr * (p.K + 1) + k];
      }
      mbar_arrive(&bar.row_sync);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, (2 * n) & 1, abort))) { failed = true; break; }
      const float Dc = sDc[r];
      const float nDr = -Dc * rWb;            // dw = (dP - D) / W_bar as one fma
      float A = 0.0f, C = 0.0f;
      // the unit loop, instantiated per grid placement so that the grid
      // loads of the element loop are shared-memory loads when the grid is
      // in shared memory (a runtime choice of pointer makes them generic)
      auto unit_loop = [&](const auto& grid, auto fold_c) {
      constexpr bool FOLD = decltype(fold_c)::value;
      for (int u = 0; u < nunits && !failed; ++u) {
        const int j = u >> 1, gu = gbase + u, rg = gu % R;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.sp_full[rg], (gu / R) & 1, abort))) { failed = true; break; }
        tc_fence_after();
        const bool edge = (p.causal && j == qt) || (j + 1) * KIA_TILE > T;
        {
          float v[16], g[16];
          const uint32_t cs = 128u * rg + 16u * part;    // this thread's 16 columns of S
          tmem_ld16(tmem + lane_addr + cs, v);
          tmem_ld16(tmem + lane_addr + cs + 64u, g);
          tmem_ld_wait_regs(v, g);
          const int key0 = 64 * u + 16 * part;
          if (!edge) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float dw = fmaf(g[i], rWb, nDr);
              v[i] = bwd_delta<V, NEED_C, FOLD>(grid, m, rh, nrh, dg, Kf, Km1f, v[i], dw, A, C);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int key = key0 + i;
              const bool ok = key < T && (!p.causal || key <= q);
              const float dw = ok ? fmaf(g[i], rWb, nDr) : 0.0f;
              v[i] = bwd_delta<V, NEED_C, FOLD>(grid, m, rh, nrh, dg, Kf, Km1f, v[i], dw, A, C);
            }
          }
          tmem_st16(tmem + lane_addr + cs, v);
          if (dS_dbg && q < T) {
            float* dst = dS_dbg + (rowbase + q) * T + key0;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (key0 + i < T) dst[i] = v[i];
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar.elem_done[rg]);
      }
      };
      if constexpr (V::MINMAX) {
        if (tab_in_smem) unit_loop(GridF{sTab + r, KIA_TILE}, std::true_type{});
        else unit_loop(GridF{st.table + qr * (p.K + 1), 1}, std::false_type{});
      } else if constexpr (V::SOFTMAX) {
        unit_loop(GridP{sPair}, std::false_type{});
      } else {
        unit_loop(make_gridz(sPair, p.K), std::false_type{});
      }
      if (failed) break;
      gbase += nunits;
      // this thread's columns of the key rows of the row's calibration terms
      // (argmax, argmin), loaded now so that their latency passes during the
      // waits below
      constexpr int kCols = D / kRowSplit;   // 16
      const uint32_t col = (uint32_t)(part * kCols);
      float4 ka4[kCols / 4], kn4[V::MINMAX ? kCols / 4 : 1];
      {
        const float4* k4 = reinterpret_cast<const float4*>(Kt + (rowbase + am) * D + col);
#pragma unroll
        for (int i = 0; i < kCols / 4; ++i) ka4[i] = k4[i];
        if constexpr (V::MINMAX) {
          const float4* n4 = reinterpret_cast<const float4*>(Kt + (rowbase + an) * D + col);
#pragma unroll
          for (int i = 0; i < kCols / 4; ++i) kn4[i] = n4[i];
        }
      }
      // row sums of the four column groups
      sAC[(part * 2 + 0) * KIA_TILE + r] = A;
      sAC[(part * 2 + 1) * KIA_TILE + r] = C;
      mbar_arrive(&bar.row_sync);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, (2 * n + 1) & 1, abort))) { failed = true; break; }
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.dq_full, n & 1, abort))) { failed = true; break; }
      tc_fence_after();
      // this thread's 16 columns of dQ, then the accumulator is free for the
      // next item
      float o[kCols];
      tmem_ld16(tmem + lane_addr + kColDQ + col, o);
      tmem_ld_wait_regs(o);
      tc_fence_before();
      mbar_arrive(&bar.dq_free);
      // calibration terms of this row (section 3, Calibration gradients;
      // Appendix B): dS gains g_m at the argmax key and g_n at the argmin key
      const float Arow = (sAC[0 * KIA_TILE + r] + sAC[2 * KIA_TILE + r]) +
                         (sAC[4 * KIA_TILE + r] + sAC[6 * KIA_TILE + r]);
      const float Crow = (sAC[1 * KIA_TILE + r] + sAC[3 * KIA_TILE + r]) +
                         (sAC[5 * KIA_TILE + r] + sAC[7 * KIA_TILE + r]);
      float gm, gn;
      calibration_coeffs(p, Arow, Crow, rh, L, gm, gn);
      const bool proj = p.grad == KIA_GRAD_PROJECT;
      const float gmq = proj ? 0.0f : gm;   // the projection shift is applied by the scan pass
      if (q < T) {
        if (gmq != 0.0f) {
#pragma unroll
          for (int i = 0; i < kCols / 4; ++i) {
            const float4 kk = ka4[i];
            o[4 * i] = fmaf(gmq, kk.x, o[4 * i]);
            o[4 * i + 1] = fmaf(gmq, kk.y, o[4 * i + 1]);
            o[4 * i + 2] = fmaf(gmq, kk.z, o[4 * i + 2]);
            o[4 * i + 3] = fmaf(gmq, kk.w, o[4 * i + 3]);
          }
        }
        if (V::MINMAX && gn != 0.0f) {
#pragma unroll
          for (int i = 0; i < kCols / 4; ++i) {
            const float4 kk = kn4[V::MINMAX ? i : 0];
            o[4 * i] = fmaf(gn, kk.x, o[4 * i]);
            o[4 * i + 1] = fmaf(gn, kk.y, o[4 * i + 1]);
            o[4 * i + 2] = fmaf(gn, kk.z, o[4 * i + 2]);
            o[4 * i + 3] = fmaf(gn, kk.w, o[4 * i + 3]);
          }
        }
      }
      // this warp's 32 rows x 16 columns of dQ, 8 columns per TMA store
      // through its staging block
      {
        float* stg = sStage + (warp - 2) * 256;
        const int row0 = qt * KIA_TILE + quad * 32;
        epilogue_store8(stg, &tmdQ, o, 1.0f, lane, (int)col, row0, bh);
        {
          // the next item's prologue operands: issued between the two
          // stores (their latency passes during the second and the next
          // item's start)
          ItemSeq peek = seq;
          const int nx = peek.next();
          if (nx >= 0) {
            load_pro(nx, pro);
            if constexpr (V::MINMAX) {
              // and its rows of the grid table into L2 (copied in its prologue)
              const int qn = item_qt(nx) * KIA_TILE + r;
              if (tab_in_smem && part == 0)
                prefetch_l2(st.table + ((long long)item_bh(nx) * T + (qn < T ? qn : T - 1)) * (p.K + 1));
            }
          }
        }
        epilogue_store8(stg, &tmdQ, o + 8, 1.0f, lane, (int)col + 8, row0, bh);
      }
      if (q < T && part == 0) {
        wk.gm[rowbase + q] = gm;
        wk.gn[rowbase + q] = gn;
        wk.am[rowbase + q] = am;
        wk.an[rowbase + q] = an;
        if (dS_dbg) {
          float* ds = dS_dbg + (rowbase + q) * T;
          if (proj) {
            for (int jj = 0; jj < L; ++jj) ds[jj] += gm;
          } else {
            ds[am] += gm;
            ds[an] += gn;
          }
        }
      }
    }
    epilogue_store_drain();
  }
  if (failed || *abort) drain_in_flight();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ key pass

template <int D, class V, bool PROJ>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQmn,
                 const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmGmn,
                 const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                 StatsView st, WorkView wk, OpParams p, int BH, int T, int tab_in_smem,
                 int nmn) {
  static_assert(D == 64, "tensor-core backward tiles are laid out for d = 64");
  constexpr uint32_t kTile = D * KIA_TILE * 4;
  if (*wk.status != 0) return;
  extern __shared__ uint8_t smraw[];
  uint8_t* base = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
  // K_j and V_j stay for an item; the queries stream through two rings of
  // half tiles (64 queries): Q and dO K-major (for S^T, dP^T) and Q and dO
  // MN-major (for dK, dV), two slots each.
  float* sK = reinterpret_cast<float*>(base);
  float* sV = reinterpret_cast<float*>(base + kTile);
  uint8_t* sQD = base + 2 * kTile;                            // [2][Q half | dO half]
  // the MN-major ring has kKvSlots slots, one when a MinMax grid table needs
  // the room (only the producer and the dV / dK issuer use it); it sits last
  // in shared memory (below), so that its depth moves no other buffer
  const int NMN = V::MINMAX ? nmn : kKvSlots;   // a constant for the other variants
  // Per-query constants of a unit (64 queries) in kSlots slots (four, or two
  // under MinMax, whose slots also hold the queries' grids), filled ahead of
  // the element warps by the constant warp: half tile g (numbered across the
  // CTA's items) uses slot g % kSlots.
  // sC4 = (m, k1, k0, 1/W_fwd): the score-gradient factor -dw/h = dP k1 + k0
  // (softmax: dw itself); sX4 (MinMax or projection) = (1/h, the degenerate
  // row's dw = dP x.y + x.z, 0 elsewhere, the projection shift c)
  constexpr int kSlots = kv_const_slots<V>(), kSlotQ = 64;
  float4* sC4 = reinterpret_cast<float4*>(sQD + kKvSlots * kHalfPair);
  float4* sX4 = sC4 + kSlots * kSlotQ;
  // calibration terms, read only where a query's argmax (argmin) key lies in
  // a warp's 32 keys: (key - tile start, coefficient bits)
  int2* sCM = reinterpret_cast<int2*>(sX4 + kSlots * kSlotQ);   // argmax key, g_m
  int2* sCN = sCM + kSlots * kSlotQ;                            // argmin key, g_n
  // which queries of a unit have their argmax (argmin) key in lanes
  // 32 quad..32 quad + 31: [slot][argmax / argmin][quad][query half]
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sCN + kSlots * kSlotQ);
  // epilogue: 1 KB per element warp to turn its rows into full-sector stores
  float* sStage = reinterpret_cast<float*>(sMask + kSlots * 2 * 4 * 2);   // [16 warps][32][8]
  float* sTab = sStage + kElemThreads / 32 * 256;   // [slot][64][K + 1]
  const int K1 = p.K + 1;
  const int tab_floats = V::SOFTMAX ? 0 : (V::MINMAX ? (tab_in_smem ? kSlots * kSlotQ * K1 : 0) : 4 * K1);
  BwdKBars& bar = *reinterpret_cast<BwdKBars*>(sTab + ((tab_floats + 31) & ~31));
  uint8_t* sQDmn =    // [NMN][Q half | dO half], MN-major, 1024-aligned
      base + ((reinterpret_cast<uint8_t*>(&bar + 1) - base + 1023) & ~(ptrdiff_t)1023);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int nitems = BH * nt;
  // item it -> (key tile, batch*head), heaviest causal tiles (most queries)
  // first; this CTA takes its items in the serpentine order of ItemSeq
  auto item_kt = [&](int it) { return it / BH; };
  auto item_bh = [&](int it) { return it % BH; };
  auto item_q0 = [&](int it) { return p.causal ? item_kt(it) : 0; };
  auto item_units = [&](int it) { return 2 * (nt - item_q0(it)); };
  constexpr int R = kBwdRegions;
  constexpr uint32_t kColDV = 128u * R, kColDK = kColDV + D;

  if (threadIdx.x == 0) {
    mbar_init(&bar.kv_full, 1);
    mbar_init(&bar.kv_empty, 1);
    for (int sl = 0; sl < kKvSlots; ++sl) {
      mbar_init(&bar.qd_full[sl], 1);
      mbar_init(&bar.qd_empty[sl], 1);
      mbar_init(&bar.mn_full[sl], 1);
      mbar_init(&bar.mn_empty[sl], 1);
    }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&bar.sp_full[b], 1);
      mbar_init(&bar.elem_done[b], kElemThreads);
      mbar_init(&bar.st_free[b], 1);
    }
    for (int sl = 0; sl < 4; ++sl) {
      mbar_init(&bar.qc_ready[sl], 32);
      mbar_init(&bar.qc_free[sl], kElemThreads);
    }
    mbar_init(&bar.acc_full, 1);
    mbar_init(&bar.acc_free, kElemThreads);
    mbar_init(&bar.acc_issued, 1);
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
    // K_j, V_j of each item once the previous item's MMAs are done with
    // them; the two query rings refill independently, each as soon as its
    // slot is free (half tiles numbered across the CTA's items).
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmQmn);
      tma_prefetch_desc(&tmG);
      tma_prefetch_desc(&tmGmn);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      ItemSeq skv(nitems), sq(nitems), sm(nitems);
      int ikv = skv.next(), nkv = 0;                 // next item for K / V
      int iq = sq.next(), uq = 0, gq = 0;             // K-major ring: item, unit, global unit
      int im = sm.next(), um = 0, gm = 0;             // MN-major ring
      PollGuard guard;
      while ((ikv >= 0 || iq >= 0 || im >= 0) && !failed) {
        bool moved = false;
        if (ikv >= 0 && mbar_test(&bar.kv_empty, (nkv & 1) ^ 1)) {
          mbar_arrive_expect_tx(&bar.kv_full, 2 * kTile);
          for (int b = 0; b < D / 32; ++b) {
            tma_load_3d(sK + b * 32 * KIA_TILE, &tmK, &bar.kv_full, b * 32, item_kt(ikv) * KIA_TILE,
                        item_bh(ikv));
            tma_load_3d(sV + b * 32 * KIA_TILE, &tmV, &bar.kv_full, b * 32, item_kt(ikv) * KIA_TILE,
                        item_bh(ikv));
          }
          ikv = skv.next();
          ++nkv;
          moved = true;
        }
        if (iq >= 0) {
          const int sl = gq % kKvSlots;
          if (mbar_test(&bar.qd_empty[sl], ((gq / kKvSlots) & 1) ^ 1)) {
            uint8_t* dst = sQD + sl * kHalfPair;
            const int row = 64 * (2 * item_q0(iq) + uq);
            mbar_arrive_expect_tx(&bar.qd_full[sl], kHalfPair);
            for (int b = 0; b < D / 32; ++b) {
              tma_load_3d(dst + b * kHalfBlockBytes, &tmQ, &bar.qd_full[sl], b * 32, row, item_bh(iq));
              tma_load_3d(dst + kHalfTile + b * kHalfBlockBytes, &tmG, &bar.qd_full[sl], b * 32,
                          row, item_bh(iq));
            }
            ++gq;
            if (++uq == item_units(iq)) { uq = 0; iq = sq.next(); }
            moved = true;
          }
        }
        if (im >= 0) {
          const int sl = gm % NMN;
          if (mbar_test(&bar.mn_empty[sl], ((gm / NMN) & 1) ^ 1)) {
            uint8_t* dst = sQDmn + sl * kHalfPair;
            const int row = 64 * (2 * item_q0(im) + um);
            mbar_arrive_expect_tx(&bar.mn_full[sl], kHalfPair);
            for (int b = 0; b < D / 32; ++b) {
              tma_load_3d(dst + b * kHalfBlockBytes, &tmQmn, &bar.mn_full[sl], b * 32, row,
                          item_bh(im));
              tma_load_3d(dst + kHalfTile + b * kHalfBlockBytes, &tmGmn, &bar.mn_full[sl], b * 32,
                          row, item_bh(im));
            }
            ++gm;
            if (++um == item_units(im)) { um = 0; im = sm.next(); }
            moved = true;
          }
        }
        if (moved) guard.progress();
        else if (!guard.idle(abort)) failed = true;
      }
    }
  } else if (warp == kScoreWarp) {
    // ------------------------------------------------- score-MMA issuer
    // (whole warp, one elected lane issuing)
    {
      const uint32_t id_s = idesc_tf32(128, 64, 0, 0);
      // descriptors built once; each MMA only adds a constant step
      const uint64_t dka = desc_kmajor(smem_u32(sK), 0), dva = desc_kmajor(smem_u32(sV), 0),
                     dqd = desc_kmajor_half(smem_u32(sQD));
      uint32_t sf_par = 0;                // per-region phase bits of the st_free waits
      int g = 0, n = 0;
      ItemSeq seq(nitems);
      for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
        if (!warp_wait(&bar.kv_full, n & 1, abort)) { failed = true; break; }
        // the previous item's last dV / dK MMAs go into the tensor pipe ahead
        // of this item's: the element warps wait for them before their
        // epilogue, while this item's first scores can wait
        if (n > 0 && !warp_wait(&bar.acc_issued, (n - 1) & 1, abort)) { failed = true; break; }
        // S^T, dP^T of half tile u (queries 64 (2 q0 + u)..) into region
        // g % R, once the dV / dK MMAs of half tile g - R have released it
        const int nunits = item_units(it);
        for (int u = 0; u < nunits; ++u, ++g) {
          const int r = g % R, sl = g % kKvSlots;
          if (g >= R) {
            if (!warp_wait(&bar.st_free[r], (sf_par >> r) & 1u, abort)) { failed = true; break; }
            sf_par ^= 1u << r;
          }
          if (!warp_wait(&bar.qd_full[sl], (g / kKvSlots) & 1, abort)) { failed = true; break; }
          const uint64_t dq = dqd + desc_step((uint32_t)sl * kHalfPair);   // Q half, dO half after it
          const uint64_t dg = dq + desc_step(kHalfTile);
          const uint32_t dst = tmem + 128u * r;
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < D / 8; ++ks)
              mma_tf32_ss(dst, dka + kstep_kmajor(ks), dq + kstep_kmajor_half(ks), id_s, ks > 0);
#pragma unroll
            for (int ks = 0; ks < D / 8; ++ks)
              mma_tf32_ss(dst + 64u, dva + kstep_kmajor(ks), dg + kstep_kmajor_half(ks), id_s, ks > 0);
            tc_commit(&bar.sp_full[r]);
            tc_commit(&bar.qd_empty[sl]);
          }
          __syncwarp();
        }
        if (!failed) {
          if (elect_one()) tc_commit(&bar.kv_empty);   // K_j, V_j free once these MMAs are done
          __syncwarp();
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------- dV / dK-MMA issuer
    // (whole warp, one elected lane issuing)
    {
      const uint32_t id_acc = idesc_tf32(128, D, 0, 1);
      const uint64_t dmn = desc_mnmajor_half(smem_u32(sQDmn));
      uint32_t ed_par = 0;                // per-region phase bits of the elem_done waits
      int g = 0, n = 0;
      ItemSeq seq(nitems);
      for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
        const int nunits = item_units(it);
        // dV += P^T dO, dK += dS^T Q for half tile u (A operands in region g % R)
        for (int u = 0; u < nunits; ++u, ++g) {
          const int r = g % R, sl = g % NMN;
          if (!warp_wait(&bar.elem_done[r], (ed_par >> r) & 1u, abort)) { failed = true; break; }
          ed_par ^= 1u << r;
          if (!warp_wait(&bar.mn_full[sl], (g / NMN) & 1, abort)) { failed = true; break; }
          // the accumulators restart with this item: the previous item's
          // epilogue must have read them
          if (u == 0 && n > 0 && !warp_wait(&bar.acc_free, (n - 1) & 1, abort)) { failed = true; break; }
          const uint64_t dqm = dmn + desc_step((uint32_t)sl * kHalfPair);   // Q half, dO half after it
          const uint64_t dgm = dqm + desc_step(kHalfTile);
          const uint32_t pa = tmem + 128u * r;
          const uint32_t acc0 = u > 0 ? 1u : 0u;
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_tf32_ts(tmem + kColDV, pa + 8u * kk, dgm + kstep_mnmajor(kk), id_acc,
                          kk > 0 ? 1u : acc0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_tf32_ts(tmem + kColDK, pa + 64u + 8u * kk, dqm + kstep_mnmajor(kk), id_acc,
                          kk > 0 ? 1u : acc0);
            tc_commit(&bar.st_free[r]);
            tc_commit(&bar.mn_empty[sl]);
          }
          __syncwarp();
        }
        if (!failed) {
          if (elect_one()) {
            tc_commit(&bar.acc_full);
            mbar_arrive(&bar.acc_issued);
          }
          __syncwarp();
        }
      }
    }
  } else if (warp == kScoreWarp + 1) {
    // -------------------------------------------- query-constant producer
    // Loads the per-query constants of each unit into its slot while the
    // element warps work on earlier units (lane l: queries l and l + 32).
    // FWM: each group's copy of the shared grid's pairs, published with the
    // first units' constants
    if (!V::SOFTMAX && !V::MINMAX) {
      // pairs k = 0..K-1, then a zero pair at K: the target of tail keys
      for (int k = lane; k <= p.K; k += 32) {
        const float2 pr = k < p.K ? make_float2(st.table[k], st.table[k + 1]) : make_float2(0.0f, 0.0f);
        reinterpret_cast<float2*>(sTab)[k] = pr;
        reinterpret_cast<float2*>(sTab)[K1 + k] = pr;
      }
    }
    // raw per-query values of one unit (lane l: queries l and l + 32), loaded
    // one unit ahead so that their latency overlaps the wait for a free slot
    struct Raw {
      float m[2], rh[2], dl[2], Wb[2], Wf[2], gm[2], gn[2];   // dl: the row's D
      int am[2], an[2];
    };
    auto load_raw = [&](int it, int u, Raw& x) {
      const long long rowbase = (long long)item_bh(it) * T;
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        const int q = 64 * (2 * item_q0(it) + u) + 32 * hq + lane;
        const long long qr = rowbase + (q < T ? q : T - 1);
        x.m[hq] = st.m[qr];
        x.rh[hq] = st.rh[qr];
        x.dl[hq] = wk.D[qr];
        x.Wb[hq] = st.Wb[qr];
        x.Wf[hq] = st.Wf[qr];
        x.gm[hq] = wk.gm[qr];
        x.gn[hq] = V::MINMAX ? wk.gn[qr] : 0.0f;
        x.am[hq] = PROJ ? 0 : wk.am[qr];
        x.an[hq] = (V::MINMAX && !PROJ) ? wk.an[qr] : 0;
      }
    };
    Raw cur;
    ItemSeq cseq(nitems);
    int it = cseq.next(), u = 0;
    if (it >= 0) load_raw(it, 0, cur);
    for (int g = 0; it >= 0 && !failed; ++g) {
      const int sl = g % kSlots;
      // the next half tile (possibly of the next item)
      int it2 = it, u2 = u + 1;
      if (u2 == item_units(it)) { u2 = 0; it2 = cseq.next(); }
      Raw nxt;
      if (it2 >= 0) load_raw(it2, u2, nxt);
      if (g >= kSlots && !__all_sync(0xffffffffu, mbar_wait(&bar.qc_free[sl], ((g / kSlots) - 1) & 1, abort))) {
        failed = true;
        break;
      }
      const int kt = item_kt(it);
      const long long rowbase = (long long)item_bh(it) * T;
      if (V::MINMAX && tab_in_smem) {
        // the unit's 64 per-query grids are consecutive rows of the stats
        // table: asynchronous copies into the slot, issued before the
        // constants below so that their latency passes meanwhile (rows past
        // T are filled with ones; their queries are masked)
        const int qf = 64 * (2 * item_q0(it) + u);
        const int nvalid = max(0, min(kSlotQ, T - qf)) * K1, ntot = kSlotQ * K1;
        const float* src = st.table + (rowbase + qf) * K1;
        float* dst = sTab + (size_t)sl * kSlotQ * K1;
        for (int x = lane; x < ntot; x += 32) {
          if (x < nvalid) cp_async4(dst + x, src + x);
          else dst[x] = 1.0f;
        }
      }
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        const int q = 64 * (2 * item_q0(it) + u) + 32 * hq + lane;
        const int e = sl * kSlotQ + 32 * hq + lane;          // its slot entry
        const int Lq = p.causal ? q + 1 : T;
        const float rWb = Lq == 1 ? 0.0f : __fdiv_rn(1.0f, cur.Wb[hq]);
        const float nD = -cur.dl[hq] * rWb;       // dw = dP rWb + nD
        // a degenerate MinMax row (1/h = 0) has dS = dw (uniform P): with its
        // grid in shared memory that comes through the slope of a patched
        // grid (below) and the factor 1 here, else through x.y, x.z
        const bool fold = V::MINMAX && tab_in_smem && cur.rh[hq] == 0.0f;
        const float nrh = (V::SOFTMAX || fold) ? 1.0f : -cur.rh[hq];
        sC4[e] = make_float4(cur.m[hq], rWb * nrh, nD * nrh, __fdiv_rn(1.0f, cur.Wf[hq]));
        // calibration terms of the query's row, added to dS^T before dK:
        // g_m at the argmax key, g_n at the argmin key, or the projection
        // shift c on every visible key
        const bool live = q < T;
        const float gm = live ? cur.gm[hq] : 0.0f, gn = live ? cur.gn[hq] : 0.0f;
        if constexpr (V::MINMAX || PROJ) {
          const float dg = (V::MINMAX && !tab_in_smem && cur.rh[hq] == 0.0f) ? 1.0f : 0.0f;
          sX4[e] = make_float4(cur.rh[hq], dg * rWb, dg * nD, PROJ ? gm : 0.0f);
        }
        if constexpr (!PROJ && !V::SOFTMAX) {
          const int ka = cur.am[hq] - kt * KIA_TILE;
          const int kn = V::MINMAX ? cur.an[hq] - kt * KIA_TILE : -1;
          sCM[e] = make_int2(ka, __float_as_int(gm));
          sCN[e] = make_int2(kn, __float_as_int(gn));
          const bool hit_m = gm != 0.0f && ka >= 0 && ka < KIA_TILE;
          const bool hit_n = V::MINMAX && gn != 0.0f && kn >= 0 && kn < KIA_TILE;
#pragma unroll
          for (int qd = 0; qd < 4; ++qd) {
            const uint32_t bm = __ballot_sync(0xffffffffu, hit_m && (ka >> 5) == qd);
            const uint32_t bn = __ballot_sync(0xffffffffu, hit_n && (kn >> 5) == qd);
            if (lane == 0) {
              sMask[((sl * 2 + 0) * 4 + qd) * 2 + hq] = bm;
              sMask[((sl * 2 + 1) * 4 + qd) * 2 + hq] = bn;
            }
          }
        }
      }
      if (V::MINMAX && tab_in_smem) cp_async_wait_all();   // the unit's grids have landed
      __syncwarp();
      if (V::MINMAX && tab_in_smem) {
        // a degenerate row's grid gets G_1 = 2 in the slot: its scores all sit
        // at node 0 (u = 0), so the slope G_1 - G_0 = 1 makes the score
        // gradient dw; its weight G_0 = 1 is unchanged
#pragma unroll
        for (int hq = 0; hq < 2; ++hq)
          if (cur.rh[hq] == 0.0f) sTab[(size_t)(sl * kSlotQ + 32 * hq + lane) * K1 + 1] = 2.0f;
        __syncwarp();
      }
      mbar_arrive(&bar.qc_ready[sl]);
      cur = nxt;
      it = it2;
      u = u2;
    }
  } else if (warp < kScoreWarp) {
    // ------------------------------------------------------ element warps
    const int quad = warp & 3;
    const int part = (warp - 2) >> 2;        // 0..3: query columns 16 part .. +15 of every unit
    const int grp = part >> 1;               // which copy of the FWM grid pairs this warp reads
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const float Kf = p.Kf, Km1f = (float)(p.K - 1);
    // FWM: each group keeps its own copy of the shared grid's pairs, with a
    // zero pair at index K that tail keys are pointed at; a pair is fetched
    // by its address computed from the floor trick's bits directly
    const float2* sPairG = reinterpret_cast<const float2*>(sTab) + grp * K1;
    const GridZ gridz = make_gridz(sPairG, p.K);
    const float rh_c = p.fwm_rh;
    int gbase = 0, n = 0;
    ItemSeq seq(nitems);
    for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
      const int kt = item_kt(it), q0 = item_q0(it), nunits = item_units(it);
      const int kj = kt * KIA_TILE + r;
      const long long rowbase = (long long)item_bh(it) * T;
      for (int u = 0; u < nunits && !failed; ++u) {
        const int gu = gbase + u;
        const int qi = q0 + (u >> 1);
        const int rg = gu % R;
        const int sl = gu % kSlots;                          // this unit's constant slot
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.qc_ready[sl], (gu / kSlots) & 1, abort))) { failed = true; break; }
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.sp_full[rg], (gu / R) & 1, abort))) { failed = true; break; }
        tc_fence_after();
        const bool edge =
            (p.causal && qi == kt) || (qi + 1) * KIA_TILE > T || (kt + 1) * KIA_TILE > T;
        {
          float v[16], g[16];
          const uint32_t cs = 128u * rg + 16u * part;        // this thread's 16 query columns
          tmem_ld16(tmem + lane_addr + cs, v);
          tmem_ld16(tmem + lane_addr + cs + 64u, g);
          tmem_ld_wait_regs(v, g);
          const int ql0 = 64 * (u & 1) + 16 * part;   // first query (in the tile) of the chunk
          const int e0 = sl * kSlotQ + 16 * part;     // its slot entry
          // the element loop, one body for every unit; the masked pairs of an
          // edge unit are zeroed afterwards (their scores are finite, so the
          // body's clamped grid index stays inside the table)
          auto body = [&](auto tabs_c) {
            [[maybe_unused]] constexpr bool TABS = decltype(tabs_c)::value;   // per-query grids in shared memory
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              [[maybe_unused]] const int ql = ql0 + i;
              const float4 cq = sC4[e0 + i];
              float4 xq = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              if constexpr (V::MINMAX || PROJ) xq = sX4[e0 + i];
              const float s = v[i], dP = g[i];
              const float dSn = fmaf(dP, cq.y, cq.z);        // -dw / h  (softmax: dw)
              float P, dS;
              if constexpr (V::SOFTMAX) {
                const float w = expf(s - cq.x);
                P = round_exp<V::EXPR>(w) * cq.w;   // the forward's (rounded) probability
                dS = w * dSn;                       // straight through the rounding
              } else {
                const float rh = V::MINMAX ? xq.x : rh_c;
                float u = __fmul_rn(__fsub_rn(cq.x, s), rh);
                if constexpr (V::MINMAX) u = fminf(u, Kf);
                const float uc = fmaxf(fminf(u, Km1f), 0.0f);
                const float tmp = __fadd_rd(uc, kMagic);
                const float t = __fsub_rn(u, __fsub_rn(tmp, kMagic));
                float2 gp;
                if constexpr (V::MINMAX) {
                  const float* gq;
                  if constexpr (TABS) gq = sTab + (e0 + i) * K1;
                  else gq = st.table + (rowbase + min(qi * KIA_TILE + ql, T - 1)) * K1;
                  gp = GridF{gq, 1}.pair(__float_as_int(tmp) - kMagicBits);
                } else {
                  // FWM tail (u > K): the zero pair, so P = 0 and dS = 0
                  gp = gridz.at(__float_as_int(tmp) - kMagicBits, u > Kf);
                }
                const float a = __fsub_rn(gp.y, gp.x);
                const float wf = V::NEAREST ? (t >= 0.5f ? gp.y : gp.x) : __fmaf_rn(t, a, gp.x);
                P = wf * cq.w;
                dS = a * dSn;
                if constexpr (V::MINMAX && !TABS) dS = fmaf(dP, xq.y, dS + xq.z);   // degenerate rows: dw
              }
              if constexpr (PROJ) dS += xq.w;
              v[i] = P;
              g[i] = dS;
            }
          };
          if constexpr (V::MINMAX) {
            if (tab_in_smem) body(std::true_type{});
            else body(std::false_type{});
          } else {
            body(std::true_type{});
          }
          if (edge) {
            // future keys, and rows or keys past T: no weight, no gradient
            const uint32_t vis = visible16(kj, qi * KIA_TILE + ql0, T, p.causal != 0);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const bool keep = (vis >> i) & 1u;
              v[i] = keep ? v[i] : 0.0f;
              g[i] = keep ? g[i] : 0.0f;
            }
          }
          if constexpr (!PROJ && !V::SOFTMAX) {
            // the chunk's queries whose argmax (argmin) key lies in this warp's
            // 32 keys (visible pairs: the edge zeroing above never meets
            // them); the masks pass through lane 0 so that the compiler sees
            // them as warp-uniform
            const int hq = part >> 1, sh = 16 * (part & 1);
            const uint32_t bm =
                __shfl_sync(0xffffffffu, (sMask[((sl * 2 + 0) * 4 + quad) * 2 + hq] >> sh) & 0xFFFFu, 0);
            const uint32_t bn = V::MINMAX
                ? __shfl_sync(0xffffffffu, (sMask[((sl * 2 + 1) * 4 + quad) * 2 + hq] >> sh) & 0xFFFFu, 0)
                : 0u;
            tmem_st16(tmem + lane_addr + cs, v);
            tmem_st16(tmem + lane_addr + cs + 64u, g);
            add_calibration_tmem(tmem + lane_addr + cs + 64u, bm, bn, sCM + e0, sCN + e0, r);
          } else {
            tmem_st16(tmem + lane_addr + cs, v);
            tmem_st16(tmem + lane_addr + cs + 64u, g);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar.elem_done[rg]);
        mbar_arrive(&bar.qc_free[sl]);
      }
      if (failed) break;
      gbase += nunits;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.acc_full, n & 1, abort))) { failed = true; break; }
      tc_fence_after();
      constexpr int kCols = D / kRowSplit;   // 16
      const uint32_t col = (uint32_t)(part * kCols);
      float v[kCols], g[kCols];
      tmem_ld16(tmem + lane_addr + kColDV + col, v);
      tmem_ld16(tmem + lane_addr + kColDK + col, g);
      tmem_ld_wait_regs(v, g);
      tc_fence_before();
      mbar_arrive(&bar.acc_free);            // the accumulators are free for the next item
      // this warp's 32 rows x 16 columns of dV and dK, 8 columns per TMA
      // store through its staging block
      float* stg = sStage + (warp - 2) * 256;
      const int row0 = kt * KIA_TILE + quad * 32;
#pragma unroll
      for (int pass = 0; pass < 4; ++pass)
        epilogue_store8(stg, pass < 2 ? &tmdV : &tmdK, (pass < 2 ? v : g) + 8 * (pass & 1), 1.0f,
                        lane, (int)col + 8 * (pass & 1), row0, item_bh(it));
    }
    epilogue_store_drain();
  }
  if (failed || *abort) drain_in_flight();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D>
size_t tc_bwd_q_smem(const OpParams& p, bool tab_in_smem, int nkv) {
  const bool minmax_tab = !p.softmax && p.cal == KIA_CAL_MINMAX;
  const int tab =
      p.softmax ? 0 : (minmax_tab ? (tab_in_smem ? (p.K + 1) * KIA_TILE : 0) : 2 * (p.K + 1));
  const size_t head = 2 * (size_t)D * KIA_TILE * 4 + kKmnSlots * (size_t)kHalfTile +
                      kElemThreads / 32 * 1024 + (2 * kRowSplit + 1) * KIA_TILE * 4 +
                      (size_t)((tab + 31) & ~31) * 4 + sizeof(BwdQBars);
  return 1024 + ((head + 1023) & ~(size_t)1023) + nkv * (size_t)kHalfPair;
}

template <int D>
size_t tc_bwd_kv_smem(const OpParams& p, bool tab_in_smem, int nmn) {
  const bool minmax_tab = !p.softmax && p.cal == KIA_CAL_MINMAX;
  const size_t slots = minmax_tab ? 2 : 4;   // kv_const_slots
  const size_t tab =
      p.softmax ? 0 : (minmax_tab ? (tab_in_smem ? slots * 64 * (p.K + 1) : 0) : 4 * (p.K + 1));
  const size_t head = 2 * (size_t)D * KIA_TILE * 4 + kKvSlots * (size_t)kHalfPair +
                      slots * 64 * (16 + 16 + 8 + 8) + slots * 2 * 4 * 2 * 4 +
                      kElemThreads / 32 * 1024 + ((tab + 31) & ~(size_t)31) * 4 + sizeof(BwdKBars);
  return 1024 + ((head + 1023) & ~(size_t)1023) + nmn * (size_t)kHalfPair;
}

template <int D, class V>
int tc_backward_v(const float* Q, const float* Kt, const float* Vv, const float* O,
                  const float* dO, const StatsView& st, const WorkView& wk, float* dQ, float* dK,
                  float* dV, float* dS_dbg, int B, int H, int T, const OpParams& p, cudaStream_t s,
                  void (*mark)(int, cudaStream_t)) {
  const int BH = B * H;
  CUtensorMap tq, tg, tk, tv, tqh, tqmh, tgh, tgmh, tkh, tkmh, tvh, tdq, tdk, tdv;
  if (!make_tmap(&tq, Q, BH, T, D) || !make_tmap(&tg, dO, BH, T, D) ||
      !make_tmap(&tk, Kt, BH, T, D) || !make_tmap(&tv, Vv, BH, T, D) ||
      !make_tmap(&tqh, Q, BH, T, D, false, 64) || !make_tmap(&tqmh, Q, BH, T, D, true, 64) ||
      !make_tmap(&tgh, dO, BH, T, D, false, 64) || !make_tmap(&tgmh, dO, BH, T, D, true, 64) ||
      !make_tmap(&tkh, Kt, BH, T, D, false, 64) || !make_tmap(&tkmh, Kt, BH, T, D, true, 64) ||
      !make_tmap(&tvh, Vv, BH, T, D, false, 64) || !make_tmap_out(&tdq, dQ, BH, T, D) ||
      !make_tmap_out(&tdk, dK, BH, T, D) || !make_tmap_out(&tdv, dV, BH, T, D))
    return KIA_ERR_CUDA;
  // MinMax grid tables in shared memory where they fit, with one ring a slot
  // shallower if that is what makes them fit; else read from global memory
  const bool need_c = V::MINMAX && (p.grad == KIA_GRAD_FULL || p.grad == KIA_GRAD_MAX_ONLY ||
                                    p.grad == KIA_GRAD_MIN_ONLY);
  const bool proj = !V::SOFTMAX && p.grad == KIA_GRAD_PROJECT;
  const size_t kMaxQ = need_c ? dyn_smem_budget(tc_bwd_q_kernel<D, V, true>)
                              : dyn_smem_budget(tc_bwd_q_kernel<D, V, false>);
  const size_t kMaxK = proj ? dyn_smem_budget(tc_bwd_kv_kernel<D, V, true>)
                            : dyn_smem_budget(tc_bwd_kv_kernel<D, V, false>);
  bool q_tab_smem = true;
  int nkv = kBwdSlots;
  if (tc_bwd_q_smem<D>(p, true, nkv) > kMaxQ) nkv = kBwdSlots - 1;
  if (tc_bwd_q_smem<D>(p, true, nkv) > kMaxQ) {
    q_tab_smem = false;
    nkv = kBwdSlots;
  }
  const size_t smq = tc_bwd_q_smem<D>(p, q_tab_smem, nkv);
  bool kv_tab_smem = true;
  int nmn = kKvSlots;
  if (tc_bwd_kv_smem<D>(p, true, nmn) > kMaxK) nmn = kKvSlots - 1;
  if (tc_bwd_kv_smem<D>(p, true, nmn) > kMaxK) {
    kv_tab_smem = false;
    nmn = kKvSlots;
  }
  const size_t smk = tc_bwd_kv_smem<D>(p, kv_tab_smem, nmn);
  if (smq > kMaxQ || smk > kMaxK) return KIA_ERR_UNSUPPORTED;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  // both passes are persistent: one CTA per SM walks the items
  const int sms = num_sms();
  if (sms <= 0) return KIA_ERR_CUDA;
  const dim3 qgrid(std::min(sms, BH * nt));
  if (need_c) {
    if (cudaFuncSetAttribute(tc_bwd_q_kernel<D, V, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smq) != cudaSuccess)
      return KIA_ERR_CUDA;
    tc_bwd_q_kernel<D, V, true><<<qgrid, kTcThreads, smq, s>>>(tq, tg, tkh, tkmh, tvh, Kt, O,
                                                              tdq, st, wk, dS_dbg, p, B, H, T,
                                                              q_tab_smem ? 1 : 0, nkv);
  } else {
    if (cudaFuncSetAttribute(tc_bwd_q_kernel<D, V, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smq) != cudaSuccess)
      return KIA_ERR_CUDA;
    tc_bwd_q_kernel<D, V, false><<<qgrid, kTcThreads, smq, s>>>(tq, tg, tkh, tkmh, tvh, Kt, O,
                                                               tdq, st, wk, dS_dbg, p, B, H, T,
                                                               q_tab_smem ? 1 : 0, nkv);
  }
  if (cudaGetLastError() != cudaSuccess) return KIA_ERR_CUDA;
  mark(4, s);
  auto launch_kv = [&](auto kern) -> int {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smk) !=
        cudaSuccess)
      return KIA_ERR_CUDA;
    kern<<<qgrid, kTcThreads, smk, s>>>(tqh, tqmh, tgh, tgmh, tk, tv, tdk, tdv, st, wk, p, BH, T,
                                        kv_tab_smem ? 1 : 0, nmn);
    return KIA_OK;
  };
  if ((proj ? launch_kv(tc_bwd_kv_kernel<D, V, true>) : launch_kv(tc_bwd_kv_kernel<D, V, false>)))
    return KIA_ERR_CUDA;
  mark(5, s);
  return cudaGetLastError() == cudaSuccess ? KIA_OK : KIA_ERR_CUDA;
}

}  // namespace kia
