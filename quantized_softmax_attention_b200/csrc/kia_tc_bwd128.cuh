// Tensor-core backward of K-interval attention at d = 128 (sm_100a).
//
// Same arithmetic as the d = 64 passes (kia_tc_bwd.cuh), laid out for fp32
// operands twice as wide.  At d = 128 a query (key) tile of 128 rows is 64 KB
// per operand, so the operands that stay for a whole item live in tensor
// memory as the A operands of TS MMAs instead of in shared memory:
//
//  query pass (tc_bwd_q128_kernel), thread = query row:
//    TMEM: Q [0, 128), dO [128, 256), dQ accumulator [256, 384), and one
//          region for a unit of 64 keys: S [384, 448), dP [448, 512)
//    S = Q K^T, dP = dO V^T  (TS: A = Q, dO from TMEM; B = 64-key halves of
//          K and V streamed through a two-slot ring)
//    dS (detached) written over S, dQ += dS K (TS: B = the K half MN-major,
//          N = 128), row sums A, C; epilogue as at d = 64
//  key pass (tc_bwd_kv128_kernel), thread = key row:
//    TMEM: K [0, 128), dV [128, 256), dK [256, 384), one region for 64
//          queries: S^T [384, 448), dP^T [448, 512)
//    S^T = K Q^T (TS), dP^T = V dO^T (SS: V stays in shared memory)
//    P^T and dS^T over S^T and dP^T, dV += P^T dO, dK += dS^T Q (TS, N = 128)
//
// With one region per pass, each unit runs as two halves of 32 keys (query
// pass) or 32 queries (key pass) side by side in the region, each with its
// own barriers: a half's N = 32 score MMAs, its element stage and its
// accumulating MMAs overlap the other half's.  All sixteen element warps work
// on every half, four threads per row, 8 columns each.  The stationary rows
// are copied into tensor memory by the element threads at the start of each
// item, once the previous item's MMAs are done with them.  Under MinMax the
// key pass keeps each half's 32 query grids in one of two shared-memory
// slots, refilled by the constant warp as the element warps release them.
#pragma once
#include "kia_tc_bwd.cuh"

namespace kia {

constexpr uint32_t kHalf128 = 64 * 128 * 4;   // one operand's 64-row half tile at d = 128

// Copies 32 consecutive floats of one row (16-byte aligned) into tensor
// memory at taddr (this thread's lane, 32 columns).
__device__ __forceinline__ void row_to_tmem32(uint32_t taddr, const float* row) {
  const float4* r4 = reinterpret_cast<const float4*>(row);
  float v[32];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 x = r4[i];
    v[4 * i] = x.x;
    v[4 * i + 1] = x.y;
    v[4 * i + 2] = x.z;
    v[4 * i + 3] = x.w;
  }
  tmem_st32(taddr, v);
}

// ---------------------------------------------------------------- query pass

// Eight columns of the warp's 32 TMEM lanes (the passes' half units).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t x[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]),
                 "=r"(x[6]), "=r"(x[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(x[i]);
}
__device__ __forceinline__ void tmem_ld_wait_regs8(float (&v)[8], float (&w)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(w[0]), "+f"(w[1]), "+f"(w[2]), "+f"(w[3]),
                 "+f"(w[4]), "+f"(w[5]), "+f"(w[6]), "+f"(w[7])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
               "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
               "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
               : "memory");
}

struct BwdQ128Bars {
  uint64_t qd_ready;               // Q, dO of the item written into TMEM (element threads)
  uint64_t qd_free;                // the item's S / dP MMAs are done with them
  uint64_t kv_full[2], kv_empty[2];    // K | V half tiles (K-major)
  uint64_t kmn_full[2], kmn_empty[2];  // K half tiles (MN-major)
  // the region holds a unit's two halves of 32 keys side by side (columns
  // S [32 h, 32 h + 32), dP the same 64 further), each with its own barriers,
  // so that one half's MMAs overlap the other half's element work
  uint64_t sp_full[2];             // S, dP of half h in the region
  uint64_t elem_done[2];           // dS of half h written over S
  uint64_t st_free[2];             // half h's dQ MMAs done: its columns free
  uint64_t dq_full, dq_free;
  uint64_t row_sync;
  uint32_t tmem_base;
  int abort;
};

template <class V, bool NEED_C>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_bwd_q128_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmKmn,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdQ,
                   const float* __restrict__ Q, const float* __restrict__ Kt,
                   const float* __restrict__ O, const float* __restrict__ dO, StatsView st,
                   WorkView wk, float* __restrict__ dS_dbg, OpParams p, int B, int H, int T,
                   int tab_in_smem, int nkmn) {
  constexpr int D = 128;
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
  uint8_t* sKV = base;                                  // [2][K half | V half]
  float* sStage = reinterpret_cast<float*>(sKV + 2 * 2 * kHalf128);   // [16 warps][32][8]
  float* sAC = sStage + kElemThreads / 32 * 256;        // [kRowSplit][2][128]
  float* sDc = sAC + 2 * kRowSplit * KIA_TILE;          // [128] centering D
  // FWM grid pairs (+ the tail's zero pair), or under MinMax the rows' own
  // grids [K + 1][128] when they fit
  float2* sPair = reinterpret_cast<float2*>(sDc + KIA_TILE);
  float* sTab = reinterpret_cast<float*>(sPair);
  const int pair_floats = V::SOFTMAX ? 0
                        : (V::MINMAX ? (tab_in_smem ? (p.K + 1) * KIA_TILE : 0) : 2 * (p.K + 1));
  BwdQ128Bars& bar =
      *reinterpret_cast<BwdQ128Bars*>(reinterpret_cast<float*>(sPair) + ((pair_floats + 31) & ~31));
  // the MN-major K ring last (1024-aligned): two slots, one when a MinMax
  // grid table needs the room (only the producer and the dQ issuer use it)
  const int NKM = V::MINMAX ? nkmn : 2;
  uint8_t* sKmn =
      base + ((reinterpret_cast<uint8_t*>(&bar + 1) - base + 1023) & ~(ptrdiff_t)1023);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = B * H;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int nitems = BH * nt;
  auto item_qt = [&](int it) { return nt - 1 - it / BH; };
  auto item_bh = [&](int it) { return it % BH; };
  auto item_units = [&](int it) { return 2 * (p.causal ? item_qt(it) + 1 : nt); };
  constexpr uint32_t kColQ = 0, kColG = 128, kColDQ = 256, kColS = 384, kColP = 448;

  if (threadIdx.x == 0) {
    mbar_init(&bar.qd_ready, kElemThreads);
    mbar_init(&bar.qd_free, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar.kv_full[s], 1);
      mbar_init(&bar.kv_empty[s], 1);
      mbar_init(&bar.kmn_full[s], 1);
      mbar_init(&bar.kmn_empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bar.sp_full[h], 1);
      mbar_init(&bar.elem_done[h], kElemThreads);
      mbar_init(&bar.st_free[h], 1);
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
    // the two key rings refill independently, each as soon as its slot is
    // free (half tiles numbered across the CTA's items)
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmKmn);
      tma_prefetch_desc(&tmV);
      ItemSeq sk(nitems), sm(nitems);
      int ik = sk.next(), uk = 0, gk = 0;
      int im = sm.next(), um = 0, gm = 0;
      PollGuard guard;
      while ((ik >= 0 || im >= 0) && !failed) {
        bool moved = false;
        if (ik >= 0) {
          const int sl = gk & 1;
          if (mbar_test(&bar.kv_empty[sl], ((gk >> 1) & 1) ^ 1)) {
            uint8_t* dst = sKV + sl * 2 * kHalf128;
            mbar_arrive_expect_tx(&bar.kv_full[sl], 2 * kHalf128);
            for (int b = 0; b < D / 32; ++b) {
              tma_load_3d(dst + b * kHalfBlockBytes, &tmK, &bar.kv_full[sl], b * 32, 64 * uk,
                          item_bh(ik));
              tma_load_3d(dst + kHalf128 + b * kHalfBlockBytes, &tmV, &bar.kv_full[sl], b * 32,
                          64 * uk, item_bh(ik));
            }
            ++gk;
            if (++uk == item_units(ik)) { uk = 0; ik = sk.next(); }
            moved = true;
          }
        }
        if (im >= 0) {
          const int sl = gm % NKM;
          if (mbar_test(&bar.kmn_empty[sl], ((gm / NKM) & 1) ^ 1)) {
            uint8_t* dst = sKmn + sl * kHalf128;
            mbar_arrive_expect_tx(&bar.kmn_full[sl], kHalf128);
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
    // S = Q K^T and dP = dO V^T with A from TMEM, one half of 32 keys at a
    // time (N = 32; the half's rows start 4 KB into each 128-byte-swizzled
    // column block of the half tile); whole warp in the loop, one elected
    // lane issuing
    const uint32_t id_s = idesc_tf32(128, 32, 0, 0);
    const uint64_t dkv = desc_kmajor_half(smem_u32(sKV));
    int g = 0, n = 0;
    ItemSeq seq(nitems);
    for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
      if (!warp_wait(&bar.qd_ready, n & 1, abort)) { failed = true; break; }
      const int nunits = item_units(it);
      for (int u = 0; u < nunits && !failed; ++u, ++g) {
        const int sl = g & 1;
        if (!warp_wait(&bar.kv_full[sl], (g >> 1) & 1, abort)) { failed = true; break; }
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          // half h's columns are free once the previous unit's half-h dQ MMAs
          // are done
          if (g > 0 && !warp_wait(&bar.st_free[h], (g - 1) & 1, abort)) { failed = true; break; }
          const uint64_t dk = dkv + desc_step((uint32_t)sl * 2 * kHalf128 + 4096u * (uint32_t)h);
          const uint64_t dv = dk + desc_step(kHalf128);
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < D / 8; ++ks)
              mma_tf32_ts(tmem + kColS + 32u * h, tmem + kColQ + 8u * ks,
                          dk + kstep_kmajor_half(ks), id_s, ks > 0 ? 1u : 0u);
#pragma unroll
            for (int ks = 0; ks < D / 8; ++ks)
              mma_tf32_ts(tmem + kColP + 32u * h, tmem + kColG + 8u * ks,
                          dv + kstep_kmajor_half(ks), id_s, ks > 0 ? 1u : 0u);
            tc_commit(&bar.sp_full[h]);
            if (h == 1) tc_commit(&bar.kv_empty[sl]);
          }
          __syncwarp();
        }
      }
      if (failed) break;
      if (elect_one()) tc_commit(&bar.qd_free);   // Q, dO in TMEM free once these MMAs are done
      __syncwarp();
    }
  } else if (warp == 1) {
    // --------------------------------------------------- dQ-MMA issuer
    const uint32_t id_dq = idesc_tf32(128, D, 0, 1);
    const uint64_t dkm = desc_mnmajor_half(smem_u32(sKmn));
    int g = 0, n = 0;
    ItemSeq seq(nitems);
    for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
      const int nunits = item_units(it);
      for (int u = 0; u < nunits && !failed; ++u, ++g) {
        const int sl = g % NKM;
        const uint64_t db = dkm + desc_step((uint32_t)sl * kHalf128);
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          // half h: keys 32 h .. 32 h + 31 of the unit, the MN-major k-steps
          // 4 h .. 4 h + 3 of the half tile
          if (!warp_wait(&bar.elem_done[h], g & 1, abort)) { failed = true; break; }
          if (h == 0 && !warp_wait(&bar.kmn_full[sl], (g / NKM) & 1, abort)) { failed = true; break; }
          // the accumulator restarts with this item: the previous item's
          // epilogue must have read it
          if (u == 0 && h == 0 && n > 0 && !warp_wait(&bar.dq_free, (n - 1) & 1, abort)) { failed = true; break; }
          const uint32_t acc0 = (u > 0 || h > 0) ? 1u : 0u;
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_tf32_ts(tmem + kColDQ, tmem + kColS + 32u * h + 8u * kk,
                          db + kstep_mnmajor(4 * h + kk), id_dq, kk > 0 ? 1u : acc0);
            tc_commit(&bar.st_free[h]);
            if (h == 1) tc_commit(&bar.kmn_empty[sl]);
          }
          __syncwarp();
        }
      }
      if (failed) break;
      if (elect_one()) tc_commit(&bar.dq_full);
      __syncwarp();
    }
  } else if (warp < kScoreWarp) {
    // ------------------------------------------------------ element warps
    const int quad = warp & 3;
    const int part = (warp - 2) >> 2;        // 0..3: 16 columns of each unit
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const float Kf = p.Kf, Km1f = (float)(p.K - 1);
    if constexpr (!V::MINMAX && !V::SOFTMAX) {
      // pairs k = 0..K-1 and the tail's zero pair at K
      for (int k = (int)threadIdx.x - 64; k <= p.K; k += kElemThreads)
        sPair[k] = k < p.K ? make_float2(st.table[k], st.table[k + 1]) : make_float2(0.0f, 0.0f);
    }
    int g = 0, n = 0;
    ItemSeq seq(nitems);
    for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
      const int qt = item_qt(it), bh = item_bh(it), nunits = item_units(it);
      const int q = qt * KIA_TILE + r;
      const long long rowbase = (long long)bh * T;
      const long long qr = rowbase + (q < T ? q : T - 1);
      // Q and dO rows into TMEM once the previous item's S / dP MMAs are done
      if (n > 0 && !__all_sync(0xffffffffu, mbar_wait(&bar.qd_free, (n - 1) & 1, abort))) { failed = true; break; }
      tc_fence_after();
      row_to_tmem32(tmem + lane_addr + kColQ + 32u * part, Q + qr * D + 32 * part);
      row_to_tmem32(tmem + lane_addr + kColG + 32u * part, dO + qr * D + 32 * part);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar.qd_ready);
      {
        // the next item's Q and dO rows into L2 now, so that their copy into
        // tensor memory at its start waits for L2 rather than DRAM
        ItemSeq peek = seq;
        const int nx = peek.next();
        if (nx >= 0) {
          const int qn = item_qt(nx) * KIA_TILE + r;
          const long long qrn = (long long)item_bh(nx) * T + (qn < T ? qn : T - 1);
          prefetch_l2(Q + qrn * D + 32 * part);
          prefetch_l2(dO + qrn * D + 32 * part);
        }
      }
      // this row's calibration and centering (written by the forward)
      const float m = st.m[qr];
      const int am = st.am[qr], an = V::MINMAX ? st.an[qr] : am;
      const float rh = st.rh[qr];
      // a degenerate MinMax row (1/h = 0) has dS = dw: with its grid in shared
      // memory through the copy patched to G_1 = 2 (below) and the factor 1,
      // else through dg
      const bool fold = V::MINMAX && tab_in_smem && rh == 0.0f;
      const float nrh = fold ? 1.0f : -rh;
      const float dg = (V::MINMAX && !tab_in_smem && rh == 0.0f) ? 1.0f : 0.0f;
      const int L = p.causal ? q + 1 : T;
      const float rWb = (L == 1) ? 0.0f : __fdiv_rn(1.0f, st.Wb[qr]);
      prefetch_l2(Kt + (rowbase + am) * D + part * 32);
      if constexpr (V::MINMAX) prefetch_l2(Kt + (rowbase + an) * D + part * 32);
      {
        // centering D = dO . O_bar, four threads per row (coalesced)
        const int e = (int)threadIdx.x - 64;
        const int rr = e >> 2, cc = e & 3;
        const int qq = qt * KIA_TILE + rr;
        const long long qrr = rowbase + (qq < T ? qq : T - 1);
        const float4* g4 = reinterpret_cast<const float4*>(dO + qrr * D) + cc * (D / 16);
        const float4* o4 =
            reinterpret_cast<const float4*>((V::PROB ? st.OL : O) + qrr * D) + cc * (D / 16);
        float acc = 0.0f;
#pragma unroll
        for (int c = 0; c < D / 16; ++c) {
          const float4 a = g4[c], b4 = o4[c];
          acc = fmaf(a.x, b4.x, acc);
          acc = fmaf(a.y, b4.y, acc);
          acc = fmaf(a.z, b4.z, acc);
          acc = fmaf(a.w, b4.w, acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (cc == 0) {
          sDc[rr] = acc;
          if (qq < T) wk.D[qrr] = acc;
        }
      }
      if constexpr (V::MINMAX) {
        // the row's grid, column r of [K + 1][128] (four threads per row)
        if (tab_in_smem)
          for (int k = part; k <= p.K; k += kRowSplit)
            sTab[k * KIA_TILE + r] = (fold && k == 1) ? 2.0f : st.table[qr * (p.K + 1) + k];
      }
      mbar_arrive(&bar.row_sync);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, (2 * n) & 1, abort))) { failed = true; break; }
      const float Dc = sDc[r];
      const float nDr = -Dc * rWb;
      float A = 0.0f, C = 0.0f;
      auto unit_loop = [&](const auto& grid, auto fold_c) {
        constexpr bool FOLD = decltype(fold_c)::value;
        for (int u = 0; u < nunits && !failed; ++u, ++g) {
          const bool edge = (p.causal && (u >> 1) == qt) || 64 * u + 64 > T;
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            // half h: this thread's 8 key columns 32 h + 8 part .. + 7
            if (!__all_sync(0xffffffffu, mbar_wait(&bar.sp_full[h], g & 1, abort))) { failed = true; break; }
            tc_fence_after();
            const int key0 = 64 * u + 32 * h + 8 * part;
            const uint32_t cS = kColS + 32u * h + 8u * part, cP = kColP + 32u * h + 8u * part;
            float v[8], gg[8];
            tmem_ld8(tmem + lane_addr + cS, v);
            tmem_ld8(tmem + lane_addr + cP, gg);
            tmem_ld_wait_regs8(v, gg);
            if (!edge) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float dw = fmaf(gg[i], rWb, nDr);
                v[i] = bwd_delta<V, NEED_C, FOLD>(grid, m, rh, nrh, dg, Kf, Km1f, v[i], dw, A, C);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int key = key0 + i;
                const bool ok = key < T && (!p.causal || key <= q);
                const float dw = ok ? fmaf(gg[i], rWb, nDr) : 0.0f;
                v[i] = bwd_delta<V, NEED_C, FOLD>(grid, m, rh, nrh, dg, Kf, Km1f, v[i], dw, A, C);
              }
            }
            tmem_st8(tmem + lane_addr + cS, v);
            if (dS_dbg && q < T) {
              float* dst = dS_dbg + (rowbase + q) * T + key0;
#pragma unroll
              for (int i = 0; i < 8; ++i)
                if (key0 + i < T) dst[i] = v[i];
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bar.elem_done[h]);
          }
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
      sAC[(part * 2 + 0) * KIA_TILE + r] = A;
      sAC[(part * 2 + 1) * KIA_TILE + r] = C;
      mbar_arrive(&bar.row_sync);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.row_sync, (2 * n + 1) & 1, abort))) { failed = true; break; }
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.dq_full, n & 1, abort))) { failed = true; break; }
      tc_fence_after();
      // this thread's 32 columns of dQ, then the accumulator is free
      const uint32_t col = (uint32_t)(part * 32);
      float o[32];
      tmem_ld32(tmem + lane_addr + kColDQ + col, o);
      tmem_ld_wait_regs(o);
      tc_fence_before();
      mbar_arrive(&bar.dq_free);
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
          const float4* k4 = reinterpret_cast<const float4*>(Kt + (rowbase + am) * D + col);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 kk = k4[i];
            o[4 * i] = fmaf(gmq, kk.x, o[4 * i]);
            o[4 * i + 1] = fmaf(gmq, kk.y, o[4 * i + 1]);
            o[4 * i + 2] = fmaf(gmq, kk.z, o[4 * i + 2]);
            o[4 * i + 3] = fmaf(gmq, kk.w, o[4 * i + 3]);
          }
        }
        if (V::MINMAX && gn != 0.0f) {
          const float4* k4 = reinterpret_cast<const float4*>(Kt + (rowbase + an) * D + col);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 kk = k4[i];
            o[4 * i] = fmaf(gn, kk.x, o[4 * i]);
            o[4 * i + 1] = fmaf(gn, kk.y, o[4 * i + 1]);
            o[4 * i + 2] = fmaf(gn, kk.z, o[4 * i + 2]);
            o[4 * i + 3] = fmaf(gn, kk.w, o[4 * i + 3]);
          }
        }
      }
      {
        float* stg = sStage + (warp - 2) * 256;
        const int row0 = qt * KIA_TILE + quad * 32;
#pragma unroll
        for (int pass = 0; pass < 4; ++pass)
          epilogue_store8(stg, &tmdQ, o + 8 * pass, 1.0f, lane, (int)col + 8 * pass, row0, bh);
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

inline size_t tc_bwd_q128_smem(const OpParams& p, bool tab_in_smem, int nkmn) {
  const bool minmax = !p.softmax && p.cal == KIA_CAL_MINMAX;
  const size_t tab = p.softmax ? 0 : (minmax ? (tab_in_smem ? (size_t)(p.K + 1) * KIA_TILE : 0)
                                              : 2 * (size_t)(p.K + 1));
  const size_t head = 2 * 2 * (size_t)kHalf128 + kElemThreads / 32 * 1024 +
                      (2 * kRowSplit + 1) * KIA_TILE * 4 + ((tab + 31) & ~(size_t)31) * 4 +
                      sizeof(BwdQ128Bars);
  return 1024 + ((head + 1023) & ~(size_t)1023) + (size_t)nkmn * kHalf128;
}


// ------------------------------------------------------------------ key pass

struct BwdKV128Bars {
  uint64_t k_ready;                // K of the item written into TMEM (element threads)
  uint64_t k_free;                 // the item's S^T MMAs are done with it
  uint64_t v_full, v_empty;        // V of the item (shared memory, K-major)
  uint64_t qd_full, qd_empty;      // Q and dO half tiles, K-major (for S^T, dP^T)
  uint64_t mn_full, mn_empty;      // Q and dO half tiles, MN-major (for dK, dV)
  // the region holds a unit's two halves of 32 queries side by side
  // (columns S [32 h, 32 h + 32), dP the same 64 further), each with its own
  // barriers, so that one half's MMAs overlap the other half's element work
  uint64_t sp_full[2];             // S^T, dP^T of half h in the region
  uint64_t qc_ready[2], qc_free[2];   // per-query constants of a unit in slot s
  uint64_t elem_done[2];           // P^T, dS^T of half h written over S^T, dP^T
  uint64_t st_free[2];             // half h's dV, dK MMAs done: its columns free
  uint64_t acc_full, acc_free;
  uint64_t acc_issued;             // the item's last dV, dK MMAs issued
  // MinMax with the queries' grids in shared memory: table slot h holds the
  // 32 grids of the current unit's half h
  uint64_t tab_ready[2];           // half h's grids copied into slot h (constant warp)
  uint64_t tab_free[2];            // the element warps done with slot h
  uint32_t tmem_base;
  int abort;
};

template <class V, bool PROJ>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_bwd_kv128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQmn,
                    const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmGmn,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdK,
                    const __grid_constant__ CUtensorMap tmdV, const float* __restrict__ Kt,
                    StatsView st, WorkView wk, OpParams p, int BH, int T, int tab_in_smem) {
  constexpr int D = 128;
  if (*wk.status != 0) return;
  extern __shared__ uint8_t smraw[];
  uint8_t* base = smraw + ((1024u - (smem_u32(smraw) & 1023u)) & 1023u);
  float* sV = reinterpret_cast<float*>(base);                     // [128 x 128], K-major
  uint8_t* sQD = base + D * KIA_TILE * 4;                           // [Q half | dO half]
  uint8_t* sQDmn = sQD + 2 * kHalf128;                              // [Q half | dO half], MN-major
  // per-query constants of a unit (64 queries) in two slots: unit g uses
  // slot g % 2; layout as in the d = 64 key pass
  constexpr int kSlots = 2, kSlotQ = 64;
  float4* sC4 = reinterpret_cast<float4*>(sQDmn + 2 * kHalf128);
  float4* sX4 = sC4 + kSlots * kSlotQ;
  int2* sCM = reinterpret_cast<int2*>(sX4 + kSlots * kSlotQ);   // argmax key, g_m bits
  int2* sCN = sCM + kSlots * kSlotQ;                            // argmin key, g_n bits
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sCN + kSlots * kSlotQ);   // [slot][max/min][quad][half]
  float* sStage = reinterpret_cast<float*>(sMask + kSlots * 2 * 4 * 2);   // [16 warps][32][8]
  float2* sPair = reinterpret_cast<float2*>(sStage + kElemThreads / 32 * 256);
  const int pair_floats = (!V::SOFTMAX && !V::MINMAX) ? 2 * (p.K + 1) : 0;
  BwdKV128Bars& bar =
      *reinterpret_cast<BwdKV128Bars*>(reinterpret_cast<float*>(sPair) + ((pair_floats + 31) & ~31));
  // MinMax: two slots of 32 queries' grids ([slot][32][K + 1]) after the barriers
  const int K1 = p.K + 1;
  const bool tabs = V::MINMAX && tab_in_smem;
  float* sTabH = reinterpret_cast<float*>(&bar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int nitems = BH * nt;
  auto item_kt = [&](int it) { return it / BH; };
  auto item_bh = [&](int it) { return it % BH; };
  auto item_q0 = [&](int it) { return p.causal ? item_kt(it) : 0; };
  auto item_units = [&](int it) { return 2 * (nt - item_q0(it)); };
  constexpr uint32_t kColK = 0, kColDV = 128, kColDK = 256, kColS = 384, kColP = 448;

  if (threadIdx.x == 0) {
    mbar_init(&bar.k_ready, kElemThreads);
    mbar_init(&bar.k_free, 1);
    mbar_init(&bar.v_full, 1);
    mbar_init(&bar.v_empty, 1);
    mbar_init(&bar.qd_full, 1);
    mbar_init(&bar.qd_empty, 1);
    mbar_init(&bar.mn_full, 1);
    mbar_init(&bar.mn_empty, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bar.sp_full[h], 1);
      mbar_init(&bar.elem_done[h], kElemThreads);
      mbar_init(&bar.st_free[h], 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&bar.qc_ready[s], 32);
      mbar_init(&bar.qc_free[s], kElemThreads);
    }
    mbar_init(&bar.acc_full, 1);
    mbar_init(&bar.acc_free, kElemThreads);
    mbar_init(&bar.acc_issued, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bar.tab_ready[h], 32);
      mbar_init(&bar.tab_free[h], kElemThreads);
    }
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
    // V of each item once the previous item's dP^T MMAs are done with it;
    // the K-major and MN-major query half tiles of each unit, each pair as
    // soon as its single slot is free
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmQmn);
      tma_prefetch_desc(&tmG);
      tma_prefetch_desc(&tmGmn);
      tma_prefetch_desc(&tmV);
      ItemSeq sv(nitems), sq(nitems), sm(nitems);
      int iv = sv.next(), nv = 0;
      int iq = sq.next(), uq = 0, gq = 0;
      int im = sm.next(), um = 0, gm = 0;
      PollGuard guard;
      while ((iv >= 0 || iq >= 0 || im >= 0) && !failed) {
        bool moved = false;
        if (iv >= 0 && mbar_test(&bar.v_empty, (nv & 1) ^ 1)) {
          mbar_arrive_expect_tx(&bar.v_full, D * KIA_TILE * 4);
          for (int b = 0; b < D / 32; ++b)
            tma_load_3d(sV + b * 32 * KIA_TILE, &tmV, &bar.v_full, b * 32,
                        item_kt(iv) * KIA_TILE, item_bh(iv));
          iv = sv.next();
          ++nv;
          moved = true;
        }
        if (iq >= 0 && mbar_test(&bar.qd_empty, (gq & 1) ^ 1)) {
          const int row = 64 * (2 * item_q0(iq) + uq);
          mbar_arrive_expect_tx(&bar.qd_full, 2 * kHalf128);
          for (int b = 0; b < D / 32; ++b) {
            tma_load_3d(sQD + b * kHalfBlockBytes, &tmQ, &bar.qd_full, b * 32, row, item_bh(iq));
            tma_load_3d(sQD + kHalf128 + b * kHalfBlockBytes, &tmG, &bar.qd_full, b * 32, row,
                        item_bh(iq));
          }
          ++gq;
          if (++uq == item_units(iq)) { uq = 0; iq = sq.next(); }
          moved = true;
        }
        if (im >= 0 && mbar_test(&bar.mn_empty, (gm & 1) ^ 1)) {
          const int row = 64 * (2 * item_q0(im) + um);
          mbar_arrive_expect_tx(&bar.mn_full, 2 * kHalf128);
          for (int b = 0; b < D / 32; ++b) {
            tma_load_3d(sQDmn + b * kHalfBlockBytes, &tmQmn, &bar.mn_full, b * 32, row,
                        item_bh(im));
            tma_load_3d(sQDmn + kHalf128 + b * kHalfBlockBytes, &tmGmn, &bar.mn_full, b * 32, row,
                        item_bh(im));
          }
          ++gm;
          if (++um == item_units(im)) { um = 0; im = sm.next(); }
          moved = true;
        }
        if (moved) guard.progress();
        else if (!guard.idle(abort)) failed = true;
      }
    }
  } else if (warp == kScoreWarp) {
    // ------------------------------------------------- score-MMA issuer
    // S^T = K Q^T (A = K from TMEM), dP^T = V dO^T (A = V from shared memory),
    // one half of 32 queries at a time (N = 32; the half's rows start 4 KB
    // into each 128-byte-swizzled column block of the half tile)
    const uint32_t id_s = idesc_tf32(128, 32, 0, 0);
    const uint64_t dva = desc_kmajor(smem_u32(sV), 0);
    const uint64_t dqd = desc_kmajor_half(smem_u32(sQD));
    const uint64_t dgd = dqd + desc_step(kHalf128);
    int g = 0, n = 0;
    ItemSeq seq(nitems);
    for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
      if (!warp_wait(&bar.k_ready, n & 1, abort)) { failed = true; break; }
      if (!warp_wait(&bar.v_full, n & 1, abort)) { failed = true; break; }
      // the previous item's last dV / dK MMAs ahead of this item's scores
      if (n > 0 && !warp_wait(&bar.acc_issued, (n - 1) & 1, abort)) { failed = true; break; }
      const int nunits = item_units(it);
      for (int u = 0; u < nunits && !failed; ++u, ++g) {
        if (!warp_wait(&bar.qd_full, g & 1, abort)) { failed = true; break; }
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          // half h's columns are free once the previous unit's half-h dV, dK
          // MMAs are done
          if (g > 0 && !warp_wait(&bar.st_free[h], (g - 1) & 1, abort)) { failed = true; break; }
          const uint64_t hq = desc_step(4096u * (uint32_t)h);
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < D / 8; ++ks)
              mma_tf32_ts(tmem + kColS + 32u * h, tmem + kColK + 8u * ks,
                          dqd + hq + kstep_kmajor_half(ks), id_s, ks > 0 ? 1u : 0u);
#pragma unroll
            for (int ks = 0; ks < D / 8; ++ks)
              mma_tf32_ss(tmem + kColP + 32u * h, dva + kstep_kmajor(ks),
                          dgd + hq + kstep_kmajor_half(ks), id_s, ks > 0 ? 1u : 0u);
            tc_commit(&bar.sp_full[h]);
            if (h == 1) tc_commit(&bar.qd_empty);
          }
          __syncwarp();
        }
      }
      if (failed) break;
      if (elect_one()) {
        tc_commit(&bar.k_free);     // K in TMEM free once these MMAs are done
        tc_commit(&bar.v_empty);    // and V's shared-memory tile
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ---------------------------------------------- dV / dK-MMA issuer
    const uint32_t id_acc = idesc_tf32(128, D, 0, 1);
    const uint64_t dqm = desc_mnmajor_half(smem_u32(sQDmn));
    const uint64_t dgm = dqm + desc_step(kHalf128);
    int g = 0, n = 0;
    ItemSeq seq(nitems);
    for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
      const int nunits = item_units(it);
      for (int u = 0; u < nunits && !failed; ++u, ++g) {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          // half h: queries 32 h .. 32 h + 31 of the unit, the MN-major
          // k-steps 4 h .. 4 h + 3 of the half tile
          if (!warp_wait(&bar.elem_done[h], g & 1, abort)) { failed = true; break; }
          if (h == 0 && !warp_wait(&bar.mn_full, g & 1, abort)) { failed = true; break; }
          if (u == 0 && h == 0 && n > 0 && !warp_wait(&bar.acc_free, (n - 1) & 1, abort)) { failed = true; break; }
          const uint32_t acc0 = (u > 0 || h > 0) ? 1u : 0u;
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_tf32_ts(tmem + kColDV, tmem + kColS + 32u * h + 8u * kk,
                          dgm + kstep_mnmajor(4 * h + kk), id_acc, kk > 0 ? 1u : acc0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_tf32_ts(tmem + kColDK, tmem + kColP + 32u * h + 8u * kk,
                          dqm + kstep_mnmajor(4 * h + kk), id_acc, kk > 0 ? 1u : acc0);
            tc_commit(&bar.st_free[h]);
            if (h == 1) tc_commit(&bar.mn_empty);
          }
          __syncwarp();
        }
      }
      if (failed) break;
      if (elect_one()) {
        tc_commit(&bar.acc_full);
        mbar_arrive(&bar.acc_issued);
      }
      __syncwarp();
    }
  } else if (warp == kScoreWarp + 1) {
    // -------------------------------------------- query-constant producer
    if (!V::SOFTMAX && !V::MINMAX) {
      for (int k = lane; k <= p.K; k += 32)
        sPair[k] = k < p.K ? make_float2(st.table[k], st.table[k + 1]) : make_float2(0.0f, 0.0f);
    }
    struct Raw {
      float m[2], rh[2], D[2], Wb[2], Wf[2], gm[2], gn[2];
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
        x.D[hq] = wk.D[qr];
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
      const int sl = g & 1;
      int it2 = it, u2 = u + 1;
      if (u2 == item_units(it)) { u2 = 0; it2 = cseq.next(); }
      Raw nxt;
      if (it2 >= 0) load_raw(it2, u2, nxt);
      if (g >= kSlots && !__all_sync(0xffffffffu, mbar_wait(&bar.qc_free[sl], ((g >> 1) - 1) & 1, abort))) {
        failed = true;
        break;
      }
      const int kt = item_kt(it);
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        const int q = 64 * (2 * item_q0(it) + u) + 32 * hq + lane;
        const int e = sl * kSlotQ + 32 * hq + lane;
        const int Lq = p.causal ? q + 1 : T;
        const float rWb = Lq == 1 ? 0.0f : __fdiv_rn(1.0f, cur.Wb[hq]);
        const float nD = -cur.D[hq] * rWb;
        // a degenerate MinMax row (1/h = 0) has dS = dw (uniform P): with the
        // grids in shared memory through its slot copy patched to G_1 = 2 and
        // the factor 1 here, else through x.y, x.z
        const bool fold = tabs && cur.rh[hq] == 0.0f;
        const float nrh = (V::SOFTMAX || fold) ? 1.0f : -cur.rh[hq];
        sC4[e] = make_float4(cur.m[hq], rWb * nrh, nD * nrh, __fdiv_rn(1.0f, cur.Wf[hq]));
        const bool live = q < T;
        const float gm = live ? cur.gm[hq] : 0.0f, gn = live ? cur.gn[hq] : 0.0f;
        if constexpr (V::MINMAX || PROJ) {
          const float dg = (V::MINMAX && !tabs && cur.rh[hq] == 0.0f) ? 1.0f : 0.0f;
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
      __syncwarp();
      mbar_arrive(&bar.qc_ready[sl]);
      if (tabs) {
        // the unit's grids, half h into slot h once the element warps are
        // done with the previous unit's half h (asynchronous copies; rows
        // past T are filled with ones, their queries are masked)
        const long long rowbase = (long long)item_bh(it) * T;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          if (g > 0 && !__all_sync(0xffffffffu, mbar_wait(&bar.tab_free[h], (g - 1) & 1, abort))) {
            failed = true;
            break;
          }
          const int qf = 64 * (2 * item_q0(it) + u) + 32 * h;
          const int nvalid = max(0, min(32, T - qf)) * K1, ntot = 32 * K1;
          const float* src = st.table + (rowbase + qf) * K1;
          float* dst = sTabH + h * 32 * K1;
          for (int x = lane; x < ntot; x += 32) {
            if (x < nvalid) cp_async4(dst + x, src + x);
            else dst[x] = 1.0f;
          }
          cp_async_wait_all();
          __syncwarp();
          // a degenerate row (this lane's query of the half) gets G_1 = 2:
          // its scores all sit at node 0, the slope 1 carries dw
          if (cur.rh[h] == 0.0f) dst[lane * K1 + 1] = 2.0f;
          __syncwarp();
          mbar_arrive(&bar.tab_ready[h]);
        }
        if (failed) break;
      }
      cur = nxt;
      it = it2;
      u = u2;
    }
  } else if (warp < kScoreWarp) {
    // ------------------------------------------------------ element warps
    const int quad = warp & 3;
    const int part = (warp - 2) >> 2;         // query columns 16 part .. +15 of each unit
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const float Kf = p.Kf, Km1f = (float)(p.K - 1);
    const GridZ gridz = make_gridz(sPair, p.K);
    const float rh_c = p.fwm_rh;
    int g = 0, n = 0;
    ItemSeq seq(nitems);
    for (int it = seq.next(); it >= 0 && !failed; it = seq.next(), ++n) {
      const int kt = item_kt(it), q0 = item_q0(it), nunits = item_units(it);
      const int kj = kt * KIA_TILE + r;
      const long long rowbase = (long long)item_bh(it) * T;
      // K rows into TMEM once the previous item's S^T MMAs are done
      if (n > 0 && !__all_sync(0xffffffffu, mbar_wait(&bar.k_free, (n - 1) & 1, abort))) { failed = true; break; }
      tc_fence_after();
      row_to_tmem32(tmem + lane_addr + kColK + 32u * part,
                    Kt + (rowbase + (kj < T ? kj : T - 1)) * D + 32 * part);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bar.k_ready);
      {
        // the next item's K row into L2 now (its copy into tensor memory then
        // waits for L2 rather than DRAM)
        ItemSeq peek = seq;
        const int nx = peek.next();
        if (nx >= 0) {
          const int kn = item_kt(nx) * KIA_TILE + r;
          prefetch_l2(Kt + ((long long)item_bh(nx) * T + (kn < T ? kn : T - 1)) * D + 32 * part);
        }
      }
      for (int u = 0; u < nunits && !failed; ++u, ++g) {
        const int qi = q0 + (u >> 1);
        const int sl = g & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.qc_ready[sl], (g >> 1) & 1, abort))) { failed = true; break; }
        const bool edge =
            (p.causal && qi == kt) || (qi + 1) * KIA_TILE > T || (kt + 1) * KIA_TILE > T;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
        // half h: this thread's 8 query columns 32 h + 8 part .. + 7
        if (tabs && !__all_sync(0xffffffffu, mbar_wait(&bar.tab_ready[h], g & 1, abort))) { failed = true; break; }
        if (!__all_sync(0xffffffffu, mbar_wait(&bar.sp_full[h], g & 1, abort))) { failed = true; break; }
        tc_fence_after();
        const uint32_t cS = kColS + 32u * h + 8u * part, cP = kColP + 32u * h + 8u * part;
        float v[8], gg[8];
        tmem_ld8(tmem + lane_addr + cS, v);
        tmem_ld8(tmem + lane_addr + cP, gg);
        tmem_ld_wait_regs8(v, gg);
        const int ql0 = 64 * (u & 1) + 32 * h + 8 * part;   // first query (in the tile) of the chunk
        const int e0 = sl * kSlotQ + 32 * h + 8 * part;     // its slot entry
        // one body for every unit; the masked pairs of an edge unit are
        // zeroed afterwards (finite scores: the clamped grid index stays in
        // the table)
        auto body = [&](auto tabs_c) {
          [[maybe_unused]] constexpr bool TABS = decltype(tabs_c)::value;   // grids in shared memory
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            [[maybe_unused]] const int ql = ql0 + i;
            const float4 cq = sC4[e0 + i];
            float4 xq = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if constexpr (V::MINMAX || PROJ) xq = sX4[e0 + i];
            const float s = v[i], dP = gg[i];
            const float dSn = fmaf(dP, cq.y, cq.z);
            float P, dS;
            if constexpr (V::SOFTMAX) {
              const float w = expf(s - cq.x);
              P = round_exp<V::EXPR>(w) * cq.w;
              dS = w * dSn;
            } else {
              const float rh = V::MINMAX ? xq.x : rh_c;
              float uu = __fmul_rn(__fsub_rn(cq.x, s), rh);
              if constexpr (V::MINMAX) uu = fminf(uu, Kf);
              const float uc = fmaxf(fminf(uu, Km1f), 0.0f);
              const float tmp = __fadd_rd(uc, kMagic);
              const float t = __fsub_rn(uu, __fsub_rn(tmp, kMagic));
              float2 gp;
              if constexpr (V::MINMAX) {
                const float* gq;
                if constexpr (TABS) gq = sTabH + (h * 32 + 8 * part + i) * K1;
                else gq = st.table + (rowbase + min(qi * KIA_TILE + ql, T - 1)) * (p.K + 1);
                gp = GridF{gq, 1}.pair(__float_as_int(tmp) - kMagicBits);
              } else {
                gp = gridz.at(__float_as_int(tmp) - kMagicBits, uu > Kf);
              }
              const float a = __fsub_rn(gp.y, gp.x);
              const float wf = V::NEAREST ? (t >= 0.5f ? gp.y : gp.x) : __fmaf_rn(t, a, gp.x);
              P = wf * cq.w;
              dS = a * dSn;
              if constexpr (V::MINMAX && !TABS) dS = fmaf(dP, xq.y, dS + xq.z);
            }
            if constexpr (PROJ) dS += xq.w;
            v[i] = P;
            gg[i] = dS;
          }
        };
        if (tabs) body(std::true_type{});
        else body(std::false_type{});
        if (tabs) mbar_arrive(&bar.tab_free[h]);   // the half's grids have been read
        if (edge) {
          // bits 0..7 of the mask of the 16 queries from ql0
          const uint32_t vis = visible16(kj, qi * KIA_TILE + ql0, T, p.causal != 0);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const bool keep = (vis >> i) & 1u;
            v[i] = keep ? v[i] : 0.0f;
            gg[i] = keep ? gg[i] : 0.0f;
          }
        }
        if constexpr (!PROJ && !V::SOFTMAX) {
          // calibration terms for the chunk's queries whose argmax (argmin) key
          // lies in this warp's 32 keys (masks of the half's 32 queries, made
          // visibly warp-uniform; this thread's 8 bits)
          const int sh = 8 * part;
          const uint32_t bm =
              __shfl_sync(0xffffffffu, (sMask[((sl * 2 + 0) * 4 + quad) * 2 + h] >> sh) & 0xFFu, 0);
          const uint32_t bn = V::MINMAX
              ? __shfl_sync(0xffffffffu, (sMask[((sl * 2 + 1) * 4 + quad) * 2 + h] >> sh) & 0xFFu, 0)
              : 0u;
          tmem_st8(tmem + lane_addr + cS, v);
          tmem_st8(tmem + lane_addr + cP, gg);
          add_calibration_tmem(tmem + lane_addr + cP, bm, bn, sCM + e0, sCN + e0, r);
        } else {
          tmem_st8(tmem + lane_addr + cS, v);
          tmem_st8(tmem + lane_addr + cP, gg);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar.elem_done[h]);
        }
        if (failed) break;
        mbar_arrive(&bar.qc_free[sl]);
      }
      if (failed) break;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar.acc_full, n & 1, abort))) { failed = true; break; }
      tc_fence_after();
      // this thread's 32 columns of dV, then of dK (one at a time: registers)
      const uint32_t col = (uint32_t)(part * 32);
      float* stg = sStage + (warp - 2) * 256;
      const int row0 = kt * KIA_TILE + quad * 32;
      float acc[32];
      tmem_ld32(tmem + lane_addr + kColDV + col, acc);
      tmem_ld_wait_regs(acc);
#pragma unroll
      for (int pass = 0; pass < 4; ++pass)
        epilogue_store8(stg, &tmdV, acc + 8 * pass, 1.0f, lane, (int)col + 8 * pass, row0,
                        item_bh(it));
      tmem_ld32(tmem + lane_addr + kColDK + col, acc);
      tmem_ld_wait_regs(acc);
      tc_fence_before();
      mbar_arrive(&bar.acc_free);
#pragma unroll
      for (int pass = 0; pass < 4; ++pass)
        epilogue_store8(stg, &tmdK, acc + 8 * pass, 1.0f, lane, (int)col + 8 * pass, row0,
                        item_bh(it));
    }
    epilogue_store_drain();
  }
  if (failed || *abort) drain_in_flight();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

inline size_t tc_bwd_kv128_smem(const OpParams& p, bool tab_in_smem) {
  const int pair_floats = (!p.softmax && p.cal != KIA_CAL_MINMAX) ? 2 * (p.K + 1) : 0;
  const size_t tab = tab_in_smem ? 2 * 32 * (size_t)(p.K + 1) * 4 : 0;
  return 1024 + 128 * KIA_TILE * 4 + 4 * (size_t)kHalf128 + 2 * 64 * (16 + 16 + 8 + 8) +
         2 * 2 * 4 * 2 * 4 + kElemThreads / 32 * 1024 + (size_t)((pair_floats + 31) & ~31) * 4 +
         sizeof(BwdKV128Bars) + tab;
}

// The d = 128 backward: query pass, then key pass (the projection's scan
// pass runs after, as at d = 64).
template <class V>
int tc_backward128_v(const float* Q, const float* Kt, const float* Vv, const float* O,
                     const float* dO, const StatsView& st, const WorkView& wk, float* dQ, float* dK,
                     float* dV, float* dS_dbg, int B, int H, int T, const OpParams& p,
                     cudaStream_t s, void (*mark)(int, cudaStream_t)) {
  constexpr int D = 128;
  const int BH = B * H;
  CUtensorMap tkh, tkmh, tvh, tqh, tqmh, tgh, tgmh, tv, tdq, tdk, tdv;
  if (!make_tmap(&tkh, Kt, BH, T, D, false, 64) || !make_tmap(&tkmh, Kt, BH, T, D, true, 64) ||
      !make_tmap(&tvh, Vv, BH, T, D, false, 64) || !make_tmap(&tqh, Q, BH, T, D, false, 64) ||
      !make_tmap(&tqmh, Q, BH, T, D, true, 64) || !make_tmap(&tgh, dO, BH, T, D, false, 64) ||
      !make_tmap(&tgmh, dO, BH, T, D, true, 64) || !make_tmap(&tv, Vv, BH, T, D) ||
      !make_tmap_out(&tdq, dQ, BH, T, D) || !make_tmap_out(&tdk, dK, BH, T, D) ||
      !make_tmap_out(&tdv, dV, BH, T, D))
    return KIA_ERR_CUDA;
  // the rows' MinMax grids in shared memory where they fit, with the
  // MN-major K ring one slot shallower if that is what makes them fit
  const bool need_c = V::MINMAX && (p.grad == KIA_GRAD_FULL || p.grad == KIA_GRAD_MAX_ONLY ||
                                    p.grad == KIA_GRAD_MIN_ONLY);
  const bool proj = !V::SOFTMAX && p.grad == KIA_GRAD_PROJECT;
  const size_t kMaxQ = need_c ? dyn_smem_budget(tc_bwd_q128_kernel<V, true>)
                              : dyn_smem_budget(tc_bwd_q128_kernel<V, false>);
  const size_t kMaxK = proj ? dyn_smem_budget(tc_bwd_kv128_kernel<V, true>)
                            : dyn_smem_budget(tc_bwd_kv128_kernel<V, false>);
  bool q_tab = true;
  int nkmn = 2;
  if (tc_bwd_q128_smem(p, true, nkmn) > kMaxQ) nkmn = 1;
  if (tc_bwd_q128_smem(p, true, nkmn) > kMaxQ) {
    q_tab = false;
    nkmn = 2;
  }
  // the key pass holds two halves' query grids where they fit
  const bool kv_tab = !p.softmax && p.cal == KIA_CAL_MINMAX && tc_bwd_kv128_smem(p, true) <= kMaxK;
  const size_t smq = tc_bwd_q128_smem(p, q_tab, nkmn), smk = tc_bwd_kv128_smem(p, kv_tab);
  if (smq > kMaxQ || smk > kMaxK) return KIA_ERR_UNSUPPORTED;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  const int sms = num_sms();
  if (sms <= 0) return KIA_ERR_CUDA;
  const dim3 grid(std::min(sms, BH * nt));
  auto launch_q = [&](auto kern) -> int {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smq) !=
        cudaSuccess)
      return KIA_ERR_CUDA;
    kern<<<grid, kTcThreads, smq, s>>>(tkh, tkmh, tvh, tdq, Q, Kt, O, dO, st, wk, dS_dbg, p, B, H,
                                       T, q_tab ? 1 : 0, nkmn);
    return cudaGetLastError() == cudaSuccess ? KIA_OK : KIA_ERR_CUDA;
  };
  int rc = need_c ? launch_q(tc_bwd_q128_kernel<V, true>) : launch_q(tc_bwd_q128_kernel<V, false>);
  if (rc) return rc;
  mark(4, s);
  auto launch_kv = [&](auto kern) -> int {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smk) !=
        cudaSuccess)
      return KIA_ERR_CUDA;
    kern<<<grid, kTcThreads, smk, s>>>(tqh, tqmh, tgh, tgmh, tv, tdk, tdv, Kt, st, wk, p, BH, T,
                                       kv_tab ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? KIA_OK : KIA_ERR_CUDA;
  };
  rc = proj ? launch_kv(tc_bwd_kv128_kernel<V, true>) : launch_kv(tc_bwd_kv128_kernel<V, false>);
  if (rc) return rc;
  mark(5, s);
  return KIA_OK;
}

// Both head sizes: d = 64 runs the passes of kia_tc_bwd.cuh, d = 128 the ones
// above.
template <int D>
int tc_backward(const float* Q, const float* Kt, const float* V, const float* O, const float* dO,
                const StatsView& st, const WorkView& wk, float* dQ, float* dK, float* dV,
                float* dS_dbg, int B, int H, int T, const OpParams& p, cudaStream_t s,
                void (*mark)(int, cudaStream_t)) {
  return dispatch_variant(p, [&]<class Vt>() {
    if constexpr (D == 64)
      return tc_backward_v<D, Vt>(Q, Kt, V, O, dO, st, wk, dQ, dK, dV, dS_dbg, B, H, T, p, s,
                                  mark);
    else
      return tc_backward128_v<Vt>(Q, Kt, V, O, dO, st, wk, dQ, dK, dV, dS_dbg, B, H, T, p, s,
                                  mark);
  });
}

}  // namespace kia
