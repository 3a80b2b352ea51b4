// Layout of the per-row statistics buffer written by the forward and read by
// the backward, and of the backward's workspace.  Everything is struct-of-
// arrays over the B*H*T rows, each array starting on a 256-byte boundary.
#pragma once
#include <stddef.h>
#include <stdint.h>

#include "kia_common.cuh"

namespace kia {

constexpr uint32_t kStatsMagic = 0x4b494131u;  // "KIA1"
constexpr int kHeaderWords = 64;

struct StatsView {
  uint32_t* header;  // kHeaderWords words: magic, shape, config
  float* m;          // row max
  float* n;          // row min
  int* am;           // lowest index of the row max
  int* an;           // lowest index of the row min
  float* rh;         // K / span (MinMax) or K / tau (FWM); 0 marks a degenerate row
  float* h;          // span / K or tau / K; 0 marks a degenerate row
  float* Wf;         // normaliser of the forward probabilities
  float* Wb;         // normaliser at the backward's normalisation point
  float* table;      // grid G_0..G_K: per row [rows][K+1] (MinMax) or one [K+1] (FWM)
  float* OL;         // LERP-point output [rows][d] (Nearest + Prob-STE only), else null
};

struct WorkView {
  float* D;     // centering dO . O_bar per row
  float* A;     // row sum of dw * a_k
  float* C;     // row sum of dw * (b - a_k u / h)
  float* gm;    // calibration coefficient added at the argmax key (or the projection shift)
  float* gn;    // calibration coefficient added at the argmin key
  int* am;      // argmax key of the row (the calibration target)
  int* an;      // argmin key of the row
  int* status;  // 0 = stats header matched the call, 1 = mismatch (kernels skip)
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct StatsLayout {
  size_t off_m, off_n, off_am, off_an, off_rh, off_h, off_Wf, off_Wb, off_table, off_OL, total;
};

__host__ __device__ inline StatsLayout stats_layout(long long rows, int d, const OpParams& p) {
  StatsLayout L;
  size_t o = align256(kHeaderWords * sizeof(uint32_t));
  const size_t r4 = align256((size_t)rows * 4);
  L.off_m = o; o += r4;
  L.off_n = o; o += r4;
  L.off_am = o; o += r4;
  L.off_an = o; o += r4;
  L.off_rh = o; o += r4;
  L.off_h = o; o += r4;
  L.off_Wf = o; o += r4;
  L.off_Wb = o; o += r4;
  L.off_table = o;
  if (!p.softmax) {
    const size_t nt = (p.cal == KIA_CAL_MINMAX) ? (size_t)rows * (p.K + 1) : (size_t)(p.K + 1);
    o += align256(nt * 4);
  }
  L.off_OL = o;
  if (needs_OL(p)) o += align256((size_t)rows * d * 4);
  L.total = o;
  return L;
}

__host__ __device__ inline StatsView stats_view(void* base, long long rows, int d,
                                               const OpParams& p) {
  const StatsLayout L = stats_layout(rows, d, p);
  char* b = static_cast<char*>(base);
  StatsView v;
  v.header = reinterpret_cast<uint32_t*>(b);
  v.m = reinterpret_cast<float*>(b + L.off_m);
  v.n = reinterpret_cast<float*>(b + L.off_n);
  v.am = reinterpret_cast<int*>(b + L.off_am);
  v.an = reinterpret_cast<int*>(b + L.off_an);
  v.rh = reinterpret_cast<float*>(b + L.off_rh);
  v.h = reinterpret_cast<float*>(b + L.off_h);
  v.Wf = reinterpret_cast<float*>(b + L.off_Wf);
  v.Wb = reinterpret_cast<float*>(b + L.off_Wb);
  v.table = p.softmax ? nullptr : reinterpret_cast<float*>(b + L.off_table);
  v.OL = needs_OL(p) ? reinterpret_cast<float*>(b + L.off_OL) : nullptr;
  return v;
}

constexpr int kWorkArrays = 7;
__host__ __device__ constexpr size_t work_bytes_c(long long rows) {
  return kWorkArrays * (((size_t)rows * 4 + 255) & ~size_t(255)) + 256;
}
__host__ __device__ inline size_t work_bytes(long long rows) { return work_bytes_c(rows); }

__host__ __device__ inline WorkView work_view(void* base, long long rows) {
  char* b = static_cast<char*>(base);
  const size_t r4 = align256((size_t)rows * 4);
  WorkView w;
  w.D = reinterpret_cast<float*>(b);
  w.A = reinterpret_cast<float*>(b + r4);
  w.C = reinterpret_cast<float*>(b + 2 * r4);
  w.gm = reinterpret_cast<float*>(b + 3 * r4);
  w.gn = reinterpret_cast<float*>(b + 4 * r4);
  w.am = reinterpret_cast<int*>(b + 5 * r4);
  w.an = reinterpret_cast<int*>(b + 6 * r4);
  w.status = reinterpret_cast<int*>(b + 7 * r4);
  return w;
}

// Header words (written by the forward, checked by the backward).
enum HeaderWord {
  HW_MAGIC = 0, HW_B, HW_H, HW_T, HW_D, HW_K, HW_CAL, HW_REC, HW_STE, HW_CAUSAL, HW_OP,
  HW_TAU_BITS, HW_COUNT
};

__device__ inline void write_header(uint32_t* hdr, int B, int H, int T, int d, const OpParams& p) {
  hdr[HW_B] = B; hdr[HW_H] = H; hdr[HW_T] = T; hdr[HW_D] = d; hdr[HW_K] = p.K;
  hdr[HW_CAL] = p.fixed_step ? KIA_CAL_FIXED : p.cal; hdr[HW_REC] = p.rec; hdr[HW_STE] = p.ste; hdr[HW_CAUSAL] = p.causal;
  hdr[HW_OP] = p.softmax ? 1 + p.exp_round : 0; hdr[HW_TAU_BITS] = __float_as_uint(p.tau);
  __threadfence();
  hdr[HW_MAGIC] = kStatsMagic;
}

__device__ inline bool header_matches(const uint32_t* hdr, int B, int H, int T, int d,
                                      const OpParams& p) {
  return hdr[HW_MAGIC] == kStatsMagic && hdr[HW_B] == (uint32_t)B && hdr[HW_H] == (uint32_t)H &&
         hdr[HW_T] == (uint32_t)T && hdr[HW_D] == (uint32_t)d && hdr[HW_K] == (uint32_t)p.K &&
         hdr[HW_CAL] == (uint32_t)(p.fixed_step ? KIA_CAL_FIXED : p.cal) &&
         hdr[HW_REC] == (uint32_t)p.rec &&
         (p.rec == KIA_REC_LERP || hdr[HW_STE] == (uint32_t)p.ste) &&
         hdr[HW_CAUSAL] == (uint32_t)p.causal && hdr[HW_OP] == (uint32_t)(p.softmax ? 1 + p.exp_round : 0) &&
         hdr[HW_TAU_BITS] == __float_as_uint(p.tau);
}

}  // namespace kia
