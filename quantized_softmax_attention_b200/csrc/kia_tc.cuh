// Tensor-core (tcgen05, kind::tf32) path: host-side tensor maps and the
// score-tile kernel behind kiattn_scores.  The fused forward and backward
// kernels are in kia_tc_fwd.cuh / kia_tc_bwd.cuh.
//
// Shared-memory operand tiles: a [128 rows x d] fp32 tile is stored as d/32
// column blocks of [128 rows x 32 fp32] (128 B per row, 16 KB per block).
// Two swizzles, both written by TMA from the same [B*H, T, d] tensor:
//  * K-major (the contraction runs over d, rows are M or N): 128-byte
//    swizzle of 16-byte atoms, 8-row groups 1024 B apart;
//  * MN-major (the contraction runs over the rows): tf32 operands must use
//    the 128-byte swizzle of 32-byte atoms, 4-row groups 512 B apart, column
//    blocks 16 KB apart.
// A tile used both ways (Q, dO, K in the backward) is loaded once per layout.
#pragma once
#include <cuda.h>

#include "kia_elem.cuh"
#include "kia_stats.cuh"

namespace kia {

constexpr uint32_t kBlockBytes = KIA_TILE * 128;  // one [128 x 32] fp32 column block

// ------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Number of SMs of the current device (cached per device; 0 on error).
// Dynamic shared memory a launch of `kern` may request: the device's opt-in
// per-block maximum less the kernel's own static shared memory (0 if either
// cannot be read).  Sizes are checked against this rather than the device
// maximum alone, which a kernel with static shared variables cannot reach.
template <class F>
inline size_t dyn_smem_budget(F* kern) {
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return 0;
  cudaFuncAttributes a;
  if (cudaFuncGetAttributes(&a, kern) != cudaSuccess) return 0;
  return optin > (int)a.sharedSizeBytes ? (size_t)optin - a.sharedSizeBytes : 0;
}

inline int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

// [BH, T, d] fp32 tensor; box = 32 columns x box_rows rows x 1, 128-byte swizzle
// (16-byte atoms for K-major use, 32-byte atoms for MN-major use),
// out-of-range rows read as zero.
inline bool make_tmap(CUtensorMap* m, const float* base, int BH, int T, int d,
                      bool mn_major = false, int box_rows = KIA_TILE) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)T * d * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            mn_major ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map for the epilogues' TMA stores: [BH, T, d] fp32, box = 8
// columns x 32 rows, no swizzle (a warp's staged block, row-major).  Rows past
// T are not written.
inline bool make_tmap_out(CUtensorMap* m, const float* base, int BH, int T, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)T * d * 4};
  cuuint32_t box[3] = {8, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// One warp writes 32 rows x 8 columns of an output: each lane puts its row's
// eight values (times `scale`) into the warp's 1 KB staging block, and one
// elected lane stores the block with TMA at (x, y, z) -- the copy engine
// writes whole lines, and no thread waits on global memory.  The block is
// rewritten only after the previous store has read it.  The elected lane is
// the same on every call (all lanes active), so its bulk groups cover every
// store of the warp; epilogue_store_drain() waits for them before exit.
__device__ __forceinline__ void epilogue_store8(float* stg, const CUtensorMap* tm,
                                                const float* src8, float scale, int lane, int x,
                                                int y, int z) {
  if (elect_one()) tma_store_wait_read();
  __syncwarp();
  *reinterpret_cast<float4*>(stg + lane * 8) =
      make_float4(src8[0] * scale, src8[1] * scale, src8[2] * scale, src8[3] * scale);
  *reinterpret_cast<float4*>(stg + lane * 8 + 4) =
      make_float4(src8[4] * scale, src8[5] * scale, src8[6] * scale, src8[7] * scale);
  fence_proxy_async_smem();
  __syncwarp();
  if (elect_one()) {
    tma_store_3d(tm, stg, x, y, z);
    tma_store_commit();
  }
  __syncwarp();
}
__device__ __forceinline__ void epilogue_store_drain() {
  if (elect_one()) tma_store_wait_all();
  __syncwarp();
}

// ------------------------------------------------------ descriptor helpers

// K-major operand, 8-element (32-byte) K step ks of a tile at smem address
// `tile`: column block ks / 4, byte offset (ks % 4) * 32 inside the 128-byte
// swizzle row.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int ks) {
  return smem_desc(tile + (uint32_t)(ks >> 2) * kBlockBytes + (uint32_t)(ks & 3) * 32u, 16u, 1024u,
                   kLayoutSW128);
}
// MN-major operand (32-byte-atom swizzle), K step ks = rows 8ks..8ks+7
// (1024 B); two 4-row groups 512 B apart, column blocks 16 KB apart.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int ks) {
  return smem_desc(tile + (uint32_t)ks * 1024u, kBlockBytes, 512u, kLayoutSW128Atom32);
}

// The start address sits in the descriptor's low 14 bits in 16-byte units
// and never carries out of them (shared memory < 256 KB), so a descriptor
// moves to another operand or K step by adding the byte offset / 16.  The
// MMA issuer builds one descriptor per tile and steps it with these.
__host__ __device__ constexpr uint64_t desc_step(uint32_t bytes) { return bytes >> 4; }
// K-major: K step ks of a tile (column block ks / 4, 32 bytes per step inside it)
__host__ __device__ constexpr uint64_t kstep_kmajor(int ks) {
  return desc_step((uint32_t)(ks >> 2) * kBlockBytes + (uint32_t)(ks & 3) * 32u);
}
// MN-major: K step ks = rows 8ks..8ks+7
__host__ __device__ constexpr uint64_t kstep_mnmajor(int ks) { return desc_step((uint32_t)ks * 1024u); }

// Half tiles (64 rows, loaded with a 64-row box): column blocks are 8 KB
// apart instead of 16 KB.
constexpr uint32_t kHalfBlockBytes = 64 * 128;
__device__ __forceinline__ uint64_t desc_kmajor_half(uint32_t tile) {
  return smem_desc(tile, 16u, 1024u, kLayoutSW128);
}
__host__ __device__ constexpr uint64_t kstep_kmajor_half(int ks) {
  return desc_step((uint32_t)(ks >> 2) * kHalfBlockBytes + (uint32_t)(ks & 3) * 32u);
}
__device__ __forceinline__ uint64_t desc_mnmajor_half(uint32_t tile) {
  return smem_desc(tile, kHalfBlockBytes, 512u, kLayoutSW128Atom32);
}

// ------------------------------------------------------ score tile kernel

template <int D>
struct ScoresSmem {
  float q[D * KIA_TILE];
  float k[D * KIA_TILE];
  uint64_t bar_tma;
  uint64_t bar_mma;
  uint32_t tmem_base;
  int abort;
};

// One 128 x 128 score tile per CTA (4 warps).  Thread t of the CTA owns
// TMEM lane t = query row t of the tile.
template <int D>
__global__ void __launch_bounds__(128)
tc_scores_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 float* __restrict__ S, OpParams p, int T) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  ScoresSmem<D>& sm = *reinterpret_cast<ScoresSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
  const int qt = blockIdx.x, kt = blockIdx.y, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int row = qt * KIA_TILE + threadIdx.x;
  const bool skip = p.causal && kt > qt;
  if (skip) {
    if (row < T) {
      float* dst = S + ((size_t)bh * T + row) * T + (size_t)kt * KIA_TILE;
      for (int c = 0; c < KIA_TILE && kt * KIA_TILE + c < T; ++c) dst[c] = 0.0f;
    }
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_tma, 1);
    mbar_init(&sm.bar_mma, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    mbar_arrive_expect_tx(&sm.bar_tma, 2u * D * KIA_TILE * 4u);
#pragma unroll
    for (int b = 0; b < D / 32; ++b) {
      tma_load_3d(sm.q + b * 32 * KIA_TILE, &tmQ, &sm.bar_tma, b * 32, qt * KIA_TILE, bh);
      tma_load_3d(sm.k + b * 32 * KIA_TILE, &tmK, &sm.bar_tma, b * 32, kt * KIA_TILE, bh);
    }
    if (mbar_wait(&sm.bar_tma, 0, abort)) {
      tc_fence_after();
      const uint32_t idesc = idesc_tf32(128, 128, 0, 0);
      const uint32_t qa = smem_u32(sm.q), ka = smem_u32(sm.k);
#pragma unroll
      for (int ks = 0; ks < D / 8; ++ks)
        mma_tf32_ss(tmem, desc_kmajor(qa, ks), desc_kmajor(ka, ks), idesc, ks > 0 ? 1u : 0u);
      tc_commit(&sm.bar_mma);
    }
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.bar_mma, 0, abort));
  tc_fence_after();
  if (ok) {
    float v[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(c * 32), v);
      tmem_ld_wait();
      if (row < T) {
        float* dst = S + ((size_t)bh * T + row) * T;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int key = kt * KIA_TILE + c * 32 + i;
          if (key < T) dst[key] = (p.causal && key > row) ? 0.0f : v[i];
        }
      }
    }
  } else {
    drain_in_flight();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

template <int D>
int tc_scores(const float* Q, const float* Kt, float* S, int B, int H, int T, const OpParams& p,
              cudaStream_t s) {
  CUtensorMap tq, tk;
  if (!make_tmap(&tq, Q, B * H, T, D) || !make_tmap(&tk, Kt, B * H, T, D)) return KIA_ERR_CUDA;
  const size_t smem = sizeof(ScoresSmem<D>) + 1024;
  if (cudaFuncSetAttribute(tc_scores_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return KIA_ERR_CUDA;
  const int nt = (T + KIA_TILE - 1) / KIA_TILE;
  dim3 grid(nt, nt, B * H);
  tc_scores_kernel<D><<<grid, 128, smem, s>>>(tq, tk, S, p, T);
  return cudaGetLastError() == cudaSuccess ? KIA_OK : KIA_ERR_CUDA;
}

// Exact-fp32 scores (same dot-product order as the exact path's kernels).
template <int D>
__global__ void simt_scores_kernel(const float* __restrict__ Q, const float* __restrict__ Kt,
                                   float* __restrict__ S, OpParams p, int T) {
  const int bh = blockIdx.y;
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (long long)T * T) return;
  const int i = (int)(e / T), j = (int)(e % T);
  const float* q = Q + ((size_t)bh * T + i) * D;
  const float* k = Kt + ((size_t)bh * T + j) * D;
  float s = 0.0f;
  for (int c = 0; c < D; ++c) s = fmaf(q[c], k[c], s);
  S[(size_t)bh * T * T + e] = (p.causal && j > i) ? 0.0f : s;
}

template <int D>
int simt_scores(const float* Q, const float* Kt, float* S, int B, int H, int T, const OpParams& p,
                cudaStream_t s) {
  dim3 grid((unsigned)(((long long)T * T + 255) / 256), B * H);
  simt_scores_kernel<D><<<grid, 256, 0, s>>>(Q, Kt, S, p, T);
  return cudaGetLastError() == cudaSuccess ? KIA_OK : KIA_ERR_CUDA;
}

// Fused kernels: filled in by kia_tc_fwd.cuh / kia_tc_bwd.cuh.
template <int D>
int tc_forward(const float* Q, const float* Kt, const float* V, float* O, void* stats, int B,
               int H, int T, const OpParams& p, cudaStream_t s);
template <int D>
int tc_backward(const float* Q, const float* Kt, const float* V, const float* O, const float* dO,
                const StatsView& st, const WorkView& wk, float* dQ, float* dK, float* dV,
                float* dS_dbg, int B, int H, int T, const OpParams& p, cudaStream_t s,
                void (*mark)(int, cudaStream_t));

}  // namespace kia

#include "kia_tc_fwd.cuh"
#include "kia_tc_bwd.cuh"
#include "kia_tc_bwd128.cuh"
