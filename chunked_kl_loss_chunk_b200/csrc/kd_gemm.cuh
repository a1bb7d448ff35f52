// kd_gemm.cuh -- what the tensor-core GEMM kernels of libkd share: tile
// constants, per-dtype MMA parameters, launch arguments, and the loss
// epilogues that drain an accumulator from TMEM.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]          (fp32 accumulate in TMEM)
//
// Output tiles are 256 columns wide; each CTA owns 128 accumulator rows and
// four epilogue warps, warp w reading TMEM lanes 32*(w%4) .. +31 (one output
// row per thread, 32 columns per tcgen05.ld).  Operands may be K-major (rows
// of K contiguous) or MN-major (rows of M/N contiguous).  The kernel itself is
// in kd_gemm2.cuh.
#pragma once

#include "kd_common.cuh"

namespace kd {

constexpr int BM = 128;                        // accumulator rows per CTA
constexpr int BN = 256;                        // output tile columns
constexpr int GEMM_THREADS = 192;              // TMA warp, MMA warp, 4 epilogue warps
constexpr int ROW_BYTES = 128;                 // K depth of a stage, in bytes
constexpr int TMEM_COLS = 2 * BN;              // two accumulators
constexpr int EPI_WARPS = 4;
constexpr int EPI_BUF_BYTES = 32 * 128;        // one 32x32 fp32 (or 32x32 bf16) output box
constexpr int EPI_SMEM_BYTES = EPI_WARPS * 2 * EPI_BUF_BYTES;   // double-buffered per warp

template <typename Elem>
struct ElemCfg;
template <>
struct ElemCfg<__nv_bfloat16> {
  static constexpr int BK = 64;        // elements per 128-byte row
  static constexpr int UMMA_K = 16;    // K per MMA instruction
  static constexpr uint32_t FMT = 1;   // bf16
  // MN-major operands: 128-byte swizzle, 8-row atoms of 1024 bytes
  static constexpr uint64_t MN_LAYOUT = UMMA_LAYOUT_SW128;
  static constexpr uint32_t MN_SBO = 1024;
};
template <>
struct ElemCfg<float> {
  static constexpr int BK = 32;
  static constexpr int UMMA_K = 8;
  static constexpr uint32_t FMT = 2;   // tf32
  // MN-major tf32 operands: 128-byte swizzle with 32-byte chunks, 4-row atoms
  static constexpr uint64_t MN_LAYOUT = UMMA_LAYOUT_SW128_ATOM32;
  static constexpr uint32_t MN_SBO = 512;
};

enum EpiKind : int {
  EPI_FWD_LSE = 0,        // logsumexp / gather partials per (row, vocabulary tile)
  EPI_BWD_DZ = 1,         // dz boxes
  EPI_STORE_H = 2,        // dH boxes in the dtype of h
  EPI_ACCUM_W = 3,        // fp32 dW boxes, stored or added
  EPI_STORE_PARTIAL = 4   // fp32 boxes of one K-split's partial dH
};

struct GemmArgs {
  int32_t M, N, K;
  int32_t m_tiles, n_tiles, k_blocks;
  int32_t m_fastest;          // tile raster: 1 = m index varies fastest
  // ---- epilogue inputs / outputs ----
  int64_t row0;               // global position of output row m = 0 (loss rows)
  int64_t V;
  int32_t Ktop;               // teacher entries per row
  float zscale;               // log2(e) / tau
  const int32_t* idx_sorted;  // [T, Ktop], ascending per row
  const float* p_sorted;      // [T, Ktop]
  const float2* row_stats;    // [T]: (S = sum p, sum p log p)
  float4* partials;           // fwd: [M, n_tiles] (max z, sum exp2((z-max) zscale), gather, -)
  const float* lse;           // bwd: [T]
  const float* grad_loss;     // bwd: device scalar or null (1)
  float inv_T_tau;            // 1 / (T tau)
  void* out;                  // dz [M, ldo] | dH rows | dW
  int64_t ldo;                // leading dimension of `out`, elements
  int32_t accumulate;         // dW: add into `out`
  int32_t k_split;            // K ranges per output tile (1 = no split)
  int32_t split_rows;         // EPI_STORE_PARTIAL: rows between consecutive splits' partials
  uint32_t* status;
  uint64_t wait_limit_ns;
};

// ----------------------------------------------------------------------------
// Output boxes.  An epilogue warp owns 32 accumulator rows; every 32-column
// block of its rows is converted, written to a shared-memory box in the TMA
// swizzle of the output tensor map, and sent out by one lane with a TMA store
// (or, for accumulating fp32 output, a TMA add-reduction).  Two boxes per warp
// alternate so that writing one overlaps the transfer of the other.
//   fp32 box: 32 rows x 128 B, 128-byte swizzle (16-byte chunk j of row r at
//             chunk j ^ (r & 7));
//   bf16 box: 32 rows x  64 B,  64-byte swizzle (chunk j of row r at
//             chunk j ^ ((r >> 1) & 3)).
// Both layouts spread a warp's 16-byte writes over all 32 banks.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void stage_box_f32(unsigned char* box, int r, const float* v) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<float4*>(box + r * 128 + ((j ^ (r & 7)) << 4)) =
        make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

__device__ __forceinline__ void stage_box_bf16(unsigned char* box, int r, const float* v) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 q;
    q.x = pack_bf16x2(v[8 * j + 0], v[8 * j + 1]);
    q.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
    q.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
    q.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
    *reinterpret_cast<uint4*>(box + r * 64 + ((j ^ ((r >> 1) & 3)) << 4)) = q;
  }
}

// Hands one staged box to TMA.  Called by every lane of the warp.
template <typename OutT>
__device__ __forceinline__ void emit_box(const CUtensorMap* tmC, unsigned char* box, int x, int y,
                                         bool reduce_add) {
  fence_proxy_async_smem();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) {
    if (reduce_add) tma_reduce_add_2d(tmC, box, x, y); else tma_store_2d(tmC, box, x, y);
    bulk_commit();
  }
}

// Before reusing a box: the transfer issued from it two blocks ago has read it.
__device__ __forceinline__ void box_reuse_wait() {
  if ((threadIdx.x & 31) == 0) bulk_wait_read<1>();
  __syncwarp();
}

// First position in the ascending list ids[0..K) holding a value >= key.
__device__ __forceinline__ int lower_bound_i32(const int32_t* ids, int K, int32_t key) {
  int lo = 0, hi = K;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(ids + mid) < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// ----------------------------------------------------------------------------
// Epilogues.  Called by the 128 epilogue threads; `taddr` addresses this
// warp's 32 TMEM lanes at the tile's first accumulator column; `boxes` is the
// warp's pair of output boxes.  Every lane of a warp executes the same sequence
// of tcgen05.ld (they are warp-collective).
// ----------------------------------------------------------------------------
template <typename Elem, int EPI>
// pace_ns (EPI_ACCUM_W): pause between two output boxes of a warp, so that a
// tile's fp32 dW boxes go out spread over the next tile's mainloop.
__device__ __forceinline__ void run_epilogue(const GemmArgs& g, const CUtensorMap* tmC, int m_base,
                                             int nb, uint32_t taddr, int quad, int lane,
                                             unsigned char* boxes, int y_extra = 0,
                                             uint32_t pace_ns = 0) {
  const int r = quad * 32 + lane;         // accumulator row of this thread
  const int m = m_base + r;               // output row within the problem
  const bool row_ok = m < g.M;
  const int n0 = nb * BN;
  const int y_box = y_extra + m_base + quad * 32;  // first output row of this warp's boxes

  if constexpr (EPI == EPI_FWD_LSE || EPI == EPI_BWD_DZ) {
    const int64_t t = g.row0 + m;         // global position
    const int32_t* ids = g.idx_sorted + t * g.Ktop;
    const float* ps = g.p_sorted + t * g.Ktop;
    int ptr = g.Ktop;
    if (row_ok) ptr = lower_bound_i32(ids, g.Ktop, n0);
    int32_t nidx = ptr < g.Ktop ? __ldg(ids + ptr) : INT32_MAX;
    float np = ptr < g.Ktop ? __ldg(ps + ptr) : 0.f;
    const float zs = g.zscale;

    if constexpr (EPI == EPI_FWD_LSE) {
      float run_m = -INFINITY, run_s = 0.f, gat = 0.f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int base = n0 + c * 32;
        if (base >= g.V) break;                       // uniform across the warp
        float v[32];
        __syncwarp();
        tmem_ld32(taddr + c * 32, v);
        if (base + 32 > g.V) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (base + j >= g.V) v[j] = -INFINITY;
        }
        if (nidx < base + 32) {                       // teacher index in this block
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (nidx == base + j) {
              gat = fmaf(np, v[j], gat);
              ++ptr;
              nidx = ptr < g.Ktop ? __ldg(ids + ptr) : INT32_MAX;
              np = ptr < g.Ktop ? __ldg(ps + ptr) : 0.f;
            }
          }
        }
        float bm = v[0];
#pragma unroll
        for (int j = 1; j < 32; ++j) bm = fmaxf(bm, v[j]);
        const float nm = fmaxf(run_m, bm);
        if (nm != -INFINITY) {
          const float off = -nm * zs;
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) s += ex2_approx(fmaf(v[j], zs, off));
          run_s = run_s * ex2_approx((run_m - nm) * zs) + s;
          run_m = nm;
        }
      }
      // every cached index inside this tile's columns was gathered
      KD_CHECK(!row_ok || static_cast<int64_t>(nidx) >= (n0 + BN < g.V ? n0 + BN : g.V), g.status);
      if (row_ok) g.partials[static_cast<int64_t>(m) * g.n_tiles + nb] =
          make_float4(run_m, run_s, gat, 0.f);
    } else {  // EPI_BWD_DZ: dz box per 32 columns; TMA clips columns >= V, rows >= M
      const float gl = g.grad_loss ? __ldg(g.grad_loss) : 1.f;
      const float coef = gl * g.inv_T_tau;
      float coefA = 0.f, off = 0.f;
      if (row_ok) {
        coefA = coef * g.row_stats[t].x;
        off = -__ldg(g.lse + t) * 1.4426950408889634f;   // -LSE * log2(e)
      }
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int base = n0 + c * 32;
        if (base >= g.V) break;
        unsigned char* box = boxes + (c & 1) * EPI_BUF_BYTES;
        box_reuse_wait();
        float v[32];
        tmem_ld32(taddr + c * 32, v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = coefA * ex2_approx(fmaf(v[j], zs, off));
        if (nidx < base + 32) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (nidx == base + j) {
              v[j] = fmaf(-coef, np, v[j]);
              ++ptr;
              nidx = ptr < g.Ktop ? __ldg(ids + ptr) : INT32_MAX;
              np = ptr < g.Ktop ? __ldg(ps + ptr) : 0.f;
            }
          }
        }
        if constexpr (sizeof(Elem) == 4) stage_box_f32(box, lane, v);
        else stage_box_bf16(box, lane, v);
        emit_box<Elem>(tmC, box, base, y_box, false);
      }
      KD_CHECK(!row_ok || static_cast<int64_t>(nidx) >= (n0 + BN < g.V ? n0 + BN : g.V), g.status);
    }
  } else {  // EPI_STORE_H (dtype of h), EPI_STORE_PARTIAL (fp32) or EPI_ACCUM_W (fp32)
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      const int base = n0 + c * 32;
      if (base >= g.N) break;
      unsigned char* box = boxes + (c & 1) * EPI_BUF_BYTES;
      box_reuse_wait();
      float v[32];
      tmem_ld32(taddr + c * 32, v);
      if constexpr (EPI == EPI_STORE_H && sizeof(Elem) == 2) stage_box_bf16(box, lane, v);
      else stage_box_f32(box, lane, v);
      emit_box<Elem>(tmC, box, base, y_box, EPI == EPI_ACCUM_W && g.accumulate);
      if (EPI == EPI_ACCUM_W && pace_ns) __nanosleep(pace_ns);
    }
  }
}

}  // namespace kd
