// kd_gemm.cuh -- persistent, warp-specialised tcgen05 GEMM for sm_100a with
// the loss epilogues fused in.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]          (fp32 accumulate in TMEM)
//
// One CTA per SM, 128x256 output tile, 128-byte-deep K stages fed by TMA with
// 128-byte swizzle, 4 stages, two TMEM accumulators (2 x 256 columns) so the
// epilogue of tile i overlaps the mainloop of tile i+1.
//   warp 0      : TMA producer (one thread)
//   warp 1      : TMEM allocator + MMA issuer (one thread)
//   warps 2..5  : epilogue; warp w reads TMEM lanes 32*(w%4) .. +31, one
//                 output row per thread, 32 columns per tcgen05.ld.
// Operands may be K-major (rows of K contiguous) or MN-major (rows of M/N
// contiguous); the UMMA descriptors and TMA boxes follow.
//
// Every wait is bounded (kd::mbar_wait); on a timeout or on an error recorded
// by another CTA, each role leaves its loop, the producer waits for its own
// copies in flight, the MMA thread for its own MMAs, and TMEM is freed.
#pragma once

#include "kd_common.cuh"

namespace kd {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int STAGES = 4;
constexpr int GEMM_THREADS = 192;
constexpr int ROW_BYTES = 128;                 // K depth of a stage, in bytes
constexpr int A_STAGE_BYTES = BM * ROW_BYTES;  // 16 KB
constexpr int B_STAGE_BYTES = BN * ROW_BYTES;  // 32 KB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int TMEM_COLS = 2 * BN;              // two accumulators
constexpr int EPI_WARPS = 4;
constexpr int EPI_BUF_BYTES = 32 * 128;        // one 32x32 fp32 (or 32x32 bf16) output box
constexpr int EPI_SMEM_BYTES = EPI_WARPS * 2 * EPI_BUF_BYTES;   // double-buffered per warp
constexpr int GEMM_SMEM_BYTES =
    STAGES * STAGE_BYTES + EPI_SMEM_BYTES + 1024 /*align*/ + 256 /*barriers*/;

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
__device__ __forceinline__ void run_epilogue(const GemmArgs& g, const CUtensorMap* tmC, int m_base,
                                             int nb, uint32_t taddr, int quad, int lane,
                                             unsigned char* boxes, int y_extra = 0) {
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
    }
  }
}

// ----------------------------------------------------------------------------
// The kernel.
// ----------------------------------------------------------------------------
template <typename Elem, int A_MN, int B_MN, int EPI>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmC, const GemmArgs g) {
  using C = ElemCfg<Elem>;
  constexpr int BK = C::BK;
  constexpr int INNER = ROW_BYTES / sizeof(Elem);        // MN elements per MN-major box
  constexpr int BOX_BYTES = ROW_BYTES * BK;               // one MN-major box
  constexpr uint32_t IDESC = umma_idesc(C::FMT, A_MN, B_MN, BM, BN);
  constexpr int KSTEPS = BK / C::UMMA_K;                  // MMAs per stage (4)

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sA = smem;
  unsigned char* sB = smem + STAGES * A_STAGE_BYTES;
  unsigned char* sEpi = smem + STAGES * STAGE_BYTES;      // [EPI_WARPS][2][EPI_BUF_BYTES]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + EPI_SMEM_BYTES);
  uint64_t* full = bars;                 // [STAGES]
  uint64_t* empty = bars + STAGES;       // [STAGES]
  uint64_t* tfull = bars + 2 * STAGES;   // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* drain = tempty + 2;          // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = g.m_tiles * g.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (EPI != EPI_FWD_LSE) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;                 // bit s: stage s has been armed
      uint32_t last_par = 0;              // bit s: parity of stage s's last arming
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int mb = g.m_fastest ? tile % g.m_tiles : tile / g.n_tiles;
        const int nb = g.m_fastest ? tile / g.m_tiles : tile % g.n_tiles;
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, g.wait_limit_ns, g.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          armed |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          unsigned char* a = sA + stage * A_STAGE_BYTES;
          unsigned char* b = sB + stage * B_STAGE_BYTES;
          if (A_MN) {
#pragma unroll
            for (int j = 0; j < BM / INNER; ++j)
              tma_load_2d(a + j * BOX_BYTES, &tmA, &full[stage], mb * BM + j * INNER, kb * BK);
          } else {
            tma_load_2d(a, &tmA, &full[stage], kb * BK, mb * BM);
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < BN / INNER; ++j)
              tma_load_2d(b + j * BOX_BYTES, &tmB, &full[stage], nb * BN + j * INNER, kb * BK);
          } else {
            tma_load_2d(b, &tmB, &full[stage], kb * BK, nb * BN);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Wait for every copy this thread started (no-op on the normal path).
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s)) mbar_drain(&full[s], (last_par >> s) & 1u, g.wait_limit_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, g.wait_limit_ns, g.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < g.k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, g.wait_limit_ns, g.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_STAGE_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * B_STAGE_BYTES);
#pragma unroll
          for (int k = 0; k < KSTEPS; ++k) {
            // K-major: advance 32 bytes inside the swizzled row (SBO = 8 rows);
            // MN-major: advance UMMA_K rows (LBO = next MN box, SBO = 8 rows).
            const uint64_t ad =
                A_MN ? umma_desc(a0 + k * C::UMMA_K * ROW_BYTES, BOX_BYTES, C::MN_SBO, C::MN_LAYOUT)
                     : umma_desc(a0 + k * 32, 16, 1024, UMMA_LAYOUT_SW128);
            const uint64_t bd =
                B_MN ? umma_desc(b0 + k * C::UMMA_K * ROW_BYTES, BOX_BYTES, C::MN_SBO, C::MN_LAYOUT)
                     : umma_desc(b0 + k * 32, 16, 1024, UMMA_LAYOUT_SW128);
            const uint32_t accum = (kb | k) != 0 ? 1u : 0u;
            if constexpr (C::FMT == 1) mma_f16(d_tmem, ad, bd, IDESC, accum);
            else mma_tf32(d_tmem, ad, bd, IDESC, accum);
          }
          mma_commit(&empty[stage]);        // frees the stage once these MMAs finish
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);            // accumulator ready for the epilogue
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // Wait for every MMA this thread issued before TMEM is released.
      mma_commit(drain);
      mbar_drain(drain, 0, g.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    unsigned char* boxes = sEpi + (warp - 2) * 2 * EPI_BUF_BYTES;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mb = g.m_fastest ? tile % g.m_tiles : tile / g.n_tiles;
      const int nb = g.m_fastest ? tile / g.m_tiles : tile % g.n_tiles;
      if (!mbar_wait(&tfull[acc], acc_phase, g.wait_limit_ns, g.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      run_epilogue<Elem, EPI>(g, &tmC, mb * BM, nb, taddr, quad, lane, boxes);
      __syncwarp();
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    // Every output box must have left shared memory and landed before exit.
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace kd
