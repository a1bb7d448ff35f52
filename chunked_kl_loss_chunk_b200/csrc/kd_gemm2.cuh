// kd_gemm2.cuh -- the same GEMM on SM pairs: tcgen05 cta_group::2.
//
// A cluster of two CTAs (two SMs) computes one 256x256 output tile:
//   CTA r (r = 0 leader, 1 peer) loads rows [r*128, r*128+128) of the tile's A
//   slab and rows [r*128, r*128+128) of its B slab (its half of N), each with
//   its own TMA loads (no multicast), whose byte counts complete on the
//   leader's stage barrier;
//   the leader's MMA thread issues tcgen05.mma.cta_group::2 (M=256, N=256),
//   which reads both CTAs' shared memory and accumulates rows r*128.. of the
//   tile into CTA r's TMEM;
//   the leader's commits arrive on the stage-free and accumulator-ready
//   barriers of both CTAs; both CTAs' epilogue warps read their own TMEM and
//   arrive on the leader's accumulator-free barrier.
// Per CTA a stage holds 16 KB of A and 16 KB of B (vs 48 KB for a 128x256 tile
// on one SM), so six stages fit and each SM pulls a third less operand data
// through L2 per flop.
//
// Tiles (and, with k_split > 1, K ranges) go to clusters round-robin; each
// role of a cluster walks its units without division (kd_unitwalk.h).  Every
// wait is bounded; on a timeout each role leaves its loop, the leader waits for
// the copies and MMAs it accounted for, and both CTAs meet at a cluster
// barrier before TMEM is freed.
#pragma once

#include "kd_gemm.cuh"
#include "kd_unitwalk.h"

namespace kd {

constexpr int STAGES2 = 6;
constexpr int HALF_BYTES = 128 * ROW_BYTES;          // 16 KB: 128 rows of one operand
constexpr int STAGE2_BYTES = 2 * HALF_BYTES;         // A half + B half, per CTA
constexpr int GEMM2_SMEM_BYTES = STAGES2 * STAGE2_BYTES + EPI_SMEM_BYTES + 1024 + 256;
constexpr int BM2 = 256;                              // tile rows per CTA pair

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}

// Address of the same shared-memory object in the cluster CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// All threads of both CTAs.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// TMA load into this CTA's shared memory whose bytes complete on the barrier
// at cluster address `bar_cluster` (the leader's).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc2(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void mma2_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma2_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once, when this thread's MMAs are done, on the barrier at this
// shared-memory offset in both CTAs of the pair (CTA mask 0b11).
__device__ __forceinline__ void mma2_commit_pair(uint64_t* bar) {
  const uint16_t mask = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}
// Same, on this CTA's barrier only.
__device__ __forceinline__ void mma2_commit_local(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// A cluster's walk over its work units (kd_unitwalk.h), started at unit cid.
__device__ __forceinline__ void walk_start(UnitWalk& w, const GemmArgs& g, int m_tiles2, int cid,
                                           int ncl) {
  walk_begin(w, m_tiles2, g.n_tiles, g.m_fastest, g.k_blocks, g.k_split, cid, ncl);
}

// Debug build: the walk's unit against its direct coordinates.
__device__ __forceinline__ void walk_check(const UnitWalk& w, const GemmArgs& g, int m_tiles2) {
  if (KD_DEBUG) {
    int s, m, n;
    unit_coords_direct(m_tiles2, g.n_tiles, g.m_fastest, w.u, s, m, n);
    KD_CHECK(s == w.split && m == w.mb2 && n == w.nb && s < g.k_split && m < m_tiles2 &&
                 n < g.n_tiles && w.kb0 == split_first_kblock(g.k_blocks, g.k_split, s) &&
                 w.kb1 == split_first_kblock(g.k_blocks, g.k_split, s + 1),
             g.status);
  }
}

template <typename Elem, int A_MN, int B_MN, int EPI>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const __grid_constant__ CUtensorMap tmC, const GemmArgs g) {
  using C = ElemCfg<Elem>;
  constexpr int BK = C::BK;
  constexpr int INNER = ROW_BYTES / sizeof(Elem);
  constexpr int BOX_BYTES = ROW_BYTES * BK;
  constexpr uint32_t IDESC = umma_idesc(C::FMT, A_MN, B_MN, BM2, BN);
  constexpr int KSTEPS = BK / C::UMMA_K;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sA = smem;                                   // [STAGES2][HALF_BYTES]
  unsigned char* sB = smem + STAGES2 * HALF_BYTES;            // [STAGES2][HALF_BYTES]
  unsigned char* sEpi = smem + STAGES2 * STAGE2_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + EPI_SMEM_BYTES);
  uint64_t* full = bars;                     // [STAGES2] (leader's used)
  uint64_t* empty = bars + STAGES2;          // [STAGES2] (both)
  uint64_t* tfull = bars + 2 * STAGES2;      // [2] (both)
  uint64_t* tempty = tfull + 2;              // [2] (leader's used)
  uint64_t* drain = tempty + 2;              // [1] (leader)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(cluster_count_x());
  const int m_tiles2 = (g.M + BM2 - 1) / BM2;
  const int units = m_tiles2 * g.n_tiles * g.k_split;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * EPI_WARPS);      // one lane per epilogue warp, both CTAs
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (EPI != EPI_FWD_LSE) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc2(tmem_slot, TMEM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  // Both CTAs' barriers are initialised and TMEM allocated before any
  // cross-CTA arrival or MMA.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The next kernel in the stream may start launching now: its CTAs take an SM
  // only as this grid's CTAs leave (shared memory), or sit beside them and
  // wait for this grid to complete before touching what it writes.
  griddep_launch_dependents();
  // What this grid reads or overwrites that earlier kernels of the stream
  // produced or still read: the epilogue's inputs (the sorted cache, lse) and
  // every output region; for dH and dW also the A operand (dz).  The operands
  // h and W of the projections are the caller's inputs, final before the
  // call's first kernel (launched in plain stream order) started, so their
  // loads need not wait: the mainloop of the first tiles overlaps the tail of
  // the kernel before.
  constexpr bool kOperandsWait = (EPI == EPI_STORE_PARTIAL || EPI == EPI_ACCUM_W);

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      if (kOperandsWait) griddep_wait();
      int stage = 0;
      uint32_t phase = 0, armed = 0, last_par = 0;
      bool ok = true;
      UnitWalk w;
      walk_start(w, g, m_tiles2, cid, ncl);
      for (; ok && w.u < units; walk_next(w)) {
        walk_check(w, g, m_tiles2);
        const int kb0 = w.kb0, kb1 = w.kb1;
        const int arow = w.mb2 * BM2 + static_cast<int>(rank) * 128;   // this CTA's A rows
        const int brow = w.nb * BN + static_cast<int>(rank) * 128;     // this CTA's B rows
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, g.wait_limit_ns, g.status)) {
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(&full[stage], 2 * STAGE2_BYTES);
            armed |= 1u << stage;
            last_par = (last_par & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          unsigned char* a = sA + stage * HALF_BYTES;
          unsigned char* b = sB + stage * HALF_BYTES;
          if (A_MN) {
#pragma unroll
            for (int j = 0; j < 128 / INNER; ++j)
              tma_load_2d_pair(a + j * BOX_BYTES, &tmA, fbar, arow + j * INNER, kb * BK);
          } else {
            tma_load_2d_pair(a, &tmA, fbar, kb * BK, arow);
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < 128 / INNER; ++j)
              tma_load_2d_pair(b + j * BOX_BYTES, &tmB, fbar, brow + j * INNER, kb * BK);
          } else {
            tma_load_2d_pair(b, &tmB, fbar, kb * BK, brow);
          }
          if (++stage == STAGES2) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (leader) {
        for (int s = 0; s < STAGES2; ++s)
          if (armed & (1u << s)) mbar_drain(&full[s], (last_par >> s) & 1u, g.wait_limit_ns);
      } else if (!ok) {
        // The peer cannot observe its copies (they complete on the leader's
        // barrier): give any still in flight a bounded moment to land.
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      UnitWalk w;
      walk_start(w, g, m_tiles2, cid, ncl);
      for (; ok && w.u < units; walk_next(w)) {
        const int kb0 = w.kb0, kb1 = w.kb1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, g.wait_limit_ns, g.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, g.wait_limit_ns, g.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * HALF_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * HALF_BYTES);
#pragma unroll
          for (int k = 0; k < KSTEPS; ++k) {
            const uint64_t ad =
                A_MN ? umma_desc(a0 + k * C::UMMA_K * ROW_BYTES, BOX_BYTES, C::MN_SBO, C::MN_LAYOUT)
                     : umma_desc(a0 + k * 32, 16, 1024, UMMA_LAYOUT_SW128);
            const uint64_t bd =
                B_MN ? umma_desc(b0 + k * C::UMMA_K * ROW_BYTES, BOX_BYTES, C::MN_SBO, C::MN_LAYOUT)
                     : umma_desc(b0 + k * 32, 16, 1024, UMMA_LAYOUT_SW128);
            const uint32_t accum = (kb != kb0 || k != 0) ? 1u : 0u;
            if constexpr (C::FMT == 1) mma2_f16(d_tmem, ad, bd, IDESC, accum);
            else mma2_tf32(d_tmem, ad, bd, IDESC, accum);
          }
          mma2_commit_pair(&empty[stage]);     // frees the stage in both CTAs
          if (++stage == STAGES2) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma2_commit_pair(&tfull[acc]);          // accumulator ready in both CTAs
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      mma2_commit_local(drain);
      mbar_drain(drain, 0, g.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    griddep_wait();
    const int quad = warp & 3;
    unsigned char* boxes = sEpi + (warp - 2) * 2 * EPI_BUF_BYTES;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    // dW: every cluster finishes its tiles at about the same moment, and each
    // CTA then adds 128 KB of fp32 into dW.  Sent as one burst, the add-
    // reductions of all clusters crowd out the operand loads of the next
    // tiles, and the MMAs wait for data (measured: the issue span of a dW tile
    // was 0.93 of its ideal tensor time, 0.99 with the boxes spread).  So the
    // epilogue spaces its boxes by 1/16 of the time between two of its tiles
    // (the tiles before), which spreads them over about half of the next
    // tile's mainloop at any clock.
    uint64_t prev_ready = 0;
    uint32_t pace_ns = 0;
    UnitWalk w;
    walk_start(w, g, m_tiles2, cid, ncl);
    for (; w.u < units; walk_next(w)) {
      walk_check(w, g, m_tiles2);
      if (!mbar_wait(&tfull[acc], acc_phase, g.wait_limit_ns, g.status)) break;
      tc_fence_after();
      if (EPI == EPI_ACCUM_W) {
        if (lane == 0) {
          const uint64_t now = globaltimer_ns();
          if (prev_ready != 0) {
            const uint64_t p = (now - prev_ready) / (2 * (BN / 32));
            pace_ns = static_cast<uint32_t>(p < 4000 ? p : 4000);
          }
          prev_ready = now;
        }
        pace_ns = __shfl_sync(0xffffffffu, pace_ns, 0);
      }
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      run_epilogue<Elem, EPI>(g, &tmC, w.mb2 * BM2 + static_cast<int>(rank) * 128, w.nb, taddr,
                              quad, lane, boxes, w.split * g.split_rows, pace_ns);
      __syncwarp();
      tc_fence_before();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  // The leader's MMAs (which write both CTAs' TMEM) are drained and both
  // epilogues are done before either CTA frees its TMEM.
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, TMEM_COLS);
  }
}

}  // namespace kd
