// kd_topk.cu -- top-K cache build (the offline teacher cache of the
// developersdigest.tech page "Distilling an LLM on One GPU", section "The two
// changes": the teacher's top-100 tokens per position are computed once).
//
// Per row of bf16 teacher logits, select the K entries ranked by
// (value descending, index ascending), +0 == -0, NaN below -inf.
//
// Design (HBM-bound streaming select).  Four 256-thread blocks per SM; each
// takes one row at a time from a counter in the workspace:
//   1. sample: the key L of the sample element ranked about 3K*S/V from the
//      top of the row's first S = min(V, 4096) elements (about 3K expected
//      survivors in the row), found in two levels of 256 bins (the key's high
//      byte, then its low byte).  On long aligned rows each thread contributes
//      the largest of its 16 sample elements instead (a packed bf16 maximum),
//      which can only lower L.  L is turned into a bf16 threshold tf with
//      key(x) >= L  <=>  x >= tf  for every non-NaN x.
//   2. stream: one coalesced pass over the row with eight 16-byte loads in
//      flight per thread; each vector is screened by its packed maximum, the
//      warp stages the vectors that may hold a survivor and tests them element
//      by element, and the survivors are appended to a shared-memory buffer.
//      One thread keeps the stream two steps ahead in L2, into the next row.
//   3. if K <= survivors <= capacity, the top K of the row are exactly the top
//      K of the survivors, ordered by the composite (key desc, index asc):
//      usually through one 256-bin histogram of key - L, otherwise by a wider
//      histogram and counting.
//   4. otherwise (ties, NaN-heavy or adversarially ordered rows) an exact
//      3-pass histogram select runs instead (passes 2-3 hit L2).
#include "kd_common.cuh"
#include "kd_internal.h"

namespace kd {

constexpr int TK_THREADS = 256;
constexpr int TK_BINS = 4096;       // bins of (order key >> 4)
constexpr int TK_SAMPLE = 4096;
constexpr int TK_CAND_CAP = 2048;
constexpr int TK_SEL_CAP = 1024;    // >= K
static_assert(TK_SEL_CAP >= KD_MAX_K, "the selection buffer holds every K the ABI accepts");
constexpr int TK_UNROLL = 8;        // 16-byte loads in flight per thread
constexpr int SAMPLE_PER_THREAD = TK_SAMPLE / TK_THREADS;   // 16

// Order-preserving 16-bit key of a bf16 bit pattern: NaN -> 0 (lowest),
// -0 -> key of +0, otherwise a monotone map of the value.
__device__ __forceinline__ uint32_t bf16_order_key(uint32_t b) {
  b &= 0xFFFFu;
  const uint32_t mag = b & 0x7FFFu;
  if (mag > 0x7F80u) return 0u;
  if (mag == 0u) return 0x8000u;
  return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
}

// 64-bit candidate: (0xFFFF - key) in bits 48..63, the index (< 2^31) in bits
// 16..46, the raw bf16 bits in bits 0..15.  Ascending order of composites is
// key descending, then index ascending (indices are distinct within a row, so
// the raw bits never decide); the raw bits give the exact output value without
// reading the row again.
__device__ __forceinline__ uint64_t composite(uint32_t key, uint32_t idx, uint32_t raw) {
  return (static_cast<uint64_t>(0xFFFFu - key) << 48) | (static_cast<uint64_t>(idx) << 16) |
         (raw & 0xFFFFu);
}
__device__ __forceinline__ uint32_t comp_key(uint64_t c) {
  return 0xFFFFu - static_cast<uint32_t>(c >> 48);
}
__device__ __forceinline__ uint32_t comp_idx(uint64_t c) {
  return static_cast<uint32_t>(c >> 16) & 0x7FFFFFFFu;
}
__device__ __forceinline__ uint32_t comp_raw(uint64_t c) { return static_cast<uint32_t>(c) & 0xFFFFu; }

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) {
  return __uint_as_float((b & 0xFFFFu) << 16);
}

constexpr int TK_WARPS = TK_THREADS / 32;

struct TopkSmem {
  uint4 stage_q[TK_WARPS][32];        // per warp: screened vectors awaiting the exact test
  uint32_t stage_base[TK_WARPS][32];  // and the row index of their first element
  uint32_t hist[TK_BINS];
  uint64_t cand[TK_CAND_CAP];
  uint64_t sel[TK_SEL_CAP];
  uint32_t warp_tot[TK_THREADS / 32 + 1];
  uint32_t hist16[16];
  uint32_t n_cand;
  uint32_t n_sel;
  unsigned long long row_slot[2];   // this CTA's current and next row
  uint32_t thr_bin;
  uint32_t thr_above;
  uint32_t eq_base;
  uint32_t wide;
};

// Exclusive block scan of one value per thread (TK_THREADS threads); also
// returns the block total.  warp_tot needs TK_THREADS/32 + 1 entries.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_tot,
                                                    uint32_t& total) {
  constexpr int NW = TK_THREADS / 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    const uint32_t t = lane < NW ? warp_tot[lane] : 0u;
    uint32_t s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NW) warp_tot[lane] = s - t;
    if (lane == NW - 1) warp_tot[NW] = s;
  }
  __syncthreads();
  const uint32_t r = warp_tot[w] + x - v;
  total = warp_tot[NW];
  __syncthreads();
  return r;
}

// Warp 0 only: among 256 bin counts h[0..256), bin 0 holding the highest keys,
// the bin b where the running count from bin 0 first reaches `target`
// (1 <= target <= total).  Writes b, the count of bins before b and the count
// of bins up to and including b.  h must be 16-byte aligned.
__device__ __forceinline__ void find_bin_256(const uint32_t* h, uint32_t target, uint32_t* out_bin,
                                             uint32_t* out_above, uint32_t* out_through) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  if (KD_DEBUG) {                       // "not found" unless a lane writes a bin below
    if (lane == 0) *out_bin = 0xFFFFFFFFu;
    __syncwarp();
  }
  const uint4 a = reinterpret_cast<const uint4*>(h)[2 * lane];
  const uint4 b = reinterpret_cast<const uint4*>(h)[2 * lane + 1];
  const uint32_t c[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t sum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) sum += c[j];
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  uint32_t run = incl - sum;
  if (run < target && incl >= target) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (run + c[j] >= target) {
        *out_bin = static_cast<uint32_t>(lane * 8 + j);
        *out_above = run;
        *out_through = run + c[j];
        break;
      }
      run += c[j];
    }
  }
}

// Highest bin b with (count of bins > b) < target <= (count of bins >= b).
// If the histogram holds fewer than `target` elements, returns bin 0.
// Writes sm.thr_bin / sm.thr_above.
__device__ void find_threshold_bin(TopkSmem& sm, uint32_t target) {
  constexpr int PER = TK_BINS / TK_THREADS;  // 8
  const int t = threadIdx.x;
  const int hi = TK_BINS - PER * t;          // thread 0 owns the top bins
  uint32_t local = 0;
#pragma unroll
  for (int j = 1; j <= PER; ++j) local += sm.hist[hi - j];
  uint32_t total;
  uint32_t above = block_excl_scan(local, sm.warp_tot, total);
  if (t == 0 && total < target) {
    sm.thr_bin = 0;
    sm.thr_above = 0;
  }
  if (above < target && above + local >= target) {
#pragma unroll 1
    for (int j = 1; j <= PER; ++j) {
      const uint32_t c = sm.hist[hi - j];
      if (above + c >= target) {
        sm.thr_bin = hi - j;
        sm.thr_above = above;
        break;
      }
      above += c;
    }
  }
  __syncthreads();
}

// In-place ascending bitonic sort of n (power of two, <= cap) entries.
__device__ void bitonic_sort(uint64_t* a, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n; i += TK_THREADS) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t x = a[i], y = a[ixj];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            a[i] = y;
            a[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

__device__ __forceinline__ int next_pow2(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}

// Visit every element of a row with 16-byte vector loads where possible.
template <class F>
__device__ __forceinline__ void for_each_elem(const uint16_t* __restrict__ row, int64_t V, F&& f) {
  const uintptr_t addr = reinterpret_cast<uintptr_t>(row);
  int64_t head = ((16 - (addr & 15)) & 15) >> 1;
  if (head > V) head = V;
  for (int64_t i = threadIdx.x; i < head; i += TK_THREADS) f(row[i], static_cast<uint32_t>(i));
  const int64_t nvec = (V - head) >> 3;
  const uint4* vp = reinterpret_cast<const uint4*>(row + head);
  // TK_UNROLL independent 16-byte loads in flight per thread before any use.
  for (int64_t j0 = threadIdx.x; j0 < nvec; j0 += TK_THREADS * TK_UNROLL) {
    uint4 q[TK_UNROLL];
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) {
      const int64_t j = j0 + static_cast<int64_t>(u) * TK_THREADS;
      q[u] = j < nvec ? __ldcs(vp + j) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) {
      const int64_t j = j0 + static_cast<int64_t>(u) * TK_THREADS;
      if (j < nvec) {
        const uint32_t base = static_cast<uint32_t>(head + (j << 3));
        const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          f(w[e] & 0xFFFFu, base + 2 * e);
          f(w[e] >> 16, base + 2 * e + 1);
        }
      }
    }
  }
  for (int64_t i = head + (nvec << 3) + threadIdx.x; i < V; i += TK_THREADS)
    f(row[i], static_cast<uint32_t>(i));
}

// Appends one element to the survivor buffer if it passes the threshold (the
// exact per-element test, for the row's unaligned head and ragged tail).
__device__ __forceinline__ void offer(TopkSmem& sm, uint32_t bits, uint32_t i, float tf) {
  if (bf16_bits_to_float(bits) >= tf) {
    const uint32_t pos = atomicAdd(&sm.n_cand, 1u);
    if (pos < TK_CAND_CAP) sm.cand[pos] = composite(bf16_order_key(bits), i, bits);
  }
}

// Exact test of the 8 elements of a screened vector: a pass mask built without
// branches, then one append per passing element (usually one).
__device__ __forceinline__ void offer8(TopkSmem& sm, uint4 q, uint32_t base, float tf) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  uint32_t m = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    m |= (__uint_as_float(w[e] << 16) >= tf ? 1u : 0u) << (2 * e);
    m |= (__uint_as_float(w[e] & 0xFFFF0000u) >= tf ? 1u : 0u) << (2 * e + 1);
  }
  while (m) {
    const int b = __ffs(m) - 1;
    m &= m - 1;
    const uint32_t bits = (w[b >> 1] >> ((b & 1) * 16)) & 0xFFFFu;
    const uint32_t pos = atomicAdd(&sm.n_cand, 1u);
    if (pos < TK_CAND_CAP) sm.cand[pos] = composite(bf16_order_key(bits), base + b, bits);
  }
}

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t x) {
  return *reinterpret_cast<__nv_bfloat162*>(&x);
}

// Packed maximum of the 8 bf16 values in q: NaN inputs are ignored by
// max.bf16x2 (the other operand is returned), so a NaN survives only where
// both operands are NaN.
__device__ __forceinline__ __nv_bfloat162 max8_packed(uint4 q) {
  return __hmax2(__hmax2(as_bf162(q.x), as_bf162(q.y)), __hmax2(as_bf162(q.z), as_bf162(q.w)));
}

// False only if both halves of m are below tb (one paired compare); a NaN
// half passes the screen and is rejected by the exact per-element test.
__device__ __forceinline__ uint32_t screen_bit(__nv_bfloat162 m, uint32_t tb2) {
  uint32_t r;
  asm("{\n\t.reg .pred p, q;\n\t"
      "setp.lt.bf16x2 p|q, %1, %2;\n\t"
      "and.pred p, p, q;\n\t"
      "selp.u32 %0, 0, 1, p;\n\t}"
      : "=r"(r)
      : "r"(*reinterpret_cast<uint32_t*>(&m)), "r"(tb2));
  return r;
}

// L2 prefetch of `bytes` (a multiple of 16) from a 16-byte-aligned global
// address, issued by one thread as a single bulk operation.
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Stage this lane's screened vectors (bit u of m: vector q[u] may hold a
// survivor; its first element is at row index base + u*TK_THREADS*8) into the
// warp's 32-entry buffer at positions from a warp prefix sum; when the buffer
// would overflow, the warp first runs the exact test on what it holds.  A
// batch of more than 32 vectors (only rows with very many survivors close
// together) is staged vector slot by vector slot instead, at most 32 at a
// time.  Warp-uniform.
__device__ __forceinline__ void flush_stage(TopkSmem& sm, const uint4* sq, const uint32_t* sb,
                                            uint32_t& cnt, float tf, int lane) {
  __syncwarp();
  if (static_cast<uint32_t>(lane) < cnt) offer8(sm, sq[lane], sb[lane], tf);
  __syncwarp();
  cnt = 0;
}

__device__ __forceinline__ void stage_vectors(TopkSmem& sm, uint4* sq, uint32_t* sb, uint32_t& cnt,
                                              uint32_t m, const uint4 (&q)[TK_UNROLL],
                                              uint32_t base, float tf, int lane, uint32_t* status) {
  const uint32_t c = __popc(m);
  uint32_t x = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const uint32_t total = __shfl_sync(0xffffffffu, x, 31);
  if (total > 32u) {
    const uint32_t lanes_below = (1u << lane) - 1u;
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) {
      const bool pass = (m >> u) & 1u;
      const uint32_t b = __ballot_sync(0xffffffffu, pass);
      if (b) {
        const uint32_t nb = __popc(b);
        if (cnt + nb > 32u) flush_stage(sm, sq, sb, cnt, tf, lane);
        if (pass) {
          const uint32_t pos = cnt + __popc(b & lanes_below);
          sq[pos] = q[u];
          sb[pos] = base + u * TK_THREADS * 8;
        }
        cnt += nb;
      }
    }
    return;
  }
  if (cnt + total > 32u) flush_stage(sm, sq, sb, cnt, tf, lane);
  uint32_t pos = cnt + x - c;
#pragma unroll
  for (int u = 0; u < TK_UNROLL; ++u) {
    if ((m >> u) & 1u) {
      KD_CHECK(pos < 32u, status);
      sq[pos] = q[u];
      sb[pos] = base + u * TK_THREADS * 8;
      ++pos;
    }
  }
  cnt += total;
}

// The streaming pass: every element of the row meets the threshold once.
// Each thread holds TK_UNROLL 16-byte vectors (64 elements) in flight, and each
// vector is screened by its packed maximum: three max.bf16x2 and one paired
// bf16x2 compare against tf (NaN operands are ignored by max.bf16x2, and tf
// is a bf16 value, never -inf or NaN, so the screen passes every vector that
// holds a survivor).  The screens of a thread's vectors form a bit mask; a
// vector that may hold a survivor is not tested on the spot, which would make
// the whole warp run the exact test for one lane: it goes to the warp's
// staging buffer, and once the buffer is full, and at the end, the warp runs
// the exact test on up to 32 staged vectors at once, one per lane.
// One thread keeps the CTA's stream two steps (64 KB) ahead in L2 with single
// bulk prefetches; near the end of the row they run on into the first steps of
// the CTA's next row (`next_vp`, or null; given only when every row starts on
// 16 bytes, so the next row has the same full steps), so that HBM keeps working
// for this CTA while it selects and samples.  Every prefetch lies inside a full
// step of this row or of the next.  Indices are 32-bit (V < 2^31).
__device__ __forceinline__ void stream_survivors(TopkSmem& sm, const uint16_t* __restrict__ row,
                                                 uint32_t V, float tf, const uint4* next_vp,
                                                 uint32_t* status) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uintptr_t addr = reinterpret_cast<uintptr_t>(row);
  uint32_t head = static_cast<uint32_t>(((16 - (addr & 15)) & 15) >> 1);
  if (head > V) head = V;
  for (uint32_t i = tid; i < head; i += TK_THREADS) offer(sm, row[i], i, tf);
  const uint32_t nvec = (V - head) >> 3;
  const uint4* vp = reinterpret_cast<const uint4*>(row + head);
  const __nv_bfloat16 tb = __float2bfloat16_rn(tf);
  const uint32_t tb2 = static_cast<uint32_t>(__bfloat16_as_ushort(tb)) * 0x10001u;
  uint4* sq = sm.stage_q[wid];
  uint32_t* sb = sm.stage_base[wid];
  uint32_t cnt = 0;                                  // staged vectors (warp-uniform)
  constexpr uint32_t STEP = TK_THREADS * TK_UNROLL;  // vectors per CTA step
  const uint32_t nfull = nvec / STEP;
  if (tid == 0 && nfull > 1) bulk_prefetch_l2(vp + STEP, STEP * 16);
  for (uint32_t it = 0; it < nfull; ++it) {
    const uint4* p = vp + it * STEP + tid;
    uint4 q[TK_UNROLL];
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) q[u] = __ldcs(p + u * TK_THREADS);
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) m |= screen_bit(max8_packed(q[u]), tb2) << u;
    if (__any_sync(0xffffffffu, m != 0u))
      stage_vectors(sm, sq, sb, cnt, m, q, head + (it * STEP + tid) * 8, tf, lane, status);
    if (tid == 0) {          // the step after next, in this row or the next one
      const uint32_t s2 = it + 2;
      if (s2 < nfull)
        bulk_prefetch_l2(p + 2 * STEP, STEP * 16);   // thread 0's p is vp + it*STEP
      else if (next_vp && s2 - nfull < nfull)     // the next row has the same nfull
        bulk_prefetch_l2(next_vp + (s2 - nfull) * STEP, STEP * 16);
    }
  }
  if (nfull * STEP < nvec) {  // the last, partial step: absent vectors read as -inf
    const uint32_t j0 = nfull * STEP + tid;
    uint4 q[TK_UNROLL];
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) {
      const uint32_t j = j0 + u * TK_THREADS;
      q[u] = j < nvec ? __ldcs(vp + j)
                      : make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
    }
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < TK_UNROLL; ++u) m |= screen_bit(max8_packed(q[u]), tb2) << u;
    if (__any_sync(0xffffffffu, m != 0u))
      stage_vectors(sm, sq, sb, cnt, m, q, head + j0 * 8, tf, lane, status);
  }
  flush_stage(sm, sq, sb, cnt, tf, lane);
  for (uint32_t i = head + (nvec << 3) + tid; i < V; i += TK_THREADS) offer(sm, row[i], i, tf);
}

__global__ void __launch_bounds__(TK_THREADS, 4)
topk_bf16_kernel(const uint16_t* __restrict__ logits, int64_t T, int64_t V, int K,
                 uint32_t sample_target, int fast_sample, float* __restrict__ out_vals,
                 int32_t* __restrict__ out_idx, uint32_t* __restrict__ status,
                 unsigned long long* __restrict__ row_counter) {
  extern __shared__ __align__(16) unsigned char tk_smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(tk_smem_raw);
  const int tid = threadIdx.x;
  const bool rows_aligned = (V & 7) == 0;            // every row starts on 16 bytes

  // Rows are handed out one at a time from a counter (zero at launch): a CTA
  // that finishes a row takes the next free one.  With a fixed share of rows
  // per CTA the build ended when its slowest CTAs did: in one cold launch at
  // 32768 x 131072 every CTA started at once with 55 or 56 rows, and they
  // finished between 1.01 and 1.56 ms (the SMs do not all stream at the same
  // rate).  A CTA takes its next row as it starts a row, so the stream's L2
  // prefetch can run on into it.
  if (tid == 0) sm.row_slot[0] = atomicAdd(row_counter, 1ull);
  __syncthreads();
  int slot = 0;
  int64_t t_next = 0;
  for (int64_t t = static_cast<int64_t>(sm.row_slot[0]); t < T; t = t_next, slot ^= 1) {
    const uint16_t* row = logits + t * V;

    // ---- 1. sample threshold -------------------------------------------------
    // L = the key of the target-th largest sample key, found in two levels of
    // 256 bins: the key's high byte, then its low byte inside the chosen
    // high-byte bin (bin 0 holds the highest keys).  The sample is the row's
    // first TK_SAMPLE elements (all of it when V <= TK_SAMPLE, with target K).
    // On the fast path (long aligned rows, small targets) each thread
    // contributes one key, the largest of its 16 sample elements (a packed
    // bf16 maximum, NaN ignored), and the target-th largest of those 256 keys
    // is L: at most the target-th largest sample element, so the expected
    // number of survivors is about the same (about 3K) and never smaller.  Any
    // L gives the exact result: survivors are every element with key >= L,
    // and rows with fewer than K of them take the fallback.
    sm.hist[tid] = 0u;
    sm.hist[TK_THREADS + tid] = 0u;
    if (tid == 0) {
      sm.n_cand = 0;
      sm.n_sel = 0;
      sm.row_slot[slot ^ 1] = atomicAdd(row_counter, 1ull);   // read after the barrier
    }
    __syncthreads();
    t_next = static_cast<int64_t>(sm.row_slot[slot ^ 1]);
    const uint32_t target = sample_target;
    uint32_t L;
    if (fast_sample) {
      const uint4* vp = reinterpret_cast<const uint4*>(row);
      const uint4 q0 = vp[tid], q1 = vp[tid + TK_THREADS];
      __nv_bfloat162 mm = __hmax2(max8_packed(q0), max8_packed(q1));
      const uint32_t w = *reinterpret_cast<uint32_t*>(&mm);
      const uint32_t k0 = bf16_order_key(w & 0xFFFFu), k1 = bf16_order_key(w >> 16);
      const uint32_t key = k0 > k1 ? k0 : k1;
      atomicAdd(&sm.hist[255u - (key >> 8)], 1u);
      __syncthreads();
      find_bin_256(sm.hist, target, &sm.thr_bin, &sm.thr_above, &sm.n_sel);
      __syncthreads();
      KD_CHECK(sm.thr_bin < 256u, status);
      const uint32_t hb = 255u - sm.thr_bin;          // high byte of L
      const uint32_t above_hb = sm.thr_above;
      if ((key >> 8) == hb) atomicAdd(&sm.hist[TK_THREADS + 255u - (key & 255u)], 1u);
      __syncthreads();
      find_bin_256(sm.hist + TK_THREADS, target - above_hb, &sm.thr_bin, &sm.thr_above,
                   &sm.n_sel);
      __syncthreads();
      KD_CHECK(sm.thr_bin < 256u, status);
      L = (hb << 8) | (255u - sm.thr_bin);
    } else {
      const int64_t S = V < TK_SAMPLE ? V : TK_SAMPLE;
      // The sample's keys stay in registers: SAMPLE_PER_THREAD per thread.
      uint32_t skey[SAMPLE_PER_THREAD];
      {
        uint32_t raw[SAMPLE_PER_THREAD];
#pragma unroll
        for (int u = 0; u < SAMPLE_PER_THREAD; ++u) {
          const int64_t i = tid + static_cast<int64_t>(u) * TK_THREADS;
          raw[u] = i < S ? row[i] : 0u;
        }
#pragma unroll
        for (int u = 0; u < SAMPLE_PER_THREAD; ++u) {
          const int64_t i = tid + static_cast<int64_t>(u) * TK_THREADS;
          skey[u] = i < S ? bf16_order_key(raw[u]) : 0xFFFFFFFFu;   // marker: not sampled
        }
      }
#pragma unroll
      for (int u = 0; u < SAMPLE_PER_THREAD; ++u)
        if (skey[u] != 0xFFFFFFFFu) atomicAdd(&sm.hist[255u - (skey[u] >> 8)], 1u);
      __syncthreads();
      // (target <= S: either S == V >= K and target == K, or V > 4096 >= 3K)
      find_bin_256(sm.hist, target, &sm.thr_bin, &sm.thr_above, &sm.n_sel);
      __syncthreads();
      KD_CHECK(sm.thr_bin < 256u, status);
      const uint32_t hb = 255u - sm.thr_bin;          // high byte of L
      const uint32_t above_hb = sm.thr_above;
#pragma unroll
      for (int u = 0; u < SAMPLE_PER_THREAD; ++u)
        if (skey[u] != 0xFFFFFFFFu && (skey[u] >> 8) == hb)
          atomicAdd(&sm.hist[TK_THREADS + 255u - (skey[u] & 255u)], 1u);
      __syncthreads();
      find_bin_256(sm.hist + TK_THREADS, target - above_hb, &sm.thr_bin, &sm.thr_above,
                   &sm.n_sel);
      __syncthreads();
      KD_CHECK(sm.thr_bin < 256u, status);
      L = (hb << 8) | (255u - sm.thr_bin);            // candidate iff order key >= L
    }
    if (tid == 0) sm.n_sel = 0u;
    // Float threshold equivalent on non-NaN values: key >= L <=> x >= tf.
    // A threshold at or below -inf (the sample's top is NaN or -inf) would
    // keep almost the whole row: such rows go straight to the exact fallback.
    const bool screen = L > 0x7Fu;
    float tf = 0.f;
    if (L == 0x7FFFu) {
      tf = 0.f;                                     // between -0's raw key and +0
    } else if (L < 0x8000u) {
      tf = bf16_bits_to_float((~L) & 0xFFFFu);      // the negative value with key L
    } else {
      tf = bf16_bits_to_float(L & 0x7FFFu);         // +0 when L == 0x8000
    }

    // ---- 2. stream the row, keep survivors ------------------------------------
    if (screen) {
      const uint4* next_vp = (rows_aligned && t_next < T)
                                 ? reinterpret_cast<const uint4*>(logits + t_next * V)
                                 : nullptr;
      stream_survivors(sm, row, static_cast<uint32_t>(V), tf, next_vp, status);
    }
    __syncthreads();
    const uint32_t n = screen ? sm.n_cand : 0u;

    if (n >= static_cast<uint32_t>(K) && n <= static_cast<uint32_t>(TK_CAND_CAP)) {
      // ---- 3. exact select among survivors -------------------------------------
      // Every survivor's key is >= L.  When they span fewer than 256 keys (the
      // usual case: few bf16 values lie near the top of a row), one histogram
      // of key - L, bin 0 holding the highest key, orders them: its prefix sums
      // are the first output slot of each key, the survivors are scattered into
      // their key's bucket, and each one's output position is its bucket's first
      // slot plus the number of bucket entries with a lower index.  Otherwise a
      // 4096-bin histogram of key >> 4, then the 16 keys of the threshold bin,
      // give the exact K-th key, and the survivors at or above it are ranked by
      // counting.
      static_assert(TK_THREADS == 256, "one narrow-histogram bin per thread");
      uint32_t* nh = sm.hist;                        // [256] counts per key - L
      uint32_t* nstart = sm.hist + 256;              // [256] first output slot per bin
      uint32_t* nfill = sm.hist + 512;               // [256] entries placed per bin
      if (tid == 0) {
        sm.wide = 0u;
        sm.n_sel = 0u;
      }
      nh[tid] = 0u;
      nfill[tid] = 0u;
      __syncthreads();
      for (int i = tid; i < static_cast<int>(n); i += TK_THREADS) {
        const uint32_t dk = comp_key(sm.cand[i]) - L;
        if (dk < 256u)
          atomicAdd(&nh[255u - dk], 1u);
        else
          sm.wide = 1u;
      }
      __syncthreads();
      if (sm.wide == 0u) {
        // warp 0: exclusive prefix of the 256 counts (8 bins per lane) and the
        // bin where the count first reaches K (bins up to it: K plus ties)
        if (tid < 32) {
          const uint4 a4 = reinterpret_cast<const uint4*>(nh)[2 * tid];
          const uint4 b4 = reinterpret_cast<const uint4*>(nh)[2 * tid + 1];
          const uint32_t c[8] = {a4.x, a4.y, a4.z, a4.w, b4.x, b4.y, b4.z, b4.w};
          uint32_t sum = 0;
#pragma unroll
          for (int j = 0; j < 8; ++j) sum += c[j];
          uint32_t incl = sum;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (tid >= o) incl += y;
          }
          uint32_t run = incl - sum;
          if (KD_DEBUG && tid == 0) sm.thr_bin = 0xFFFFFFFFu;
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            nstart[8 * tid + j] = run;
            if (run < static_cast<uint32_t>(K) && run + c[j] >= static_cast<uint32_t>(K)) {
              sm.thr_bin = static_cast<uint32_t>(8 * tid + j);   // last bin kept
              sm.thr_above = run + c[j];                          // entries kept (K + ties)
            }
            run += c[j];
          }
        }
        __syncthreads();
        KD_CHECK(sm.thr_bin < 256u, status);
        const uint32_t last_bin = sm.thr_bin;
        const uint32_t ns = sm.thr_above;
        if (ns <= static_cast<uint32_t>(TK_SEL_CAP)) {
          for (int i = tid; i < static_cast<int>(n); i += TK_THREADS) {
            const uint64_t c = sm.cand[i];
            const uint32_t b = 255u - (comp_key(c) - L);
            if (b <= last_bin) sm.sel[nstart[b] + atomicAdd(&nfill[b], 1u)] = c;
          }
          __syncthreads();
          for (int s2 = tid; s2 < static_cast<int>(ns); s2 += TK_THREADS) {
            const uint64_t c = sm.sel[s2];
            const uint32_t b = 255u - (comp_key(c) - L);
            const uint32_t lo = nstart[b], hi = lo + nh[b];
            uint32_t r = lo;
            for (uint32_t j = lo; j < hi; ++j) r += sm.sel[j] < c ? 1u : 0u;
            if (r < static_cast<uint32_t>(K)) {
              out_idx[t * K + r] = static_cast<int32_t>(comp_idx(c));
              out_vals[t * K + r] = bf16_bits_to_float(comp_raw(c));
            }
          }
          __syncthreads();
          continue;
        }
        // more than TK_SEL_CAP entries tie at the K-th key: rank in place below
        __syncthreads();                              // every thread has read thr_bin
        if (tid == 0) sm.thr_bin = L + 255u - last_bin;   // exact K-th key
        __syncthreads();
      } else {
        for (int b = tid; b < TK_BINS; b += TK_THREADS) sm.hist[b] = 0u;
        if (tid < 16) sm.hist16[tid] = 0u;
        __syncthreads();
        for (int i = tid; i < static_cast<int>(n); i += TK_THREADS)
          atomicAdd(&sm.hist[comp_key(sm.cand[i]) >> 4], 1u);
        __syncthreads();
        find_threshold_bin(sm, static_cast<uint32_t>(K));
        const uint32_t cb = sm.thr_bin;
        for (int i = tid; i < static_cast<int>(n); i += TK_THREADS) {
          const uint32_t key = comp_key(sm.cand[i]);
          if ((key >> 4) == cb) atomicAdd(&sm.hist16[key & 15u], 1u);
        }
        __syncthreads();
        if (tid == 0) {
          uint32_t above = sm.thr_above, nib = 0, at = 0;
          for (int j = 15; j >= 0; --j) {
            if (above + sm.hist16[j] >= static_cast<uint32_t>(K)) {
              nib = static_cast<uint32_t>(j);
              at = sm.hist16[j];
              break;
            }
            above += sm.hist16[j];
          }
          sm.thr_bin = (cb << 4) | nib;     // exact K-th key
          sm.thr_above = above + at;        // survivors with key >= it
        }
        __syncthreads();
      }
      const uint32_t Tk = sm.thr_bin;
      const bool compact = sm.thr_above <= static_cast<uint32_t>(TK_SEL_CAP);
      // keep the survivors with key >= Tk (the top K plus ties at Tk);
      if (compact) {
        for (int i = tid; i < static_cast<int>(n); i += TK_THREADS) {
          const uint64_t c = sm.cand[i];
          if (comp_key(c) >= Tk) {
            const uint32_t p = atomicAdd(&sm.n_sel, 1u);
            KD_CHECK(p < static_cast<uint32_t>(TK_SEL_CAP), status);
            if (p < static_cast<uint32_t>(TK_SEL_CAP)) sm.sel[p] = c;
          }
        }
        __syncthreads();
      }
      // rank: the composites are distinct (they contain the index), so an
      // entry's output position is the number of entries ordered before it;
      // those below K write themselves there, already in order.
      const uint64_t* set = compact ? sm.sel : sm.cand;
      const int ns = compact ? static_cast<int>(sm.n_sel) : static_cast<int>(n);
      KD_CHECK(ns >= K && (!compact || static_cast<uint32_t>(ns) == sm.thr_above), status);
      for (int i = tid; i < ns; i += TK_THREADS) {
        const uint64_t c = set[i];
        int rank = 0;
#pragma unroll 8
        for (int j = 0; j < ns; ++j) rank += set[j] < c ? 1 : 0;
        if (rank < K) {
          out_idx[t * K + rank] = static_cast<int32_t>(comp_idx(c));
          out_vals[t * K + rank] = bf16_bits_to_float(comp_raw(c));
        }
      }
      __syncthreads();
      continue;
    }

    // ---- 4. exact 3-pass fallback --------------------------------------------
    // Pass A: full-row histogram of key >> 4.
    for (int b = tid; b < TK_BINS; b += TK_THREADS) sm.hist[b] = 0u;
    if (tid < 16) sm.hist16[tid] = 0u;
    if (tid == 0) {
      sm.n_sel = 0;
      sm.eq_base = 0;
    }
    __syncthreads();
    for_each_elem(row, V, [&](uint32_t bits, uint32_t) {
      atomicAdd(&sm.hist[bf16_order_key(bits) >> 4], 1u);
    });
    __syncthreads();
    find_threshold_bin(sm, static_cast<uint32_t>(K));
    const uint32_t b1 = sm.thr_bin, above1 = sm.thr_above;
    if (tid == 0) sm.n_sel = 0;
    __syncthreads();
    // Pass B: keep bins above b1; histogram the low nibble inside b1.
    for_each_elem(row, V, [&](uint32_t bits, uint32_t i) {
      const uint32_t key = bf16_order_key(bits);
      const uint32_t b = key >> 4;
      if (b > b1) {
        const uint32_t pos = atomicAdd(&sm.n_sel, 1u);
        KD_CHECK(pos < static_cast<uint32_t>(K), status);
        if (pos < static_cast<uint32_t>(TK_SEL_CAP)) sm.sel[pos] = composite(key, i, bits);
      } else if (b == b1) {
        atomicAdd(&sm.hist16[key & 15u], 1u);
      }
    });
    __syncthreads();
    if (tid == 0) {
      uint32_t above = above1;
      uint32_t nib = 0;
      for (int j = 15; j >= 0; --j) {
        if (above + sm.hist16[j] >= static_cast<uint32_t>(K)) {
          nib = static_cast<uint32_t>(j);
          break;
        }
        above += sm.hist16[j];
      }
      sm.thr_bin = (b1 << 4) | nib;   // exact threshold key
      sm.thr_above = above;           // number of keys strictly above it
    }
    __syncthreads();
    const uint32_t Tk = sm.thr_bin;
    const uint32_t need = static_cast<uint32_t>(K) - sm.thr_above;
    // Pass C: keys in (Tk, bin b1 top] appended; keys == Tk taken in index order.
    for (int64_t base = 0; base < V; base += 8 * TK_THREADS) {
      const int64_t i0 = base + 8 * tid;
      uint32_t eq_mask = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t i = i0 + u;
        if (i < V) {
          const uint32_t bits = row[i];
          const uint32_t key = bf16_order_key(bits);
          if ((key >> 4) == b1 && key > Tk) {
            const uint32_t pos = atomicAdd(&sm.n_sel, 1u);
            KD_CHECK(pos < static_cast<uint32_t>(K), status);
            if (pos < static_cast<uint32_t>(TK_SEL_CAP))
              sm.sel[pos] = composite(key, static_cast<uint32_t>(i), bits);
          } else if (key == Tk) {
            eq_mask |= 1u << u;
          }
        }
      }
      uint32_t tile_total;
      const uint32_t rank = block_excl_scan(__popc(eq_mask), sm.warp_tot, tile_total);
      const uint32_t eb = sm.eq_base;
      uint32_t r = eb + rank;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (eq_mask & (1u << u)) {
          if (r < need) {
            const uint32_t pos = atomicAdd(&sm.n_sel, 1u);
            KD_CHECK(pos < static_cast<uint32_t>(K), status);
            if (pos < static_cast<uint32_t>(TK_SEL_CAP))
              sm.sel[pos] = composite(Tk, static_cast<uint32_t>(i0 + u), row[i0 + u]);
          }
          ++r;
        }
      }
      __syncthreads();
      if (tid == 0) sm.eq_base = eb + tile_total;
      __syncthreads();
    }
    KD_CHECK(sm.n_sel == static_cast<uint32_t>(K), status);   // exactly the top K
    const int np = next_pow2(K);
    for (int i = K + tid; i < np; i += TK_THREADS) sm.sel[i] = ~0ull;
    __syncthreads();
    bitonic_sort(sm.sel, np);
    for (int k = tid; k < K; k += TK_THREADS) {
      const uint64_t c = sm.sel[k];
      out_idx[t * K + k] = static_cast<int32_t>(comp_idx(c));
      out_vals[t * K + k] = bf16_bits_to_float(comp_raw(c));
    }
    __syncthreads();
  }
}

}  // namespace kd

// ----------------------------------------------------------------------------
// Host launcher (called from kd_api.cu after argument validation).
// ----------------------------------------------------------------------------
namespace kd {

cudaError_t launch_topk_bf16(const void* logits, int64_t T, int64_t V, int K, float* out_vals,
                             int32_t* out_idx, uint32_t* status, unsigned long long* row_counter,
                             cudaStream_t stream, int num_sms) {
  const size_t smem = sizeof(TopkSmem);
  cudaError_t e = cudaFuncSetAttribute(topk_bf16_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_bf16_kernel, TK_THREADS, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t grid = static_cast<int64_t>(num_sms) * per_sm;
  if (grid > T) grid = T;
  // Sample rank of the threshold: about 3K expected survivors over the row
  // (all K when the sample is the whole row).  Integer ceil(3*K*S / V).
  uint32_t target;
  if (V <= TK_SAMPLE) {
    target = static_cast<uint32_t>(K);
  } else {
    const int64_t num = 3 * static_cast<int64_t>(K) * TK_SAMPLE;
    target = static_cast<uint32_t>((num + V - 1) / V);
    if (target < 1u) target = 1u;
  }
  // one key per thread (the largest of its 16 sample elements) when rows are
  // long and 16-byte aligned and the target is a small share of the 256 keys
  const int fast = (V > TK_SAMPLE && (V & 7) == 0 && target <= 32u) ? 1 : 0;
  topk_bf16_kernel<<<static_cast<unsigned>(grid), TK_THREADS, smem, stream>>>(
      static_cast<const uint16_t*>(logits), T, V, K, target, fast, out_vals, out_idx, status,
      row_counter);
  count_launch();
  return cudaGetLastError();
}

}  // namespace kd
