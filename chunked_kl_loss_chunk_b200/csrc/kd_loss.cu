// kd_loss.cu -- the fused chunked top-K KL loss: cache preparation, the chunk
// loop of the forward (projection + logsumexp + gather fused into the GEMM
// epilogue, then a per-row combine) and of the backward (projection recomputed
// with dz formed in the epilogue, then dH = dz W and dW += dz^T h).
//
// Method: developersdigest.tech "Distilling an LLM on One GPU", section "The two
// changes" (one chunk of positions at a time: project to logits for that chunk,
// fold into the running loss, discard; the backward recomputes each chunk);
// scitechpulse.com "New distillation trick ..." (the output projection is
// folded into the loss so the student's logits grid is never materialised).
#include <math.h>
#include <string.h>

#include <atomic>

#include "kd_gemm.cuh"
#include "kd_gemm2.cuh"
#include "kd_internal.h"

namespace kd {

// Factor on the loss and on every gradient: tau^2 under KD_KL_TAU_SQUARED
// (the usual temperature compensation of distillation), else 1.
static inline double loss_weight(float tau, uint32_t flags) {
  return (flags & KD_KL_TAU_SQUARED) ? static_cast<double>(tau) * tau : 1.0;
}

// ----------------------------------------------------------------------------
// K2: cache prep.  One warp per position: p = softmax(vals / tau) over the K
// cached logits (or, for a cache of full-vocabulary log-probabilities,
// p = exp(vals) with no renormalisation), S = sum p, sum p log p, then the
// (index, p) pairs sorted by index ascending.  Indices outside [0, V) or
// repeated in a row record KD_ERR_BAD_INDEX; such entries get p = 0 and are
// moved past V.
// ----------------------------------------------------------------------------
constexpr int PREP_WARPS = 4;
constexpr int PREP_MAXK = KD_MAX_K;

__global__ void __launch_bounds__(PREP_WARPS * 32)
prep_kernel(const float* __restrict__ vals, const int32_t* __restrict__ idx, int64_t T, int K,
            int64_t V, float inv_tau, int logprob, int32_t* __restrict__ idx_sorted,
            float* __restrict__ p_sorted, float2* __restrict__ stats, uint32_t* status) {
  extern __shared__ __align__(16) unsigned char prep_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* buf = reinterpret_cast<uint64_t*>(prep_smem) + warp * PREP_MAXK;
  int np = 1;
  while (np < K) np <<= 1;

  for (int64_t t = static_cast<int64_t>(blockIdx.x) * PREP_WARPS + warp; t < T;
       t += static_cast<int64_t>(gridDim.x) * PREP_WARPS) {
    const float* vr = vals + t * K;
    const int32_t* ir = idx + t * K;
    // cached logits: p = softmax over the K entries at temperature tau;
    // cached log-probabilities: p = exp(vals) as given (S <= 1).
    float mx = 0.f, inv_se = 1.f;
    if (!logprob) {
      mx = -INFINITY;
      for (int k = lane; k < K; k += 32) mx = fmaxf(mx, vr[k] * inv_tau);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float se = 0.f;
      for (int k = lane; k < K; k += 32) se += expf(vr[k] * inv_tau - mx);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) se += __shfl_xor_sync(0xffffffffu, se, o);
      inv_se = 1.f / se;
    }
    float S = 0.f, plogp = 0.f;
    bool bad = false;
    for (int k = lane; k < K; k += 32) {
      const float b = logprob ? vr[k] : vr[k] * inv_tau - mx;
      float p = expf(b) * inv_se;
      int32_t i = ir[k];
      if (i < 0 || static_cast<int64_t>(i) >= V) {
        bad = true;
        p = 0.f;
        i = INT32_MAX;
      }
      S += p;
      if (p > 0.f) plogp += p * (logprob ? b : logf(p));
      buf[k] = (static_cast<uint64_t>(static_cast<uint32_t>(i)) << 32) | __float_as_uint(p);
    }
    for (int k = K + lane; k < np; k += 32) buf[k] = ~0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      S += __shfl_xor_sync(0xffffffffu, S, o);
      plogp += __shfl_xor_sync(0xffffffffu, plogp, o);
    }
    __syncwarp();
    // bitonic sort of np entries by index (upper 32 bits), ascending
    for (int kk = 2; kk <= np; kk <<= 1) {
      for (int j = kk >> 1; j > 0; j >>= 1) {
        for (int i = lane; i < np; i += 32) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const uint64_t x = buf[i], y = buf[ixj];
            const bool up = (i & kk) == 0;
            if ((x > y) == up) {
              buf[i] = y;
              buf[ixj] = x;
            }
          }
        }
        __syncwarp();
      }
    }
    for (int k = lane; k < K; k += 32) {
      const uint64_t e = buf[k];
      const uint32_t i = static_cast<uint32_t>(e >> 32);
      if (k > 0 && i != 0x7FFFFFFFu && static_cast<uint32_t>(buf[k - 1] >> 32) == i) bad = true;
      idx_sorted[t * K + k] = static_cast<int32_t>(i);
      p_sorted[t * K + k] = __uint_as_float(static_cast<uint32_t>(e));
    }
    if (lane == 0) stats[t] = make_float2(S, plogp);
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, KD_ERR_BAD_INDEX);
    __syncwarp();
  }
}

// The same preparation for K <= 128, with the (index, p) pairs of a row held
// in registers, four per lane (entry e = lane + 32*r), and sorted by a bitonic
// network over the next power of two >= K whose exchanges are warp shuffles
// (distances < 32) or register swaps (distances 32 and 64).  No shared memory,
// so the kernel runs beside the first GEMM of the chunk loop, which may start
// while it runs (programmatic dependent launch; it waits for this kernel's
// results before reading them).
constexpr int PREP_REG_MAXK = 128;

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t x, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(x), m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(x >> 32), m);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}
__device__ __forceinline__ uint64_t shfl_u64(uint64_t x, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, static_cast<uint32_t>(x), src);
  const uint32_t hi = __shfl_sync(0xffffffffu, static_cast<uint32_t>(x >> 32), src);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}
__device__ __forceinline__ uint64_t shfl_up_u64(uint64_t x, int d) {
  const uint32_t lo = __shfl_up_sync(0xffffffffu, static_cast<uint32_t>(x), d);
  const uint32_t hi = __shfl_up_sync(0xffffffffu, static_cast<uint32_t>(x >> 32), d);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

__global__ void __launch_bounds__(PREP_WARPS * 32)
prep_reg_kernel(const float* __restrict__ vals, const int32_t* __restrict__ idx, int64_t T, int K,
                int64_t V, float inv_tau, int logprob, int32_t* __restrict__ idx_sorted,
                float* __restrict__ p_sorted, float2* __restrict__ stats, uint32_t* status) {
  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int np = 1;
  while (np < K) np <<= 1;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * PREP_WARPS + warp; t < T;
       t += static_cast<int64_t>(gridDim.x) * PREP_WARPS) {
    const float* vr = vals + t * K;
    const int32_t* ir = idx + t * K;
    float v[4];
    int32_t ix[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int k = lane + 32 * r;
      v[r] = k < K ? vr[k] : 0.f;
      ix[r] = k < K ? ir[k] : 0;
    }
    float mx = 0.f, inv_se = 1.f;
    if (!logprob) {
      mx = -INFINITY;
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (lane + 32 * r < K) mx = fmaxf(mx, v[r] * inv_tau);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float se = 0.f;
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (lane + 32 * r < K) se += expf(v[r] * inv_tau - mx);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) se += __shfl_xor_sync(0xffffffffu, se, o);
      inv_se = 1.f / se;
    }
    float S = 0.f, plogp = 0.f;
    bool bad = false;
    uint64_t a[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      if (lane + 32 * r < K) {
        const float b = logprob ? v[r] : v[r] * inv_tau - mx;
        float p = expf(b) * inv_se;
        int32_t i = ix[r];
        if (i < 0 || static_cast<int64_t>(i) >= V) {
          bad = true;
          p = 0.f;
          i = INT32_MAX;
        }
        S += p;
        if (p > 0.f) plogp += p * (logprob ? b : logf(p));
        a[r] = (static_cast<uint64_t>(static_cast<uint32_t>(i)) << 32) | __float_as_uint(p);
      } else {
        a[r] = ~0ull;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      S += __shfl_xor_sync(0xffffffffu, S, o);
      plogp += __shfl_xor_sync(0xffffffffu, plogp, o);
    }
    // bitonic sort of entries [0, np) ascending (the entries above np are padding)
    for (int kk = 2; kk <= np; kk <<= 1) {
      for (int j = kk >> 1; j > 0; j >>= 1) {
        if (j >= 32) {
          // entries e and e + j are this lane's registers r and r + j/32
          auto cas = [&](uint64_t& x, uint64_t& y, int r) {
            const bool asc = ((lane + 32 * r) & kk) == 0;
            const bool swap = (x > y) == asc;
            const uint64_t lo = swap ? y : x, hi = swap ? x : y;
            x = lo;
            y = hi;
          };
          if (j == 32) {
            cas(a[0], a[1], 0);
            cas(a[2], a[3], 2);
          } else {
            cas(a[0], a[2], 0);
            cas(a[1], a[3], 1);
          }
        } else {
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int e = lane + 32 * r;
            const uint64_t other = shfl_xor_u64(a[r], j);
            const bool lower = (e & j) == 0, asc = (e & kk) == 0;
            const bool take_min = lower == asc;
            a[r] = take_min ? (other < a[r] ? other : a[r]) : (other > a[r] ? other : a[r]);
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int k = lane + 32 * r;
      uint64_t prev = shfl_up_u64(a[r], 1);
      const uint64_t last_prev = shfl_u64(a[r > 0 ? r - 1 : 0], 31);
      if (lane == 0) prev = last_prev;
      if (k < K) {
        const uint32_t i = static_cast<uint32_t>(a[r] >> 32);
        if (k > 0 && i != 0x7FFFFFFFu && static_cast<uint32_t>(prev >> 32) == i) bad = true;
        idx_sorted[t * K + k] = static_cast<int32_t>(i);
        p_sorted[t * K + k] = __uint_as_float(static_cast<uint32_t>(a[r]));
      }
    }
    if (lane == 0) stats[t] = make_float2(S, plogp);
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, KD_ERR_BAD_INDEX);
  }
}

// ----------------------------------------------------------------------------
// K4: combine the per-(row, vocab tile) partials of one chunk.  One warp per
// row; lane l merges tiles l, l+32, ... in order, then a fixed shuffle tree.
//   LSE_t = M/tau + ln S,  KL_t = sum p log p - G/tau + (sum p) LSE_t
// ----------------------------------------------------------------------------
__device__ __forceinline__ void merge_lse(float& m, float& s, float m2, float s2, float zs) {
  const float nm = fmaxf(m, m2);
  if (nm == -INFINITY) return;
  s = s * exp2f((m - nm) * zs) + s2 * exp2f((m2 - nm) * zs);
  m = nm;
}

__global__ void __launch_bounds__(256)
combine_kernel(const float4* __restrict__ partials, int rows, int n_tiles, int64_t row0,
               float zscale, float inv_tau, const float2* __restrict__ stats,
               float* __restrict__ lse, float* __restrict__ kl) {
  griddep_launch_dependents();
  griddep_wait();                       // the chunk's GEMM has written the partials
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const float4* pr = partials + static_cast<int64_t>(warp) * n_tiles;
  float m = -INFINITY, s = 0.f, gsum = 0.f;
  for (int j = lane; j < n_tiles; j += 32) {
    const float4 q = pr[j];
    merge_lse(m, s, q.x, q.y, zscale);
    gsum += q.z;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const float g2 = __shfl_xor_sync(0xffffffffu, gsum, o);
    // xor partners combine symmetrically; use a canonical operand order so that
    // both lanes compute bit-identical results.
    if (lane & o) {
      float mm = m2, ss = s2;
      merge_lse(mm, ss, m, s, zscale);
      m = mm;
      s = ss;
      gsum = g2 + gsum;
    } else {
      merge_lse(m, s, m2, s2, zscale);
      gsum = gsum + g2;
    }
  }
  if (lane == 0) {
    const int64_t t = row0 + warp;
    const float L = m * inv_tau + logf(s);
    const float2 st = stats[t];
    lse[t] = L;
    kl[t] = st.y - gsum * inv_tau + st.x * L;
  }
}

// dH rows of a chunk = sum over K-splits of the fp32 partials, in split order.
// One thread per 4 consecutive elements (d % 8 == 0), grid-stride over a grid
// small enough to be resident at once (so that the next kernel can launch
// while this one waits for the dH GEMM).
template <typename Elem>
__global__ void __launch_bounds__(256)
dh_reduce_kernel(const float* __restrict__ part, int k_split, int64_t split_rows, int rows,
                 int64_t d, Elem* __restrict__ dH) {
  griddep_launch_dependents();
  griddep_wait();                       // the dH GEMM has written the partials
  const int64_t per_row = d / 4;
  const int64_t n = static_cast<int64_t>(rows) * per_row;
  for (int64_t q = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < n;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = q / per_row, j = (q - m * per_row) * 4;
    float4 acc = reinterpret_cast<const float4*>(part + m * d + j)[0];
    for (int s = 1; s < k_split; ++s) {
      const float4 x = reinterpret_cast<const float4*>(part + (s * split_rows + m) * d + j)[0];
      acc.x += x.x;
      acc.y += x.y;
      acc.z += x.z;
      acc.w += x.w;
    }
    if constexpr (sizeof(Elem) == 4) {
      reinterpret_cast<float4*>(dH + m * d + j)[0] = acc;
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&lo);
      w.y = *reinterpret_cast<uint32_t*>(&hi);
      reinterpret_cast<uint2*>(dH + m * d + j)[0] = w;
    }
  }
}

// Deterministic sum of kl[0..T) divided by T_norm (T itself, or the positions
// of the whole batch when these T rows are one data-parallel shard of it): one
// block, fixed per-thread strides, fixed tree; fp64 accumulation.
__global__ void __launch_bounds__(1024)
mean_kernel(const float* __restrict__ kl, int64_t T, int64_t T_norm, double scale,
            float* __restrict__ loss) {
  __shared__ double part[1024];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < T; i += 1024) acc += static_cast<double>(kl[i]);
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 512; s > 0; s >>= 1) {
    if (threadIdx.x < s) part[threadIdx.x] += part[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = static_cast<float>(scale * (part[0] / static_cast<double>(T_norm)));
}

// Failure-detection probe: waits on a barrier that nothing arrives at.
__global__ void wait_probe_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, limit_ns, status);
}

// ----------------------------------------------------------------------------
// Host side.
// ----------------------------------------------------------------------------
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// 2-D row-major tensor [outer, inner] with the given row pitch (elements),
// zero fill out of bounds.  Swizzle: 128 bytes of 16-byte chunks, except for
// fp32 tiles read MN-major by the tensor cores (mn_major && f32), which need
// 128 bytes of 32-byte chunks to match the MMA's tf32 MN-major layout.
bool make_map(CUtensorMap* map, const void* base, bool f32, uint64_t inner, uint64_t outer,
              uint64_t pitch_elems, uint32_t box_inner, uint32_t box_outer,
              bool mn_major = false, int swizzle_override = -1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_elems * es};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                  2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_override >= 0 ? static_cast<CUtensorMapSwizzle>(swizzle_override)
                  : (mn_major && f32)   ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                                        : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Output box map for the epilogues: 32 x 32 elements, 128-byte swizzle for
// fp32 boxes (128-byte rows), 64-byte swizzle for bf16 boxes (64-byte rows).
bool make_out_map(CUtensorMap* map, const void* base, bool f32, uint64_t inner, uint64_t outer,
                  uint64_t pitch_elems) {
  return make_map(map, base, f32, inner, outer, pitch_elems, 32, 32, false,
                  f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// Launches a small kernel with programmatic stream serialization (it may start
// while the kernel before it runs, and waits inside for that kernel's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Cache preparation for fwd_impl / bwd_impl.  K <= 128: the register sort, a
// grid small enough to be resident at once, so that the first GEMM (launched
// with programmatic serialization) can start while it runs.  Larger K: the
// shared-memory sort.
cudaError_t launch_prep(const float* t_vals, const int32_t* t_idx, int64_t T, int K, int64_t V,
                        float inv_tau, int logprob, int32_t* idx_s, float* p_s, float2* stats,
                        uint32_t* status, cudaStream_t s, int num_sms) {
  const int64_t blocks64 = (T + PREP_WARPS - 1) / PREP_WARPS;
  if (K <= PREP_REG_MAXK) {
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    const unsigned blocks = static_cast<unsigned>(blocks64 < cap ? blocks64 : cap);
    prep_reg_kernel<<<blocks, PREP_WARPS * 32, 0, s>>>(t_vals, t_idx, T, K, V, inv_tau, logprob,
                                                        idx_s, p_s, stats, status);
  } else {
    const int blocks = static_cast<int>(blocks64 < 65535 * 16 ? blocks64 : 65535 * 16);
    prep_kernel<<<blocks, PREP_WARPS * 32, PREP_WARPS * PREP_MAXK * 8, s>>>(
        t_vals, t_idx, T, K, V, inv_tau, logprob, idx_s, p_s, stats, status);
  }
  count_launch();
  return cudaGetLastError();
}

// Clusters of two CTAs that can be resident at once for this kernel, cached
// per device (atomics: calls may come from several host threads).
constexpr int KD_MAX_DEVICES = 64;
template <typename Kern>
int max_pair_clusters(Kern kern, int num_sms) {
  static std::atomic<int> cache[KD_MAX_DEVICES];
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cacheable = dev >= 0 && dev < KD_MAX_DEVICES;
  if (cacheable) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms / 2));
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = GEMM2_SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = num_sms / 2;
  }
  if (cacheable) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <typename Elem, int A_MN, int B_MN, int EPI>
cudaError_t launch_gemm2(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc,
                         GemmArgs g, cudaStream_t s, int num_sms) {
  static constexpr int kKind[5] = {KD_GEMM_FWD_LSE, KD_GEMM_BWD_DZ, KD_GEMM_DH, KD_GEMM_DW,
                                   KD_GEMM_DH};
  auto kern = gemm2_kernel<Elem, A_MN, B_MN, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       GEMM2_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int units = ((g.M + BM2 - 1) / BM2) * g.n_tiles * g.k_split;
  const int maxc = max_pair_clusters(kern, num_sms);
  const int nclusters = units < maxc ? units : maxc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * nclusters);
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = GEMM2_SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // may start while the kernel before it runs (the kernel waits inside for
  // whatever that kernel writes)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  profile_before(kKind[EPI], 2.0 * g.M * static_cast<double>(g.N) * g.K, s);
  e = cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, g);
  count_launch();
  profile_after(s);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// K-splits (1..KD_DH_MAX_SPLIT, never more than k_blocks) for dH that best
// fill the pair clusters.
int choose_dh_split(int units1, int nclusters, int k_blocks) {
  int best = 1;
  double best_eff = 0.0;
  const int kmax = k_blocks < KD_DH_MAX_SPLIT ? k_blocks : KD_DH_MAX_SPLIT;
  for (int k = 1; k <= kmax; ++k) {
    const int u = units1 * k;
    const int rounds = (u + nclusters - 1) / nclusters;
    const double eff = static_cast<double>(u) / (static_cast<double>(rounds) * nclusters);
    if (eff > best_eff + 0.01) {
      best_eff = eff;
      best = k;
    }
  }
  return best;
}

inline int cdiv(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

}  // namespace

namespace {

// size_t arithmetic that saturates at SIZE_MAX and clears `ok` on overflow.
struct CheckedSize {
  bool ok = true;
  size_t mul(size_t a, size_t b) {
    size_t r;
    if (!ok || __builtin_mul_overflow(a, b, &r)) return fail();
    return r;
  }
  size_t add(size_t a, size_t b) {
    size_t r;
    if (!ok || __builtin_add_overflow(a, b, &r)) return fail();
    return r;
  }
  size_t align(size_t x) {   // round up to KD_WS_ALIGN
    const size_t r = add(x, KD_WS_ALIGN - 1);
    return ok ? (r & ~(KD_WS_ALIGN - 1)) : r;
  }
  size_t fail() {
    ok = false;
    return SIZE_MAX;
  }
};

}  // namespace

WsLayout ws_layout(int64_t T, int64_t d, int64_t V, int K, int64_t chunk, int dtype) {
  WsLayout L;
  CheckedSize c;
  const size_t es = dtype == KD_DTYPE_F32 ? 4 : 2;
  const size_t t = static_cast<size_t>(T), k = static_cast<size_t>(K);
  size_t off = KD_WS_ALIGN;  // status word + reserved
  L.p_sorted = off;
  off = c.align(c.add(off, c.mul(c.mul(t, k), 4)));
  L.idx_sorted = off;
  off = c.align(c.add(off, c.mul(c.mul(t, k), 4)));
  L.stats = off;
  off = c.align(c.add(off, c.mul(t, 8)));
  L.kl = off;
  off = c.align(c.add(off, c.mul(t, 4)));
  const int64_t rows = chunk < T ? chunk : T;
  L.ldz = ((V + 63) / 64) * 64;
  const size_t n_tiles = static_cast<size_t>((V + BN - 1) / BN);
  const size_t part = c.mul(c.mul(static_cast<size_t>(rows), n_tiles), 16);
  const size_t dz = c.mul(c.mul(c.mul(KD_DW_GROUP, static_cast<size_t>(rows)),
                                static_cast<size_t>(L.ldz)), es);
  L.scratch = off;
  L.fwd_end = c.add(off, part);
  off = c.align(c.add(off, part > dz ? part : dz));
  L.rows_pad = ((rows + 255) / 256) * 256;
  L.hpart = off;
  off = c.align(c.add(off, c.mul(c.mul(KD_DH_MAX_SPLIT, static_cast<size_t>(L.rows_pad)),
                                 c.mul(static_cast<size_t>(d), 4))));
  L.total = off;
  L.ok = c.ok;
  if (!L.ok) L.total = L.fwd_end = SIZE_MAX;
  return L;
}

template <typename Elem>
static kd_status fwd_impl(const void* h, const void* W, int64_t T, int64_t T_norm, int64_t d,
                          int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                          int64_t chunk, float tau, uint32_t flags, float* loss, float* lse,
                          float* kl_rows, void* ws, cudaStream_t s, int num_sms,
                          uint64_t limit_ns) {
  constexpr bool F32 = sizeof(Elem) == 4;
  constexpr int BK = ElemCfg<Elem>::BK;
  const WsLayout L = ws_layout(T, d, V, K, chunk, F32 ? KD_DTYPE_F32 : KD_DTYPE_BF16);
  unsigned char* w = static_cast<unsigned char*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(w);
  int32_t* idx_s = reinterpret_cast<int32_t*>(w + L.idx_sorted);
  float* p_s = reinterpret_cast<float*>(w + L.p_sorted);
  float2* stats = reinterpret_cast<float2*>(w + L.stats);
  float* kl = kl_rows ? kl_rows : reinterpret_cast<float*>(w + L.kl);
  float4* part = reinterpret_cast<float4*>(w + L.scratch);

  if (cudaMemsetAsync(status, 0, 4, s) != cudaSuccess) return KD_ERR_CUDA;
  const float inv_tau = 1.f / tau;
  if (launch_prep(t_vals, t_idx, T, K, V, inv_tau, (flags & KD_KL_LOGPROB_CACHE) ? 1 : 0, idx_s,
                  p_s, stats, status, s, num_sms) != cudaSuccess)
    return KD_ERR_CUDA;
  CUtensorMap tW;
  if (!make_map(&tW, W, F32, d, V, d, BK, 128)) return KD_ERR_CUDA;
  const float zscale = 1.4426950408889634f * inv_tau;
  for (int64_t c0 = 0; c0 < T; c0 += chunk) {
    const int64_t rows = (T - c0) < chunk ? (T - c0) : chunk;
    CUtensorMap tH;
    const Elem* hc = static_cast<const Elem*>(h) + c0 * d;
    if (!make_map(&tH, hc, F32, d, rows, d, BK, BM)) return KD_ERR_CUDA;
    GemmArgs g;
    memset(&g, 0, sizeof(g));
    g.M = static_cast<int32_t>(rows);
    g.N = static_cast<int32_t>(V);
    g.K = static_cast<int32_t>(d);
    g.m_tiles = cdiv(rows, BM);
    g.n_tiles = cdiv(V, BN);
    g.k_blocks = cdiv(d, BK);
    g.m_fastest = 1;
    g.k_split = 1;
    g.row0 = c0;
    g.V = V;
    g.Ktop = K;
    g.zscale = zscale;
    g.idx_sorted = idx_s;
    g.p_sorted = p_s;
    g.row_stats = stats;
    g.partials = part;
    g.status = status;
    g.wait_limit_ns = limit_ns;
    if (launch_gemm2<Elem, 0, 0, EPI_FWD_LSE>(tH, tW, tH /*no output box*/, g, s, num_sms) !=
        cudaSuccess)
      return KD_ERR_CUDA;
    const int cblocks = cdiv(rows * 32, 256);
    if (launch_pdl(combine_kernel, static_cast<unsigned>(cblocks), 256u, s,
                   static_cast<const float4*>(part), static_cast<int>(rows), g.n_tiles, c0, zscale,
                   inv_tau, static_cast<const float2*>(stats), lse, kl) != cudaSuccess)
      return KD_ERR_CUDA;
  }
  mean_kernel<<<1, 1024, 0, s>>>(kl, T, T_norm, loss_weight(tau, flags), loss);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return KD_ERR_CUDA;
  return KD_OK;
}

template <typename Elem>
static kd_status bwd_impl(const void* h, const void* W, int64_t T, int64_t T_norm, int64_t d,
                          int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                          int64_t chunk, float tau, uint32_t flags, const float* lse,
                          const float* grad_loss, void* dH, float* dW, int accumulate, void* ws,
                          cudaStream_t s, int num_sms, uint64_t limit_ns) {
  constexpr bool F32 = sizeof(Elem) == 4;
  constexpr int BK = ElemCfg<Elem>::BK;
  constexpr int INNER = ROW_BYTES / sizeof(Elem);
  const WsLayout L = ws_layout(T, d, V, K, chunk, F32 ? KD_DTYPE_F32 : KD_DTYPE_BF16);
  unsigned char* w = static_cast<unsigned char*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(w);
  int32_t* idx_s = reinterpret_cast<int32_t*>(w + L.idx_sorted);
  float* p_s = reinterpret_cast<float*>(w + L.p_sorted);
  float2* stats = reinterpret_cast<float2*>(w + L.stats);
  Elem* dz = reinterpret_cast<Elem*>(w + L.scratch);

  if (cudaMemsetAsync(status, 0, 4, s) != cudaSuccess) return KD_ERR_CUDA;
  const float inv_tau = 1.f / tau;
  if (launch_prep(t_vals, t_idx, T, K, V, inv_tau, (flags & KD_KL_LOGPROB_CACHE) ? 1 : 0, idx_s,
                  p_s, stats, status, s, num_sms) != cudaSuccess)
    return KD_ERR_CUDA;
  CUtensorMap tW_k, tW_mn;
  if (!make_map(&tW_k, W, F32, d, V, d, BK, 128)) return KD_ERR_CUDA;     // [V, d], K = d
  if (!make_map(&tW_mn, W, F32, d, V, d, INNER, BK, true)) return KD_ERR_CUDA;  // K = V, N = d
  CUtensorMap tDW_out, tHP_out;
  if (!make_out_map(&tDW_out, dW, true, d, V, d)) return KD_ERR_CUDA;
  float* hpart = reinterpret_cast<float*>(w + L.hpart);
  if (!make_out_map(&tHP_out, hpart, true, d, KD_DH_MAX_SPLIT * L.rows_pad, d)) return KD_ERR_CUDA;
  const float zscale = 1.4426950408889634f * inv_tau;
  const float inv_T_tau =
      static_cast<float>(loss_weight(tau, flags) / (static_cast<double>(T_norm) * tau));
  // dz of KD_DW_GROUP consecutive chunks is kept side by side, so that dW is
  // updated once per group with K = the group's rows (halving dW's
  // read-modify-write traffic); dz and dH are formed chunk by chunk.
  const int64_t group_rows = chunk * KD_DW_GROUP;
  for (int64_t g0 = 0; g0 < T; g0 += group_rows) {
    const int64_t grows = (T - g0) < group_rows ? (T - g0) : group_rows;
    for (int64_t off = 0; off < grows; off += chunk) {
      const int64_t c0 = g0 + off;
      const int64_t rows = (grows - off) < chunk ? (grows - off) : chunk;
      const Elem* hc = static_cast<const Elem*>(h) + c0 * d;
      Elem* dzc = dz + off * L.ldz;                 // this chunk's rows of the group's dz
      CUtensorMap tH_k, tDz_k, tDz_out;
      if (!make_out_map(&tDz_out, dzc, F32, V, rows, L.ldz)) return KD_ERR_CUDA;
      if (!make_map(&tH_k, hc, F32, d, rows, d, BK, BM)) return KD_ERR_CUDA;
      if (!make_map(&tDz_k, dzc, F32, V, rows, L.ldz, BK, BM)) return KD_ERR_CUDA;

      // (1) recompute z = h_c W^T; epilogue writes dz_c [rows, ldz]
      GemmArgs g;
      memset(&g, 0, sizeof(g));
      g.M = static_cast<int32_t>(rows);
      g.N = static_cast<int32_t>(V);
      g.K = static_cast<int32_t>(d);
      g.m_tiles = cdiv(rows, BM);
      g.n_tiles = cdiv(V, BN);
      g.k_blocks = cdiv(d, BK);
      g.m_fastest = 1;
      g.k_split = 1;
      g.row0 = c0;
      g.V = V;
      g.Ktop = K;
      g.zscale = zscale;
      g.idx_sorted = idx_s;
      g.p_sorted = p_s;
      g.row_stats = stats;
      g.lse = lse;
      g.grad_loss = grad_loss;
      g.inv_T_tau = inv_T_tau;
      g.out = dzc;
      g.ldo = L.ldz;
      g.status = status;
      g.wait_limit_ns = limit_ns;
      if (launch_gemm2<Elem, 0, 0, EPI_BWD_DZ>(tH_k, tW_k, tDz_out, g, s, num_sms) != cudaSuccess)
        return KD_ERR_CUDA;

      // (2) dH_c = dz_c W : M = rows, N = d, K = V; A K-major, B MN-major;
      //     K split into even ranges whose fp32 partials are summed in order
      GemmArgs gh = g;
      gh.N = static_cast<int32_t>(d);
      gh.K = static_cast<int32_t>(V);
      gh.n_tiles = cdiv(d, BN);
      gh.k_blocks = cdiv(V, BK);
      gh.m_fastest = 1;
      gh.out = hpart;
      gh.ldo = d;
      gh.row0 = 0;
      gh.split_rows = static_cast<int32_t>(L.rows_pad);
      {
        const int units1 = ((gh.M + BM2 - 1) / BM2) * gh.n_tiles;
        gh.k_split = choose_dh_split(units1,
                                     max_pair_clusters(gemm2_kernel<Elem, 0, 1, EPI_STORE_PARTIAL>,
                                                       num_sms),
                                     gh.k_blocks);
      }
      if (launch_gemm2<Elem, 0, 1, EPI_STORE_PARTIAL>(tDz_k, tW_mn, tHP_out, gh, s, num_sms) !=
          cudaSuccess)
        return KD_ERR_CUDA;
      {
        const int64_t n4 = rows * (d / 4);
        int64_t blocks = (n4 + 255) / 256;
        if (blocks > 4 * static_cast<int64_t>(num_sms)) blocks = 4 * static_cast<int64_t>(num_sms);
        if (launch_pdl(dh_reduce_kernel<Elem>, static_cast<unsigned>(blocks), 256u, s,
                       static_cast<const float*>(hpart), gh.k_split,
                       static_cast<int64_t>(L.rows_pad), static_cast<int>(rows), d,
                       static_cast<Elem*>(dH) + c0 * d) != cudaSuccess)
          return KD_ERR_CUDA;
      }
    }

    // (3) dW (+)= dz_g^T h_g over the group: M = V, N = d, K = grows; both
    //     operands MN-major
    const Elem* hg = static_cast<const Elem*>(h) + g0 * d;
    CUtensorMap tH_mn, tDz_mn;
    if (!make_map(&tH_mn, hg, F32, d, grows, d, INNER, BK, true)) return KD_ERR_CUDA;
    if (!make_map(&tDz_mn, dz, F32, V, grows, L.ldz, INNER, BK, true)) return KD_ERR_CUDA;
    GemmArgs gw;
    memset(&gw, 0, sizeof(gw));
    gw.M = static_cast<int32_t>(V);
    gw.N = static_cast<int32_t>(d);
    gw.K = static_cast<int32_t>(grows);
    gw.m_tiles = cdiv(V, BM);
    gw.n_tiles = cdiv(d, BN);
    gw.k_blocks = cdiv(grows, BK);
    gw.m_fastest = 0;              // tiles sharing one dz slab run together
    gw.k_split = 1;
    gw.V = V;
    gw.out = dW;
    gw.ldo = d;
    gw.accumulate = (accumulate || g0 > 0) ? 1 : 0;
    gw.status = status;
    gw.wait_limit_ns = limit_ns;
    if (launch_gemm2<Elem, 1, 1, EPI_ACCUM_W>(tDz_mn, tH_mn, tDW_out, gw, s, num_sms) !=
        cudaSuccess)
      return KD_ERR_CUDA;
  }
  return KD_OK;
}

kd_status fused_fwd(const void* h, const void* W, int dtype, int64_t T, int64_t T_norm, int64_t d,
                    int64_t V, const float* t_vals, const int32_t* t_idx, int K, int64_t chunk,
                    float tau, uint32_t flags, float* loss, float* lse, float* kl_rows, void* ws,
                    cudaStream_t s, int num_sms, uint64_t limit_ns) {
  if (dtype == KD_DTYPE_F32)
    return fwd_impl<float>(h, W, T, T_norm, d, V, t_vals, t_idx, K, chunk, tau, flags, loss, lse,
                           kl_rows, ws, s, num_sms, limit_ns);
  return fwd_impl<__nv_bfloat16>(h, W, T, T_norm, d, V, t_vals, t_idx, K, chunk, tau, flags, loss,
                                 lse, kl_rows, ws, s, num_sms, limit_ns);
}

kd_status fused_bwd(const void* h, const void* W, int dtype, int64_t T, int64_t T_norm, int64_t d,
                    int64_t V, const float* t_vals, const int32_t* t_idx, int K, int64_t chunk,
                    float tau, uint32_t flags, const float* lse, const float* grad_loss, void* dH,
                    float* dW, int accumulate, void* ws, cudaStream_t s, int num_sms,
                    uint64_t limit_ns) {
  if (dtype == KD_DTYPE_F32)
    return bwd_impl<float>(h, W, T, T_norm, d, V, t_vals, t_idx, K, chunk, tau, flags, lse,
                           grad_loss, dH, dW, accumulate, ws, s, num_sms, limit_ns);
  return bwd_impl<__nv_bfloat16>(h, W, T, T_norm, d, V, t_vals, t_idx, K, chunk, tau, flags, lse,
                                 grad_loss, dH, dW, accumulate, ws, s, num_sms, limit_ns);
}

cudaError_t launch_wait_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  count_launch();
  return cudaGetLastError();
}

}  // namespace kd
