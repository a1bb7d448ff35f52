// kd_noalloc.cu -- kd_fused_kl_fwd_noalloc: the fused chunked KL forward for
// callers that cannot hand the library a workspace.
//
// Some callers have no way to obtain device memory at call time: a plugin that
// is given only its input and output pointers, or a host program whose device
// memory is owned entirely by another framework's pool.  This entry point takes
// its scratch (the sorted teacher cache, per-row KL, the per-tile logsumexp
// partials and the device status word) from a fixed array compiled into the
// library instead, and calls no allocating routine.
//
// The array is a file-scope __device__ object, so every GPU that loads this
// library holds KD_NOALLOC_SCRATCH_BYTES of it until the process exits.  In host
// code its name is only a stand-in for the device object: its device address is
// looked up once per device with cudaGetSymbolAddress (on the first call made
// with that device current) and cached.
#include <math.h>

#include <mutex>

#include "kd_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_kd_noalloc_scratch[KD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).  Returns nullptr and sets *err on failure.
void* scratch_on_current_device(kd_status* err) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err = KD_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kd_noalloc_scratch) != cudaSuccess || !p) {
      *err = KD_ERR_CUDA;
      return nullptr;
    }
    g_addr[dev] = p;
  }
  return g_addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" kd_status kd_fused_kl_fwd_noalloc(const void* h, const void* W, int dtype, int64_t T,
                                             int64_t d, int64_t V, const float* t_vals,
                                             const int32_t* t_idx, int K, int64_t chunk,
                                             float temperature, float* loss, float* lse,
                                             float* kl_rows, void* stream) {
  if (!h || !W || !t_vals || !t_idx || !loss || !lse) return KD_ERR_INVALID_ARG;
  if (T < 1 || d < 1 || V < 1 || K < 1 || K > V || chunk < 1) return KD_ERR_INVALID_ARG;
  if (!(temperature > 0.f) || !isfinite(temperature)) return KD_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(W) || !aligned16(t_vals) || !aligned16(t_idx) ||
      !aligned16(lse) || (kl_rows && !aligned16(kl_rows)) ||
      (reinterpret_cast<uintptr_t>(loss) & 3u))
    return KD_ERR_INVALID_ARG;
  if (dtype != KD_DTYPE_BF16 && dtype != KD_DTYPE_F32) return KD_ERR_UNSUPPORTED;
  if (d % 8 != 0 || K > 1024 || V >= (int64_t(1) << 31) - 256 || d >= (int64_t(1) << 31))
    return KD_ERR_UNSUPPORTED;
  // The forward uses the workspace up to the end of its partials region.
  const kd::WsLayout L = kd::ws_layout(T, d, V, K, chunk, dtype);
  const int64_t rows = chunk < T ? chunk : T;
  const size_t need = L.scratch + static_cast<size_t>(rows) * ((V + 255) / 256) * 16;
  if (need > KD_NOALLOC_SCRATCH_BYTES) return KD_ERR_WORKSPACE;

  kd_status err = KD_OK;
  void* ws = scratch_on_current_device(&err);
  if (!ws) return err;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return KD_ERR_CUDA;
  // fused_fwd clears the status word itself and overwrites every other region
  // it reads, so nothing left by a previous call leaks into this one.
  return kd::fused_fwd(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, 0u, loss,
                       lse, kl_rows, ws, static_cast<cudaStream_t>(stream), sms,
                       kd::wait_limit_ns());
}
