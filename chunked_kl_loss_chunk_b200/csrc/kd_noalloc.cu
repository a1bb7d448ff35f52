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
// looked up with cudaGetSymbolAddress, with the device current, the first time
// a call runs in a given CUDA context, and cached under that context's unique
// id (so a context made after cudaDeviceReset, or a caller's own driver-API
// context on the same device, gets its own lookup).
#include <cuda.h>
#include <math.h>

#include <mutex>

#include "kd_internal.h"

namespace {

// The forward's workspace contract: the base and every region are
// KD_WS_ALIGN-aligned (ws_layout places the regions at multiples of it).
static __device__ __align__(1024) unsigned char g_kd_noalloc_scratch[KD_NOALLOC_SCRATCH_BYTES];
static_assert(kd::KD_WS_ALIGN == 1024, "the scratch array's alignment is the workspace contract");

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id (cuCtxGetId) of the calling thread's current context; 0 if there
// is none yet or the driver entry points are unavailable.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

constexpr int kSlots = 64;
struct Slot {
  unsigned long long ctx_id;
  void* addr;
};
std::mutex g_mu;
Slot g_slots[kSlots] = {};
int g_next = 0;

// Device address of the scratch array in the current context.  The lookup
// (cudaGetSymbolAddress, which also makes the device's primary context current
// when the thread has none) runs once per context.  Returns nullptr on failure.
void* scratch_in_current_context() {
  unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  if (id != 0) {
    for (const Slot& s : g_slots)
      if (s.ctx_id == id) return s.addr;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_kd_noalloc_scratch) != cudaSuccess || !p) {
    cudaGetLastError();
    return nullptr;
  }
  if (id == 0) id = current_context_id();   // the lookup made a context current
  if (id != 0) {
    g_slots[g_next] = Slot{id, p};
    g_next = (g_next + 1) % kSlots;
  }
  return p;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" kd_status kd_fused_kl_fwd_noalloc(const void* h, const void* W, int dtype, int64_t T,
                                             int64_t d, int64_t V, const float* t_vals,
                                             const int32_t* t_idx, int K, int64_t chunk,
                                             float temperature, float* loss, float* lse,
                                             float* kl_rows, void* stream) {
  // The same input checks as kd_fused_kl_fwd (one shared routine).
  const kd_status st =
      kd::validate_loss_inputs(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature);
  if (st != KD_OK) return st;
  if (!loss || !lse) return KD_ERR_INVALID_ARG;
  if (!aligned(loss, 4) || !aligned(lse, 16) || (kl_rows && !aligned(kl_rows, 16)))
    return KD_ERR_INVALID_ARG;
  // The forward uses the workspace up to the end of its partials region; every
  // size is computed with overflow checks.
  const kd::WsLayout L = kd::ws_layout(T, d, V, K, chunk, dtype);
  if (!L.ok || L.fwd_end > KD_NOALLOC_SCRATCH_BYTES) return KD_ERR_WORKSPACE;

  void* ws = scratch_in_current_context();
  if (!ws) return KD_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return KD_ERR_CUDA;
  // fused_fwd clears the status word itself and overwrites every other region
  // it reads before reading it, so nothing left by a previous call leaks into
  // this one.
  return kd::fused_fwd(h, W, dtype, T, T, d, V, t_vals, t_idx, K, chunk, temperature, 0u, loss,
                       lse, kl_rows, ws, static_cast<cudaStream_t>(stream), sms,
                       kd::wait_limit_ns());
}
