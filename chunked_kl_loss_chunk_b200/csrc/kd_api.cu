// kd_api.cu -- the C ABI declared in include/kd.h: argument validation,
// workspace sizing, device status, and dispatch to the kernels.
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "kd_internal.h"

namespace {

std::atomic<uint64_t> g_wait_limit_ns{4000000000ull};  // 4 s; set from any host thread
std::atomic<uint64_t> g_launches{0};

struct Profile {
  void* const* start = nullptr;
  void* const* end = nullptr;
  int* kinds = nullptr;
  double* flops = nullptr;
  int capacity = 0, mask = 0, n = 0;
  bool armed = false;   // set between profile_before and profile_after
} g_prof;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int num_sms_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

using kd::KD_MAX_K;

}  // namespace

namespace kd {

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

// While `s` is being captured into a CUDA graph the record must be external to
// become an event node of the graph (timed on every replay); outside capture
// it is a plain record.  A failed record is cleared so that it can never be
// reported as the failure of the launch it brackets.
static void record_profile_event(void* ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) cs = cudaStreamCaptureStatusNone;
  const cudaError_t e =
      cs == cudaStreamCaptureStatusActive
          ? cudaEventRecordWithFlags(static_cast<cudaEvent_t>(ev), s, cudaEventRecordExternal)
          : cudaEventRecord(static_cast<cudaEvent_t>(ev), s);
  if (e != cudaSuccess) cudaGetLastError();
}

void profile_before(int kind, double flops, cudaStream_t s) {
  g_prof.armed = false;
  if (!g_prof.start || !(g_prof.mask & kind) || g_prof.n >= g_prof.capacity) return;
  record_profile_event(g_prof.start[g_prof.n], s);
  if (g_prof.kinds) g_prof.kinds[g_prof.n] = kind;
  if (g_prof.flops) g_prof.flops[g_prof.n] = flops;
  g_prof.armed = true;
}

void profile_after(cudaStream_t s) {
  if (!g_prof.armed) return;
  record_profile_event(g_prof.end[g_prof.n], s);
  ++g_prof.n;
  g_prof.armed = false;
}

kd_status validate_loss_inputs(const void* h, const void* W, int dtype, int64_t T, int64_t d,
                               int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                               int64_t chunk, float tau) {
  if (!h || !W || !t_vals || !t_idx) return KD_ERR_INVALID_ARG;
  if (T < 1 || d < 1 || V < 1 || K < 1 || K > V || chunk < 1) return KD_ERR_INVALID_ARG;
  if (!(tau > 0.f) || !isfinite(tau)) return KD_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(W, 16) || !aligned(t_vals, 16) || !aligned(t_idx, 16))
    return KD_ERR_INVALID_ARG;
  if (dtype != KD_DTYPE_BF16 && dtype != KD_DTYPE_F32) return KD_ERR_UNSUPPORTED;
  if (d % 8 != 0 || K > KD_MAX_K || V >= (int64_t(1) << 31) - 256 ||
      d >= (int64_t(1) << 31) || T >= (int64_t(1) << 40))
    return KD_ERR_UNSUPPORTED;
  // Rows per chunk: the backward contracts dW over two chunks' rows in one
  // 32-bit GEMM extent.
  if ((chunk < T ? chunk : T) > (int64_t(1) << 30)) return KD_ERR_UNSUPPORTED;
  return KD_OK;
}

}  // namespace kd

extern "C" {

const char* kd_status_string(int status) {
  switch (status) {
    case KD_OK: return "KD_OK";
    case KD_ERR_INVALID_ARG: return "KD_ERR_INVALID_ARG";
    case KD_ERR_UNSUPPORTED: return "KD_ERR_UNSUPPORTED";
    case KD_ERR_WORKSPACE: return "KD_ERR_WORKSPACE";
    case KD_ERR_BAD_INDEX: return "KD_ERR_BAD_INDEX";
    case KD_ERR_TIMEOUT: return "KD_ERR_TIMEOUT";
    case KD_ERR_CUDA: return "KD_ERR_CUDA";
    case KD_ERR_INTERNAL: return "KD_ERR_INTERNAL";
    default: return "KD_ERR_UNKNOWN";
  }
}

int kd_version(void) { return (1 << 16) | 0; }

size_t kd_topk_workspace_size(int64_t T, int64_t V, int K) {
  (void)T;
  (void)V;
  (void)K;
  return 1024;
}

kd_status kd_topk_build(const void* logits, int dtype, int64_t T, int64_t V, int K,
                        float* out_vals, int32_t* out_idx, void* ws, size_t ws_bytes,
                        void* stream) {
  if (!logits || !out_vals || !out_idx || !ws) return KD_ERR_INVALID_ARG;
  if (T < 1 || V < 1 || K < 1 || K > V) return KD_ERR_INVALID_ARG;
  if (!aligned(logits, 16) || !aligned(out_vals, 16) || !aligned(out_idx, 16) ||
      !aligned(ws, 1024))
    return KD_ERR_INVALID_ARG;
  if (dtype != KD_DTYPE_BF16) return KD_ERR_UNSUPPORTED;
  if (K > KD_MAX_K || V >= (int64_t(1) << 31)) return KD_ERR_UNSUPPORTED;
  if (ws_bytes < kd_topk_workspace_size(T, V, K)) return KD_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = num_sms_current();
  if (sms <= 0) return KD_ERR_CUDA;
  // status word and row counter, both zero before the build
  if (cudaMemsetAsync(ws, 0, kd::KD_TOPK_COUNTER_OFFSET + 8, s) != cudaSuccess) return KD_ERR_CUDA;
  unsigned long long* row_counter = reinterpret_cast<unsigned long long*>(
      static_cast<char*>(ws) + kd::KD_TOPK_COUNTER_OFFSET);
  if (kd::launch_topk_bf16(logits, T, V, K, out_vals, out_idx, static_cast<uint32_t*>(ws),
                           row_counter, s, sms) != cudaSuccess)
    return KD_ERR_CUDA;
  return KD_OK;
}

size_t kd_fused_kl_workspace_size(int64_t T, int64_t d, int64_t V, int K, int64_t chunk,
                                  int dtype) {
  if (T < 1 || d < 1 || V < 1 || K < 1 || chunk < 1) return 0;
  const kd::WsLayout L = kd::ws_layout(T, d, V, K, chunk, dtype);
  return L.ok ? L.total : 0;
}

static kd_status validate_loss(const void* h, const void* W, int dtype, int64_t T, int64_t d,
                               int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                               int64_t chunk, float tau, void* ws, size_t ws_bytes) {
  const kd_status st = kd::validate_loss_inputs(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, tau);
  if (st != KD_OK) return st;
  if (!ws || !aligned(ws, kd::KD_WS_ALIGN)) return KD_ERR_INVALID_ARG;
  const kd::WsLayout L = kd::ws_layout(T, d, V, K, chunk, dtype);
  if (!L.ok || ws_bytes < L.total) return KD_ERR_WORKSPACE;
  return KD_OK;
}

}  // extern "C"

// The forward and backward behind every fused-loss entry point; T_norm is the
// count the loss and gradients are normalised by (T, or a whole batch's
// positions for a data-parallel shard of it).
static kd_status fwd_entry(const void* h, const void* W, int dtype, int64_t T, int64_t T_norm,
                           int64_t d, int64_t V, const float* t_vals, const int32_t* t_idx,
                           int K, int64_t chunk, float temperature, uint32_t flags, float* loss,
                           float* lse, float* kl_rows, void* ws, size_t ws_bytes, void* stream) {
  kd_status st =
      validate_loss(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, ws, ws_bytes);
  if (st != KD_OK) return st;
  if ((flags & ~KD_KL_KNOWN_FLAGS) != 0u) return KD_ERR_INVALID_ARG;
  if (T_norm < T) return KD_ERR_INVALID_ARG;
  if (T_norm >= (int64_t(1) << 40)) return KD_ERR_UNSUPPORTED;
  if (!loss || !lse) return KD_ERR_INVALID_ARG;
  if (!aligned(loss, 4) || !aligned(lse, 16) || (kl_rows && !aligned(kl_rows, 16)))
    return KD_ERR_INVALID_ARG;
  const int sms = num_sms_current();
  if (sms <= 0) return KD_ERR_CUDA;
  return kd::fused_fwd(h, W, dtype, T, T_norm, d, V, t_vals, t_idx, K, chunk, temperature, flags,
                       loss, lse, kl_rows, ws, static_cast<cudaStream_t>(stream), sms,
                       kd::wait_limit_ns());
}

static kd_status bwd_entry(const void* h, const void* W, int dtype, int64_t T, int64_t T_norm,
                           int64_t d, int64_t V, const float* t_vals, const int32_t* t_idx,
                           int K, int64_t chunk, float temperature, uint32_t flags,
                           const float* lse, const float* grad_loss, void* dH, float* dW,
                           int accumulate_dW, void* ws, size_t ws_bytes, void* stream) {
  kd_status st =
      validate_loss(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, ws, ws_bytes);
  if (st != KD_OK) return st;
  if ((flags & ~KD_KL_KNOWN_FLAGS) != 0u) return KD_ERR_INVALID_ARG;
  if (T_norm < T) return KD_ERR_INVALID_ARG;
  if (T_norm >= (int64_t(1) << 40)) return KD_ERR_UNSUPPORTED;
  if (!lse || !dH || !dW) return KD_ERR_INVALID_ARG;
  if (!aligned(lse, 16) || !aligned(dH, 16) || !aligned(dW, 16) ||
      (grad_loss && !aligned(grad_loss, 4)))
    return KD_ERR_INVALID_ARG;
  const int sms = num_sms_current();
  if (sms <= 0) return KD_ERR_CUDA;
  return kd::fused_bwd(h, W, dtype, T, T_norm, d, V, t_vals, t_idx, K, chunk, temperature, flags,
                       lse, grad_loss, dH, dW, accumulate_dW, ws,
                       static_cast<cudaStream_t>(stream), sms, kd::wait_limit_ns());
}

extern "C" {

kd_status kd_fused_kl_fwd_ex(const void* h, const void* W, int dtype, int64_t T, int64_t d,
                             int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                             int64_t chunk, float temperature, uint32_t flags, float* loss,
                             float* lse, float* kl_rows, void* ws, size_t ws_bytes,
                             void* stream) {
  return fwd_entry(h, W, dtype, T, T, d, V, t_vals, t_idx, K, chunk, temperature, flags, loss, lse,
                   kl_rows, ws, ws_bytes, stream);
}

kd_status kd_fused_kl_fwd(const void* h, const void* W, int dtype, int64_t T, int64_t d,
                          int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                          int64_t chunk, float temperature, float* loss, float* lse,
                          float* kl_rows, void* ws, size_t ws_bytes, void* stream) {
  return fwd_entry(h, W, dtype, T, T, d, V, t_vals, t_idx, K, chunk, temperature, 0u, loss, lse,
                   kl_rows, ws, ws_bytes, stream);
}

kd_status kd_fused_kl_fwd_shard(const void* h, const void* W, int dtype, int64_t T, int64_t d,
                                int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                                int64_t chunk, float temperature, uint32_t flags, int64_t T_total,
                                float* loss, float* lse, float* kl_rows, void* ws,
                                size_t ws_bytes, void* stream) {
  return fwd_entry(h, W, dtype, T, T_total, d, V, t_vals, t_idx, K, chunk, temperature, flags,
                   loss, lse, kl_rows, ws, ws_bytes, stream);
}

kd_status kd_fused_kl_bwd_ex(const void* h, const void* W, int dtype, int64_t T, int64_t d,
                             int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                             int64_t chunk, float temperature, uint32_t flags, const float* lse,
                             const float* grad_loss, void* dH, float* dW, int accumulate_dW,
                             void* ws, size_t ws_bytes, void* stream) {
  return bwd_entry(h, W, dtype, T, T, d, V, t_vals, t_idx, K, chunk, temperature, flags, lse,
                   grad_loss, dH, dW, accumulate_dW, ws, ws_bytes, stream);
}

kd_status kd_fused_kl_bwd(const void* h, const void* W, int dtype, int64_t T, int64_t d,
                          int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                          int64_t chunk, float temperature, const float* lse,
                          const float* grad_loss, void* dH, float* dW, int accumulate_dW,
                          void* ws, size_t ws_bytes, void* stream) {
  return bwd_entry(h, W, dtype, T, T, d, V, t_vals, t_idx, K, chunk, temperature, 0u, lse,
                   grad_loss, dH, dW, accumulate_dW, ws, ws_bytes, stream);
}

kd_status kd_fused_kl_bwd_shard(const void* h, const void* W, int dtype, int64_t T, int64_t d,
                                int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                                int64_t chunk, float temperature, uint32_t flags, int64_t T_total,
                                const float* lse, const float* grad_loss, void* dH, float* dW,
                                int accumulate_dW, void* ws, size_t ws_bytes, void* stream) {
  return bwd_entry(h, W, dtype, T, T_total, d, V, t_vals, t_idx, K, chunk, temperature, flags, lse,
                   grad_loss, dH, dW, accumulate_dW, ws, ws_bytes, stream);
}

kd_status kd_read_device_status(const void* ws, void* stream) {
  if (!ws) return KD_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return KD_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KD_ERR_CUDA;
  return static_cast<kd_status>(v);
}

uint64_t kd_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

kd_status kd_profile_attach(void* const* start_events, void* const* end_events, int* kinds,
                            double* flops, int capacity, int kind_mask) {
  if (!start_events || !end_events || capacity < 1) return KD_ERR_INVALID_ARG;
  g_prof.start = start_events;
  g_prof.end = end_events;
  g_prof.kinds = kinds;
  g_prof.flops = flops;
  g_prof.capacity = capacity;
  g_prof.mask = kind_mask;
  g_prof.n = 0;
  g_prof.armed = false;
  return KD_OK;
}

int kd_profile_detach(void) {
  const int n = g_prof.n;
  g_prof = Profile{};
  return n;
}

kd_status kd_set_wait_limit_ns(uint64_t limit_ns) {
  if (limit_ns < 1000) return KD_ERR_INVALID_ARG;
  g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
  return KD_OK;
}

kd_status kd_debug_wait_probe(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream) {
  if (!ws || ws_bytes < 1024 || !aligned(ws, 1024)) return KD_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 10000000000ull) return KD_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return KD_ERR_CUDA;
  if (kd::launch_wait_probe(static_cast<uint32_t*>(ws), limit_ns, s) != cudaSuccess)
    return KD_ERR_CUDA;
  return KD_OK;
}

}  // extern "C"
