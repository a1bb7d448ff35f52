// kd_internal.h -- declarations shared by the translation units of libkd.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "kd.h"

namespace kd {

// Largest number of K-splits used for dH = dz W (its fp32 partials live in
// the workspace).
constexpr int KD_DH_MAX_SPLIT = 4;

// Consecutive chunks whose dz the backward keeps side by side, so that dW is
// updated once per group (its read-modify-write traffic falls by this factor).
constexpr int KD_DW_GROUP = 2;

// Largest number of cached teacher entries per position (the prep kernel
// sorts a row's entries in shared memory, and the top-K build keeps up to this
// many in its selection buffer).
constexpr int KD_MAX_K = 1024;

// Alignment of every region of a fused-loss workspace, and of its base: the
// tensor maps encoded over the dz scratch and the dH partials need at least
// 16 bytes, and the regions are placed at multiples of this.
constexpr size_t KD_WS_ALIGN = 1024;

// Byte offsets of the regions of a fused-loss workspace.
// Every size is computed with overflow checks: when a byte count does not fit
// in size_t, `ok` is false and every offset from that point on, and `total`,
// read SIZE_MAX, so no finite workspace is ever accepted for such sizes.
struct WsLayout {
  size_t p_sorted = 0, idx_sorted = 0, stats = 0, kl = 0, scratch = 0, hpart = 0, total = 0;
  size_t fwd_end = 0;    // end of the forward's partials (the forward uses nothing beyond)
  int64_t ldz = 0;       // row pitch (elements) of the dz scratch
  int64_t rows_pad = 0;  // chunk rows rounded up to 256 (rows per dH partial)
  bool ok = true;
};

WsLayout ws_layout(int64_t T, int64_t d, int64_t V, int K, int64_t chunk, int dtype);

// Host validation shared by every fused-loss entry point, for everything but
// the workspace and the outputs: non-null, 16-byte-aligned inputs; positive
// sizes with K <= V; a finite tau > 0 (KD_ERR_INVALID_ARG); a supported dtype,
// d % 8 == 0, K <= KD_MAX_K, V < 2^31 - 256, d < 2^31, T < 2^40 and
// min(chunk, T) <= 2^30 (KD_ERR_UNSUPPORTED).  Makes no CUDA call.
kd_status validate_loss_inputs(const void* h, const void* W, int dtype, int64_t T, int64_t d,
                               int64_t V, const float* t_vals, const int32_t* t_idx, int K,
                               int64_t chunk, float tau);

// The fused loss over T positions whose loss and gradients are normalised by
// T_norm >= T: T_norm == T for a whole batch, the batch's total positions when
// these T rows are one data-parallel shard of it (then the shards' losses and
// dW contributions sum to the batch's).
kd_status fused_fwd(const void* h, const void* W, int dtype, int64_t T, int64_t T_norm, int64_t d,
                    int64_t V, const float* t_vals, const int32_t* t_idx, int K, int64_t chunk,
                    float tau, uint32_t flags, float* loss, float* lse, float* kl_rows, void* ws,
                    cudaStream_t s, int num_sms, uint64_t limit_ns);

kd_status fused_bwd(const void* h, const void* W, int dtype, int64_t T, int64_t T_norm, int64_t d,
                    int64_t V, const float* t_vals, const int32_t* t_idx, int K, int64_t chunk,
                    float tau, uint32_t flags, const float* lse, const float* grad_loss, void* dH,
                    float* dW, int accumulate, void* ws, cudaStream_t s, int num_sms,
                    uint64_t limit_ns);

// The top-K build's workspace: the status word at byte 0 and the row counter
// (zero before each build) at byte 8.
constexpr size_t KD_TOPK_COUNTER_OFFSET = 8;
cudaError_t launch_topk_bf16(const void* logits, int64_t T, int64_t V, int K, float* out_vals,
                             int32_t* out_idx, uint32_t* status, unsigned long long* row_counter,
                             cudaStream_t stream, int num_sms);

cudaError_t launch_wait_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t s);

// Current time limit of device-side waits (kd_set_wait_limit_ns).
uint64_t wait_limit_ns();

// Launch accounting and optional per-GEMM event recording.
void count_launch();
void profile_before(int kind, double flops, cudaStream_t s);
void profile_after(cudaStream_t s);

}  // namespace kd
