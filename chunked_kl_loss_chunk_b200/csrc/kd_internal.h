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

// Byte offsets of the regions of a fused-loss workspace.
struct WsLayout {
  size_t p_sorted = 0, idx_sorted = 0, stats = 0, kl = 0, scratch = 0, hpart = 0, total = 0;
  int64_t ldz = 0;       // row pitch (elements) of the dz scratch
  int64_t rows_pad = 0;  // chunk rows rounded up to 256 (rows per dH partial)
};

WsLayout ws_layout(int64_t T, int64_t d, int64_t V, int K, int64_t chunk, int dtype);

kd_status fused_fwd(const void* h, const void* W, int dtype, int64_t T, int64_t d, int64_t V,
                    const float* t_vals, const int32_t* t_idx, int K, int64_t chunk, float tau,
                    uint32_t flags, float* loss, float* lse, float* kl_rows, void* ws, cudaStream_t s,
                    int num_sms, uint64_t limit_ns);

kd_status fused_bwd(const void* h, const void* W, int dtype, int64_t T, int64_t d, int64_t V,
                    const float* t_vals, const int32_t* t_idx, int K, int64_t chunk, float tau,
                    uint32_t flags, const float* lse, const float* grad_loss, void* dH, float* dW,
                    int accumulate, void* ws, cudaStream_t s, int num_sms, uint64_t limit_ns);

cudaError_t launch_topk_bf16(const void* logits, int64_t T, int64_t V, int K, float* out_vals,
                             int32_t* out_idx, uint32_t* status, cudaStream_t stream, int num_sms);

cudaError_t launch_wait_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t s);

// Current time limit of device-side waits (kd_set_wait_limit_ns).
uint64_t wait_limit_ns();

// Launch accounting and optional per-GEMM event recording.
void count_launch();
void profile_before(int kind, double flops, cudaStream_t s);
void profile_after(cudaStream_t s);

}  // namespace kd
