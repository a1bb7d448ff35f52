"""kd_fused_kl_fwd_noalloc: the forward for callers that cannot provide a
workspace (for instance a plugin handed only input/output pointers, or a host
program whose device memory all belongs to another framework's pool).  Its
scratch is a fixed array inside the library, so two calls in a row share it;
each must still reproduce kd_fused_kl_fwd exactly as the other tests require.

This file sorts last so that a stop-at-first-failure run has already run every
other test before it."""

import numpy as np
import pytest
import torch

from chunked_kl_loss_chunk_b200 import inputs, kd
from gpu_util import require_gpu

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3   # the suite's loss tolerance
LSE_ATOL = 1e-3    # the suite's lse tolerance (bf16 operands)


def _noalloc(h, W, vals, idx, chunk, tau):
    T, d = h.shape
    V, K = W.shape[0], vals.shape[1]
    loss = torch.empty((), dtype=torch.float32, device=h.device)
    lse = torch.empty((T,), dtype=torch.float32, device=h.device)
    kl = torch.empty((T,), dtype=torch.float32, device=h.device)
    st = kd.kd_fused_kl_fwd_noalloc(h.data_ptr(), W.data_ptr(), kd.KD_DTYPE_BF16, T, d, V,
                                    vals.data_ptr(), idx.data_ptr(), K, chunk, tau, loss.data_ptr(),
                                    lse.data_ptr(), kl.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == kd.KD_OK, kd.status_string(st)
    return loss, lse, kl


def test_noalloc_forward_matches_workspace_forward_twice():
    require_gpu()
    # Two different problems back to back: the second call must not see the
    # first call's leftovers in the shared scratch array.
    cases = [(300, 200, 5000, 16, 100, 1.0, 11), (513, 128, 9000, 32, 256, 1.5, 12)]
    for T, d, V, K, chunk, tau, seed in cases:
        h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=torch.bfloat16, seed=seed,
                                                  device="cuda")
        ref_loss, ref_lse, ref_kl, _ = kd.fused_kl_fwd(h, W, vals, idx, chunk, tau, kl_rows=True)
        loss, lse, kl = _noalloc(h, W, vals, idx, chunk, tau)
        torch.cuda.synchronize()
        r = float(ref_loss.item())
        assert abs(float(loss.item()) - r) <= LOSS_RTOL * abs(r)
        assert (lse - ref_lse).abs().max().item() <= LSE_ATOL
        assert (kl - ref_kl).abs().max().item() <= 10 * LSE_ATOL


def test_noalloc_rejects_sizes_beyond_its_scratch():
    require_gpu()
    # T * K * 8 bytes of sorted cache alone exceeds the 64 MiB array: rejected
    # on the host before anything is launched (the pointers are never used).
    fake = 0x7F0000000000
    st = kd.kd_fused_kl_fwd_noalloc(fake, fake, kd.KD_DTYPE_BF16, 1 << 20, 64, 4096, fake, fake, 100,
                                    1024, 1.0, fake, fake, None, None)
    assert st == kd.KD_ERR_WORKSPACE
