"""kd_fused_kl_fwd_noalloc: the forward for callers that cannot provide a
workspace (for instance a plugin handed only input/output pointers, or a host
program whose device memory all belongs to another framework's pool).  Its
scratch is a fixed array inside the library, so consecutive calls share it.

Both entry points run the same deterministic kernels on the same inputs (a
fixed-order per-row combine, a one-block fp64 mean), so the call without a
workspace must reproduce kd_fused_kl_fwd bit for bit -- on every call, whatever
the previous call left in the shared array -- and, like every forward, match
the fp64 oracle within the suite's tolerances.

This file sorts last so that a stop-at-first-failure run has already run every
other test before it."""

import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_chunk_b200 import inputs, kd
from gpu_util import require_gpu, to_np_exact

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3   # the suite's loss tolerance
LSE_ATOL = 1e-3    # the suite's lse tolerance (bf16 operands)


def _noalloc(h, W, vals, idx, chunk, tau, with_kl=True):
    T, d = h.shape
    V, K = W.shape[0], vals.shape[1]
    code = kd.KD_DTYPE_F32 if h.dtype == torch.float32 else kd.KD_DTYPE_BF16
    loss = torch.empty((), dtype=torch.float32, device=h.device)
    lse = torch.empty((T,), dtype=torch.float32, device=h.device)
    kl = torch.empty((T,), dtype=torch.float32, device=h.device) if with_kl else None
    st = kd.kd_fused_kl_fwd_noalloc(h.data_ptr(), W.data_ptr(), code, T, d, V,
                                    vals.data_ptr(), idx.data_ptr(), K, chunk, tau, loss.data_ptr(),
                                    lse.data_ptr(), None if kl is None else kl.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    assert st == kd.KD_OK, kd.status_string(st)
    return loss, lse, kl


# Different problems back to back: no call may see the previous call's leftovers
# in the shared scratch array.  The second case is larger than the first (its
# sorted cache and partials reach further into the array); the third is smaller
# again and runs without kl_rows, so per-row KL lives in the array itself.
CASES = [
    dict(T=300, d=200, V=5000, K=16, chunk=100, tau=1.0, seed=11, kl=True, dtype=torch.bfloat16),
    dict(T=513, d=128, V=9000, K=32, chunk=256, tau=1.5, seed=12, kl=True, dtype=torch.bfloat16),
    dict(T=200, d=64, V=3000, K=8, chunk=64, tau=0.7, seed=13, kl=False, dtype=torch.bfloat16),
    dict(T=160, d=96, V=2000, K=12, chunk=48, tau=1.0, seed=14, kl=True, dtype=torch.float32),
]


def test_noalloc_forward_matches_workspace_forward_and_oracle():
    require_gpu()
    for c in CASES:
        h, W, vals, idx = inputs.make_loss_inputs(c["T"], c["d"], c["V"], c["K"],
                                                  dtype=c["dtype"], seed=c["seed"], device="cuda")
        ref_loss, ref_lse, ref_kl, _ = kd.fused_kl_fwd(h, W, vals, idx, c["chunk"], c["tau"],
                                                       kl_rows=True)
        for _ in range(2):                               # two calls in a row on one input
            loss, lse, kl = _noalloc(h, W, vals, idx, c["chunk"], c["tau"], with_kl=c["kl"])
            torch.cuda.synchronize()
            assert torch.equal(loss, ref_loss)
            assert torch.equal(lse, ref_lse)
            if kl is not None:
                assert torch.equal(kl, ref_kl)
        lo, lse_o, kl_o = oracle.forward(to_np_exact(h), to_np_exact(W), vals.cpu().numpy(),
                                         idx.cpu().numpy(), c["tau"])
        lse_tol = 5 * LSE_ATOL if c["dtype"] == torch.float32 else LSE_ATOL   # tf32 products
        assert abs(float(loss.item()) - lo) <= LOSS_RTOL * abs(lo)
        assert np.abs(lse.cpu().numpy() - lse_o).max() <= lse_tol
        if kl is not None:
            assert np.abs(kl.cpu().numpy() - kl_o).max() <= 10 * lse_tol


def test_noalloc_rejects_sizes_beyond_its_scratch():
    require_gpu()
    # T * K * 8 bytes of sorted cache alone exceeds the 64 MiB array: rejected
    # on the host before anything is launched (the pointers are never used).
    fake = 0x7F0000000000
    st = kd.kd_fused_kl_fwd_noalloc(fake, fake, kd.KD_DTYPE_BF16, 1 << 20, 64, 4096, fake, fake, 100,
                                    1024, 1.0, fake, fake, None, None)
    assert st == kd.KD_ERR_WORKSPACE
