"""The debug build (libkd_debug.so: the same kernels compiled with -DKD_DEBUG=1,
whose device-side invariant checks record KD_ERR_INTERNAL instead of trapping)
on parity cases: every status word must read KD_OK and the results must still
match the oracle.  This stands in for a memory checker, which is not available
on the GPUs these tests run on."""

import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_chunk_b200 import build, inputs, kd
from gpu_util import rel_maxabs, require_gpu, to_np_exact

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def debug_lib():
    require_gpu()
    path = build.build(debug=True)
    prev = kd.use_library(path)
    yield path
    kd.use_library(prev)


def _topk_checked(x, K):
    T, V = x.shape
    ws = kd.alloc_workspace(kd.kd_topk_workspace_size(T, V, K), x.device)
    vals, idx = kd.topk_build(x, K, ws=ws)
    assert kd.read_device_status(ws) == kd.KD_OK
    ov, oi = oracle.topk_rows(to_np_exact(x), K)
    assert np.array_equal(idx.cpu().numpy(), oi)
    assert np.array_equal(vals.cpu().numpy().view(np.uint32), ov.view(np.uint32))


def test_debug_topk_random_and_ragged(debug_lib):
    _topk_checked(inputs.make_teacher_logits(64, 4096, seed=1, device="cuda"), 100)
    _topk_checked(inputs.make_teacher_logits(37, 1003, seed=2, device="cuda"), 7)
    _topk_checked(inputs.make_teacher_logits(5, 8191, seed=3, device="cuda"), 1024)


def test_debug_topk_fallback_rows(debug_lib):
    """Rows that take the exact 3-pass path: all equal, mostly NaN, ascending."""
    V, K = 3000, 50
    rows = [torch.full((V,), 1.5), torch.full((V,), float("nan")), torch.arange(V) / 7.0,
            torch.where(torch.arange(V) % 3 == 0, torch.tensor(-0.0), torch.tensor(0.0))]
    rows[1][::97] = 2.0
    x = torch.stack(rows).to(torch.bfloat16).cuda()
    _topk_checked(x, K)


@pytest.mark.parametrize("T,d,V,K,chunk,dtype", [
    (300, 200, 5000, 16, 100, torch.bfloat16),
    (77, 72, 1003, 7, 33, torch.float32),
    (520, 264, 2304, 100, 512, torch.bfloat16),
    # several work units per cluster (the forward and dz GEMMs: 4 x 128 tile
    # pairs; dW: 128), so the clusters' unit walks advance under the checks
    (1024, 256, 32768, 16, 1024, torch.bfloat16),
])
def test_debug_loss_parity(debug_lib, T, d, V, K, chunk, dtype):
    h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=dtype, seed=T, device="cuda")
    loss, lse, _, ws = kd.fused_kl_fwd(h, W, vals, idx, chunk, 1.0)
    assert kd.read_device_status(ws) == kd.KD_OK
    dH, dW, _ = kd.fused_kl_bwd(h, W, vals, idx, lse, chunk, 1.0, ws=ws)
    assert kd.read_device_status(ws) == kd.KD_OK
    hn, Wn = to_np_exact(h), to_np_exact(W)
    v, i = vals.cpu().numpy(), idx.cpu().numpy()
    lo, lse_o, _ = oracle.forward(hn, Wn, v, i, 1.0)
    assert abs(loss.item() - lo) <= 1e-3 * abs(lo)
    dHo, dWo = oracle.backward(hn, Wn, v, i, 1.0)
    assert rel_maxabs(dH.float().cpu().numpy(), dHo) <= 2e-2
    assert rel_maxabs(dW.cpu().numpy(), dWo) <= 2e-2


def test_debug_build_is_the_library_in_use(debug_lib):
    assert kd.LIB_PATH == debug_lib
