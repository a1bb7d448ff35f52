"""Data-parallel shards of the fused loss through the C ABI, on one GPU.

kd_fused_kl_fwd_shard / kd_fused_kl_bwd_shard normalise by the batch's T_total
instead of the shard's own T, so the shards of a batch, run one after the other
on one device (dW chained with accumulate_dW, the losses summed), must give the
batch's loss and gradients: bit for bit where the shards' chunk and dW-group
boundaries are the batch's own, within the suite's tolerances otherwise, and
against the fp64 oracle of the whole batch.  (On several GPUs the same sums are
all-reduces; ``chunked_kl_loss_chunk_b200.dp`` does that, and its partitioning
and reduction are tested on CPU ranks.)
"""

import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_chunk_b200 import dp, inputs, kd
from gpu_util import rel_maxabs, require_gpu, to_np_exact

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
GRAD_TOL = 2e-2


def _shards_on_one_gpu(h, W, vals, idx, bounds, chunk, tau, **var):
    T_total = h.shape[0]
    losses, lses, dHs = [], [], []
    dW = torch.empty((W.shape[0], W.shape[1]), dtype=torch.float32, device="cuda")
    for i, (a, b) in enumerate(zip(bounds, bounds[1:])):
        sl = slice(a, b)
        loss, lse, _, ws = kd.fused_kl_fwd(h[sl], W, vals[sl], idx[sl], chunk, tau,
                                           T_total=T_total, **var)
        dH, _, _ = kd.fused_kl_bwd(h[sl], W, vals[sl], idx[sl], lse, chunk, tau, ws=ws, dW=dW,
                                   accumulate_dW=i > 0, T_total=T_total, **var)
        losses.append(loss)
        lses.append(lse)
        dHs.append(dH)
        assert kd.read_device_status(ws) == kd.KD_OK
    torch.cuda.synchronize()
    return (torch.stack(losses).double().sum().item(), torch.cat(lses), torch.cat(dHs), dW)


def test_chunk_aligned_shards_are_the_batch_bit_for_bit():
    """Three shards of 200 rows = one dW group (two 100-row chunks) each: every
    launch is the batch's own launch, so lse, dH and dW are bit-identical."""
    require_gpu()
    T, d, V, K, chunk, tau = 600, 128, 3000, 20, 100, 1.3
    h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=torch.bfloat16, seed=21, device="cuda")
    loss_b, lse_b, _, ws = kd.fused_kl_fwd(h, W, vals, idx, chunk, tau)
    dH_b, dW_b, _ = kd.fused_kl_bwd(h, W, vals, idx, lse_b, chunk, tau, ws=ws)
    loss_s, lse_s, dH_s, dW_s = _shards_on_one_gpu(h, W, vals, idx, [0, 200, 400, 600], chunk, tau)
    assert torch.equal(lse_s, lse_b)
    assert torch.equal(dH_s, dH_b)
    assert torch.equal(dW_s, dW_b)
    assert abs(loss_s - loss_b.item()) <= 1e-6 * abs(loss_b.item())
    # and the batch itself against the oracle
    hn, Wn = to_np_exact(h), to_np_exact(W)
    lo, _, _ = oracle.forward(hn, Wn, vals.cpu().numpy(), idx.cpu().numpy(), tau)
    assert abs(loss_s - lo) <= LOSS_RTOL * abs(lo)


@pytest.mark.parametrize("cache,tau_sq,dtype", [("logits", False, torch.bfloat16),
                                                ("logprobs", True, torch.bfloat16),
                                                ("logits", False, torch.float32)])
def test_uneven_shards_match_the_oracle_of_the_batch(cache, tau_sq, dtype):
    """Shards from dp.shard_rows over 3 ranks of an odd batch (blocks that cut
    chunks and dW groups), both cache kinds, with the tau^2 factor, and fp32
    operands (tf32 tensor cores)."""
    require_gpu()
    T, d, V, K, chunk, tau = 517, 96, 2500, 16, 64, 2.0
    h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=dtype, seed=22, device="cuda")
    if cache == "logprobs":
        vals, _ = inputs.make_logprob_cache(T, K, seed=22, device="cuda")
    sh = [dp.shard_rows(T, 3, r) for r in range(3)]
    bounds = [s.row0 for s in sh] + [T]
    var = dict(cache=cache, tau_squared=tau_sq)
    loss_s, lse_s, dH_s, dW_s = _shards_on_one_gpu(h, W, vals, idx, bounds, chunk, tau, **var)
    hn, Wn = to_np_exact(h), to_np_exact(W)
    v, i = vals.cpu().numpy(), idx.cpu().numpy()
    lo, lse_o, _ = oracle.forward(hn, Wn, v, i, tau, cache=cache, tau_sq=tau_sq)
    dH_o, dW_o = oracle.backward(hn, Wn, v, i, tau, cache=cache, tau_sq=tau_sq)
    assert abs(loss_s - lo) <= LOSS_RTOL * abs(lo)
    assert np.abs(lse_s.cpu().numpy() - lse_o).max() <= (5e-3 if dtype == torch.float32 else 1e-3)
    assert rel_maxabs(dH_s.float().cpu().numpy(), dH_o) <= GRAD_TOL
    assert rel_maxabs(dW_s.cpu().numpy(), dW_o) <= GRAD_TOL


def test_shard_with_its_own_T_is_the_plain_call_bit_for_bit():
    require_gpu()
    T, d, V, K, chunk = 300, 64, 2000, 12, 128
    h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=torch.bfloat16, seed=23, device="cuda")
    loss_a, lse_a, _, ws = kd.fused_kl_fwd(h, W, vals, idx, chunk, 0.8)
    dH_a, dW_a, _ = kd.fused_kl_bwd(h, W, vals, idx, lse_a, chunk, 0.8, ws=ws)
    loss_b, lse_b, _, ws = kd.fused_kl_fwd(h, W, vals, idx, chunk, 0.8, T_total=T)
    dH_b, dW_b, _ = kd.fused_kl_bwd(h, W, vals, idx, lse_b, chunk, 0.8, ws=ws, T_total=T)
    torch.cuda.synchronize()
    assert torch.equal(loss_a, loss_b) and torch.equal(lse_a, lse_b)
    assert torch.equal(dH_a, dH_b) and torch.equal(dW_a, dW_b)


def test_dp_shard_step_single_rank_on_gpu():
    """dp.shard_step with the GPU computation and no process group (one rank):
    the whole batch is the rank's shard."""
    require_gpu()
    T, d, V, K, chunk = 256, 64, 1500, 10, 64
    h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=torch.bfloat16, seed=24, device="cuda")
    loss, dH, dW = dp.shard_step(h, W, vals, idx, T, chunk, 1.0)
    torch.cuda.synchronize()
    hn, Wn = to_np_exact(h), to_np_exact(W)
    lo, _, _ = oracle.forward(hn, Wn, vals.cpu().numpy(), idx.cpu().numpy(), 1.0)
    dH_o, dW_o = oracle.backward(hn, Wn, vals.cpu().numpy(), idx.cpu().numpy(), 1.0)
    assert abs(loss.item() - lo) <= LOSS_RTOL * abs(lo)
    assert rel_maxabs(dH.float().cpu().numpy(), dH_o) <= GRAD_TOL
    assert rel_maxabs(dW.cpu().numpy(), dW_o) <= GRAD_TOL
