"""GPU parity of the fused chunked KL loss (forward and backward) against the
fp64 oracle, through the C ABI.

Tolerances (the parity bar, written here):
  * loss: relative error <= 1e-3;
  * dH, dW: max|gpu - oracle| / max|oracle| <= 2e-2;
  * lse: absolute error <= 1e-3 (bf16 operands multiply exactly and accumulate
    in fp32, so z is good to ~1e-6 relative); <= 5e-3 for fp32 operands, which
    the tensor cores read as tf32 (10-bit mantissa, ~5e-4 relative per operand).
"""

import math

import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_chunk_b200 import inputs, kd
from gpu_util import rel_maxabs, require_gpu, to_np_exact

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-3
GRAD_TOL = 2e-2


def _run(T, d, V, K, chunk, dtype, tau=1.0, g=None, seed=0, acc_init=None, cache="logits",
         tau_sq=False):
    h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=dtype, seed=seed, device="cuda")
    if cache == "logprobs":
        vals, _ = inputs.make_logprob_cache(T, K, seed=seed, device="cuda")
    var = dict(cache=cache, tau_squared=tau_sq)
    loss, lse, kl, ws = kd.fused_kl_fwd(h, W, vals, idx, chunk, tau, kl_rows=True, **var)
    gl = None if g is None else torch.tensor(g, dtype=torch.float32, device="cuda")
    dW0 = None
    if acc_init is not None:
        dW0 = torch.full((V, d), acc_init, dtype=torch.float32, device="cuda")
    dH, dW, _ = kd.fused_kl_bwd(h, W, vals, idx, lse, chunk, tau, grad_loss=gl, ws=ws, dW=dW0,
                                accumulate_dW=acc_init is not None, **var)
    torch.cuda.synchronize()
    assert kd.read_device_status(ws) == kd.KD_OK
    return dict(h=h, W=W, vals=vals, idx=idx, loss=loss, lse=lse, kl=kl, dH=dH, dW=dW,
                cache=cache, tau_sq=tau_sq)


def _full_parity(r, tau=1.0, g=1.0, lse_tol=1e-3, acc_init=None):
    h, W = to_np_exact(r["h"]), to_np_exact(r["W"])
    vals, idx = r["vals"].cpu().numpy(), r["idx"].cpu().numpy()
    var = dict(cache=r["cache"], tau_sq=r["tau_sq"])
    loss, lse, kl = oracle.forward(h, W, vals, idx, tau, **var)
    dH, dW = oracle.backward(h, W, vals, idx, tau, g, **var)
    if acc_init is not None:
        dW = dW + acc_init
    gl = float(r["loss"].item())
    assert abs(gl - loss) <= LOSS_RTOL * abs(loss), (gl, loss)
    assert np.abs(r["lse"].cpu().numpy() - lse).max() <= lse_tol
    assert np.abs(r["kl"].cpu().numpy() - kl).max() <= 10 * lse_tol
    assert rel_maxabs(r["dH"].float().cpu().numpy(), dH) <= GRAD_TOL
    assert rel_maxabs(r["dW"].cpu().numpy(), dW) <= GRAD_TOL
    return dict(loss=loss, lse=lse, dH=dH, dW=dW)


def test_tiny_fp32_config():
    """T=256, d=256, V=4096, K=16, chunk=64, fp32 (the correctness config)."""
    require_gpu()
    r = _run(256, 256, 4096, 16, 64, torch.float32)
    _full_parity(r, lse_tol=5e-3)


@pytest.mark.parametrize("T,d,V,K,chunk,dtype", [
    (300, 200, 5000, 16, 100, torch.bfloat16),     # ragged T, chunk, d (not /64), V (not /32)
    (77, 72, 1003, 7, 33, torch.float32),          # odd V, tiny chunk
    (129, 64, 257, 1, 129, torch.bfloat16),        # K = 1, V just over one tile
    (64, 64, 64, 64, 16, torch.bfloat16),          # K = V
    (520, 264, 2304, 100, 512, torch.bfloat16),    # several M and N tiles, K = 100
])
def test_ragged_shapes(T, d, V, K, chunk, dtype):
    require_gpu()
    r = _run(T, d, V, K, chunk, dtype, seed=T)
    _full_parity(r, lse_tol=5e-3 if dtype == torch.float32 else 1e-3)


@pytest.mark.parametrize("T,d,V,K,chunk,dtype", [
    (1, 8, 40, 3, 1, torch.bfloat16),              # one position, minimum d
    (33, 8, 300, 5, 1, torch.float32),             # chunk = 1: one launch per position
    (5, 16, 1030, 1024, 2, torch.bfloat16),        # K at its maximum
    (3, 4104, 513, 9, 7, torch.bfloat16),          # d > 4096 and not a multiple of 64, T < chunk
    (40, 64, 1024, 1024, 40, torch.bfloat16),      # K = V = 1024
])
def test_edge_shapes(T, d, V, K, chunk, dtype):
    require_gpu()
    r = _run(T, d, V, K, chunk, dtype, seed=T + d)
    _full_parity(r, lse_tol=5e-3 if dtype == torch.float32 else 1e-3)


def test_temperature_grad_scale_and_accumulate():
    require_gpu()
    r = _run(200, 128, 3000, 20, 64, torch.bfloat16, tau=2.0, g=3.0, acc_init=0.25)
    _full_parity(r, tau=2.0, g=3.0, acc_init=0.25)


@pytest.mark.parametrize("T,d,V,K,chunk,dtype,tau,g,tau_sq", [
    (300, 200, 5000, 16, 100, torch.bfloat16, 1.0, None, False),
    (256, 256, 4096, 16, 64, torch.float32, 1.5, 2.0, False),
    (520, 264, 2304, 100, 512, torch.bfloat16, 2.0, 0.5, True),
])
def test_logprob_cache_parity(T, d, V, K, chunk, dtype, tau, g, tau_sq):
    """Cache of full-vocabulary teacher log-probabilities (S < 1, no
    renormalisation; tau scales the student only)."""
    require_gpu()
    r = _run(T, d, V, K, chunk, dtype, tau=tau, g=g, seed=T + 1, cache="logprobs", tau_sq=tau_sq)
    S = torch.exp(r["vals"]).sum(dim=1)
    assert float(S.max()) < 0.96 and float(S.min()) > 0.29
    _full_parity(r, tau=tau, g=1.0 if g is None else g,
                 lse_tol=5e-3 if dtype == torch.float32 else 1e-3)


def test_tau_squared_parity():
    require_gpu()
    r = _run(200, 128, 3000, 20, 64, torch.bfloat16, tau=2.0, g=0.5, tau_sq=True, acc_init=-0.5)
    _full_parity(r, tau=2.0, g=0.5, acc_init=-0.5)


def test_flags_zero_is_the_plain_entry_point_bitwise():
    """kd_fused_kl_fwd_ex / _bwd_ex with flags = 0 are the plain calls."""
    require_gpu()
    T, d, V, K, chunk = 200, 128, 3000, 20, 64
    h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=torch.bfloat16, seed=8,
                                              device="cuda")
    loss_ex, lse_ex, _, ws = kd.fused_kl_fwd(h, W, vals, idx, chunk, 1.3)
    dH_ex, dW_ex, _ = kd.fused_kl_bwd(h, W, vals, idx, lse_ex, chunk, 1.3, ws=ws)
    loss = torch.empty((), dtype=torch.float32, device="cuda")
    lse = torch.empty((T,), dtype=torch.float32, device="cuda")
    dH, dW = torch.empty_like(h), torch.empty((V, d), dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert kd.kd_fused_kl_fwd(h.data_ptr(), W.data_ptr(), kd.KD_DTYPE_BF16, T, d, V,
                              vals.data_ptr(), idx.data_ptr(), K, chunk, 1.3, loss.data_ptr(),
                              lse.data_ptr(), None, ws.data_ptr(), ws.numel(), s) == kd.KD_OK
    assert kd.kd_fused_kl_bwd(h.data_ptr(), W.data_ptr(), kd.KD_DTYPE_BF16, T, d, V,
                              vals.data_ptr(), idx.data_ptr(), K, chunk, 1.3, lse.data_ptr(), None,
                              dH.data_ptr(), dW.data_ptr(), 0, ws.data_ptr(), ws.numel(),
                              s) == kd.KD_OK
    torch.cuda.synchronize()
    assert torch.equal(loss, loss_ex) and torch.equal(lse, lse_ex)
    assert torch.equal(dH, dH_ex) and torch.equal(dW, dW_ex)


def test_chunk_invariance_bitwise():
    """Per-row results do not depend on the chunk size; the loss is bit-identical."""
    require_gpu()
    h, W, vals, idx = inputs.make_loss_inputs(384, 128, 6000, 16, dtype=torch.bfloat16, seed=3,
                                              device="cuda")
    outs = [kd.fused_kl_fwd(h, W, vals, idx, c, 1.0) for c in (384, 128, 100, 7)]
    torch.cuda.synchronize()
    for loss, lse, _, _ in outs[1:]:
        assert torch.equal(loss, outs[0][0])
        assert torch.equal(lse, outs[0][1])
    dHs = [kd.fused_kl_bwd(h, W, vals, idx, outs[0][1], c, 1.0)[:2] for c in (384, 100)]
    torch.cuda.synchronize()
    assert torch.equal(dHs[0][0], dHs[1][0])                       # dH rows independent
    assert rel_maxabs(dHs[1][1].cpu().numpy(), dHs[0][1].cpu().numpy()) <= 1e-5


def test_zero_loss_when_student_reproduces_teacher():
    """d = V = 64, W = I, h = teacher logits (bf16-exact) at idx and -60 elsewhere:
    exact KL ~ 1e-24; fp32 cancellation of O(5) terms leaves ~1e-6."""
    require_gpu()
    T, V, K = 256, 64, 8
    _, _, vals, idx = inputs.make_loss_inputs(T, V, V, K, dtype=torch.bfloat16, seed=5, device="cuda")
    vals = vals.to(torch.bfloat16).float()
    W = torch.eye(V, dtype=torch.bfloat16, device="cuda")
    h = torch.full((T, V), -60.0, dtype=torch.float32, device="cuda")
    h.scatter_(1, idx.long(), vals)
    h = h.to(torch.bfloat16)
    loss, lse, kl, _ = kd.fused_kl_fwd(h, W, vals.contiguous(), idx, 64, 1.0, kl_rows=True)
    torch.cuda.synchronize()
    assert abs(loss.item()) < 1e-5
    assert kl.abs().max().item() < 1e-4


def test_bad_index_recorded_not_faulted():
    require_gpu()
    h, W, vals, idx = inputs.make_loss_inputs(64, 64, 500, 8, dtype=torch.bfloat16, seed=1, device="cuda")
    idx = idx.clone()
    idx[3, 2] = 500 + 7          # out of range
    idx[9, 1] = idx[9, 4]        # duplicate
    loss, lse, _, ws = kd.fused_kl_fwd(h, W, vals, idx, 32, 1.0)
    assert kd.read_device_status(ws) == kd.KD_ERR_BAD_INDEX
    kd.fused_kl_bwd(h, W, vals, idx, lse, 32, 1.0, ws=ws)
    assert kd.read_device_status(ws) == kd.KD_ERR_BAD_INDEX
    # status is cleared by the next call on clean inputs
    _, _, vals2, idx2 = inputs.make_loss_inputs(64, 64, 500, 8, dtype=torch.bfloat16, seed=1, device="cuda")
    kd.fused_kl_fwd(h, W, vals2, idx2, 32, 1.0, ws=ws)
    assert kd.read_device_status(ws) == kd.KD_OK


def test_bounded_wait_times_out_and_context_survives():
    """A wait on a barrier nothing arrives at returns KD_ERR_TIMEOUT by itself."""
    require_gpu()
    ws = kd.alloc_workspace(4096, "cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert kd.kd_debug_wait_probe(ws.data_ptr(), ws.numel(), 2_000_000, st) == kd.KD_OK
    assert kd.read_device_status(ws) == kd.KD_ERR_TIMEOUT
    r = _run(128, 64, 1000, 8, 64, torch.bfloat16)          # the context still works
    _full_parity(r)


def test_autograd_function():
    require_gpu()
    h, W, vals, idx = inputs.make_loss_inputs(96, 64, 777, 10, dtype=torch.bfloat16, seed=2, device="cuda")
    h.requires_grad_(True)
    W.requires_grad_(True)
    loss = kd.FusedTopKKLLoss.apply(h, W, vals, idx, 40, 1.0)
    (2.0 * loss).backward()
    torch.cuda.synchronize()
    hn, Wn = to_np_exact(h), to_np_exact(W)
    dH, dW = oracle.backward(hn, Wn, vals.cpu().numpy(), idx.cpu().numpy(), 1.0, 2.0)
    assert rel_maxabs(h.grad.float().cpu().numpy(), dH) <= GRAD_TOL
    assert rel_maxabs(W.grad.float().cpu().numpy(), dW) <= GRAD_TOL


def test_autograd_function_logprob_cache_tau_squared():
    require_gpu()
    T, d, V, K = 96, 64, 777, 10
    h, W, _, idx = inputs.make_loss_inputs(T, d, V, K, dtype=torch.bfloat16, seed=4, device="cuda")
    vals, _ = inputs.make_logprob_cache(T, K, seed=4, device="cuda")
    h.requires_grad_(True)
    W.requires_grad_(True)
    loss = kd.FusedTopKKLLoss.apply(h, W, vals, idx, 40, 1.5, "logprobs", True)
    (0.75 * loss).backward()
    torch.cuda.synchronize()
    hn, Wn = to_np_exact(h), to_np_exact(W)
    v, i = vals.cpu().numpy(), idx.cpu().numpy()
    lo, _, _ = oracle.forward(hn, Wn, v, i, 1.5, cache="logprobs", tau_sq=True)
    assert abs(loss.item() - lo) <= LOSS_RTOL * abs(lo)
    dH, dW = oracle.backward(hn, Wn, v, i, 1.5, 0.75, cache="logprobs", tau_sq=True)
    assert rel_maxabs(h.grad.float().cpu().numpy(), dH) <= GRAD_TOL
    assert rel_maxabs(W.grad.float().cpu().numpy(), dW) <= GRAD_TOL


def test_chain_topk_build_then_loss():
    """The offline pipeline end to end: teacher logits [T, V] -> kd_topk_build
    -> cache -> fused forward and backward, against the oracle's own top-K and
    loss on the same teacher logits."""
    require_gpu()
    T, d, V, K, chunk = 160, 96, 3000, 20, 64
    h, W, _, _ = inputs.make_loss_inputs(T, d, V, K, dtype=torch.bfloat16, seed=6, device="cuda")
    x = inputs.make_teacher_logits(T, V, seed=6, device="cuda")
    vals, idx = kd.topk_build(x, K)
    loss, lse, _, ws = kd.fused_kl_fwd(h, W, vals, idx, chunk, 1.0)
    dH, dW, _ = kd.fused_kl_bwd(h, W, vals, idx, lse, chunk, 1.0, ws=ws)
    torch.cuda.synchronize()
    assert kd.read_device_status(ws) == kd.KD_OK
    ov, oi = oracle.topk_rows(to_np_exact(x), K)
    assert np.array_equal(idx.cpu().numpy(), oi)
    assert np.array_equal(vals.cpu().numpy().view(np.uint32), ov.view(np.uint32))
    hn, Wn = to_np_exact(h), to_np_exact(W)
    lo, _, _ = oracle.forward(hn, Wn, ov, oi, 1.0)
    assert abs(loss.item() - lo) <= LOSS_RTOL * abs(lo)
    dHo, dWo = oracle.backward(hn, Wn, ov, oi, 1.0)
    assert rel_maxabs(dH.float().cpu().numpy(), dHo) <= GRAD_TOL
    assert rel_maxabs(dW.cpu().numpy(), dWo) <= GRAD_TOL


# ------------------------------------------------------------------ full-size

def _sampled_full_size(name, n_rows, n_vrows=0):
    cfg = inputs.WORKLOADS[name]
    T, d, V, K, chunk = cfg["T"], cfg["d"], cfg["V"], cfg["K"], cfg["chunk"]
    r = _run(T, d, V, K, chunk, torch.bfloat16)
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(T, n_rows, replace=False))
    rows[0] = 0
    rows[-1] = T - 1                                 # both ends of the last (ragged) chunk
    hn, Wn = to_np_exact(r["h"]), to_np_exact(r["W"])
    vals, idx = r["vals"].cpu().numpy(), r["idx"].cpu().numpy()
    lse_o, kl_o = oracle.forward_rows(hn, Wn, vals, idx, 1.0, rows)
    assert np.abs(r["lse"].cpu().numpy()[rows] - lse_o).max() <= 1e-3
    assert np.abs(r["kl"].cpu().numpy()[rows] - kl_o).max() <= 1e-2
    dH_o = oracle.backward_dH_rows(hn, Wn, vals, idx, 1.0, rows, T)
    assert rel_maxabs(r["dH"].float().cpu().numpy()[rows], dH_o) <= GRAD_TOL
    # the loss is the mean of the per-row KL (checked above on sampled rows)
    kl_all = r["kl"].cpu().numpy().astype(np.float64)
    assert abs(r["loss"].item() - kl_all.mean()) <= 1e-6 * abs(kl_all.mean())
    # zero-sum invariant: sum_v dz = 0 (S = 1) => sum_v dW[v, :] = 0
    dW = r["dW"]
    colsum = dW.double().sum(dim=0).abs().max().item()
    assert colsum <= 1e-3 * dW.abs().max().item() * math.sqrt(V)
    return r


def test_toy_head_8k_sampled():
    """T=8192, d=4096, V=131072, K=100, chunk=1024 (bench launch config)."""
    require_gpu()
    _sampled_full_size("head-8k", 32)


@pytest.mark.slow
def test_toy_head_32k_sampled():
    """T=32768, d=4096, V=131072, K=100, chunk=2048 (the headline workload)."""
    require_gpu()
    _sampled_full_size("head-32k", 24)


@pytest.mark.slow
def test_large_vocab_sampled():
    """4 x 8192 positions, d=2880, V=201088 (V % 256 = 128), K=100, chunk=2048."""
    require_gpu()
    _sampled_full_size("vocab-201k", 16)


@pytest.mark.slow
def test_long_context_256k_sampled():
    """T=262144, d=4096, V=131072, K=100, chunk=4096."""
    require_gpu()
    _sampled_full_size("long-256k", 8)


def test_dW_sampled_vocab_rows_full_width():
    """Full d and V with a short T so the oracle's all-row LSE stays cheap:
    T=384, d=4096, V=131072, K=100, chunk=256; 48 vocabulary rows of dW
    (including every teacher index of row 0)."""
    require_gpu()
    T, d, V, K, chunk = 384, 4096, 131072, 100, 256
    r = _run(T, d, V, K, chunk, torch.bfloat16)
    hn, Wn = to_np_exact(r["h"]), to_np_exact(r["W"])
    vals, idx = r["vals"].cpu().numpy(), r["idx"].cpu().numpy()
    vrows = np.unique(np.concatenate([idx[0, :24], np.random.default_rng(2).choice(V, 24, replace=False),
                                      [0, V - 1]]))
    dW_o = oracle.backward_dW_rows(hn, Wn, vals, idx, 1.0, vrows)
    assert rel_maxabs(r["dW"].cpu().numpy()[vrows], dW_o) <= GRAD_TOL
    loss_o, _, _ = oracle.forward(hn, Wn, vals, idx, 1.0)
    assert abs(r["loss"].item() - loss_o) <= LOSS_RTOL * abs(loss_o)


def _dW_rows_parity_accumulating(T, d, V, K, chunk, tail_rows=0, n_random=32, seed=0):
    """dW element by element on sampled vocabulary rows, at full d and V, over a
    backward whose dW launches mostly ADD into dW (one launch per group of two
    chunks: the first stores, every later one reduce-adds).  The reference is
    the oracle's own: it computes LSE_t of every position itself (one full fp64
    projection) and never reads the GPU's lse.  The rows checked are 0, V-1,
    every teacher index of three positions (one in the first group, one in a
    middle group, the last position), random rows and, optionally, the last
    `tail_rows` rows (the ragged last M tile of the dW GEMM when V % 256 != 0).
    A lost, doubled or stored-instead-of-added group changes every one of them."""
    groups = -(-T // (2 * chunk))
    assert groups >= 3, "the check wants at least two accumulating dW launches"
    r = _run(T, d, V, K, chunk, torch.bfloat16, seed=seed)
    hn, Wn = to_np_exact(r["h"]), to_np_exact(r["W"])
    vals, idx = r["vals"].cpu().numpy(), r["idx"].cpu().numpy()
    rng = np.random.default_rng(seed + 7)
    pos = [0, T // 2 + 1, T - 1]
    vrows = np.unique(np.concatenate([idx[pos].ravel(), rng.choice(V, n_random, replace=False),
                                      [0, V - 1], np.arange(V - tail_rows, V)]).astype(np.int64))
    dW_o = oracle.backward_dW_rows(hn, Wn, vals, idx, 1.0, vrows)
    dW_g = r["dW"][torch.as_tensor(vrows, device="cuda")].cpu().numpy()
    err = rel_maxabs(dW_g, dW_o)
    assert err <= GRAD_TOL, err
    # every checked row is non-trivial (a zeroed row would fail the bar above)
    assert np.abs(dW_o).max(axis=1).min() > 0.0
    return err


@pytest.mark.slow
def test_dW_full_size_head_8k_accumulating():
    """T=8192, d=4096, V=131072, K=100, chunk=1024: four dW launches, three of
    them reduce-adding into dW."""
    require_gpu()
    cfg = inputs.WORKLOADS["head-8k"]
    _dW_rows_parity_accumulating(cfg["T"], cfg["d"], cfg["V"], cfg["K"], cfg["chunk"])


@pytest.mark.slow
def test_dW_full_size_large_vocab_accumulating():
    """d=2880, V=201088 (V % 256 = 128), K=100, chunk=1024, T=6144: three dW
    launches, two of them reduce-adding, and the last 128 vocabulary rows (the
    ragged M tail of every dW launch) checked element by element."""
    require_gpu()
    cfg = inputs.WORKLOADS["vocab-201k"]
    _dW_rows_parity_accumulating(6144, cfg["d"], cfg["V"], cfg["K"], 1024, tail_rows=128)


@pytest.mark.slow
def test_peak_memory_linear_in_T():
    """Peak device memory of fwd + bwd grows linearly in T (the pages: memory
    grows only linearly with sequence length), with a per-token slope close to
    h + dH (bf16) + the cache and its prepared copy + lse, and far below the
    dense [T, V] fp32 logits grid (512 KB per token at V = 131072)."""
    require_gpu()
    d, V, K, chunk = 4096, 131072, 100, 2048
    Ts = [4096, 8192, 16384, 32768]
    peaks = []
    dev = torch.device("cuda")
    for T in Ts:
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        base = torch.cuda.memory_allocated(dev)
        h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=torch.bfloat16, seed=1, device=dev)
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats(dev)        # the generator's temporaries are gone
        loss, lse, kl, ws = kd.fused_kl_fwd(h, W, vals, idx, chunk, 1.0)
        dH, dW, ws_b = kd.fused_kl_bwd(h, W, vals, idx, lse, chunk, 1.0, ws=ws)
        torch.cuda.synchronize()
        assert kd.read_device_status(ws) == kd.KD_OK
        peaks.append(torch.cuda.max_memory_allocated(dev) - base)
        # drop every reference (the workspace is returned twice), so that the
        # next T's baseline holds none of this T's buffers
        del h, W, vals, idx, loss, lse, kl, ws, ws_b, dH, dW
    x = np.array(Ts, np.float64)
    y = np.array(peaks, np.float64)
    b, a = np.polyfit(x, y, 1)
    r2 = 1 - ((y - (a + b * x)) ** 2).sum() / ((y - y.mean()) ** 2).sum()
    expected = 2 * d * 2 + 8 * K + 8 * K + 12 + 4          # h, dH, cache, prepared cache, stats, lse
    assert r2 > 0.999, (peaks, r2)
    assert 0.9 * expected <= b <= 1.25 * expected, (b, expected)
    assert b < 0.05 * V * 4


def test_repeated_steps_bit_identical():
    """The kernels of a call overlap their neighbours (programmatic dependent
    launch) and wait inside for what those write; a missing wait would show as
    run-to-run differences.  Many chunks (so many GEMM/combine/reduce hand-offs),
    two dW groups with a ragged last chunk, run five times on one stream with
    other work in between: every output bit-identical every time."""
    require_gpu()
    T, d, V, K, chunk = 1000, 256, 9000, 32, 96
    h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=torch.bfloat16, seed=31, device="cuda")
    outs = []
    scratch = torch.empty(1 << 24, dtype=torch.float32, device="cuda")
    for rep in range(5):
        scratch.uniform_()                          # unrelated work on the same stream
        loss, lse, kl, ws = kd.fused_kl_fwd(h, W, vals, idx, chunk, 1.0, kl_rows=True)
        dH, dW, _ = kd.fused_kl_bwd(h, W, vals, idx, lse, chunk, 1.0, ws=ws)
        torch.cuda.synchronize()
        assert kd.read_device_status(ws) == kd.KD_OK
        outs.append([t.clone() for t in (loss, lse, kl, dH, dW)])
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert torch.equal(a, b)
    hn, Wn = to_np_exact(h), to_np_exact(W)
    lo, _, _ = oracle.forward(hn, Wn, vals.cpu().numpy(), idx.cpu().numpy(), 1.0)
    assert abs(outs[0][0].item() - lo) <= LOSS_RTOL * abs(lo)
