"""GPU parity of kd_topk_build against the oracle's brute-force stable sort.

Indices and values must be bit-exact (integer/index work)."""

import math

import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_chunk_b200 import inputs, kd
from gpu_util import require_gpu, to_np_exact

pytestmark = pytest.mark.gpu


def _check_rows(logits, K, rows=None):
    vals, idx = kd.topk_build(logits, K)
    torch.cuda.synchronize()
    x = to_np_exact(logits)
    gv, gi = vals.cpu().numpy(), idx.cpu().numpy()
    if rows is not None:
        x, gv, gi = x[rows], gv[rows], gi[rows]
    ov, oi = oracle.topk_rows(x, K)
    assert np.array_equal(gi, oi), np.argwhere(gi != oi)[:5]
    assert np.array_equal(gv.view(np.uint32), ov.view(np.uint32))


def test_topk_small_random():
    require_gpu()
    x = inputs.make_teacher_logits(64, 4096, seed=1, device="cuda")
    _check_rows(x, 16)
    _check_rows(x, 100)


@pytest.mark.parametrize("T,V,K", [(37, 1003, 7), (5, 4096 + 8 * 3 + 5, 100), (3, 131072, 1),
                                   (9, 300, 300), (17, 8191, 1024), (2, 1, 1)])
def test_topk_ragged_shapes(T, V, K):
    require_gpu()
    x = inputs.make_teacher_logits(T, V, seed=T + V, device="cuda")
    _check_rows(x, K)


def _bf16(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def test_topk_adversarial_rows():
    """Ties, signed zeros, infinities and NaNs (exact fallback path)."""
    require_gpu()
    V = 5000
    rows = []
    rows.append(np.full(V, 3.0))                                  # all equal
    rows.append(np.where(np.arange(V) % 2 == 0, 1.0, 2.0))        # two values
    r = np.zeros(V); r[[7, 4000, 11]] = [5.0, 9.0, 5.0]; rows.append(r)   # K-1 above a wide tie
    r = np.full(V, -math.inf); r[123] = 0.0; rows.append(r)       # -inf run
    r = np.where(np.arange(V) % 3 == 0, -0.0, 0.0); r[4999] = 1.0; rows.append(r)  # +-0
    r = np.full(V, math.nan); r[10] = -math.inf; r[20] = 1.0; rows.append(r)       # NaN heavy
    rows.append(np.arange(V, dtype=np.float64) / 64.0)            # ascending (bad sample)
    rows.append(-np.arange(V, dtype=np.float64) / 64.0)           # descending
    r = np.round(np.random.default_rng(0).standard_normal(V) * 2) / 2; rows.append(r)  # heavy ties
    x = _bf16(np.stack(rows)).cuda().contiguous()
    for K in (1, 3, 100, 1024):
        _check_rows(x, K)


def test_topk_toy_head_8k_sampled():
    """8192 x 131072 bf16 N(0,3) (the cache-build workload); 256 sampled rows."""
    require_gpu()
    x = inputs.make_teacher_logits(8192, 131072, seed=0, device="cuda")
    rows = np.random.default_rng(0).choice(8192, 256, replace=False)
    _check_rows(x, 100, rows)


@pytest.mark.slow
def test_topk_large_vocab_sampled():
    """32768 x 201088 bf16 N(0,3); 128 sampled rows."""
    require_gpu()
    x = inputs.make_teacher_logits(32768, 201088, seed=0, device="cuda")
    rows = np.random.default_rng(1).choice(32768, 128, replace=False)
    _check_rows(x, 100, rows)
