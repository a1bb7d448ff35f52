"""Seeded synthetic inputs for the distillation-loss workloads.

This module holds random-number plumbing only: it contains none of the loss or
top-K arithmetic.  Both the CUDA path and the CPU checks consume the tensors it
returns (the checks always read back the exact bytes the GPU used).

Distributions (the toy output head of the andresseo.expert page, section "What a
Single H200 GPU Can Now Do That Once Required Four Nodes": d=4096, V=131072):

* student hidden states ``h ~ N(0, 1)``;
* output head ``W ~ N(0, 1/d)`` (nn.Linear layout ``[V, d]``, no bias);
* teacher cache indices: K distinct uniform draws per row (Floyd's sampling);
* teacher cache values ``~ N(0, 2)`` (variance 2) as float32 logits;
* teacher logits for the cache build ``~ N(0, 3)`` (variance 3), rounded to bf16;
* for a cache of full-vocabulary teacher log-probabilities: the same N(0, 2)
  draws shifted per row so that the K cached probabilities sum to a row mass
  ``S ~ U(0.3, 0.95)`` (the rest is the tail the cache dropped).

Every tensor has its own stream: generator seed = ``seed * 1000 + tensor_id``
with ids h=0, W=1, vals=2, idx=3, teacher logits=4, row mass=5.
"""

from __future__ import annotations

import math

import torch

TENSOR_IDS = {"h": 0, "W": 1, "vals": 2, "idx": 3, "logits": 4, "mass": 5}


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + TENSOR_IDS[name])
    return g


def _randn(shape, std: float, dtype, seed: int, name: str, device, rows_per_block: int = 4096):
    """N(0, std^2) drawn in fp32 and rounded to ``dtype``; generated in row
    blocks so that only one fp32 block is alive at a time."""
    g = _gen(seed, name, device)
    out = torch.empty(shape, dtype=dtype, device=device)
    R = shape[0]
    for r0 in range(0, R, rows_per_block):
        r1 = min(R, r0 + rows_per_block)
        blk = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=g, device=device,
                          dtype=torch.float32)
        if std != 1.0:
            blk.mul_(std)
        out[r0:r1].copy_(blk)
        del blk
    return out


def distinct_uniform_indices(T: int, V: int, K: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """K distinct indices per row, uniform over K-subsets of [0, V) (Floyd)."""
    if not (1 <= K <= V):
        raise ValueError("need 1 <= K <= V")
    g = _gen(seed, "idx", device)
    sel = torch.empty((T, K), dtype=torch.int64, device=device)
    for j, top in enumerate(range(V - K, V)):
        r = torch.randint(0, top + 1, (T,), generator=g, device=device, dtype=torch.int64)
        if j:
            dup = (sel[:, :j] == r[:, None]).any(dim=1)
            r = torch.where(dup, torch.full_like(r, top), r)
        sel[:, j] = r
    return sel.to(torch.int32)


def make_loss_inputs(T: int, d: int, V: int, K: int, dtype=torch.bfloat16, seed: int = 0,
                     device="cpu"):
    """(h [T,d], W [V,d], vals f32 [T,K], idx i32 [T,K]) for the fused KL loss."""
    h = _randn((T, d), 1.0, dtype, seed, "h", device)
    W = _randn((V, d), 1.0 / math.sqrt(d), dtype, seed, "W", device)
    vals = _randn((T, K), math.sqrt(2.0), torch.float32, seed, "vals", device)
    idx = distinct_uniform_indices(T, V, K, seed, device)
    return h, W, vals, idx


def make_logprob_cache(T: int, K: int, seed: int = 0, device="cpu", mass=(0.3, 0.95)):
    """Teacher log-probabilities [T, K] f32 of K tokens that carry a row mass
    S_t ~ U(mass) of a full-vocabulary distribution: log S_t plus the
    log-softmax of N(0, 2) draws.  Returns (vals, S)."""
    x = _randn((T, K), math.sqrt(2.0), torch.float32, seed, "vals", device)
    g = _gen(seed, "mass", device)
    S = torch.empty((T,), dtype=torch.float32, device=device).uniform_(mass[0], mass[1], generator=g)
    return torch.log_softmax(x, dim=1) + torch.log(S)[:, None], S


def make_teacher_logits(T: int, V: int, seed: int = 0, device="cpu", dtype=torch.bfloat16,
                        rows_per_block: int = 1024):
    """Teacher logits [T, V] ~ N(0, 3) for the top-K cache build."""
    return _randn((T, V), math.sqrt(3.0), dtype, seed, "logits", device, rows_per_block)


# Workloads, named by what they are.
WORKLOADS = {
    "tiny-fp32": dict(T=256, d=256, V=4096, K=16, chunk=64, dtype="f32"),
    "head-8k": dict(T=8192, d=4096, V=131072, K=100, chunk=1024, dtype="bf16"),
    "head-32k": dict(T=32768, d=4096, V=131072, K=100, chunk=2048, dtype="bf16"),
    "vocab-201k": dict(T=32768, d=2880, V=201088, K=100, chunk=2048, dtype="bf16"),
    "long-256k": dict(T=262144, d=4096, V=131072, K=100, chunk=4096, dtype="bf16"),
    # one and two 2048-position chunks of the 32K head: small cases for profiles
    "head-2k": dict(T=2048, d=4096, V=131072, K=100, chunk=2048, dtype="bf16"),
    "head-4k": dict(T=4096, d=4096, V=131072, K=100, chunk=2048, dtype="bf16"),
    # two pairs of 2048-row chunks: the second dW launch adds into dW
    "head-8k-c2048": dict(T=8192, d=4096, V=131072, K=100, chunk=2048, dtype="bf16"),
}

TOPK_WORKLOADS = {
    "topk-8k": dict(T=8192, V=131072, K=100),
    "topk-201k": dict(T=32768, V=201088, K=100),
}
