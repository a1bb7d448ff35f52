"""Plain, slow, obviously-correct fp64 CPU oracle (TEST INFRASTRUCTURE ONLY).

What the pages fix, and the readings taken where they are silent:

* Offline cache ([DD] "The two changes"; [GX] "Detailed Chronology and
  Technical Evolution"; [AS] "Offline Top-K"): the teacher is run once and the
  top-100 tokens of every position are cached as (logit value, token index).
  Reading: the cache holds the teacher *logits*; ties at the boundary go to the
  lower token index; the list is ordered by value descending, index ascending;
  +0 and -0 compare equal; NaN ranks below -inf.
* Fused chunked KL ([DD] "The two changes"; [ST]; [AS] "Fused Chunked KL"):
  per chunk of positions, project hidden states to logits, fold the chunk's KL
  into the running loss, discard the chunk; the backward recomputes each chunk.
  The pages state (in [AS] "Caching Once, Training Forever") that neither change
  alters the mathematical objective, so the oracle is the plain definition:

      z[t,v]   = sum_j h[t,j] W[v,j]
      a[t,v]   = z[t,v] / tau,    LSE_t = log sum_v exp(a[t,v])
      p[t,k]   = softmax_k(vals[t,k] / tau)        (renormalised teacher top-K)
      S_t      = sum_k p[t,k]
      KL_t     = sum_k p[t,k] (log p[t,k] - (a[t,idx[t,k]] - LSE_t))
      loss     = (1/T) sum_t KL_t
      dz[t,v]  = g / (T tau) * (S_t exp(a[t,v] - LSE_t) - sum_k p[t,k] [v == idx[t,k]])
      dH       = dz W,      dW = dz^T h

  Readings: KL(p_teacher || q_student); temperature divides both teacher and
  student logits, no tau^2 factor; the reduction is the mean over all T
  positions; 0 log 0 := 0.

Two variants of the same objective (every function takes them as keywords):

* ``cache="logprobs"``: the cache holds the teacher's log-probabilities from a
  softmax over the FULL vocabulary, so the K cached entries carry only part of
  the mass: p[t,k] = exp(vals[t,k]) as given (no renormalisation, no
  temperature: it was applied when the teacher ran), S_t = sum_k p <= 1, and
  sum p log p = sum_k p[t,k] vals[t,k].  The formulas above then hold with this
  p and S unchanged (the gradient keeps its S_t softmax - p form).
* ``tau_sq=True``: the loss and every gradient are multiplied by tau^2, the
  usual temperature compensation of distillation; the per-row KL_t is returned
  unscaled.

All arithmetic is fp64.  Inputs are the exact values the GPU consumed (bf16 bit
patterns are widened exactly).  Rows are processed in blocks only to bound host
memory; every row's result is computed independently from its definition.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "topk_rows",
    "teacher_distribution",
    "loss_weight",
    "forward",
    "forward_rows",
    "backward",
    "backward_dH_rows",
    "backward_dW_rows",
    "dense_bruteforce_loss",
]


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns (uint16/int16) to float64.

    A bfloat16 value is the upper half of the float32 with the same bits, so the
    widening is a 16-bit left shift into a float32 followed by an exact cast.
    """
    u = np.asarray(bits).view(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def _as_f64(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.uint16 or x.dtype == np.int16:
        return bf16_bits_to_f64(x)
    return x.astype(np.float64, copy=False)


# ---------------------------------------------------------------------------
# a1: top-K cache build  ([DD] "The two changes": top-100 tokens per position)
# ---------------------------------------------------------------------------

def topk_rows(x, K: int):
    """Per row, the K entries ranked by (value descending, index ascending).

    ``x``: [T, V] teacher logits (bf16 bit patterns or floats).  Returns
    ``vals`` float32 [T, K] (exact copies of the selected logits) and ``idx``
    int32 [T, K].  Ranking: NaN below everything (including -inf); +0 == -0;
    among equal values the lower index first.  Implemented as a full stable
    sort of every row, i.e. by brute force.
    """
    xv = _as_f64(x)
    T, V = xv.shape
    if not (1 <= K <= V):
        raise ValueError("need 1 <= K <= V")
    out_v = np.empty((T, K), np.float32)
    out_i = np.empty((T, K), np.int32)
    cols = np.arange(V)
    for t in range(T):
        row = xv[t]
        isnan = np.isnan(row)
        # +0.0 turns -0.0 into +0.0, so the two compare (and sort) equal.
        val = np.where(isnan, 0.0, row) + 0.0
        # lexsort: last key is primary.  Primary: non-NaN first; then value
        # descending; then index ascending.
        order = np.lexsort((cols, -val, isnan))[:K]
        out_i[t] = order
        out_v[t] = row[order].astype(np.float32)
    return out_v, out_i


# ---------------------------------------------------------------------------
# a2: renormalised teacher distribution over the cached K entries
# ---------------------------------------------------------------------------

CACHE_KINDS = ("logits", "logprobs")


def teacher_distribution(vals, tau: float, cache: str = "logits"):
    """Teacher probabilities at the K cached entries.

    ``cache="logits"``: p = softmax over the K cached logits at temperature tau
    (renormalised, S = 1).  ``cache="logprobs"``: p = exp(vals), the teacher's
    own full-vocabulary probabilities, S <= 1.

    Returns (p [T,K], S [T] = sum_k p, plogp [T] = sum_k p log p with 0 log 0 = 0).
    """
    if cache not in CACHE_KINDS:
        raise ValueError(f"cache must be one of {CACHE_KINDS}")
    v = _as_f64(vals)
    if cache == "logprobs":
        p = np.exp(v)
        S = p.sum(axis=1)
        plogp = np.where(p > 0.0, p * np.where(p > 0.0, v, 0.0), 0.0).sum(axis=1)
        return p, S, plogp
    b = v / tau
    bmax = b.max(axis=1, keepdims=True)
    e = np.exp(b - bmax)
    p = e / e.sum(axis=1, keepdims=True)
    S = p.sum(axis=1)
    safe = np.where(p > 0.0, p, 1.0)
    plogp = np.where(p > 0.0, p * np.log(safe), 0.0).sum(axis=1)
    return p, S, plogp


def loss_weight(tau: float, tau_sq: bool) -> float:
    """Factor on the loss and its gradients: tau^2 with ``tau_sq``, else 1."""
    return tau * tau if tau_sq else 1.0


def _row_block_stats(h_rows, W, tau):
    """z, a = z/tau and LSE for a block of rows (full vocabulary)."""
    z = h_rows @ W.T
    a = z / tau
    amax = a.max(axis=1, keepdims=True)
    lse = amax[:, 0] + np.log(np.exp(a - amax).sum(axis=1))
    return z, a, lse


def _kl_from(a_rows, lse_rows, p_rows, idx_rows):
    """KL_t = sum_k p (log p - (a_at_idx - LSE)), 0 log 0 = 0."""
    a_at = np.take_along_axis(a_rows, idx_rows.astype(np.int64), axis=1)
    logq = a_at - lse_rows[:, None]
    safe = np.where(p_rows > 0.0, p_rows, 1.0)
    terms = np.where(p_rows > 0.0, p_rows * (np.log(safe) - logq), 0.0)
    return terms.sum(axis=1)


# ---------------------------------------------------------------------------
# a3/a4: forward  (project, full-vocab logsumexp, gather at idx, fold, discard)
# ---------------------------------------------------------------------------

def forward(h, W, vals, idx, tau: float = 1.0, row_block: int = 256, cache: str = "logits",
            tau_sq: bool = False, T_norm: int | None = None):
    """Full forward: returns (loss, lse [T], kl [T]); loss carries the tau^2
    factor when ``tau_sq``, kl does not.

    ``T_norm`` (default T) is the number of positions the mean divides by:
    when these T rows are one shard of a batch of T_norm positions, the loss
    returned is this shard's part of the batch's mean, (1/T_norm) sum_t KL_t.

    ``row_block`` only bounds host memory (each row is independent); results do
    not depend on it except through fp64 rounding of the final mean.
    """
    h64, W64 = _as_f64(h), _as_f64(W)
    idx = np.asarray(idx)
    T = h64.shape[0]
    p, _, _ = teacher_distribution(vals, tau, cache)
    lse = np.empty(T)
    kl = np.empty(T)
    for t0 in range(0, T, row_block):
        t1 = min(T, t0 + row_block)
        _, a, l = _row_block_stats(h64[t0:t1], W64, tau)
        lse[t0:t1] = l
        kl[t0:t1] = _kl_from(a, l, p[t0:t1], idx[t0:t1])
    n = T if T_norm is None else T_norm
    return loss_weight(tau, tau_sq) * (kl.sum() / n), lse, kl


def forward_rows(h, W, vals, idx, tau: float, rows, cache: str = "logits"):
    """lse and KL_t (unscaled) for a subset of rows (exact per row)."""
    rows = np.asarray(rows)
    h64 = _as_f64(np.asarray(h)[rows])
    p, _, _ = teacher_distribution(np.asarray(vals)[rows], tau, cache)
    _, a, l = _row_block_stats(h64, _as_f64(W), tau)
    return l, _kl_from(a, l, p, np.asarray(idx)[rows])


# ---------------------------------------------------------------------------
# a5-a8: backward  (recompute, dz = (S softmax - p)/(T tau) * g, dH, dW)
# ---------------------------------------------------------------------------

def _dz_block(a, lse, p, S, idx, scale):
    q = np.exp(a - lse[:, None])
    dz = S[:, None] * q
    r = np.arange(a.shape[0])[:, None]
    np.subtract.at(dz, (np.broadcast_to(r, idx.shape), idx.astype(np.int64)), p)
    return dz * scale


def backward(h, W, vals, idx, tau: float = 1.0, g: float = 1.0, row_block: int = 256,
             cache: str = "logits", tau_sq: bool = False, T_norm: int | None = None):
    """Full backward: returns (dH [T,d], dW [V,d]) in fp64.  ``T_norm`` as in
    ``forward``: the gradients of this shard's part of a batch's mean."""
    h64, W64 = _as_f64(h), _as_f64(W)
    idx = np.asarray(idx)
    T = h64.shape[0]
    p, S, _ = teacher_distribution(vals, tau, cache)
    n = T if T_norm is None else T_norm
    scale = loss_weight(tau, tau_sq) * g / (n * tau)
    dH = np.empty_like(h64)
    dW = np.zeros_like(W64)
    for t0 in range(0, T, row_block):
        t1 = min(T, t0 + row_block)
        _, a, l = _row_block_stats(h64[t0:t1], W64, tau)
        dz = _dz_block(a, l, p[t0:t1], S[t0:t1], idx[t0:t1], scale)
        dH[t0:t1] = dz @ W64
        dW += dz.T @ h64[t0:t1]
    return dH, dW


def backward_dH_rows(h, W, vals, idx, tau: float, rows, T_total: int, g: float = 1.0,
                     cache: str = "logits", tau_sq: bool = False):
    """dH for a subset of rows; each row needs only its own LSE."""
    rows = np.asarray(rows)
    h64 = _as_f64(np.asarray(h)[rows])
    W64 = _as_f64(W)
    p, S, _ = teacher_distribution(np.asarray(vals)[rows], tau, cache)
    _, a, l = _row_block_stats(h64, W64, tau)
    dz = _dz_block(a, l, p, S, np.asarray(idx)[rows],
                   loss_weight(tau, tau_sq) * g / (T_total * tau))
    return dz @ W64


def backward_dW_rows(h, W, vals, idx, tau: float, vrows, g: float = 1.0,
                     lse=None, row_block: int = 256, cache: str = "logits",
                     tau_sq: bool = False):
    """dW[v,:] for a subset of vocabulary rows v.

    Needs LSE_t of every position (one full fp64 projection) unless the
    oracle's own ``lse`` is passed in.
    """
    vrows = np.asarray(vrows)
    h64 = _as_f64(h)
    W64 = _as_f64(W)
    idx = np.asarray(idx)
    T = h64.shape[0]
    if lse is None:
        lse = np.empty(T)
        for t0 in range(0, T, row_block):
            t1 = min(T, t0 + row_block)
            lse[t0:t1] = _row_block_stats(h64[t0:t1], W64, tau)[2]
    p, S, _ = teacher_distribution(vals, tau, cache)
    a_sel = (h64 @ W64[vrows].T) / tau                       # [T, |vrows|]
    dz = S[:, None] * np.exp(a_sel - lse[:, None])           # softmax part
    for j, v in enumerate(vrows):
        hit = idx == v                                        # [T, K]
        dz[:, j] -= (p * hit).sum(axis=1)                     # scatter part
    dz *= loss_weight(tau, tau_sq) * g / (T * tau)
    return dz.T @ h64                                         # [|vrows|, d]


# ---------------------------------------------------------------------------
# Dense brute force: the [T, V] grid the fused method avoids
# ---------------------------------------------------------------------------

def dense_bruteforce_loss(h, W, vals, idx, tau: float = 1.0, cache: str = "logits",
                          tau_sq: bool = False):
    """Materialise full student log-probs and a dense scattered teacher
    distribution over [T, V] and sum p (log p - log q) over its support.
    Only for tiny shapes ([DD] "The two changes" describes this grid as what a
    naive KL builds).  Uses scipy's softmax routines rather than this module's
    own arithmetic so that it checks the per-row path independently.
    """
    from scipy.special import log_softmax, softmax

    h64, W64 = _as_f64(h), _as_f64(W)
    idx = np.asarray(idx).astype(np.int64)
    T, V = h64.shape[0], W64.shape[0]
    logq = log_softmax((h64 @ W64.T) / tau, axis=1)          # [T, V]
    if cache == "logprobs":
        pt = np.exp(_as_f64(vals))                            # teacher's own probabilities
    else:
        pt = softmax(_as_f64(vals) / tau, axis=1)             # [T, K]
    P = np.zeros((T, V))
    for t in range(T):
        for k in range(idx.shape[1]):
            P[t, idx[t, k]] += pt[t, k]
    total = 0.0
    for t in range(T):
        sup = P[t] > 0
        total += float((P[t, sup] * (np.log(P[t, sup]) - logq[t, sup])).sum())
    return (tau * tau if tau_sq else 1.0) * total / T
