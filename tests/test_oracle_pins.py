"""Pins for the fp64 oracle: each check compares it with something other than
itself -- hand-derived fixtures, closed forms, library routines on special
cases, brute force and finite differences -- chosen so that a dropped term, a
wrong sign or index, or a transposed operand fails at least one of them."""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from chunked_kl_loss_chunk_b200 import inputs


def _tiny(T=9, d=6, V=23, K=5, seed=0, tau=1.0):
    rng = np.random.default_rng(seed)
    h = rng.standard_normal((T, d))
    W = rng.standard_normal((V, d)) / math.sqrt(d)
    vals = rng.standard_normal((T, K)) * math.sqrt(2.0)
    idx = np.stack([rng.choice(V, K, replace=False) for _ in range(T)]).astype(np.int32)
    return h, W, vals, idx


# ---------------------------------------------------------------- widening

def test_bf16_widening_known_patterns():
    bits = np.array([0x3F80, 0xC000, 0x7F80, 0xFF80, 0x0001, 0x8000, 0x3EAB], np.uint16)
    got = oracle.bf16_bits_to_f64(bits)
    assert got[0] == 1.0 and got[1] == -2.0
    assert got[2] == math.inf and got[3] == -math.inf
    assert got[4] == 2.0 ** -133                       # smallest bf16 subnormal
    assert got[5] == 0.0 and math.copysign(1.0, got[5]) == -1.0
    assert got[6] == (0x2B | 0x80) / 128.0 * 2.0 ** (0x7D - 127)


# ---------------------------------------------------------------- top-K

def _parse(v):
    return {"-inf": -math.inf, "inf": math.inf, "nan": math.nan, "-0": -0.0}.get(v, v) \
        if isinstance(v, str) else float(v)


def test_topk_golden_rows(golden_dir):
    cases = json.load(open(os.path.join(golden_dir, "topk_rows.json")))["cases"]
    for c in cases:
        row = np.array([[_parse(v) for v in c["row"]]], np.float64)
        vals, idx = oracle.topk_rows(row, c["K"])
        assert idx[0].tolist() == c["idx"], c["name"]
        exp_vals = row[0, c["idx"]].astype(np.float32)
        # exact copies, sign of zero and NaN-ness preserved
        assert np.array_equal(vals[0].view(np.uint32), exp_vals.view(np.uint32)), c["name"]


def test_topk_bruteforce_python_sort():
    rng = np.random.default_rng(3)
    for trial in range(40):
        V = int(rng.integers(1, 40))
        K = int(rng.integers(1, V + 1))
        # small integers force heavy ties; sprinkle specials
        row = rng.integers(-3, 4, V).astype(np.float64)
        for j in range(V):
            u = rng.random()
            if u < 0.05:
                row[j] = math.nan
            elif u < 0.1:
                row[j] = -math.inf
            elif u < 0.15:
                row[j] = -0.0
            elif u < 0.18:
                row[j] = math.inf
        exp = sorted(range(V), key=lambda i: (math.isnan(row[i]),
                                              0.0 if math.isnan(row[i]) else -row[i], i))[:K]
        _, idx = oracle.topk_rows(row[None], K)
        assert idx[0].tolist() == exp


def test_topk_bf16_bits_match_float_path():
    x = inputs.make_teacher_logits(4, 300, seed=5)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    v1, i1 = oracle.topk_rows(bits, 17)
    v2, i2 = oracle.topk_rows(x.float().numpy(), 17)
    assert np.array_equal(i1, i2) and np.array_equal(v1, v2)


# ---------------------------------------------------------------- teacher p

def test_teacher_distribution_golden():
    vals = np.array([[0.0, math.log(2.0), math.log(3.0)]])
    p, S, plogp = oracle.teacher_distribution(vals, 1.0)
    assert np.allclose(p, [[1 / 6, 1 / 3, 1 / 2]], rtol=0, atol=1e-15)
    assert abs(S[0] - 1.0) < 1e-15
    exp = (1 / 6) * math.log(1 / 6) + (1 / 3) * math.log(1 / 3) + 0.5 * math.log(0.5)
    assert abs(plogp[0] - exp) < 1e-14
    # temperature divides the teacher logits
    p2, _, _ = oracle.teacher_distribution(2.0 * vals, 2.0)
    assert np.allclose(p2, p, atol=1e-15)


# ---------------------------------------------------------------- loss

def test_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "worked_example.json")))
    i, e = g["inputs"], g["expected"]
    h, W = np.array(i["h"]), np.array(i["W"])
    vals, idx = np.array(i["vals"]), np.array(i["idx"], np.int32)
    loss, lse, kl = oracle.forward(h, W, vals, idx, i["tau"])
    assert abs(loss - e["loss"]) < 1e-15
    assert np.allclose(lse, e["lse"], atol=1e-15)
    dH, dW = oracle.backward(h, W, vals, idx, i["tau"])
    assert np.allclose(dH, e["dH"], atol=1e-15)
    assert np.allclose(dW, e["dW"], atol=1e-15)


def test_uniform_student_closed_form():
    """W = 0 -> q uniform -> KL_t = sum p log p + S log V."""
    h, W, vals, idx = _tiny()
    W = np.zeros_like(W)
    for tau in (1.0, 0.7):
        loss, lse, kl = oracle.forward(h, W, vals, idx, tau)
        p, S, plogp = oracle.teacher_distribution(vals, tau)
        V = W.shape[0]
        assert np.allclose(kl, plogp + S * math.log(V), atol=1e-13)
        assert np.allclose(lse, math.log(V), atol=1e-13)


def test_k1_is_cross_entropy():
    h, W, vals, idx = _tiny(K=1)
    for tau in (1.0, 2.5):
        loss, _, _ = oracle.forward(h, W, vals, idx, tau)
        logits = torch.tensor(h @ W.T / tau, dtype=torch.float64)
        ce = torch.nn.functional.cross_entropy(logits, torch.tensor(idx[:, 0], dtype=torch.long))
        assert abs(loss - ce.item()) < 1e-12


def test_k_equals_v_is_full_kl():
    T, d, V = 7, 5, 11
    h, W, vals, idx = _tiny(T=T, d=d, V=V, K=V)
    for tau in (1.0, 1.7):
        loss, _, _ = oracle.forward(h, W, vals, idx, tau)
        # dense teacher logits in vocabulary order
        tl = np.zeros((T, V))
        for t in range(T):
            tl[t, idx[t]] = vals[t]
        logq = torch.log_softmax(torch.tensor(h @ W.T / tau), dim=1)
        pt = torch.softmax(torch.tensor(tl / tau), dim=1)
        ref = torch.nn.functional.kl_div(logq, pt, reduction="sum").item() / T
        assert abs(loss - ref) < 1e-12


def test_zero_loss_when_student_reproduces_teacher():
    """d = V, W = I, h = teacher logits at idx and -60 elsewhere -> KL ~ 0."""
    T, V, K = 6, 32, 5
    _, _, vals, idx = _tiny(T=T, d=V, V=V, K=K)
    W = np.eye(V)
    h = np.full((T, V), -60.0)
    for t in range(T):
        h[t, idx[t]] = vals[t]
    loss, _, kl = oracle.forward(h, W, vals, idx, 1.0)
    # exact value is log(1 + tail/sum) ~ 1e-24; fp64 rounding leaves ~1e-17
    assert abs(loss) < 1e-14
    assert np.all(np.abs(kl) < 1e-14)


def test_gibbs_nonnegative_and_dense_bruteforce():
    h, W, vals, idx = _tiny(T=13, d=7, V=29, K=6)
    for tau in (1.0, 0.5):
        dense = oracle.dense_bruteforce_loss(h, W, vals, idx, tau)
        for rb in (1, 7, 64, 13):
            loss, _, kl = oracle.forward(h, W, vals, idx, tau, row_block=rb)
            assert abs(loss - dense) < 1e-12
            assert np.all(kl >= -1e-14)


def test_temperature_identity():
    """L(h, W, vals, tau) = L(h, W/tau, vals/tau, 1)."""
    h, W, vals, idx = _tiny()
    tau = 1.9
    a, _, _ = oracle.forward(h, W, vals, idx, tau)
    b, _, _ = oracle.forward(h, W / tau, vals / tau, idx, 1.0)
    assert abs(a - b) < 1e-13


def test_forward_rows_matches_forward():
    h, W, vals, idx = _tiny(T=17)
    _, lse, kl = oracle.forward(h, W, vals, idx, 1.3)
    rows = np.array([0, 5, 16, 3])
    l2, k2 = oracle.forward_rows(h, W, vals, idx, 1.3, rows)
    assert np.allclose(l2, lse[rows], atol=1e-14) and np.allclose(k2, kl[rows], atol=1e-14)


# ---------------------------------------------------------------- gradients

def _fd_check(tau, g):
    h, W, vals, idx = _tiny(T=5, d=4, V=13, K=4, seed=11)
    dH, dW = oracle.backward(h, W, vals, idx, tau, g)
    rng = np.random.default_rng(1)
    eps = 1e-6
    for _ in range(25):
        t, j = rng.integers(5), rng.integers(4)
        hp, hm = h.copy(), h.copy()
        hp[t, j] += eps
        hm[t, j] -= eps
        fd = g * (oracle.forward(hp, W, vals, idx, tau)[0] - oracle.forward(hm, W, vals, idx, tau)[0]) / (2 * eps)
        assert abs(fd - dH[t, j]) <= 1e-6 * max(1.0, abs(dH[t, j])) + 1e-9
        v, j = rng.integers(13), rng.integers(4)
        Wp, Wm = W.copy(), W.copy()
        Wp[v, j] += eps
        Wm[v, j] -= eps
        fd = g * (oracle.forward(h, Wp, vals, idx, tau)[0] - oracle.forward(h, Wm, vals, idx, tau)[0]) / (2 * eps)
        assert abs(fd - dW[v, j]) <= 1e-6 * max(1.0, abs(dW[v, j])) + 1e-9


def test_gradients_finite_differences():
    _fd_check(1.0, 1.0)
    _fd_check(0.6, 2.5)


def test_gradient_invariants():
    h, W, vals, idx = _tiny(T=8, d=5, V=19, K=4)
    W[:, 2] = 0.37                                  # constant column of W
    dH, dW = oracle.backward(h, W, vals, idx, 1.0)
    assert np.allclose(dW.sum(axis=0), 0.0, atol=1e-15)   # sum_v dz = 0 when S = 1
    assert np.allclose(dH[:, 2], 0.0, atol=1e-15)


def test_sampled_gradients_match_full():
    h, W, vals, idx = _tiny(T=11, d=5, V=17, K=4)
    dH, dW = oracle.backward(h, W, vals, idx, 0.8, 1.5)
    rows = np.array([2, 10, 0])
    assert np.allclose(oracle.backward_dH_rows(h, W, vals, idx, 0.8, rows, 11, 1.5), dH[rows], atol=1e-15)
    vr = np.array([0, 16, 4, int(idx[3, 1])])
    assert np.allclose(oracle.backward_dW_rows(h, W, vals, idx, 0.8, vr, 1.5), dW[vr], atol=1e-15)


def test_backward_chunk_invariance():
    h, W, vals, idx = _tiny(T=13)
    ref = oracle.backward(h, W, vals, idx, 1.0, row_block=13)
    for rb in (1, 4, 7):
        dH, dW = oracle.backward(h, W, vals, idx, 1.0, row_block=rb)
        assert np.allclose(dH, ref[0], atol=1e-15) and np.allclose(dW, ref[1], atol=1e-14)


# ---------------------------------------------------------------- variants:
# a cache of full-vocabulary teacher log-probabilities (S = sum p < 1), and the
# tau^2 factor on loss and gradients

def _logprob_cache(T, K, seed=5, mass=(0.3, 0.95)):
    """Unnormalised teacher log-probs: K entries of a distribution whose other
    entries (the tail the cache dropped) hold 1 - S of the mass."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, K)) * math.sqrt(2.0)
    S = rng.uniform(*mass, size=T)
    lp = torch.log_softmax(torch.tensor(x), dim=1).numpy() + np.log(S)[:, None]
    return lp, S


def test_logprob_cache_hand_example():
    """V = 2, d = 1, W = [ln 3, 0], h = 1: z = (ln 3, 0), q = (3/4, 1/4),
    LSE = ln 4.  One cached entry, token 0 with p = 1/2 (S = 1/2):
    KL = (1/2)(ln 1/2 - ln 3/4) = (1/2) ln 2/3;  dz = S q - p~ = (-1/8, 1/8);
    dH = dz W = -(ln 3)/8;  dW = dz^T h = (-1/8, 1/8).
    With tau = 2 and the tau^2 factor: q0 = sqrt3/(1 + sqrt3) = (3 - sqrt3)/2,
    loss = 4 (1/2)(ln 1/2 - ln q0), dz = 4/(1*2) (S q - p~) = (q0 - 1, 1 - q0)."""
    h = np.array([[1.0]])
    W = np.array([[math.log(3.0)], [0.0]])
    vals = np.array([[math.log(0.5)]])
    idx = np.array([[0]], np.int32)
    loss, lse, kl = oracle.forward(h, W, vals, idx, 1.0, cache="logprobs")
    assert abs(loss - 0.5 * math.log(2.0 / 3.0)) < 1e-15
    assert abs(lse[0] - math.log(4.0)) < 1e-15
    dH, dW = oracle.backward(h, W, vals, idx, 1.0, cache="logprobs")
    assert abs(dH[0, 0] + math.log(3.0) / 8) < 1e-15
    assert np.allclose(dW[:, 0], [-0.125, 0.125], atol=1e-16)

    q0 = (3.0 - math.sqrt(3.0)) / 2.0
    loss2, lse2, kl2 = oracle.forward(h, W, vals, idx, 2.0, cache="logprobs", tau_sq=True)
    assert abs(loss2 - 4 * 0.5 * (math.log(0.5) - math.log(q0))) < 1e-14
    assert abs(kl2[0] - 0.5 * (math.log(0.5) - math.log(q0))) < 1e-15     # kl unscaled
    assert abs(lse2[0] - math.log(math.sqrt(3.0) + 1.0)) < 1e-15
    dH2, dW2 = oracle.backward(h, W, vals, idx, 2.0, cache="logprobs", tau_sq=True)
    assert np.allclose(dW2[:, 0], [q0 - 1.0, 1.0 - q0], atol=1e-15)
    assert abs(dH2[0, 0] - (q0 - 1.0) * math.log(3.0)) < 1e-15


def test_logprob_uniform_student_closed_form():
    """W = 0 -> q = 1/V -> KL_t = sum_k p log p + S ln V with p = exp(vals)."""
    T, d, V, K = 9, 6, 23, 5
    h, W, _, idx = _tiny(T=T, d=d, V=V, K=K)
    lp, S = _logprob_cache(T, K)
    for tau in (1.0, 0.7):
        loss, lse, kl = oracle.forward(h, np.zeros_like(W), lp, idx, tau, cache="logprobs")
        p = np.exp(lp)
        assert np.allclose(p.sum(axis=1), S, atol=1e-14)
        p2, S2, plogp2 = oracle.teacher_distribution(lp, tau, cache="logprobs")
        assert np.allclose(S2, S, atol=1e-14) and np.allclose(plogp2, (p * lp).sum(axis=1), atol=1e-14)
        assert np.allclose(kl, (p * lp).sum(axis=1) + S * math.log(V), atol=1e-13)
        assert np.all(kl < (p * lp).sum(axis=1) + math.log(V))  # S < 1 lowers the loss


def test_logprob_full_vocab_is_full_kl():
    """K = V, vals = the teacher's log-softmax -> the full KL of torch's kl_div."""
    T, d, V = 7, 5, 11
    h, W, tl, idx = _tiny(T=T, d=d, V=V, K=V)
    lp = torch.log_softmax(torch.tensor(tl), dim=1).numpy()
    for tau in (1.0, 1.7):
        loss, _, _ = oracle.forward(h, W, lp, idx, tau, cache="logprobs")
        logq = torch.log_softmax(torch.tensor(h @ W.T / tau), dim=1)
        # teacher log-probs in vocabulary order
        lpv = np.zeros((T, V))
        for t in range(T):
            lpv[t, idx[t]] = lp[t]
        ref = torch.nn.functional.kl_div(logq, torch.tensor(lpv), reduction="sum",
                                         log_target=True).item() / T
        assert abs(loss - ref) < 1e-12


def test_logprob_cache_of_renormalised_teacher_equals_logits_cache():
    """vals' = log softmax_K(vals / tau) read as log-probs gives the logits
    cache's loss and gradients at the same tau."""
    h, W, vals, idx = _tiny(T=8, d=5, V=19, K=4)
    for tau in (1.0, 0.8):
        lp = torch.log_softmax(torch.tensor(vals / tau), dim=1).numpy()
        a = oracle.forward(h, W, vals, idx, tau)
        b = oracle.forward(h, W, lp, idx, tau, cache="logprobs")
        assert abs(a[0] - b[0]) < 1e-14 and np.allclose(a[2], b[2], atol=1e-14)
        ga = oracle.backward(h, W, vals, idx, tau, 1.3)
        gb = oracle.backward(h, W, lp, idx, tau, 1.3, cache="logprobs")
        assert np.allclose(ga[0], gb[0], atol=1e-15) and np.allclose(ga[1], gb[1], atol=1e-15)


def test_logprob_dense_bruteforce():
    T, d, V, K = 13, 7, 29, 6
    h, W, _, idx = _tiny(T=T, d=d, V=V, K=K)
    lp, _ = _logprob_cache(T, K, seed=2)
    for tau, sq in ((1.0, False), (0.5, True), (2.0, True)):
        dense = oracle.dense_bruteforce_loss(h, W, lp, idx, tau, cache="logprobs", tau_sq=sq)
        loss, _, kl = oracle.forward(h, W, lp, idx, tau, cache="logprobs", tau_sq=sq)
        assert abs(loss - dense) < 1e-12


def _fd_check_variant(tau, g, cache, tau_sq):
    T, d, V, K = 5, 4, 13, 4
    h, W, vals, idx = _tiny(T=T, d=d, V=V, K=K, seed=11)
    if cache == "logprobs":
        vals, _ = _logprob_cache(T, K, seed=4)
    kw = dict(cache=cache, tau_sq=tau_sq)
    dH, dW = oracle.backward(h, W, vals, idx, tau, g, **kw)
    rng = np.random.default_rng(7)
    eps = 1e-6
    f = lambda hh, WW: oracle.forward(hh, WW, vals, idx, tau, **kw)[0]
    for _ in range(20):
        t, j = rng.integers(T), rng.integers(d)
        hp, hm = h.copy(), h.copy()
        hp[t, j] += eps
        hm[t, j] -= eps
        fd = g * (f(hp, W) - f(hm, W)) / (2 * eps)
        assert abs(fd - dH[t, j]) <= 1e-6 * max(1.0, abs(dH[t, j])) + 1e-9
        v, j = rng.integers(V), rng.integers(d)
        Wp, Wm = W.copy(), W.copy()
        Wp[v, j] += eps
        Wm[v, j] -= eps
        fd = g * (f(h, Wp) - f(h, Wm)) / (2 * eps)
        assert abs(fd - dW[v, j]) <= 1e-6 * max(1.0, abs(dW[v, j])) + 1e-9


def test_variant_gradients_finite_differences():
    _fd_check_variant(1.0, 1.0, "logprobs", False)
    _fd_check_variant(0.6, 2.5, "logprobs", True)
    _fd_check_variant(1.7, 0.5, "logits", True)


def test_tau_sq_high_temperature_limit_is_logit_matching():
    """With a dense teacher (K = V) and the tau^2 factor, as tau grows the loss
    tends to (1/(2 V T)) sum_t |w_t - u_t|^2 and dz to g (w - u)/(T V), where u, w
    are the teacher's and the student's logits with their row means removed
    (the high-temperature limit of distillation).  Both errors shrink as 1/tau."""
    T, d, V = 6, 5, 11
    h, W, x, idx = _tiny(T=T, d=d, V=V, K=V, seed=9)
    z = h @ W.T
    xv = np.zeros((T, V))
    for t in range(T):
        xv[t, idx[t]] = x[t]
    u = xv - xv.mean(axis=1, keepdims=True)
    w = z - z.mean(axis=1, keepdims=True)
    lim_loss = ((w - u) ** 2).sum() / (2 * V * T)
    lim_dW = ((w - u) / (T * V)).T @ h
    errs = []
    for tau in (1e2, 1e3):
        loss, _, _ = oracle.forward(h, W, x, idx, tau, tau_sq=True)
        _, dW = oracle.backward(h, W, x, idx, tau, tau_sq=True)
        errs.append((abs(loss - lim_loss) / lim_loss,
                     np.abs(dW - lim_dW).max() / np.abs(lim_dW).max()))
    assert errs[1][0] < 2e-3 and errs[1][1] < 2e-3
    assert errs[1][0] < 0.2 * errs[0][0] and errs[1][1] < 0.2 * errs[0][1]
    # without the factor the loss vanishes as 1/tau^2
    plain, _, _ = oracle.forward(h, W, x, idx, 1e3)
    assert abs(plain * 1e6 - lim_loss) / lim_loss < 2e-3


def test_unknown_cache_kind_rejected():
    with pytest.raises(ValueError):
        oracle.teacher_distribution(np.zeros((1, 2)), 1.0, cache="probs")


# ---------------------------------------------------------------- inputs

def test_logprob_cache_generator_row_mass():
    """make_logprob_cache: K log-probabilities per row whose probabilities sum to
    the drawn row mass S in [0.3, 0.95], the same for every call with a seed."""
    vals, S = inputs.make_logprob_cache(64, 20, seed=4)
    assert vals.shape == (64, 20) and vals.dtype == torch.float32 and S.shape == (64,)
    assert float(S.min()) >= 0.3 and float(S.max()) <= 0.95
    assert torch.allclose(torch.exp(vals.double()).sum(dim=1), S.double(), rtol=1e-5)
    assert bool((vals < 0).all())                      # every entry below probability 1
    v2, S2 = inputs.make_logprob_cache(64, 20, seed=4)
    assert torch.equal(v2, vals) and torch.equal(S2, S)


def test_input_generator_shapes_and_distinct_indices():
    h, W, vals, idx = inputs.make_loss_inputs(64, 32, 500, 16, dtype=torch.float32, seed=0)
    assert h.shape == (64, 32) and W.shape == (500, 32) and vals.shape == (64, 16)
    assert idx.dtype == torch.int32 and int(idx.min()) >= 0 and int(idx.max()) < 500
    s, _ = torch.sort(idx.long(), dim=1)
    assert bool((s[:, 1:] != s[:, :-1]).all())
    h2, W2, vals2, idx2 = inputs.make_loss_inputs(64, 32, 500, 16, dtype=torch.float32, seed=0)
    assert torch.equal(h, h2) and torch.equal(idx, idx2)
    # K = V is a permutation
    p = inputs.distinct_uniform_indices(3, 9, 9, seed=1)
    assert sorted(p[0].tolist()) == list(range(9))
