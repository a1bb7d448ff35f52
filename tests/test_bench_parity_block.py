"""The bench's parity block (the CPU leg's check of the GPU outputs on sampled
rows), run on the CPU with the oracle's own outputs standing in for the GPU's:
exact outputs pass, and planted mistakes are caught."""

import numpy as np
import torch

import bench
import oracle
from chunked_kl_loss_chunk_b200 import inputs


def _fake_gpu(T=48, d=32, V=600, K=8, seed=3):
    h, W, _, _ = inputs.make_loss_inputs(T, d, V, 1, dtype=torch.bfloat16, seed=seed)
    x = inputs.make_teacher_logits(T, V, seed=seed)
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    vo, io = oracle.topk_rows(bits(x), K)
    _, lse, _ = oracle.forward(bits(h), bits(W), vo, io)
    dH, _ = oracle.backward(bits(h), bits(W), vo, io)
    gpu = dict(h=h, W=W, logits=x, vals=torch.tensor(vo), idx=torch.tensor(io),
               lse=torch.tensor(lse, dtype=torch.float32), dH=torch.tensor(dH, dtype=torch.float32))
    return gpu, dict(T=T, d=d, V=V, K=K)


def _parity(gpu, w, rows=12):
    return bench.cpu_baseline(w, rows=rows, gpu=gpu, single_core_rows=2)["parity"]


def test_exact_outputs_pass():
    gpu, w = _fake_gpu()
    p = _parity(gpu, w)
    assert p["pass"] and p["topk_bit_exact"] and p["rows"] == 12
    assert p["lse_max_abs_err"] < 1e-6 and p["dH_rel_maxabs_err"] < 1e-6


def test_planted_mistakes_fail():
    gpu, w = _fake_gpu()
    T = w["T"]
    sel = np.unique(np.linspace(0, T - 1, 12).round().astype(np.int64))
    # two top-K entries of a sampled row swapped
    bad = dict(gpu, idx=gpu["idx"].clone())
    bad["idx"][sel[3], [0, 1]] = bad["idx"][sel[3], [1, 0]]
    p = _parity(bad, w)
    assert not p["topk_bit_exact"] and not p["pass"]
    # one lse off by 2e-3
    bad = dict(gpu, lse=gpu["lse"].clone())
    bad["lse"][sel[5]] += 2e-3
    p = _parity(bad, w)
    assert p["topk_bit_exact"] and p["lse_max_abs_err"] > 1e-3 and not p["pass"]
    # one dH row scaled by 1.05
    bad = dict(gpu, dH=gpu["dH"].clone())
    bad["dH"][sel[-1]] *= 1.05
    p = _parity(bad, w)
    assert p["dH_rel_maxabs_err"] > 2e-2 and not p["pass"]


def test_clock_samples_parse_power_and_reasons():
    """The bench's nvidia-smi sampler: median SM clock and board power, the
    highest max clock, every throttle reason seen active; unparsable power
    fields are skipped, malformed lines ignored, no samples give None."""
    import bench
    lines = ["0, 1350, 1965, 998.50, 0x4, Not Active, Not Active, Not Active, Active",
             "0, 1365, 1965, 1001.20, 0x4, Not Active, Not Active, Not Active, Active",
             "0, 1290, 1965, [N/A], 0x4, Active, Not Active, Not Active, Not Active",
             "no, data"]
    r = bench.parse_clock_samples(lines)
    assert r["sm_mhz"] == 1350.0 and r["sm_max_mhz"] == 1965.0 and r["samples"] == 3
    assert r["power_w"] == (998.50 + 1001.20) / 2
    assert r["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert bench.parse_clock_samples(["garbage"]) is None
