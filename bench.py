#!/usr/bin/env python
"""Benchmark of the fused chunked top-K KL distillation loss on B200.

One step = the whole hot path over one batch of synthetic input:
  top-K cache build of the batch's teacher logits [T, V] (bf16)
  -> fused chunked KL forward (loss, lse) -> fused chunked KL backward (dH, dW),
with the cache the build produced feeding the loss.

Default workload: the toy output head at 32K tokens (T=32768, d=4096,
V=131072, K=100, chunk=2048, bf16 operands, fp32 accumulation).

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--dp]

Prints ONE JSON line (rank 0).  The K timed steps are captured in one CUDA
graph and timed as one replay, with CUDA events per step (the top-K build,
forward and backward times) and around the GEMMs of the last step.  Multi-GPU
runs are independent replicas by default (weak scaling, no collective on the
data path); with --dp each rank's batch is one shard of a batch N times as
large, and dW and the loss are summed over the ranks.  Time is the max over
ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "tokens/s & TFLOP/s (8TdV) fused top-K KL fwd+bwd; % BF16 tensor peak; peak mem"
UNIT = "tokens/s"

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of launches shaped exactly like the bench's (a head-8k-c2048 step:
# 2048-row chunks at d=4096, V=131072), valid only for the GEMM sources with
# this digest; the roofline's "traffic" is null for any other source.
NCU_TRAFFIC = {
    "source_sha256_16": "0ec119d57cec7fff",
    # dram__bytes_read.sum + dram__bytes_write.sum per launch of each GEMM kind,
    # from captures of one or two launches of a head-8k-c2048 step (2048-row
    # chunks at d=4096, V=131072: the launch shapes of the 32K head); fwd_lse is
    # the mean of two launches; dW is the mix of a 32K step, one storing launch
    # (4.075 GB) and seven adding ones (5.833 GB)
    "per_launch_bytes": {"fwd_lse": 1.112e9, "bwd_dz": 1.630e9, "dH": 2.617e9, "dW": 5.613e9},
}


def _gemm_source_digest():
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "chunked_kl_loss_chunk_b200", "csrc")
    for f in ("kd_common.cuh", "kd_gemm.cuh", "kd_gemm2.cuh", "kd_unitwalk.h", "kd_internal.h",
              "kd_loss.cu"):
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kd", choices=["kd", "reference"])
    ap.add_argument("--workload", default="head-32k")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time K eager steps instead of K replays of a captured step")
    ap.add_argument("--cpu-rows", type=int, default=0, help="oracle rows per CPU step (0 = auto)")
    ap.add_argument("--dp", action="store_true",
                    help="data-parallel shards: each rank's T rows are one shard of a batch of "
                         "T x N positions; dW and the loss are summed over the ranks (NCCL)")
    ap.add_argument("--no-topk-alone", action="store_true",
                    help="skip timing the top-K build on its own after the timed steps")
    ap.add_argument("--sweep-memory", action="store_true",
                    help="print the peak-memory vs T sweep instead of the bench line")
    return ap.parse_args()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _workload(name):
    from chunked_kl_loss_chunk_b200 import inputs
    return dict(inputs.WORKLOADS[name])


def _config(w, name, extra=None):
    c = {"workload": name, "T": w["T"], "d": w["d"], "V": w["V"], "K": w["K"],
         "chunk": w["chunk"], "temperature": 1.0,
         "step": "top-K cache build of teacher logits [T,V] + fused fwd + fused bwd (dH, dW)",
         "l2": "inputs larger than L2 (W and teacher logits exceed 126 MB); no flush"}
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------ CPU oracle

def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _cpu_sample_step(W64, h_rows, logits_rows, K, tau=1.0):
    """One bounded sample of the step on the host cores with the fp64 oracle."""
    import oracle
    vals, idx = oracle.topk_rows(logits_rows, K)
    _, lse, _ = oracle.forward(h_rows, W64, vals, idx, tau)
    oracle.backward(h_rows, W64, vals, idx, tau)


def _cpu_setup(w, rows, seed=0):
    import numpy as np
    import torch
    import oracle
    from chunked_kl_loss_chunk_b200 import inputs
    # The same distributions as the GPU arm, drawn on the host.
    g = torch.Generator().manual_seed(seed * 1000 + 1)
    W = (torch.randn((w["V"], w["d"]), generator=g) / math.sqrt(w["d"])).to(torch.bfloat16)
    Wn = W.view(torch.int16).numpy().view(np.uint16)
    W64 = oracle.bf16_bits_to_f64(Wn)
    h, _, _, _ = inputs.make_loss_inputs(rows, w["d"], 8, 1, dtype=torch.bfloat16, seed=seed)
    hn = h.view(torch.int16).numpy().view(np.uint16)
    x = inputs.make_teacher_logits(rows, w["V"], seed=seed)
    xn = x.view(torch.int16).numpy().view(np.uint16)
    return W64, hn, xn


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def _cpu_from_gpu(gpu, rows):
    """Host copies of `rows` evenly spaced positions of the bench's own batch
    (exact bf16 bit patterns) and of the full output head, widened to fp64."""
    import numpy as np
    import torch
    import oracle
    T = gpu["h"].shape[0]
    sel = np.unique(np.linspace(0, T - 1, min(rows, T)).round().astype(np.int64))
    st = torch.as_tensor(sel, device=gpu["h"].device)

    def bits(t):
        t = t.detach().cpu().contiguous()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()
    W64 = oracle.bf16_bits_to_f64(bits(gpu["W"])) if gpu["W"].dtype == torch.bfloat16 \
        else gpu["W"].double().cpu().numpy()
    return W64, bits(gpu["h"][st]), bits(gpu["logits"][st]), sel


def _gpu_parity(gpu, W64, hn, xn, sel, K):
    """The GPU's outputs on the sampled positions against the oracle: top-K
    (bit-exact), lse (absolute error) and dH rows (max-abs error over the
    oracle's max-abs), with the bars the tests use."""
    import numpy as np
    import oracle
    T = gpu["h"].shape[0]
    vals_g = gpu["vals"][sel].cpu().numpy()
    idx_g = gpu["idx"][sel].cpu().numpy()
    vals_o, idx_o = oracle.topk_rows(xn, K)
    topk_exact = bool(np.array_equal(idx_g, idx_o) and
                      np.array_equal(vals_g.view(np.uint32), vals_o.view(np.uint32)))
    rows = np.arange(len(sel))
    lse_o, _ = oracle.forward_rows(hn, W64, vals_o, idx_o, 1.0, rows)
    lse_err = float(np.abs(gpu["lse"][sel].cpu().numpy().astype(np.float64) - lse_o).max())
    dH_o = oracle.backward_dH_rows(hn, W64, vals_o, idx_o, 1.0, rows, T)
    dH_g = gpu["dH"][sel].float().cpu().numpy().astype(np.float64)
    dH_err = float(np.abs(dH_g - dH_o).max() / max(np.abs(dH_o).max(), 1e-300))
    return {"rows": int(len(sel)), "topk_bit_exact": topk_exact, "lse_max_abs_err": lse_err,
            "dH_rel_maxabs_err": dH_err,
            "bars": {"topk": "bit-exact", "lse_max_abs_err": 1e-3, "dH_rel_maxabs_err": 2e-2},
            "pass": bool(topk_exact and lse_err <= 1e-3 and dH_err <= 2e-2)}


def cpu_baseline(w, rows=0, steps=1, single_core_rows=32, gpu=None):
    """Oracle tokens/s on a bounded sample (rows positions per step), on all
    host cores and, on a smaller sample, on one core.  Given the bench's device
    tensors (`gpu`), the sample is rows of the bench's own batch and the GPU's
    outputs on those rows are checked against the oracle's."""
    if rows <= 0:
        rows = 16
    sel = None
    if gpu is not None:
        W64, hn, xn, sel = _cpu_from_gpu(gpu, rows)
        rows = len(sel)
    else:
        W64, hn, xn = _cpu_setup(w, rows)
    t0 = time.perf_counter()
    for _ in range(steps):
        _cpu_sample_step(W64, hn, xn, w["K"])
    dt = time.perf_counter() - t0
    out = {"value": rows * steps / dt, "unit": UNIT, "cores": _cpu_threads(), "kind": "oracle",
           "cpu_model": _cpu_model(), "nproc": os.cpu_count(),
           "sample": f"{rows} positions x {steps} step(s) of the {w['T']}-position batch: "
                     f"fp64 top-K (full stable sort of V={w['V']}), forward and backward "
                     f"(d={w['d']}); {dt:.2f} s"}
    if single_core_rows > 0:
        from threadpoolctl import threadpool_limits
        n1 = min(single_core_rows, rows)
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            _cpu_sample_step(W64, hn[:n1], xn[:n1], w["K"])
            dt1 = time.perf_counter() - t0
        out["single_core"] = {"value": n1 / dt1, "unit": UNIT, "cores": 1,
                              "sample": f"{n1} positions of the same sample; {dt1:.2f} s"}
    if gpu is not None:
        out["sample"] = (f"{rows} evenly spaced positions of the bench's own batch (T={w['T']}): "
                         + out["sample"].split(": ", 1)[1])
        out["parity"] = _gpu_parity(gpu, W64, hn, xn, sel, w["K"])
    return out


def run_reference(args, rank):
    """Reference arm: the fp64 CPU oracle as it stands, rank 0 only."""
    if rank != 0:
        return
    w = _workload(args.workload)
    rows = args.cpu_rows or 8
    W64, hn, xn = _cpu_setup(w, rows)
    for _ in range(args.warmup):
        _cpu_sample_step(W64, hn, xn, w["K"])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _cpu_sample_step(W64, hn, xn, w["K"])
    dt = time.perf_counter() - t0
    v = rows * args.steps / dt
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(w, args.workload, {"sample_rows_per_step": rows}),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": _cpu_threads(), "kind": "oracle",
                             "sample": f"{rows} positions per step (top-K, forward, backward) of "
                                       f"the {w['T']}-position workload"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    def __init__(self, dev_index):
        self.proc = None
        self.path = None
        self.dev = dev_index

    def start(self):
        import torch
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        ident = str(self.dev)
        try:
            u = torch.cuda.get_device_properties(self.dev).uuid
            ident = "GPU-" + str(u) if not str(u).startswith("GPU-") else str(u)
        except Exception:
            pass
        self.ident = ident
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={ident}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        result = parse_clock_samples(open(self.path).read().splitlines())
        os.unlink(self.path)
        if result is not None:
            result["power_limit_w"] = self.power_limit()
        return result

    def power_limit(self):
        """The board's enforced power limit in watts (one nvidia-smi query;
        None if it cannot be read)."""
        try:
            out = subprocess.run(["nvidia-smi", f"--id={self.ident}",
                                  "--query-gpu=enforced.power.limit",
                                  "--format=csv,noheader,nounits"],
                                 capture_output=True, text=True, timeout=10).stdout
            return float(out.strip().splitlines()[0])
        except Exception:
            return None


def parse_clock_samples(lines):
    """nvidia-smi CSV lines (index, clocks.sm, clocks.max.sm, power.draw, the
    active-reasons bitmask, then hw_slowdown, hw_thermal_slowdown,
    sw_thermal_slowdown, sw_power_cap) -> the median SM clock, the highest max
    clock, every reason seen active, the median board power and the number of
    samples; None without a parsable line."""
    sm, mx, pw, reasons = [], [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        f = [x.strip() for x in ln.split(",")]
        if len(f) < 9:
            continue
        try:
            sm.append(float(f[1]))
            mx.append(float(f[2]))
        except ValueError:
            continue
        try:
            pw.append(float(f[3]))
        except ValueError:
            pass
        for n, v in zip(names, f[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
            "power_w": statistics.median(pw) if pw else None, "samples": len(sm)}


# ------------------------------------------------------------------ GPU arm

def job_throughput(ms_local, tokens_per_rank, world, device):
    """Whole-job throughput of independent replicas: the timed region is the
    slowest rank's (max over ranks), the work is every rank's.  Returns
    (ms of the slowest rank, tokens/s over all ranks)."""
    ms = float(ms_local)
    if world > 1:
        import torch
        import torch.distributed as dist
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms, tokens_per_rank * world / (ms / 1000.0)


def run_kd(args, rank, world):
    import torch
    import torch.distributed as dist
    from chunked_kl_loss_chunk_b200 import build as kbuild
    from chunked_kl_loss_chunk_b200 import inputs, kd

    kbuild.build()
    kd.load()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = _workload(args.workload)
    T, d, V, K, chunk = w["T"], w["d"], w["V"], w["K"], w["chunk"]
    dt = torch.bfloat16 if w["dtype"] == "bf16" else torch.float32

    # inputs of this rank's replica (seeded by rank)
    h, W, _, _ = inputs.make_loss_inputs(T, d, V, 1, dtype=dt, seed=rank, device=dev)
    logits = inputs.make_teacher_logits(T, V, seed=rank, device=dev)
    vals = torch.empty((T, K), dtype=torch.float32, device=dev)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    ws_topk = kd.alloc_workspace(kd.kd_topk_workspace_size(T, V, K), dev)
    ws = kd.workspace_for(h, W, K, chunk)
    loss_vec = torch.empty((1,), dtype=torch.float32, device=dev)
    loss = loss_vec[0]
    lse = torch.empty((T,), dtype=torch.float32, device=dev)
    dH = torch.empty_like(h)
    dW = torch.empty((V, d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    code = kd.KD_DTYPE_BF16 if dt == torch.bfloat16 else kd.KD_DTYPE_F32

    def step(ev=None, inp=None):
        """One step; `ev` (4 timing events) marks its start and the ends of the
        top-K build, the forward and the backward on the launching stream."""
        hh, WW, xx = inp if inp is not None else (h, W, logits)
        sp = torch.cuda.current_stream().cuda_stream     # the capture stream while capturing
        nvtx = torch.cuda.nvtx
        if ev is not None:
            ev[0].record()
        nvtx.range_push("kd_topk_build")
        st = kd.kd_topk_build(xx.data_ptr(), kd.KD_DTYPE_BF16, T, V, K, vals.data_ptr(),
                              idx.data_ptr(), ws_topk.data_ptr(), ws_topk.numel(), sp)
        nvtx.range_pop()
        if ev is not None:
            ev[1].record()
        nvtx.range_push("kd_fused_kl_fwd")
        if args.dp:     # this rank's rows are one shard of a batch of T * world positions
            st |= kd.kd_fused_kl_fwd_shard(hh.data_ptr(), WW.data_ptr(), code, T, d, V,
                                           vals.data_ptr(), idx.data_ptr(), K, chunk, 1.0, 0,
                                           T * world, loss.data_ptr(), lse.data_ptr(), None,
                                           ws.data_ptr(), ws.numel(), sp)
        else:
            st |= kd.kd_fused_kl_fwd(hh.data_ptr(), WW.data_ptr(), code, T, d, V, vals.data_ptr(),
                                     idx.data_ptr(), K, chunk, 1.0, loss.data_ptr(), lse.data_ptr(),
                                     None, ws.data_ptr(), ws.numel(), sp)
        nvtx.range_pop()
        if ev is not None:
            ev[2].record()
        nvtx.range_push("kd_fused_kl_bwd")
        if args.dp:
            st |= kd.kd_fused_kl_bwd_shard(hh.data_ptr(), WW.data_ptr(), code, T, d, V,
                                           vals.data_ptr(), idx.data_ptr(), K, chunk, 1.0, 0,
                                           T * world, lse.data_ptr(), None, dH.data_ptr(),
                                           dW.data_ptr(), 0, ws.data_ptr(), ws.numel(), sp)
        else:
            st |= kd.kd_fused_kl_bwd(hh.data_ptr(), WW.data_ptr(), code, T, d, V, vals.data_ptr(),
                                     idx.data_ptr(), K, chunk, 1.0, lse.data_ptr(), None,
                                     dH.data_ptr(), dW.data_ptr(), 0, ws.data_ptr(), ws.numel(), sp)
        nvtx.range_pop()
        if args.dp and world > 1:
            # the batch's dW and loss: one sum over the ranks (NCCL)
            dist.all_reduce(dW, op=dist.ReduceOp.SUM)
            dist.all_reduce(loss_vec, op=dist.ReduceOp.SUM)
        if ev is not None:
            ev[3].record()
        if st != 0:
            raise RuntimeError(f"libkd call failed ({st})")

    def barrier():
        if world > 1:
            dist.barrier()

    def capture(fn, n_launch_out):
        """Capture fn() into a CUDA graph on a side stream; returns the graph,
        or None (after printing why) when capture fails."""
        try:
            side = torch.cuda.Stream(device=dev)
            side.wait_stream(stream)
            g = torch.cuda.CUDAGraph()
            nc = kd.kd_launch_count()
            # thread_local: other threads of the process (e.g. a process group's
            # watchdog) may keep making CUDA calls while this thread captures
            with torch.cuda.graph(g, stream=side, capture_error_mode="thread_local"):
                fn()
            n_launch_out.append(kd.kd_launch_count() - nc)
            stream.wait_stream(side)
            g.replay()                                   # upload; untimed
            torch.cuda.synchronize()
            return g
        except Exception as exc:
            print(f"bench: CUDA graph capture failed ({exc!r}); timing eager steps",
                  file=sys.stderr, flush=True)
            torch.cuda.synchronize()
            return None

    # warm-up
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert kd.read_device_status(ws) == kd.KD_OK

    # The timed region: K steps captured, one after the other, in ONE CUDA graph
    # (the library allocates nothing and never synchronises inside a call) and
    # run by one replay.  Each step carries its own four timing events and
    # every GEMM launch its own pair (external event nodes of the graph), so
    # the top-K, forward and backward times, and the per-GEMM figures, are
    # those of the K timed steps themselves.  --no-graph times K eager steps,
    # with the same events.
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
           for _ in range(args.steps)]
    per_step_launches = 4 * ((T + chunk - 1) // chunk) + 16
    # Per-GEMM events go around the launches of the LAST timed step only: an
    # event between two kernels stops the second from starting while the first
    # finishes (programmatic dependent launch), so the other steps run as a
    # user's would.
    prof = kd.GemmProfiler(capacity=per_step_launches)

    def steps_once():
        for i in range(args.steps):
            if i == args.steps - 1:
                with prof:
                    step(evs[i])
            else:
                step(evs[i])
    graph = None
    graph_launches = []
    if args.dp and world > 1 and args.graph:
        # the step holds NCCL collectives: time eager steps rather than capture them
        args.graph = False
    if args.graph:
        graph = capture(steps_once, graph_launches)
        if graph is None:
            prof = kd.GemmProfiler(capacity=per_step_launches)
        else:
            assert kd.read_device_status(ws) == kd.KD_OK
    sampler = ClockSampler(local) if rank == 0 else None
    torch.cuda.reset_peak_memory_stats(dev)
    barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    n0 = kd.kd_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graph is not None:
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        n_launch = graph_launches[0]                      # a replay runs no host code
    else:
        e0.record()
        steps_once()
        e1.record()
        torch.cuda.synchronize()
        n_launch = kd.kd_launch_count() - n0
    assert kd.read_device_status(ws) == kd.KD_OK
    clocks = sampler.stop() if sampler else None
    barrier()
    peak_bytes = torch.cuda.max_memory_allocated(dev)
    ms_total, value = job_throughput(e0.elapsed_time(e1), T * args.steps, world, dev)
    ms_step = ms_total / args.steps
    flop_step = 8.0 * T * d * V

    # components of the timed steps (sums over the K steps, per step below)
    topk_sum = sum(e[0].elapsed_time(e[1]) for e in evs)
    fwd_sum = sum(e[1].elapsed_time(e[2]) for e in evs)
    bwd_sum = sum(e[2].elapsed_time(e[3]) for e in evs)
    gaps_sum = sum(evs[i][3].elapsed_time(evs[i + 1][0]) for i in range(args.steps - 1))
    local_region_ms = e0.elapsed_time(e1)
    topk_ms = topk_sum / args.steps
    fwd_ms = fwd_sum / args.steps
    bwd_ms = bwd_sum / args.steps

    # per-GEMM-kind breakdown from the live events
    res = prof.results()
    kinds = {}
    for k, f, ms in res:
        e = kinds.setdefault(kd.GEMM_KIND_NAMES[k], {"launches": 0, "ms": 0.0, "flops": 0.0})
        e["launches"] += 1
        e["ms"] += ms
        e["flops"] += f
    dom = max(kinds.items(), key=lambda kv: kv[1]["ms"])
    peaks, peak_src = _peaks()
    peak_sus = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    achieved = dom[1]["flops"] / (dom[1]["ms"] / 1000.0) / 1e12
    gemm_ms_step = sum(v["ms"] for v in kinds.values())        # the last timed step
    loss_ms = fwd_ms + bwd_ms
    loss_tflops = flop_step / (loss_ms / 1000.0) / 1e12
    topk_bytes = T * V * 2 + T * K * 8

    # The top-K build timed alone: R builds in one graph, clocks sampled, after
    # the timed region (so it is not part of the step's number).
    topk_alone = None
    if rank == 0 and not args.no_topk_alone:
        R = 20
        ev_a = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]

        def topk_only():
            sp_ = torch.cuda.current_stream().cuda_stream
            ev_a[0].record()
            for _ in range(R):
                st_ = kd.kd_topk_build(logits.data_ptr(), kd.KD_DTYPE_BF16, T, V, K,
                                       vals.data_ptr(), idx.data_ptr(), ws_topk.data_ptr(),
                                       ws_topk.numel(), sp_)
                if st_ != 0:
                    raise RuntimeError(f"kd_topk_build failed ({st_})")
            ev_a[1].record()
        gt = capture(topk_only, []) if args.graph else None
        samp = ClockSampler(local)
        torch.cuda.synchronize()
        samp.start()
        time.sleep(0.3)
        for _ in range(3):
            if gt is not None:
                gt.replay()
            else:
                topk_only()
        torch.cuda.synchronize()
        ck = samp.stop()
        assert kd.read_device_status(ws_topk) == kd.KD_OK
        ms_a = ev_a[0].elapsed_time(ev_a[1]) / R           # the last replay's R builds
        topk_alone = {"ms": ms_a, "gbs": topk_bytes / (ms_a / 1000.0) / 1e9,
                      "frac_hbm_peak": topk_bytes / (ms_a / 1000.0) / 1e9 / float(peaks["hbm_gbs"]),
                      "builds": R, "clocks": ck,
                      "note": "the same build timed alone, back to back, outside the step"}
        del gt

    # loss-path memory: what the fused loss holds (inputs, cache, outputs, workspace)
    loss_path_bytes = (h.numel() * h.element_size() + W.numel() * W.element_size()
                       + vals.numel() * 4 + idx.numel() * 4 + lse.numel() * 4
                       + dH.numel() * dH.element_size() + dW.numel() * 4 + ws.numel())

    # e2e: host-resident inputs through the same public API, copies inside the
    # timed region.  Each step's inputs (h, W, teacher logits) are copied from
    # pinned host memory on a copy stream into one of two device buffer sets,
    # so step i+1's copy overlaps step i's kernels; each step's loss is read
    # back to the host.  The region runs from the first copy to the last
    # read-back.
    e2e = None
    if not args.no_e2e:
        h_host = h.cpu().pin_memory()
        W_host = W.cpu().pin_memory()
        x_host = logits.cpu().pin_memory()
        loss_host = torch.empty((args.steps,), dtype=torch.float32).pin_memory()
        h2d = h.numel() * h.element_size() + W.numel() * W.element_size() + x_host.numel() * 2
        sets = [(h, W, logits), (torch.empty_like(h), torch.empty_like(W), torch.empty_like(logits))]
        copy_stream = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        consumed = [torch.cuda.Event() for _ in range(2)]
        for e in consumed:
            e.record(stream)
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(copy_stream)
        for i in range(args.steps):
            buf = sets[i % 2]
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(consumed[i % 2])
                buf[0].copy_(h_host, non_blocking=True)
                buf[1].copy_(W_host, non_blocking=True)
                buf[2].copy_(x_host, non_blocking=True)
                copied[i % 2].record(copy_stream)
            stream.wait_event(copied[i % 2])
            step(inp=buf)
            loss_host[i].copy_(loss, non_blocking=True)
            consumed[i % 2].record(stream)
        b.record(stream)
        torch.cuda.synchronize()
        ems, e2e_value = job_throughput(a.elapsed_time(b), T * args.steps, world, dev)
        assert bool(torch.isfinite(loss_host).all())
        e2e = {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": 4, "ms_per_step": ems / args.steps,
               "overlap": "inputs of step i+1 copied while step i computes (2 buffer sets)"}
        del sets

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        torch.cuda.nvtx.range_push("cpu_baseline")
        cpu = cpu_baseline(w, rows=args.cpu_rows or 128,
                           gpu=dict(h=h, W=W, logits=logits, vals=vals, idx=idx, lse=lse, dH=dH))
        torch.cuda.nvtx.range_pop()

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if dt == torch.bfloat16 else "f32",
        "data": "synthetic",
        "config": _config(w, args.workload, {
            "parallelism": (f"dp{world} (T-sharded batch of {T * world} positions, "
                            "all-reduce of dW and the loss)" if args.dp else f"replicas x{world}"),
            "timed_steps": ("K steps captured in one CUDA graph, run by one replay"
                            if graph is not None else "K eager steps")}),
        "loss_fwd_bwd": {"ms": loss_ms, "tokens_per_s": T / (loss_ms / 1000.0),
                          "tflops": loss_tflops,
                          "frac_bf16_peak_sustained": loss_tflops / peak_sus,
                          "frac_bf16_peak_burst": loss_tflops / float(peaks["bf16_tflops"]),
                          "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
                          "gemm_ms": gemm_ms_step},
        "topk_build": {"ms": topk_ms, "gbs": topk_bytes / (topk_ms / 1000.0) / 1e9,
                       "frac_hbm_peak": topk_bytes / (topk_ms / 1000.0) / 1e9
                       / float(peaks["hbm_gbs"]),
                       "bytes": int(topk_bytes)},
        "topk_build_alone": topk_alone,
        "components": {
            "source": "CUDA events of the timed steps (inside the timed region)",
            "topk_ms": topk_ms, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
            "between_steps_ms": gaps_sum / args.steps,
            "sum_over_ms_per_step": (topk_sum + fwd_sum + bwd_sum + gaps_sum)
            / max(local_region_ms, 1e-9)},
        "gemm_kernels": {k: {"launches": v["launches"], "ms_per_launch": v["ms"] / v["launches"],
                             "tflops": v["flops"] / (v["ms"] / 1000.0) / 1e12}
                         for k, v in kinds.items()},
        "peak_mem_bytes": int(peak_bytes),
        "loss_path_bytes": int(loss_path_bytes),
        "dense_logits_grid_bytes_fp32": int(T * V * 4),
        "roofline": {"bound": "tensor", "kernel": f"gemm2_kernel ({dom[0]})",
                     "achieved": achieved, "peak": peak_sus, "unit": "TFLOP/s",
                     "frac": achieved / peak_sus,
                     "traffic": (NCU_TRAFFIC["per_launch_bytes"].get(dom[0])
                                 if _gemm_source_digest() == NCU_TRAFFIC["source_sha256_16"]
                                 else None),
                     "peak_source": f"{peak_src} bf16_tflops_sustained (kernel inside a long step)"},
        "gpu_launches": int(n_launch),
        "clocks": clocks,
        # board power sampled during the timed steps (rank 0's GPU): the
        # energy of one step, and the step's 8TdV flops per joule of it
        "energy": (None if not clocks or clocks.get("power_w") is None else {
            "power_w_median": clocks["power_w"],
            "joules_per_step": clocks["power_w"] * ms_step / 1e3,
            "tflop_per_joule": flop_step / 1e12 / (clocks["power_w"] * ms_step / 1e3)}),
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def sweep_memory(args):
    """Peak device memory of the fused loss (fwd + bwd) vs T at d=4096, V=131072."""
    import torch
    from chunked_kl_loss_chunk_b200 import build as kbuild
    from chunked_kl_loss_chunk_b200 import inputs, kd
    kbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    torch.empty(1, device=dev)          # initialise the caching allocator
    d, V, K, chunk = 4096, 131072, 100, 4096
    out = []
    for T in (4096, 8192, 16384, 32768, 65536, 131072, 262144):
        torch.cuda.empty_cache()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        h, W, vals, idx = inputs.make_loss_inputs(T, d, V, K, dtype=torch.bfloat16, seed=0, device=dev)
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats(dev)
        loss, lse, kl, ws = kd.fused_kl_fwd(h, W, vals, idx, chunk, 1.0)
        dH, dW, ws_b = kd.fused_kl_bwd(h, W, vals, idx, lse, chunk, 1.0, ws=ws)
        torch.cuda.synchronize()
        peak = torch.cuda.max_memory_allocated(dev) - base
        out.append({"T": T, "peak_bytes": int(peak), "dense_grid_fp32_bytes": T * V * 4})
        del h, W, vals, idx, loss, lse, kl, ws, ws_b, dH, dW
    xs = [o["T"] for o in out]
    ys = [o["peak_bytes"] for o in out]
    n = len(xs)
    mx, my = sum(xs) / n, sum(ys) / n
    b = sum((x - mx) * (y - my) for x, y in zip(xs, ys)) / sum((x - mx) ** 2 for x in xs)
    a = my - b * mx
    ss_res = sum((y - (a + b * x)) ** 2 for x, y in zip(xs, ys))
    ss_tot = sum((y - my) ** 2 for y in ys)
    print(json.dumps({"sweep": out, "fit": {"intercept_bytes": a, "bytes_per_token": b,
                                            "r2": 1 - ss_res / ss_tot}}), flush=True)


def main():
    args = _args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.sweep_memory:
        sweep_memory(args)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        run_kd(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
