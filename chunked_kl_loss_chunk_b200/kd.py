"""Thin Python binding of libkd (the C ABI in include/kd.h).

Argument marshalling only: every step of the top-K build and of the fused
chunked KL loss runs in the library's CUDA kernels.  PyTorch supplies device
memory and the current stream.  There is no CPU fallback: if libkd.so is
missing or fails to load, every call raises.

Low-level functions carry the C names (``kd_topk_build``, ``kd_fused_kl_fwd``,
``kd_fused_kl_bwd`` ...) and take raw integers (device pointers, sizes, stream
handle).  ``topk_build``, ``fused_kl_fwd``, ``fused_kl_bwd`` and
``FusedTopKKLLoss`` wrap them for torch tensors.
"""

from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libkd.so")
DEBUG_LIB_PATH = os.path.join(_PKG_DIR, "libkd_debug.so")   # built with -DKD_DEBUG=1
HEADER_PATH = os.path.join(os.path.dirname(_PKG_DIR), "include", "kd.h")

KD_OK, KD_ERR_INVALID_ARG, KD_ERR_UNSUPPORTED, KD_ERR_WORKSPACE = 0, 1, 2, 3
KD_ERR_BAD_INDEX, KD_ERR_TIMEOUT, KD_ERR_CUDA, KD_ERR_INTERNAL = 4, 5, 6, 7
KD_DTYPE_F32, KD_DTYPE_BF16 = 0, 1
KD_KL_LOGPROB_CACHE, KD_KL_TAU_SQUARED = 0x1, 0x2
CACHE_KINDS = ("logits", "logprobs")

_c_i64, _c_int, _c_sz, _c_vp, _c_u64 = ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_uint64
_c_u32 = ctypes.c_uint32

_SIGNATURES = {
    "kd_status_string": (ctypes.c_char_p, [_c_int]),
    "kd_version": (_c_int, []),
    "kd_topk_workspace_size": (_c_sz, [_c_i64, _c_i64, _c_int]),
    "kd_topk_build": (_c_int, [_c_vp, _c_int, _c_i64, _c_i64, _c_int, _c_vp, _c_vp, _c_vp, _c_sz, _c_vp]),
    "kd_fused_kl_workspace_size": (_c_sz, [_c_i64, _c_i64, _c_i64, _c_int, _c_i64, _c_int]),
    "kd_fused_kl_fwd": (_c_int, [_c_vp, _c_vp, _c_int, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp, _c_int,
                                 _c_i64, ctypes.c_float, _c_vp, _c_vp, _c_vp, _c_vp, _c_sz, _c_vp]),
    "kd_fused_kl_bwd": (_c_int, [_c_vp, _c_vp, _c_int, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp, _c_int,
                                 _c_i64, ctypes.c_float, _c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_vp,
                                 _c_sz, _c_vp]),
    "kd_fused_kl_fwd_ex": (_c_int, [_c_vp, _c_vp, _c_int, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp, _c_int,
                                    _c_i64, ctypes.c_float, _c_u32, _c_vp, _c_vp, _c_vp, _c_vp, _c_sz,
                                    _c_vp]),
    "kd_fused_kl_bwd_ex": (_c_int, [_c_vp, _c_vp, _c_int, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp, _c_int,
                                    _c_i64, ctypes.c_float, _c_u32, _c_vp, _c_vp, _c_vp, _c_vp, _c_int,
                                    _c_vp, _c_sz, _c_vp]),
    "kd_fused_kl_fwd_shard": (_c_int, [_c_vp, _c_vp, _c_int, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp,
                                       _c_int, _c_i64, ctypes.c_float, _c_u32, _c_i64, _c_vp, _c_vp,
                                       _c_vp, _c_vp, _c_sz, _c_vp]),
    "kd_fused_kl_bwd_shard": (_c_int, [_c_vp, _c_vp, _c_int, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp,
                                       _c_int, _c_i64, ctypes.c_float, _c_u32, _c_i64, _c_vp, _c_vp,
                                       _c_vp, _c_vp, _c_int, _c_vp, _c_sz, _c_vp]),
    "kd_read_device_status": (_c_int, [_c_vp, _c_vp]),
    "kd_set_wait_limit_ns": (_c_int, [_c_u64]),
    "kd_debug_wait_probe": (_c_int, [_c_vp, _c_sz, _c_u64, _c_vp]),
    "kd_launch_count": (_c_u64, []),
    "kd_fused_kl_fwd_noalloc": (_c_int, [_c_vp, _c_vp, _c_int, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp,
                                         _c_int, _c_i64, ctypes.c_float, _c_vp, _c_vp, _c_vp, _c_vp]),
    "kd_profile_attach": (_c_int, [_c_vp, _c_vp, _c_vp, _c_vp, _c_int, _c_int]),
    "kd_profile_detach": (_c_int, []),
}

KD_GEMM_FWD_LSE, KD_GEMM_BWD_DZ, KD_GEMM_DH, KD_GEMM_DW = 1, 2, 4, 8
GEMM_KIND_NAMES = {1: "fwd_lse", 2: "bwd_dz", 4: "dH", 8: "dW", 12: "dH+dW"}

_lib = None


def header_symbols():
    """Names of the functions declared in include/kd.h."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kd_[a-z0-9_]+)\s*\(", text)))


def load():
    """Load libkd.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libkd.so not built ({LIB_PATH}); run chunked_kl_loss_chunk_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def use_library(path: str):
    """Route every later call to the library at `path` (e.g. DEBUG_LIB_PATH,
    whose kernels also check internal invariants); returns the previous path."""
    global _lib, LIB_PATH
    prev = LIB_PATH
    LIB_PATH = path
    _lib = None
    load()
    return prev


class KDError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def status_string(status: int) -> str:
    return load().kd_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != KD_OK:
        raise KDError(status, where)


# ---------------------------------------------------------------- raw C names

def kd_topk_workspace_size(T, V, K):
    return load().kd_topk_workspace_size(T, V, K)


def kd_topk_build(logits, dtype, T, V, K, out_vals, out_idx, ws, ws_bytes, stream):
    return load().kd_topk_build(logits, dtype, T, V, K, out_vals, out_idx, ws, ws_bytes, stream)


def kd_fused_kl_workspace_size(T, d, V, K, chunk, dtype):
    return load().kd_fused_kl_workspace_size(T, d, V, K, chunk, dtype)


def kd_fused_kl_fwd(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, loss, lse, kl_rows,
                    ws, ws_bytes, stream):
    return load().kd_fused_kl_fwd(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, loss,
                                  lse, kl_rows, ws, ws_bytes, stream)


def kd_fused_kl_bwd(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, lse, grad_loss, dH,
                    dW, accumulate_dW, ws, ws_bytes, stream):
    return load().kd_fused_kl_bwd(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, lse,
                                  grad_loss, dH, dW, accumulate_dW, ws, ws_bytes, stream)


def kd_fused_kl_fwd_ex(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, flags, loss, lse,
                       kl_rows, ws, ws_bytes, stream):
    return load().kd_fused_kl_fwd_ex(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature,
                                     flags, loss, lse, kl_rows, ws, ws_bytes, stream)


def kd_fused_kl_bwd_ex(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, flags, lse,
                       grad_loss, dH, dW, accumulate_dW, ws, ws_bytes, stream):
    return load().kd_fused_kl_bwd_ex(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature,
                                     flags, lse, grad_loss, dH, dW, accumulate_dW, ws, ws_bytes,
                                     stream)


def kd_fused_kl_fwd_shard(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, flags,
                          T_total, loss, lse, kl_rows, ws, ws_bytes, stream):
    return load().kd_fused_kl_fwd_shard(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature,
                                        flags, T_total, loss, lse, kl_rows, ws, ws_bytes, stream)


def kd_fused_kl_bwd_shard(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, flags,
                          T_total, lse, grad_loss, dH, dW, accumulate_dW, ws, ws_bytes, stream):
    return load().kd_fused_kl_bwd_shard(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature,
                                        flags, T_total, lse, grad_loss, dH, dW, accumulate_dW, ws,
                                        ws_bytes, stream)


def kd_fused_kl_fwd_noalloc(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature, loss, lse,
                            kl_rows, stream):
    """Forward for callers that cannot provide a workspace (scratch is a fixed
    array inside the library; see include/kd.h for its limit and caveats)."""
    return load().kd_fused_kl_fwd_noalloc(h, W, dtype, T, d, V, t_vals, t_idx, K, chunk, temperature,
                                          loss, lse, kl_rows, stream)


def kd_read_device_status(ws, stream):
    return load().kd_read_device_status(ws, stream)


def kd_set_wait_limit_ns(limit_ns):
    return load().kd_set_wait_limit_ns(limit_ns)


def kd_debug_wait_probe(ws, ws_bytes, limit_ns, stream):
    return load().kd_debug_wait_probe(ws, ws_bytes, limit_ns, stream)


def kd_launch_count():
    return load().kd_launch_count()


def kd_profile_attach(start_events, end_events, kinds, flops, capacity, kind_mask):
    return load().kd_profile_attach(start_events, end_events, kinds, flops, capacity, kind_mask)


def kd_profile_detach():
    return load().kd_profile_detach()


class GemmProfiler:
    """Records CUDA events around every tensor-core GEMM launch (per kind)
    while active; ``results()`` gives (kind, flops, ms) per launch."""

    def __init__(self, capacity: int = 4096, kind_mask: int = 15):
        self.capacity = capacity
        self.kind_mask = kind_mask
        self.start = [torch.cuda.Event(enable_timing=True) for _ in range(capacity)]
        self.end = [torch.cuda.Event(enable_timing=True) for _ in range(capacity)]
        for e in self.start + self.end:      # materialise the event handles
            e.record()
        torch.cuda.synchronize()
        self._s = (ctypes.c_void_p * capacity)(*[e.cuda_event for e in self.start])
        self._e = (ctypes.c_void_p * capacity)(*[e.cuda_event for e in self.end])
        self._k = (ctypes.c_int * capacity)()
        self._f = (ctypes.c_double * capacity)()
        self.n = 0

    def __enter__(self):
        _check(kd_profile_attach(self._s, self._e, self._k, self._f, self.capacity, self.kind_mask),
               "kd_profile_attach")
        return self

    def __exit__(self, *exc):
        self.n = kd_profile_detach()
        return False

    def results(self):
        torch.cuda.synchronize()
        return [(int(self._k[i]), float(self._f[i]), self.start[i].elapsed_time(self.end[i]))
                for i in range(self.n)]


# ---------------------------------------------------------------- torch helpers

def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KD_DTYPE_BF16
    if t.dtype == torch.float32:
        return KD_DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """Caller-owned workspace: a 1024-byte-aligned uint8 view of ``nbytes``."""
    n = max(int(nbytes), 1024)
    buf = torch.empty(n + 1024, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % 1024
    ws = buf[off:off + n]
    assert ws.data_ptr() % 1024 == 0
    return ws


def read_device_status(ws: torch.Tensor, stream=None) -> int:
    return kd_read_device_status(ws.data_ptr(), _stream(stream))


def topk_build(logits: torch.Tensor, K: int, ws: torch.Tensor | None = None, stream=None):
    """Top-K cache of bf16 teacher logits [T, V] -> (vals f32 [T,K], idx i32 [T,K])."""
    assert logits.is_cuda and logits.is_contiguous() and logits.dim() == 2
    T, V = logits.shape
    vals = torch.empty((T, K), dtype=torch.float32, device=logits.device)
    idx = torch.empty((T, K), dtype=torch.int32, device=logits.device)
    need = kd_topk_workspace_size(T, V, K)
    if ws is None:
        ws = alloc_workspace(need, logits.device)
    _check(kd_topk_build(logits.data_ptr(), _dtype_code(logits), T, V, K, vals.data_ptr(),
                         idx.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)),
           "kd_topk_build")
    return vals, idx


def workspace_for(h: torch.Tensor, W: torch.Tensor, K: int, chunk: int) -> torch.Tensor:
    T, d = h.shape
    V = W.shape[0]
    return alloc_workspace(kd_fused_kl_workspace_size(T, d, V, K, chunk, _dtype_code(h)), h.device)


def kl_flags(cache: str = "logits", tau_squared: bool = False) -> int:
    """The C ABI's flag bits for a cache kind ("logits": renormalised top-K
    logits; "logprobs": full-vocabulary teacher log-probabilities, S <= 1) and
    the optional tau^2 factor."""
    if cache not in CACHE_KINDS:
        raise ValueError(f"cache must be one of {CACHE_KINDS}")
    return (KD_KL_LOGPROB_CACHE if cache == "logprobs" else 0) | (KD_KL_TAU_SQUARED if tau_squared else 0)


def fused_kl_fwd(h, W, t_vals, t_idx, chunk: int, temperature: float = 1.0, ws=None,
                 kl_rows: bool = False, stream=None, cache: str = "logits",
                 tau_squared: bool = False, T_total: int | None = None):
    """Returns (loss [] f32, lse [T] f32, kl [T] f32 or None, ws).  With
    ``T_total`` the rows are one data-parallel shard of a batch of T_total
    positions (kd_fused_kl_fwd_shard): the loss is this shard's part of the
    batch's mean."""
    for t in (h, W, t_vals, t_idx):
        assert t.is_cuda and t.is_contiguous()
    T, d = h.shape
    V = W.shape[0]
    K = t_vals.shape[1]
    flags = kl_flags(cache, tau_squared)
    if ws is None:
        ws = workspace_for(h, W, K, chunk)
    loss = torch.empty((), dtype=torch.float32, device=h.device)
    lse = torch.empty((T,), dtype=torch.float32, device=h.device)
    kl = torch.empty((T,), dtype=torch.float32, device=h.device) if kl_rows else None
    if T_total is None:
        _check(kd_fused_kl_fwd_ex(h.data_ptr(), W.data_ptr(), _dtype_code(h), T, d, V,
                                  t_vals.data_ptr(), t_idx.data_ptr(), K, chunk, float(temperature),
                                  flags, loss.data_ptr(), lse.data_ptr(), _ptr(kl), ws.data_ptr(),
                                  ws.numel(), _stream(stream)),
               "kd_fused_kl_fwd_ex")
    else:
        _check(kd_fused_kl_fwd_shard(h.data_ptr(), W.data_ptr(), _dtype_code(h), T, d, V,
                                     t_vals.data_ptr(), t_idx.data_ptr(), K, chunk,
                                     float(temperature), flags, int(T_total), loss.data_ptr(),
                                     lse.data_ptr(), _ptr(kl), ws.data_ptr(), ws.numel(),
                                     _stream(stream)),
               "kd_fused_kl_fwd_shard")
    return loss, lse, kl, ws


def fused_kl_bwd(h, W, t_vals, t_idx, lse, chunk: int, temperature: float = 1.0, grad_loss=None,
                 ws=None, dH=None, dW=None, accumulate_dW: bool = False, stream=None,
                 cache: str = "logits", tau_squared: bool = False, T_total: int | None = None):
    """Returns (dH [T,d] dtype of h, dW [V,d] f32, ws).  With ``T_total`` the
    rows are one data-parallel shard of a batch of T_total positions
    (kd_fused_kl_bwd_shard): dH is the batch gradient's rows of this shard and
    dW this shard's term of the batch's dW."""
    T, d = h.shape
    V = W.shape[0]
    K = t_vals.shape[1]
    flags = kl_flags(cache, tau_squared)
    if ws is None:
        ws = workspace_for(h, W, K, chunk)
    if dH is None:
        dH = torch.empty_like(h)
    if dW is None:
        dW = torch.empty((V, d), dtype=torch.float32, device=h.device)
    if T_total is None:
        _check(kd_fused_kl_bwd_ex(h.data_ptr(), W.data_ptr(), _dtype_code(h), T, d, V,
                                  t_vals.data_ptr(), t_idx.data_ptr(), K, chunk, float(temperature),
                                  flags, lse.data_ptr(), _ptr(grad_loss), dH.data_ptr(),
                                  dW.data_ptr(), int(accumulate_dW), ws.data_ptr(), ws.numel(),
                                  _stream(stream)),
               "kd_fused_kl_bwd_ex")
    else:
        _check(kd_fused_kl_bwd_shard(h.data_ptr(), W.data_ptr(), _dtype_code(h), T, d, V,
                                     t_vals.data_ptr(), t_idx.data_ptr(), K, chunk,
                                     float(temperature), flags, int(T_total), lse.data_ptr(),
                                     _ptr(grad_loss), dH.data_ptr(), dW.data_ptr(),
                                     int(accumulate_dW), ws.data_ptr(), ws.numel(),
                                     _stream(stream)),
               "kd_fused_kl_bwd_shard")
    return dH, dW, ws


class FusedTopKKLLoss(torch.autograd.Function):
    """Drop-in loss: forward = kd_fused_kl_fwd_ex, backward = kd_fused_kl_bwd_ex.

    ``loss = FusedTopKKLLoss.apply(h, W, t_vals, t_idx, chunk, temperature)``,
    optionally followed by ``cache`` ("logits" or "logprobs") and
    ``tau_squared``; gradients flow to h and W (W's gradient is returned in
    W's dtype).
    """

    @staticmethod
    def forward(ctx, h, W, t_vals, t_idx, chunk, temperature, cache="logits", tau_squared=False):
        loss, lse, _, ws = fused_kl_fwd(h, W, t_vals, t_idx, chunk, temperature, cache=cache,
                                        tau_squared=tau_squared)
        ctx.save_for_backward(h, W, t_vals, t_idx, lse)
        ctx.chunk, ctx.temperature, ctx.ws = chunk, temperature, ws
        ctx.cache, ctx.tau_squared = cache, tau_squared
        return loss

    @staticmethod
    def backward(ctx, g):
        h, W, t_vals, t_idx, lse = ctx.saved_tensors
        g = g.to(torch.float32).contiguous()
        dH, dW, _ = fused_kl_bwd(h, W, t_vals, t_idx, lse, ctx.chunk, ctx.temperature,
                                 grad_loss=g, ws=ctx.ws, cache=ctx.cache,
                                 tau_squared=ctx.tau_squared)
        return dH, dW.to(W.dtype), None, None, None, None, None, None
