"""Host-side tests of the C ABI (no GPU needed, no kernel launched).

Every call below fails argument validation, which returns before any CUDA call,
so these run on a CPU-only machine and are harmless on a GPU machine.
"""

import ctypes
import os

import pytest

from chunked_kl_loss_chunk_b200 import kd

FAKE = 0x7F0000000000  # 1024-aligned fake device address; never dereferenced


@pytest.fixture(scope="module")
def lib():
    from chunked_kl_loss_chunk_b200 import build
    build.build()
    return kd.load()


def test_every_header_symbol_is_exported(lib):
    names = kd.header_symbols()
    assert {"kd_topk_build", "kd_fused_kl_fwd", "kd_fused_kl_bwd", "kd_read_device_status",
            "kd_status_string", "kd_topk_workspace_size", "kd_fused_kl_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in [(0, "KD_OK"), (1, "KD_ERR_INVALID_ARG"), (2, "KD_ERR_UNSUPPORTED"),
                       (3, "KD_ERR_WORKSPACE"), (4, "KD_ERR_BAD_INDEX"), (5, "KD_ERR_TIMEOUT"),
                       (6, "KD_ERR_CUDA"), (7, "KD_ERR_INTERNAL")]:
        assert kd.status_string(code) == name
    assert kd.status_string(99) == "KD_ERR_UNKNOWN"
    assert kd.load().kd_version() >> 16 == 1


def test_workspace_sizes(lib):
    assert kd.kd_topk_workspace_size(8192, 131072, 100) >= 4
    # fused: status + sorted cache (8 B/entry) + stats + kl + max(partials, dz)
    T, d, V, K, c = 32768, 4096, 131072, 100, 2048
    n = kd.kd_fused_kl_workspace_size(T, d, V, K, c, kd.KD_DTYPE_BF16)
    dz = 2 * c * V * 2             # the backward keeps dz of two consecutive chunks
    cache = T * K * 8
    hpart = 4 * c * d * 4          # fp32 partials of up to 4 K-splits of dH
    assert dz + cache + hpart <= n <= dz + cache + hpart + T * 16 + 64 * 1024
    # constant in T apart from the O(T) cache/stat terms (linear memory)
    n2 = kd.kd_fused_kl_workspace_size(2 * T, d, V, K, c, kd.KD_DTYPE_BF16)
    assert n2 - n <= T * (8 * K + 12) + 4096
    # fp32 dz is twice as wide
    nf = kd.kd_fused_kl_workspace_size(256, 256, 4096, 16, 64, kd.KD_DTYPE_F32)
    nb = kd.kd_fused_kl_workspace_size(256, 256, 4096, 16, 64, kd.KD_DTYPE_BF16)
    assert nf > nb
    assert kd.kd_fused_kl_workspace_size(0, 8, 8, 1, 1, 1) == 0


def _topk(**kw):
    a = dict(logits=FAKE, dtype=kd.KD_DTYPE_BF16, T=4, V=64, K=8, vals=FAKE, idx=FAKE, ws=FAKE,
             ws_bytes=1 << 20, stream=None)
    a.update(kw)
    return kd.kd_topk_build(a["logits"], a["dtype"], a["T"], a["V"], a["K"], a["vals"], a["idx"],
                            a["ws"], a["ws_bytes"], a["stream"])


def test_topk_validation(lib):
    assert _topk(logits=None) == kd.KD_ERR_INVALID_ARG
    assert _topk(vals=None) == kd.KD_ERR_INVALID_ARG
    assert _topk(K=65) == kd.KD_ERR_INVALID_ARG           # K > V
    assert _topk(K=0) == kd.KD_ERR_INVALID_ARG
    assert _topk(T=0) == kd.KD_ERR_INVALID_ARG
    assert _topk(logits=FAKE + 2) == kd.KD_ERR_INVALID_ARG  # misaligned
    assert _topk(ws=FAKE + 256) == kd.KD_ERR_INVALID_ARG    # ws not 1024-aligned
    assert _topk(dtype=kd.KD_DTYPE_F32) == kd.KD_ERR_UNSUPPORTED
    assert _topk(V=5000, K=1025) == kd.KD_ERR_UNSUPPORTED  # K above the maximum
    assert _topk(ws_bytes=16) == kd.KD_ERR_WORKSPACE


def _fwd(**kw):
    a = dict(h=FAKE, W=FAKE, dtype=kd.KD_DTYPE_BF16, T=256, d=256, V=4096, vals=FAKE, idx=FAKE,
             K=16, chunk=64, tau=1.0, loss=FAKE, lse=FAKE, kl=None, ws=FAKE, ws_bytes=1 << 40,
             stream=None)
    a.update(kw)
    return kd.kd_fused_kl_fwd(a["h"], a["W"], a["dtype"], a["T"], a["d"], a["V"], a["vals"], a["idx"],
                              a["K"], a["chunk"], a["tau"], a["loss"], a["lse"], a["kl"], a["ws"],
                              a["ws_bytes"], a["stream"])


def _bwd(**kw):
    a = dict(h=FAKE, W=FAKE, dtype=kd.KD_DTYPE_BF16, T=256, d=256, V=4096, vals=FAKE, idx=FAKE,
             K=16, chunk=64, tau=1.0, lse=FAKE, g=None, dH=FAKE, dW=FAKE, acc=0, ws=FAKE,
             ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return kd.kd_fused_kl_bwd(a["h"], a["W"], a["dtype"], a["T"], a["d"], a["V"], a["vals"], a["idx"],
                              a["K"], a["chunk"], a["tau"], a["lse"], a["g"], a["dH"], a["dW"],
                              a["acc"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("call", [_fwd, _bwd])
def test_loss_validation(lib, call):
    E = kd
    assert call(h=None) == E.KD_ERR_INVALID_ARG
    assert call(W=None) == E.KD_ERR_INVALID_ARG
    assert call(vals=None) == E.KD_ERR_INVALID_ARG
    assert call(idx=None) == E.KD_ERR_INVALID_ARG
    assert call(ws=None) == E.KD_ERR_INVALID_ARG
    assert call(T=0) == E.KD_ERR_INVALID_ARG
    assert call(chunk=0) == E.KD_ERR_INVALID_ARG
    assert call(K=4097) == E.KD_ERR_INVALID_ARG            # K > V
    assert call(tau=0.0) == E.KD_ERR_INVALID_ARG
    assert call(tau=-1.0) == E.KD_ERR_INVALID_ARG
    assert call(tau=float("inf")) == E.KD_ERR_INVALID_ARG
    assert call(tau=float("nan")) == E.KD_ERR_INVALID_ARG
    assert call(h=FAKE + 8) == E.KD_ERR_INVALID_ARG         # misaligned
    assert call(ws=FAKE + 512) == E.KD_ERR_INVALID_ARG
    assert call(dtype=7) == E.KD_ERR_UNSUPPORTED
    assert call(d=12) == E.KD_ERR_UNSUPPORTED               # d % 8 != 0
    assert call(K=1025) == E.KD_ERR_UNSUPPORTED             # K above the maximum
    assert call(ws_bytes=1024) == E.KD_ERR_WORKSPACE
    assert call(T=1 << 40) == E.KD_ERR_UNSUPPORTED
    assert call(T=(1 << 30) + 1, chunk=(1 << 30) + 1) == E.KD_ERR_UNSUPPORTED   # rows per chunk
    assert call(T=(1 << 31), chunk=1 << 30, ws_bytes=1024) == E.KD_ERR_WORKSPACE   # 2^30 rows pass


def test_fwd_output_pointers(lib):
    assert _fwd(loss=None) == kd.KD_ERR_INVALID_ARG
    assert _fwd(lse=None) == kd.KD_ERR_INVALID_ARG
    assert _fwd(lse=FAKE + 4) == kd.KD_ERR_INVALID_ARG


def test_bwd_output_pointers(lib):
    assert _bwd(dH=None) == kd.KD_ERR_INVALID_ARG
    assert _bwd(dW=None) == kd.KD_ERR_INVALID_ARG
    assert _bwd(lse=None) == kd.KD_ERR_INVALID_ARG


def _fwd_ex(flags, **kw):
    a = dict(h=FAKE, W=FAKE, dtype=kd.KD_DTYPE_BF16, T=256, d=256, V=4096, vals=FAKE, idx=FAKE,
             K=16, chunk=64, tau=1.0, loss=FAKE, lse=FAKE, kl=None, ws=FAKE, ws_bytes=1 << 40,
             stream=None)
    a.update(kw)
    return kd.kd_fused_kl_fwd_ex(a["h"], a["W"], a["dtype"], a["T"], a["d"], a["V"], a["vals"],
                                 a["idx"], a["K"], a["chunk"], a["tau"], flags, a["loss"], a["lse"],
                                 a["kl"], a["ws"], a["ws_bytes"], a["stream"])


def _bwd_ex(flags, **kw):
    a = dict(h=FAKE, W=FAKE, dtype=kd.KD_DTYPE_BF16, T=256, d=256, V=4096, vals=FAKE, idx=FAKE,
             K=16, chunk=64, tau=1.0, lse=FAKE, g=None, dH=FAKE, dW=FAKE, acc=0, ws=FAKE,
             ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return kd.kd_fused_kl_bwd_ex(a["h"], a["W"], a["dtype"], a["T"], a["d"], a["V"], a["vals"],
                                 a["idx"], a["K"], a["chunk"], a["tau"], flags, a["lse"], a["g"],
                                 a["dH"], a["dW"], a["acc"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("call", [_fwd_ex, _bwd_ex])
def test_variant_flags_validation(lib, call):
    E = kd
    for bad in (0x4, 0x80000000, 0xFFFFFFFF, kd.KD_KL_LOGPROB_CACHE | 0x10):
        assert call(bad) == E.KD_ERR_INVALID_ARG
    # the shared checks still come first for valid flags
    for ok in (0, kd.KD_KL_LOGPROB_CACHE, kd.KD_KL_TAU_SQUARED, 3):
        assert call(ok, h=None) == E.KD_ERR_INVALID_ARG
        assert call(ok, tau=0.0) == E.KD_ERR_INVALID_ARG
        assert call(ok, d=12) == E.KD_ERR_UNSUPPORTED
        assert call(ok, ws_bytes=1024) == E.KD_ERR_WORKSPACE


def test_kl_flags_helper():
    assert kd.kl_flags() == 0
    assert kd.kl_flags("logprobs") == kd.KD_KL_LOGPROB_CACHE
    assert kd.kl_flags("logits", True) == kd.KD_KL_TAU_SQUARED
    assert kd.kl_flags("logprobs", True) == 3
    with pytest.raises(ValueError):
        kd.kl_flags("probs")


def test_debug_api_validation(lib):
    assert kd.kd_set_wait_limit_ns(10) == kd.KD_ERR_INVALID_ARG
    assert kd.kd_debug_wait_probe(None, 4096, 10 ** 6, None) == kd.KD_ERR_INVALID_ARG
    assert kd.kd_debug_wait_probe(FAKE, 16, 10 ** 6, None) == kd.KD_ERR_INVALID_ARG
    assert kd.kd_debug_wait_probe(FAKE, 4096, 10, None) == kd.KD_ERR_INVALID_ARG
    assert kd.kd_read_device_status(None, None) == kd.KD_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(kd, "_lib", None)
    monkeypatch.setattr(kd, "LIB_PATH", "/nonexistent/libkd.so")
    with pytest.raises(RuntimeError):
        kd.load()


def _fwd_noalloc(**kw):
    a = dict(h=FAKE, W=FAKE, dtype=kd.KD_DTYPE_BF16, T=256, d=256, V=4096, vals=FAKE, idx=FAKE,
             K=16, chunk=64, tau=1.0, loss=FAKE, lse=FAKE, kl=None, stream=None)
    a.update(kw)
    return kd.kd_fused_kl_fwd_noalloc(a["h"], a["W"], a["dtype"], a["T"], a["d"], a["V"], a["vals"],
                                      a["idx"], a["K"], a["chunk"], a["tau"], a["loss"], a["lse"],
                                      a["kl"], a["stream"])


def test_noalloc_validation_matches_the_workspace_forward(lib):
    """The entry point without a workspace checks its arguments with the same
    routine as kd_fused_kl_fwd: same ranges, same status codes, before any CUDA
    call (so these run without a GPU)."""
    for kw, want in [
        (dict(h=None), kd.KD_ERR_INVALID_ARG),
        (dict(lse=None), kd.KD_ERR_INVALID_ARG),
        (dict(loss=None), kd.KD_ERR_INVALID_ARG),
        (dict(T=0), kd.KD_ERR_INVALID_ARG),
        (dict(K=4097), kd.KD_ERR_INVALID_ARG),
        (dict(tau=float("nan")), kd.KD_ERR_INVALID_ARG),
        (dict(h=FAKE + 8), kd.KD_ERR_INVALID_ARG),
        (dict(kl=FAKE + 4), kd.KD_ERR_INVALID_ARG),
        (dict(dtype=7), kd.KD_ERR_UNSUPPORTED),
        (dict(d=12), kd.KD_ERR_UNSUPPORTED),
        (dict(K=1025), kd.KD_ERR_UNSUPPORTED),
        (dict(V=(1 << 31) - 200), kd.KD_ERR_UNSUPPORTED),
        (dict(T=1 << 40), kd.KD_ERR_UNSUPPORTED),
        (dict(T=1 << 62, K=4), kd.KD_ERR_UNSUPPORTED),   # T*K*4 etc. would wrap in size_t
        (dict(T=1 << 31, chunk=1 << 31), kd.KD_ERR_UNSUPPORTED),  # chunk rows above 2^30
    ]:
        assert _fwd_noalloc(**kw) == want, kw
        if "kl" not in kw and "loss" not in kw and "lse" not in kw:
            assert _fwd(**{k: v for k, v in kw.items()}) == want, kw


def test_noalloc_rejects_what_does_not_fit(lib):
    # 2^20 positions x K=100: 800 MB of sorted cache, far above the 64 MiB array
    assert _fwd_noalloc(T=1 << 20, K=100, V=131072) == kd.KD_ERR_WORKSPACE
    # the largest T under 2^40 with K = 1024 still needs more than the array
    assert _fwd_noalloc(T=(1 << 40) - 1, K=1024, V=131072) == kd.KD_ERR_WORKSPACE


def test_workspace_size_reports_zero_when_it_cannot_be_represented(lib):
    # four fp32 dH partials of 2^30 chunk rows x d ~ 2^31: 2^65 bytes
    d = (1 << 31) - 8
    assert kd.kd_fused_kl_workspace_size(1 << 30, d, 4096, 1, 1 << 30, kd.KD_DTYPE_F32) == 0
    # and the fused calls reject that size with KD_ERR_WORKSPACE, never a wrapped size
    assert _fwd(T=1 << 30, d=d, V=4096, K=1, chunk=1 << 30, dtype=kd.KD_DTYPE_F32,
                ws_bytes=(1 << 64) - 1) == kd.KD_ERR_WORKSPACE
    assert _bwd(T=1 << 30, d=d, V=4096, K=1, chunk=1 << 30, dtype=kd.KD_DTYPE_F32,
                ws_bytes=(1 << 64) - 1) == kd.KD_ERR_WORKSPACE


def _fwd_shard(**kw):
    a = dict(h=FAKE, W=FAKE, dtype=kd.KD_DTYPE_BF16, T=256, d=256, V=4096, vals=FAKE, idx=FAKE,
             K=16, chunk=64, tau=1.0, flags=0, T_total=512, loss=FAKE, lse=FAKE, kl=None, ws=FAKE,
             ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return kd.kd_fused_kl_fwd_shard(a["h"], a["W"], a["dtype"], a["T"], a["d"], a["V"], a["vals"],
                                    a["idx"], a["K"], a["chunk"], a["tau"], a["flags"], a["T_total"],
                                    a["loss"], a["lse"], a["kl"], a["ws"], a["ws_bytes"], a["stream"])


def _bwd_shard(**kw):
    a = dict(h=FAKE, W=FAKE, dtype=kd.KD_DTYPE_BF16, T=256, d=256, V=4096, vals=FAKE, idx=FAKE,
             K=16, chunk=64, tau=1.0, flags=0, T_total=512, lse=FAKE, g=None, dH=FAKE, dW=FAKE,
             acc=0, ws=FAKE, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return kd.kd_fused_kl_bwd_shard(a["h"], a["W"], a["dtype"], a["T"], a["d"], a["V"], a["vals"],
                                    a["idx"], a["K"], a["chunk"], a["tau"], a["flags"], a["T_total"],
                                    a["lse"], a["g"], a["dH"], a["dW"], a["acc"], a["ws"],
                                    a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("call", [_fwd_shard, _bwd_shard])
def test_shard_validation(lib, call):
    assert call(T_total=255) == kd.KD_ERR_INVALID_ARG        # fewer batch positions than rows
    assert call(T_total=0) == kd.KD_ERR_INVALID_ARG
    assert call(T_total=1 << 40) == kd.KD_ERR_UNSUPPORTED
    assert call(flags=0x80) == kd.KD_ERR_INVALID_ARG
    assert call(h=None) == kd.KD_ERR_INVALID_ARG             # the shared input checks
    assert call(K=1025) == kd.KD_ERR_UNSUPPORTED
    assert call(ws_bytes=16) == kd.KD_ERR_WORKSPACE
