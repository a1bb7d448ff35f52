"""Helpers shared by the GPU tests (no method arithmetic here)."""

import numpy as np
import torch


def to_np_exact(t: torch.Tensor) -> np.ndarray:
    """Host copy holding the exact bytes the GPU used (bf16 -> uint16 bits)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def rel_maxabs(got, ref) -> float:
    """max |got - ref| / max |ref|  (the gradient parity measure)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-300))


def require_gpu():
    import pytest
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from chunked_kl_loss_chunk_b200 import build, kd
    build.build()
    kd.load()
    major, minor = torch.cuda.get_device_capability()
    assert (major, minor) == (10, 0), f"library is built for sm_100a, device is sm_{major}{minor}"
