"""The library allocates nothing and never synchronises inside a call, so a
whole step (top-K cache build, fused forward, fused backward) can be captured
in one CUDA graph.  Replays must match eager execution bit for bit, also after
new inputs are copied into the captured buffers."""

import pytest
import torch

from chunked_kl_loss_chunk_b200 import inputs, kd
from gpu_util import require_gpu

pytestmark = pytest.mark.gpu


def _buffers(T, d, V, K, seed):
    h, W, _, _ = inputs.make_loss_inputs(T, d, V, 1, dtype=torch.bfloat16, seed=seed, device="cuda")
    x = inputs.make_teacher_logits(T, V, seed=seed, device="cuda")
    return h, W, x


def test_step_captured_in_one_cuda_graph():
    require_gpu()
    T, d, V, K, chunk = 600, 256, 5000, 32, 256
    h, W, x = _buffers(T, d, V, K, seed=11)
    vals = torch.empty((T, K), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    ws_topk = kd.alloc_workspace(kd.kd_topk_workspace_size(T, V, K), h.device)
    ws = kd.workspace_for(h, W, K, chunk)
    loss = torch.empty((), dtype=torch.float32, device="cuda")
    lse = torch.empty((T,), dtype=torch.float32, device="cuda")
    dH = torch.empty_like(h)
    dW = torch.empty((V, d), dtype=torch.float32, device="cuda")
    code = kd.KD_DTYPE_BF16

    def step(stream):
        s = stream.cuda_stream
        st = kd.kd_topk_build(x.data_ptr(), code, T, V, K, vals.data_ptr(), idx.data_ptr(),
                              ws_topk.data_ptr(), ws_topk.numel(), s)
        st |= kd.kd_fused_kl_fwd(h.data_ptr(), W.data_ptr(), code, T, d, V, vals.data_ptr(),
                                 idx.data_ptr(), K, chunk, 1.0, loss.data_ptr(), lse.data_ptr(),
                                 None, ws.data_ptr(), ws.numel(), s)
        st |= kd.kd_fused_kl_bwd(h.data_ptr(), W.data_ptr(), code, T, d, V, vals.data_ptr(),
                                 idx.data_ptr(), K, chunk, 1.0, lse.data_ptr(), None,
                                 dH.data_ptr(), dW.data_ptr(), 0, ws.data_ptr(), ws.numel(), s)
        assert st == kd.KD_OK

    def snapshot():
        return [t.clone() for t in (vals, idx, loss, lse, dH, dW)]

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step(side)                                   # eager, also warms up
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = snapshot()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(torch.cuda.current_stream())
    n0 = kd.kd_launch_count()
    g.replay()
    torch.cuda.synchronize()
    assert kd.kd_launch_count() == n0                 # a replay launches from the graph only
    assert kd.read_device_status(ws) == kd.KD_OK
    for a, b in zip(snapshot(), eager):
        assert torch.equal(a, b)

    # new inputs in the same buffers: replay == eager on them
    h2, W2, x2 = _buffers(T, d, V, K, seed=12)
    h.copy_(h2)
    W.copy_(W2)
    x.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    replayed = snapshot()
    step(torch.cuda.current_stream())
    torch.cuda.synchronize()
    for a, b in zip(replayed, snapshot()):
        assert torch.equal(a, b)
    assert not torch.equal(replayed[5], eager[5])     # the inputs did change
