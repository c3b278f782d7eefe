"""The layer inside a CUDA graph: moe_forward (and the int8 layer) are captured once
and replayed; every replay equals an eager call on the same inputs bit for bit,
including after new activations are copied into the captured input buffers. The
library launches only on the caller's stream, allocates nothing and never
synchronises inside these entry points, which is what capture requires."""
import pytest
import torch

from sparse_mixture_experts_09_b200 import moe as M
from sparse_mixture_experts_09_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _capture(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):          # first calls set kernel attributes outside the capture
            fn()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        fn()
    return graph


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_forward_graph_replay_equals_eager(name):
    w = W.WORKLOADS[name]
    inp = W.draw(w, "cuda")
    k = w.num_experts_per_tok
    shape = M.make_shape(*w.shape)
    ws = M.make_workspace(shape)
    x = inp.x.clone()
    out = torch.empty_like(x)

    def fn():
        M.forward(x, inp.w_router, inp.w1, inp.w3, inp.w2, k, residual=inp.residual, ws=ws, out=out)

    graph = _capture(fn)
    for attempt in range(2):
        if attempt:
            x.copy_(W.redraw_x_rows(w, torch.arange(w.num_tokens), 1).to(x.device))
        graph.replay()
        torch.cuda.synchronize()
        want = M.forward(x, inp.w_router, inp.w1, inp.w3, inp.w2, k, residual=inp.residual)
        torch.cuda.synchronize()
        assert torch.equal(out, want)
    M.device_status(ws)


def test_int8_forward_graph_replay_equals_eager():
    w = W.WORKLOADS["decode"]
    inp = W.draw(w, "cuda")
    q = M.quantize_int8(inp.w1, inp.w3, inp.w2)
    ws = M.make_workspace(M.make_shape(*w.shape))
    out = torch.empty_like(inp.x)

    def fn():
        M.forward_w8(inp.x, inp.w_router, q, 2, residual=inp.residual, ws=ws, out=out)

    graph = _capture(fn)
    graph.replay()
    torch.cuda.synchronize()
    want = M.forward_w8(inp.x, inp.w_router, q, 2, residual=inp.residual)
    torch.cuda.synchronize()
    assert torch.equal(out, want)
