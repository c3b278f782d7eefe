"""Failure detection without a GPU fault: a bounded wait that nothing completes must
give up, be reported as MOE_ERR_TIMEOUT through the workspace status word, and leave
the context usable for the next layer."""
import time

import pytest
import torch

from sparse_mixture_experts_09_b200 import moe as M
from sparse_mixture_experts_09_b200 import workloads as W

from ._cases import assert_layer_close, screened, to_cpu

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_survives():
    w = W.WORKLOADS["tiny"]
    ws = M.make_workspace(M.make_shape(*w.shape))
    M.device_status(ws)                          # clean to start with
    t0 = time.perf_counter()
    M.selftest_wait_timeout(ws, 50_000_000)      # 50 ms
    with pytest.raises(M.MoeError) as err:
        M.device_status(ws)                      # waits for the stream, reads the word
    assert err.value.status == 5                 # MOE_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 10.0
    M.device_status(ws)                          # the word was cleared
    # the same context still runs the layer correctly
    from oracle import moe_oracle as O
    inp, _ = screened(w)
    out = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, 2, ws=ws)
    M.device_status(ws)
    c = to_cpu(inp)
    ref = O.moe_layer(c.x, c.w_router, c.w1, c.w3, c.w2, 2, mode="bf16_storage")
    assert_layer_close(O.to_f64(out.cpu()), ref["out"])
    torch.cuda.synchronize()
