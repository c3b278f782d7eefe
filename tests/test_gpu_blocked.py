"""Expert weights in the blocked layout (MOE_WEIGHTS_BLOCKED): moe_pack_weights'
reordering, and the layer run on packed weights equals the layer on row-major
weights bit for bit (same arithmetic, only the addresses of the weight tiles
change), including the CTA-pair down GEMM and the last-wave pieces."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_09_b200 import moe as M
from sparse_mixture_experts_09_b200 import workloads as W

from ._cases import assert_layer_close, sample_tokens, screened, to_cpu
from .test_gpu_kernels import SMALL

pytestmark = pytest.mark.gpu


def _blocked_reference(t):
    # [E, R, K] -> [E*R/128, K/64, 128, 64]: a 128 x 64 tile is contiguous
    e, r, k = t.shape
    return t.reshape(e * r // 128, 128, k // 64, 64).permute(0, 2, 1, 3).contiguous().reshape(e, r, k)


def test_pack_weights_matches_reordering():
    w = SMALL["ragged"]
    _, w1, w3, w2 = W.draw_weights(w, "cuda")
    p1, p3, p2 = M.pack_weights(w1, w3, w2)
    torch.cuda.synchronize()
    for got, src in ((p1, w1), (p3, w3), (p2, w2)):
        assert torch.equal(got, _blocked_reference(src))


@pytest.mark.parametrize("name", ["tiny", "ragged", "e5k3", "k32_waves", "bn128_split", "pair_down"])
def test_blocked_layer_equals_row_major_layer(name):
    w = SMALL[name]
    inp, _ = screened(w)
    k = w.num_experts_per_tok
    ref = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, k, residual=inp.residual,
                    logit_bias=inp.logit_bias)
    p1, p3, p2 = M.pack_weights(inp.w1, inp.w3, inp.w2)
    got = M.forward(inp.x, inp.w_router, p1, p3, p2, k, residual=inp.residual,
                    logit_bias=inp.logit_bias, weight_layout=M.BLOCKED)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_blocked_full_size_against_oracle(name):
    w = W.WORKLOADS[name]
    inp, near = screened(w)
    assert near.numel() == 0
    p1, p3, p2 = M.pack_weights(inp.w1, inp.w3, inp.w2)
    out = M.forward(inp.x, inp.w_router, p1, p3, p2, 2, weight_layout=M.BLOCKED)
    torch.cuda.synchronize()
    tokens = sample_tokens(w.num_tokens)
    c = to_cpu(inp)
    ref = O.moe_layer(c.x, c.w_router, c.w1, c.w3, c.w2, 2, mode="bf16_storage", tokens=tokens)
    assert_layer_close(O.to_f64(out.cpu())[tokens], ref["out"], name)
