"""The mixture half of the decoder block on the GPU (moe_forward_rmsnorm): RMSNorm
fused into the router and the gather, the layer, and the residual add, against the
oracle's moe_block on the same seeded inputs (nnterp "Mixtral", "The block, in
order": out = h + mlp(post_attention_layernorm(h)))."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from oracle.screen import screen_margin
from sparse_mixture_experts_09_b200 import moe as M
from sparse_mixture_experts_09_b200 import workloads as W

from ._cases import assert_layer_close, sample_tokens

pytestmark = pytest.mark.gpu

EPS = W.RMS_NORM_EPS

CASES = {
    "tiny": W.WORKLOADS["tiny"],                                        # 8 warps per token
    "t1000": W.Workload("t1000", 1000, 384, 640, 8, 2, seed=21),        # 8 warps per token
    "t3000": W.Workload("t3000", 3000, 256, 256, 8, 2, seed=22),        # 2 warps per token
    "t6000": W.Workload("t6000", 6000, 256, 256, 8, 2, seed=23),        # 1 warp per token
    "decode": W.WORKLOADS["decode"],
}


def _screened_block(w):
    wr, w1, w3, w2 = W.draw_weights(w, "cuda")
    g = W.draw_norm_weight(w)
    h = W.draw_x(w, "cpu")
    wr_c = wr.cpu()
    prep = lambda rows: O.round_bf16(O.rms_norm(rows, g, EPS))  # noqa: E731
    h, _, near = screen_margin(h, wr_c, None, w.num_experts_per_tok,
                               lambda rows, a: W.redraw_x_rows(w, rows, a), prep=prep)
    return h, g, wr, w1, w3, w2, near


@pytest.mark.parametrize("name", list(CASES))
def test_block_matches_oracle(name):
    w = CASES[name]
    h, g, wr, w1, w3, w2, near = _screened_block(w)
    assert near.numel() == 0
    out = M.forward_rmsnorm(h.cuda(), g.cuda(), EPS, wr, w1, w3, w2, w.num_experts_per_tok)
    torch.cuda.synchronize()
    tokens = sample_tokens(w.num_tokens, 512)
    ref = O.moe_block(h, g, EPS, wr.cpu(), w1.cpu(), w3.cpu(), w2.cpu(), w.num_experts_per_tok,
                      mode="bf16_storage", tokens=tokens)
    got = O.to_f64(out.cpu())[tokens]
    assert_layer_close(got, ref["out"], name)
    # the routed part alone, against the oracle's routed output (the bf16 rounding of
    # the sum bounds the difference by one bf16 step of |out|)
    routed_gpu = got - O.to_f64(h)[tokens]
    err = np.abs(routed_gpu - ref["routed"])
    assert np.all(err <= 2.0 ** -8 * np.abs(ref["out"]) + 1e-3 * np.abs(ref["routed"]).max())


def test_block_without_norm_gain_change_equals_layer_on_normed_input():
    # with gain 1 and the normed rows fed to the plain layer, both entry points agree
    w = CASES["t1000"]
    h, _, wr, w1, w3, w2, _ = _screened_block(w)
    ones = torch.ones(w.hidden_size, dtype=torch.bfloat16)
    out = M.forward_rmsnorm(h.cuda(), ones.cuda(), EPS, wr, w1, w3, w2, 2)
    xn = torch.from_numpy(O.round_bf16(O.rms_norm(h, ones, EPS))).to(torch.bfloat16)
    lay = M.forward(xn.cuda(), wr, w1, w3, w2, 2, residual=h.cuda())
    torch.cuda.synchronize()
    # the two differ only where the GPU's fp32 norm and the fp64 one round apart
    diff = (O.to_f64(out.cpu()) - O.to_f64(lay.cpu()))
    assert np.abs(diff).max() <= 0.05 and np.mean(diff != 0) < 0.2
