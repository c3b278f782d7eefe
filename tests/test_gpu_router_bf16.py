"""The router's bf16-logit mode (shape.router_bf16_logits = 1): logits rounded to bf16
before scoring, as in a bf16 load of the model; equal rounded logits go to the lower
expert. On inputs whose logits sit away from bf16 rounding half-way points, the GPU's
rounded logits and the routing are bit-exact against the oracle."""
import numpy as np
import pytest

from oracle import moe_oracle as O
from sparse_mixture_experts_09_b200 import moe as M
from sparse_mixture_experts_09_b200 import workloads as W

from ._cases import W_ABS, assert_layer_close, decision_window, screened_bf16_logits, to_cpu
from .test_gpu_kernels import SMALL

pytestmark = pytest.mark.gpu

CASES = {"tiny": W.WORKLOADS["tiny"], "ragged": SMALL["ragged"], "e64k8": SMALL["e64k8"],
         "decode": W.WORKLOADS["decode"], "prefill": W.WORKLOADS["prefill"]}


@pytest.mark.parametrize("name", list(CASES))
def test_bf16_logit_router_is_bit_exact(name):
    w = CASES[name]
    inp, bad = screened_bf16_logits(w)
    assert bad.numel() == 0
    k = w.num_experts_per_tok
    idx, wt, logits = M.router_topk(inp.x, inp.w_router, k, return_logits=True,
                                    router_bf16_logits=True)
    c = to_cpu(inp)
    ref_logits = O.router_logits(c.x, c.w_router, bf16_logits=True)
    ref_idx, ref_w, _ = O.route_topk(ref_logits, k)
    got = logits.cpu().double().numpy()
    # logits that decide the routing round identically; the rest within one bf16 step
    win = decision_window(O.router_logits(c.x, c.w_router), k)
    assert np.array_equal(got[win], ref_logits[win])
    step = np.ldexp(1.0, np.frexp(np.abs(ref_logits) + 1e-30)[1] - 8)
    assert np.all(np.abs(got - ref_logits) <= step)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert np.abs(wt.cpu().double().numpy() - ref_w).max() <= W_ABS
    ties = (np.diff(-np.sort(-ref_logits, axis=1)[:, :k + 1], axis=1) == 0).any(axis=1).sum()
    print(f"{name}: {ties} tokens with tied bf16 logits among the top {k + 1}")


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_bf16_logit_layer_matches_oracle(name):
    w = CASES[name]
    inp, bad = screened_bf16_logits(w)
    assert bad.numel() == 0
    out = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, 2, router_bf16_logits=True)
    c = to_cpu(inp)
    ref = O.moe_layer(c.x, c.w_router, c.w1, c.w3, c.w2, 2, mode="bf16_storage", bf16_logits=True)
    assert_layer_close(O.to_f64(out.cpu()), ref["out"], name)
