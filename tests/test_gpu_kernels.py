"""Per-step GPU parity through the C ABI: router, permutation, grouped GEMMs, combine.

Every expected value comes from the fp64 oracle on the same seeded inputs.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_09_b200 import moe as M
from sparse_mixture_experts_09_b200 import workloads as W

from ._cases import W_ABS, assert_layer_close, screened, to_cpu

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": W.WORKLOADS["tiny"],
    "ragged": W.Workload("ragged", 1000, 384, 640, 8, 2, seed=11),
    "e5k3": W.Workload("e5k3", 777, 256, 256, 5, 3, seed=12),
    "e64k8": W.Workload("e64k8", 100, 128, 128, 64, 8, seed=13),
    "one_token": W.Workload("one_token", 1, 128, 256, 8, 2, seed=14),
    "skewed": W.Workload("skewed", 2000, 256, 256, 8, 2, seed=15,
                         logit_bias=(3.0, 0, 0, 0, 0, 0, -2.0, -2.0)),
    # deeper K (16 and 32 k-blocks), one row tile per expert (k16) and several row
    # tiles per expert with more than five waves of tiles (k32_waves)
    "k16": W.Workload("k16", 300, 1024, 1024, 8, 2, seed=17),
    "k32_waves": W.Workload("k32_waves", 3000, 1024, 2048, 8, 2, seed=18),
    # hidden 640: the down GEMM uses 128-column tiles, and its last wave is cut
    # into 32-column pieces
    "bn128_split": W.Workload("bn128_split", 4000, 640, 512, 8, 2, seed=19),
    # at least 1024 routed rows per expert: the down GEMM runs on CTA pairs
    # (tcgen05 cta_group::2), experts with odd and even row-tile counts
    "pair_down": W.Workload("pair_down", 4500, 512, 512, 8, 2, seed=20),
}


@pytest.fixture(scope="module", params=list(SMALL))
def case(request):
    w = SMALL[request.param]
    inp, near = screened(w)
    return w, inp, near


def test_router_matches_oracle(case):
    w, inp, near = case
    assert near.numel() == 0
    idx, wt, logits = M.router_topk(inp.x, inp.w_router, w.num_experts_per_tok, inp.logit_bias,
                                    return_logits=True)
    c = to_cpu(inp)
    ref_logits = O.router_logits(c.x, c.w_router, c.logit_bias)
    ref_idx, ref_w, _ = O.route_topk(ref_logits, w.num_experts_per_tok)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert np.abs(wt.cpu().double().numpy() - ref_w).max() <= W_ABS
    assert np.abs(wt.cpu().double().numpy().sum(1) - 1).max() <= 2 ** -22
    # fp32 accumulation of H products against the exact fp64 sum
    bound = 1e-5 * (np.abs(O.to_f64(c.x)) @ np.abs(O.to_f64(c.w_router)).T) + 1e-6
    assert np.all(np.abs(logits.cpu().double().numpy() - ref_logits) <= bound)


def test_permute_matches_oracle(case):
    w, inp, _ = case
    c = to_cpu(inp)
    ref_idx, _, _ = O.route_topk(O.router_logits(c.x, c.w_router, c.logit_bias), w.num_experts_per_tok)
    shape = M.make_shape(*w.shape)
    ws = M.make_workspace(shape)
    got = M.permute(torch.from_numpy(ref_idx).cuda(), inp.x, w.num_experts, w.intermediate_size, ws)
    count, offset, row_of, tok = O.stable_permute(ref_idx, w.num_experts)
    assert np.array_equal(got["counts"].cpu().numpy(), count)
    assert np.array_equal(got["offsets"].cpu().numpy(), offset)
    assert np.array_equal(got["row_of"].cpu().numpy(), row_of)
    r = int(offset[-1])
    assert np.array_equal(got["token_of_row"][:r].cpu().numpy(), tok)
    assert torch.all(got["token_of_row"][r:] == -2)          # untouched past R_pad
    xp = got["x_perm"][:r].cpu()
    real = torch.from_numpy(tok >= 0)
    assert torch.equal(xp[real], c.x[torch.from_numpy(tok[tok >= 0])])
    assert torch.all(xp[~real] == 0)


def test_grouped_swiglu_matches_oracle(case):
    w, inp, _ = case
    c = to_cpu(inp)
    k = w.num_experts_per_tok
    ref = O.moe_layer(c.x, c.w_router, c.w1, c.w3, c.w2, k, logit_bias=c.logit_bias, mode="bf16_storage")
    shape = M.make_shape(*w.shape)
    ws = M.make_workspace(shape)
    p = M.permute(torch.from_numpy(ref["idx"]).cuda(), inp.x, w.num_experts, w.intermediate_size, ws)
    y = M.grouped_swiglu(p["x_perm"], p["offsets"], inp.w1, inp.w3, inp.w2, w.num_tokens, k, ws)
    M.device_status(ws)
    row_of = p["row_of"].cpu().numpy().astype(np.int64)
    got = y.cpu().double().numpy()[row_of]                  # [T, k, H]
    assert_layer_close(got, ref["y"], "y")
    # pad rows hold zero activations, so their outputs are exactly zero
    tok = p["token_of_row"][: int(p["offsets"][-1])].cpu().numpy()
    assert np.all(y.cpu().numpy()[: tok.size][tok < 0] == 0)


def test_combine_matches_fp64_definition(case):
    w, inp, _ = case
    c = to_cpu(inp)
    k = w.num_experts_per_tok
    ref_idx, ref_w, _ = O.route_topk(O.router_logits(c.x, c.w_router, c.logit_bias), k)
    _, offset, row_of, _ = O.stable_permute(ref_idx, w.num_experts)
    g = torch.Generator().manual_seed(5)
    rmax = int(M.max_padded_rows(M.make_shape(*w.shape)))
    y = torch.randn(rmax, w.hidden_size, generator=g, dtype=torch.float32)
    wt = torch.from_numpy(ref_w.astype(np.float32))
    ro = torch.from_numpy(row_of.astype(np.int32))
    for residual in (None, c.residual):
        out = M.combine(y.cuda(), ro.cuda(), wt.cuda(), None if residual is None else residual.cuda(),
                        w.num_experts, w.intermediate_size)
        yd = y.double().numpy()[row_of]                     # [T, k, H]
        terms = wt.double().numpy()[:, :, None] * yd
        exact = terms.sum(1)
        mag = np.abs(terms).sum(1)
        if residual is not None:
            exact = exact + O.to_f64(residual)
            mag = mag + np.abs(O.to_f64(residual))
        want = O.round_bf16(exact)
        got = O.to_f64(out.cpu())
        # the fp32 sum (k + 1 roundings of at most 2^-24 of the running magnitude) can
        # move the value across a bf16 rounding boundary: one bf16 step of the result
        # plus the fp32 error, and rarely
        ulp = np.ldexp(1.0, np.frexp(np.abs(want) + 1e-30)[1] - 8)
        assert np.all(np.abs(got - want) <= ulp + (k + 2) * 2.0 ** -24 * mag)
        assert np.mean(got != want) < 5e-3
