"""Whole-layer GPU parity through the C ABI (moe_forward), in the benchmark's launch
configuration, against the fp64 oracle; plus the invariants the nnterp "Mixtral"
page states for the layer, checked on the GPU."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_09_b200 import moe as M
from sparse_mixture_experts_09_b200 import workloads as W

from ._cases import assert_layer_close, layer_errors, sample_tokens, screened, to_cpu
from .test_gpu_kernels import SMALL

pytestmark = pytest.mark.gpu

SINGLE_EXPERT = W.Workload("single_expert", 200, 128, 256, 1, 1, seed=16)


def _forward_and_check(w, inp, tokens=None, residual=True):
    res = inp.residual if residual else None
    shape = M.make_shape(*w.shape)
    ws = M.make_workspace(shape)
    out = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, w.num_experts_per_tok,
                    residual=res, logit_bias=inp.logit_bias, ws=ws)
    M.device_status(ws)
    c = to_cpu(inp)
    ref = O.moe_layer(c.x, c.w_router, c.w1, c.w3, c.w2, w.num_experts_per_tok,
                      residual=None if res is None else c.residual, logit_bias=c.logit_bias,
                      mode="bf16_storage", tokens=tokens)
    got = O.to_f64(out.cpu())
    if tokens is not None:
        got = got[tokens]
    return got, ref, out


@pytest.mark.parametrize("name", list(SMALL) + ["single_expert"])
def test_forward_small(name):
    w = SINGLE_EXPERT if name == "single_expert" else SMALL[name]
    inp, near = screened(w)
    assert near.numel() == 0
    # the gate is on the routed output (no residual), which a unit-RMS residual would mask
    got, ref, _ = _forward_and_check(w, inp, residual=False)
    assert_layer_close(got, ref["out"], name)
    got, ref, _ = _forward_and_check(w, inp, residual=True)
    assert_layer_close(got, ref["out"], name + "+residual")


# At most 256 tokens the bf16 layer runs both expert GEMMs as one swap-operand kernel:
# 16-, 32- and 64-row sub-tiles up to 64 tokens (7, 17, 24, 48, 50 and 64 tokens; N = 32
# and 48 on 2 experts at 24 and 48 tokens; E = 64 with k = 8; a hidden size that is not
# a multiple of 256), 64-row sub-tiles above that while experts average at most 56 rows
# (160 tokens with one expert holding 155 rows: sub-tiles of 64, 64 and 27; 96 tokens
# with one at 66), else 128-row sub-tiles (65 tokens on 2 experts: N = 80; 200 tokens on
# 2 experts: 128 and 72 rows, an intermediate size that is not a multiple of 256; 256
# tokens on 8 experts).
SWAP_128 = {
    "t200_e2": W.Workload("t200_e2", 200, 256, 384, 2, 2, seed=43),
    "t256_e8": W.Workload("t256_e8", 256, 512, 768, 8, 2, seed=44),
}


@pytest.mark.parametrize("name", ["ts_k1", "t17_e4", "t24_e2", "t48_e2", "ts_e64k8", "ts_h640",
                                  "t64_edge", "t160_skew", "t96_e4", "t65_edge", "t200_e2",
                                  "t256_e8"])
def test_forward_swap_operand_widths(name):
    from .test_gpu_w8 import SMALL_BATCH
    w = SWAP_128[name] if name in SWAP_128 else SMALL_BATCH[name]
    inp, near = screened(w)
    assert near.numel() == 0
    for residual in (False, True):
        got, ref, _ = _forward_and_check(w, inp, residual=residual)
        assert_layer_close(got, ref["out"], f"{name} residual={residual}")


def test_single_expert_is_plain_swiglu():
    # E = 1, k = 1: the layer is w2 (silu(w1 x) * w3 x), checked here against torch's
    # own fp64 F.linear / F.silu on the same bf16 values
    import torch.nn.functional as F
    w = SINGLE_EXPERT
    inp, _ = screened(w)
    got, _, _ = _forward_and_check(w, inp, residual=False)
    c = to_cpu(inp)
    x = c.x.double()
    want = F.linear(F.silu(F.linear(x, c.w1[0].double())) * F.linear(x, c.w3[0].double()),
                    c.w2[0].double()).numpy()
    max_rel, mae = layer_errors(got, want)
    assert max_rel <= 2e-2 and mae <= 5e-3       # h rounded to bf16 on the GPU, not in `want`


def test_forward_is_deterministic_and_host_entry_matches():
    w = SMALL["ragged"]
    inp, _ = screened(w)
    a = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, 2, residual=inp.residual)
    b = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, 2, residual=inp.residual)
    assert torch.equal(a, b)
    xh = inp.x.cpu().pin_memory()
    rh = inp.residual.cpu().pin_memory()
    h = M.forward_host(xh, inp.w_router, inp.w1, inp.w3, inp.w2, 2, residual_host=rh)
    assert torch.equal(h, a.cpu())


def test_ablating_an_expert_changes_exactly_its_tokens():
    # nnterp "Mixtral", "Ablating an expert": zero expert e's weight where it was chosen;
    # the output changes on exactly the tokens that chose e.
    w = SMALL["ragged"]
    inp, _ = screened(w)
    shape = M.make_shape(*w.shape)
    ws = M.make_workspace(shape)
    idx, wt = M.router_topk(inp.x, inp.w_router, 2)
    p = M.permute(idx, inp.x, w.num_experts, w.intermediate_size, ws)
    y = M.grouped_swiglu(p["x_perm"], p["offsets"], inp.w1, inp.w3, inp.w2, w.num_tokens, 2, ws)
    clean = M.combine(y, p["row_of"], wt, inp.residual, w.num_experts, w.intermediate_size)
    for e in (0, 3, 7):
        abl_w = wt.masked_fill(idx == e, 0.0)
        ablated = M.combine(y, p["row_of"], abl_w, inp.residual, w.num_experts, w.intermediate_size)
        changed = (ablated != clean).any(-1)
        assert torch.equal(changed, (idx == e).any(-1))


@pytest.mark.parametrize("name", ["decode", "prefill", "imbalanced_a", "imbalanced_b", "larger"])
def test_forward_full_size(name):
    w = W.WORKLOADS[name]
    inp, near = screened(w)
    assert near.numel() <= max(1, w.num_tokens // 1000)
    c = to_cpu(inp)
    # routing of every token, bit-exact
    idx, wt = M.router_topk(inp.x, inp.w_router, 2, inp.logit_bias)
    ref_idx, ref_w, _ = O.route_topk(O.router_logits(c.x, c.w_router, c.logit_bias), 2)
    ok = np.ones(w.num_tokens, dtype=bool)
    ok[near.numpy()] = False
    assert np.array_equal(idx.cpu().numpy()[ok], ref_idx[ok])
    # counts, padded offsets and the permutation, bit-exact against the oracle's
    # counting sort. With no near-tie rows the GPU's indices are the oracle's, so this is
    # the oracle's permutation of the oracle's routing; a near-tie row (at most one per
    # thousand tokens) may go either way, and then the oracle permutes the GPU's choice.
    gpu_idx = idx.cpu().numpy()
    if near.numel() == 0:
        assert np.array_equal(gpu_idx, ref_idx)
    count, offset, row_of, tok = O.stable_permute(gpu_idx, w.num_experts)
    ws = M.make_workspace(M.make_shape(*w.shape))
    p = M.permute(idx, inp.x, w.num_experts, w.intermediate_size, ws)
    M.device_status(ws)
    assert np.array_equal(p["counts"].cpu().numpy(), count)
    assert np.array_equal(p["offsets"].cpu().numpy(), offset)
    assert np.array_equal(p["row_of"].cpu().numpy(), row_of)
    n_rows = int(offset[-1])
    assert np.array_equal(p["token_of_row"][:n_rows].cpu().numpy(), tok)
    # the gathered rows: x_perm[row] = x[token], pad rows zero
    tok_d = p["token_of_row"][:n_rows].long()
    real = tok_d >= 0
    assert torch.equal(p["x_perm"][:n_rows][real], inp.x[tok_d[real]])
    assert not p["x_perm"][:n_rows][~real].any()
    if w.logit_bias is not None:
        assert count[0] > 0.4 * count.sum()          # about half the slots go to expert 0
    # outputs on sampled tokens (all tokens when T <= 256)
    tokens = sample_tokens(w.num_tokens)
    got, ref, _ = _forward_and_check(w, inp, tokens=tokens, residual=False)
    assert_layer_close(got, ref["out"], name)


@pytest.mark.parametrize("t", W.DECODE_SWEEP_TOKENS)
def test_forward_decode_sweep(t):
    w = W.WORKLOADS["larger"].with_tokens(t)
    inp, near = screened(w)
    assert near.numel() == 0
    got, ref, _ = _forward_and_check(w, inp, residual=False)
    assert_layer_close(got, ref["out"], w.name)


# Every token on experts 0 and 1 (bias +30): two experts with 3000 rows each (24 row
# tiles), six empty experts; the routing margin between the two is still screened.
ALL_ON_TWO = W.Workload("all_on_two", 3000, 256, 512, 8, 2, seed=41,
                        logit_bias=(30.0, 30.0, 0, 0, 0, 0, 0, 0))
# 100k tokens: the multi-block histogram / scan / rank path with 3125 token blocks
MANY_TOKENS = W.Workload("many_tokens", 100_000, 128, 128, 8, 2, seed=42)


@pytest.mark.parametrize("w", [ALL_ON_TWO, MANY_TOKENS], ids=lambda w: w.name)
def test_forward_extreme_batches(w):
    inp, near = screened(w)
    assert near.numel() == 0
    tokens = sample_tokens(w.num_tokens, 512)
    got, ref, out = _forward_and_check(w, inp, tokens=tokens, residual=False)
    assert_layer_close(got, ref["out"], w.name)
    idx, _ = M.router_topk(inp.x, inp.w_router, 2, inp.logit_bias)
    counts = torch.bincount(idx.reshape(-1).long(), minlength=w.num_experts).cpu()
    if w is ALL_ON_TWO:
        assert counts[:2].tolist() == [w.num_tokens] * 2 and int(counts[2:].sum()) == 0
    assert int(counts.sum()) == 2 * w.num_tokens


def test_int8_extreme_imbalance():
    w = ALL_ON_TWO
    inp, _ = screened(w)
    q = M.quantize_int8(inp.w1, inp.w3, inp.w2)
    out = M.forward_w8(inp.x, inp.w_router, q, 2, logit_bias=inp.logit_bias)
    torch.cuda.synchronize()
    c = to_cpu(inp)
    deq = []
    for full in (c.w1, c.w3, c.w2):
        qq, s = O.quantize_int8_rows(full)
        deq.append(qq.astype(np.float64) * s.astype(np.float64)[..., None])
    tokens = sample_tokens(w.num_tokens, 512)
    ref = O.moe_layer(c.x, c.w_router, deq[0], deq[1], deq[2], 2, logit_bias=c.logit_bias,
                      mode="f16_experts", tokens=tokens)
    assert_layer_close(O.to_f64(out.cpu())[tokens], ref["out"], "int8 all_on_two")


def test_forward_host_async_steps_queue_on_one_stream():
    # three steps with different activations enqueued back to back on one stream and
    # one workspace, one wait at the end: each equals the device-resident forward
    w = SMALL["ragged"]
    inp, _ = screened(w)
    shape = M.make_shape(*w.shape)
    ws = M.make_workspace(shape, "cuda", host=True)
    xs = [W.redraw_x_rows(w, torch.arange(w.num_tokens), a).pin_memory() for a in (1, 2, 3)]
    rh = inp.residual.cpu().pin_memory()
    outs = [torch.empty_like(x).pin_memory() for x in xs]
    for x, o in zip(xs, outs):
        M.forward_host(x, inp.w_router, inp.w1, inp.w3, inp.w2, w.num_experts_per_tok,
                       residual_host=rh, ws=ws, out_host=o, wait=False)
    torch.cuda.synchronize()
    for x, o in zip(xs, outs):
        want = M.forward(x.cuda(), inp.w_router, inp.w1, inp.w3, inp.w2, w.num_experts_per_tok,
                         residual=inp.residual)
        assert torch.equal(o, want.cpu())


def test_forward_host_async_steps_of_different_sizes_share_a_workspace():
    # a serving loop whose batch size changes from step to step, enqueued back to back on
    # one stream and one workspace sized for the largest batch: every region of the
    # workspace moves with the batch size, so each step's copies in must not land on
    # memory the step before is still using. Each output equals the device forward.
    w = SMALL["ragged"]
    inp, _ = screened(w)
    t_max = w.num_tokens
    sizes = [t_max, 7, t_max // 2 + 3, t_max, 1, t_max, t_max - 5, 33]
    ws = M.make_workspace(M.make_shape(*w.shape), "cuda", host=True)
    xs = [W.redraw_x_rows(w, torch.arange(t), a + 1).pin_memory() for a, t in enumerate(sizes)]
    rs = [W.redraw_x_rows(w, torch.arange(t), a + 40).pin_memory() for a, t in enumerate(sizes)]
    outs = [torch.empty_like(x).pin_memory() for x in xs]
    for x, r, o in zip(xs, rs, outs):
        M.forward_host(x, inp.w_router, inp.w1, inp.w3, inp.w2, w.num_experts_per_tok,
                       residual_host=r, ws=ws, out_host=o, wait=False)
    torch.cuda.synchronize()
    M.device_status(ws)
    for x, r, o in zip(xs, rs, outs):
        want = M.forward(x.cuda(), inp.w_router, inp.w1, inp.w3, inp.w2, w.num_experts_per_tok,
                         residual=r.cuda())
        assert torch.equal(o, want.cpu())


# Few routed rows: the down GEMM's tiles do not fill the SMs, so moe_forward splits each
# tile's K range into parts (at least 8 k-blocks each) and the last part of a tile sums
# the parts in order. 8 parts; 3 uneven parts (26 k-blocks); 4 parts on 128-column tiles
# (a hidden size that is not a multiple of 256).
SPLIT_K = {
    "sk_t5": W.Workload("sk_t5", 5, 256, 4096, 8, 2, seed=51),
    "sk_uneven": W.Workload("sk_uneven", 3, 512, 1664, 8, 2, seed=52),
    "sk_h384": W.Workload("sk_h384", 7, 384, 2048, 4, 2, seed=53),
}


@pytest.mark.parametrize("name", list(SPLIT_K))
def test_split_k_down_gemm_matches_oracle_and_repeats_exactly(name):
    w = SPLIT_K[name]
    inp, near = screened(w)
    assert near.numel() == 0
    got, ref, out = _forward_and_check(w, inp, residual=False)
    assert_layer_close(got, ref["out"], name)
    # the parts are summed in a fixed order: a second call gives the same bits
    again = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, w.num_experts_per_tok,
                      logit_bias=inp.logit_bias)
    assert torch.equal(again, out)
    # against the unsplit GEMM (the split entry points do not split): within a rounding
    shape = M.make_shape(*w.shape)
    ws = M.make_workspace(shape)
    idx, wt = M.router_topk(inp.x, inp.w_router, w.num_experts_per_tok, inp.logit_bias)
    p = M.permute(idx, inp.x, w.num_experts, w.intermediate_size, ws)
    y = M.grouped_swiglu(p["x_perm"], p["offsets"], inp.w1, inp.w3, inp.w2, w.num_tokens,
                         w.num_experts_per_tok, ws)
    plain = M.combine(y, p["row_of"], wt, None, w.num_experts, w.intermediate_size)
    g, f = out.float(), plain.float()
    # one bf16 rounding step, or an fp32-sized difference where the output cancels to ~0
    tol = 2.0 ** -7 * torch.maximum(g.abs(), f.abs()) + 1e-5 * f.pow(2).mean().sqrt()
    assert ((g - f).abs() <= tol).all()
