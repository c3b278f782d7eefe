"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each check is independent of the oracle's own code path: closed forms, library
routines (torch's bf16 conversion, F.silu, F.linear), brute force over tiny inputs,
and the invariants the nnterp "Mixtral" page states for the layer.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import moe_oracle as O
from oracle.screen import min_gap, screen_margin
from sparse_mixture_experts_09_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_torch_on_float32_values():
    g = torch.Generator().manual_seed(0)
    a = torch.randn(200000, generator=g, dtype=torch.float32) * torch.exp(
        torch.randn(200000, generator=g) * 10)
    want = a.to(torch.bfloat16).double().numpy()
    got = O.round_bf16(a.double().numpy())
    assert np.array_equal(got, want)


def test_round_bf16_ties_to_even_closed_form():
    # 1 + 2^-8 is half-way between 1 and 1 + 2^-7 (bf16 spacing at 1 is 2^-7)
    assert O.round_bf16(1 + 2.0 ** -8) == 1.0
    assert O.round_bf16(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    assert O.round_bf16(-(1 + 3 * 2.0 ** -8)) == -(1 + 2.0 ** -6)
    # just above half-way rounds up
    assert O.round_bf16(1 + 2.0 ** -8 + 2.0 ** -30) == 1 + 2.0 ** -7
    # smallest bf16 subnormal is 2^-133
    assert O.round_bf16(2.0 ** -133 * 0.75) == 2.0 ** -133
    assert O.round_bf16(0.0) == 0.0


# ---------------------------------------------------------------- silu

def test_silu_closed_forms():
    l3 = math.log(3.0)
    # sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4
    assert O.silu(np.array([l3]))[0] == pytest.approx(0.75 * l3, rel=1e-15)
    assert O.silu(np.array([-l3]))[0] == pytest.approx(-0.25 * l3, rel=1e-15)
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert O.silu(np.array([800.0]))[0] == 800.0
    assert O.silu(np.array([-800.0]))[0] == 0.0


def test_silu_matches_torch():
    g = np.linspace(-30, 30, 10001)
    want = F.silu(torch.from_numpy(g)).numpy()
    assert np.allclose(O.silu(g), want, rtol=1e-14, atol=1e-300)


# ---------------------------------------------------------------- router

def test_router_logits_pick_columns():
    # x = unit vector e_h selects column h of W_r: logits[t, e] = W_r[e, h]
    rng = np.random.default_rng(0)
    wr = rng.standard_normal((5, 7))
    x = np.eye(7)[[3, 0, 6]]
    assert np.array_equal(O.router_logits(x, wr), wr[:, [3, 0, 6]].T)
    bias = np.arange(5.0)
    assert np.array_equal(O.router_logits(x, wr, bias), wr[:, [3, 0, 6]].T + bias)


def test_route_closed_form_example():
    # logits ln[1, 4, 2, 1]: softmax = [1, 4, 2, 1] / 8; top-2 = experts 1, 2;
    # renormalised weights 4/6 and 2/6.
    logits = np.log(np.array([[1.0, 4.0, 2.0, 1.0]]))
    idx, w, p = O.route_topk(logits, 2)
    assert idx.tolist() == [[1, 2]]
    assert np.allclose(p, [[1 / 8, 4 / 8, 2 / 8, 1 / 8]], rtol=1e-15)
    assert np.allclose(w, [[2 / 3, 1 / 3]], rtol=1e-15)


def test_route_weights_sum_to_one_and_match_two_logit_softmax():
    rng = np.random.default_rng(1)
    logits = rng.standard_normal((500, 8)) * 3
    idx, w, _ = O.route_topk(logits, 2)
    # "a token's weights are p and 1 - p"
    assert np.all(np.abs(w.sum(1) - 1) <= 1e-15)
    # softmax -> top-2 -> renormalise == softmax over the two selected logits
    l0 = np.take_along_axis(logits, idx.astype(np.int64)[:, :1], 1)[:, 0]
    l1 = np.take_along_axis(logits, idx.astype(np.int64)[:, 1:], 1)[:, 0]
    assert np.allclose(w[:, 0], 1 / (1 + np.exp(l1 - l0)), rtol=1e-14)
    assert np.all(w[:, 0] >= w[:, 1])


def test_route_brute_force_pair_search():
    # The top-2 set is the pair of experts with the largest total probability.
    rng = np.random.default_rng(2)
    logits = rng.standard_normal((200, 6)) * 2
    idx, _, p = O.route_topk(logits, 2)
    for t in range(200):
        best = max(itertools.combinations(range(6), 2), key=lambda ab: p[t, ab[0]] + p[t, ab[1]])
        assert set(idx[t].tolist()) == set(best)
        assert p[t, idx[t, 0]] >= p[t, idx[t, 1]]


def test_route_ties_to_lower_index_and_k1():
    idx, w, _ = O.route_topk(np.array([[0.5, 2.0, 2.0, 2.0]]), 2)
    assert idx.tolist() == [[1, 2]]
    assert np.allclose(w, [[0.5, 0.5]])
    idx1, w1, _ = O.route_topk(np.array([[0.1, 0.9, 0.3]]), 1)
    assert idx1.tolist() == [[1]] and w1.tolist() == [[1.0]]


def test_route_topk_ranks_float32_logits_ties_low():
    # the reading: the top-k decision is taken on the logits rounded to float32 and equal
    # float32 logits go to the lower expert index. 1 and 1 + 2**-30 differ in fp64 but
    # round to the same float32, so expert 0 wins; the weights still use fp64 logits.
    logits = np.array([[1.0, 1.0 + 2.0 ** -30, 0.5]])
    idx, w, p = O.route_topk(logits, 2)
    assert idx.tolist() == [[0, 1]]
    assert w[0, 0] < w[0, 1] and abs(w.sum() - 1.0) < 1e-15
    idx1, _, _ = O.route_topk(logits, 1)
    assert idx1.tolist() == [[0]]
    # a difference float32 keeps decides the order as usual
    idx2, _, _ = O.route_topk(np.array([[1.0, 1.0 + 2.0 ** -20, 0.5]]), 1)
    assert idx2.tolist() == [[1]]


# ---------------------------------------------------------------- permutation

@pytest.mark.parametrize("t_count,e_count,k", [(37, 8, 2), (300, 5, 3), (1, 8, 2), (64, 1, 1)])
def test_stable_permute_against_library_sort(t_count, e_count, k):
    rng = np.random.default_rng(t_count)
    idx = np.stack([rng.permutation(e_count)[:k] for _ in range(t_count)]).astype(np.int32)
    count, offset, row_of, tok = O.stable_permute(idx, e_count)
    assert count.sum() == t_count * k
    assert np.all(offset[1:] % 128 == 0) and offset[0] == 0
    # order of (expert, token, slot) keys by a library stable sort
    flat = idx.reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")       # flat index = t*k + j, already in (t, j) order
    for e in range(e_count):
        members = order[flat[order] == e]
        rows = offset[e] + np.arange(members.size)
        assert np.array_equal(row_of.reshape(-1)[members], rows)
        assert np.array_equal(tok[rows], members // k)
        assert np.all(tok[offset[e] + members.size: offset[e + 1]] == -1)
    assert np.unique(row_of).size == t_count * k


def test_stable_permute_offsets_closed_form():
    # groups of 0, 1, 128, 129 and 256 rows take 0, 128, 128, 256 and 256 padded rows:
    # an empty expert takes none, an exact multiple of 128 takes no extra tile
    counts = [0, 1, 128, 129, 256]
    idx = np.concatenate([np.full(c, e, dtype=np.int32) for e, c in enumerate(counts)])[:, None]
    count, offset, row_of, tok = O.stable_permute(idx, len(counts))
    assert count.tolist() == counts
    assert offset.tolist() == [0, 0, 128, 256, 512, 768]
    assert tok.size == 768 and int((tok >= 0).sum()) == sum(counts)


# ---------------------------------------------------------------- experts and layer

def _tiny_layer(seed, t_count=24, h=16, i=32, e_count=4, k=2):
    rng = np.random.default_rng(seed)
    x = O.round_bf16(rng.standard_normal((t_count, h)))
    wr = O.round_bf16(rng.standard_normal((e_count, h)) / math.sqrt(h))
    w1 = O.round_bf16(rng.standard_normal((e_count, i, h)) / math.sqrt(h))
    w3 = O.round_bf16(rng.standard_normal((e_count, i, h)) / math.sqrt(h))
    w2 = O.round_bf16(rng.standard_normal((e_count, h, i)) / math.sqrt(i))
    res = O.round_bf16(rng.standard_normal((t_count, h)))
    return x, wr, w1, w3, w2, res


def test_single_expert_top1_is_plain_swiglu_mlp():
    # E = 1, k = 1: the layer is the SwiGLU MLP down(silu(gate x) * up x), written
    # here with torch's own F.linear and F.silu in float64.
    x, wr, w1, w3, w2, res = _tiny_layer(3, e_count=1, k=1)
    got = O.moe_layer(x, wr[:1], w1, w3, w2, k=1)["out"]
    xt = torch.from_numpy(x)
    want = F.linear(F.silu(F.linear(xt, torch.from_numpy(w1[0]))) * F.linear(xt, torch.from_numpy(w3[0])),
                    torch.from_numpy(w2[0])).numpy()
    assert np.allclose(got, want, rtol=1e-12, atol=1e-14)


def test_diagonal_experts_closed_form():
    # H = I with diagonal weights: y_i = c_i * silu(a_i x_i) * b_i x_i.
    h = 8
    a, b, c = np.linspace(0.5, 2, h), np.linspace(-1, 1, h), np.linspace(1, 3, h)
    x = np.linspace(-2, 2, h)[None, :]
    y = O.swiglu_expert(x, np.diag(a), np.diag(b), np.diag(c))
    want = c * (a * x / (1 + np.exp(-a * x))) * (b * x)
    assert np.allclose(y, want, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("seed,k", [(4, 2), (5, 2), (6, 3)])
def test_sparse_layer_equals_dense_masked_evaluation(seed, k):
    # Evaluate all E experts on every token and mix them with a dense gate that is
    # zero off the top-k and the renormalised softmax on it (brute force).
    x, wr, w1, w3, w2, res = _tiny_layer(seed, k=k)
    got = O.moe_layer(x, wr, w1, w3, w2, k=k, residual=res)
    logits = x @ wr.T
    e_count = wr.shape[0]
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    dense = np.zeros_like(x)
    for t in range(x.shape[0]):
        top = sorted(range(e_count), key=lambda e: -p[t, e])[:k]
        gate = np.zeros(e_count)
        gate[top] = p[t, top] / p[t, top].sum()
        for e in range(e_count):
            xt = torch.from_numpy(x[t:t + 1])
            ye = F.linear(F.silu(F.linear(xt, torch.from_numpy(w1[e]))) * F.linear(xt, torch.from_numpy(w3[e])),
                          torch.from_numpy(w2[e])).numpy()[0]
            dense[t] += gate[e] * ye
    assert np.allclose(got["routed"], dense, rtol=1e-12, atol=1e-13)
    assert np.allclose(got["out"], res + dense, rtol=1e-12, atol=1e-13)


def test_slot_sum_and_ablation_invariants():
    x, wr, w1, w3, w2, res = _tiny_layer(7)
    r = O.moe_layer(x, wr, w1, w3, w2, k=2)
    # expert_outputs sums over its slot axis to routed_output
    assert np.array_equal(r["expert_outputs"].sum(1), r["routed"])
    # zeroing expert e's weight changes the output on exactly the tokens that chose e
    for e in range(wr.shape[0]):
        w_abl = np.where(r["idx"] == e, 0.0, r["weights"])
        ablated = (w_abl[:, :, None] * r["y"]).sum(1)
        changed = (ablated != r["routed"]).any(-1)
        assert np.array_equal(changed, (r["idx"] == e).any(-1))


def test_token_subset_matches_full_layer():
    x, wr, w1, w3, w2, res = _tiny_layer(8)
    full = O.moe_layer(x, wr, w1, w3, w2, k=2, residual=res, mode="bf16_storage")
    sub = [0, 5, 17, 23]
    part = O.moe_layer(x, wr, w1, w3, w2, k=2, residual=res, mode="bf16_storage", tokens=sub)
    for key in ("idx", "weights", "routed", "out"):
        assert np.array_equal(part[key], full[key][sub])


def test_bf16_storage_mode_rounds_h_and_out_closed_form():
    # one expert, one unit, x = gate = up = 1: h = silu(1) is stored as its nearest bf16;
    # y = bf16(silu(1)) * w2 stays wide, and the output is y rounded once to bf16
    # (nearest values from torch's bf16 conversion, not the oracle's rounding)
    import math
    bf = lambda v: float(torch.tensor(v, dtype=torch.float64).to(torch.bfloat16))
    one = torch.ones((1, 1), dtype=torch.bfloat16)
    w2 = torch.full((1, 1, 1), 1 + 2.0 ** -7, dtype=torch.bfloat16)
    r = O.moe_layer(one, one, one.view(1, 1, 1), one.view(1, 1, 1), w2, 1, mode="bf16_storage")
    h = bf(1.0 / (1.0 + math.exp(-1.0)))
    assert h != 1.0 / (1.0 + math.exp(-1.0))
    assert r["y"][0, 0, 0] == h * (1 + 2.0 ** -7)
    assert r["out"][0, 0] == bf(h * (1 + 2.0 ** -7)) != r["routed"][0, 0]


def test_storage_mode_differs_only_by_bf16_rounding():
    x, wr, w1, w3, w2, _ = _tiny_layer(9)
    ex = O.moe_layer(x, wr, w1, w3, w2, k=2, mode="exact")
    st = O.moe_layer(x, wr, w1, w3, w2, k=2, mode="bf16_storage")
    assert np.array_equal(ex["idx"], st["idx"])
    # bound: h rounded with relative error <= 2^-9 feeds |w2| |h|; then one more 2^-9
    bound = np.zeros_like(ex["routed"])
    for e in range(wr.shape[0]):
        tok, slot = np.nonzero(ex["idx"] == e)
        g = x[tok] @ w1[e].T
        u = x[tok] @ w3[e].T
        hmag = np.abs(O.silu(g) * u)
        contrib = (hmag @ np.abs(w2[e]).T) * 2.0 ** -9 * ex["weights"][tok, slot][:, None]
        np.add.at(bound, tok, contrib)
    bound = bound * (1 + 1e-9) + np.abs(ex["routed"] + bound) * 2.0 ** -9 + 1e-300
    assert np.all(np.abs(st["out"] - ex["routed"]) <= bound)
    assert np.any(st["out"] != ex["routed"])


# ---------------------------------------------------------------- margin screen

def test_margin_screen_enforces_gaps():
    w = W.WORKLOADS["tiny"]
    inp = W.draw(w)
    x, att, near = screen_margin(inp.x, inp.w_router, None, 2,
                                 lambda rows, a: W.redraw_x_rows(w, rows, a))
    gaps = min_gap(O.router_logits(x, inp.w_router), 2)
    ok = np.ones(x.shape[0], dtype=bool)
    ok[near.numpy()] = False
    assert np.all(gaps[ok] >= 1e-2)
    assert int(att.max()) >= 0 and near.numel() == 0
    # rows that were never redrawn are untouched
    same = att == 0
    assert torch.equal(x[same], inp.x[same])


# ---------------------------------------------------------------- the pages' printed values

def _golden_config():
    vals = {}
    with open(os.path.join(GOLDEN, "mixtral_8x7b_config.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split()
                vals[k] = float(v)
    return vals


def test_workload_shapes_match_printed_config():
    g = _golden_config()
    for name in ("decode", "prefill", "imbalanced_a", "imbalanced_b"):
        w = W.WORKLOADS[name]
        assert w.hidden_size == g["hidden_size"] and w.intermediate_size == g["intermediate_size"]
        assert w.num_experts == g["num_local_experts"] and w.num_experts_per_tok == g["num_experts_per_tok"]
    assert W.WORKLOADS["larger"].intermediate_size == g["intermediate_size_8x22b"]


def test_parameter_count_reconciles_45b_and_47b():
    # Experts: layers * E * 3 * H * I. Attention: q, k, v, o projections. Plus
    # untied embedding and head. The pages print 45B (doc) and 47B (model card):
    # the first is the expert total, the second the model total.
    g = _golden_config()
    h, i, layers = g["hidden_size"], g["intermediate_size"], g["num_hidden_layers"]
    experts = layers * g["num_local_experts"] * 3 * h * i
    attn = layers * h * (g["q_proj_out"] + g["k_proj_out"] + g["v_proj_out"] + g["o_proj_out"])
    router = layers * g["num_local_experts"] * h
    embed = 2 * g["vocab_size"] * h
    total = experts + attn + router + embed
    assert round(experts / 1e9) == g["params_total_billion_doc"]
    assert round(total / 1e9) == g["params_total_billion_card"]


# ---------------------------------------------------------------- RMSNorm (the block's norm)

def test_rms_norm_matches_torch_and_closed_form():
    rng = np.random.default_rng(10)
    h = rng.standard_normal((50, 64)) * 3
    g = 1 + 0.1 * rng.standard_normal(64)
    want = F.rms_norm(torch.from_numpy(h), (64,), torch.from_numpy(g), eps=1e-5).numpy()
    assert np.allclose(O.rms_norm(h, g, 1e-5), want, rtol=1e-13, atol=1e-14)
    # a constant row c: c / sqrt(c^2 + eps) * g
    c = -2.5
    got = O.rms_norm(np.full((1, 8), c), np.arange(1.0, 9.0), 1e-5)
    assert np.allclose(got, c / math.sqrt(c * c + 1e-5) * np.arange(1.0, 9.0), rtol=1e-15)
    # scale invariance with eps = 0
    assert np.allclose(O.rms_norm(7.0 * h, g, 0.0), O.rms_norm(h, g, 0.0), rtol=1e-13)


def test_block_is_residual_plus_layer_on_normed_input():
    x, wr, w1, w3, w2, res = _tiny_layer(11)
    g = 1 + 0.1 * np.random.default_rng(3).standard_normal(x.shape[1])
    blk = O.moe_block(res, g, 1e-5, wr, w1, w3, w2, 2, mode="exact")
    xn = O.rms_norm(res, g, 1e-5)
    lay = O.moe_layer(xn, wr, w1, w3, w2, 2, mode="exact")
    assert np.allclose(blk["out"], res + lay["routed"], rtol=1e-14, atol=1e-14)
    sub = O.moe_block(res, g, 1e-5, wr, w1, w3, w2, 2, mode="bf16_storage", tokens=[1, 4])
    full = O.moe_block(res, g, 1e-5, wr, w1, w3, w2, 2, mode="bf16_storage")
    assert np.array_equal(sub["out"], full["out"][[1, 4]])


def test_bf16_logits_round_before_scoring_and_ties_go_low():
    # exact logits 1.001, 1.003, 0.5: as bf16 (spacing 2^-7 at 1) the first two are both
    # 1.0, a tie that goes to the lower expert with equal weights; in fp32 expert 1 wins
    x = np.array([[1.0, 0.0, 0.0]])
    wr = np.array([[1.001, 0, 0], [1.003, 0, 0], [0.5, 0, 0]]).astype(np.float64)
    lb = O.router_logits(x, wr, bf16_logits=True)
    assert lb.tolist() == [[1.0, 1.0, 0.5]]
    idx, w, _ = O.route_topk(lb, 2)
    assert idx.tolist() == [[0, 1]] and np.allclose(w, [[0.5, 0.5]], rtol=0, atol=0)
    idx32, _, _ = O.route_topk(O.router_logits(x, wr), 2)
    assert idx32.tolist() == [[1, 0]]


# ---------------------------------------------------------------- int8 weight-only codes

def test_int8_rows_bounds_and_extremes():
    rng = np.random.default_rng(12)
    w = O.round_bf16(rng.standard_normal((3, 40, 64)) / 8)
    w[1, 5] = 0.0                                   # an all-zero row
    q, s = O.quantize_int8_rows(w)
    assert q.dtype == np.int8 and s.dtype == np.float32 and s.shape == (3, 40)
    assert q.min() >= -127 and q.max() <= 127
    deq = q.astype(np.float64) * s[..., None].astype(np.float64)
    # |w - q s| <= s / 2, plus the float32 rounding of w / s (<= 127 * 2^-24 of s)
    assert np.all(np.abs(w - deq) <= s[..., None] * (0.5 + 127 * 2.0 ** -23))
    # the largest |w| of every non-zero row maps to +-127
    amax_idx = np.abs(w).argmax(-1)
    top = np.take_along_axis(q, amax_idx[..., None], -1)[..., 0]
    nz = np.abs(w).max(-1) > 0
    assert np.all(np.abs(top[nz]) == 127)
    assert np.all(q[1, 5] == 0) and s[1, 5] == 1.0


def test_int8_codes_match_torch_float32_arithmetic():
    # same decision in float32 with torch's own ops: amax / 127, w / s, round half even
    rng = np.random.default_rng(13)
    w = O.round_bf16(rng.standard_normal((64, 96)) * 0.05)
    q, s = O.quantize_int8_rows(w)
    wt = torch.from_numpy(w).float()
    st = wt.abs().amax(-1) / 127.0
    qt = torch.round(wt / st[:, None]).clamp(-127, 127).to(torch.int8)
    assert np.array_equal(s, st.numpy()) and np.array_equal(q, qt.numpy())


# ---------------------------------------------------------------- 4-bit group codes

def test_int4_groups_closed_form():
    # every group holds integer multiples k * 2**-6 with k in [-7, 7] and reaches |k| = 7:
    # s = 7 * 2**-6 / 7 = 2**-6 exactly, so the codes are the k and the weights come back
    rng = np.random.default_rng(21)
    k = rng.integers(-7, 8, size=(2, 5, 192))
    k[..., ::64] = 7 * np.where(rng.random((2, 5, 3)) < 0.5, -1, 1)
    w = k * 2.0 ** -6
    q, s16 = O.quantize_int4_groups(w)
    assert q.dtype == np.int8 and s16.dtype == np.float16 and s16.shape == (2, 5, 3)
    assert np.all(s16 == np.float16(2.0 ** -6)) and np.array_equal(q, k)
    assert np.array_equal(O.dequantize_int4_groups(q, s16), w)


def test_int4_groups_nearest_code_brute_force():
    # each code is, of the 15 levels q * s16, the one nearest to w (clamped at +-7)
    rng = np.random.default_rng(22)
    w = O.round_bf16(rng.standard_normal((6, 128)) * 0.02)
    w[2, 70] = 0.5                                    # one outlier in a group
    q, s16 = O.quantize_int4_groups(w)
    s = np.repeat(s16.astype(np.float64), 64, axis=-1)
    levels = np.arange(-7, 8, dtype=np.float64)
    err = np.abs(w[..., None] - levels * s[..., None])
    best = err.min(axis=-1)
    mine = np.abs(w - q.astype(np.float64) * s)
    assert np.all(mine <= best + s * 2.0 ** -20)
    # the group's largest magnitude takes code +-7 (its scale is within a half's rounding)
    g = np.abs(w).reshape(6, 2, 64)
    top = np.take_along_axis(q.reshape(6, 2, 64), g.argmax(-1)[..., None], -1)[..., 0]
    assert np.all(np.abs(top) == 7)


def test_int4_groups_degenerate_groups_and_bound():
    rng = np.random.default_rng(23)
    w = O.round_bf16(rng.standard_normal((4, 256)) * 0.05)
    w[0, 64:128] = 0.0                   # all zeros: scale 1, codes 0
    w[1, :64] = 0.0
    w[1, 10] = 2.0 ** -30                # amax / 7 underflows a half: scale 1, codes 0
    w[2, 128:192] = 0.0                  # a subnormal scale: amax / 7 = (10/7) 2**-24
    w[2, 130] = 10 * 2.0 ** -24          # rounds to the half 2**-24, so w / s = 10: clamped
    w[2, 131] = -3 * 2.0 ** -24
    w[2, 132] = -9 * 2.0 ** -24          # clamped at -7, not -8
    q, s16 = O.quantize_int4_groups(w)
    assert s16[0, 1] == 1.0 and np.all(q[0, 64:128] == 0)
    assert s16[1, 0] == 1.0 and np.all(q[1, :64] == 0)
    assert s16[2, 2] == np.float16(2.0 ** -24) and q[2, 130] == 7 and q[2, 131] == -3
    assert q[2, 132] == -7
    assert np.all(q[2, 128:130] == 0) and np.all(q[2, 133:192] == 0)
    deq = O.dequantize_int4_groups(q, s16)
    s = np.repeat(s16.astype(np.float64), 64, axis=-1)
    # |w - f16(q s16)| <= s16 / 2 (nearest level; no clamping when s16 >= amax / 7) plus
    # the half rounding of the product (2**-11 relative)
    unclamped = np.repeat(s16.astype(np.float64) * 7 >= np.abs(w).reshape(4, 4, 64).max(-1), 64, -1)
    bound = s / 2 + np.abs(deq) * 2.0 ** -11
    assert np.all((np.abs(w - deq) <= bound)[unclamped])
    # with a normal half scale (relative rounding 2**-11), a clamped level sits at most one
    # half-rounding of the scale further out (the subnormal group above is checked exactly)
    normal = s >= 2.0 ** -14
    err_ok = np.abs(w - deq) <= s / 2 + 7 * s * 2.0 ** -10 + np.abs(deq) * 2.0 ** -11
    assert np.all(err_ok[normal]) and not np.all(normal)


def test_int4_groups_match_torch_arithmetic():
    # the same decisions with torch's float32 and half ops: amax / 7, rounded to half;
    # w / s, round half even, clamp; the product q * s formed in half precision
    rng = np.random.default_rng(24)
    w = O.round_bf16(rng.standard_normal((32, 192)) * 0.03)
    q, s16 = O.quantize_int4_groups(w)
    wt = torch.from_numpy(w).float().reshape(32, 3, 64)
    st = (wt.abs().amax(-1) / 7.0).half()
    st = torch.where(st == 0, torch.ones_like(st), st)
    qt = torch.round(wt / st.float()[..., None]).clamp(-7, 7)
    assert np.array_equal(s16, st.numpy()) and np.array_equal(q, qt.reshape(32, 192).to(torch.int8).numpy())
    dt = (qt.half() * st[..., None]).reshape(32, 192).double().numpy()
    assert np.array_equal(O.dequantize_int4_groups(q, s16), dt)


def test_round_f16_closed_forms():
    # IEEE binary16: 11 significant bits, smallest normal 2**-14, subnormal step 2**-24,
    # largest finite 65504; ties go to the even significand
    for v in (0.0, 1.0, -2.5, 65504.0, 2.0 ** -14, 2.0 ** -24, 1 + 2.0 ** -10):
        assert O.round_f16(v) == v
    assert O.round_f16(1 + 2.0 ** -11) == 1.0                      # tie, to even
    assert O.round_f16(1 + 3 * 2.0 ** -11) == 1 + 2.0 ** -9        # tie, to even
    assert O.round_f16(2049.0) == 2048.0 and O.round_f16(2051.0) == 2052.0
    assert O.round_f16(2.0 ** -25) == 0.0                          # subnormal tie
    assert O.round_f16(3 * 2.0 ** -25) == 2.0 ** -23
    assert O.round_f16(65519.0) == 65504.0
    assert np.isinf(O.round_f16(65520.0)) and O.round_f16(-1e6) == -np.inf


def test_round_f16_matches_numpy_half_cast():
    g = np.random.default_rng(3)
    a = np.concatenate([g.standard_normal(4000) * 10.0 ** g.integers(-9, 6, 4000),
                        g.standard_normal(100) * 1e-7, [7e4, -7e4, 65519.9, 65520.0]])
    with np.errstate(over="ignore"):
        want = a.astype(np.float16).astype(np.float64)
    assert np.array_equal(O.round_f16(a), want)


def test_bf16_values_in_f16_normal_range_are_exact_in_f16():
    # 8 significant bits fit in 11: the half-precision expert path reads bf16 inputs
    # unchanged when 2**-14 <= |x| <= 65504
    g = np.random.default_rng(4)
    x = O.round_bf16(g.standard_normal(5000) * 10.0 ** g.integers(-4, 4, 5000))
    x = x[(np.abs(x) >= 2.0 ** -14) & (np.abs(x) <= 65504)]
    assert np.array_equal(O.round_f16(x), x)


def test_f16_expert_mode_reads_x_rounded_to_half():
    # one expert, one unit: x = 2**-20 (1 + 2**-7) is a bf16 value below half's normal
    # range, where half spacing is 2**-24, so the experts read x16 = 2**-20. With gate and
    # up weights 2**20, g = u = 1 and h = silu(1), stored as the nearest half; the down
    # weight 1 passes it through. Unrounded x would give g = u = 1 + 2**-7 instead.
    x = torch.tensor([[2.0 ** -20 * (1 + 2.0 ** -7)]], dtype=torch.bfloat16)
    one = torch.ones((1, 1), dtype=torch.bfloat16)
    big = torch.full((1, 1, 1), 2.0 ** 20, dtype=torch.bfloat16)
    r = O.moe_layer(x, one, big, big, torch.ones((1, 1, 1), dtype=torch.bfloat16), 1,
                    mode="f16_experts")
    assert r["y"][0, 0, 0] == float(np.float16(1.0 / (1.0 + np.exp(-1.0))))
    # values beyond half's largest finite value overflow when the experts read them
    xl = torch.tensor([[70000.0]], dtype=torch.bfloat16)
    rl = O.moe_layer(xl, one, one.view(1, 1, 1), one.view(1, 1, 1),
                     torch.ones((1, 1, 1), dtype=torch.bfloat16), 1, mode="f16_experts")
    assert not np.isfinite(rl["y"][0, 0, 0])
    assert np.isfinite(O.moe_layer(xl, one, one.view(1, 1, 1), one.view(1, 1, 1),
                                   torch.ones((1, 1, 1), dtype=torch.bfloat16), 1,
                                   mode="exact")["y"][0, 0, 0])


def test_f16_expert_mode_differs_from_exact_by_f16_rounding_of_h():
    # with inputs exact in float16, the f16 expert mode equals the exact layer up to
    # the float16 rounding of h (and the final bf16 rounding)
    g = torch.Generator().manual_seed(9)
    t, hd, i, e, k = 24, 32, 48, 4, 2
    x = (torch.randn(t, hd, generator=g)).to(torch.bfloat16)
    wr = (torch.randn(e, hd, generator=g) * 0.2).to(torch.bfloat16)
    w1 = (torch.randn(e, i, hd, generator=g) * 0.2).to(torch.bfloat16)
    w3 = (torch.randn(e, i, hd, generator=g) * 0.2).to(torch.bfloat16)
    w2 = (torch.randn(e, hd, i, generator=g) * 0.2).to(torch.bfloat16)
    ex = O.moe_layer(x, wr, w1, w3, w2, k, mode="exact")
    f16 = O.moe_layer(x, wr, w1, w3, w2, k, mode="f16_experts")
    assert np.array_equal(ex["idx"], f16["idx"])
    # h relative rounding <= 2**-11, so each y moves by at most that times sum |w2| |h|
    xs = O.to_f64(x)
    for tt in range(t):
        for j in range(k):
            ee = ex["idx"][tt, j]
            h = O.silu(xs[tt] @ O.to_f64(w1[ee]).T) * (xs[tt] @ O.to_f64(w3[ee]).T)
            bound = 2.0 ** -11 * (np.abs(O.to_f64(w2[ee])) @ np.abs(h)) + 1e-12
            assert np.all(np.abs(f16["y"][tt, j] - ex["y"][tt, j]) <= bound)
    assert not np.array_equal(f16["y"], ex["y"])
    assert np.array_equal(f16["out"], O.round_bf16(f16["routed"]))
