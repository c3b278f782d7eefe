"""Weight-only int8 experts: the quantiser's codes and scales equal the oracle's bit
for bit, and the int8 grouped GEMMs and the whole int8 layer match the oracle's
half-precision expert mode run on the dequantised weights q * s."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_09_b200 import moe as M
from sparse_mixture_experts_09_b200 import workloads as W

from ._cases import assert_layer_close, sample_tokens, screened, to_cpu
from .test_gpu_kernels import SMALL

pytestmark = pytest.mark.gpu


def _unblock(q):
    """Tiled offset-binary codes -> row-major int8 [E, R, K]. Tile (row tile, column
    tile) is 8 KiB: [column chunk v (16 columns)][row][16 columns]."""
    e, r, k = q.shape
    t = q.reshape(e * r // 128, k // 64, 4, 128, 16).permute(0, 3, 1, 2, 4).reshape(e, r, k)
    return (t.to(torch.int16) - 128).to(torch.int8)


def _oracle_experts(c):
    """The oracle's codes and scales of (w1, w3, w2) and the dequantised weights."""
    out = []
    for w in (c.w1, c.w3, c.w2):
        q, s = O.quantize_int8_rows(w)
        out.append((q, s, q.astype(np.float64) * s.astype(np.float64)[..., None]))
    return out


class _Dequantised:
    """Expert e of q * s on demand (the oracle's codes), one expert in memory at a time."""

    def __init__(self, w):
        self.w = w

    def __getitem__(self, e):
        q, s = O.quantize_int8_rows(self.w[e])
        return q.astype(np.float64) * s.astype(np.float64)[:, None]


@pytest.mark.parametrize("name", ["tiny", "ragged", "e5k3", "bn128_split"])
def test_quantize_matches_oracle(name):
    w = SMALL[name]
    _, w1, w3, w2 = W.draw_weights(w, "cuda")
    # an all-zero row (scale 1, codes 0) and a row with one large entry
    w1[0, 5].zero_()
    w2[-1, 3, 7] = 40.0
    ex = M.quantize_int8(w1, w3, w2)
    torch.cuda.synchronize()
    for q_gpu, s_gpu, src in ((ex.q1, ex.s1, w1), (ex.q3, ex.s3, w3), (ex.q2, ex.s2, w2)):
        q, s = O.quantize_int8_rows(src.cpu())
        assert np.array_equal(_unblock(q_gpu).cpu().numpy(), q)
        assert np.array_equal(s_gpu.cpu().numpy().view(np.uint32), s.view(np.uint32))
    codes = _unblock(ex.q1)
    assert float(ex.s1[0, 5]) == 1.0 and int(codes[0, 5].abs().max()) == 0
    assert int(codes.to(torch.int16).abs().max()) == 127


# Few tokens (one row tile per expert, mostly padding; at most 64 tokens run on 64-row
# tiles): an odd token count, many experts with k = 8, a hidden size that is not a
# multiple of 256, k = 1, and both sides of the 64-token switch with every token on
# both of 2 experts (64 and 65 rows per expert).
SMALL_BATCH = {
    "ts_t33": W.Workload("ts_t33", 33, 256, 384, 8, 2, seed=31),
    "ts_e64k8": W.Workload("ts_e64k8", 50, 256, 256, 64, 8, seed=32),
    "ts_h640": W.Workload("ts_h640", 48, 640, 512, 16, 4, seed=33),
    "ts_k1": W.Workload("ts_k1", 7, 128, 1024, 4, 1, seed=34),
    # 64 tokens is the last batch on 64-row tiles; 65 takes the 128-row tiles
    "t64_edge": W.Workload("t64_edge", 64, 256, 256, 2, 2, seed=35),
    "t65_edge": W.Workload("t65_edge", 65, 256, 256, 2, 2, seed=36),
    # the swap-operand kernel's row widths: 17 and 24 tokens take its 32-row variant (24
    # rows per expert: N = 32), 48 tokens its 64-row variant with N = 48
    "t17_e4": W.Workload("t17_e4", 17, 512, 512, 4, 2, seed=37),
    "t24_e2": W.Workload("t24_e2", 24, 256, 512, 2, 2, seed=38),
    "t48_e2": W.Workload("t48_e2", 48, 384, 768, 2, 2, seed=39),
    # above 64 tokens (at most 48 routed rows per expert on average) an expert's rows are
    # cut into 64-row sub-tiles over the same weight tiles: 160 tokens with expert 0
    # favoured give it 155 rows (sub-tiles of 64, 64 and 27); 96 tokens on 4 experts
    # with expert 0 slightly favoured give it 66 rows (64 and 2)
    "t160_skew": W.Workload("t160_skew", 160, 256, 512, 8, 2, seed=45,
                            logit_bias=(3.0, 0, 0, 0, 0, 0, 0, 0)),
    "t96_e4": W.Workload("t96_e4", 96, 384, 512, 4, 2, seed=46, logit_bias=(0.5, 0, 0, 0)),
}
CASES = {**SMALL, **SMALL_BATCH}


@pytest.mark.parametrize("name", list(CASES))
def test_grouped_swiglu_w8_matches_oracle(name):
    w = CASES[name]
    inp, _ = screened(w)
    c = to_cpu(inp)
    k = w.num_experts_per_tok
    (q1, _, d1), (q3, _, d3), (q2, _, d2) = _oracle_experts(c)
    ref = O.moe_layer(c.x, c.w_router, d1, d3, d2, k, logit_bias=c.logit_bias, mode="f16_experts")
    ex = M.quantize_int8(inp.w1, inp.w3, inp.w2)
    shape = M.make_shape(*w.shape)
    ws = M.make_workspace(shape)
    p = M.permute(torch.from_numpy(ref["idx"]).cuda(), inp.x, w.num_experts, w.intermediate_size, ws)
    y = M.grouped_swiglu_w8(p["x_perm"], p["offsets"], ex, w.num_tokens, k, ws)
    M.device_status(ws)
    assert np.array_equal(_unblock(ex.q2).cpu().numpy(), q2)
    row_of = p["row_of"].cpu().numpy().astype(np.int64)
    got = y.cpu().double().numpy()[row_of]
    assert_layer_close(got, ref["y"], f"{name} y")
    tok = p["token_of_row"][: int(p["offsets"][-1])].cpu().numpy()
    assert np.all(y.cpu().numpy()[: tok.size][tok < 0] == 0)


@pytest.mark.parametrize("name", ["tiny", "ragged", "e5k3", "one_token", "skewed", "bn128_split",
                                  "ts_t33", "ts_e64k8", "ts_h640", "t64_edge", "t65_edge",
                                  "t17_e4", "t24_e2", "t48_e2", "t160_skew", "t96_e4"])
def test_forward_w8_matches_oracle(name):
    w = CASES[name]
    inp, near = screened(w)
    assert near.numel() == 0
    c = to_cpu(inp)
    k = w.num_experts_per_tok
    (_, _, d1), (_, _, d3), (_, _, d2) = _oracle_experts(c)
    ex = M.quantize_int8(inp.w1, inp.w3, inp.w2)
    ws = M.make_workspace(M.make_shape(*w.shape))
    for residual in (None, inp.residual):
        out = M.forward_w8(inp.x, inp.w_router, ex, k, residual=residual, logit_bias=inp.logit_bias,
                           ws=ws)
        M.device_status(ws)
        ref = O.moe_layer(c.x, c.w_router, d1, d3, d2, k,
                          residual=None if residual is None else c.residual,
                          logit_bias=c.logit_bias, mode="f16_experts")
        assert_layer_close(O.to_f64(out.cpu()), ref["out"], name)


@pytest.mark.parametrize("name", ["decode", "prefill", "larger_decode_T1", "larger_decode_T64",
                                  "larger_decode_T256"])
def test_forward_w8_full_size_against_oracle(name):
    w = W.workload(name)
    inp, near = screened(w)
    assert near.numel() == 0
    ex = M.quantize_int8(inp.w1, inp.w3, inp.w2)
    ws = M.make_workspace(M.make_shape(*w.shape))
    out = M.forward_w8(inp.x, inp.w_router, ex, 2, ws=ws)
    M.device_status(ws)
    # deterministic: repeated runs agree bit for bit (no ordering-dependent reads)
    for _ in range(3):
        again = M.forward_w8(inp.x, inp.w_router, ex, 2, ws=ws)
        assert torch.equal(again, out)
    tokens = sample_tokens(w.num_tokens)
    c = to_cpu(inp)
    deq = [_Dequantised(t) for t in (c.w1, c.w3, c.w2)]
    ref = O.moe_layer(c.x, c.w_router, deq[0], deq[1], deq[2], 2, mode="f16_experts", tokens=tokens)
    assert_layer_close(O.to_f64(out.cpu())[tokens], ref["out"], name)
    # the int8 layer stays close to the bf16 layer (quantisation and half rounding)
    out_bf16 = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, 2)
    rel = (out.double() - out_bf16.double()).norm() / out_bf16.double().norm()
    assert float(rel) < 4e-2
