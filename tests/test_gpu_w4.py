"""Weight-only 4-bit experts: the quantiser's codes and group scales equal the oracle's
bit for bit, and the 4-bit grouped GEMMs and the whole 4-bit layer match the oracle's
half-precision expert mode run on the dequantised weights half(q * s)."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_09_b200 import moe as M
from sparse_mixture_experts_09_b200 import workloads as W

from ._cases import assert_layer_close, sample_tokens, screened, to_cpu
from .test_gpu_kernels import SMALL
from .test_gpu_w8 import SMALL_BATCH

pytestmark = pytest.mark.gpu

CASES = {**SMALL, **SMALL_BATCH}


def unblock4(q, s):
    """Tiled 4-bit codes and tile-ordered scales -> row-major int8 codes [E, R, K] and
    float16 scales [E, R, K / 64]. A 4 KiB tile is [column half v][row][4 words]; word m
    of a row's 16 bytes holds columns 32 v + 8 m .. + 7, column 2j in nibble j and column
    2j + 1 in nibble j + 4."""
    e, r, k2 = q.shape
    k = 2 * k2
    b = np.ascontiguousarray(q.cpu().numpy()).reshape(e * r // 128, k // 64, 2, 128, 16)
    words = b.transpose(0, 3, 1, 2, 4).reshape(e * r, k // 8, 4).view(np.uint32)[..., 0]
    codes = np.empty((e * r, k // 8, 8), dtype=np.int8)
    for nib in range(8):
        col = 2 * nib if nib < 4 else 2 * (nib - 4) + 1
        codes[:, :, col] = ((words >> (4 * nib)) & 15).astype(np.int8) - 8
    sc = s.cpu().numpy().transpose(0, 1, 3, 2).reshape(e, r, k // 64)
    return codes.reshape(e, r, k), sc


def _dequantised(c):
    out = []
    for w in (c.w1, c.w3, c.w2):
        q, s = O.quantize_int4_groups(w)
        out.append((q, s, O.dequantize_int4_groups(q, s)))
    return out


class _Dequantised:
    """Expert e of half(q * s) on demand (the oracle's codes), one expert at a time."""

    def __init__(self, w):
        self.w = w

    def __getitem__(self, e):
        q, s = O.quantize_int4_groups(self.w[e])
        return O.dequantize_int4_groups(q, s)


@pytest.mark.parametrize("name", ["tiny", "ragged", "e5k3", "bn128_split"])
def test_quantize4_matches_oracle(name):
    w = SMALL[name]
    _, w1, w3, w2 = W.draw_weights(w, "cuda")
    # an all-zero group (scale 1, codes 0), a group whose scale underflows a half, and a
    # group with one large entry
    w1[0, 5, :64].zero_()
    w3[0, 2, 64:128].zero_()
    w3[0, 2, 70] = 2.0 ** -30
    w2[-1, 3, 7] = 40.0
    ex = M.quantize_int4(w1, w3, w2)
    torch.cuda.synchronize()
    for q_gpu, s_gpu, src in ((ex.q1, ex.s1, w1), (ex.q3, ex.s3, w3), (ex.q2, ex.s2, w2)):
        q, s = O.quantize_int4_groups(src.cpu())
        got_q, got_s = unblock4(q_gpu, s_gpu)
        assert np.array_equal(got_q, q)
        assert np.array_equal(got_s.view(np.uint16), s.view(np.uint16))
    q1, s1 = unblock4(ex.q1, ex.s1)
    assert s1[0, 5, 0] == 1.0 and np.all(q1[0, 5, :64] == 0)
    q3, s3 = unblock4(ex.q3, ex.s3)
    assert s3[0, 2, 1] == 1.0 and np.all(q3[0, 2, 64:128] == 0)
    assert int(np.abs(q1).max()) == 7


@pytest.mark.parametrize("name", list(CASES))
def test_grouped_swiglu_w4_matches_oracle(name):
    w = CASES[name]
    inp, _ = screened(w)
    c = to_cpu(inp)
    k = w.num_experts_per_tok
    (_, _, d1), (_, _, d3), (_, _, d2) = _dequantised(c)
    ref = O.moe_layer(c.x, c.w_router, d1, d3, d2, k, logit_bias=c.logit_bias, mode="f16_experts")
    ex = M.quantize_int4(inp.w1, inp.w3, inp.w2)
    shape = M.make_shape(*w.shape)
    ws = M.make_workspace(shape)
    p = M.permute(torch.from_numpy(ref["idx"]).cuda(), inp.x, w.num_experts, w.intermediate_size, ws)
    y = M.grouped_swiglu_w4(p["x_perm"], p["offsets"], ex, w.num_tokens, k, ws)
    M.device_status(ws)
    row_of = p["row_of"].cpu().numpy().astype(np.int64)
    got = y.cpu().double().numpy()[row_of]
    assert_layer_close(got, ref["y"], f"{name} y")
    tok = p["token_of_row"][: int(p["offsets"][-1])].cpu().numpy()
    assert np.all(y.cpu().numpy()[: tok.size][tok < 0] == 0)


@pytest.mark.parametrize("name", ["tiny", "ragged", "e5k3", "one_token", "skewed", "bn128_split",
                                  "ts_t33", "ts_e64k8", "ts_h640", "ts_k1", "t64_edge", "t65_edge",
                                  "t17_e4", "t24_e2", "t48_e2", "t160_skew", "t96_e4"])
def test_forward_w4_matches_oracle(name):
    w = CASES[name]
    inp, near = screened(w)
    assert near.numel() == 0
    c = to_cpu(inp)
    k = w.num_experts_per_tok
    (_, _, d1), (_, _, d3), (_, _, d2) = _dequantised(c)
    ex = M.quantize_int4(inp.w1, inp.w3, inp.w2)
    ws = M.make_workspace(M.make_shape(*w.shape))
    for residual in (None, inp.residual):
        out = M.forward_w4(inp.x, inp.w_router, ex, k, residual=residual, logit_bias=inp.logit_bias,
                           ws=ws)
        M.device_status(ws)
        ref = O.moe_layer(c.x, c.w_router, d1, d3, d2, k,
                          residual=None if residual is None else c.residual,
                          logit_bias=c.logit_bias, mode="f16_experts")
        assert_layer_close(O.to_f64(out.cpu()), ref["out"], name)


@pytest.mark.parametrize("name", ["decode", "prefill", "larger_decode_T1", "larger_decode_T64",
                                  "larger_decode_T256"])
def test_forward_w4_full_size_against_oracle(name):
    w = W.workload(name)
    inp, near = screened(w)
    assert near.numel() == 0
    ex = M.quantize_int4(inp.w1, inp.w3, inp.w2)
    ws = M.make_workspace(M.make_shape(*w.shape))
    out = M.forward_w4(inp.x, inp.w_router, ex, 2, ws=ws)
    M.device_status(ws)
    # deterministic: repeated runs agree bit for bit (no ordering-dependent reads)
    for _ in range(3):
        again = M.forward_w4(inp.x, inp.w_router, ex, 2, ws=ws)
        assert torch.equal(again, out)
    tokens = sample_tokens(w.num_tokens)
    c = to_cpu(inp)
    deq = [_Dequantised(t) for t in (c.w1, c.w3, c.w2)]
    ref = O.moe_layer(c.x, c.w_router, deq[0], deq[1], deq[2], 2, mode="f16_experts", tokens=tokens)
    assert_layer_close(O.to_f64(out.cpu())[tokens], ref["out"], name)
    # 15 levels per 64-column group move the layer ~0.2 (relative norm) from the bf16
    # layer on these Gaussian weights; a wrong layout or scale lands near 1 or beyond
    out_bf16 = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, 2)
    rel = (out.double() - out_bf16.double()).norm() / out_bf16.double().norm()
    assert float(rel) < 0.3
