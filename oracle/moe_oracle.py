"""fp64 CPU oracle of the Mixtral sparse-MoE feed-forward layer.

TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import or run this module. The CUDA path never
does, and this module imports nothing from it: it shares no code, table or helper
with the kernels. Inputs arrive as arrays of bf16 values (torch CPU tensors or numpy
arrays); everything below is numpy in float64.

What it computes, in the pages' own order (nnterp encyclopedia, "Mixtral"):

1. router logits   l = x W_r^T, one per expert, no bias ("Values, by host":
                   router_logits is the output of the router's F.linear, before the
                   scoring; "Attention has no window": no projection has a bias);
2. scoring         softmax over all E experts, keep the k largest, divide them by
                   their sum; slot 0 holds the larger weight ("The router
                   renormalizes its top 2, in float32");
3. experts         per routed slot, down(act(gate x) * up x) with act = silu
                   ("Values, by host": mlp_neurons is act(gate)*up, what the down
                   projection receives; Hugging Face "Mixtral" doc, MixtralConfig:
                   hidden_act silu);
4. combine         expert_outputs[t, j] = w[t, j] * y[t, j]; routed_output is their
                   sum over the slot axis ("expert_outputs needs the default experts
                   implementation"); mlp_output == routed_output (no shared expert);
                   the block adds it to the residual ("The block, in order").

Two modes. ``exact`` rounds nothing. ``bf16_storage`` rounds, to the nearest bf16
with ties to even, at the two places where a bf16 load stores bf16 values on this
path: the expert's hidden activation h (mlp_neurons) and the block's output
("The router renormalizes its top 2, in float32": in a bf16 load routed_output is
bf16 while expert_weights stay float32).

Readings where the pages are silent:
* The top-k decision is taken on the router logits rounded to float32 (the scoring
  precision the pages fix; softmax is strictly increasing, so ranking logits ranks
  probabilities); equal float32 logits go to the lower expert index. The weights
  themselves are computed in fp64 from the unrounded logits.
* The expert-contiguous order of routed rows is a stable counting sort on
  (expert, token, slot); every expert group is padded to a multiple of ``pad`` rows,
  pad rows carry token -1.
* With k = 1 the single weight is renormalised to exactly 1.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "to_f64", "round_bf16", "round_f16", "silu", "router_logits", "route_topk", "stable_permute",
    "swiglu_expert", "moe_layer", "rms_norm", "moe_block", "quantize_int8_rows",
    "quantize_int4_groups", "dequantize_int4_groups",
]


def to_f64(a) -> np.ndarray:
    """float64 numpy copy of ``a`` (a torch tensor of any float dtype, or an array)."""
    if hasattr(a, "detach"):
        return a.detach().cpu().double().numpy()
    return np.asarray(a, dtype=np.float64)


def round_bf16(a) -> np.ndarray:
    """Nearest bf16 value of each fp64 element, ties to even, returned as fp64.

    bf16 keeps 8 significant bits and float32's exponent range (smallest normal
    2**-126, subnormal spacing 2**-133). For |a| = m * 2**e with 0.5 <= m < 1 the
    spacing of bf16 values near a is 2**(e - 8), floored at 2**-133; dividing by a
    power of two is exact, and np.rint rounds half-way cases to even.
    """
    a = np.asarray(a, dtype=np.float64)
    _, e = np.frexp(a)
    quantum = np.ldexp(1.0, np.maximum(e, -125) - 8)
    return np.rint(a / quantum) * quantum


def round_f16(a) -> np.ndarray:
    """Nearest IEEE half-precision (float16) value of each fp64 element, ties to even,
    returned as fp64; magnitudes that round past the largest finite value 65504 become
    infinite.

    float16 keeps 11 significant bits; its smallest normal is 2**-14 and its subnormal
    spacing 2**-24. For |a| = m * 2**e with 0.5 <= m < 1 the spacing near a is
    2**(e - 11), floored at 2**-24.
    """
    a = np.asarray(a, dtype=np.float64)
    _, e = np.frexp(a)
    quantum = np.ldexp(1.0, np.maximum(e, -13) - 11)
    r = np.rint(a / quantum) * quantum
    return np.where(np.abs(r) > 65504.0, np.copysign(np.inf, a), r)


def silu(g: np.ndarray) -> np.ndarray:
    """silu(g) = g * sigmoid(g) = g / (1 + exp(-g))."""
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def router_logits(x, w_router, logit_bias=None, bf16_logits: bool = False) -> np.ndarray:
    """[T, E] fp64 logits l[t, e] = sum_h x[t, h] * W_r[e, h] (+ logit_bias[e] if given).

    ``logit_bias`` is not part of Mixtral; the benchmark's imbalanced workload uses it
    to skew routing. With ``bf16_logits`` each logit is rounded to bf16 first, as in a
    bf16 load, whose router returns bf16 logits that the scoring casts to float32
    ("The router renormalizes its top 2, in float32").
    """
    logits = to_f64(x) @ to_f64(w_router).T
    if bf16_logits:
        logits = round_bf16(logits)
    if logit_bias is not None:
        logits = logits + to_f64(logit_bias)[None, :]
    return logits


def route_topk(logits: np.ndarray, k: int):
    """Softmax over all experts, the k largest, renormalised to sum to one.

    Returns (idx [T, k] int32, weights [T, k] fp64, probs [T, E] fp64); slot 0 holds
    the largest weight.
    """
    logits = np.asarray(logits, dtype=np.float64)
    t_count, e_count = logits.shape
    shifted = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(shifted)
    p = p / p.sum(axis=1, keepdims=True)
    key32 = logits.astype(np.float32)
    idx = np.empty((t_count, k), dtype=np.int32)
    for t in range(t_count):
        # stable sort of -key keeps lower expert indices first among equal keys
        order = np.argsort(-key32[t].astype(np.float64), kind="stable")
        idx[t] = order[:k]
    top = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    weights = top / top.sum(axis=1, keepdims=True)
    return idx, weights, p


def stable_permute(idx: np.ndarray, num_experts: int, pad: int = 128):
    """Expert-contiguous order of the routed (token, slot) pairs.

    Counting sort: count[e] = #{(t, j): idx[t, j] == e}; group e starts at
    offset[e] = sum_{e' < e} pad_up(count[e']); within a group rows follow token,
    then slot, order. Returns (count [E], offset [E+1], row_of [T, k],
    token_of_row [offset[E]] with -1 on pad rows).
    """
    idx = np.asarray(idx)
    t_count, k = idx.shape
    count = np.zeros(num_experts, dtype=np.int64)
    for e in idx.reshape(-1):
        count[e] += 1
    padded = (count + pad - 1) // pad * pad
    offset = np.zeros(num_experts + 1, dtype=np.int64)
    offset[1:] = np.cumsum(padded)
    cursor = offset[:-1].copy()
    row_of = np.empty((t_count, k), dtype=np.int64)
    token_of_row = np.full(int(offset[-1]), -1, dtype=np.int64)
    for t in range(t_count):
        for j in range(k):
            e = idx[t, j]
            row_of[t, j] = cursor[e]
            token_of_row[cursor[e]] = t
            cursor[e] += 1
    return count, offset, row_of, token_of_row


def swiglu_expert(x_rows: np.ndarray, w1_e, w3_e, w2_e, h_bf16: bool = False) -> np.ndarray:
    """y = down(silu(gate x) * up x) for each row of ``x_rows`` ([n, H] fp64).

    gate = w1 [I, H], up = w3 [I, H], down = w2 [H, I], all in nn.Linear
    [out, in] form. With ``h_bf16`` the hidden activation is rounded to bf16 before
    the down projection, as a bf16 load stores it.
    """
    g = x_rows @ to_f64(w1_e).T
    u = x_rows @ to_f64(w3_e).T
    h = silu(g) * u
    if h_bf16:
        h = round_bf16(h)
    return h @ to_f64(w2_e).T


def moe_layer(x, w_router, w1, w3, w2, k: int, residual=None, logit_bias=None,
              mode: str = "exact", tokens=None, bf16_logits: bool = False) -> dict:
    """The layer on tokens ``tokens`` (all tokens when None).

    ``mode``: ``exact`` rounds nothing; ``bf16_storage`` rounds h and the output to
    bf16 (a bf16 load); ``f16_experts`` is a half-precision expert path, as a float16
    load computes it (Hugging Face "Mixtral" doc, "Shrinking down Mixtral using
    quantization": the model in half precision, float16): the experts read x rounded
    to float16 and store h as float16, the router and the combine are as in
    ``bf16_storage``.

    Returns a dict of fp64 arrays over the chosen tokens: ``logits`` [n, E], ``idx``
    [n, k], ``weights`` [n, k], ``y`` [n, k, H] (unweighted expert outputs),
    ``expert_outputs`` [n, k, H] (weighted), ``routed`` [n, H] and ``out`` [n, H]
    (residual + routed; rounded to bf16 in ``bf16_storage`` mode).
    """
    if mode not in ("exact", "bf16_storage", "f16_experts"):
        raise ValueError(mode)
    storage = mode != "exact"
    xs = to_f64(x)
    if tokens is not None:
        tokens = np.asarray(tokens, dtype=np.int64)
        xs = xs[tokens]
    n, hidden = xs.shape
    logits = router_logits(xs, w_router, logit_bias, bf16_logits)
    idx, weights, _ = route_topk(logits, k)
    num_experts = logits.shape[1]
    # f16_experts: the experts read x as float16 and store h as float16
    x_experts = round_f16(xs) if mode == "f16_experts" else xs
    y = np.zeros((n, k, hidden), dtype=np.float64)
    for e in range(num_experts):
        tok, slot = np.nonzero(idx == e)
        if tok.size == 0:
            continue
        if mode == "f16_experts":
            h = silu(x_experts[tok] @ to_f64(w1[e]).T) * (x_experts[tok] @ to_f64(w3[e]).T)
            y[tok, slot] = round_f16(h) @ to_f64(w2[e]).T
        else:
            y[tok, slot] = swiglu_expert(xs[tok], w1[e], w3[e], w2[e], h_bf16=storage)
    expert_outputs = weights[:, :, None] * y
    routed = np.zeros((n, hidden), dtype=np.float64)
    for j in range(k):
        routed = routed + expert_outputs[:, j]
    out = routed.copy()
    if residual is not None:
        res = to_f64(residual)
        if tokens is not None:
            res = res[tokens]
        out = res + routed
    if storage:
        out = round_bf16(out)
    return {"logits": logits, "idx": idx, "weights": weights, "y": y,
            "expert_outputs": expert_outputs, "routed": routed, "out": out}


def rms_norm(h, weight, eps: float) -> np.ndarray:
    """RMSNorm of each row: h / sqrt(mean(h^2) + eps) * weight, in fp64.

    The block norms the residual stream before the mixture (nnterp "Mixtral", "The
    block, in order": out = h + mlp(post_attention_layernorm(h)); Printout:
    MixtralRMSNorm((4096,), eps=1e-05); Config: rms_norm_eps 1e-05). The pages name the
    norm and its epsilon but do not write it out; this is the standard root-mean-square
    layer norm with a learned per-channel gain and no bias, eps inside the root.
    """
    h = to_f64(h)
    ms = (h * h).mean(axis=1, keepdims=True)
    return h / np.sqrt(ms + eps) * to_f64(weight)[None, :]


def moe_block(h, norm_weight, eps: float, w_router, w1, w3, w2, k: int, logit_bias=None,
              mode: str = "exact", tokens=None) -> dict:
    """The mixture half of the decoder block: out = h + moe(rms_norm(h)).

    In ``bf16_storage`` mode the normed activations are rounded to bf16 (they are the
    mixture's bf16 input in a bf16 load) and the output is rounded once.
    """
    hs = to_f64(h)
    if tokens is not None:
        hs = hs[np.asarray(tokens, dtype=np.int64)]
    x = rms_norm(hs, norm_weight, eps)
    if mode == "bf16_storage":
        x = round_bf16(x)
    r = moe_layer(x, w_router, w1, w3, w2, k, residual=hs, logit_bias=logit_bias, mode=mode)
    r["x_norm"] = x
    return r


def quantize_int8_rows(w):
    """Symmetric per-row int8 codes of a weight matrix (or a stack of them).

    The pages load Mixtral in int8 or 4 bits to shrink its ~90 GB of bf16 weights
    (Hugging Face "Mixtral" doc, "Shrinking down Mixtral using quantization"; "Welcome
    Mixtral", "Quantizing Mixtral") but leave the scheme to the quantisation library.
    This is the plain weight-only scheme: for every output row (channel), scale s =
    max|w| / 127 and code q = round-half-even(w / s), so w ~ q * s with |w - q s| <= s/2.
    The code is an integer that floating point decides, so it is decided in float32 (s
    and w / s correctly rounded in float32, as the kernel does); an all-zero row has
    s = 1 and q = 0. Returns (q int8 array, s float32 array [..., rows]).
    """
    w = np.asarray(to_f64(w), dtype=np.float32)
    amax = np.abs(w).max(axis=-1)
    s = np.where(amax > 0, amax / np.float32(127.0), np.float32(1.0)).astype(np.float32)
    q = np.rint(w / s[..., None]).astype(np.float32)
    q = np.clip(q, -127, 127).astype(np.int8)
    return q, s


def quantize_int4_groups(w, group: int = 64):
    """Symmetric 4-bit codes with one half-precision scale per ``group`` columns of a row.

    The pages also load Mixtral in 4 bits (Hugging Face "Mixtral" doc, "Shrinking down
    Mixtral using quantization"; "Welcome Mixtral", "Quantizing Mixtral") and leave the
    format to the quantisation library. Fifteen levels cannot cover a whole row well, so
    the scale is per run of ``group`` consecutive columns of a row (a group), in the
    manner of block-wise 4-bit schemes: for each group, s = max|w| / 7 in float32, then
    rounded to the nearest IEEE half (s16; a group whose s16 is zero, all zeros or too
    small for a half, takes s16 = 1); code q = round-half-even(w / s16) in float32,
    clamped to [-7, 7]. The code is decided in float32 as the kernel decides it. A
    group whose largest |w| exceeds 7 * 65504 has an infinite half scale (outside the
    format: its weights dequantise to NaN).
    Returns (q int8 [..., rows, K], s16 float16 [..., rows, K / group]).
    """
    w = np.asarray(to_f64(w), dtype=np.float32)
    k = w.shape[-1]
    if k % group:
        raise ValueError(f"row length {k} is not a multiple of the group {group}")
    g = w.reshape(*w.shape[:-1], k // group, group)
    amax = np.abs(g).max(axis=-1)
    s = (amax / np.float32(7.0)).astype(np.float32)
    s16 = round_f16(s.astype(np.float64))
    s16 = np.where(s16 == 0, 1.0, s16).astype(np.float16)
    q = np.rint(g / s16.astype(np.float32)[..., None])
    q = np.clip(q, -7, 7).astype(np.int8).reshape(w.shape)
    return q, s16


def dequantize_int4_groups(q, s16, group: int = 64) -> np.ndarray:
    """The weight a 4-bit expert multiplies: q * s16 rounded once to the nearest half
    (the product of a code and a half scale, formed in half precision), as fp64."""
    q = np.asarray(q)
    k = q.shape[-1]
    prod = (q.astype(np.float64).reshape(*q.shape[:-1], k // group, group)
            * np.asarray(s16, dtype=np.float64)[..., None])
    return round_f16(prod).reshape(q.shape)
