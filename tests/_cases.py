"""Shared helpers of the GPU parity tests: screened inputs and the tolerance gate."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as O
from oracle.screen import screen_margin
from sparse_mixture_experts_09_b200 import workloads as W

# Float tolerance of the layer output (normwise max relative error and mean absolute
# error relative to the RMS of the reference), against the oracle's bf16-storage mode.
MAX_REL = 2e-2
MAE_RMS = 1e-3
# Routing weights: fp32 softmax and renormalisation against the fp64 oracle.
W_ABS = 2e-6


def screened(w: W.Workload, device="cuda"):
    """Inputs of ``w`` with the routing margin enforced on x (weights drawn on
    ``device``, x drawn and screened on the CPU). Returns (LayerInputs on device,
    near-tie rows)."""
    wr, w1, w3, w2 = W.draw_weights(w, device)
    x = W.draw_x(w, "cpu")
    bias = None if w.logit_bias is None else torch.tensor(w.logit_bias, dtype=torch.float32)
    x, _, near = screen_margin(x, wr.cpu(), bias, w.num_experts_per_tok,
                               lambda rows, a: W.redraw_x_rows(w, rows, a))
    res = W.synth.normal_rows_unit_rms(w.num_tokens, w.hidden_size, w.seed, W.RESIDUAL_ID, 0, "cpu")
    inp = W.LayerInputs(x.to(device), wr, w1, w3, w2, res.to(device),
                        None if bias is None else bias.to(device))
    return inp, near


def to_cpu(inp: W.LayerInputs) -> W.LayerInputs:
    return W.LayerInputs(*(None if t is None else t.cpu() for t in
                           (inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, inp.residual, inp.logit_bias)))


def layer_errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    max_rel = float(err.max() / max(np.abs(ref).max(), 1e-300))
    mae_rms = float(err.mean() / max(np.sqrt((ref ** 2).mean()), 1e-300))
    return max_rel, mae_rms


def assert_layer_close(got, ref, what=""):
    max_rel, mae_rms = layer_errors(got, ref)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), what
    assert max_rel <= MAX_REL and mae_rms <= MAE_RMS, (what, max_rel, mae_rms)
    return max_rel, mae_rms


def sample_tokens(t_count: int, n: int = 256, seed: int = 1234) -> np.ndarray:
    if t_count <= n:
        return np.arange(t_count)
    g = np.random.default_rng(seed)
    pick = g.choice(np.arange(1, t_count - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, t_count - 1], pick]))


def bf16_np(t: torch.Tensor) -> np.ndarray:
    return O.to_f64(t)


def bf16_midpoint_distance(v: np.ndarray) -> np.ndarray:
    """Distance of each fp64 value to the nearest half-way point between bf16 values."""
    _, e = np.frexp(v)
    q = np.ldexp(1.0, np.maximum(e, -125) - 8)
    u = v / q
    return np.abs((u - np.floor(u)) - 0.5) * q


def decision_window(exact: np.ndarray, k: int) -> np.ndarray:
    """Logits that can decide a bf16-logit top-k: the k largest and any within two bf16
    steps below the k-th (the renormalised weights depend on the selected logits only)."""
    kth = -np.sort(-exact, axis=1)[:, k - 1:k]
    _, e = np.frexp(kth)
    step = np.ldexp(1.0, np.maximum(e, -125) - 8)
    return exact >= kth - 2 * step


def screened_bf16_logits(w: W.Workload, device="cuda", max_attempts: int = 64):
    """Inputs whose router logits all sit far enough from bf16 rounding half-way points
    that the GPU's fp32 sum and the exact sum round to the same bf16 value (redrawing
    x rows that do not). Returns (LayerInputs on device, rows still failing)."""
    wr, w1, w3, w2 = W.draw_weights(w, device)
    wr_c = wr.cpu()
    x = W.draw_x(w, "cpu")
    absw = np.abs(O.to_f64(wr_c)).T

    def bad_rows(xs):
        exact = O.to_f64(xs) @ O.to_f64(wr_c).T
        bound = 1e-5 * (np.abs(O.to_f64(xs)) @ absw) + 1e-6
        near = bf16_midpoint_distance(exact) <= bound
        return np.nonzero((near & decision_window(exact, w.num_experts_per_tok)).any(axis=1))[0]

    bad = bad_rows(x)
    attempt = 0
    while bad.size and attempt < max_attempts:
        attempt += 1
        rows = torch.from_numpy(bad.astype(np.int64))
        x[rows] = W.redraw_x_rows(w, rows, attempt)
        still = bad_rows(x[rows])
        bad = bad[still]
    res = W.synth.normal_rows_unit_rms(w.num_tokens, w.hidden_size, w.seed, W.RESIDUAL_ID, 0, "cpu")
    inp = W.LayerInputs(x.to(device), wr, w1, w3, w2, res.to(device), None)
    return inp, torch.from_numpy(bad.astype(np.int64))
