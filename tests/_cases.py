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
