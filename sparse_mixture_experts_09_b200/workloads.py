"""Named synthetic workloads of the Mixtral sparse-MoE feed-forward layer.

Shapes follow the Mixtral pages: hidden_size 4096, intermediate_size 14336,
num_local_experts 8, num_experts_per_tok 2 for 8x7B (Hugging Face "Mixtral" doc,
MixtralConfig; nnterp encyclopedia "Mixtral", Config), intermediate_size 16384 for
8x22B (nnterp "Mixtral", The Notes, "The block, in order"). Token counts, seeds,
distributions and the logit bias of the imbalanced case are the benchmark's own
choices: there is no dataset behind any of them.

Distributions: router, w1 and w3 weights ~ N(0, 1/hidden_size); w2 ~ N(0,
1/intermediate_size); x ~ N(0, 1) (tiny case) or N(0, 1) rows scaled to RMS 1 (all
others); the residual stream is drawn like x. All stored as bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import synth

# tensor ids of the generator streams
X_ID, ROUTER_ID, W1_ID, W3_ID, W2_ID, RESIDUAL_ID, NORM_ID = range(7)
RMS_NORM_EPS = 1e-5  # rms_norm_eps of every Mixtral checkpoint


@dataclass(frozen=True)
class Workload:
    name: str
    num_tokens: int
    hidden_size: int
    intermediate_size: int
    num_experts: int = 8
    num_experts_per_tok: int = 2
    seed: int = 0
    x_unit_rms: bool = True
    logit_bias: Optional[Tuple[float, ...]] = None
    note: str = ""

    @property
    def shape(self):
        return (self.num_tokens, self.hidden_size, self.intermediate_size,
                self.num_experts, self.num_experts_per_tok)

    def with_tokens(self, t: int, name: Optional[str] = None) -> "Workload":
        return Workload(name or f"{self.name}_T{t}", t, self.hidden_size, self.intermediate_size,
                        self.num_experts, self.num_experts_per_tok, self.seed, self.x_unit_rms,
                        self.logit_bias, self.note)

    def expert_bytes(self) -> int:
        """bf16 bytes of one expert's w1, w3 and w2."""
        return 3 * self.hidden_size * self.intermediate_size * 2

    def routed_flops(self) -> int:
        """Multiply-add flops of the experts: 3 GEMMs of 2*H*I per routed (token, slot)."""
        return 6 * self.num_tokens * self.num_experts_per_tok * self.hidden_size * self.intermediate_size

    def router_flops(self) -> int:
        return 2 * self.num_tokens * self.hidden_size * self.num_experts


WORKLOADS = {
    "tiny": Workload("tiny", 64, 128, 256, 8, 2, seed=0, x_unit_rms=False,
                     note="T=64, hidden 128, intermediate 256, x ~ N(0,1)"),
    "decode": Workload("decode", 16, 4096, 14336, 8, 2, seed=1,
                       note="8x7B-shaped layer, batch 16 x seq 1"),
    "prefill": Workload("prefill", 4096, 4096, 14336, 8, 2, seed=2,
                        note="8x7B-shaped layer, batch 1 x seq 4096"),
    "imbalanced_a": Workload("imbalanced_a", 8192, 4096, 14336, 8, 2, seed=3,
                             logit_bias=(3.0, 0, 0, 0, 0, 0, 0, 0),
                             note="+3.0 on expert 0's router logit"),
    "imbalanced_b": Workload("imbalanced_b", 8192, 4096, 14336, 8, 2, seed=3,
                             logit_bias=(3.0, 0, 0, 0, 0, 0, -2.0, -2.0),
                             note="+3.0 on expert 0, -2.0 on experts 6 and 7"),
    "larger": Workload("larger", 2048, 6144, 16384, 8, 2, seed=4,
                       note="8x22B-width experts, hidden 6144"),
}
DECODE_SWEEP_TOKENS = (1, 4, 16, 64, 256)


def decode_sweep():
    return [WORKLOADS["larger"].with_tokens(t, f"larger_decode_T{t}") for t in DECODE_SWEEP_TOKENS]


def workload(name: str) -> "Workload":
    """A named workload, or one of the decode sweep's (larger_decode_T<t>)."""
    if name in WORKLOADS:
        return WORKLOADS[name]
    sweep = {w.name: w for w in decode_sweep()}
    if name in sweep:
        return sweep[name]
    raise KeyError(f"unknown workload {name!r}: one of {sorted(WORKLOADS) + sorted(sweep)}")


@dataclass
class LayerInputs:
    """bf16 tensors of one layer: x [T,H], w_router [E,H], w1/w3 [E,I,H], w2 [E,H,I],
    residual [T,H]; logit_bias [E] fp32 or None."""
    x: torch.Tensor
    w_router: torch.Tensor
    w1: torch.Tensor
    w3: torch.Tensor
    w2: torch.Tensor
    residual: torch.Tensor
    logit_bias: Optional[torch.Tensor]
    x_attempt: Optional[torch.Tensor] = None  # per-row draw attempt (None: all attempt 0)


def draw_x(w: Workload, device="cpu") -> torch.Tensor:
    if w.x_unit_rms:
        return synth.normal_rows_unit_rms(w.num_tokens, w.hidden_size, w.seed, X_ID, 0, device)
    return synth.normal((w.num_tokens, w.hidden_size), 1.0, w.seed, X_ID, 0, device)


def redraw_x_rows(w: Workload, rows: torch.Tensor, attempt: int) -> torch.Tensor:
    """Attempt ``attempt`` of the given rows of x (same distribution as ``draw_x``)."""
    return synth.rows_at(rows, w.hidden_size, 1.0, w.seed, X_ID, attempt, w.x_unit_rms)


def draw_weights(w: Workload, device="cpu"):
    h, i, e = w.hidden_size, w.intermediate_size, w.num_experts
    sh, si = 1.0 / math.sqrt(h), 1.0 / math.sqrt(i)
    wr = synth.normal((e, h), sh, w.seed, ROUTER_ID, 0, device)
    w1 = synth.normal((e, i, h), sh, w.seed, W1_ID, 0, device)
    w3 = synth.normal((e, i, h), sh, w.seed, W3_ID, 0, device)
    w2 = synth.normal((e, h, i), si, w.seed, W2_ID, 0, device)
    return wr, w1, w3, w2


def draw(w: Workload, device="cpu") -> LayerInputs:
    """All inputs of workload ``w`` on ``device`` (no routing-margin screen)."""
    wr, w1, w3, w2 = draw_weights(w, device)
    res = synth.normal_rows_unit_rms(w.num_tokens, w.hidden_size, w.seed, RESIDUAL_ID, 0, device)
    bias = None
    if w.logit_bias is not None:
        bias = torch.tensor(w.logit_bias, dtype=torch.float32, device=device)
    return LayerInputs(draw_x(w, device), wr, w1, w3, w2, res, bias)


def draw_norm_weight(w: Workload, device="cpu") -> torch.Tensor:
    """RMSNorm gain [H] bf16: 1 + 0.1 N(0, 1) (a trained gain sits near one)."""
    z = synth.normal((w.hidden_size,), 0.1, w.seed, NORM_ID, 0, device, dtype=torch.float64)
    return (1.0 + z).to(torch.bfloat16)
