"""fp64 CPU oracle of the sparse-MoE layer: test infrastructure only.

Only the test suite, the package smoke check and the benchmark's CPU-baseline leg
may import this package. The CUDA path never imports it and shares no code with it.
"""
from .moe_oracle import (to_f64, round_bf16, round_f16, silu, router_logits, route_topk,  # noqa: F401
                         stable_permute, swiglu_expert, moe_layer, rms_norm, moe_block,
                         quantize_int8_rows, quantize_int4_groups, dequantize_int4_groups)
