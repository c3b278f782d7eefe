"""The oracle's pins are strong enough: each mistake below, planted in an in-memory
copy of the oracle (on the CPU; the oracle's file is untouched), makes at least one
of the named pins in test_oracle.py fail. Every mistake is a plausible slip in one
step of the layer: a wrong sign, a dropped term or rounding, a swapped operand, an
off-by-one in a constant."""
import inspect
import types

import pytest

from oracle import moe_oracle as O

from . import test_oracle as T

# (planted change: exact text -> replacement, pins that must catch it)
MUTATIONS = [
    ("to_f64(x) @ to_f64(w_router).T", "to_f64(x) @ to_f64(w_router).T * 1.001",
     ["test_router_logits_pick_columns"]),
    ("logits = logits + to_f64(logit_bias)[None, :]", "logits = logits - to_f64(logit_bias)[None, :]",
     ["test_router_logits_pick_columns"]),
    ("        logits = round_bf16(logits)", "        logits = logits",
     ["test_bf16_logits_round_before_scoring_and_ties_go_low"]),
    ("p = p / p.sum(axis=1, keepdims=True)", "p = p / p.sum(axis=1, keepdims=True) ** 0.999",
     ["test_route_closed_form_example", "test_route_weights_sum_to_one_and_match_two_logit_softmax"]),
    ("weights = top / top.sum(axis=1, keepdims=True)", "weights = top",
     ["test_route_closed_form_example", "test_route_weights_sum_to_one_and_match_two_logit_softmax"]),
    ('order = np.argsort(-key32[t].astype(np.float64), kind="stable")',
     'order = np.argsort(key32[t].astype(np.float64), kind="stable")[::-1]',
     ["test_route_ties_to_lower_index_and_k1", "test_route_brute_force_pair_search"]),
    ("key32 = logits.astype(np.float32)", "key32 = logits",
     ["test_route_topk_ranks_float32_logits_ties_low"]),
    ("padded = (count + pad - 1) // pad * pad", "padded = (count + pad) // pad * pad",
     ["test_stable_permute_offsets_closed_form"]),
    ("    for t in range(t_count):\n        for j in range(k):\n            e = idx[t, j]",
     "    for j in range(k):\n        for t in range(t_count):\n            e = idx[t, j]",
     [("test_stable_permute_against_library_sort", (37, 8, 2))]),
    ("return g / (1.0 + np.exp(-g))", "return g / (1.0 + np.exp(g))",
     ["test_silu_closed_forms"]),
    ("    h = silu(g) * u", "    h = silu(u) * g",
     ["test_single_expert_top1_is_plain_swiglu_mlp"]),
    ("    if h_bf16:\n        h = round_bf16(h)", "    if h_bf16:\n        h = h",
     ["test_bf16_storage_mode_rounds_h_and_out_closed_form"]),
    ("    expert_outputs = weights[:, :, None] * y", "    expert_outputs = y",
     ["test_slot_sum_and_ablation_invariants", ("test_sparse_layer_equals_dense_masked_evaluation", (4, 2))]),
    ("        out = res + routed", "        out = res - routed",
     ["test_block_is_residual_plus_layer_on_normed_input"]),
    ("    if storage:\n        out = round_bf16(out)", "    if storage:\n        out = out",
     ["test_bf16_storage_mode_rounds_h_and_out_closed_form"]),
    ('    x_experts = round_f16(xs) if mode == "f16_experts" else xs', "    x_experts = xs",
     ["test_f16_expert_mode_reads_x_rounded_to_half"]),
    ("            y[tok, slot] = round_f16(h) @ to_f64(w2[e]).T", "            y[tok, slot] = h @ to_f64(w2[e]).T",
     ["test_f16_expert_mode_differs_from_exact_by_f16_rounding_of_h"]),
    ("quantum = np.ldexp(1.0, np.maximum(e, -125) - 8)", "quantum = np.ldexp(1.0, np.maximum(e, -125) - 9)",
     ["test_round_bf16_ties_to_even_closed_form"]),
    ("quantum = np.ldexp(1.0, np.maximum(e, -13) - 11)", "quantum = np.ldexp(1.0, np.maximum(e, -14) - 11)",
     ["test_round_f16_closed_forms"]),
    ("return h / np.sqrt(ms + eps) * to_f64(weight)[None, :]",
     "return h / (np.sqrt(ms) + eps) * to_f64(weight)[None, :]",
     ["test_rms_norm_matches_torch_and_closed_form"]),
    ("return h / np.sqrt(ms + eps) * to_f64(weight)[None, :]", "return h / np.sqrt(ms + eps)",
     ["test_rms_norm_matches_torch_and_closed_form"]),
    ("residual=hs, logit_bias=logit_bias, mode=mode)", "residual=x, logit_bias=logit_bias, mode=mode)",
     ["test_block_is_residual_plus_layer_on_normed_input"]),
    ("amax / np.float32(127.0)", "amax / np.float32(128.0)",
     ["test_int8_rows_bounds_and_extremes", "test_int8_codes_match_torch_float32_arithmetic"]),
    ("(amax / np.float32(7.0))", "(amax / np.float32(8.0))",
     ["test_int4_groups_closed_form"]),
    ("q = np.rint(g / s16.astype(np.float32)[..., None])", "q = np.floor(g / s16.astype(np.float32)[..., None])",
     ["test_int4_groups_nearest_code_brute_force"]),
    ("q = np.clip(q, -7, 7)", "q = np.clip(q, -8, 7)",
     ["test_int4_groups_degenerate_groups_and_bound"]),
    ("s16 = np.where(s16 == 0, 1.0, s16)", "s16 = np.where(s16 == 0, 0.0, s16)",
     ["test_int4_groups_degenerate_groups_and_bound"]),
    ("return round_f16(prod).reshape(q.shape)", "return prod.reshape(q.shape)",
     ["test_int4_groups_match_torch_arithmetic"]),
]


def _mutant(old: str, new: str):
    src = inspect.getsource(O)
    assert src.count(old) == 1, f"the planted text must occur once: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = O.__file__
    exec(compile(src.replace(old, new), O.__file__, "exec"), mod.__dict__)
    return mod


def test_unmutated_oracle_passes_the_named_pins(monkeypatch):
    monkeypatch.setattr(T, "O", _mutant("def silu(", "def silu("))
    for _, _, pins in MUTATIONS:
        for pin in pins:
            name, args = pin if isinstance(pin, tuple) else (pin, ())
            getattr(T, name)(*args)


@pytest.mark.parametrize("old,new,pins", MUTATIONS, ids=[f"m{i}" for i in range(len(MUTATIONS))])
def test_planted_mistake_fails_a_pin(monkeypatch, old, new, pins):
    monkeypatch.setattr(T, "O", _mutant(old, new))
    failed = []
    for pin in pins:
        name, args = pin if isinstance(pin, tuple) else (pin, ())
        try:
            with _quiet():
                getattr(T, name)(*args)
        except AssertionError:
            failed.append(name)
    assert failed, f"no pin caught {new!r}"


class _quiet:
    def __enter__(self):
        import warnings
        self._w = warnings.catch_warnings()
        self._w.__enter__()
        warnings.simplefilter("ignore")

    def __exit__(self, *exc):
        return self._w.__exit__(*exc)
