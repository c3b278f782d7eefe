"""The benchmark's roofline arithmetic against closed forms: the algorithmic bytes and
flops it divides by the measured kernel time, the bound it picks, and the fraction."""
import bench
from sparse_mixture_experts_09_b200 import workloads as W

PEAKS = {"hbm_gbs": 6556.2, "bf16_tflops": 1613.7, "bf16_tflops_sustained": 1342.7}


def test_decode_gate_up_bytes_and_hbm_bound():
    w = W.WORKLOADS["decode"]            # T=16, H=4096, I=14336, E=8, k=2
    stage_ms = {"router": 0.01, "permute": 0.01, "gate_up": 0.3, "down": 0.15, "combine": 0.01}
    r = bench.kernel_roofline(w, stage_ms, [4] * 8, PEAKS, "measured", False)
    per_expert = 2 * 14336 * 4096 * 2    # w1 + w3 rows of one expert: 234.9 MB
    assert per_expert == 234_881_024
    routed = 16 * 2
    assert r["algorithmic_bytes"] == 8 * per_expert + routed * 4096 * 2 + routed * 14336 * 2
    assert r["kernel"] == "gate_up" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - r["algorithmic_bytes"] / 0.3e-3 / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 6556.2) < 1e-12
    # only experts that received rows are streamed
    r2 = bench.kernel_roofline(w, stage_ms, [16, 16, 0, 0, 0, 0, 0, 0], PEAKS, "measured", False)
    assert r2["active_experts"] == 2
    assert r2["algorithmic_bytes"] == 2 * per_expert + routed * 4096 * 2 + routed * 14336 * 2


def test_prefill_flops_and_tensor_bound():
    w = W.WORKLOADS["prefill"]           # T=4096: 8192 routed rows
    stage_ms = {"router": 0.01, "permute": 0.02, "gate_up": 1.7, "down": 0.85, "combine": 0.03}
    r = bench.kernel_roofline(w, stage_ms, [1024] * 8, PEAKS, "measured", False)
    assert r["kernel"] == "gate_up" and r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["algorithmic_flops"] == 4 * 8192 * 4096 * 14336
    assert r["peak"] == 1613.7 and r["peak_source"] == "measured burst"
    # the whole layer's expert work, 6 R H I = 2.886 TFLOP
    down = bench.kernel_roofline(w, {"down": 1.0}, [1024] * 8, PEAKS, "measured", False)
    assert round((r["algorithmic_flops"] + down["algorithmic_flops"]) / 1e12, 3) == 2.886
    # a long timed region takes the sustained tensor peak
    r_long = bench.kernel_roofline(w, stage_ms, [1024] * 8, PEAKS, "measured", True)
    assert r_long["peak"] == 1342.7 and r_long["peak_source"] == "measured sustained"


class _Proc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler_with(rows):
    import tempfile
    s = bench.ClockSampler()
    s.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
    s.file.write("\n".join(rows) + "\n")
    s.proc = _Proc()
    return s


def test_clock_sampler_reads_loaded_samples_and_reasons():
    # index, bus, util %, sm MHz, max sm MHz, W, active mask, hw_slowdown,
    # hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
    row = "0, 00000000:1B:00.0, {u}, {sm}, 1965, {w}, 0x4, Not Active, Not Active, Not Active, {cap}"
    rows = [row.format(u=0, sm=345, w=120.0, cap="Not Active"),       # idle: ignored
            row.format(u=100, sm=1845, w=700.5, cap="Active"),
            row.format(u=97, sm=1800, w=690.0, cap="Not Active"),
            row.format(u=100, sm=1900, w=707.2, cap="Active")]
    c = _sampler_with(rows).stop()
    assert c["sm_mhz"] == 1845.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"] and c["samples_under_load"] == 3
    assert c["power_w_max"] == 707.2


def test_clock_sampler_reports_slowdowns_and_tolerates_no_samples():
    row = "0, 00000000:1B:00.0, 100, 1200, 1965, 600, 0x8, {hw}, Not Active, {sw}, Not Active"
    c = _sampler_with([row.format(hw="Active", sw="Not Active"),
                       row.format(hw="Not Active", sw="Active")]).stop()
    assert c["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert _sampler_with(["garbage"]).stop() is None
    assert bench.ClockSampler().stop() is None          # nvidia-smi never started


def test_kernels_per_forward_matches_the_launch_lists():
    # the ncu launch lists: 5 kernels per forward at decode (router, plan, gather, the
    # swap-operand kernel for both GEMMs, combine), up to 256 tokens; 6 from 257 tokens
    # (two GEMMs); 8 above 1024 tokens (histogram, scan and rank replace the plan)
    assert bench.kernels_per_forward(16) == 5
    assert bench.kernels_per_forward(64) == 5
    assert bench.kernels_per_forward(65) == 5
    assert bench.kernels_per_forward(256) == 5
    assert bench.kernels_per_forward(257) == 6
    assert bench.kernels_per_forward(16, 4096, 384) == 5
    assert bench.kernels_per_forward(1024) == 6
    assert bench.kernels_per_forward(1025) == 8
    assert bench.kernels_per_forward(4096) == 8
    assert bench.fused_experts(64, 6144, 16384) and not bench.fused_experts(16, 4160, 14336)


def test_experts_stage_roofline_counts_both_gemms():
    w = W.WORKLOADS["decode"]
    H, I, T = w.hidden_size, w.intermediate_size, w.num_tokens
    R = T * 2
    r = bench.kernel_roofline(w, {"router": 0.01, "experts": 0.4}, [4] * 8, PEAKS, "measured", False)
    assert r["kernel"] == "experts" and r["bound"] == "hbm"
    assert r["algorithmic_bytes"] == 8 * 3 * I * H * 2 + R * H * 2 + 2 * R * I * 2 + R * H * 4
    assert r["algorithmic_flops"] == 6 * R * H * I


class _Inputs:
    x = w_router = w1 = w3 = w2 = residual = logit_bias = None


def test_oracle_timing_runs_exactly_max_runs():
    # the reference arm asks for a number of runs with no time budget: every one of
    # them must run (a budget of 0 s must not stop the loop after the first)
    calls = []
    w = W.WORKLOADS["decode"]
    per, runs, n_tok, _ = bench.oracle_timing(_Inputs(), w, budget_s=0.0, max_runs=3,
                                              layer=lambda *a, **kw: calls.append(kw["mode"]))
    assert calls == ["exact"] * 3 and runs == 3 and n_tok == 16
    # with a budget and no run count, at least one run and then the budget decides
    calls.clear()
    bench.oracle_timing(_Inputs(), w, budget_s=0.0, layer=lambda *a, **kw: calls.append(1))
    assert len(calls) == 1


def test_both_arms_print_the_same_config():
    w = W.WORKLOADS["prefill"]
    c = bench.workload_config(w, 1)
    assert c == bench.workload_config(w, 1)
    assert c["parallelism"] == "replicas x1" and c["num_tokens"] == 4096
    # the weights every step reads (at least k experts' 352.3 MB) exceed the L2
    assert "0.70 GB" in c["l2"]


def test_near_tie_tokens_counts_small_gaps_among_the_top_k_plus_one():
    import torch
    logits = torch.tensor([[3.0, 2.0, 1.0, 0.0],      # clear
                           [3.0, 2.995, 1.0, 0.0],    # 1st-2nd tie
                           [3.0, 2.0, 1.995, 0.0],    # 2nd-3rd tie (decides the top 2)
                           [3.0, 2.0, 1.0, 0.995]])   # 3rd-4th: outside the k+1 largest
    assert bench.near_tie_tokens(logits, 2) == 2
    assert bench.near_tie_tokens(logits, 3) == 3
    assert bench.near_tie_tokens(logits[:1], 2) == 0


def test_layer_roofline_against_nominal_and_measured_peaks():
    dec = W.WORKLOADS["decode"]
    r = bench.layer_roofline(dec, 0.5, [4] * 8, PEAKS, "measured", False)
    b = 8 * dec.expert_bytes() + 3 * 16 * 4096 * 2 + 8 * 4096 * 2 + 16 * 2 * 8
    assert r["bound"] == "hbm" and r["algorithmic_bytes"] == b
    assert abs(r["achieved"] - b / 0.5e-3 / 1e9) < 1e-9
    assert abs(r["frac_of_nominal"] - r["achieved"] / 8000.0) < 1e-12
    assert abs(r["frac_of_measured"] - r["achieved"] / 6556.2) < 1e-12
    pre = W.WORKLOADS["prefill"]
    r = bench.layer_roofline(pre, 2.14, [1024] * 8, PEAKS, "measured", False)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    flops = 6 * 8192 * 4096 * 14336 + 2 * 4096 * 4096 * 8
    assert r["algorithmic_flops"] == flops
    # the prefill target: 60% of 2.25 PFLOP/s is a 2.14 ms layer
    assert abs(r["frac_of_nominal"] - 0.6) < 0.002


def test_quantised_layer_roofline_counts_codes_and_scales():
    # decode workload, all 8 experts active: int8 codes are 1 byte per weight plus 4-byte
    # row scales, 4-bit codes half a byte plus one 2-byte scale per 64 weights
    w = W.WORKLOADS["decode"]
    H, I, T = w.hidden_size, w.intermediate_size, w.num_tokens
    peaks = {"hbm_gbs": 6556.0}
    acts = 3 * T * H * 2 + w.num_experts * H * 2 + T * 2 * 8
    r8 = bench.quant_layer_roofline(w, 1.0, [1] * 8, peaks, "measured", 8)
    assert r8["algorithmic_bytes"] == 8 * (3 * H * I + (2 * I + H) * 4) + acts
    r4 = bench.quant_layer_roofline(w, 1.0, [1] * 8, peaks, "measured", 4)
    assert r4["algorithmic_bytes"] == 8 * (3 * H * I // 2 + 3 * H * I // 32) + acts
    # 1 ms per step: GB/s = bytes / 1e6
    assert abs(r8["achieved"] - r8["algorithmic_bytes"] / 1e6) < 1e-6
    assert r4["bound"] == "hbm" and abs(r4["frac_of_measured"] - r4["achieved"] / 6556.0) < 1e-12
    # inactive experts carry no weight bytes
    r8_two = bench.quant_layer_roofline(w, 1.0, [3, 0, 0, 0, 0, 0, 0, 2], peaks, "measured", 8)
    assert r8_two["algorithmic_bytes"] == 2 * (3 * H * I + (2 * I + H) * 4) + acts
