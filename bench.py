#!/usr/bin/env python
"""Throughput of the Mixtral sparse-MoE feed-forward layer on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill|...]
    python bench.py --impl reference ...     # the fp64 CPU oracle on the host cores

A step is one pass of the whole layer (router, scoring, permutation, both expert
GEMMs, combine) over the workload's synthetic batch. ``value`` is tokens/s with every
input resident in HBM, timed with CUDA events around K back-to-back moe_forward calls.
A second loop of K steps runs the same kernels through the split entry points with
events between stages, which gives each kernel's average duration for the roofline
line. ``e2e`` times K calls of moe_forward_host: host-to-device copy of x and the
residual from pinned memory, the layer, device-to-host copy of the output.

Under torchrun every rank runs its own replica of the workload (the layer shards
over independent batches; there is no data-path collective): ``value`` is all ranks'
tokens over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and % of roofline (BF16 tensor peak / HBM BW) at 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "ncu_traffic.json")
GEMM_SOURCE = os.path.join(ROOT, "sparse_mixture_experts_09_b200", "csrc", "gemm_sm100.cu")


def fused_experts(num_tokens: int, hidden: int, inter: int) -> bool:
    """Whether the bf16 layer runs both expert GEMMs as one swap-operand kernel: at most
    256 tokens, hidden and intermediate multiples of 128 (64-row sub-tiles when the
    intermediate size is a multiple of 256 and the batch is small, else 128-row ones)."""
    return num_tokens <= 256 and hidden % 128 == 0 and inter % 128 == 0


def kernels_per_forward(num_tokens: int, hidden: int = 4096, inter: int = 14336) -> int:
    """Kernels one moe_forward launches: router, the permutation (one planning kernel
    up to 1024 tokens, else histogram + scan + rank; then the gather), the expert GEMMs
    (one swap-operand kernel at small batches, else gate/up and down) and the combine."""
    plan = 1 if (num_tokens + 31) // 32 <= 32 else 3
    gemms = 1 if fused_experts(num_tokens, hidden, inter) else 2
    return 1 + plan + 1 + gemms + 1


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="leave out the prefill sub-record of the default line")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_config(w, world=1):
    """The ``config`` object of the JSON line; both arms print the same one."""
    routed_gb = w.num_experts_per_tok * w.expert_bytes() / 1e9
    return {"workload": w.name, "num_tokens": w.num_tokens, "hidden_size": w.hidden_size,
            "intermediate_size": w.intermediate_size, "num_experts": w.num_experts,
            "num_experts_per_tok": w.num_experts_per_tok,
            "logit_bias": list(w.logit_bias) if w.logit_bias else None,
            "parallelism": f"replicas x{world}",
            "l2": ("no flush: every step reads the weights of each routed expert, at least "
                   "%.2f GB, more than the 126 MB L2" % routed_gb)}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock, power and throttle reasons while running."""
    QUERY = ("index,pci.bus_id,utilization.gpu,clocks.sm,clocks.max.sm,power.draw,"
             "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id=None):
        self.bus_id = bus_id
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            cmd = ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.bus_id:
                cmd += ["-i", self.bus_id]
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        with open(self.file.name) as f:
            rows = [r.split(", ") for r in f.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        rows = [r for r in rows if len(r) >= 11]
        if not rows:
            return None
        loaded = [r for r in rows if r[2].strip().isdigit() and int(r[2]) >= 30] or rows
        sm = [float(r[3]) for r in loaded if _isnum(r[3])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(4) if r[7 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(loaded[0][4]) if _isnum(loaded[0][4]) else None,
                "reasons": reasons, "samples_under_load": len(loaded),
                "power_w_max": max(float(r[5]) for r in loaded if _isnum(r[5])) if loaded else None}


def _isnum(s):
    try:
        float(s)
        return True
    except ValueError:
        return False


# ------------------------------------------------------------------ CPU oracle baseline

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else None
    except Exception:
        return None


def oracle_timing(inp_cpu, w, budget_s=0.0, max_runs=None, tokens=None, layer=None):
    """Run the oracle (as it stands) on the workload: exactly ``max_runs`` times when it
    is given, else until ``budget_s`` seconds have passed (at least once). Returns
    (seconds per run, runs, tokens per run, torch threads)."""
    import torch
    if layer is None:
        from oracle import moe_oracle as O
        layer = O.moe_layer
    runs, t0 = 0, time.perf_counter()
    while True:
        layer(inp_cpu.x, inp_cpu.w_router, inp_cpu.w1, inp_cpu.w3, inp_cpu.w2,
              w.num_experts_per_tok, residual=inp_cpu.residual, logit_bias=inp_cpu.logit_bias,
              mode="exact", tokens=tokens)
        runs += 1
        el = time.perf_counter() - t0
        if max_runs is not None:
            if runs >= max_runs:
                break
        elif el >= budget_s:
            break
    n_tok = w.num_tokens if tokens is None else len(tokens)
    return el / runs, runs, n_tok, torch.get_num_threads()


def cpu_sample_tokens(w):
    """Token subset for the CPU baseline: whole batch up to 64 tokens, else 64 tokens."""
    if w.num_tokens <= 64:
        return None
    step = w.num_tokens // 64
    return list(range(0, w.num_tokens, step))[:64]


# ------------------------------------------------------------------ reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    from sparse_mixture_experts_09_b200 import workloads as W
    w = W.workload(args.workload)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = W.draw(w, dev)
    inp = W.LayerInputs(*(None if t is None else t.cpu() for t in
                          (inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, inp.residual, inp.logit_bias)))
    tokens = cpu_sample_tokens(w)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    # probe one step, then size the run to a few minutes
    per_step, _, n_tok, threads = oracle_timing(inp, w, max_runs=1, tokens=tokens)
    budget = 150.0
    steps = max(1, min(args.steps, int((budget - per_step) / per_step) - args.warmup))
    warm = min(args.warmup, max(0, int(budget / per_step) - steps - 1))
    if warm:
        oracle_timing(inp, w, max_runs=warm, tokens=tokens)
    per_step, steps, n_tok, threads = oracle_timing(inp, w, max_runs=steps, tokens=tokens)
    value = n_tok / per_step
    sample = (f"{'all ' if tokens is None else ''}{n_tok} tokens of the {w.name} batch per step, "
              f"fp64 exact mode, {steps} timed steps after {warm} warm-up")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 0,
            "steps": steps, "warmup": warm, "ms_per_step": 1e3 * per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads() or threads,
                             "kind": "oracle", "sample": sample, "host_cpus": os.cpu_count()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def kernel_roofline(w, stage_ms, counts, peaks, peak_kind, long_run):
    """Roofline object of the dominant kernel (largest average duration)."""
    H, I, k, T = w.hidden_size, w.intermediate_size, w.num_experts_per_tok, w.num_tokens
    R = T * k
    n_active = int(sum(1 for c in counts if c > 0))
    wbytes = 2  # bf16
    work = {
        # name: (bytes per launch, flops per launch)
        "router": (T * H * wbytes + w.num_experts * H * wbytes + T * k * 8, 2 * T * H * w.num_experts),
        "permute": (2 * R * H * wbytes + T * k * 12, 0),
        "gate_up": (n_active * 2 * I * H * wbytes + R * H * wbytes + R * I * wbytes, 4 * R * H * I),
        "down": (n_active * H * I * wbytes + R * I * wbytes + R * H * 4, 2 * R * H * I),
        # both GEMMs as one kernel: the weights once, the routed rows, h written and read
        # back, y written
        "experts": (n_active * 3 * I * H * wbytes + R * H * wbytes + 2 * R * I * wbytes + R * H * 4,
                    6 * R * H * I),
        "combine": (R * H * 4 + 2 * T * H * wbytes + T * k * 8, 2 * R * H),
    }
    name = max(stage_ms, key=stage_ms.get)
    bytes_, flops = work[name]
    sec = stage_ms[name] * 1e-3
    hbm_peak = peaks["hbm_gbs"]
    tensor_peak = peaks["bf16_tflops_sustained" if long_run else "bf16_tflops"]
    hbm_time = bytes_ / (hbm_peak * 1e9)
    tensor_time = flops / (tensor_peak * 1e12) if flops else 0.0
    if name in ("gate_up", "down", "experts") and tensor_time > hbm_time:
        r = {"bound": "tensor", "achieved": flops / sec / 1e12, "peak": tensor_peak,
             "unit": "TFLOP/s"}
    else:
        r = {"bound": "hbm", "achieved": bytes_ / sec / 1e9, "peak": hbm_peak, "unit": "GB/s"}
    r["frac"] = r["achieved"] / r["peak"]
    r["kernel"] = name
    r["peak_source"] = peak_kind + (" sustained" if (r["bound"] == "tensor" and long_run) else " burst")
    r["algorithmic_bytes"] = bytes_
    r["algorithmic_flops"] = flops
    r["active_experts"] = n_active
    r["traffic"] = ncu_traffic(w.name, name)
    return r


def ncu_traffic(workload, kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current GEMM source; else None."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
        with open(GEMM_SOURCE, "rb") as f:
            src = hashlib.sha256(f.read()).hexdigest()[:16]
        e = d.get(workload, {}).get(kernel)
        if e and e.get("source_sha256_16") == src:
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def slowest_rank(ms, e2e_ms, world, device):
    """Per-step times of the slowest rank (max over ranks; identity for one rank)."""
    if world == 1:
        return ms, e2e_ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms, e2e_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t[0]), float(t[1])


def job_throughput(tokens_per_rank, world, ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (ms * 1e-3)


NOMINAL = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}   # B200 spec: HBM3e, dense bf16


def layer_roofline(w, ms, counts, peaks, peak_kind, long_run):
    """Whole-layer fraction of roofline: the layer's algorithmic bytes (decode) or expert
    flops (prefill) over the step time, against the nominal B200 peaks (8 TB/s, 2.25
    PFLOP/s dense bf16) and the measured ones."""
    H, I, k, T, E = (w.hidden_size, w.intermediate_size, w.num_experts_per_tok, w.num_tokens,
                     w.num_experts)
    n_active = int(sum(1 for c in counts if c > 0))
    bytes_ = n_active * w.expert_bytes() + 3 * T * H * 2 + E * H * 2 + T * k * 8
    flops = w.routed_flops() + w.router_flops()
    sec = ms * 1e-3
    if flops / (NOMINAL["bf16_tflops"] * 1e12) > bytes_ / (NOMINAL["hbm_gbs"] * 1e9):
        achieved = flops / sec / 1e12
        meas = peaks["bf16_tflops_sustained" if long_run else "bf16_tflops"]
        return {"bound": "tensor", "achieved": achieved, "unit": "TFLOP/s",
                "nominal_peak": NOMINAL["bf16_tflops"], "frac_of_nominal": achieved / NOMINAL["bf16_tflops"],
                "measured_peak": meas, "frac_of_measured": achieved / meas,
                "measured_peak_source": peak_kind + (" sustained" if long_run else " burst"),
                "algorithmic_flops": flops}
    achieved = bytes_ / sec / 1e9
    return {"bound": "hbm", "achieved": achieved, "unit": "GB/s",
            "nominal_peak": NOMINAL["hbm_gbs"], "frac_of_nominal": achieved / NOMINAL["hbm_gbs"],
            "measured_peak": peaks["hbm_gbs"], "frac_of_measured": achieved / peaks["hbm_gbs"],
            "measured_peak_source": peak_kind, "algorithmic_bytes": bytes_}


def quant_layer_roofline(w, ms, counts, peaks, peak_kind, bits):
    """Whole-layer fraction of the HBM roofline for weight-only int8 (bits = 8) or 4-bit
    (bits = 4, plus one 2-byte scale per 64 weights) experts: the active experts' code
    and scale bytes plus the activations' bytes, over the step time. The int8 per-row
    fp32 scales (4 bytes per weight row) are counted too."""
    H, I, k, T, E = (w.hidden_size, w.intermediate_size, w.num_experts_per_tok, w.num_tokens,
                     w.num_experts)
    n_active = int(sum(1 for c in counts if c > 0))
    elems = 3 * H * I  # weights per expert
    per_expert = elems * bits // 8 + (elems // 64 * 2 if bits == 4 else (2 * I + H) * 4)
    bytes_ = n_active * per_expert + 3 * T * H * 2 + E * H * 2 + T * k * 8
    achieved = bytes_ / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "unit": "GB/s",
            "nominal_peak": NOMINAL["hbm_gbs"], "frac_of_nominal": achieved / NOMINAL["hbm_gbs"],
            "measured_peak": peaks["hbm_gbs"], "frac_of_measured": achieved / peaks["hbm_gbs"],
            "measured_peak_source": peak_kind, "algorithmic_bytes": bytes_}


def near_tie_tokens(logits, k, margin=1e-2):
    """Tokens whose float32 router logits have a gap below ``margin`` between any two
    neighbours among their k + 1 largest (the ranks that decide the top-k and its slot
    order). Reported only; the benchmark draws x without the parity tests' screen."""
    import torch
    top = torch.topk(logits, min(k + 1, logits.shape[1]), dim=1).values
    gaps = top[:, :-1] - top[:, 1:]
    return int((gaps < margin).any(dim=1).sum().item())


def _time_loop(fn, K, stream, barrier, dev):
    import torch
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    return e0.elapsed_time(e1) / K


class Bf16Layer:
    """The default (bf16, blocked weights) layer of one workload, ready to time: whole
    forwards, and the split entry points with events between the stages."""

    def __init__(self, w, dev, keep_row_major=False):
        import torch
        from sparse_mixture_experts_09_b200 import moe
        from sparse_mixture_experts_09_b200 import workloads as W
        self.w, self.dev, self.moe = w, dev, moe
        inp = W.draw(w, dev)
        self.inp = inp
        # the expert weights live in the library's blocked layout, converted once at load
        # time (not timed)
        self.bw = moe.pack_weights(inp.w1, inp.w3, inp.w2)
        if not keep_row_major:
            inp.w1 = inp.w3 = inp.w2 = None
            torch.cuda.empty_cache()
        self.k = k = w.num_experts_per_tok
        self.shape = moe.make_shape(*w.shape, moe.BLOCKED)
        self.ws = moe.make_workspace(self.shape, dev)
        self.out = torch.empty((w.num_tokens, w.hidden_size), dtype=torch.bfloat16, device=dev)
        self.stream = torch.cuda.current_stream(dev)
        rmax = moe.max_padded_rows(self.shape)
        T, E = w.num_tokens, w.num_experts
        self.idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.wt = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.logits = torch.empty((T, E), dtype=torch.float32, device=dev)
        self.perm = {"counts": torch.empty(E, dtype=torch.int32, device=dev),
                     "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
                     "row_of": torch.empty((T, k), dtype=torch.int32, device=dev),
                     "token_of_row": torch.empty(rmax, dtype=torch.int32, device=dev),
                     "x_perm": torch.empty((rmax, w.hidden_size), dtype=torch.bfloat16, device=dev)}
        self.hbuf = torch.empty((rmax, w.intermediate_size), dtype=torch.bfloat16, device=dev)
        self.ybuf = torch.empty((rmax, w.hidden_size), dtype=torch.float32, device=dev)
        # at small batches the forward runs both expert GEMMs as one kernel: the split
        # timing then takes them together (the grouped entry point) as stage "experts"
        self.fused = fused_experts(T, w.hidden_size, w.intermediate_size)
        self.stage_names = (["router", "permute", "experts", "combine"] if self.fused
                            else ["router", "permute", "gate_up", "down", "combine"])

    def step(self):
        i, (b1, b3, b2) = self.inp, self.bw
        self.moe.forward(i.x, i.w_router, b1, b3, b2, self.k, residual=i.residual,
                         logit_bias=i.logit_bias, ws=self.ws, out=self.out,
                         weight_layout=self.moe.BLOCKED)

    def split_step(self, ev, logits=False):
        import ctypes
        moe, L, i = self.moe, self.moe.lib(), self.inp
        sp, st = ctypes.byref(self.shape), self.stream.cuda_stream
        p = lambda t: t.data_ptr()  # noqa: E731
        bias = None if i.logit_bias is None else p(i.logit_bias)
        perm, ws = self.perm, self.ws
        ev[0].record(self.stream)
        moe._check(L.moe_router_topk(sp, p(i.x), p(i.w_router), bias, p(self.idx), p(self.wt),
                                     p(self.logits) if logits else None, st))
        ev[1].record(self.stream)
        moe._check(L.moe_permute(sp, p(self.idx), p(i.x), p(perm["counts"]), p(perm["offsets"]),
                                 p(perm["row_of"]), p(perm["token_of_row"]), p(perm["x_perm"]),
                                 p(ws), ws.numel(), st))
        ev[2].record(self.stream)
        if self.fused:
            moe._check(L.moe_grouped_swiglu(sp, p(perm["x_perm"]), p(perm["offsets"]),
                                            p(self.bw[0]), p(self.bw[1]), p(self.bw[2]),
                                            p(self.ybuf), p(ws), ws.numel(), st))
        else:
            moe._check(L.moe_expert_gate_up(sp, p(perm["x_perm"]), p(perm["offsets"]),
                                            p(self.bw[0]), p(self.bw[1]), p(self.hbuf), p(ws),
                                            ws.numel(), st))
            ev[3].record(self.stream)
            moe._check(L.moe_expert_down(sp, p(self.hbuf), p(perm["offsets"]), p(self.bw[2]),
                                         p(self.ybuf), p(ws), ws.numel(), st))
        ev[4 if not self.fused else 3].record(self.stream)
        moe._check(L.moe_combine(sp, p(self.ybuf), p(perm["row_of"]), p(self.wt), p(i.residual),
                                 p(self.out), st))
        ev[5 if not self.fused else 4].record(self.stream)

    def warm(self, n):
        import torch
        scratch = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
        for _ in range(n):
            self.step()
        self.split_step(scratch, logits=True)
        torch.cuda.synchronize(self.dev)
        self.moe.device_status(self.ws)

    def time_forward(self, K, barrier):
        return _time_loop(self.step, K, self.stream, barrier, self.dev)

    def time_stages(self, K):
        import torch
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
        torch.cuda.synchronize(self.dev)
        for i in range(K):
            self.split_step(evs[i])
        torch.cuda.synchronize(self.dev)
        self.moe.device_status(self.ws)
        return {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(K))
                for j, n in enumerate(self.stage_names)}

    def routing_report(self):
        """Expert counts and near-tie tokens of the last split step (untimed)."""
        return (self.perm["counts"].cpu().tolist(),
                near_tie_tokens(self.logits, self.k))


def run_ours(args):
    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_09_b200 import moe
    from sparse_mixture_experts_09_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    moe.lib()  # fail loudly if the library is missing
    w = W.workload(args.workload)
    layer = Bf16Layer(w, dev, keep_row_major=True)
    inp, k = layer.inp, layer.k
    ws, out, stream = layer.ws, layer.out, layer.stream
    bw1, bw3, bw2 = layer.bw
    step = layer.step

    # weight-only int8 experts, quantised once at load time (not timed)
    w8 = moe.quantize_int8(inp.w1, inp.w3, inp.w2)
    ws8 = moe.make_workspace(moe.make_shape(*w.shape), dev)

    def step_w8():
        moe.forward_w8(inp.x, inp.w_router, w8, k, residual=inp.residual,
                       logit_bias=inp.logit_bias, ws=ws8, out=out)

    # weight-only 4-bit experts (a half scale per 64-column group), quantised once
    w4 = moe.quantize_int4(inp.w1, inp.w3, inp.w2)
    ws4 = moe.make_workspace(moe.make_shape(*w.shape), dev)

    def step_w4():
        moe.forward_w4(inp.x, inp.w_router, w4, k, residual=inp.residual,
                       logit_bias=inp.logit_bias, ws=ws4, out=out)

    def step_row_major():
        moe.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, k, residual=inp.residual,
                    logit_bias=inp.logit_bias, ws=ws, out=out)

    xh = inp.x.cpu().pin_memory()
    rh = inp.residual.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    wsh = moe.make_workspace(layer.shape, dev, host=True)

    def host_step(wait=True):
        moe.forward_host(xh, inp.w_router, bw1, bw3, bw2, k, residual_host=rh,
                         logit_bias=inp.logit_bias, ws=wsh, out_host=oh, weight_layout=moe.BLOCKED,
                         wait=wait)

    # the prefill layer rides along with the default (decode) line: the tensor-bound
    # half of the metric
    pre = None
    if args.workload != "prefill" and not args.no_prefill:
        pre = Bf16Layer(W.workload("prefill"), dev)

    K, Wm = args.steps, max(3, args.warmup)
    for _ in range(Wm):
        step_row_major()
        step_w8()
        step_w4()
    layer.warm(Wm)
    if pre is not None:
        pre.warm(Wm)
    for _ in range(3):
        host_step()
    torch.cuda.synchronize(dev)
    # the same forward captured once in a CUDA graph (replayed in loop 5)
    # thread-local capture: other threads (a process group's watchdog) may use CUDA
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        step()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize(dev)
    moe.device_status(ws)
    counts, near_ties = layer.routing_report()
    barrier()

    bus = None
    try:
        props = torch.cuda.get_device_properties(dev)
        bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    except Exception:
        pass
    clocks = ClockSampler(bus)
    clocks.start()
    time.sleep(0.3)

    # (1) value: K back-to-back moe_forward calls, inputs resident in HBM
    ms = layer.time_forward(K, barrier)
    # (2) per-kernel breakdown through the split entry points
    stage_ms = layer.time_stages(K)
    # (2b) the same layer with row-major expert weights
    rm_ms = _time_loop(step_row_major, K, stream, barrier, dev)
    # (3) end to end from pinned host memory, waiting after every call
    e2e_sync_ms = _time_loop(host_step, K, stream, barrier, dev)
    # (3b) the same host path as a serving loop runs it: every step enqueued back to back
    #      (moe_forward_host_async: copy in, layer, copy out), one wait at the end
    e2e_ms = _time_loop(lambda: host_step(wait=False), K, stream, barrier, dev)
    # (4) the same layer with weight-only int8 experts, (4b) 4-bit experts
    w8_ms = _time_loop(step_w8, K, stream, barrier, dev)
    w4_ms = _time_loop(step_w4, K, stream, barrier, dev)
    # (5) the default forward replayed from a CUDA graph
    graph_ms = _time_loop(graph.replay, K, stream, barrier, dev)
    clk = clocks.stop()
    for b in (ws, wsh, ws8, ws4):
        moe.device_status(b)

    # (6) the prefill layer: whole forwards, then the stage breakdown
    pre_rec = None
    if pre is not None:
        pclk = ClockSampler(bus)
        pclk.start()
        time.sleep(0.3)
        pms = pre.time_forward(K, barrier)
        pstage = pre.time_stages(K)
        pclocks = pclk.stop()
        pms, _ = slowest_rank(pms, pms, world, dev)
        pcounts, pnear = pre.routing_report()
        peaks, peak_kind = load_peaks()
        plong = pms * K > 1000.0
        pre_rec = {"workload": pre.w.name, "config": workload_config(pre.w, world),
                   "value": job_throughput(pre.w.num_tokens, world, pms), "unit": "tokens/s",
                   "ms_per_step": pms, "steps": K,
                   "layer_roofline": layer_roofline(pre.w, pms, pcounts, peaks, peak_kind, plong),
                   "roofline": kernel_roofline(pre.w, pstage, pcounts, peaks, peak_kind, plong),
                   "kernels_ms": pstage, "expert_counts": pcounts, "near_ties": pnear,
                   "clocks": pclocks,
                   "gpu_launches": kernels_per_forward(pre.w.num_tokens, pre.w.hidden_size,
                                                       pre.w.intermediate_size) * K}

    ms, e2e_ms = slowest_rank(ms, e2e_ms, world, dev)
    e2e_sync_ms, _ = slowest_rank(e2e_sync_ms, e2e_sync_ms, world, dev)
    rm_ms, _ = slowest_rank(rm_ms, rm_ms, world, dev)
    w8_ms, _ = slowest_rank(w8_ms, w8_ms, world, dev)
    w4_ms, _ = slowest_rank(w4_ms, w4_ms, world, dev)
    graph_ms, _ = slowest_rank(graph_ms, graph_ms, world, dev)

    peaks, peak_kind = load_peaks()
    long_run = ms * K > 1000.0
    roof = kernel_roofline(w, stage_ms, counts, peaks, peak_kind, long_run)

    line = None
    if rank == 0:
        bytes_io = w.num_tokens * w.hidden_size * 2
        n_active = roof["active_experts"]
        line = {
            "metric": METRIC, "value": job_throughput(w.num_tokens, world, ms), "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": Wm, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded SplitMix64/Box-Muller draws, weights ~N(0,1/fan_in), x rows RMS 1",
            "config": workload_config(w, world),
            "weight_layout": "blocked (moe_pack_weights once at load, untimed)",
            "roofline": roof,
            "layer_roofline": layer_roofline(w, ms, counts, peaks, peak_kind, long_run),
            "kernels_ms": stage_ms,
            "row_major_weights": {"ms_per_step": rm_ms,
                                  "value": job_throughput(w.num_tokens, world, rm_ms)},
            "cuda_graph": {"ms_per_step": graph_ms,
                           "value": job_throughput(w.num_tokens, world, graph_ms),
                           "note": "the default forward captured once, replayed"},
            "int8_experts": {"ms_per_step": w8_ms,
                             "value": job_throughput(w.num_tokens, world, w8_ms),
                             "api": "moe_forward_w8",
                             "weight_gb_per_step": n_active * w.expert_bytes() / 2e9,
                             "layer_roofline": quant_layer_roofline(w, w8_ms, counts, peaks,
                                                                    peak_kind, 8),
                             "note": "weight-only int8 experts, half-precision expert math, "
                                     "quantised once at load (untimed); not the headline"},
            "int4_experts": {"ms_per_step": w4_ms,
                             "value": job_throughput(w.num_tokens, world, w4_ms),
                             "api": "moe_forward_w4",
                             "weight_gb_per_step": (n_active * w.expert_bytes()
                                                    * (1 / 4 + 1 / 64) / 1e9),
                             "layer_roofline": quant_layer_roofline(w, w4_ms, counts, peaks,
                                                                    peak_kind, 4),
                             "note": "weight-only 4-bit experts (a half scale per 64-column "
                                     "group), half-precision expert math, quantised once at "
                                     "load (untimed); not the headline"},
            "e2e": {"value": job_throughput(w.num_tokens, world, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": 2 * bytes_io, "d2h_bytes_per_step": bytes_io,
                    "api": "moe_forward_host_async, steps enqueued back to back, one wait",
                    "per_call_wait": {"value": job_throughput(w.num_tokens, world, e2e_sync_ms),
                                      "api": "moe_forward_host (waits every step)"}},
            "gpu_launches": kernels_per_forward(w.num_tokens, w.hidden_size,
                                                w.intermediate_size) * K,
            "clocks": clk,
            "expert_counts": counts,
            "near_ties": {"tokens": near_ties, "margin": 1e-2,
                          "rule": "float32 router logits, gap below the margin between neighbours "
                                  "among the k+1 largest"},
        }
        if pre_rec is not None:
            line["prefill"] = pre_rec
            line["gpu_launches"] += pre_rec["gpu_launches"]
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            cpu = W.LayerInputs(*(None if t is None else t.cpu() for t in
                                  (inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, inp.residual,
                                   inp.logit_bias)))
            tokens = cpu_sample_tokens(w)
            per, runs, n_tok, threads = oracle_timing(cpu, w, args.cpu_seconds, tokens=tokens)
            line["cpu_baseline"] = {
                "value": n_tok / per, "unit": "tokens/s", "cores": blas_threads() or threads,
                "kind": "oracle", "host_cpus": os.cpu_count(),
                "sample": (f"{'all ' if tokens is None else ''}{n_tok} tokens of the {w.name} batch "
                           f"through the fp64 oracle (exact mode), {runs} runs, {per:.2f} s each")}
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
