"""A few forwards of one workload, for a profiler to capture (nothing is timed here).

    python -m sparse_mixture_experts_09_b200.profile_run [--path bf16|int8|int4] <workload>

Draws the workload's inputs on the GPU, converts the expert weights once (bf16: the
blocked layout; int8 / int4: the quantised codes), frees the row-major bf16 copies so
that only what the chosen path reads stays on the device, then runs the whole layer
three times and checks the workspace status. A profiler's kernel filter with a skip
count then selects a launch of the second or third forward.
"""
import argparse

import torch

from . import moe as M
from . import workloads as W


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("workload")
    ap.add_argument("--path", choices=("bf16", "int8", "int4"), default="bf16")
    args = ap.parse_args(argv)
    w = W.workload(args.workload)
    inp = W.draw(w, "cuda")
    k = w.num_experts_per_tok
    if args.path == "bf16":
        p1, p3, p2 = M.pack_weights(inp.w1, inp.w3, inp.w2)
        run = lambda ws: M.forward(inp.x, inp.w_router, p1, p3, p2, k, residual=inp.residual,
                                   logit_bias=inp.logit_bias, ws=ws, weight_layout=M.BLOCKED)
        layout = M.BLOCKED
    else:
        quantize, forward = ((M.quantize_int8, M.forward_w8) if args.path == "int8"
                             else (M.quantize_int4, M.forward_w4))
        ex = quantize(inp.w1, inp.w3, inp.w2)
        run = lambda ws: forward(inp.x, inp.w_router, ex, k, residual=inp.residual,
                                 logit_bias=inp.logit_bias, ws=ws)
        layout = M.ROW_MAJOR
    del inp.w1, inp.w3, inp.w2
    torch.cuda.empty_cache()
    ws = M.make_workspace(M.make_shape(*w.shape, layout))
    for _ in range(3):
        out = run(ws)
    torch.cuda.synchronize()
    M.device_status(ws)
    print("ok", args.path, w.name, float(out.float().abs().mean()),
          "%.2f GB peak" % (torch.cuda.max_memory_allocated() / 1e9))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
