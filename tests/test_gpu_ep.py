"""Expert parallelism on one GPU: the row-gather kernel; the expert-parallel layer over
a one-rank NCCL group, whose exchanges are then identities, equal to moe_forward bit
for bit (same routing, same groups, same GEMM tiles) and to the fp64 oracle; and the
layer over two ranks (two processes on the GPU, rows exchanged through host memory)
against the oracle, with bf16, int8 and 4-bit experts."""
import datetime
import socket

import pytest
import torch
import torch.distributed as dist

from sparse_mixture_experts_09_b200 import ep
from sparse_mixture_experts_09_b200 import moe as M
from sparse_mixture_experts_09_b200 import workloads as W

from ._cases import screened
from .test_gpu_kernels import SMALL

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,width", [(torch.bfloat16, 136), (torch.float32, 4096),
                                         (torch.bfloat16, 8)])
def test_gather_rows_matches_indexing(dtype, width):
    g = torch.Generator(device="cuda").manual_seed(3)
    src = torch.randn(1000, width, generator=g, device="cuda").to(dtype)
    index = torch.randint(-3, 1003, (2500,), generator=g, device="cuda")
    out = M.gather_rows(src, index)
    torch.cuda.synchronize()
    ok = (index >= 0) & (index < src.shape[0])
    want = torch.zeros_like(out)
    want[ok] = src[index[ok]]
    assert torch.equal(out, want)
    assert M.gather_rows(src, index[:0]).shape == (0, width)


def test_gather_rows_rejects_bad_rows():
    src = torch.zeros(4, 3, dtype=torch.bfloat16, device="cuda")   # 6-byte rows
    with pytest.raises(M.MoeError):
        M.gather_rows(src, torch.zeros(2, dtype=torch.int64, device="cuda"))


@pytest.fixture(scope="module")
def one_rank_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield None
    dist.destroy_process_group()


@pytest.mark.parametrize("name", ["tiny", "ragged", "e64k8", "skewed"])
def test_expert_parallel_one_rank_equals_forward(one_rank_group, name):
    w = SMALL[name]
    inp, _ = screened(w)
    k = w.num_experts_per_tok
    want = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, k, residual=inp.residual,
                     logit_bias=inp.logit_bias)
    l1, l3, l2 = ep.shard_experts(inp.w1, inp.w3, inp.w2, 0, 1)
    got = ep.forward_ep(inp.x, inp.w_router, l1, l3, l2, k, w.num_experts,
                        residual=inp.residual, logit_bias=inp.logit_bias)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    # and the routed output against the fp64 oracle
    routed = ep.forward_ep(inp.x, inp.w_router, l1, l3, l2, k, w.num_experts,
                           logit_bias=inp.logit_bias)
    from oracle import moe_oracle as O
    from ._cases import assert_layer_close
    assert_layer_close(O.to_f64(routed.cpu()), _oracle_out(w, inp, "bf16"), name)


@pytest.mark.parametrize("mode", ["int8", "int4"])
def test_expert_parallel_quantized_one_rank_matches_oracle(one_rank_group, mode):
    from oracle import moe_oracle as O
    from ._cases import assert_layer_close
    w = SMALL["ragged"]
    inp, _ = screened(w)
    quant = M.quantize_int8 if mode == "int8" else M.quantize_int4
    local = ep.shard_quantized(quant(inp.w1, inp.w3, inp.w2), 0, 1)
    got = ep.forward_ep_quantized(inp.x, inp.w_router, local, w.num_experts_per_tok,
                                  w.num_experts, logit_bias=inp.logit_bias)
    torch.cuda.synchronize()
    assert_layer_close(O.to_f64(got.cpu()), _oracle_out(w, inp, mode), mode)


def test_expert_parallel_one_rank_decode(one_rank_group):
    # moe_forward sums the experts' products in another fp32 order than the expert-
    # parallel path at small batches (a split down GEMM, or the swap-operand kernel's
    # partial sums), so a few outputs may round to the neighbouring bf16 value: both
    # against the oracle, and within one bf16 unit in the last place of each other (at
    # most 2^-7 of the largest output), with a tight mean
    from oracle import moe_oracle as O
    from ._cases import assert_layer_close
    w = W.WORKLOADS["decode"]
    inp, near = screened(w)
    assert near.numel() == 0
    want = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, 2)
    got = ep.forward_ep(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, 2, w.num_experts)
    torch.cuda.synchronize()
    ref = _oracle_out(w, inp, "bf16")
    assert_layer_close(O.to_f64(got.cpu()), ref, "decode, expert parallel")
    assert_layer_close(O.to_f64(want.cpu()), ref, "decode, moe_forward")
    from ._cases import layer_errors
    max_rel, mae = layer_errors(O.to_f64(got.cpu()), O.to_f64(want.cpu()))
    assert max_rel <= 2.0 ** -7 and mae <= 1e-4, (max_rel, mae)


# ---- two ranks on one GPU, the exchange staged through gloo on the host ----
#
# Each rank is its own process with its own CUDA context on the same GPU. The rows cross
# between ranks through torch.distributed's gloo all_to_all on host copies, so no kernel
# ever waits on another rank: every wait is in the host collective. The layer's steps
# are the library's kernels (CudaOps), the exchange plan is ep.exchange_plan, and the
# two ranks' outputs together are checked against the fp64 oracle.

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _host_exchange(out, inp, out_splits=None, in_splits=None, group=None):
    """all_to_all_single through host memory (gloo); rows of 2-D tensors move as bytes."""
    cast = (lambda t: t.view(torch.uint8)) if inp.dim() == 2 else (lambda t: t)
    got = torch.empty(out.shape, dtype=out.dtype)
    dist.all_to_all_single(cast(got), cast(inp.contiguous().cpu()), out_splits, in_splits,
                           group=group)
    out.copy_(got)


def _token_split(t, world):
    cuts = [0, (3 * t) // 8, t] if world == 2 else [round(t * r / world) for r in range(world + 1)]
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def _ep_rank(rank, world, port, q, name, mode):
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as D
    from sparse_mixture_experts_09_b200 import ep as EP
    from sparse_mixture_experts_09_b200 import moe as MM
    from tests._cases import screened as scr
    from tests.test_gpu_kernels import SMALL as S
    D.init_process_group("gloo", rank=rank, world_size=world,
                         timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(0)
    w = S[name]
    inp, _ = scr(w)
    lo, hi = _token_split(w.num_tokens, world)[rank]
    k, e = w.num_experts_per_tok, w.num_experts
    if mode == "bf16":
        l1, l3, l2 = EP.shard_experts(inp.w1, inp.w3, inp.w2, rank, world)
        out = EP.forward_ep(inp.x[lo:hi], inp.w_router, l1, l3, l2, k, e,
                            logit_bias=inp.logit_bias, exchange=_host_exchange)
    else:
        quant = MM.quantize_int8 if mode == "int8" else MM.quantize_int4
        local = EP.shard_quantized(quant(inp.w1, inp.w3, inp.w2), rank, world)
        out = EP.forward_ep_quantized(inp.x[lo:hi], inp.w_router, local, k, e,
                                      logit_bias=inp.logit_bias, exchange=_host_exchange)
    torch.cuda.synchronize()
    q.put((rank, out.cpu().view(torch.int16).numpy().copy()))
    D.barrier()
    D.destroy_process_group()


def _oracle_out(w, inp, mode):
    import numpy as np
    from oracle import moe_oracle as O
    from ._cases import to_cpu
    c = to_cpu(inp)
    k = w.num_experts_per_tok
    if mode == "bf16":
        return O.moe_layer(c.x, c.w_router, c.w1, c.w3, c.w2, k, logit_bias=c.logit_bias,
                           mode="bf16_storage")["out"]
    if mode == "int8":
        deq = []
        for t in (c.w1, c.w3, c.w2):
            qq, s = O.quantize_int8_rows(t)
            deq.append(qq.astype(np.float64) * s.astype(np.float64)[..., None])
    else:
        deq = [O.dequantize_int4_groups(*O.quantize_int4_groups(t)) for t in (c.w1, c.w3, c.w2)]
    return O.moe_layer(c.x, c.w_router, *deq, k, logit_bias=c.logit_bias, mode="f16_experts")["out"]


@pytest.mark.parametrize("name,mode", [("ragged", "bf16"), ("e64k8", "bf16"), ("skewed", "bf16"),
                                       ("ragged", "int8"), ("ragged", "int4")])
def test_expert_parallel_two_ranks_matches_oracle(name, mode):
    import numpy as np
    import torch.multiprocessing as mp
    from oracle import moe_oracle as O
    from ._cases import assert_layer_close
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_rank, args=(r, world, port, q, name, mode))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    bits = np.concatenate([got[r] for r in range(world)])
    out = torch.from_numpy(bits).view(torch.bfloat16)
    w = SMALL[name]
    inp, near = screened(w)
    assert near.numel() == 0
    assert_layer_close(O.to_f64(out), _oracle_out(w, inp, mode), f"{name} {mode} over 2 ranks")


# ---- the peer-memory exchange (ep.peer_plan, moe_scatter_rows_peer, moe_combine_peer) ----
#
# An emulated world in one process: every rank's receive buffers are separate
# allocations on the one GPU, addressed through the same pointer tables a multi-GPU run
# builds from IPC mappings. The steps run rank after rank (route and permute, store the
# rows into the owners' groups, every owner's experts, every rank's combine), so no
# kernel waits on another rank. The outputs are checked against the fp64 oracle.

def _emulated_peer_world(w, inp, world, mode):
    ops = ep.CudaOps()
    k, e = w.num_experts_per_tok, w.num_experts
    h, inter = w.hidden_size, w.intermediate_size
    e_loc = e // world
    splits = _token_split(w.num_tokens, world)
    rows = ep.peer_rows_needed(max(hi - lo for lo, hi in splits), k, world, e_loc)
    xs = [torch.zeros((rows, h), dtype=torch.bfloat16, device="cuda") for _ in range(world)]
    ys = [torch.zeros((rows, h), dtype=torch.float32, device="cuda") for _ in range(world)]
    x_bases = torch.tensor([t.data_ptr() for t in xs], dtype=torch.int64, device="cuda")
    y_bases = torch.tensor([t.data_ptr() for t in ys], dtype=torch.int64, device="cuda")
    perms, wts = [], []
    for lo, hi in splits:
        if hi > lo:
            idx, wt = ops.router_topk(inp.x[lo:hi], inp.w_router, k, inp.logit_bias)
            perm = ops.permute(idx, inp.x[lo:hi], e, inter)
        else:
            wt = None
            perm = {"offsets": torch.zeros(e + 1, dtype=torch.int32, device="cuda"),
                    "counts": torch.zeros(e, dtype=torch.int32, device="cuda"),
                    "x_perm": torch.empty((0, h), dtype=torch.bfloat16, device="cuda")}
        perms.append(perm)
        wts.append(wt)
    counts_all = torch.stack([p["counts"].to(torch.int64) for p in perms])
    plans = [ep.peer_plan(perms[r]["offsets"], counts_all, r, world, device="cuda")
             for r in range(world)]
    for r in range(world):
        ops.scatter_rows_peer(perms[r]["x_perm"], plans[r]["send_index"], plans[r]["dst_rank"],
                              plans[r]["dst_row"], x_bases, rows)
    torch.cuda.synchronize()
    if mode == "bf16":
        shards = [ep.shard_experts(inp.w1, inp.w3, inp.w2, r, world) for r in range(world)]
    else:
        quant = M.quantize_int8 if mode == "int8" else M.quantize_int4
        full = quant(inp.w1, inp.w3, inp.w2)
        shards = [ep.shard_quantized(full, r, world) for r in range(world)]
    for r in range(world):
        n_recv = plans[r]["n_recv"]
        rows_buf = ops.padded_rows(n_recv, e_loc)
        assert rows_buf <= rows
        off = torch.tensor(plans[r]["local_offsets"], dtype=torch.int32, device="cuda")
        if mode == "bf16":
            ops.grouped_swiglu(xs[r][:rows_buf], off, *shards[r], n_recv, y=ys[r][:rows_buf])
        else:
            ops.grouped_swiglu_quantized(xs[r][:rows_buf], off, shards[r], n_recv,
                                         y=ys[r][:rows_buf])
    torch.cuda.synchronize()
    outs = []
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    for r, (lo, hi) in enumerate(splits):
        if hi == lo:
            continue
        row_of = perms[r]["row_of"].to(torch.int64).reshape(-1)
        slot_rank = plans[r]["row_rank"][row_of].contiguous()
        slot_row = plans[r]["row_dst"][row_of].contiguous()
        outs.append(M.combine_peer(y_bases, rows, slot_rank, slot_row, wts[r], h, bad=bad))
    torch.cuda.synchronize()
    assert int(bad) == 0
    return torch.cat(outs)


@pytest.mark.parametrize("name,world,mode", [("ragged", 2, "bf16"), ("ragged", 4, "bf16"),
                                             ("e64k8", 4, "bf16"), ("skewed", 2, "bf16"),
                                             ("one_token", 2, "bf16"), ("ragged", 2, "int8"),
                                             ("ragged", 4, "int4")])
def test_peer_exchange_emulated_world_matches_oracle(name, world, mode):
    from oracle import moe_oracle as O
    from ._cases import assert_layer_close
    w = SMALL[name]
    inp, near = screened(w)
    assert near.numel() == 0
    out = _emulated_peer_world(w, inp, world, mode)
    assert_layer_close(O.to_f64(out.cpu()), _oracle_out(w, inp, mode),
                       f"{name} {mode}, {world} emulated ranks over peer buffers")


def test_peer_scatter_and_combine_skip_and_count_bad_indices():
    # out-of-range ranks and rows are skipped (no access leaves the buffers) and counted
    src = torch.arange(4 * 8, dtype=torch.float32, device="cuda").reshape(4, 8)
    dst = [torch.full((3, 8), -1.0, device="cuda") for _ in range(2)]
    bases = torch.tensor([t.data_ptr() for t in dst], dtype=torch.int64, device="cuda")
    bad = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = torch.tensor([0, 1, 2, 3, 9], dtype=torch.int64, device="cuda")
    rank = torch.tensor([0, 1, 2, 1, 0], dtype=torch.int32, device="cuda")
    row = torch.tensor([2, 0, 0, 5, 1], dtype=torch.int64, device="cuda")
    M.scatter_rows_peer(src, idx, rank, row, bases, 3, bad=bad)
    torch.cuda.synchronize()
    assert int(bad) == 3
    assert torch.equal(dst[0][2], src[0]) and torch.equal(dst[1][0], src[1])
    assert (dst[0][:2] == -1).all() and (dst[1][1:] == -1).all()
    y = [torch.ones((2, 8), device="cuda"), 2 * torch.ones((2, 8), device="cuda")]
    y_bases = torch.tensor([t.data_ptr() for t in y], dtype=torch.int64, device="cuda")
    bad.zero_()
    w = torch.tensor([[0.5, 0.25], [1.0, 1.0]], device="cuda")
    out = M.combine_peer(y_bases, 2, torch.tensor([[0, 1], [1, 7]], dtype=torch.int32, device="cuda"),
                         torch.tensor([[1, 0], [3, 0]], dtype=torch.int64, device="cuda"), w, 8, bad=bad)
    torch.cuda.synchronize()
    assert int(bad) == 2
    assert (out[0].float() == 1.0).all() and (out[1].float() == 0.0).all()


# Two processes on the one GPU, each with its own context: the buffers are the
# library's IPC allocations (PeerBuffers), each process maps the other's, and the layer
# runs through ep.forward_ep_peer. Counts, handles and barriers go through gloo on the
# host; the stores and loads go to the other process's memory directly.

def _ep_peer_rank(rank, world, port, q, name, mode):
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as D
    from sparse_mixture_experts_09_b200 import ep as EP
    from sparse_mixture_experts_09_b200 import moe as MM
    from tests._cases import screened as scr
    from tests.test_gpu_kernels import SMALL as S
    D.init_process_group("gloo", rank=rank, world_size=world,
                         timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(0)
    w = S[name]
    inp, _ = scr(w)
    lo, hi = _token_split(w.num_tokens, world)[rank]
    k, e = w.num_experts_per_tok, w.num_experts
    longest = max(b - a for a, b in _token_split(w.num_tokens, world))
    bufs = EP.PeerBuffers(EP.peer_rows_needed(longest, k, world, e // world), w.hidden_size)

    def gather_counts(c):
        parts = [torch.empty_like(c.cpu()) for _ in range(world)]
        D.all_gather(parts, c.cpu())
        return torch.stack(parts).cuda()

    if mode == "bf16":
        l1, l3, l2 = EP.shard_experts(inp.w1, inp.w3, inp.w2, rank, world)
        out = EP.forward_ep_peer(inp.x[lo:hi], inp.w_router, l1, l3, l2, k, e, bufs,
                                 logit_bias=inp.logit_bias, gather_counts=gather_counts)
    else:
        quant = MM.quantize_int8 if mode == "int8" else MM.quantize_int4
        local = EP.shard_quantized(quant(inp.w1, inp.w3, inp.w2), rank, world)
        out = EP.forward_ep_peer_quantized(inp.x[lo:hi], inp.w_router, local, k, e, bufs,
                                           logit_bias=inp.logit_bias, gather_counts=gather_counts)
    torch.cuda.synchronize()
    q.put((rank, out.cpu().view(torch.int16).numpy().copy()))
    bufs.close()
    D.barrier()
    D.destroy_process_group()


@pytest.mark.parametrize("name,mode", [("ragged", "bf16"), ("skewed", "bf16"), ("ragged", "int8")])
def test_peer_exchange_two_processes_match_oracle(name, mode):
    import numpy as np
    import torch.multiprocessing as mp
    from oracle import moe_oracle as O
    from ._cases import assert_layer_close
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_peer_rank, args=(r, world, port, q, name, mode))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    bits = np.concatenate([got[r] for r in range(world)])
    out = torch.from_numpy(bits).view(torch.bfloat16)
    w = SMALL[name]
    inp, near = screened(w)
    assert near.numel() == 0
    assert_layer_close(O.to_f64(out), _oracle_out(w, inp, mode),
                       f"{name} {mode} over 2 processes, peer buffers")
