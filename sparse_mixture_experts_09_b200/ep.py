"""Expert parallelism: the layer with its experts spread over the ranks of a process
group, one process per GPU.

The pages note that a Mixtral config's experts may be split across devices
(Hugging Face "Mixtral" doc, MixtralConfig: num_local_experts, the experts on each
device). With W ranks and E experts, rank r owns experts [r E/W, (r+1) E/W) and keeps
only their weights; every rank keeps the router and routes its own tokens. One layer:

1. route and permute this rank's tokens (the library's router and permutation): rows
   grouped by expert, each group padded to 128 rows, so the rows bound for rank r are
   one contiguous block;
2. exchange per-expert padded row counts (all_to_all of E/W integers per peer);
3. exchange the rows themselves (all_to_all_single, uneven splits): rank r receives,
   from every source rank in turn, the padded groups of its own experts;
4. regroup the received rows expert-contiguously (the library's row gather), run the
   grouped SwiGLU experts on them, and restore the received order (row gather);
5. send every expert output back to the rank its token came from (all_to_all_single,
   the splits of step 3 reversed), then combine into the residual there.

Every arithmetic step runs in the library's kernels; this module only plans the
exchange on the host (it reads the E+1 group offsets back, one synchronisation) and
calls torch.distributed, whose collectives are NCCL on GPUs. The compute steps are
reached through an ``ops`` object (``CudaOps`` by default), so the same plan can be
exercised with other implementations of the steps.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class CudaOps:
    """The layer's steps on CUDA tensors, through the library's C ABI."""

    def __init__(self):
        from . import moe
        self.moe = moe

    def router_topk(self, x, w_router, k, logit_bias):
        idx, wt = self.moe.router_topk(x, w_router, k, logit_bias)
        return idx, wt

    def permute(self, idx, x, num_experts, intermediate_size):
        shape = self.moe.make_shape(x.shape[0], x.shape[1], intermediate_size, num_experts,
                                    idx.shape[1])
        ws = self.moe.make_workspace(shape, x.device)
        return self.moe.permute(idx, x, num_experts, intermediate_size, ws)

    def gather_rows(self, src, index):
        return self.moe.gather_rows(src, index)

    def grouped_swiglu(self, x_groups, offsets, w1, w3, w2, rows):
        """The experts on `rows` routed rows in expert groups (x_groups holds
        padded_rows(rows, E) rows)."""
        e, i, h = w1.shape
        rows = max(rows, 1)
        shape = self.moe.make_shape(rows, h, i, e, 1)
        ws = self.moe.make_workspace(shape, x_groups.device)
        return self.moe.grouped_swiglu(x_groups, offsets, w1, w3, w2, rows, 1, ws)

    def combine(self, y_perm, row_of, topk_w, residual, num_experts, intermediate_size):
        return self.moe.combine(y_perm, row_of, topk_w, residual, num_experts, intermediate_size)

    def padded_rows(self, rows, num_experts):
        """Rows the grouped GEMM's buffers need for `rows` routed rows in num_experts
        groups (its moe_max_padded_rows)."""
        shape = self.moe.make_shape(max(rows, 1), 128, 128, num_experts, 1)
        return self.moe.max_padded_rows(shape)


def exchange_plan(offsets, world: int, recv_counts):
    """Host-side plan of one exchange.

    offsets: this rank's padded group offsets [E+1] (E = world * E_loc experts);
    recv_counts: [world, E_loc] padded rows this rank receives for each of its experts
    from each source rank.
    Returns (send_rows [world], recv_rows [world], local_offsets [E_loc+1],
    to_local [n_recv], to_recv [n_recv]): rows sent to / received from each rank; the
    expert-contiguous layout of the received rows (expert e's rows from source 0, then
    source 1, ...); and the two row maps, local row -> received row and back.
    """
    offsets = [int(v) for v in offsets]
    e_total = len(offsets) - 1
    e_loc = e_total // world
    send_rows = [offsets[(r + 1) * e_loc] - offsets[r * e_loc] for r in range(world)]
    counts = [[int(c) for c in row] for row in recv_counts]
    recv_rows = [sum(row) for row in counts]
    # start of the (source s, expert e) segment in the received buffer
    seg = [[0] * e_loc for _ in range(world)]
    pos = 0
    for s in range(world):
        for e in range(e_loc):
            seg[s][e] = pos
            pos += counts[s][e]
    n_recv = pos
    local_offsets = [0]
    to_local = []
    for e in range(e_loc):
        for s in range(world):
            to_local.extend(range(seg[s][e], seg[s][e] + counts[s][e]))
        local_offsets.append(len(to_local))
    to_recv = [0] * n_recv
    for dst, src in enumerate(to_local):
        to_recv[src] = dst
    return send_rows, recv_rows, local_offsets, to_local, to_recv


def forward_ep(x, w_router, w1_local, w3_local, w2_local, k: int, num_experts: int,
               group=None, residual=None, logit_bias=None, ops=None):
    """The layer for this rank's tokens x [T, H], its experts' weights w1_local,
    w3_local [E/W, I, H] and w2_local [E/W, H, I] (rank r owns experts r E/W ..), and the
    full router w_router [E, H]. Returns out [T, H] = residual + routed output.

    Every rank of ``group`` must call it (the collectives are collective); T may differ
    between ranks. E must be a multiple of the group size.
    """
    ops = ops or CudaOps()
    world = dist.get_world_size(group)
    if num_experts % world:
        raise ValueError(f"num_experts {num_experts} is not a multiple of the group size {world}")
    e_loc = num_experts // world
    if w1_local.shape[0] != e_loc:
        raise ValueError(f"this rank must hold {e_loc} experts, got {w1_local.shape[0]}")
    inter = w1_local.shape[1]
    dev = x.device

    # 1. route and permute this rank's tokens (a rank without tokens sends nothing but
    #    still takes part in every exchange)
    if x.shape[0] == 0:
        wt = None
        perm = {"offsets": torch.zeros(num_experts + 1, dtype=torch.int64),
                "x_perm": torch.empty((0, x.shape[1]), dtype=x.dtype, device=dev)}
    else:
        idx, wt = ops.router_topk(x, w_router, k, logit_bias)
        perm = ops.permute(idx, x, num_experts, inter)
    offsets = perm["offsets"].to("cpu", torch.int64)
    r_pad = int(offsets[-1])

    # 2. padded rows per expert, E/W to each owner
    padded = (offsets[1:] - offsets[:-1]).to(dev)
    recv_counts = torch.empty(world * e_loc, dtype=torch.int64, device=dev)
    dist.all_to_all_single(recv_counts, padded, group=group)
    recv_counts = recv_counts.view(world, e_loc).cpu()
    send_rows, recv_rows, local_offsets, to_local, to_recv = exchange_plan(offsets, world,
                                                                          recv_counts)

    # 3. the rows
    x_perm = perm["x_perm"][:r_pad].contiguous()
    x_recv = torch.empty((sum(recv_rows), x.shape[1]), dtype=x_perm.dtype, device=dev)
    dist.all_to_all_single(x_recv, x_perm, recv_rows, send_rows, group=group)

    # 4. regroup by local expert (padded to the grouped GEMM's buffer size), the experts,
    #    and back to the received order
    n_local = len(to_local)
    rows_buf = ops.padded_rows(n_local, e_loc)
    index = torch.full((rows_buf,), -1, dtype=torch.int64)
    index[:n_local] = torch.tensor(to_local, dtype=torch.int64)
    x_local = ops.gather_rows(x_recv, index.to(dev))
    loc_off = torch.tensor(local_offsets, dtype=torch.int32, device=dev)
    y_local = ops.grouped_swiglu(x_local, loc_off, w1_local, w3_local, w2_local, n_local)
    y_recv = ops.gather_rows(y_local, torch.tensor(to_recv, dtype=torch.int64, device=dev))

    # 5. outputs back to their tokens' ranks, then the combine
    y_back = torch.empty((max(r_pad, 1), x.shape[1]), dtype=y_recv.dtype, device=dev)
    dist.all_to_all_single(y_back[:r_pad], y_recv, send_rows, recv_rows, group=group)
    if x.shape[0] == 0:
        return torch.empty((0, x.shape[1]), dtype=x.dtype, device=dev)
    return ops.combine(y_back, perm["row_of"], wt, residual, num_experts, inter)


def shard_experts(w1, w3, w2, rank: int, world: int):
    """This rank's slice of the stacked expert weights (contiguous copies)."""
    e = w1.shape[0]
    if e % world:
        raise ValueError(f"{e} experts do not split over {world} ranks")
    lo, hi = rank * e // world, (rank + 1) * e // world
    return w1[lo:hi].contiguous(), w3[lo:hi].contiguous(), w2[lo:hi].contiguous()

