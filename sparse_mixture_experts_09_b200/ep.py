"""Expert parallelism: the layer with its experts spread over the ranks of a process
group, one process per GPU.

The pages note that a Mixtral config's experts may be split across devices
(Hugging Face "Mixtral" doc, MixtralConfig: num_local_experts, the experts on each
device). With W ranks and E experts, rank r owns experts [r E/W, (r+1) E/W) and keeps
only their weights; every rank keeps the router and routes its own tokens. One layer:

1. route and permute this rank's tokens (the library's router and permutation): rows
   grouped by expert, each group padded to 128 rows, so the rows bound for rank r are
   one contiguous block;
2. exchange per-expert routed row counts (all_to_all of E/W integers per peer);
3. exchange the rows themselves, without pad rows (a row gather packs them;
   all_to_all_single, uneven splits): rank r receives, from every source rank in turn,
   the rows of its own experts;
4. regroup the received rows into expert groups padded to 128 rows (row gather), run
   the grouped SwiGLU experts on them, and restore the received order (row gather);
5. send every expert output back to the rank its token came from (all_to_all_single,
   the splits of step 3 reversed), put it back in the permuted order (row gather) and
   combine into the residual there.

Every arithmetic step of the layer runs in the library's kernels; this module plans
the exchange with whole-tensor index operations on the rows' device (the host reads
only the sizes, once per layer, because the collectives need host-side split sizes)
and calls torch.distributed, whose collectives are NCCL on GPUs. The compute steps are
reached through an ``ops`` object (``CudaOps`` by default), so the same plan can be
exercised with other implementations of the steps.
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist


class CudaOps:
    """The layer's steps on CUDA tensors, through the library's C ABI. Workspaces are
    kept between calls, one per purpose and device, and grow to the largest shape seen."""

    def __init__(self):
        from . import moe
        self.moe = moe
        self._ws = {}

    def _workspace(self, purpose, shape, device):
        need = self.moe.workspace_size(shape)
        key = (purpose, str(device))
        ws = self._ws.get(key)
        if ws is None or ws.numel() < need:
            ws = self.moe.make_workspace(shape, device)
            self._ws[key] = ws
        return ws

    def router_topk(self, x, w_router, k, logit_bias):
        idx, wt = self.moe.router_topk(x, w_router, k, logit_bias)
        return idx, wt

    def permute(self, idx, x, num_experts, intermediate_size):
        shape = self.moe.make_shape(x.shape[0], x.shape[1], intermediate_size, num_experts,
                                    idx.shape[1])
        ws = self._workspace("permute", shape, x.device)
        return self.moe.permute(idx, x, num_experts, intermediate_size, ws)

    def gather_rows(self, src, index):
        return self.moe.gather_rows(src, index)

    def grouped_swiglu(self, x_groups, offsets, w1, w3, w2, rows):
        """The experts on `rows` routed rows in expert groups (x_groups holds
        padded_rows(rows, E) rows)."""
        e, i, h = w1.shape
        rows = max(rows, 1)
        shape = self.moe.make_shape(rows, h, i, e, 1)
        ws = self._workspace("experts", shape, x_groups.device)
        return self.moe.grouped_swiglu(x_groups, offsets, w1, w3, w2, rows, 1, ws)

    def grouped_swiglu_quantized(self, x_groups, offsets, experts, rows):
        """The same with int8 (Int8Experts) or 4-bit (Int4Experts) expert weights."""
        e, i, _ = experts.q1.shape
        h = x_groups.shape[1]
        rows = max(rows, 1)
        shape = self.moe.make_shape(rows, h, i, e, 1)
        ws = self._workspace("experts", shape, x_groups.device)
        fn = (self.moe.grouped_swiglu_w4 if isinstance(experts, self.moe.Int4Experts)
              else self.moe.grouped_swiglu_w8)
        return fn(x_groups, offsets, experts, rows, 1, ws)

    def combine(self, y_perm, row_of, topk_w, residual, num_experts, intermediate_size):
        return self.moe.combine(y_perm, row_of, topk_w, residual, num_experts, intermediate_size)

    def padded_rows(self, rows, num_experts):
        """Rows the grouped GEMM's buffers need for `rows` routed rows in num_experts
        groups (its moe_max_padded_rows)."""
        shape = self.moe.make_shape(max(rows, 1), 128, 128, num_experts, 1)
        return self.moe.max_padded_rows(shape)


def _pad(n):
    return (n + 127) // 128 * 128


def _starts(sizes):
    """Exclusive prefix sums: where each of consecutive segments of these sizes starts."""
    return torch.cumsum(sizes, 0) - sizes


def _segment_ranks(sizes, total: int):
    """For segments of the given sizes laid end to end (``total`` elements in all):
    (segment of each element, position of each element inside its segment)."""
    seg = torch.repeat_interleave(torch.arange(sizes.numel(), device=sizes.device), sizes,
                                  output_size=total)
    pos = torch.arange(total, device=sizes.device) - _starts(sizes)[seg]
    return seg, pos


def exchange_plan(offsets, counts, world: int, recv_counts, device=None):
    """Plan of one exchange, in whole-tensor index arithmetic (no loop over rows). Only
    real rows cross between ranks; groups are padded to 128 rows where they are
    computed.

    offsets: this rank's padded group offsets [E+1]; counts: its routed rows per expert
    [E] (E = world * E_loc); recv_counts: [world, E_loc] rows this rank receives for each
    of its experts from each source rank. The index tensors are built on ``device``
    (default the CPU); the sizes come to the host in one read. Split sizes and offsets
    are Python ints. Returns a dict:
      send_index [n_send]: rows of this rank's x_perm to send, grouped by owner rank
        (expert order), without pad rows;
      send_rows [world], recv_rows [world]: rows sent to / received from each rank;
      local_offsets [E_loc+1]: expert groups of the received rows, each padded to 128;
      to_local [local_offsets[-1]]: received row of each local row (-1 on pad rows);
      to_recv [n_recv]: local row of each received row;
      back_index [offsets[-1]]: position in the returned rows of each x_perm row (-1 on
        pad rows).
    """
    i64 = dict(dtype=torch.int64, device=device)
    offsets = torch.as_tensor(offsets, **i64).reshape(-1)
    counts = torch.as_tensor(counts, **i64).reshape(-1)
    e_total = counts.numel()
    e_loc = e_total // world
    rc = torch.as_tensor(recv_counts, **i64).reshape(world, e_loc)
    # the sizes, read once: padded rows of this rank, its counts, the received counts
    host = torch.cat([offsets[-1:], counts, rc.reshape(-1)]).cpu()
    n_rows = int(host[0])
    counts_h = host[1:1 + e_total]
    rc_h = host[1 + e_total:].reshape(world, e_loc)
    n_send, n_recv = int(counts_h.sum()), int(rc_h.sum())
    send_rows = counts_h.reshape(world, e_loc).sum(1).tolist()
    recv_rows = rc_h.sum(1).tolist()
    local_offsets = [0] + torch.cumsum(_pad(rc_h.sum(0)), 0).tolist()

    # the real rows of each group, in expert order; group e's sit at offsets[e] + j
    grp, j = _segment_ranks(counts, n_send)
    send_index = offsets[:-1][grp] + j
    back_index = torch.full((n_rows,), -1, **i64)
    back_index[send_index] = torch.arange(n_send, **i64)
    # the received buffer holds segments (source s, expert e), source-major; local expert
    # e gathers its segments from every source in turn, padded to 128 rows
    seg_start = _starts(rc.reshape(-1)).reshape(world, e_loc)
    before = (torch.cumsum(rc, 0) - rc).t()        # [e_loc, world]: rows of e from sources < s
    dst_start = torch.as_tensor(local_offsets[:-1], **i64)[:, None] + before
    seg, pos = _segment_ranks(rc.t().reshape(-1), n_recv)   # segments in (expert, source) order
    src = seg_start.t().reshape(-1)[seg] + pos
    dst = dst_start.reshape(-1)[seg] + pos
    to_local = torch.full((local_offsets[-1],), -1, **i64)
    to_local[dst] = src
    to_recv = torch.empty(n_recv, **i64)
    to_recv[src] = dst
    return {"send_index": send_index, "send_rows": send_rows, "recv_rows": recv_rows,
            "local_offsets": local_offsets, "to_local": to_local, "to_recv": to_recv,
            "back_index": back_index}


def _all_to_all(out, inp, out_splits=None, in_splits=None, group=None):
    dist.all_to_all_single(out, inp, out_splits, in_splits, group=group)


def forward_ep(x, w_router, w1_local, w3_local, w2_local, k: int, num_experts: int,
               group=None, residual=None, logit_bias=None, ops=None, exchange=None):
    """The layer for this rank's tokens x [T, H], its experts' weights w1_local,
    w3_local [E/W, I, H] and w2_local [E/W, H, I] (rank r owns experts r E/W ..), and the
    full router w_router [E, H]. Returns out [T, H] = residual + routed output.

    Every rank of ``group`` must call it (the collectives are collective); T may differ
    between ranks, and may be 0. E must be a multiple of the group size. ``exchange``
    (default: torch.distributed's all_to_all_single) moves the rows: it is called as
    exchange(out, inp, out_splits, in_splits, group=group).
    """
    ops = ops or _default_ops()
    return _forward_ep(
        x, w_router, k, num_experts, w1_local.shape[0], w1_local.shape[1],
        lambda xl, off, n: ops.grouped_swiglu(xl, off, w1_local, w3_local, w2_local, n),
        group, residual, logit_bias, ops, exchange or _all_to_all)


def forward_ep_quantized(x, w_router, experts_local, k: int, num_experts: int, group=None,
                         residual=None, logit_bias=None, ops=None, exchange=None):
    """forward_ep with this rank's experts as weight-only int8 or 4-bit codes
    (moe.Int8Experts / moe.Int4Experts holding E/W experts, e.g. from shard_quantized).
    Routing and the exchanges are the bf16 layer's; the experts compute as the
    library's quantised grouped entry points do (half precision)."""
    ops = ops or _default_ops()
    e_loc, inter = experts_local.q1.shape[0], experts_local.q1.shape[1]
    return _forward_ep(
        x, w_router, k, num_experts, e_loc, inter,
        lambda xl, off, n: ops.grouped_swiglu_quantized(xl, off, experts_local, n),
        group, residual, logit_bias, ops, exchange or _all_to_all)


_ops = None


def _default_ops():
    """One CudaOps per process, so its workspaces serve every layer call."""
    global _ops
    if _ops is None:
        _ops = CudaOps()
    return _ops


def _forward_ep(x, w_router, k, num_experts, held, inter, run_experts, group, residual,
                logit_bias, ops, exchange):
    world = dist.get_world_size(group)
    if num_experts % world:
        raise ValueError(f"num_experts {num_experts} is not a multiple of the group size {world}")
    e_loc = num_experts // world
    if held != e_loc:
        raise ValueError(f"this rank must hold {e_loc} experts, got {held}")
    hidden = x.shape[1]
    dev = x.device

    # 1. route and permute this rank's tokens (a rank without tokens sends nothing but
    #    still takes part in every exchange)
    if x.shape[0] == 0:
        wt = None
        perm = {"offsets": torch.zeros(num_experts + 1, dtype=torch.int64),
                "counts": torch.zeros(num_experts, dtype=torch.int64),
                "x_perm": torch.empty((0, hidden), dtype=x.dtype, device=dev)}
    else:
        idx, wt = ops.router_topk(x, w_router, k, logit_bias)
        perm = ops.permute(idx, x, num_experts, inter)
    offsets = perm["offsets"].to(dev, torch.int64)
    counts = perm["counts"].to(dev, torch.int64)

    # 2. routed rows per expert, E/W to each owner
    recv_counts = torch.empty(world * e_loc, dtype=torch.int64, device=dev)
    exchange(recv_counts, counts, group=group)
    # the index arithmetic runs where the rows are; only the split sizes come to the host
    plan = exchange_plan(offsets, counts, world, recv_counts.view(world, e_loc), device=dev)

    # 3. the rows, without padding
    x_send = ops.gather_rows(perm["x_perm"], plan["send_index"])
    x_recv = torch.empty((sum(plan["recv_rows"]), hidden), dtype=x_send.dtype, device=dev)
    exchange(x_recv, x_send, plan["recv_rows"], plan["send_rows"], group=group)

    # 4. expert groups padded to 128 rows (to the grouped GEMM's buffer size), the
    #    experts, and back to the received order
    n_local = plan["local_offsets"][-1]
    rows_buf = ops.padded_rows(n_local, e_loc)
    to_local = torch.cat([plan["to_local"],
                          torch.full((rows_buf - n_local,), -1, dtype=torch.int64, device=dev)])
    x_local = ops.gather_rows(x_recv, to_local)
    loc_off = torch.tensor(plan["local_offsets"], dtype=torch.int32, device=dev)
    y_local = run_experts(x_local, loc_off, n_local)
    y_recv = ops.gather_rows(y_local, plan["to_recv"])

    # 5. outputs back to their tokens' ranks, into the permuted order, then the combine
    y_back = torch.empty((sum(plan["send_rows"]), hidden), dtype=y_recv.dtype, device=dev)
    exchange(y_back, y_recv, plan["send_rows"], plan["recv_rows"], group=group)
    if x.shape[0] == 0:
        return torch.empty((0, hidden), dtype=x.dtype, device=dev)
    y_perm = ops.gather_rows(y_back, plan["back_index"])
    return ops.combine(y_perm, perm["row_of"], wt, residual, num_experts, inter)


def shard_quantized(experts, rank: int, world: int):
    """This rank's slice of quantised experts (Int8Experts or Int4Experts). Codes and
    scales are stored expert after expert (an expert's rows fill whole 128-row tiles),
    so a slice along the expert axis is itself a valid layout for E/W experts."""
    e = experts.q1.shape[0]
    if e % world:
        raise ValueError(f"{e} experts do not split over {world} ranks")
    lo, hi = rank * e // world, (rank + 1) * e // world
    return dataclasses.replace(experts, **{f.name: getattr(experts, f.name)[lo:hi].contiguous()
                                           for f in dataclasses.fields(experts)})


def shard_experts(w1, w3, w2, rank: int, world: int):
    """This rank's slice of the stacked expert weights (contiguous copies)."""
    e = w1.shape[0]
    if e % world:
        raise ValueError(f"{e} experts do not split over {world} ranks")
    lo, hi = rank * e // world, (rank + 1) * e // world
    return w1[lo:hi].contiguous(), w3[lo:hi].contiguous(), w2[lo:hi].contiguous()

