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

    def grouped_swiglu(self, x_groups, offsets, w1, w3, w2, rows, y=None):
        """The experts on `rows` routed rows in expert groups (x_groups holds
        padded_rows(rows, E) rows); into `y` when given."""
        e, i, h = w1.shape
        rows = max(rows, 1)
        shape = self.moe.make_shape(rows, h, i, e, 1)
        ws = self._workspace("experts", shape, x_groups.device)
        return self.moe.grouped_swiglu(x_groups, offsets, w1, w3, w2, rows, 1, ws, y=y)

    def grouped_swiglu_quantized(self, x_groups, offsets, experts, rows, y=None):
        """The same with int8 (Int8Experts) or 4-bit (Int4Experts) expert weights."""
        e, i, _ = experts.q1.shape
        h = x_groups.shape[1]
        rows = max(rows, 1)
        shape = self.moe.make_shape(rows, h, i, e, 1)
        ws = self._workspace("experts", shape, x_groups.device)
        fn = (self.moe.grouped_swiglu_w4 if isinstance(experts, self.moe.Int4Experts)
              else self.moe.grouped_swiglu_w8)
        return fn(x_groups, offsets, experts, rows, 1, ws, y=y)

    def scatter_rows_peer(self, src, src_index, dst_rank, dst_row, dst_bases, dst_rows):
        self.moe.scatter_rows_peer(src, src_index, dst_rank, dst_row, dst_bases, dst_rows)

    def combine_peer(self, y_bases, y_rows, slot_rank, slot_row, topk_w, hidden, residual):
        return self.moe.combine_peer(y_bases, y_rows, slot_rank, slot_row, topk_w, hidden,
                                     residual)

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



# ---- the same layer with the exchanges as peer-memory loads and stores ----
#
# Every rank allocates its receive buffers once (PeerBuffers: x_local [rows, H] bf16,
# the expert groups the grouped GEMM reads, and y_local [rows, H] fp32, what it writes)
# and maps every other rank's through CUDA IPC. One layer, after routing and permuting
# as above:
#
# 1. all-gather every rank's routed rows per expert (world x E integers), so each rank
#    knows every owner's group layout;
# 2. store each real routed row straight into its owner's x_local, at its final place:
#    the owner's group for that expert, after the rows of lower source ranks (one
#    kernel of plain stores; it replaces the all-to-all and both regrouping gathers);
# 3. barrier; every owner runs its experts from x_local into y_local;
# 4. barrier; each rank's combine reads its slots' outputs from the owners' y_local
#    (plain loads) and adds them into the residual; barrier, so the buffers are free
#    for the next layer.
#
# The barriers order the ranks between kernels: no kernel waits on another rank.


def peer_plan(offsets, counts_all, rank: int, world: int, device=None):
    """Plan of the peer-memory exchange for rank `rank`, in whole-tensor index
    arithmetic. offsets: this rank's padded group offsets [E+1]; counts_all [world, E]:
    every rank's routed rows per expert (E = world * E_loc). Returns a dict:
      send_index [n_send] int64: this rank's x_perm rows to send (real rows, expert order);
      dst_rank [n_send] int32: the owner of each; dst_row [n_send] int64: its row in the
        owner's x_local (the owner's group for the expert, each group padded to 128 rows
        and holding the source ranks' rows in rank order);
      local_offsets [E_loc+1] (ints): this rank's own groups as an owner;
      n_recv (int): the real rows this rank receives in them; owner_recv [world] (ints):
        the real rows every owner receives (the same list on every rank);
      row_rank [offsets[-1]] int32, row_dst [offsets[-1]] int64: for each x_perm row,
        the owner and row of its expert output (-1 on pad rows).
    The sizes come to the host in one read."""
    i64 = dict(dtype=torch.int64, device=device)
    offsets = torch.as_tensor(offsets, **i64).reshape(-1)
    c = torch.as_tensor(counts_all, **i64).reshape(world, -1)
    e_total = c.shape[1]
    if e_total % world:
        raise ValueError(f"{e_total} experts do not split over {world} ranks")
    e_loc = e_total // world
    padded = _pad(c.sum(0)).reshape(world, e_loc)            # rows of each owner's groups
    group_start = (torch.cumsum(padded, 1) - padded).reshape(-1)
    before = (torch.cumsum(c, 0) - c)[rank]                  # rows of expert e from ranks < rank
    counts = c[rank]
    owners = c.sum(0).reshape(world, e_loc).sum(1)             # real rows each owner receives
    host = torch.cat([offsets[-1:], counts.sum().reshape(1), owners, padded[rank]]).cpu()
    n_rows, n_send = int(host[0]), int(host[1])
    owner_recv = host[2:2 + world].tolist()
    n_recv = owner_recv[rank]
    local_offsets = [0] + torch.cumsum(host[2 + world:], 0).tolist()
    grp, j = _segment_ranks(counts, n_send)
    send_index = offsets[:-1][grp] + j
    dst_rank = (grp // e_loc).to(torch.int32)
    dst_row = group_start[grp] + before[grp] + j
    row_rank = torch.full((n_rows,), -1, dtype=torch.int32, device=device)
    row_rank[send_index] = dst_rank
    row_dst = torch.full((n_rows,), -1, **i64)
    row_dst[send_index] = dst_row
    return {"send_index": send_index, "dst_rank": dst_rank, "dst_row": dst_row,
            "local_offsets": local_offsets, "n_recv": n_recv, "owner_recv": owner_recv,
            "row_rank": row_rank, "row_dst": row_dst}


def peer_rows_needed(max_tokens: int, k: int, world: int, e_loc: int) -> int:
    """Rows an owner's buffers need: every rank's tokens all routed to this owner
    (world * max_tokens * k rows) in E_loc groups, as the grouped GEMM sizes them."""
    r = world * max_tokens * k
    return (r + 127) // 128 * 128 + 128 * e_loc


class PeerBuffers:
    """This rank's receive buffers of the peer-memory layer and every rank's addresses.

    x_local [rows, hidden] bf16 and y_local [rows, hidden] fp32 are allocated by the
    library (moe_ipc_alloc) and zeroed; ``share`` (default: all_gather_object over
    ``group``) gives every rank's IPC handles, and the other ranks' buffers are mapped
    (moe_ipc_open). x_bases / y_bases: int64 device tensors of the world's addresses,
    indexed by rank. ``close()`` unmaps, waits for every rank, and frees."""

    def __init__(self, rows: int, hidden: int, group=None, device=None, share=None):
        from . import moe
        self.moe = moe
        self.rows, self.hidden, self.group = rows, hidden, group
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.rank = dist.get_rank(group)
        world = dist.get_world_size(group)
        self._own, self._mapped = [], []
        try:
            self._setup(moe, rows, hidden, group, world, share)
        except BaseException:
            # nothing half-made stays behind: unmap what was mapped, free what was made
            for p in self._mapped:
                moe.ipc_close(p)
            for p in self._own:
                moe.ipc_free(p)
            self._own, self._mapped = [], []
            raise

    def _setup(self, moe, rows, hidden, group, world, share):
        x_ptr, x_h = moe.ipc_alloc(rows * hidden * 2)
        self._own.append(x_ptr)
        y_ptr, y_h = moe.ipc_alloc(rows * hidden * 4)
        self._own.append(y_ptr)
        self.x_local = moe.tensor_at(x_ptr, (rows, hidden), torch.bfloat16, self.device)
        self.y_local = moe.tensor_at(y_ptr, (rows, hidden), torch.float32, self.device)
        self.x_local.zero_()
        self.y_local.zero_()
        torch.cuda.synchronize(self.device)
        if share is None:
            def share(obj):
                out = [None] * world
                dist.all_gather_object(out, obj, group=group)
                return out
        handles = share((x_h, y_h, rows, hidden))
        # the stores and loads index every rank's buffers with this rank's row count
        if any((rr, hh) != (rows, hidden) for _, _, rr, hh in handles):
            raise ValueError("every rank's PeerBuffers must have the same rows and hidden size: "
                             f"{[(rr, hh) for _, _, rr, hh in handles]}")
        xs, ys = [], []
        for r, (xh, yh, _, _) in enumerate(handles):
            if r == self.rank:
                xs.append(x_ptr)
                ys.append(y_ptr)
            else:
                xs.append(moe.ipc_open(xh))
                self._mapped.append(xs[-1])
                ys.append(moe.ipc_open(yh))
                self._mapped.append(ys[-1])
        self.x_bases = torch.tensor(xs, dtype=torch.int64, device=self.device)
        self.y_bases = torch.tensor(ys, dtype=torch.int64, device=self.device)

    def close(self, barrier=None):
        """Unmap the other ranks' buffers, wait at ``barrier`` (default: a group
        barrier) until every rank has done the same, then free this rank's."""
        for p in self._mapped:
            self.moe.ipc_close(p)
        self._mapped = []
        (barrier or (lambda: dist.barrier(group=self.group)))()
        self.x_local = self.y_local = None
        for p in self._own:
            self.moe.ipc_free(p)
        self._own = []


def _default_barrier(group, device):
    def barrier():
        torch.cuda.current_stream(device).synchronize()
        dist.barrier(group=group)
    return barrier


def _default_gather_counts(group, world):
    def gather(counts):
        parts = [torch.empty_like(counts) for _ in range(world)]
        dist.all_gather(parts, counts, group=group)
        return torch.stack(parts)
    return gather


def forward_ep_peer(x, w_router, w1_local, w3_local, w2_local, k: int, num_experts: int,
                    bufs: PeerBuffers, group=None, residual=None, logit_bias=None, ops=None,
                    gather_counts=None, barrier=None):
    """forward_ep with the exchanges as peer-memory stores and loads (PeerBuffers).
    ``gather_counts(counts [E] int64) -> [world, E]`` (default: all_gather over
    ``group``) and ``barrier()`` (default: wait for this rank's stream, then a group
    barrier) can be replaced, e.g. by host-side collectives in tests."""
    ops = ops or _default_ops()
    return _forward_ep_peer(
        x, w_router, k, num_experts, w1_local.shape[0], w1_local.shape[1],
        lambda xl, off, n, y: ops.grouped_swiglu(xl, off, w1_local, w3_local, w2_local, n, y=y),
        bufs, group, residual, logit_bias, ops, gather_counts, barrier)


def forward_ep_peer_quantized(x, w_router, experts_local, k: int, num_experts: int,
                              bufs: PeerBuffers, group=None, residual=None, logit_bias=None,
                              ops=None, gather_counts=None, barrier=None):
    """forward_ep_peer with this rank's experts as int8 or 4-bit codes."""
    ops = ops or _default_ops()
    e_loc, inter = experts_local.q1.shape[0], experts_local.q1.shape[1]
    return _forward_ep_peer(
        x, w_router, k, num_experts, e_loc, inter,
        lambda xl, off, n, y: ops.grouped_swiglu_quantized(xl, off, experts_local, n, y=y),
        bufs, group, residual, logit_bias, ops, gather_counts, barrier)


def _forward_ep_peer(x, w_router, k, num_experts, held, inter, run_experts, bufs, group,
                     residual, logit_bias, ops, gather_counts, barrier):
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if num_experts % world:
        raise ValueError(f"num_experts {num_experts} is not a multiple of the group size {world}")
    e_loc = num_experts // world
    if held != e_loc:
        raise ValueError(f"this rank must hold {e_loc} experts, got {held}")
    hidden = x.shape[1]
    if hidden != bufs.hidden:
        raise ValueError(f"the buffers hold rows of {bufs.hidden}, x has {hidden}")
    dev = x.device
    gather_counts = gather_counts or _default_gather_counts(group, world)
    barrier = barrier or _default_barrier(group, dev)

    # routing and permutation of this rank's tokens (none: it only takes part)
    if x.shape[0] == 0:
        wt = None
        perm = {"offsets": torch.zeros(num_experts + 1, dtype=torch.int64, device=dev),
                "counts": torch.zeros(num_experts, dtype=torch.int64, device=dev),
                "x_perm": torch.empty((0, hidden), dtype=x.dtype, device=dev)}
    else:
        idx, wt = ops.router_topk(x, w_router, k, logit_bias)
        perm = ops.permute(idx, x, num_experts, inter)
    offsets = perm["offsets"].to(dev, torch.int64)
    counts = perm["counts"].to(dev, torch.int64)

    # 1. every rank's counts; 2. the rows into their owners' groups
    counts_all = gather_counts(counts).to(dev, torch.int64).reshape(world, num_experts)
    plan = peer_plan(offsets, counts_all, rank, world, device=dev)
    n_recv = plan["n_recv"]
    # the grouped GEMM's buffer rows for n_recv rows in E_loc groups (they cover the
    # padded groups: local_offsets[-1] <= n_recv + 127 E_loc). Every rank checks every
    # owner from the same counts, so all ranks raise together and none is left waiting.
    need = max(ops.padded_rows(n, e_loc) for n in plan["owner_recv"])
    if need > bufs.rows:
        raise ValueError(f"an owner receives {max(plan['owner_recv'])} rows; the grouped GEMM "
                         f"needs {need} buffer rows, the buffers hold {bufs.rows}")
    rows_buf = ops.padded_rows(n_recv, e_loc)
    ops.scatter_rows_peer(perm["x_perm"], plan["send_index"], plan["dst_rank"], plan["dst_row"],
                          bufs.x_bases, bufs.rows)
    barrier()
    # 3. this rank's experts on the rows every rank stored here
    loc_off = torch.tensor(plan["local_offsets"], dtype=torch.int32, device=dev)
    run_experts(bufs.x_local[:rows_buf], loc_off, n_recv, bufs.y_local[:rows_buf])
    barrier()
    # 4. the combine reads each slot's output where its owner wrote it
    if x.shape[0] == 0:
        out = torch.empty((0, hidden), dtype=x.dtype, device=dev)
    else:
        row_of = perm["row_of"].to(dev, torch.int64).reshape(-1)
        slot_rank = plan["row_rank"][row_of].contiguous()
        slot_row = plan["row_dst"][row_of].contiguous()
        out = ops.combine_peer(bufs.y_bases, bufs.rows, slot_rank, slot_row, wt, hidden,
                               residual)
    barrier()
    return out
