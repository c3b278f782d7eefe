"""Expert parallelism on CPU with gloo ranks: the exchange plan, and the whole
expert-parallel layer with oracle stand-ins for the compute steps, against the
single-process oracle layer (experts split over 2 and 4 ranks, uneven token counts,
ranks that own no routed rows)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_mixture_experts_09_b200 import ep


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The layer's steps from the fp64 oracle on CPU tensors (test infrastructure)."""

    def __init__(self):
        from oracle import moe_oracle as O
        self.O = O

    def router_topk(self, x, w_router, k, logit_bias):
        O = self.O
        idx, w, _ = O.route_topk(O.router_logits(x, w_router, logit_bias), k)
        return torch.from_numpy(idx), torch.from_numpy(w)

    def permute(self, idx, x, num_experts, intermediate_size):
        O = self.O
        count, offset, row_of, tok = O.stable_permute(idx.numpy(), num_experts)
        # rows keep x's dtype (exact copies), as the library's gather does
        x_perm = torch.zeros((int(offset[-1]), x.shape[1]), dtype=x.dtype)
        real = torch.from_numpy(tok >= 0)
        x_perm[real] = x[torch.from_numpy(tok)[real]]
        return {"counts": torch.from_numpy(count), "offsets": torch.from_numpy(offset),
                "row_of": torch.from_numpy(row_of), "x_perm": x_perm}

    def gather_rows(self, src, index):
        out = torch.zeros((index.numel(), src.shape[1]), dtype=src.dtype)
        ok = (index >= 0) & (index < src.shape[0])
        out[ok] = src[index[ok]]
        return out

    def grouped_swiglu(self, x_groups, offsets, w1, w3, w2, rows, y=None):
        out = torch.zeros((x_groups.shape[0], w2.shape[1]), dtype=torch.float64)
        off = offsets.tolist()
        for e in range(w1.shape[0]):
            a, b = off[e], off[e + 1]
            if b > a:
                rows_e = self.O.to_f64(x_groups[a:b])
                out[a:b] = torch.from_numpy(self.O.swiglu_expert(rows_e, w1[e], w3[e], w2[e]))
        if y is None:
            return out
        y[:out.shape[0]] = out
        return y

    def scatter_rows_peer(self, src, src_index, dst_rank, dst_row, dst_bases, dst_rows):
        """dst_bases: every rank's x_local (CPU tensors in shared memory)."""
        for i, r, d in zip(src_index.tolist(), dst_rank.tolist(), dst_row.tolist()):
            assert 0 <= d < dst_rows
            dst_bases[r][d] = src[i]

    def combine_peer(self, y_bases, y_rows, slot_rank, slot_row, topk_w, hidden, residual):
        t, k = topk_w.shape
        out = torch.zeros((t, hidden), dtype=torch.float64)
        ranks, rows = slot_rank.reshape(t, k), slot_row.reshape(t, k)
        for i in range(t):
            for j in range(k):
                out[i] += topk_w[i, j] * y_bases[int(ranks[i, j])][int(rows[i, j])]
        if residual is not None:
            out += residual.double()
        return out

    def grouped_swiglu_quantized(self, x_groups, offsets, experts, rows, y=None):
        """Half-precision experts on dequantised weights (experts.deq = fp64 w1, w3, w2
        of this rank's experts), as the oracle's f16_experts mode computes them."""
        O = self.O
        d1, d3, d2 = experts.deq
        out = torch.zeros((x_groups.shape[0], d2.shape[1]), dtype=torch.float64)
        off = offsets.tolist()
        for e in range(d1.shape[0]):
            a, b = off[e], off[e + 1]
            if b > a:
                x16 = O.round_f16(O.to_f64(x_groups[a:b]))
                h = O.silu(x16 @ d1[e].T) * (x16 @ d3[e].T)
                out[a:b] = torch.from_numpy(O.round_f16(h) @ d2[e].T)
        if y is None:
            return out
        y[:out.shape[0]] = out
        return y

    def combine(self, y_perm, row_of, topk_w, residual, num_experts, intermediate_size):
        out = torch.zeros((row_of.shape[0], y_perm.shape[1]), dtype=torch.float64)
        for j in range(row_of.shape[1]):
            out += topk_w[:, j:j + 1] * y_perm[row_of[:, j]]
        if residual is not None:
            out += residual.double()
        return out

    def padded_rows(self, rows, num_experts):
        return (max(rows, 1) + 127) // 128 * 128 + 128 * num_experts


def _layer_inputs(t_total, hd, inter, e, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(t_total, hd, generator=g).to(torch.bfloat16)
    wr = (torch.randn(e, hd, generator=g) / hd ** 0.5).to(torch.bfloat16)
    w1 = (torch.randn(e, inter, hd, generator=g) / hd ** 0.5).to(torch.bfloat16)
    w3 = (torch.randn(e, inter, hd, generator=g) / hd ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(e, hd, inter, generator=g) / inter ** 0.5).to(torch.bfloat16)
    res = torch.randn(t_total, hd, generator=g).to(torch.bfloat16)
    return x, wr, w1, w3, w2, res


def _dequantised_4bit(w1, w3, w2):
    from oracle import moe_oracle as O
    return [O.dequantize_int4_groups(*O.quantize_int4_groups(w)) for w in (w1, w3, w2)]


def _rank(rank, world, port, q, tokens, e, k, bias, quant=False):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from sparse_mixture_experts_09_b200 import ep as EP
    from tests.test_ep import OracleOps, _layer_inputs
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    hd, inter = (128, 128) if quant else (32, 48)
    x, wr, w1, w3, w2, res = _layer_inputs(sum(tokens), hd, inter, e, seed=7)
    lo = sum(tokens[:rank])
    mine = slice(lo, lo + tokens[rank])
    b = None if bias is None else torch.tensor(bias, dtype=torch.float64)
    if quant:
        from types import SimpleNamespace
        from tests.test_ep import _dequantised_4bit
        d = _dequantised_4bit(w1, w3, w2)
        el = e // world
        part = [t[rank * el:(rank + 1) * el] for t in d]
        local = SimpleNamespace(q1=torch.from_numpy(part[0]), deq=part)
        out = EP.forward_ep_quantized(x[mine], wr, local, k, e, residual=res[mine], logit_bias=b,
                                      ops=OracleOps())
    else:
        l1, l3, l2 = EP.shard_experts(w1, w3, w2, rank, world)
        out = EP.forward_ep(x[mine], wr, l1, l3, l2, k, e, residual=res[mine], logit_bias=b,
                            ops=OracleOps())
    q.put((rank, out.double().numpy()))
    dist.barrier()
    dist.destroy_process_group()


def _run(world, tokens, e, k, bias=None, quant=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q, tokens, e, k, bias, quant))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    return np.concatenate([got[r] for r in range(world)])


@pytest.mark.parametrize("world,tokens,e,k,bias", [
    (2, [5, 9], 4, 2, None),
    (4, [3, 0, 11, 6], 8, 2, None),
    # all tokens go to experts 0 and 1 (rank 0): the other ranks receive nothing
    (2, [7, 4], 4, 2, [30.0, 30.0, -30.0, -30.0]),
    (2, [6, 6], 2, 1, None),
])
def test_expert_parallel_layer_equals_single_process_layer(world, tokens, e, k, bias):
    from oracle import moe_oracle as O
    got = _run(world, tokens, e, k, bias)
    x, wr, w1, w3, w2, res = _layer_inputs(sum(tokens), 32, 48, e, seed=7)
    b = None if bias is None else np.asarray(bias)
    ref = O.moe_layer(x, wr, w1, w3, w2, k, residual=res, logit_bias=b, mode="exact")
    np.testing.assert_allclose(got, ref["out"], rtol=1e-12, atol=1e-12)


def test_exchange_plan_sends_real_rows_and_pads_per_expert():
    # E = 4 over 2 ranks; this rank routed 3, 130, 0, 5 rows (padded offsets below) and
    # receives, for its experts 0 and 1, 3 and 0 rows from rank 0, 7 and 2 from rank 1
    offsets = [0, 128, 384, 384, 512]
    counts = [3, 130, 0, 5]
    p = _lists(ep.exchange_plan(offsets, counts, 2, [[3, 0], [7, 2]]))
    assert p["send_rows"] == [133, 5] and p["recv_rows"] == [3, 9]
    assert p["send_index"] == [0, 1, 2] + list(range(128, 258)) + [384, 385, 386, 387, 388]
    # every x_perm row maps to its place in the packed rows, pad rows to -1
    back = p["back_index"]
    assert len(back) == 512 and sum(b >= 0 for b in back) == 138
    assert all(p["send_index"][back[r]] == r for r in range(512) if back[r] >= 0)
    # local expert 0: source 0 rows 0..2, source 1 rows 3..9, padded to 128; expert 1:
    # source 1 rows 10..11, padded
    assert p["local_offsets"] == [0, 128, 256]
    tl = p["to_local"]
    assert tl[:10] == list(range(10)) and tl[10:128] == [-1] * 118
    assert tl[128:130] == [10, 11] and tl[130:] == [-1] * 126
    assert all(tl[p["to_recv"][i]] == i for i in range(12))


def _lists(plan):
    """The plan with its index tensors as Python lists."""
    return {k: v.tolist() if torch.is_tensor(v) else v for k, v in plan.items()}


def test_exchange_plan_empty_rank():
    p = _lists(ep.exchange_plan([0, 0, 0, 0, 0], [0, 0, 0, 0], 2, [[0, 0], [4, 0]]))
    assert p["send_rows"] == [0, 0] and p["send_index"] == [] and p["back_index"] == []
    assert p["local_offsets"] == [0, 128, 128] and p["to_recv"] == [0, 1, 2, 3]


def _simulate_world(counts):
    """All ranks' plans of one exchange, run on the host: counts[r][e] rows routed by
    rank r to global expert e. Rows are tagged (rank, expert, j); the all-to-all is
    emulated as concatenation by source rank. Returns what every owner computes on and
    what every source gets back."""
    world, e_total = len(counts), len(counts[0])
    e_loc = e_total // world
    pad = lambda n: (n + 127) // 128 * 128
    x_perm, plans = [], []
    for r in range(world):
        offs = [0]
        rows = []
        for e in range(e_total):
            rows += [(r, e, j) for j in range(counts[r][e])]
            rows += [None] * (pad(counts[r][e]) - counts[r][e])
            offs.append(len(rows))
        x_perm.append(rows)
        recv = [[counts[s][r * e_loc + e] for e in range(e_loc)] for s in range(world)]
        plans.append(_lists(ep.exchange_plan(offs, counts[r], world, recv)))
    sent = []
    for r in range(world):
        rows = [x_perm[r][i] for i in plans[r]["send_index"]]
        pieces, at = [], 0
        for s in range(world):
            pieces.append(rows[at:at + plans[r]["send_rows"][s]])
            at += plans[r]["send_rows"][s]
        sent.append(pieces)
    local, back = [], []
    for s in range(world):
        received = [row for r in range(world) for row in sent[r][s]]
        assert len(received) == sum(plans[s]["recv_rows"])
        local.append([received[i] if i >= 0 else None for i in plans[s]["to_local"]])
        # the experts keep rows in place; the reply goes out in received order
        reply = [local[s][i] for i in plans[s]["to_recv"]]
        back.append(reply)
    returned = []
    for r in range(world):
        rows, at = [], 0
        for s in range(world):
            # rank s replies to r with the segment it received from r, in order
            start = sum(plans[s]["recv_rows"][:r])
            rows += back[s][start:start + plans[s]["recv_rows"][r]]
        returned.append([rows[i] if i >= 0 else None for i in plans[r]["back_index"]])
    return x_perm, plans, local, returned


def test_exchange_plan_random_worlds_round_trip():
    rng = np.random.default_rng(41)
    for trial in range(60):
        world = int(rng.choice([1, 2, 4]))
        e_loc = int(rng.integers(1, 4))
        # mostly small groups, some past one or two 128-row tiles, some empty
        counts = rng.choice([0, 1, 3, 17, 127, 128, 129, 260], size=(world, world * e_loc))
        counts = counts.tolist()
        x_perm, plans, local, returned = _simulate_world(counts)
        for s in range(world):
            lo = plans[s]["local_offsets"]
            assert len(lo) == e_loc + 1 and all(v % 128 == 0 for v in lo)
            for e in range(e_loc):
                group = local[s][lo[e]:lo[e + 1]]
                real = [g for g in group if g is not None]
                # expert group e of owner s: every source's rows for it, by source, then j
                want = [(r, s * e_loc + e, j) for r in range(world)
                        for j in range(counts[r][s * e_loc + e])]
                assert real == want and group[len(real):] == [None] * (len(group) - len(real))
        for r in range(world):
            # every row comes back to its own place; pad rows stay empty
            assert returned[r] == x_perm[r]
            for s in range(world):
                assert plans[r]["send_rows"][s] == plans[s]["recv_rows"][r]


def test_expert_parallel_4bit_layer_equals_single_process_layer():
    # experts as 4-bit codes: each rank computes its experts in half precision on the
    # dequantised weights; the result is the oracle's half-precision layer (before its
    # output rounding) plus the residual
    from oracle import moe_oracle as O
    tokens, e, k = [6, 11], 4, 2
    got = _run(2, tokens, e, k, quant=True)
    x, wr, w1, w3, w2, res = _layer_inputs(sum(tokens), 128, 128, e, seed=7)
    d1, d3, d2 = _dequantised_4bit(w1, w3, w2)
    ref = O.moe_layer(x, wr, d1, d3, d2, k, mode="f16_experts")
    np.testing.assert_allclose(got, O.to_f64(res) + ref["routed"], rtol=1e-12, atol=1e-12)


def test_shard_quantized_slices_are_valid_layouts():
    # 4-bit codes packed by the header's layout statement, sliced per rank, decode to
    # exactly the codes and scales of that rank's experts
    from oracle import moe_oracle as O
    from sparse_mixture_experts_09_b200 import moe as M
    from .test_gpu_w4 import unblock4
    from .test_w4_layout import _pack_from_header, _scales_from_header
    rng = np.random.default_rng(42)
    e, i, h = 4, 256, 128
    mats = {"1": (i, h), "3": (i, h), "2": (h, i)}
    codes, fields = {}, {}
    for name, (r, kk) in mats.items():
        w = O.round_bf16(rng.standard_normal((e * r, kk)) * 0.05)
        q, s16 = O.quantize_int4_groups(w)
        codes[name] = (q, s16)
        fields["q" + name] = torch.from_numpy(_pack_from_header(q, kk).copy()).reshape(e, r, kk // 2)
        fields["s" + name] = torch.from_numpy(_scales_from_header(s16, e * r, kk)).reshape(
            e, r // 128, kk // 64, 128)
    ex = M.Int4Experts(**fields)
    for rank in range(2):
        part = ep.shard_quantized(ex, rank, 2)
        lo, hi = rank * 2, rank * 2 + 2
        for name, (r, kk) in mats.items():
            got_q, got_s = unblock4(getattr(part, "q" + name), getattr(part, "s" + name))
            q, s16 = codes[name]
            assert np.array_equal(got_q.reshape(-1, kk), q[lo * r:hi * r])
            assert np.array_equal(got_s.reshape(-1, kk // 64), s16[lo * r:hi * r])
    with pytest.raises(ValueError):
        ep.shard_quantized(ex, 0, 3)


# ---- the peer-memory exchange (ep.peer_plan, ep.forward_ep_peer) ----

def test_peer_plan_random_worlds_place_rows_as_the_exchange_does():
    # every rank stores its rows straight into the owners' groups; the owners' groups
    # must hold what the all-to-all path regroups there, pad rows untouched, and every
    # x_perm row must know where its output is
    rng = np.random.default_rng(43)
    for trial in range(60):
        world = int(rng.choice([1, 2, 4]))
        e_loc = int(rng.integers(1, 4))
        e_total = world * e_loc
        counts = rng.choice([0, 1, 3, 17, 127, 128, 129, 260], size=(world, e_total)).tolist()
        x_perm, plans, local, _ = _simulate_world(counts)
        offs = [[0] + np.cumsum([(n + 127) // 128 * 128 for n in counts[r]]).tolist()
                for r in range(world)]
        peer = [_lists(ep.peer_plan(offs[r], counts, r, world)) for r in range(world)]
        owners = [[None] * peer[s]["local_offsets"][-1] for s in range(world)]
        for r in range(world):
            p = peer[r]
            assert p["send_index"] == plans[r]["send_index"]
            for i, d, row in zip(p["send_index"], p["dst_rank"], p["dst_row"]):
                assert owners[d][row] is None          # no row is written twice
                owners[d][row] = x_perm[r][i]
            n_rows = len(x_perm[r])
            assert len(p["row_rank"]) == n_rows and len(p["row_dst"]) == n_rows
            for i in range(n_rows):
                if x_perm[r][i] is None:
                    assert p["row_rank"][i] == -1 and p["row_dst"][i] == -1
        for s in range(world):
            assert peer[s]["local_offsets"] == plans[s]["local_offsets"]
            assert peer[s]["n_recv"] == sum(plans[s]["recv_rows"])
            assert peer[s]["owner_recv"] == [sum(plans[o]["recv_rows"]) for o in range(world)]
            assert owners[s] == local[s]
        for r in range(world):
            for i, row in enumerate(x_perm[r]):
                if row is not None:
                    assert owners[peer[r]["row_rank"][i]][peer[r]["row_dst"][i]] == row


def test_peer_rows_needed_covers_every_routing():
    # all of every rank's rows routed to one owner, in E_loc groups
    for world, t, k, e_loc in ((1, 5, 2, 4), (2, 300, 2, 4), (4, 129, 8, 2)):
        worst = world * t * k
        groups = [(worst + 127) // 128 * 128] + [0] * (e_loc - 1)
        assert sum(groups) <= ep.peer_rows_needed(t, k, world, e_loc)


def _rank_peer(rank, world, port, q, tokens, e, k, bias, shared, quant=False):
    import datetime
    import sys
    from types import SimpleNamespace
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from sparse_mixture_experts_09_b200 import ep as EP
    from tests.test_ep import OracleOps, _layer_inputs
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    hd, inter = (128, 128) if quant else (32, 48)
    x, wr, w1, w3, w2, res = _layer_inputs(sum(tokens), hd, inter, e, seed=7)
    lo = sum(tokens[:rank])
    mine = slice(lo, lo + tokens[rank])
    b = None if bias is None else torch.tensor(bias, dtype=torch.float64)
    # the world's receive buffers: CPU tensors in shared memory, indexed by rank
    bufs = SimpleNamespace(rows=shared[0][0].shape[0], hidden=hd, x_local=shared[rank][0],
                           y_local=shared[rank][1], x_bases=[t[0] for t in shared],
                           y_bases=[t[1] for t in shared])
    try:
        if quant:
            from tests.test_ep import _dequantised_4bit
            d = _dequantised_4bit(w1, w3, w2)
            el = e // world
            part = [t[rank * el:(rank + 1) * el] for t in d]
            local = SimpleNamespace(q1=torch.from_numpy(part[0]), deq=part)
            out = EP.forward_ep_peer_quantized(x[mine], wr, local, k, e, bufs,
                                               residual=res[mine], logit_bias=b,
                                               ops=OracleOps(), barrier=dist.barrier)
        else:
            l1, l3, l2 = EP.shard_experts(w1, w3, w2, rank, world)
            out = EP.forward_ep_peer(x[mine], wr, l1, l3, l2, k, e, bufs, residual=res[mine],
                                     logit_bias=b, ops=OracleOps(), barrier=dist.barrier)
        q.put((rank, out.double().numpy()))
    except ValueError as err:
        q.put((rank, f"raised: {err}"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,tokens,e,k,bias", [
    (2, [5, 9], 4, 2, None),
    (4, [3, 0, 11, 6], 8, 2, None),
    (2, [7, 4], 4, 2, [30.0, 30.0, -30.0, -30.0]),
])
def test_peer_layer_equals_single_process_layer(world, tokens, e, k, bias):
    from oracle import moe_oracle as O
    rows = ep.peer_rows_needed(max(tokens), k, world, e // world)
    got = _run_peer(world, tokens, e, k, bias, rows)
    got = np.concatenate([got[r] for r in range(world)])
    x, wr, w1, w3, w2, res = _layer_inputs(sum(tokens), 32, 48, e, seed=7)
    b = None if bias is None else np.asarray(bias)
    ref = O.moe_layer(x, wr, w1, w3, w2, k, residual=res, logit_bias=b, mode="exact")
    np.testing.assert_allclose(got, ref["out"], rtol=1e-12, atol=1e-12)


def test_peer_layer_too_small_buffers_raise_on_every_rank():
    # all tokens routed to rank 0's experts: rank 0 would need more rows than the
    # buffers hold; every rank sees it from the gathered counts and raises (none waits)
    got = _run_peer(2, [7, 4], 4, 2, [30.0, 30.0, -30.0, -30.0], rows=256)
    assert all(isinstance(v, str) and v.startswith("raised") for v in got.values()), got


def _run_peer(world, tokens, e, k, bias, rows, quant=False):
    hd = 128 if quant else 32
    shared = [(torch.zeros((rows, hd), dtype=torch.bfloat16).share_memory_(),
               torch.zeros((rows, hd), dtype=torch.float64).share_memory_()) for _ in range(world)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_peer, args=(r, world, port, q, tokens, e, k, bias, shared,
                                                  quant))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    return got


def test_peer_layer_4bit_equals_single_process_layer():
    # forward_ep_peer_quantized: each owner computes its experts in half precision on
    # the dequantised weights, from the rows the ranks stored into its buffer
    from oracle import moe_oracle as O
    tokens, e, k = [6, 11], 4, 2
    rows = ep.peer_rows_needed(max(tokens), k, 2, e // 2)
    got = _run_peer(2, tokens, e, k, None, rows, quant=True)
    got = np.concatenate([got[r] for r in range(2)])
    x, wr, w1, w3, w2, res = _layer_inputs(sum(tokens), 128, 128, e, seed=7)
    d1, d3, d2 = _dequantised_4bit(w1, w3, w2)
    ref = O.moe_layer(x, wr, d1, d3, d2, k, mode="f16_experts")
    np.testing.assert_allclose(got, O.to_f64(res) + ref["routed"], rtol=1e-12, atol=1e-12)

