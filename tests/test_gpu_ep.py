"""Expert parallelism on one GPU: the row-gather kernel, and the expert-parallel layer
over a one-rank NCCL group, whose exchanges are then identities, equal to moe_forward
bit for bit (same routing, same groups, same GEMM tiles)."""
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


def test_expert_parallel_one_rank_decode(one_rank_group):
    w = W.WORKLOADS["decode"]
    inp = W.draw(w, "cuda")
    want = M.forward(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, 2, residual=inp.residual)
    got = ep.forward_ep(inp.x, inp.w_router, inp.w1, inp.w3, inp.w2, 2, w.num_experts,
                        residual=inp.residual)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
