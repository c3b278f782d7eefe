"""moe_permute_static, the allocation-free permutation, checked against moe_permute.

moe_permute_static serves callers that cannot call cudaMalloc (so cannot hand the
library a workspace): its scratch table is a static device array inside libmoe.so.
The GPU test calls it three times in a row, on different shapes that all need the
table (more than 1024 tokens), the last one filling it exactly, and compares every
output with moe_permute's and, for two of the shapes, with the oracle's. It
sits in a file of its own, collected last, and needs nothing from other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

from sparse_mixture_experts_09_b200 import build_lib
from sparse_mixture_experts_09_b200 import moe as M


def _routing(t, h, e, k, seed):
    g = torch.Generator().manual_seed(seed)
    # k distinct experts per token
    idx = torch.rand(t, e, generator=g).topk(k, dim=1).indices.to(torch.int32)
    x = torch.randn(t, h, generator=g).to(torch.bfloat16)
    return idx.cuda(), x.cuda()


@pytest.mark.gpu
def test_static_permute_matches_workspace_permute_on_two_calls():
    # the last shape fills the static table exactly: ceil(262144 / 32) * 8 = 65536 entries
    build_lib.build()
    for t, h, e, k, seed in ((3000, 256, 8, 2, 1), (2500, 384, 5, 3, 2), (262144, 128, 8, 2, 3)):
        idx, x = _routing(t, h, e, k, seed)
        ws = M.make_workspace(M.make_shape(t, h, 128, e, k))
        want = M.permute(idx, x, e, 128, ws)
        got = M.permute_static(idx, x, e, 128)
        torch.cuda.synchronize()
        for key in ("counts", "offsets", "row_of", "token_of_row", "x_perm"):
            assert torch.equal(got[key], want[key]), (t, key)
        if seed != 2:
            # both share their kernels, so also against the oracle's counting sort
            count, offset, row_of, tok = O.stable_permute(idx.cpu().numpy(), e)
            assert np.array_equal(got["counts"].cpu().numpy(), count), t
            assert np.array_equal(got["offsets"].cpu().numpy(), offset), t
            assert np.array_equal(got["row_of"].cpu().numpy(), row_of), t
            assert np.array_equal(got["token_of_row"][:int(offset[-1])].cpu().numpy(), tok), t


def test_static_permute_rejects_oversized_shapes():
    # 262176 tokens x 8 experts needs 65544 table entries, more than the 65536 it holds;
    # the check runs on the host before any CUDA call
    build_lib.build()
    L = M.lib()
    shape = M.make_shape(262176, 128, 128, 8, 2)
    st = L.moe_permute_static(ctypes.byref(shape), 16, 16, 16, 16, 16, 16, 16, None)
    assert st == 2
    assert b"static table" in L.moe_last_error()
