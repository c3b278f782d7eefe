"""The C-ABI library: it builds, loads, exports every declared symbol, and rejects bad
arguments on the host before any CUDA call (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

from sparse_mixture_experts_09_b200 import build_lib
from sparse_mixture_experts_09_b200 import moe as M

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    build_lib.build()
    return M.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_router_topk", "moe_permute", "moe_grouped_swiglu", "moe_combine",
                     "moe_forward", "moe_workspace_size", "moe_last_error"):
        assert required in names
    assert set(names) == set(M.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def shape(t=64, h=128, i=256, e=8, k=2, layout=0):
    return M.make_shape(t, h, i, e, k, layout)


def test_workspace_and_padded_rows(L):
    s = shape()
    assert M.max_padded_rows(s) == 128 + 128 * 8
    assert M.workspace_size(s) > 0
    assert M.workspace_size_host(s) > M.workspace_size(s)
    big = shape(t=4096, h=4096, i=14336)
    rmax = M.max_padded_rows(big)
    # x_perm + h + y dominate
    assert M.workspace_size(big) >= rmax * (4096 * 2 + 14336 * 2 + 4096 * 4)


@pytest.mark.parametrize("bad", [dict(t=0), dict(h=100), dict(i=200), dict(e=0), dict(e=65),
                                 dict(k=0), dict(k=9, e=16), dict(k=3, e=2), dict(layout=2),
                                 dict(layout=-1)])
def test_invalid_shapes_are_rejected(L, bad):
    s = shape(**bad)
    assert M.workspace_size(s) == 0
    assert M.max_padded_rows(s) == -1
    st = L.moe_forward(ctypes.byref(s), 16, 16, None, 16, 16, 16, None, 16, 256, 1 << 30, None)
    assert st in (1, 2)
    assert L.moe_last_error()


def test_null_and_misaligned_pointers_are_rejected(L):
    s = shape()
    st = L.moe_forward(ctypes.byref(s), None, 16, None, 16, 16, 16, None, 16, 256, 1 << 30, None)
    assert st == 1 and b"x is NULL" in L.moe_last_error()
    st = L.moe_forward(ctypes.byref(s), 24, 16, None, 16, 16, 16, None, 16, 256, 1 << 30, None)
    assert st == 1 and b"aligned" in L.moe_last_error()
    st = L.moe_router_topk(ctypes.byref(s), 16, 16, None, 16, None, None, None)
    assert st == 1 and b"topk_w" in L.moe_last_error()


def test_small_workspace_is_rejected(L):
    s = shape()
    need = M.workspace_size(s)
    st = L.moe_forward(ctypes.byref(s), 16, 16, None, 16, 16, 16, None, 16, 256, need - 1, None)
    assert st == 3 and b"workspace too small" in L.moe_last_error()
    st = L.moe_forward(ctypes.byref(s), 16, 16, None, 16, 16, 16, None, 16, 128, need, None)
    assert st == 3
    st = L.moe_grouped_swiglu(ctypes.byref(s), 16, 16, 16, 16, 16, 16, 256, 10, None)
    assert st == 3


def test_binding_refuses_cpu_tensors(L):
    import torch
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        M.router_topk(x, torch.zeros(8, 128, dtype=torch.bfloat16), 2)


@pytest.mark.parametrize("t,h,i,e,k", [(1, 128, 128, 1, 1), (16, 4096, 14336, 8, 2),
                                       (777, 256, 256, 5, 3), (4096, 640, 512, 64, 8),
                                       (100000, 4096, 14336, 8, 2)])
def test_workspace_holds_every_region(L, t, h, i, e, k):
    s = M.make_shape(t, h, i, e, k)
    rmax = M.max_padded_rows(s)
    assert rmax == (t * k + 127) // 128 * 128 + 128 * e
    ws = M.workspace_size(s)
    # routed-row buffers (x_perm and h as 2-byte values, y fp32) and the per-slot tables
    assert ws >= rmax * (h * 2 + i * 2 + h * 4) + rmax * 4 + 3 * t * k * 4 + 256
    # host entry points: two staging slots for x and the residual, one for the output
    assert M.workspace_size_host(s) - ws >= 5 * t * h * 2
    assert ws % 256 == 0 and M.workspace_size_host(s) % 256 == 0


def test_peer_memory_entry_points_validate_on_the_host(L):
    # every rejection below happens before any CUDA call
    ok, invalid, unsupported = 0, 1, 2
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: each call fails validation first
    ptr = ctypes.c_void_p()
    handle = ctypes.create_string_buffer(64)
    assert L.moe_ipc_alloc(0, ctypes.byref(ptr), ctypes.cast(handle, ctypes.c_void_p)) == invalid
    assert L.moe_ipc_alloc(16, None, ctypes.cast(handle, ctypes.c_void_p)) == invalid
    assert L.moe_ipc_open(None, ctypes.byref(ptr)) == invalid
    assert L.moe_ipc_close(None) == ok and L.moe_ipc_free(None) == ok
    # scatter: bad row size, bad world, negative counts; zero rows is a no-op
    assert L.moe_scatter_rows_peer(fake, 4, fake, fake, fake, 2, fake, 2, 4, 10, None, None) == invalid
    assert L.moe_scatter_rows_peer(fake, 4, fake, fake, fake, 2, fake, 0, 4, 16, None, None) == invalid
    assert L.moe_scatter_rows_peer(fake, 4, fake, fake, fake, -1, fake, 2, 4, 16, None, None) == invalid
    assert L.moe_scatter_rows_peer(None, 0, None, None, None, 0, None, 2, 4, 16, None, None) == ok
    assert L.moe_scatter_rows_peer(fake, 4, None, fake, fake, 2, fake, 2, 4, 16, None, None) == invalid
    # combine: k outside [1, 8], hidden not a multiple of 8, bad world; no tokens is a no-op
    args = lambda k, h, world, t=3: (fake, world, 4, fake, fake, fake, None, fake, t, k, h, None, None)
    assert L.moe_combine_peer(*args(9, 64, 2)) == unsupported
    assert b"k must be in [1, 8]" in L.moe_last_error()
    assert L.moe_combine_peer(*args(2, 60, 2)) == unsupported
    assert b"hidden" in L.moe_last_error()
    assert L.moe_combine_peer(*args(2, 64, 0)) == invalid
    assert L.moe_combine_peer(*args(2, 64, 2, t=0)) == ok
