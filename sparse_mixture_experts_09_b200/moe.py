"""ctypes binding of libmoe.so (include/moe.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels. PyTorch supplies device
memory and the current stream; nothing here computes any part of the layer, and
there is no fallback: if the library is missing or a tensor is not on a CUDA device,
the call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# MOE_LIB_PATH selects another build of the same library (it must exist)
LIB_PATH = os.environ.get("MOE_LIB_PATH") or os.path.join(_HERE, "libmoe.so")
ROW_PAD = 128

STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT"}

EXPORTS = ("moe_workspace_size", "moe_workspace_size_host", "moe_max_padded_rows",
           "moe_router_topk", "moe_permute", "moe_grouped_swiglu", "moe_expert_gate_up",
           "moe_expert_down", "moe_combine", "moe_forward",
           "moe_forward_host", "moe_device_status", "moe_last_error", "moe_permute_static",
           "moe_selftest_wait_timeout", "moe_forward_rmsnorm", "moe_pack_weights",
           "moe_quantize_int8", "moe_grouped_swiglu_w8", "moe_forward_w8", "moe_gather_rows",
           "moe_forward_host_async", "moe_quantize_int4", "moe_grouped_swiglu_w4", "moe_forward_w4",
           "moe_ipc_alloc", "moe_ipc_open", "moe_ipc_close", "moe_ipc_free",
           "moe_scatter_rows_peer", "moe_combine_peer")


@dataclass
class Int8Experts:
    """Weight-only int8 experts as written by quantize_int8: codes q1, q3 [E, I, H] and
    q2 [E, H, I] (uint8, offset-binary q + 128, in the library's tiled code layout of
    include/moe.h; same number of elements), per-row scales s1, s3 [E, I] and s2 [E, H]
    fp32."""
    q1: torch.Tensor
    q3: torch.Tensor
    q2: torch.Tensor
    s1: torch.Tensor
    s3: torch.Tensor
    s2: torch.Tensor

    def pointers(self):
        return [_dev(self.q1, "q1", torch.uint8), _dev(self.q3, "q3", torch.uint8),
                _dev(self.q2, "q2", torch.uint8), _dev(self.s1, "s1", torch.float32),
                _dev(self.s3, "s3", torch.float32), _dev(self.s2, "s2", torch.float32)]


@dataclass
class Int4Experts:
    """Weight-only 4-bit experts as written by quantize_int4: codes q1, q3 [E, I, H/2] and
    q2 [E, H, I/2] (uint8, two offset-binary codes q + 8 to a byte, in the library's
    tiled 4-bit layout of include/moe.h) and float16 scales, one per row and 64-column
    group in tile order: s1, s3 [E, I/128, H/64, 128] and s2 [E, H/128, I/64, 128]."""
    q1: torch.Tensor
    q3: torch.Tensor
    q2: torch.Tensor
    s1: torch.Tensor
    s3: torch.Tensor
    s2: torch.Tensor

    def pointers(self):
        return [_dev(self.q1, "q1", torch.uint8), _dev(self.q3, "q3", torch.uint8),
                _dev(self.q2, "q2", torch.uint8), _dev(self.s1, "s1", torch.float16),
                _dev(self.s3, "s3", torch.float16), _dev(self.s2, "s2", torch.float16)]


class MoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


ROW_MAJOR, BLOCKED = 0, 1  # MOE_WEIGHTS_* layouts of the expert weights


class Shape(ctypes.Structure):
    _fields_ = [("num_tokens", ctypes.c_int64), ("hidden_size", ctypes.c_int32),
                ("intermediate_size", ctypes.c_int32), ("num_experts", ctypes.c_int32),
                ("num_experts_per_tok", ctypes.c_int32), ("weight_layout", ctypes.c_int32),
                ("router_bf16_logits", ctypes.c_int32)]


_lib = None
_P = ctypes.c_void_p
_SZ = ctypes.c_size_t


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_mixture_experts_09_b200.build_lib`")
        L = ctypes.CDLL(LIB_PATH)
        sp = ctypes.POINTER(Shape)
        st = ctypes.c_int
        L.moe_workspace_size.argtypes = [sp]
        L.moe_workspace_size.restype = _SZ
        L.moe_workspace_size_host.argtypes = [sp]
        L.moe_workspace_size_host.restype = _SZ
        L.moe_max_padded_rows.argtypes = [sp]
        L.moe_max_padded_rows.restype = ctypes.c_int64
        L.moe_router_topk.argtypes = [sp, _P, _P, _P, _P, _P, _P, _P]
        L.moe_router_topk.restype = st
        L.moe_permute.argtypes = [sp, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.moe_permute.restype = st
        L.moe_grouped_swiglu.argtypes = [sp, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.moe_grouped_swiglu.restype = st
        L.moe_expert_gate_up.argtypes = [sp, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.moe_expert_gate_up.restype = st
        L.moe_expert_down.argtypes = [sp, _P, _P, _P, _P, _P, _SZ, _P]
        L.moe_expert_down.restype = st
        L.moe_combine.argtypes = [sp, _P, _P, _P, _P, _P, _P]
        L.moe_combine.restype = st
        L.moe_forward.argtypes = [sp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.moe_forward.restype = st
        L.moe_forward_rmsnorm.argtypes = [sp, _P, _P, ctypes.c_float, _P, _P, _P, _P, _P, _P, _P,
                                          _SZ, _P]
        L.moe_forward_rmsnorm.restype = st
        L.moe_pack_weights.argtypes = [sp, _P, _P, _P, _P, _P, _P, _P]
        L.moe_pack_weights.restype = st
        L.moe_forward_host.argtypes = [sp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.moe_forward_host_async.argtypes = [sp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.moe_forward_host_async.restype = st
        L.moe_forward_host.restype = st
        L.moe_device_status.argtypes = [_P, _SZ, _P]
        L.moe_device_status.restype = st
        L.moe_permute_static.argtypes = [sp, _P, _P, _P, _P, _P, _P, _P, _P]
        L.moe_permute_static.restype = st
        L.moe_selftest_wait_timeout.argtypes = [_P, _SZ, ctypes.c_uint64, _P]
        L.moe_selftest_wait_timeout.restype = st
        L.moe_quantize_int8.argtypes = [sp] + [_P] * 10
        L.moe_quantize_int8.restype = st
        L.moe_grouped_swiglu_w8.argtypes = [sp] + [_P] * 10 + [_SZ, _P]
        L.moe_grouped_swiglu_w8.restype = st
        L.moe_forward_w8.argtypes = [sp] + [_P] * 12 + [_SZ, _P]
        L.moe_forward_w8.restype = st
        L.moe_quantize_int4.argtypes = [sp] + [_P] * 10
        L.moe_quantize_int4.restype = st
        L.moe_grouped_swiglu_w4.argtypes = [sp] + [_P] * 10 + [_SZ, _P]
        L.moe_grouped_swiglu_w4.restype = st
        L.moe_forward_w4.argtypes = [sp] + [_P] * 12 + [_SZ, _P]
        L.moe_forward_w4.restype = st
        L.moe_gather_rows.argtypes = [_P, ctypes.c_int64, _P, ctypes.c_int64, ctypes.c_int64, _P, _P]
        L.moe_gather_rows.restype = st
        L.moe_ipc_alloc.argtypes = [_SZ, ctypes.POINTER(_P), _P]
        L.moe_ipc_alloc.restype = st
        L.moe_ipc_open.argtypes = [_P, ctypes.POINTER(_P)]
        L.moe_ipc_open.restype = st
        L.moe_ipc_close.argtypes = [_P]
        L.moe_ipc_close.restype = st
        L.moe_ipc_free.argtypes = [_P]
        L.moe_ipc_free.restype = st
        L.moe_scatter_rows_peer.argtypes = [_P, ctypes.c_int64, _P, _P, _P, ctypes.c_int64, _P,
                                            ctypes.c_int, ctypes.c_int64, ctypes.c_int64, _P, _P]
        L.moe_scatter_rows_peer.restype = st
        L.moe_combine_peer.argtypes = [_P, ctypes.c_int, ctypes.c_int64, _P, _P, _P, _P, _P,
                                       ctypes.c_int64, ctypes.c_int, ctypes.c_int, _P, _P]
        L.moe_combine_peer.restype = st
        L.moe_last_error.argtypes = []
        L.moe_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != 0:
        raise MoeError(status, lib().moe_last_error().decode(errors="replace"))


def make_shape(num_tokens: int, hidden_size: int, intermediate_size: int, num_experts: int,
               num_experts_per_tok: int, weight_layout: int = ROW_MAJOR,
               router_bf16_logits: bool = False) -> Shape:
    return Shape(int(num_tokens), int(hidden_size), int(intermediate_size), int(num_experts),
                 int(num_experts_per_tok), int(weight_layout), int(bool(router_bf16_logits)))


def _dev(t: Optional[torch.Tensor], name: str, dtype=None, nullable=False) -> Optional[int]:
    if t is None:
        if nullable:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _sized(name: str, t: Optional[torch.Tensor], n: int, at_least: bool = False) -> None:
    """The kernels index a buffer by the layer's shape alone (the C ABI takes bare
    pointers), so one of the wrong size would be read or written out of bounds: refuse
    it here, before any pointer is taken."""
    if t is None:
        return
    if t.numel() < n or (t.numel() != n and not at_least):
        need = f"at least {n}" if at_least else f"{n}"
        raise ValueError(f"{name} has {t.numel()} elements; the layer's shape needs {need}")


def _layer_sizes(t: int, h: int, e: int, i: int, w_router=None, logit_bias=None, residual=None,
                 out=None, **weights) -> None:
    """Element counts of the tensors of a whole-layer call: w_router [E, H], logit_bias
    [E], residual and out [T, H], and each keyword ``name=(tensor, count)``."""
    _sized("w_router", w_router, e * h)
    _sized("logit_bias", logit_bias, e)
    _sized("residual", residual, t * h)
    _sized("out", out, t * h)
    for name, (tensor, n) in weights.items():
        # x_perm may be a larger buffer: the kernels read its first R_max rows
        _sized(name, tensor, n, at_least=name == "x_perm")


def _bf16_weights(e: int, i: int, h: int, w1, w3, w2) -> dict:
    return {"w1": (w1, e * i * h), "w3": (w3, e * i * h), "w2": (w2, e * h * i)}


def _quant_weights(e: int, i: int, h: int, ex, bits: int) -> dict:
    """Codes and scales of Int8Experts (bits 8) or Int4Experts (bits 4)."""
    per = (lambda n: n) if bits == 8 else (lambda n: n // 2)
    sc = (lambda rows, k: rows) if bits == 8 else (lambda rows, k: rows * k // 64)
    return {"q1": (ex.q1, per(e * i * h)), "q3": (ex.q3, per(e * i * h)),
            "q2": (ex.q2, per(e * h * i)), "s1": (ex.s1, sc(e * i, h)),
            "s3": (ex.s3, sc(e * i, h)), "s2": (ex.s2, sc(e * h, i))}


def _stream(stream) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def workspace_size(shape: Shape) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(shape)))


def workspace_size_host(shape: Shape) -> int:
    return int(lib().moe_workspace_size_host(ctypes.byref(shape)))


def max_padded_rows(shape: Shape) -> int:
    return int(lib().moe_max_padded_rows(ctypes.byref(shape)))


def make_workspace(shape: Shape, device="cuda", host: bool = False) -> torch.Tensor:
    """A zeroed device workspace (zero status word) big enough for ``shape``."""
    n = workspace_size_host(shape) if host else workspace_size(shape)
    if n == 0:
        raise MoeError(2, lib().moe_last_error().decode(errors="replace"))
    return torch.zeros(n, dtype=torch.uint8, device=device)


def router_topk(x, w_router, k: int, logit_bias=None, return_logits=False, stream=None,
                router_bf16_logits: bool = False):
    """(topk_idx [T,k] int32, topk_w [T,k] fp32[, logits [T,E] fp32])."""
    t, h = x.shape
    e = w_router.shape[0]
    shape = make_shape(t, h, ROW_PAD, e, k, router_bf16_logits=router_bf16_logits)
    _layer_sizes(t, h, e, ROW_PAD, w_router, logit_bias)
    idx = torch.empty((t, k), dtype=torch.int32, device=x.device)
    w = torch.empty((t, k), dtype=torch.float32, device=x.device)
    logits = torch.empty((t, e), dtype=torch.float32, device=x.device) if return_logits else None
    _check(lib().moe_router_topk(ctypes.byref(shape), _dev(x, "x", torch.bfloat16),
                                 _dev(w_router, "w_router", torch.bfloat16),
                                 _dev(logit_bias, "logit_bias", torch.float32, True),
                                 _dev(idx, "idx"), _dev(w, "w"), _dev(logits, "logits", None, True),
                                 _stream(stream)))
    return (idx, w, logits) if return_logits else (idx, w)


def permute(topk_idx, x, num_experts: int, intermediate_size: int, ws, stream=None) -> dict:
    """Expert-contiguous permutation of the routed rows (see moe_permute)."""
    t, k = topk_idx.shape
    h = x.shape[1]
    shape = make_shape(t, h, intermediate_size, num_experts, k)
    _sized("x", x, t * h, at_least=True)      # the gather reads rows 0 .. T-1
    rmax = max_padded_rows(shape)
    dev = x.device
    out = {
        "counts": torch.empty(num_experts, dtype=torch.int32, device=dev),
        "offsets": torch.empty(num_experts + 1, dtype=torch.int32, device=dev),
        "row_of": torch.empty((t, k), dtype=torch.int32, device=dev),
        "token_of_row": torch.full((rmax,), -2, dtype=torch.int32, device=dev),
        "x_perm": torch.zeros((rmax, h), dtype=torch.bfloat16, device=dev),
    }
    _check(lib().moe_permute(ctypes.byref(shape), _dev(topk_idx, "topk_idx", torch.int32),
                             _dev(x, "x", torch.bfloat16), _dev(out["counts"], "counts"),
                             _dev(out["offsets"], "offsets"), _dev(out["row_of"], "row_of"),
                             _dev(out["token_of_row"], "token_of_row"), _dev(out["x_perm"], "x_perm"),
                             _dev(ws, "ws"), ws.numel(), _stream(stream)))
    return out


def permute_static(topk_idx, x, num_experts: int, intermediate_size: int, stream=None) -> dict:
    """moe_permute_static: the permutation without a workspace, for callers that cannot
    allocate device memory (its scratch is a static array in the library; calls that
    overlap on the GPU race on it). Same results as ``permute``."""
    t, k = topk_idx.shape
    h = x.shape[1]
    shape = make_shape(t, h, intermediate_size, num_experts, k)
    _sized("x", x, t * h, at_least=True)      # the gather reads rows 0 .. T-1
    rmax = max_padded_rows(shape)
    dev = x.device
    out = {
        "counts": torch.empty(num_experts, dtype=torch.int32, device=dev),
        "offsets": torch.empty(num_experts + 1, dtype=torch.int32, device=dev),
        "row_of": torch.empty((t, k), dtype=torch.int32, device=dev),
        "token_of_row": torch.full((rmax,), -2, dtype=torch.int32, device=dev),
        "x_perm": torch.zeros((rmax, h), dtype=torch.bfloat16, device=dev),
    }
    _check(lib().moe_permute_static(ctypes.byref(shape), _dev(topk_idx, "topk_idx", torch.int32),
                                    _dev(x, "x", torch.bfloat16), _dev(out["counts"], "counts"),
                                    _dev(out["offsets"], "offsets"), _dev(out["row_of"], "row_of"),
                                    _dev(out["token_of_row"], "token_of_row"),
                                    _dev(out["x_perm"], "x_perm"), _stream(stream)))
    return out


def _out_rows(y, rows: int, h: int, device):
    """The experts' fp32 output: y itself (its first rows x h elements are written; it
    must hold at least that many), or a new zeroed [rows, h] tensor."""
    if y is None:
        return torch.zeros((rows, h), dtype=torch.float32, device=device)
    _sized("y_perm", y, rows * h, at_least=True)
    return y


def grouped_swiglu(x_perm, offsets, w1, w3, w2, num_tokens: int, k: int, ws, stream=None,
                   weight_layout: int = ROW_MAJOR, y=None):
    """y_perm [R_max, H] fp32 = w2[e] (silu(w1[e] x) * w3[e] x) per routed row (into
    `y` when given: an fp32 CUDA tensor of at least R_max x H elements)."""
    e, i, h = w1.shape
    shape = make_shape(num_tokens, h, i, e, k, weight_layout)
    _layer_sizes(0, h, e, i, x_perm=(x_perm, max_padded_rows(shape) * h),
                 offsets=(offsets, e + 1), **_bf16_weights(e, i, h, w1, w3, w2))
    y = _out_rows(y, max_padded_rows(shape), h, x_perm.device)
    _check(lib().moe_grouped_swiglu(ctypes.byref(shape), _dev(x_perm, "x_perm", torch.bfloat16),
                                    _dev(offsets, "offsets", torch.int32),
                                    _dev(w1, "w1", torch.bfloat16), _dev(w3, "w3", torch.bfloat16),
                                    _dev(w2, "w2", torch.bfloat16), _dev(y, "y_perm"),
                                    _dev(ws, "ws"), ws.numel(), _stream(stream)))
    return y


def expert_gate_up(x_perm, offsets, w1, w3, num_tokens: int, k: int, ws, h=None, stream=None,
                   weight_layout: int = ROW_MAJOR):
    """h [R_max, I] bf16 = bf16(silu(x_perm w1[e]^T) * (x_perm w3[e]^T)) (GEMM1 alone)."""
    e, i, hd = w1.shape
    shape = make_shape(num_tokens, hd, i, e, k, weight_layout)
    if h is None:
        h = torch.zeros((max_padded_rows(shape), i), dtype=torch.bfloat16, device=x_perm.device)
    _check(lib().moe_expert_gate_up(ctypes.byref(shape), _dev(x_perm, "x_perm", torch.bfloat16),
                                    _dev(offsets, "offsets", torch.int32),
                                    _dev(w1, "w1", torch.bfloat16), _dev(w3, "w3", torch.bfloat16),
                                    _dev(h, "h", torch.bfloat16), _dev(ws, "ws"), ws.numel(),
                                    _stream(stream)))
    return h


def expert_down(h, offsets, w2, num_tokens: int, k: int, ws, y=None, stream=None,
                weight_layout: int = ROW_MAJOR):
    """y_perm [R_max, H] fp32 = h w2[e]^T (GEMM2 alone)."""
    e, hd, i = w2.shape
    shape = make_shape(num_tokens, hd, i, e, k, weight_layout)
    if y is None:
        y = torch.zeros((max_padded_rows(shape), hd), dtype=torch.float32, device=h.device)
    _check(lib().moe_expert_down(ctypes.byref(shape), _dev(h, "h", torch.bfloat16),
                                 _dev(offsets, "offsets", torch.int32), _dev(w2, "w2", torch.bfloat16),
                                 _dev(y, "y_perm", torch.float32), _dev(ws, "ws"), ws.numel(),
                                 _stream(stream)))
    return y


def combine(y_perm, row_of, topk_w, residual=None, num_experts: int = 8, intermediate_size: int = ROW_PAD,
            stream=None):
    """out [T,H] bf16 = residual + sum_j topk_w[:,j] * y_perm[row_of[:,j]]."""
    t, k = row_of.shape
    h = y_perm.shape[1]
    shape = make_shape(t, h, intermediate_size, max(num_experts, k), k)
    _sized("topk_w", topk_w, t * k)
    _sized("residual", residual, t * h)
    out = torch.empty((t, h), dtype=torch.bfloat16, device=y_perm.device)
    _check(lib().moe_combine(ctypes.byref(shape), _dev(y_perm, "y_perm", torch.float32),
                             _dev(row_of, "row_of", torch.int32), _dev(topk_w, "topk_w", torch.float32),
                             _dev(residual, "residual", torch.bfloat16, True), _dev(out, "out"),
                             _stream(stream)))
    return out


def forward(x, w_router, w1, w3, w2, k: int, residual=None, logit_bias=None, ws=None, out=None,
            stream=None, weight_layout: int = ROW_MAJOR, router_bf16_logits: bool = False):
    """The whole layer on device tensors; returns out [T,H] bf16."""
    t, h = x.shape
    e, i, _ = w1.shape
    shape = make_shape(t, h, i, e, k, weight_layout, router_bf16_logits)
    _layer_sizes(t, h, e, i, w_router, logit_bias, residual, out,
                 **_bf16_weights(e, i, h, w1, w3, w2))
    if ws is None:
        ws = make_workspace(shape, x.device)
    if out is None:
        out = torch.empty((t, h), dtype=torch.bfloat16, device=x.device)
    _check(lib().moe_forward(ctypes.byref(shape), _dev(x, "x", torch.bfloat16),
                             _dev(w_router, "w_router", torch.bfloat16),
                             _dev(logit_bias, "logit_bias", torch.float32, True),
                             _dev(w1, "w1", torch.bfloat16), _dev(w3, "w3", torch.bfloat16),
                             _dev(w2, "w2", torch.bfloat16),
                             _dev(residual, "residual", torch.bfloat16, True), _dev(out, "out"),
                             _dev(ws, "ws"), ws.numel(), _stream(stream)))
    return out


def forward_rmsnorm(h, norm_weight, eps: float, w_router, w1, w3, w2, k: int, logit_bias=None,
                    ws=None, out=None, stream=None, weight_layout: int = ROW_MAJOR):
    """out = h + moe(rms_norm(h)) on device tensors (the mixture half of the block)."""
    t, hd = h.shape
    e, i, _ = w1.shape
    shape = make_shape(t, hd, i, e, k, weight_layout)
    _layer_sizes(t, hd, e, i, w_router, logit_bias, None, out, norm_weight=(norm_weight, hd),
                 **_bf16_weights(e, i, hd, w1, w3, w2))
    if ws is None:
        ws = make_workspace(shape, h.device)
    if out is None:
        out = torch.empty((t, hd), dtype=torch.bfloat16, device=h.device)
    _check(lib().moe_forward_rmsnorm(ctypes.byref(shape), _dev(h, "h", torch.bfloat16),
                                     _dev(norm_weight, "norm_weight", torch.bfloat16), float(eps),
                                     _dev(w_router, "w_router", torch.bfloat16),
                                     _dev(logit_bias, "logit_bias", torch.float32, True),
                                     _dev(w1, "w1", torch.bfloat16), _dev(w3, "w3", torch.bfloat16),
                                     _dev(w2, "w2", torch.bfloat16), _dev(out, "out"),
                                     _dev(ws, "ws"), ws.numel(), _stream(stream)))
    return out


def forward_host(x_host, w_router, w1, w3, w2, k: int, residual_host=None, logit_bias=None,
                 ws=None, out_host=None, stream=None, weight_layout: int = ROW_MAJOR,
                 wait: bool = True):
    """The layer with host (ideally pinned) activations; returns out_host. With
    wait=False the call only enqueues (moe_forward_host_async): out_host is ready once
    the stream has been synchronised."""
    t, h = x_host.shape
    e, i, _ = w1.shape
    shape = make_shape(t, h, i, e, k, weight_layout)
    _layer_sizes(t, h, e, i, w_router, logit_bias, residual_host=(residual_host, t * h),
                 out_host=(out_host, t * h), **_bf16_weights(e, i, h, w1, w3, w2))
    for name, a in (("x_host", x_host), ("residual_host", residual_host), ("out_host", out_host)):
        if a is not None and (a.is_cuda or a.dtype != torch.bfloat16 or not a.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous bf16 host tensor")
    if ws is None:
        ws = make_workspace(shape, w1.device, host=True)
    if out_host is None:
        out_host = torch.empty((t, h), dtype=torch.bfloat16, pin_memory=True)
    fn = lib().moe_forward_host if wait else lib().moe_forward_host_async
    _check(fn(ctypes.byref(shape), x_host.data_ptr(),
                                  _dev(w_router, "w_router", torch.bfloat16),
                                  _dev(logit_bias, "logit_bias", torch.float32, True),
                                  _dev(w1, "w1", torch.bfloat16), _dev(w3, "w3", torch.bfloat16),
                                  _dev(w2, "w2", torch.bfloat16),
                                  None if residual_host is None else residual_host.data_ptr(),
                                  out_host.data_ptr(), _dev(ws, "ws"), ws.numel(), _stream(stream)))
    return out_host


def selftest_wait_timeout(ws, timeout_ns: int, stream=None) -> None:
    """Launch the bounded-wait check: a wait that nothing completes gives up after
    ``timeout_ns`` and records MOE_ERR_TIMEOUT in ``ws``'s status word."""
    _check(lib().moe_selftest_wait_timeout(_dev(ws, "ws"), ws.numel(), int(timeout_ns), _stream(stream)))


def pack_weights(w1, w3, w2, stream=None):
    """Row-major expert weights -> the blocked layout (new tensors of the same shapes);
    pass weight_layout=BLOCKED with them."""
    e, i, h = w1.shape
    shape = make_shape(1, h, i, e, 1)
    out = [torch.empty_like(t) for t in (w1, w3, w2)]
    _check(lib().moe_pack_weights(ctypes.byref(shape), _dev(w1, "w1", torch.bfloat16),
                                  _dev(w3, "w3", torch.bfloat16), _dev(w2, "w2", torch.bfloat16),
                                  _dev(out[0], "w1_blocked"), _dev(out[1], "w3_blocked"),
                                  _dev(out[2], "w2_blocked"), _stream(stream)))
    return tuple(out)


def device_status(ws, stream=None) -> None:
    """Raise MoeError(MOE_ERR_TIMEOUT) if a kernel gave up a bounded wait since last checked."""
    _check(lib().moe_device_status(_dev(ws, "ws"), ws.numel(), _stream(stream)))


def quantize_int8(w1, w3, w2, stream=None) -> Int8Experts:
    """Row-major bf16 expert weights -> Int8Experts (per-row symmetric int8)."""
    e, i, h = w1.shape
    shape = make_shape(1, h, i, e, 1)
    dev = w1.device
    q = [torch.empty(t.shape, dtype=torch.uint8, device=dev) for t in (w1, w3, w2)]
    sc = [torch.empty((e, i), dtype=torch.float32, device=dev),
          torch.empty((e, i), dtype=torch.float32, device=dev),
          torch.empty((e, h), dtype=torch.float32, device=dev)]
    out = Int8Experts(q[0], q[1], q[2], sc[0], sc[1], sc[2])
    _check(lib().moe_quantize_int8(ctypes.byref(shape), _dev(w1, "w1", torch.bfloat16),
                                   _dev(w3, "w3", torch.bfloat16), _dev(w2, "w2", torch.bfloat16),
                                   *out.pointers(), _stream(stream)))
    return out


def grouped_swiglu_w8(x_perm, offsets, experts: Int8Experts, num_tokens: int, k: int, ws,
                      stream=None, y=None):
    """grouped_swiglu with int8 expert weights: y_perm [R_max, H] fp32 (into `y` when
    given)."""
    e, i, h = experts.q1.shape
    shape = make_shape(num_tokens, h, i, e, k)
    _layer_sizes(0, h, e, i, x_perm=(x_perm, max_padded_rows(shape) * h),
                 offsets=(offsets, e + 1), **_quant_weights(e, i, h, experts, 8))
    y = _out_rows(y, max_padded_rows(shape), h, x_perm.device)
    _check(lib().moe_grouped_swiglu_w8(ctypes.byref(shape), _dev(x_perm, "x_perm", torch.bfloat16),
                                       _dev(offsets, "offsets", torch.int32), *experts.pointers(),
                                       _dev(y, "y_perm"), _dev(ws, "ws"), ws.numel(),
                                       _stream(stream)))
    return y


def forward_w8(x, w_router, experts: Int8Experts, k: int, residual=None, logit_bias=None,
               ws=None, out=None, stream=None, router_bf16_logits: bool = False):
    """The whole layer with int8 expert weights; returns out [T,H] bf16."""
    t, h = x.shape
    e, i, _ = experts.q1.shape
    shape = make_shape(t, h, i, e, k, ROW_MAJOR, router_bf16_logits)
    _layer_sizes(t, h, e, i, w_router, logit_bias, residual, out,
                 **_quant_weights(e, i, h, experts, 8))
    if ws is None:
        ws = make_workspace(shape, x.device)
    if out is None:
        out = torch.empty((t, h), dtype=torch.bfloat16, device=x.device)
    _check(lib().moe_forward_w8(ctypes.byref(shape), _dev(x, "x", torch.bfloat16),
                                _dev(w_router, "w_router", torch.bfloat16),
                                _dev(logit_bias, "logit_bias", torch.float32, True),
                                *experts.pointers(),
                                _dev(residual, "residual", torch.bfloat16, True), _dev(out, "out"),
                                _dev(ws, "ws"), ws.numel(), _stream(stream)))
    return out


def quantize_int4(w1, w3, w2, stream=None) -> Int4Experts:
    """Row-major bf16 expert weights -> Int4Experts (symmetric 4-bit, a half scale per
    64-column group of a row)."""
    e, i, h = w1.shape
    shape = make_shape(1, h, i, e, 1)
    dev = w1.device
    q = [torch.empty((e, i, h // 2), dtype=torch.uint8, device=dev),
         torch.empty((e, i, h // 2), dtype=torch.uint8, device=dev),
         torch.empty((e, h, i // 2), dtype=torch.uint8, device=dev)]
    sc = [torch.empty((e, i // 128, h // 64, 128), dtype=torch.float16, device=dev),
          torch.empty((e, i // 128, h // 64, 128), dtype=torch.float16, device=dev),
          torch.empty((e, h // 128, i // 64, 128), dtype=torch.float16, device=dev)]
    out = Int4Experts(q[0], q[1], q[2], sc[0], sc[1], sc[2])
    _check(lib().moe_quantize_int4(ctypes.byref(shape), _dev(w1, "w1", torch.bfloat16),
                                   _dev(w3, "w3", torch.bfloat16), _dev(w2, "w2", torch.bfloat16),
                                   *out.pointers(), _stream(stream)))
    return out


def grouped_swiglu_w4(x_perm, offsets, experts: Int4Experts, num_tokens: int, k: int, ws,
                      stream=None, y=None):
    """grouped_swiglu with 4-bit expert weights: y_perm [R_max, H] fp32 (into `y` when
    given)."""
    e, i, h2 = experts.q1.shape
    shape = make_shape(num_tokens, 2 * h2, i, e, k)
    _layer_sizes(0, 2 * h2, e, i, x_perm=(x_perm, max_padded_rows(shape) * 2 * h2),
                 offsets=(offsets, e + 1), **_quant_weights(e, i, 2 * h2, experts, 4))
    y = _out_rows(y, max_padded_rows(shape), 2 * h2, x_perm.device)
    _check(lib().moe_grouped_swiglu_w4(ctypes.byref(shape), _dev(x_perm, "x_perm", torch.bfloat16),
                                       _dev(offsets, "offsets", torch.int32), *experts.pointers(),
                                       _dev(y, "y_perm"), _dev(ws, "ws"), ws.numel(),
                                       _stream(stream)))
    return y


def forward_w4(x, w_router, experts: Int4Experts, k: int, residual=None, logit_bias=None,
               ws=None, out=None, stream=None, router_bf16_logits: bool = False):
    """The whole layer with 4-bit expert weights; returns out [T,H] bf16."""
    t, h = x.shape
    e, i, _ = experts.q1.shape
    shape = make_shape(t, h, i, e, k, ROW_MAJOR, router_bf16_logits)
    _layer_sizes(t, h, e, i, w_router, logit_bias, residual, out,
                 **_quant_weights(e, i, h, experts, 4))
    if ws is None:
        ws = make_workspace(shape, x.device)
    if out is None:
        out = torch.empty((t, h), dtype=torch.bfloat16, device=x.device)
    _check(lib().moe_forward_w4(ctypes.byref(shape), _dev(x, "x", torch.bfloat16),
                                _dev(w_router, "w_router", torch.bfloat16),
                                _dev(logit_bias, "logit_bias", torch.float32, True),
                                *experts.pointers(),
                                _dev(residual, "residual", torch.bfloat16, True), _dev(out, "out"),
                                _dev(ws, "ws"), ws.numel(), _stream(stream)))
    return out


def gather_rows(src, index, stream=None):
    """out[i] = src[index[i]] (a zero row where index[i] is outside [0, len(src))); src is
    a 2-D CUDA tensor whose rows are a multiple of 16 bytes, index an int64 CUDA tensor."""
    if src.dim() != 2:
        raise ValueError("src must be 2-D")
    n = index.numel()
    out = torch.empty((n, src.shape[1]), dtype=src.dtype, device=src.device)
    row_bytes = src.shape[1] * src.element_size()
    _check(lib().moe_gather_rows(_dev(src, "src") if src.shape[0] else None, src.shape[0],
                                 _dev(index, "index", torch.int64) if n else None, n, row_bytes,
                                 _dev(out, "dst") if n else None, _stream(stream)))
    return out


# ---- expert parallelism over peer memory ----

IPC_HANDLE_BYTES = 64


def ipc_alloc(nbytes: int):
    """A device buffer other processes can map: (device address, IPC handle bytes). The
    caller frees it with ipc_free once every other process has unmapped it."""
    ptr = _P()
    handle = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    _check(lib().moe_ipc_alloc(int(nbytes), ctypes.byref(ptr), ctypes.cast(handle, _P)))
    return int(ptr.value), handle.raw


def ipc_open(handle: bytes) -> int:
    """Address in this process of another process's ipc_alloc buffer."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {IPC_HANDLE_BYTES} bytes, got {len(handle)}")
    buf = ctypes.create_string_buffer(bytes(handle), IPC_HANDLE_BYTES)
    ptr = _P()
    _check(lib().moe_ipc_open(ctypes.cast(buf, _P), ctypes.byref(ptr)))
    return int(ptr.value)


def ipc_close(ptr: int) -> None:
    _check(lib().moe_ipc_close(ptr))


def ipc_free(ptr: int) -> None:
    _check(lib().moe_ipc_free(ptr))


class _DeviceArray:
    """A contiguous device array described to torch by its address
    (__cuda_array_interface__); torch.as_tensor then wraps it without copying."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 2, "strides": None}


_TYPESTR = {torch.bfloat16: ("<i2", torch.int16), torch.float32: ("<f4", torch.float32),
            torch.int32: ("<i4", torch.int32), torch.int64: ("<i8", torch.int64)}


def tensor_at(ptr: int, shape, dtype, device) -> torch.Tensor:
    """A tensor over device memory this library allocated (it does not own the memory:
    keep the buffer alive while the tensor is used)."""
    typestr, base = _TYPESTR[dtype]
    t = torch.as_tensor(_DeviceArray(ptr, shape, typestr), device=device)
    return t.view(dtype) if base != dtype else t


def scatter_rows_peer(src, src_index, dst_rank, dst_row, dst_bases, dst_rows: int, bad=None,
                      stream=None) -> None:
    """Row dst_row[i] of buffer dst_bases[dst_rank[i]] = src[src_index[i]] for every i.
    src: 2-D CUDA tensor (rows a multiple of 16 bytes); src_index, dst_row int64 and
    dst_rank int32 CUDA tensors of one length; dst_bases: int64 CUDA tensor of device
    addresses (this GPU's buffers or ipc_open mappings), each buffer dst_rows rows of
    src's row size. Out-of-range rows are skipped and counted into `bad` (int32 CUDA
    tensor of one element) when given."""
    if src.dim() != 2:
        raise ValueError("src must be 2-D")
    n = src_index.numel()
    if dst_rank.numel() != n or dst_row.numel() != n:
        raise ValueError("src_index, dst_rank and dst_row must have the same length")
    if n == 0:
        return
    _check(lib().moe_scatter_rows_peer(
        _dev(src, "src") if src.shape[0] else None, src.shape[0],
        _dev(src_index, "src_index", torch.int64), _dev(dst_rank, "dst_rank", torch.int32),
        _dev(dst_row, "dst_row", torch.int64), n, _dev(dst_bases, "dst_bases", torch.int64),
        dst_bases.numel(), int(dst_rows), src.shape[1] * src.element_size(),
        _dev(bad, "bad", torch.int32, True), _stream(stream)))


def combine_peer(y_bases, y_rows: int, slot_rank, slot_row, topk_w, hidden: int, residual=None,
                 bad=None, stream=None):
    """out [T, hidden] bf16 = residual + sum_j topk_w[:, j] * (row slot_row[t k + j] of
    the fp32 buffer y_bases[slot_rank[t k + j]]), moe_combine's arithmetic. y_bases:
    int64 CUDA tensor of device addresses, each buffer y_rows x hidden fp32; slot_rank
    int32 and slot_row int64 CUDA tensors [T, k]; topk_w fp32 [T, k]."""
    t, k = topk_w.shape
    _sized("slot_rank", slot_rank, t * k)
    _sized("slot_row", slot_row, t * k)
    _sized("residual", residual, t * hidden)
    out = torch.empty((t, hidden), dtype=torch.bfloat16, device=topk_w.device)
    if t == 0:
        return out
    _check(lib().moe_combine_peer(
        _dev(y_bases, "y_bases", torch.int64), y_bases.numel(), int(y_rows),
        _dev(slot_rank, "slot_rank", torch.int32), _dev(slot_row, "slot_row", torch.int64),
        _dev(topk_w, "topk_w", torch.float32), _dev(residual, "residual", torch.bfloat16, True),
        _dev(out, "out"), t, k, hidden, _dev(bad, "bad", torch.int32, True), _stream(stream)))
    return out

