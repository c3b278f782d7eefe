"""The binding refuses tensors whose element counts do not fit the layer's shape
before it takes any pointer (the C ABI sees bare pointers, so the kernels would read or
write past a short buffer). Runs on CPU: well-sized CPU tensors get past the size checks
and are then refused as not being on a CUDA device."""
import pytest
import torch

from sparse_mixture_experts_09_b200 import moe as M

T, H, I, E, K = 5, 128, 256, 4, 2


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def _layer():
    return dict(x=_bf16(T, H), w_router=_bf16(E, H), w1=_bf16(E, I, H), w3=_bf16(E, I, H),
                w2=_bf16(E, H, I), residual=_bf16(T, H), out=_bf16(T, H),
                logit_bias=torch.zeros(E, dtype=torch.float32))


def _int8():
    u8 = lambda *s: torch.zeros(s, dtype=torch.uint8)
    f32 = lambda *s: torch.zeros(s, dtype=torch.float32)
    return M.Int8Experts(u8(E, I, H), u8(E, I, H), u8(E, H, I), f32(E, I), f32(E, I), f32(E, H))


def _int4():
    u8 = lambda *s: torch.zeros(s, dtype=torch.uint8)
    f16 = lambda *s: torch.zeros(s, dtype=torch.float16)
    return M.Int4Experts(u8(E, I, H // 2), u8(E, I, H // 2), u8(E, H, I // 2),
                         f16(E, I // 128, H // 64, 128), f16(E, I // 128, H // 64, 128),
                         f16(E, H // 128, I // 64, 128))


def _forward(a):
    return M.forward(a["x"], a["w_router"], a["w1"], a["w3"], a["w2"], K, residual=a["residual"],
                     logit_bias=a["logit_bias"], out=a["out"])


def test_well_sized_layer_reaches_the_device_check():
    with pytest.raises(ValueError, match="CUDA"):
        _forward(_layer())
    a = _layer()
    with pytest.raises(ValueError, match="CUDA"):
        M.forward_rmsnorm(a["x"], _bf16(H), 1e-5, a["w_router"], a["w1"], a["w3"], a["w2"], K,
                          out=a["out"])
    with pytest.raises(ValueError, match="CUDA"):
        M.forward_w8(a["x"], a["w_router"], _int8(), K, residual=a["residual"], out=a["out"])
    with pytest.raises(ValueError, match="CUDA"):
        M.forward_w4(a["x"], a["w_router"], _int4(), K, residual=a["residual"], out=a["out"])
    with pytest.raises(ValueError, match="CUDA"):
        M.forward_host(a["x"], a["w_router"], a["w1"], a["w3"], a["w2"], K,
                       residual_host=a["residual"], out_host=a["out"])
    rmax = M.max_padded_rows(M.make_shape(T, H, I, E, K))
    offsets = torch.zeros(E + 1, dtype=torch.int32)
    for x_perm in (_bf16(rmax, H), _bf16(rmax + 7, H)):        # a larger buffer is fine
        with pytest.raises(ValueError, match="CUDA"):
            M.grouped_swiglu(x_perm, offsets, a["w1"], a["w3"], a["w2"], T, K, torch.zeros(8))
    with pytest.raises(ValueError, match="CUDA"):
        M.grouped_swiglu_w8(_bf16(rmax, H), offsets, _int8(), T, K, torch.zeros(8))
    with pytest.raises(ValueError, match="CUDA"):
        M.grouped_swiglu_w4(_bf16(rmax, H), offsets, _int4(), T, K, torch.zeros(8))


@pytest.mark.parametrize("name,bad", [
    ("w2", _bf16(E, H + 128, I)),          # the hidden size of another layer
    ("w3", _bf16(E - 1, I, H)),
    ("w_router", _bf16(E, H // 2)),
    ("residual", _bf16(T - 1, H)),
    ("out", _bf16(T, H // 2)),
    ("logit_bias", torch.zeros(E + 1, dtype=torch.float32)),
])
def test_mis_sized_layer_tensor_is_refused(name, bad):
    a = _layer()
    a[name] = bad
    with pytest.raises(ValueError, match=name):
        _forward(a)


def test_mis_sized_quantised_experts_and_buffers_are_refused():
    a = _layer()
    ex = _int8()
    ex.s2 = torch.zeros(E, I, dtype=torch.float32)     # the scales of w1, not w2
    with pytest.raises(ValueError, match="s2"):
        M.forward_w8(a["x"], a["w_router"], ex, K, out=a["out"])
    ex4 = _int4()
    ex4.q2 = torch.zeros(E, H, I, dtype=torch.uint8)   # int8-sized codes
    with pytest.raises(ValueError, match="q2"):
        M.forward_w4(a["x"], a["w_router"], ex4, K, out=a["out"])
    rmax = M.max_padded_rows(M.make_shape(T, H, I, E, K))
    with pytest.raises(ValueError, match="x_perm"):
        M.grouped_swiglu(_bf16(rmax - 1, H), torch.zeros(E + 1, dtype=torch.int32),
                         a["w1"], a["w3"], a["w2"], T, K, torch.zeros(8))
    with pytest.raises(ValueError, match="offsets"):
        M.grouped_swiglu(_bf16(rmax, H), torch.zeros(E, dtype=torch.int32),
                         a["w1"], a["w3"], a["w2"], T, K, torch.zeros(8))
    with pytest.raises(ValueError, match="out_host"):
        M.forward_host(a["x"], a["w_router"], a["w1"], a["w3"], a["w2"], K,
                       out_host=_bf16(T - 1, H))


def test_split_entry_points_check_sizes():
    x = _bf16(T, H)
    with pytest.raises(ValueError, match="CUDA"):
        M.router_topk(x, _bf16(E, H), K, torch.zeros(E, dtype=torch.float32))
    with pytest.raises(ValueError, match="w_router"):
        M.router_topk(x, _bf16(E, H // 2), K)
    with pytest.raises(ValueError, match="logit_bias"):
        M.router_topk(x, _bf16(E, H), K, torch.zeros(E - 1, dtype=torch.float32))
    idx = torch.zeros((T, K), dtype=torch.int32)
    for fn, extra in ((M.permute, (torch.zeros(8),)), (M.permute_static, ())):
        with pytest.raises(ValueError, match="CUDA"):
            fn(idx, _bf16(T + 3, H), E, I, *extra)           # more rows than tokens is fine
        with pytest.raises(ValueError, match="x has"):
            fn(idx, _bf16(T - 1, H), E, I, *extra)
    y = torch.zeros((40, H), dtype=torch.float32)           # rows as the caller's groups need
    row_of = torch.zeros((T, K), dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        M.combine(y, row_of, torch.zeros((T, K)), _bf16(T, H), E, I)
    with pytest.raises(ValueError, match="topk_w"):
        M.combine(y, row_of, torch.zeros((T, K + 1)), None, E, I)
    with pytest.raises(ValueError, match="residual"):
        M.combine(y, row_of, torch.zeros((T, K)), _bf16(T, H + 128), E, I)


def test_profile_driver_parses_and_needs_a_gpu():
    import pytest as _pt
    from sparse_mixture_experts_09_b200 import profile_run
    with _pt.raises(SystemExit) as e:
        profile_run.main(["--help"])
    assert e.value.code == 0
    if not torch.cuda.is_available():
        # no CPU fallback: drawing the inputs on a CUDA device fails loudly
        with _pt.raises((RuntimeError, AssertionError)):
            profile_run.main(["--path", "int4", "tiny"])
