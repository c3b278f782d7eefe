"""The quantised kernels' widening steps, restated in numpy half arithmetic and checked
exhaustively on CPU:
- int8: the half with high byte 0x64 and low byte u is 1024 + u, and 1024 + u - 1152
  is u - 128 exactly, for every code byte u;
- 4-bit: 0x6400 | n is 1024 + n and 1024 + n - 1032 is n - 8 exactly, and the packed
  half multiply by a group scale s rounds q * s once, which is what the oracle's
  dequantisation defines, for all 15 codes and every positive finite half scale
  (subnormal ones included)."""
import numpy as np

from oracle import moe_oracle as O


def _half(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16)


def test_int8_codes_widen_exactly():
    u = np.arange(256, dtype=np.uint16)
    h = _half(0x6400 | u)
    assert np.array_equal(h.astype(np.float64), 1024.0 + u)
    q = h - _half(0x6480)                       # 1152 = 1024 + 128
    assert np.array_equal(q.astype(np.float64), u.astype(np.float64) - 128)


def test_int4_codes_widen_and_scale_as_the_oracle_dequantises():
    n = np.arange(16, dtype=np.uint16)
    h = _half(0x6400 | n)
    assert np.array_equal(h.astype(np.float64), 1024.0 + n)
    q = (h - _half(0x6408))[1:]                 # 1032 = 1024 + 8; codes 1 .. 15
    assert np.array_equal(q.astype(np.float64), np.arange(-7, 8, dtype=np.float64))
    scales = _half(np.arange(1, 0x7C00, dtype=np.uint16))       # every positive finite half
    with np.errstate(over="ignore"):             # 7 * s beyond 65504 rounds to infinity
        prod = (q[:, None] * scales[None, :]).astype(np.float64)  # numpy: one rounding to half
    codes = np.broadcast_to(np.arange(-7, 8, dtype=np.int8)[:, None], prod.shape)
    # one 64-column "group" per (code, scale) pair: the oracle's dequantisation
    want = O.dequantize_int4_groups(np.repeat(codes[..., None], 64, -1).reshape(-1, 64),
                                    np.broadcast_to(scales, prod.shape).reshape(-1, 1))
    assert np.array_equal(want[:, 0], prod.reshape(-1))
