"""The 4-bit code layout as the C header states it: codes packed here from that
statement, byte by byte, are decoded back by the GPU tests' helper (so the helper that
the 4-bit parity tests read the library's codes with is itself checked), and the
header's scale order matches the scale tensors' shape."""
import numpy as np
import torch

from oracle import moe_oracle as O

from .test_gpu_w4 import unblock4


def _pack_from_header(q, k):
    """Offset-binary u = q + 8; tile (row / 128, col / 64) is 4 KiB block number
    (row / 128) * (K / 64) + col / 64; inside, the 32-bit word at byte (c / 32) * 2048 +
    r * 16 + ((c % 32) / 8) * 4 holds the code in nibble (c % 8) / 2 for even c, 4 +
    (c % 8) / 2 for odd c (r = row % 128, c = col % 64)."""
    rows = q.shape[0]
    words = np.zeros(rows * k // 8, dtype=np.uint32)
    for row in range(rows):
        for col in range(k):
            r, c = row % 128, col % 64
            block = (row // 128) * (k // 64) + col // 64
            byte = block * 4096 + (c // 32) * 2048 + r * 16 + ((c % 32) // 8) * 4
            nib = (c % 8) // 2 if c % 2 == 0 else 4 + (c % 8) // 2
            words[byte // 4] |= np.uint32((int(q[row, col]) + 8) << (4 * nib))
    return words.view(np.uint8)


def _scales_from_header(s16, rows, k):
    out = np.zeros(rows * k // 64, dtype=np.float16)
    for row in range(rows):
        for g in range(k // 64):
            out[((row // 128) * (k // 64) + g) * 128 + row % 128] = s16[row, g]
    return out


def test_unblock4_inverts_the_header_layout():
    rng = np.random.default_rng(31)
    e, r, k = 2, 256, 192
    w = O.round_bf16(rng.standard_normal((e * r, k)) * 0.05)
    q, s16 = O.quantize_int4_groups(w)
    packed = torch.from_numpy(_pack_from_header(q, k).copy()).reshape(e, r, k // 2)
    scales = torch.from_numpy(_scales_from_header(s16, e * r, k)).reshape(e, r // 128, k // 64, 128)
    got_q, got_s = unblock4(packed, scales)
    assert np.array_equal(got_q.reshape(e * r, k), q)
    assert np.array_equal(got_s.reshape(e * r, k // 64), s16)
