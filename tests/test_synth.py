"""The seeded generator: SplitMix64 bits, Box-Muller normals, bf16 storage."""
import math

import pytest
import torch

from sparse_mixture_experts_09_b200 import synth, workloads


def test_splitmix64_published_vector():
    # Outputs 1..5 of SplitMix64 seeded with 1234567, as printed by the reference C
    # implementation that accompanies the SplitMix64 paper (Vigna's splitmix64.c).
    expected = [6457827717110365317, 3203168211198807973, 9817491932198370423,
                4593380528125082431, 16408922859458223821]
    got = [synth.splitmix64_scalar(1234567 + n * 0x9E3779B97F4A7C15) for n in range(1, 6)]
    assert got == expected


def test_tensor_splitmix_matches_scalar():
    key = synth.stream_key(7, 3, 1)
    idx = torch.arange(0, 4096, dtype=torch.int64) * 7919 + 123456789
    bits = synth.uniform_bits(key, idx)
    for i in range(0, 4096, 97):
        want = synth.splitmix64_scalar(key + int(idx[i]) * 0x9E3779B97F4A7C15)
        assert int(bits[i]) & ((1 << 64) - 1) == want


def test_normals_moments():
    z = synth.standard_normal_f64(synth.stream_key(0, 0), 0, 1 << 20, "cpu")
    assert abs(float(z.mean())) < 5e-3
    assert abs(float(z.var()) - 1.0) < 5e-3
    # fourth moment of N(0,1) is 3
    assert abs(float((z ** 4).mean()) - 3.0) < 0.05


def test_normal_is_chunk_and_slice_invariant():
    full = synth.normal((64, 96), 0.5, 3, 2)
    part = synth.normal((16, 96), 0.5, 3, 2, first_row=20)
    assert torch.equal(full[20:36], part)
    rows = torch.tensor([0, 5, 63])
    assert torch.equal(synth.rows_at(rows, 96, 0.5, 3, 2, 0, False), full[rows])
    u = synth.normal_rows_unit_rms(64, 96, 3, 2)
    assert torch.equal(synth.rows_at(rows, 96, 1.0, 3, 2, 0, True), u[rows])


def test_unit_rms_rows():
    u = synth.normal_rows_unit_rms(32, 4096, 1, 0).double()
    rms = u.pow(2).mean(dim=1).sqrt()
    assert torch.allclose(rms, torch.ones_like(rms), atol=4e-3)


def test_weight_scale():
    w = workloads.WORKLOADS["tiny"]
    wr, w1, w3, w2 = workloads.draw_weights(w)
    assert w1.shape == (8, 256, 128) and w2.shape == (8, 128, 256)
    assert abs(float(w1.double().std()) - 1 / math.sqrt(128)) < 2e-3
    assert abs(float(w2.double().std()) - 1 / math.sqrt(256)) < 2e-3
    assert w1.dtype == torch.bfloat16


def test_streams_are_distinct():
    a = synth.normal((1024,), 1.0, 0, 2)
    b = synth.normal((1024,), 1.0, 0, 3)
    c = synth.normal((1024,), 1.0, 0, 2, attempt=1)
    assert not torch.equal(a, b) and not torch.equal(a, c)


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_workload_shapes_follow_config(name):
    w = workloads.WORKLOADS[name]
    assert w.hidden_size % 128 == 0 and w.intermediate_size % 128 == 0
    assert w.num_experts == 8 and w.num_experts_per_tok == 2


def test_workload_names_resolve():
    import pytest as _pt
    from sparse_mixture_experts_09_b200 import workloads as W
    assert W.workload("decode") is W.WORKLOADS["decode"]
    for t in (1, 4, 16, 64, 256):
        w = W.workload(f"larger_decode_T{t}")
        assert (w.num_tokens, w.hidden_size, w.intermediate_size) == (t, 6144, 16384)
    with _pt.raises(KeyError):
        W.workload("larger_decode_T3")
