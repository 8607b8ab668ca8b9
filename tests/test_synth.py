"""The seeded input generator shared by the oracle and the GPU path: splitmix64 against
its published reference outputs (state 0), the uniform and normal streams' ranges and
moments, and the BF16 rounding of the generated tensors."""
import numpy as np

import synth


def test_splitmix64_reference_outputs():
    # the first three outputs of Vigna's splitmix64 started from state 0
    z = synth._splitmix64(0, 3)
    assert [int(v) for v in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_streams_are_seeded_and_distinct():
    a = synth.uniform(1, 1000)
    assert np.array_equal(a, synth.uniform(1, 1000))
    assert not np.array_equal(a, synth.uniform(2, 1000))
    assert np.all((a > 0) & (a < 1))


def test_normal_moments():
    n = synth.normal(3, 200000)
    assert abs(n.mean()) < 0.01 and abs(n.std() - 1.0) < 0.01
    # the tail is Gaussian: about 0.27% beyond 3 sigma
    assert 0.0020 < np.mean(np.abs(n) > 3.0) < 0.0034


def test_bf16_tensors_are_rounded_values_of_the_stream():
    g = synth.gaussian_bf16(4, (8, 16), std=2.0)
    v = synth.bf16_bits_to_f64(g)
    ref = 2.0 * synth.normal(4, 128).reshape(8, 16)
    assert np.all(np.abs(v - ref) <= 2.0 ** -8 * np.abs(ref))       # one BF16 rounding
    assert np.array_equal(synth.f64_to_bf16_bits(v), g)               # BF16 values round-trip


def test_stream_offsets_continue_the_stream():
    """A stream started at an (even) offset is the same stream's continuation, so
    tensors generated in chunks equal tensors generated at once."""
    full = synth.normal(5, 1000)
    assert np.array_equal(synth.normal(5, 300, offset=700), full[700:])
    assert np.array_equal(synth.uniform(5, 10, offset=20), synth.uniform(5, 30)[20:])
    old = synth._CHUNK
    try:
        synth._CHUNK = 64                       # force many chunks, one of them ragged
        chunked = synth.gaussian_bf16(6, (9, 50), std=0.5, mean=1.0)
    finally:
        synth._CHUNK = old
    assert np.array_equal(chunked, synth.f64_to_bf16_bits(1.0 + 0.5 * synth.normal(6, 450)).reshape(9, 50))
