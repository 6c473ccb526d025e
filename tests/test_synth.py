"""The shared input generator: determinism and the structure the configs ask
for (no NaN codes, distinct needles, scale ranges).  No method arithmetic."""
import numpy as np

import synth


def test_streams_are_deterministic_and_distinct():
    a = synth.hashes(synth.stream_key(1, 2, 3, 4), 0, 100)
    b = synth.hashes(synth.stream_key(1, 2, 3, 4), 50, 50)
    assert np.array_equal(a[50:], b)
    c = synth.hashes(synth.stream_key(1, 2, 3, 5), 0, 100)
    assert not np.array_equal(a, c)
    # SplitMix64 reference value (seed 0 state after one step, Vigna's splitmix64.c)
    assert int(synth.mix64(np.uint64(0x9E3779B97F4A7C15))) == 0xE220A8397B1DCDAF


def test_mxfp4_rows_slices_agree():
    full = synth.mxfp4_rows(5, 1, 2, 7, 0, 0, 64, 512, rownorm_key=synth.stream_key(5, synth.T_ROWNORM, 7))
    part = synth.mxfp4_rows(5, 1, 2, 7, 0, 40, 10, 512, rownorm_key=synth.stream_key(5, synth.T_ROWNORM, 7))
    assert np.array_equal(full[0][40:50], part[0]) and np.array_equal(full[1][40:50], part[1])
    assert full[1].min() >= 123 and full[1].max() <= 129


def test_e4m3_rows_have_no_nan():
    w = synth.e4m3_rows(3, synth.T_WIN, 0, 0, 0, 2048)
    assert not np.any((w & 0x7F) == 0x7F)
    assert ((w >> 3) & 15).min() >= 9


def test_needles_distinct_and_in_range():
    for L in [300, 8192, 1 << 20]:
        p = synth.needle_positions(9, 1, 0, L, 256)
        assert len(np.unique(p)) == len(p) and p.min() >= 0 and p.max() < max(L - 128, 1)


def test_normal_like_values():
    v = synth.bf16_bits_to_f32(synth.normal_bf16(1, synth.T_Q, 0, 0, 100000))
    assert abs(v.mean()) < 0.02 and abs(v.std() - 1) < 0.02
    w = synth.head_weights(1, 0, 0, 1000)
    assert w.min() >= 0.5 and w.max() < 1.5


def test_bf16_rounding_is_rne():
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20], np.float32)
    got = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))
    assert got.tolist() == [1.0, 1.0 + 2 ** -6, -1.0, 1.0 + 2 ** -7]
