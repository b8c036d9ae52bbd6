"""Seeded input generators (no GPU)."""
import numpy as np
import pytest

from exact_io_aware_92_b200 import workloads as wl


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa wins (1.0);
    # 1 + 3*2^-8 ties between 1 + 2^-7 and 1 + 2^-6: even wins (1 + 2^-6).
    x = np.array([1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-8 + 2**-20, -2.5, 0.0], np.float32)
    b = wl.round_to_bf16_bits(x)
    np.testing.assert_array_equal(wl.bf16_bits_to_f32(b),
                                  np.array([1.0, 1.0 + 2**-6, 1.0 + 2**-7, -2.5, 0.0], np.float32))


def test_small_and_large_rounding_paths_agree():
    x = np.random.default_rng(0).standard_normal(3 << 20, dtype=np.float32)
    big = wl.round_to_bf16_bits(x)
    small = np.concatenate([wl.round_to_bf16_bits(c) for c in np.split(x, 6)])
    np.testing.assert_array_equal(big, small)


def test_rejects_non_finite():
    with pytest.raises(ValueError):
        wl.round_to_bf16_bits(np.array([1.0, np.inf], np.float32))


def test_draw_is_seeded_and_shaped():
    a = wl.draw(2, 4, 2, 33, 64, seed=7, seqlen_range=(3, 9))
    b = wl.draw(2, 4, 2, 33, 64, seed=7, seqlen_range=(3, 9))
    assert a.q_bits.shape == (2, 4, 33, 64) and a.k_bits.shape == (2, 2, 33, 64)
    assert np.array_equal(a.q_bits, b.q_bits) and np.array_equal(a.seqlens, b.seqlens)
    assert np.all((a.seqlens >= 3) & (a.seqlens <= 9))
    # K scaling by a power of two is exact
    c = wl.draw(1, 1, 1, 8, 64, seed=3, k_scale=2.0)
    d = wl.draw(1, 1, 1, 8, 64, seed=3)
    np.testing.assert_array_equal(c.k_f32, 2.0 * d.k_f32)


def test_flop_counts():
    assert wl.flops(wl.LLAMA_GQA) == pytest.approx(1.0995e12, rel=1e-4)
    assert wl.flops(wl.GPT2) == pytest.approx(1.288e10, rel=1e-3)
    assert wl.flops(wl.TINY) == 4 * 1 * 2 * 256 * 256 * 64
    assert wl.flops(wl.LONG) == pytest.approx(4.398e12, rel=1e-3)


def test_sample_rows_sorted_unique():
    r = wl.sample_rows(wl.LONG)
    assert r.shape == (16, 256)
    assert all(len(set(row)) == 256 and np.all(np.diff(row) > 0) for row in r)
