"""The coupling's stream format, checked on the CPU.

The device path carries the reversible coupling's two streams as fp32 values
that are multiples of 2^-16 and below 256 in magnitude, so that every
coupling add and subtract is exact and the inverse returns the forward's
inputs bit for bit at any depth. These tests pin the arithmetic facts that
claim rests on, in numpy fp32, independently of the GPU:

* the sum and difference of two grid values below 256 are exact in fp32, so
  (a + b) - b == a;
* without the grid the same round trip loses bits (why the format exists);
* every bf16 value of magnitude 2^-9 or more already lies on the grid;
* a smaller bf16 value, put on the grid (half to even), stays a bf16 value
  and moves by at most 2^-17.
"""
import numpy as np

from tests.gpu_util import stream_grid

GRID = 2.0 ** -16
LIMIT = 256.0


def _grid_values(rng, n, bound):
    k = rng.integers(-int(bound / GRID) + 1, int(bound / GRID), size=n, dtype=np.int64)
    return (k.astype(np.float64) * GRID)


def test_grid_adds_and_subtracts_are_exact_in_fp32():
    rng = np.random.default_rng(0)
    a = _grid_values(rng, 200_000, LIMIT / 2)
    b = _grid_values(rng, 200_000, LIMIT / 2)
    a32, b32 = a.astype(np.float32), b.astype(np.float32)
    assert np.array_equal(a32.astype(np.float64), a) and np.array_equal(b32.astype(np.float64), b)
    s32 = a32 + b32
    assert np.array_equal(s32.astype(np.float64), a + b)          # exact sum
    assert np.array_equal(s32 - b32, a32)                         # exact inverse
    d32 = a32 - b32
    assert np.array_equal(d32 + b32, a32)


def test_round_trip_loses_bits_off_the_grid():
    rng = np.random.default_rng(1)
    a = rng.standard_normal(200_000).astype(np.float32) * np.float32(1e-3)
    b = rng.standard_normal(200_000).astype(np.float32)
    assert not np.array_equal((a + b) - b, a)


def _all_bf16_finite():
    bits = np.arange(1 << 16, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    return v[np.isfinite(v)].astype(np.float64)


def _is_bf16(v):
    f = np.asarray(v, np.float32)
    return np.array_equal(((f.view(np.uint32) >> 16) << 16).view(np.float32), f)


def test_bf16_values_from_two_to_the_minus_nine_lie_on_the_grid():
    v = _all_bf16_finite()
    big = v[(np.abs(v) >= 2.0 ** -9) & (np.abs(v) < LIMIT)]
    assert big.size == 2 * 17 * 128          # both signs, 17 binades of 128 values
    assert np.array_equal(stream_grid(big), big)


def test_small_bf16_values_move_by_at_most_half_a_grid_step_and_stay_bf16():
    v = _all_bf16_finite()
    small = v[np.abs(v) < 2.0 ** -9]
    g = stream_grid(small)
    assert np.max(np.abs(g - small)) <= 2.0 ** -17
    assert _is_bf16(g)
    assert np.any(g != small)          # the grid does move some of them


def test_grid_rounding_is_half_to_even():
    half = 2.0 ** -17
    assert stream_grid(np.array([half]))[0] == 0.0
    assert stream_grid(np.array([3 * half]))[0] == 2 * GRID
    assert stream_grid(np.array([-half]))[0] == 0.0
