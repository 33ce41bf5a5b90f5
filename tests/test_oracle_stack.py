"""Pins of the oracle's stack wiring (bf16 rounding and fp32 summation order)."""

import numpy as np

from oracle import stack


def test_next_input_rounds_to_nearest_even():
    # 1 + 2^-8 lies halfway between the bf16 neighbours 1 and 1 + 2^-7: ties go to the even one (1).
    assert stack.next_input(np.float32(1.0), np.float32(2.0 ** -8)) == np.float32(1.0)
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    assert stack.next_input(np.float32(1.0 + 2.0 ** -7), np.float32(2.0 ** -8)) == np.float32(1.0 + 2.0 ** -6)
    # Just above the halfway point rounds up; truncation would give 1.
    assert stack.next_input(np.float32(1.0), np.float32(2.0 ** -8 + 2.0 ** -12)) == np.float32(1.0 + 2.0 ** -7)
    # Exact sums stay exact, signs included.
    assert stack.next_input(np.float32(-3.0), np.float32(1.0)) == np.float32(-2.0)


def test_grad_sum_is_sequential_fp32_in_the_stated_order():
    big = np.float32(2.0 ** 24)
    dX = {"q": big, "k": np.float32(1.0), "v": -big, "o": np.float32(0.0), "gate": np.float32(0.0),
          "up": np.float32(0.0)}
    # fp32: (2^24 + 1) rounds to 2^24 (tie to even), then cancels: 0, not the exact sum 1.
    assert stack.grad_sum(dX) == np.float32(0.0)
    # Another order of the same terms (k first) keeps the 1.
    dX2 = dict(dX, q=np.float32(1.0), k=big)
    assert stack.grad_sum(dX2) == np.float32(0.0)
    dX3 = dict(dX, v=np.float32(1.0), k=-big)
    assert stack.grad_sum(dX3) == np.float32(1.0)


def test_grad_sum_of_bf16_values_equals_fp64_sum_when_exact():
    g = np.random.default_rng(5)
    vals = {n: (g.integers(-64, 64, size=(3, 5)) / 8.0).astype(np.float32) for n in stack.READS_H}
    exact = sum(v.astype(np.float64) for v in vals.values())
    np.testing.assert_array_equal(stack.grad_sum(vals), exact.astype(np.float32))
