"""The precision of the bf16 hi/lo split the tensor-core and prefill kernels
feed to the tensor cores (CPU).

A float value x enters a bf16 product as two parts, hi = bf16(x) and
lo = bf16(x - hi), both rounded to nearest even. bf16 keeps 8 significant
bits, so |x - hi| <= 2^-8 |x| and |x - hi - lo| <= 2^-8 |x - hi| <= 2^-16 |x|:
the pair carries about 16 bits. A product of two split values is formed as
hi_x hi_y + hi_x lo_y + lo_x hi_y, each bf16 product exact in the fp32
accumulator; the dropped lo_x lo_y is at most 2^-16 of |x y|. These are the
bounds the kernels' precision rests on; they are checked here in exact
float64 arithmetic with the oracle's bf16 rounding (pinned separately).
"""
import numpy as np

from oracle.gdr_oracle import bf16_round


def split(x):
    hi = bf16_round(x)
    lo = bf16_round(x - hi)
    return hi, lo


def values(rng, n):
    mag = 2.0 ** rng.uniform(-60, 60, n)
    return rng.choice([-1.0, 1.0], n) * mag * rng.uniform(1.0, 2.0, n)


def test_hi_lo_carries_sixteen_bits():
    rng = np.random.default_rng(1)
    x = values(rng, 200000).astype(np.float32).astype(np.float64)  # fp32 inputs
    hi, lo = split(x)
    assert np.all(np.abs(x - hi) <= 2.0 ** -8 * np.abs(x))
    assert np.all(np.abs(x - hi - lo) <= 2.0 ** -16 * np.abs(x))


def test_split_product_drops_only_the_lo_lo_term():
    rng = np.random.default_rng(2)
    x = values(rng, 200000).astype(np.float32).astype(np.float64)
    y = values(rng, 200000).astype(np.float32).astype(np.float64)
    hx, lx = split(x)
    hy, ly = split(y)
    approx = hx * hy + hx * ly + lx * hy  # each term exact; the sum as the accumulator forms it
    exact = x * y
    # the two representation errors (2^-16 each) and the dropped lo lo term (2^-16)
    assert np.all(np.abs(approx - exact) <= 3.01 * 2.0 ** -16 * np.abs(exact))
    assert np.all(np.abs(lx * ly) <= 2.0 ** -16 * np.abs(exact) * 1.0001)


def test_one_part_alone_is_not_enough():
    """bf16 alone (hi only) is off by up to 2^-8: the lo part is what brings a
    product to the 2^-7 relative parity bar with margin over many terms."""
    rng = np.random.default_rng(3)
    x = values(rng, 200000).astype(np.float32).astype(np.float64)
    hi, _ = split(x)
    worst = np.max(np.abs(x - hi) / np.abs(x))
    assert worst > 2.0 ** -9  # the hi part alone really is an 8-bit value
