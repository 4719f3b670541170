"""The index kernel's path for E4M3 keys and bf16 queries splits each query element x (scaled by a
power of two so that its head's largest magnitude lies in [2^7, 2^8)) into hi = E4M3(x) and
lo = E4M3(x - hi), and feeds both to 8-bit MMAs that sum into one accumulator.  Its claims,
checked here on every bf16 value of each range with the oracle's E4M3 codec (round to nearest,
saturating): hi + lo == x exactly for 2^-2 <= |x| < 2^8, and |hi + lo - x| <= 2^-10 below that
(2^-17 of the head's largest magnitude).  The GPU tests check the kernel itself."""
import numpy as np

import oracle


def bf16_values(e_lo: int, e_hi: int) -> np.ndarray:
    """Every normal bf16 value with exponent in [e_lo, e_hi], both signs (128 per binade)."""
    mant = 1.0 + np.arange(128) / 128.0
    v = np.concatenate([mant * 2.0 ** e for e in range(e_lo, e_hi + 1)])
    return np.concatenate([v, -v])


def split(x: np.ndarray):
    hi = oracle.e4m3_decode(oracle.e4m3_encode(x))
    lo = oracle.e4m3_decode(oracle.e4m3_encode(x - hi))
    return hi, lo


def test_split_is_exact_within_two_to_the_nine_of_the_maximum():
    x = bf16_values(-2, 7)
    hi, lo = split(x)
    assert np.array_equal(hi + lo, x)
    assert np.max(np.abs(hi)) <= 256.0 and np.max(np.abs(lo)) <= 8.0   # far from saturation


def test_split_error_below_that_is_under_two_to_the_minus_ten():
    x = np.concatenate([bf16_values(-40, -3), [0.0]])
    hi, lo = split(x)
    assert np.max(np.abs(hi + lo - x)) <= 2.0 ** -10


def test_split_needs_the_second_part():
    # hi alone keeps 4 significant bits: most bf16 values in range are not E4M3 values
    x = bf16_values(-2, 7)
    hi, _ = split(x)
    assert np.mean(hi != x) > 0.8
