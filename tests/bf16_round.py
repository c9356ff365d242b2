"""Round-to-nearest-even to bf16 of fp64 values, written out from the format's definition
(8 significant bits, so neighbouring bf16 values of x in [2^(e-1), 2^e) are 2^(e-8) apart),
for tests that check a bf16 output is a correct rounding of a reference value."""
import numpy as np


def bf16_neighbours(x):
    """The two bf16 values around each fp64 value (lower <= x <= upper), the one nearest to
    it (ties to the even significand), and the midpoint between the neighbours."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(np.where(x == 0, 1.0, np.abs(x)))  # |x| = m 2^e, m in [0.5, 1)
    ulp = np.ldexp(1.0, e - 8)                           # 8 significant bits
    lo = np.floor(np.abs(x) / ulp) * ulp
    hi = lo + ulp
    mid = lo + ulp / 2
    odd = (np.floor(np.abs(x) / ulp) % 2) == 1
    near = np.where(np.abs(x) < mid, lo, np.where(np.abs(x) > mid, hi, np.where(odd, hi, lo)))
    sgn = np.sign(x)
    return sgn * near, sgn * np.where(near == lo, hi, lo), sgn * mid
