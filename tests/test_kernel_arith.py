"""CPU checks of arithmetic identities the CUDA kernels rely on (no GPU).

The quantizer divides a block's max |x| (a BF16 value) by 6 with three
operations -- q0 = RN(a * RN(1/6)), r = RN(a - 6 q0) by FMA, q = RN(r * RN(1/6)
+ q0) -- instead of an IEEE division.  This must equal the correctly rounded
binary32 quotient for every non-negative finite BF16 input, or the block
scales would differ from the definition.  Checked here exhaustively with exact
rational arithmetic.
"""
from fractions import Fraction

import numpy as np


def _rn32(x: Fraction) -> float:
    lo = np.float32(float(x))
    cands = [np.nextafter(lo, np.float32(-np.inf)), lo, np.nextafter(lo, np.float32(np.inf))]
    return float(min(cands, key=lambda c: (abs(Fraction(float(c)) - x),
                                           int(np.float32(c).view(np.uint32)) & 1)))


def test_div6_by_fma_is_correctly_rounded_for_all_bf16():
    bits = np.arange(0, 0x7F80, dtype=np.uint32) << 16          # every non-negative finite bf16
    a = bits.view(np.float32)
    ref = a / np.float32(6.0)                                     # IEEE binary32 division
    inv6 = np.float32(1.0) / np.float32(6.0)
    q0 = a * inv6                                                 # RN(a * RN(1/6))
    # r = RN(a - 6 q0): 6 q0 and the difference are exact in binary64
    r = (a.astype(np.float64) - 6.0 * q0.astype(np.float64)).astype(np.float32)
    # q = RN(r * inv6 + q0): exact rational, then one rounding
    inv6f = Fraction(float(inv6))
    bad = [i for i in range(a.size)
           if _rn32(Fraction(float(r[i])) * inv6f + Fraction(float(q0[i]))) != float(ref[i])]
    assert not bad, bad[:5]
