"""4-bit codebooks for the blockwise quantizer: NF4 and two baselines.
Test infrastructure: see ``oracle/__init__``.

What the pages fix:
  [P4 "The three ideas behind QLoRA", 1. 4-bit NormalFloat]  NF4 beats the
      standard 4-bit integer and float formats on normally distributed data.
  [P5 figure 3 "NF4 - bins shaped like the weights"]  INT4 and FP4 spread
      their sixteen values evenly (uniform bins) and so waste levels where
      weights rarely fall; NF4 is worth about a point of MMLU over FP4.

The pages name the two baselines but do not define them.  Readings taken:

* ``fp4``: the standard 4-bit float with 1 sign, 2 exponent and 1 mantissa
  bits (e2m1, exponent bias 1, no infinities or NaN).  Its eight magnitudes
  are 0, 0.5, 1, 1.5, 2, 3, 4, 6; divided by the largest, 6, so that an
  absmax-normalised block spans [-1, 1] like NF4's.  The sixteen codes in
  ascending order: code 7 = -0 and code 8 = +0, code 0 = -1, code 15 = +1.
  A normalised weight of exactly 0 takes code 7 (the lower index of a tie,
  as for every midpoint), whose level is -0.
* ``int4``: symmetric absmax integer quantization, levels i/7 for
  i = -7..7 at codes 0..14; code 15 repeats +1 and is never produced
  (its midpoint with code 14 is 1, and |w / absmax| <= 1).

Both keep NF4's block of 64, its double-quantized constants and its decision
rule (code = #{i : x > T_i}, T_i = fp32(fp32(L_i + L_{i+1}) * 0.5)), so the
comparison isolates the choice of the sixteen values.  Levels are exact
rationals rounded once to fp32.
"""

from fractions import Fraction

import numpy as np

from . import nf4

NAMES = ("nf4", "fp4", "int4")


def fp4_magnitudes() -> list:
    """The eight e2m1 magnitudes, ascending, as exact fractions."""
    return [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4),
            Fraction(6)]


def levels_exact(name: str) -> list:
    """The 16 levels of a baseline codebook as exact fractions, ascending."""
    if name == "fp4":
        mags = [m / 6 for m in fp4_magnitudes()]
        return [-m for m in reversed(mags)] + mags          # -1 .. -0, +0 .. 1
    if name == "int4":
        return [Fraction(i, 7) for i in range(-7, 8)] + [Fraction(1)]
    raise ValueError(name)


def levels_f32(name: str) -> np.ndarray:
    """The 16 levels of ``name`` rounded once to fp32 (code order)."""
    if name == "nf4":
        return nf4.levels_f32()
    lv = np.array([float(v) for v in levels_exact(name)], dtype=np.float64).astype(np.float32)
    if name == "fp4":
        lv[7] = np.float32(-0.0)                           # the negative zero of code 7
    return lv


def midpoints_f32(name: str) -> np.ndarray:
    """T_i = fp32(fp32(L_i + L_{i+1}) * 0.5), i = 0..14, as for NF4."""
    if name == "nf4":
        return nf4.midpoints_f32()
    lv = levels_f32(name)
    s = (lv[:-1] + lv[1:]).astype(np.float32)
    return (s * np.float32(0.5)).astype(np.float32)
