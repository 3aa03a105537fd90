"""NF4 (4-bit NormalFloat) codebook.  Test infrastructure: see ``oracle/__init__``.

What the pages fix:
  [P3 "The idea"]  16 levels spaced at the quantiles of a standard normal.
  [P4 "The three ideas behind QLoRA", 1. NF4]  levels at normal quantiles, so
      each level is used about equally often.
  [P5 figure 3 "NF4 - bins shaped like the weights"]  equal mass per bin,
      dense near zero, sparse in the tails.
  [P5 figure 4]  weights are scaled per block of 64 by an absmax constant, so
      the normalised weight lies in [-1, 1].

What the pages leave open, and the reading taken here:
  Sixteen symmetric quantiles can hold neither an exact zero nor the finite
  endpoints +-1 that an absmax-normalised block needs (the absmax element
  itself maps to +-1, and zero weights must stay zero).  The construction used
  is the asymmetric one of the paper the pages cite (arXiv:2305.14314, named on
  [P4 "What is QLoRA?"]):

  * a tail probability o = 1 - (1/32 + 1/30)/2, the mean of the last bin
    centre for 16 and for 15 equal-mass bins;
  * 8 positive levels Phi^-1(p) for p equally spaced from o down to 1/2,
    9 points with the point 1/2 dropped;
  * 7 negative levels -Phi^-1(p) for p equally spaced from o down to 1/2,
    8 points with the point 1/2 dropped;
  * the level 0;
  * all divided by Phi^-1(o) so that the extremes are exactly -1 and +1.

  Equal normal mass per bin then holds within each half: the probability
  spacing is (o - 1/2)/8 above zero and (o - 1/2)/7 below it.

The levels are computed in double with ``statistics.NormalDist.inv_cdf`` and
rounded once to fp32.  Index 0 = -1, index 7 = 0, index 15 = +1.
"""

from statistics import NormalDist

import numpy as np

# Tail probability of the extreme level (the reading described above).
TAIL_P = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)

N_POS = 8  # positive levels
N_NEG = 7  # negative levels


def levels_f64() -> np.ndarray:
    """The 16 NF4 levels in double, ascending, before fp32 rounding."""
    phi_inv = NormalDist().inv_cdf
    o = TAIL_P
    pos = [phi_inv(o - i * (o - 0.5) / N_POS) for i in range(N_POS)]
    neg = [-phi_inv(o - i * (o - 0.5) / N_NEG) for i in range(N_NEG)]
    top = phi_inv(o)
    vals = sorted(neg + [0.0] + pos)
    return np.array([v / top for v in vals], dtype=np.float64)


def levels_f32() -> np.ndarray:
    """The 16 NF4 levels rounded once to fp32 (the stored codebook)."""
    return levels_f64().astype(np.float32)


def midpoints_f32() -> np.ndarray:
    """Decision thresholds T_i = fp32(fp32(L_i + L_{i+1}) * 0.5), i = 0..14.

    A normalised weight x gets code #{i : x > T_i}: the nearest level, with a
    value exactly on a midpoint going to the lower index (the pages give no
    tie rule; this is the reading taken).
    """
    lv = levels_f32()
    s = (lv[:-1] + lv[1:]).astype(np.float32)
    return (s * np.float32(0.5)).astype(np.float32)
