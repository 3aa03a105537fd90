"""Double quantization of the block absmax with a mean offset and 8-bit floats.
Test infrastructure: see ``oracle/__init__``.

The pages fix double quantization as 8-bit codes in blocks of 256 with one
fp32 constant per block [P5 figure 4; P1 "Summary"; P4 "2. Double
quantization": the constants of the first quantization are quantized again].
The paper they cite (arXiv:2305.14314, P4 "What is QLoRA?") describes a
variant in which the constants are 8-bit floats and their mean is subtracted
first, to centre them around zero and use a symmetric format.  The pages do
not spell that variant out; the reading taken here, a second storage format
beside the unsigned linear one of ``oracle.quant``:

  mean   mu = fp32(T / nb), T the fp64 sum of the nb block absmax values
         c_b, added in a fixed order: each group of 256 (the last possibly
         partial) is summed by pairwise halving (``pairwise_sum``), then the
         group sums are summed the same way.  Every c_b is exact in fp64; the
         order makes the result reproducible.
  offset d_b = fp32(c_b - mu)
  scale  S_g = max |d_b| over the group (fp32)
  code   q_b = E4M3(fp32(fp32(d_b / S_g) * 448)), round to nearest, ties to
         even; 448 is the largest finite E4M3 value, so |.| <= 448 needs no
         saturation.  S_g == 0 gives q_b = 0.
  stored absmax_q[b] = q_b (the E4M3 bit pattern), group_scale[g] =
         fp32(S_g / 448) for g < ng, and group_scale[ng] = mu.
  decode c'_b = fp32(fp32(E4M3(q_b) * group_scale[g]) + mu)

E4M3 is the 8-bit float with 1 sign bit, 4 exponent bits (bias 7) and 3
mantissa bits; exponent field 0 holds the subnormals m/8 * 2^-6; the pattern
S.1111.111 is NaN and there are no infinities (largest finite 448).

The weights themselves are still quantized against the fp32 c_b (reading 5
of the two-stage scheme); only the stored constants change.  Storage: 8 bits
per block, 32 bits per group of 256 and 32 bits per tensor, the same
0.127 bit per weight as the linear format.
"""

import numpy as np

from . import codebooks, quant

GROUP = quant.GROUP
E4M3_MAX = 448.0


def e4m3_decode(code) -> np.ndarray:
    """fp32 value of each E4M3 bit pattern (NaN for S.1111.111)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return (s * mag).astype(np.float32)


_POS = e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)   # codes 0x00..0x7E, ascending


def e4m3_encode(x) -> np.ndarray:
    """Round fp32 values in [-448, 448] to the nearest E4M3 pattern, ties to
    the even pattern (even mantissa)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64).reshape(-1)
    if np.any(~np.isfinite(x)) or np.any(np.abs(x) > E4M3_MAX):
        raise ValueError("values must be finite and within +-448")
    a = np.abs(x)
    hi = np.searchsorted(_POS, a, side="left")          # first code with value >= a
    hi = np.minimum(hi, _POS.size - 1)
    lo = np.maximum(hi - 1, 0)
    dlo = a - _POS[lo]
    dhi = _POS[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0) & (hi != lo))
    code = np.where(a == _POS[hi], hi, np.where(pick_hi, hi, lo)).astype(np.int64)
    sign = np.where(np.signbit(x), 0x80, 0)
    return (code | sign).astype(np.uint8)


def pairwise_sum(values) -> float:
    """fp64 sum by repeated halving: adjacent pairs are added level by level,
    an odd last element carried to the next level unchanged."""
    v = [float(t) for t in np.asarray(values, dtype=np.float64).reshape(-1)]
    if not v:
        return 0.0
    while len(v) > 1:
        nxt = [v[i] + v[i + 1] for i in range(0, len(v) - 1, 2)]
        if len(v) % 2:
            nxt.append(v[-1])
        v = nxt
    return v[0]


def _pairwise_rows(a: np.ndarray) -> np.ndarray:
    """pairwise_sum of each row of a [rows x 2^j] fp64 array (vectorised)."""
    a = np.asarray(a, dtype=np.float64)
    while a.shape[1] > 1:
        a = a[:, 0::2] + a[:, 1::2]
    return a[:, 0]


def tensor_mean(absmax) -> np.float32:
    """mu: group sums by pairwise halving, then their pairwise sum, / nb."""
    c = np.asarray(absmax, dtype=np.float32).reshape(-1).astype(np.float64)
    nb = c.size
    full = nb // GROUP
    sums = list(_pairwise_rows(c[:full * GROUP].reshape(full, GROUP))) if full else []
    if nb % GROUP:
        sums.append(pairwise_sum(c[full * GROUP:]))
    return np.float32(pairwise_sum(sums) / nb)


def double_quantize_fp8(absmax):
    """absmax fp32 [nb] -> (q uint8 [nb] E4M3 patterns, group_scale fp32
    [ng + 1] = (fp32(S_g / 448) for each group, then mu))."""
    c = np.asarray(absmax, dtype=np.float32).reshape(-1)
    nb = c.size
    ng = (nb + GROUP - 1) // GROUP
    mu = tensor_mean(c)
    d = (c - mu).astype(np.float32)
    q = np.zeros(nb, dtype=np.uint8)
    gs = np.zeros(ng + 1, dtype=np.float32)
    for g in range(ng):
        dg = d[g * GROUP:(g + 1) * GROUP]
        sg = np.float32(np.max(np.abs(dg)))
        gs[g] = np.float32(sg / np.float32(E4M3_MAX))
        if sg > 0:
            ratio = (dg / sg).astype(np.float32)
            scaled = (ratio * np.float32(E4M3_MAX)).astype(np.float32)
            q[g * GROUP:(g + 1) * GROUP] = e4m3_encode(scaled)
    gs[ng] = mu
    return q, gs


def absmax_dequant_fp8(q, group_scale) -> np.ndarray:
    """c'_b = fp32(fp32(E4M3(q_b) * group_scale[g]) + mu)."""
    q = np.asarray(q, dtype=np.uint8).reshape(-1)
    gs = np.asarray(group_scale, dtype=np.float32).reshape(-1)
    mu = gs[-1]
    g = np.arange(q.size) // GROUP
    prod = (e4m3_decode(q) * gs[g]).astype(np.float32)
    return (prod + mu).astype(np.float32)


def quantize(w_flat, codebook: str = "nf4"):
    """Blockwise quantization with this double quantization: (packed codes,
    q [nb], group_scale [ng + 1], absmax [nb]).  The codes are those of
    ``quant.quantize_nf4_dq`` (they depend on the fp32 absmax only)."""
    c = quant.block_absmax(w_flat)
    codes = quant.nf4_codes(w_flat, c, codebook)
    q, gs = double_quantize_fp8(c)
    return quant.pack_codes(codes), q, gs, c


def dequant_bf16_bits(packed, q, group_scale, codebook: str = "nf4") -> np.ndarray:
    """W^ = bf16_rne(fp32(L[code] * c')) as bit patterns, flat row-major."""
    codes = quant.unpack_codes(packed)
    cprime = absmax_dequant_fp8(q, group_scale)
    lv = codebooks.levels_f32(codebook)
    vals = (lv[codes].reshape(-1, quant.BLOCK) * cprime.reshape(-1, 1)).astype(np.float32)
    return quant.bf16_rne_bits(vals.reshape(-1))


def dequant_bf16_values(packed, q, group_scale, codebook: str = "nf4") -> np.ndarray:
    """W^ as the fp64 values of its bf16 entries."""
    return quant.bf16_bits_to_f32(dequant_bf16_bits(packed, q, group_scale, codebook)).astype(np.float64)
