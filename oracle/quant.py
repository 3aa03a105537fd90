"""Blockwise NF4 quantization with double-quantized absmax.  Test infrastructure.

Storage format (the readings are listed where the pages are silent):

  W is fp32 [n x k], row-major, k a multiple of 64.  Flattened row-major it is
  cut into nb = n*k/64 blocks of 64 consecutive weights
  [P5 figure 4: "each block of 64 weights carries a 32-bit scaling constant";
   P3 "Worked example": block size 64 in fp32].

  a1  c_b = max |w| over block b (fp32, exact).
  a2  x = fp32(w / c_b) (IEEE round-to-nearest division); code = #{i : x > T_i}
      with T the 15 fp32 midpoints of ``oracle.nf4``; c_b == 0 gives code 7
      (the zero level) without dividing.  Codes are packed two per byte
      [P3 "Worked example": 0.5 byte per parameter]; the pages do not give the
      nibble order, and the reading taken is: byte j = (code[2j] << 4) |
      code[2j+1], the even element in the high nibble.
  a3  Double quantization [P1 "Summary": scales quantized to 8-bit integers;
      P5 figure 4: "8-bit, blocks of 256", 0.127 bit per parameter].  The
      pages disagree on "a single global scale" (P1) versus blocks of 256
      (P5); 0.127 = 8/64 + 32/(64*256) fixes one fp32 constant per 256
      absmax values.  Reading taken: unsigned linear 8-bit codes (absmax is
      never negative), group g = absmax values [256g, 256g+256), the last
      group possibly partial:
          S_g = max c over the group (fp32)
          q   = rint_half_even(fp32(fp32(c / S_g) * 255))  -> uint8
          S_g == 0 gives q = 0.
  a4  Dequantize [P2 "Storage precision is not calculation precision";
      P5 figure 2: dequantized block by block to bf16]:
          t_g = fp32(S_g / 255)
          c'  = fp32(float(q) * t_g)
          W^  = bf16_rne(fp32(L[code] * c'))
      Weights are quantized against the fp32 c_b, then the constants are
      compressed (the two-stage reading of P1 and P5).

The same functions take a ``codebook`` name (``oracle.codebooks``): the FP4
and INT4 baselines change only the sixteen levels and their midpoints.

Inputs must be finite; that precondition is checked here only.
"""

import numpy as np

from . import codebooks, nf4

BLOCK = 64
GROUP = 256


# ---------------------------------------------------------------------------
# bf16 round-to-nearest-even by bit manipulation
# ---------------------------------------------------------------------------

def bf16_rne_bits(x) -> np.ndarray:
    """fp32 -> bf16 bit pattern (uint16), round to nearest, ties to even.

    Finite inputs only.  The top 16 bits of the fp32 pattern are kept after
    adding 0x7FFF plus the lowest kept bit (so an exact half rounds to the
    even neighbour)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """bf16 bit pattern (uint16) -> the exactly equal fp32 value."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---------------------------------------------------------------------------
# a1 - a3: quantize
# ---------------------------------------------------------------------------

def block_absmax(w_flat: np.ndarray) -> np.ndarray:
    """a1: fp32 absmax of each block of 64 consecutive weights."""
    w = np.asarray(w_flat, dtype=np.float32).reshape(-1)
    if w.size % BLOCK:
        raise ValueError("length must be a multiple of 64")
    if not np.all(np.isfinite(w)):
        raise ValueError("weights must be finite")
    return np.max(np.abs(w.reshape(-1, BLOCK)), axis=1).astype(np.float32)


def nf4_codes(w_flat: np.ndarray, absmax: np.ndarray, codebook: str = "nf4") -> np.ndarray:
    """a2: one code (0..15, uint8) per weight, from the fp32 block absmax; the
    decision midpoints are those of ``codebook`` (NF4 unless a baseline of
    ``oracle.codebooks`` is named)."""
    w = np.asarray(w_flat, dtype=np.float32).reshape(-1, BLOCK)
    c = np.asarray(absmax, dtype=np.float32).reshape(-1, 1)
    safe = np.where(c > 0, c, np.float32(1.0)).astype(np.float32)
    x = (w / safe).astype(np.float32)          # IEEE fp32 division
    x = np.where(c > 0, x, np.float32(0.0)).astype(np.float32)
    t = codebooks.midpoints_f32(codebook)
    codes = np.zeros(x.shape, dtype=np.uint8)
    for ti in t:                                # count of midpoints below x
        codes += (x > ti).astype(np.uint8)
    return codes.reshape(-1)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte, the even element in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    if c.size % 2:
        raise ValueError("even number of codes required")
    return ((c[0::2] << np.uint8(4)) | c[1::2]).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p >> np.uint8(4)
    out[1::2] = p & np.uint8(0x0F)
    return out


def double_quantize(absmax: np.ndarray):
    """a3: absmax fp32 [nb] -> (q uint8 [nb], S fp32 [ceil(nb/256)])."""
    c = np.asarray(absmax, dtype=np.float32).reshape(-1)
    nb = c.size
    ng = (nb + GROUP - 1) // GROUP
    q = np.zeros(nb, dtype=np.uint8)
    S = np.zeros(ng, dtype=np.float32)
    for g in range(ng):
        cg = c[g * GROUP:(g + 1) * GROUP]
        sg = np.float32(np.max(cg))
        S[g] = sg
        if sg > 0:
            ratio = (cg / sg).astype(np.float32)
            scaled = (ratio * np.float32(255.0)).astype(np.float32)
            q[g * GROUP:(g + 1) * GROUP] = np.rint(scaled).astype(np.uint8)
    return q, S


def quantize_nf4_dq(w_flat: np.ndarray, codebook: str = "nf4"):
    """a1-a3 for a flat row-major weight whose length is a multiple of 64.

    Returns (packed codes uint8 [len/2], q uint8 [nb], S fp32 [ng],
    absmax fp32 [nb]).  Groups are counted from the start of ``w_flat``, so a
    slice that starts on a 16384-element boundary of a larger weight gives
    exactly that weight's groups."""
    c = block_absmax(w_flat)
    codes = nf4_codes(w_flat, c, codebook)
    q, S = double_quantize(c)
    return pack_codes(codes), q, S, c


# ---------------------------------------------------------------------------
# a4: dequantize
# ---------------------------------------------------------------------------

def absmax_dequant(q: np.ndarray, S: np.ndarray) -> np.ndarray:
    """c' = fp32(float(q) * fp32(S_g / 255)) for every block."""
    q = np.asarray(q, dtype=np.uint8).reshape(-1)
    S = np.asarray(S, dtype=np.float32).reshape(-1)
    t = (S / np.float32(255.0)).astype(np.float32)
    g = np.arange(q.size) // GROUP
    return (q.astype(np.float32) * t[g]).astype(np.float32)


def dequant_f32(packed: np.ndarray, q: np.ndarray, S: np.ndarray, codebook: str = "nf4") -> np.ndarray:
    """fp32(L[code] * c') for every weight, before the bf16 cast."""
    codes = unpack_codes(packed)
    cprime = absmax_dequant(q, S)
    lv = codebooks.levels_f32(codebook)
    vals = lv[codes].reshape(-1, BLOCK)
    return (vals * cprime.reshape(-1, 1)).astype(np.float32).reshape(-1)


def dequant_bf16_bits(packed: np.ndarray, q: np.ndarray, S: np.ndarray, codebook: str = "nf4") -> np.ndarray:
    """a4: W^ as bf16 bit patterns (uint16), flat row-major."""
    return bf16_rne_bits(dequant_f32(packed, q, S, codebook))


def dequant_bf16_values(packed: np.ndarray, q: np.ndarray, S: np.ndarray, codebook: str = "nf4") -> np.ndarray:
    """a4: W^ as the fp64 values of its bf16 entries (exact)."""
    return bf16_bits_to_f32(dequant_bf16_bits(packed, q, S, codebook)).astype(np.float64)
