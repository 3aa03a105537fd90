"""LoRA dropout on the adapter input, with a counter-based random mask.
Test infrastructure: see ``oracle/__init__``.

What the pages fix:
  [P3 "In code"]  ``LoraConfig(r=16, lora_alpha=32, lora_dropout=0.05, ...)``:
      the adapter branch is trained with dropout probability 0.05.

What they leave open, and the readings taken:
* Where dropout acts.  As in the LoRA configuration the pages use: on the
  adapter's input only.  The frozen product sees X, the adapter sees
  Xd = D * X / (1 - p) (inverted dropout, D the keep mask):
      Y  = X . W^T + s . (Xd . A^T) . B^T
      dX = dY . W^ + D * (s . (dY . B) . A) / (1 - p)
      dA = s . (dY . B)^T . Xd          dB = s . dY^T . (Xd . A^T)
* The random numbers.  Philox4x64 with 10 rounds (Salmon, Moraes, Dror and
  Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011): a counter
  of four 64-bit words is scrambled by ten rounds of two 64 x 64 -> 128-bit
  multiplications under a key of two 64-bit words that is bumped by two
  Weyl constants between rounds.  Element e of X (row-major flat index)
  draws the 16-bit lane e mod 16 of the output for the counter
  (e div 16, offset, 0, 0) under the key (seed, 0); it is kept when that
  16-bit value is >= round(p * 65536) (p resolved to 1/65536).  ``offset``
  separates the masks of different calls (step, layer); the backward pass
  regenerates the forward's mask from the same (seed, offset).
* The arithmetic of Xd.  1 - p and its reciprocal are rounded to fp32, and a
  kept element becomes bf16_rne(fp32(x * fp32(1 / fp32(1 - p)))), the bf16
  tensor the adapter multiplies; a dropped element becomes +0.
"""

import numpy as np

from . import quant

MASK64 = (1 << 64) - 1
# Philox4x64 round multipliers and key increments (the published constants).
PHILOX_M0 = 0xD2E7470EE14C6C93
PHILOX_M1 = 0xCA5A826395121157
PHILOX_W0 = 0x9E3779B97F4A7C15
PHILOX_W1 = 0xBB67AE8584CAA73B


def philox4x64_10(counter, key) -> list:
    """Ten Philox4x64 rounds of the 4-word counter under the 2-word key."""
    x0, x1, x2, x3 = (int(v) & MASK64 for v in counter)
    k0, k1 = (int(v) & MASK64 for v in key)
    for _ in range(10):
        p0 = PHILOX_M0 * x0
        p1 = PHILOX_M1 * x2
        x0, x1, x2, x3 = (((p1 >> 64) ^ x1 ^ k0) & MASK64, p1 & MASK64,
                          ((p0 >> 64) ^ x3 ^ k1) & MASK64, p0 & MASK64)
        k0 = (k0 + PHILOX_W0) & MASK64
        k1 = (k1 + PHILOX_W1) & MASK64
    return [x0, x1, x2, x3]


def threshold(p: float) -> int:
    """round(p * 65536) for the keep test u16 >= threshold (p in [0, 1))."""
    p32 = float(np.float32(p))
    if not 0.0 <= p32 < 1.0:
        raise ValueError("dropout probability must lie in [0, 1)")
    return int(np.rint(p32 * 65536.0))


def uniforms16(numel: int, seed: int, offset: int) -> np.ndarray:
    """The 16-bit uniform of every flat element index 0 .. numel-1."""
    out = np.empty(numel, dtype=np.uint32)
    for blk in range((numel + 15) // 16):
        words = philox4x64_10((blk, offset, 0, 0), (seed, 0))
        for lane in range(min(16, numel - 16 * blk)):
            out[16 * blk + lane] = (words[lane >> 2] >> (16 * (lane & 3))) & 0xFFFF
    return out


def keep_mask(m: int, k: int, p: float, seed: int, offset: int) -> np.ndarray:
    """D [m x k]: True where the element of the adapter input is kept."""
    return (uniforms16(m * k, seed, offset) >= threshold(p)).reshape(m, k)


def keep_scale(p: float) -> np.float32:
    """fp32(1 / fp32(1 - p))."""
    return np.float32(np.float32(1.0) / np.float32(np.float32(1.0) - np.float32(p)))


def dropout_bf16_bits(X: np.ndarray, keep: np.ndarray, p: float) -> np.ndarray:
    """Xd as bf16 bit patterns: bf16_rne(fp32(x * keep_scale)) where kept, +0
    elsewhere.  X holds the fp32 values of a bf16 tensor."""
    x = np.asarray(X, dtype=np.float32)
    scaled = (x * keep_scale(p)).astype(np.float32)
    bits = quant.bf16_rne_bits(scaled).reshape(x.shape)
    return np.where(keep, bits, np.uint16(0)).astype(np.uint16)


def dropout_values(X: np.ndarray, keep: np.ndarray, p: float) -> np.ndarray:
    """Xd as the fp64 values of its bf16 entries."""
    return quant.bf16_bits_to_f32(dropout_bf16_bits(X, keep, p)).astype(np.float64)


def fwd(X, W_hat, A, B, s, Xd) -> np.ndarray:
    """Y = X . W^T + s . (Xd . A^T) . B^T (fp64)."""
    X, W_hat, A, B, Xd = (np.asarray(a, dtype=np.float64) for a in (X, W_hat, A, B, Xd))
    return X @ W_hat.T + s * (Xd @ A.T) @ B.T


def bwd_dx(dY, W_hat, A, B, s, keep, p) -> np.ndarray:
    """dX = dY . W^ + D * (s . (dY . B) . A) * fp32(1 / fp32(1 - p)) (fp64)."""
    dY, W_hat, A, B = (np.asarray(a, dtype=np.float64) for a in (dY, W_hat, A, B))
    return dY @ W_hat + np.where(keep, float(keep_scale(p)), 0.0) * (s * (dY @ B) @ A)


def lora_grads(Xd, dY, A, B, s):
    """dA = s . (dY . B)^T . Xd and dB = s . dY^T . (Xd . A^T) (fp64)."""
    Xd, dY, A, B = (np.asarray(a, dtype=np.float64) for a in (Xd, dY, A, B))
    return s * (dY @ B).T @ Xd, s * dY.T @ (Xd @ A.T)
