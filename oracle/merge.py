"""Adapter merge: fold the trained LoRA update into the dequantized base.
Test infrastructure: see ``oracle/__init__``.

What the pages fix:
  [P2 "Curiosity question: is the final model permanently 4-bit?", "Training
  setup versus deployment setup"]  after training, the quantized base and the
  adapter may be served apart, merged into another checkpoint, or moved to
  another serving precision.
  [P2 "Common misconception"; P5 "Nothing about LoRA changes" before figure
  3]  QLoRA keeps LoRA's mergeability: the two small matrices fold back into
  the frozen weight.

The merged weight is the one whose plain product equals the layer's forward
(``oracle.linear.fwd``): X . W'^T = X . W^^T + s . (X . A^T) . B^T for every X,
so W' = W^ + s . B . A with W^ the dequantized base (the only base a quantized
checkpoint has) and s = alpha / r.

Readings (the pages give no precision or export format): W' is formed in
fp32, the layer's accumulation type, and exported either as fp32 (to be
re-quantized by the blockwise quantizer into a new 4-bit checkpoint) or
rounded once to bf16, the compute type.  The reference below is the exact
value in fp64; its bf16 export is bf16_rne(fp32(W')).
"""

import numpy as np

from . import quant


def merge_f64(W_hat, A, B, s) -> np.ndarray:
    """W' = W^ + s . B . A in fp64: W^ [n x k], A [r x k], B [n x r]."""
    W_hat = np.asarray(W_hat, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    return W_hat + float(s) * (B @ A)


def merge_bf16_bits(W_hat, A, B, s) -> np.ndarray:
    """The bf16 export: bf16_rne(fp32(W')) as uint16 bit patterns."""
    return quant.bf16_rne_bits(merge_f64(W_hat, A, B, s).astype(np.float32))
