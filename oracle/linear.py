"""Forward and backward of the QLoRA linear layer, by definition, in fp64.
Test infrastructure: see ``oracle/__init__``.

The layer [P2 "The simple definition", "Storage precision is not calculation
precision"; P3 "The idea"; P4 "What is QLoRA?"; P5 figure 2 "A 4-bit statue
with 16-bit hands"]: the frozen base weight is dequantized to bf16 for the
matrix product and a trainable low-rank adapter is added beside it, with the
LoRA scaling s = alpha / r of the ``LoraConfig(r, lora_alpha)`` knobs shown on
[P3 "In code"]:

    Y  = X . W^T + s . (X . A^T) . B^T            X [m x k], W^ [n x k]
                                                  A [r x k], B [n x r]
Gradients flow through the frozen W^ into the input and into the adapters
only; W gets none [P2 "Follow one QLoRA training step", step 4; P4 "What is
QLoRA?"; P5 figure 2].  For an upstream gradient dY [m x n]:

    dX = dY . W^ + s . (dY . B) . A
    dA = s . (dY . B)^T . X
    dB = s . dY^T . (X . A^T)

All arguments are the exact values of bf16 tensors (as float arrays); the
products are accumulated in fp64 with ``numpy.matmul``.  The intermediate
rank-r products are kept in fp64 here; the GPU may round them to bf16, which
the stated tolerance covers.
"""

import numpy as np


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def lora_t(X, A, s):
    """T = s . X . A^T  [m x r]."""
    return s * (_f64(X) @ _f64(A).T)


def lora_u(dY, B, s):
    """U = s . dY . B  [m x r]."""
    return s * (_f64(dY) @ _f64(B))


def fwd(X, W_hat, A=None, B=None, s=0.0):
    """Y = X . W^T + s . (X . A^T) . B^T ; A or B None means no adapter."""
    y = _f64(X) @ _f64(W_hat).T
    if A is not None and B is not None:
        y = y + lora_t(X, A, s) @ _f64(B).T
    return y


def bwd_dx(dY, W_hat, A=None, B=None, s=0.0):
    """dX = dY . W^ + s . (dY . B) . A."""
    dx = _f64(dY) @ _f64(W_hat)
    if A is not None and B is not None:
        dx = dx + lora_u(dY, B, s) @ _f64(A)
    return dx


def lora_grads(X, dY, A, B, s):
    """(dA, dB) = (s . (dY . B)^T . X,  s . dY^T . (X . A^T))."""
    dA = lora_u(dY, B, s).T @ _f64(X)
    dB = _f64(dY).T @ lora_t(X, A, s)
    return dA, dB


def max_abs_normalised_error(got, ref) -> float:
    """max |got - ref| / max |ref|  (0 when both are all zero)."""
    got = _f64(got)
    ref = _f64(ref)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    if den == 0.0:
        return num
    return num / den
