"""Oracle-side reference helpers for the GPU parity tests.

Everything here calls only ``oracle/`` (plus NumPy) on inputs drawn from
``bit_nf4_quantized_qlora_b200.workloads``; nothing reads a CUDA result.
"""
import numpy as np
import torch

from oracle import linear, quant

GROUP_ELEMS = 64 * 256


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 values of a bf16 torch tensor (CPU or GPU)."""
    return t.detach().to("cpu").to(torch.float32).numpy().astype(np.float64)


def quantize(W: torch.Tensor, codebook: str = "nf4"):
    """Oracle quantization of a whole fp32 weight: (packed, q, S)."""
    packed, q, S, _ = quant.quantize_nf4_dq(W.reshape(-1).numpy(), codebook)
    return packed, q, S


def quantize_groups(W: torch.Tensor, groups):
    """Oracle quantization of selected groups of 256 blocks (16384 weights):
    {g: (packed, q, S)}; a group is independent of all others."""
    flat = W.reshape(-1).numpy()
    out = {}
    for g in groups:
        sl = flat[g * GROUP_ELEMS:(g + 1) * GROUP_ELEMS]
        p, q, S, _ = quant.quantize_nf4_dq(sl)
        out[int(g)] = (p, q, S)
    return out


def dequant_rows(W: torch.Tensor, rows) -> np.ndarray:
    """Oracle W^ (fp64 values of bf16) for selected rows of a large weight,
    each computed from the group-aligned slice that covers it."""
    n, k = W.shape
    flat = W.reshape(-1).numpy()
    res = np.empty((len(rows), k), dtype=np.float64)
    for i, r in enumerate(rows):
        lo = (int(r) * k) // GROUP_ELEMS * GROUP_ELEMS
        hi = min(((int(r) + 1) * k + GROUP_ELEMS - 1) // GROUP_ELEMS * GROUP_ELEMS, n * k)
        p, q, S, _ = quant.quantize_nf4_dq(flat[lo:hi])
        vals = quant.dequant_bf16_values(p, q, S)
        off = int(r) * k - lo
        res[i] = vals[off:off + k]
    return res


def dequant_full(W: torch.Tensor, codebook: str = "nf4") -> np.ndarray:
    p, q, S = quantize(W, codebook)
    return quant.dequant_bf16_values(p, q, S, codebook).reshape(W.shape)


def fwd(X, W_hat, A, B, s):
    return linear.fwd(X, W_hat, A, B, s)


def bwd_dx(dY, W_hat, A, B, s):
    return linear.bwd_dx(dY, W_hat, A, B, s)


def lora_grads(X, dY, A, B, s):
    return linear.lora_grads(X, dY, A, B, s)


err = linear.max_abs_normalised_error
