"""GPU parity of the E4M3 + mean absmax format (QLORA_DQ_FP8_MEAN) against
``oracle/dq_fp8.py``.

* Quantization is bit-exact: the packed codes, the E4M3 absmax codes and the
  ng + 1 group entries (the fp32 scales S_g / 448, then the tensor mean mu,
  whose fp64 pairwise sums must be added in the oracle's order).  Shapes
  cover one block, one partial group, many groups with a partial last group
  of fewer than 8 blocks, whole groups only, and the degenerate weights (all
  zero; every block with the same absmax, where mu is exact and every offset
  is zero).
* Dequantization is bit-exact, for NF4 and the FP4 baseline codebook.
* Every product path decodes the format: the forward at m = 1 (the three
  absmax-code load modes of the decode-sized kernel: k/64 a multiple of 16,
  of 4, and neither), m = 12 (CTA-ring kernel), m = 96 (one-CTA tcgen05
  kernel) and m = 300 (paired kernel); the input gradient at m = 16
  (split-K) and m = 300 (paired kernel); all within 2e-2 of the oracle's
  fp64 products with the oracle's W^.
* The merge exports W^ + s B A within the merge's own bound.
"""
import numpy as np
import pytest
import torch

import oracle_refs as R
from bit_nf4_quantized_qlora_b200 import binding as B
from bit_nf4_quantized_qlora_b200 import workloads as WL
from oracle import dq_fp8, linear, merge

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 2e-2


def _quantize(W: torch.Tensor, codebook: str = "nf4"):
    return B.qlora_quantize_4bit_dq(W.to(DEV), B.CODEBOOKS[codebook], dq_format=B.QLORA_DQ_FP8_MEAN)


def _np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)


def _w_hat(W: torch.Tensor, codebook: str = "nf4") -> np.ndarray:
    packed, q, gs, _ = dq_fp8.quantize(W.reshape(-1).numpy(), codebook)
    return dq_fp8.dequant_bf16_values(packed, q, gs, codebook).reshape(W.shape)


SHAPES = [(1, 64), (7, 1088), (300, 1088), (515, 64), (1024, 1024), (776, 1280)]


@pytest.mark.parametrize("nk", SHAPES, ids=lambda s: f"n{s[0]}_k{s[1]}")
def test_quantize_and_dequant_bit_exact(nk):
    n, k = nk
    W = WL.weight(n, k, 0.02, seed=7000 + n)
    w = _quantize(W)
    absmax = torch.empty(n * k // 64, dtype=torch.float32, device=DEV)
    w2 = B.qlora_quantize_4bit_dq(W.to(DEV), B.QLORA_CODEBOOK_NF4, absmax_fp32=absmax,
                                  dq_format=B.QLORA_DQ_FP8_MEAN)
    Wh = B.qlora_dequant(w)
    torch.cuda.synchronize()
    packed, q, gs, c = dq_fp8.quantize(W.reshape(-1).numpy())
    assert w.group_scale.numel() == gs.size
    assert np.array_equal(_np(w.codes), packed)
    assert np.array_equal(_np(w.absmax_q), q)
    assert np.array_equal(_np(w.group_scale).view(np.uint32), gs.view(np.uint32))
    assert np.array_equal(_np(absmax).view(np.uint32), c.view(np.uint32))
    assert np.array_equal(_np(w2.absmax_q), q)
    assert np.array_equal(_bits(Wh), dq_fp8.dequant_bf16_bits(packed, q, gs))


def test_fp4_codebook_in_the_fp8_format():
    W = WL.weight(264, 576, 0.02, seed=7100)
    w = _quantize(W, "fp4")
    Wh = B.qlora_dequant(w)
    torch.cuda.synchronize()
    packed, q, gs, _ = dq_fp8.quantize(W.reshape(-1).numpy(), "fp4")
    assert np.array_equal(_np(w.codes), packed) and np.array_equal(_np(w.absmax_q), q)
    assert np.array_equal(_bits(Wh), dq_fp8.dequant_bf16_bits(packed, q, gs, "fp4"))


@pytest.mark.parametrize("kind", ["zero", "equal_absmax"])
def test_degenerate_weights(kind):
    n, k = 520, 640
    if kind == "zero":
        W = torch.zeros(n, k)
    else:
        sign = torch.sign(WL.normal((n, k), 1.0, 7200))
        W = torch.where(sign == 0, torch.ones_like(sign), sign) * 0.03
    w = _quantize(W)
    Wh = B.qlora_dequant(w)
    torch.cuda.synchronize()
    packed, q, gs, _ = dq_fp8.quantize(W.reshape(-1).numpy())
    assert np.all(q == 0)
    assert np.array_equal(_np(w.absmax_q), q)
    assert np.array_equal(_np(w.group_scale).view(np.uint32), gs.view(np.uint32))
    assert np.array_equal(_bits(Wh), dq_fp8.dequant_bf16_bits(packed, q, gs))


def _case(n, k, m, r, seed):
    W = WL.weight(n, k, 0.02, seed=seed)
    X = WL.bf16(WL.normal((m, k), 1.0, seed + 1))
    dY = WL.bf16(WL.normal((m, n), 1.0, seed + 2))
    A = WL.bf16(WL.normal((r, k), 0.05, seed + 3))
    Bm = WL.bf16(WL.normal((n, r), 0.05, seed + 4))
    return W, X, dY, A, Bm


@pytest.mark.parametrize("n,k,m", [(776, 1024, 1), (776, 1280, 1), (776, 1088, 1), (520, 1088, 12),
                                   (776, 1088, 96), (776, 1088, 300)])
def test_forward_paths(n, k, m):
    r, s = 16, 2.0
    W, X, _, A, Bm = _case(n, k, m, r, 7300 + m + k)
    w = _quantize(W)
    Y = B.qlora_linear_fwd(X.to(DEV), w, A.to(DEV), Bm.to(DEV), r, s)
    torch.cuda.synchronize()
    Xf, Af, Bf = (R.bf16_to_f64(t) for t in (X, A, Bm))
    assert R.err(R.bf16_to_f64(Y), linear.fwd(Xf, _w_hat(W), Af, Bf, s)) <= TOL


@pytest.mark.parametrize("m", [16, 300])
def test_input_gradient_and_adapter_grads(m):
    n, k, r, s = 776, 1088, 64, 2.0
    W, X, dY, A, Bm = _case(n, k, m, r, 7400 + m)
    w = _quantize(W)
    dX, dA, dB = B.qlora_linear_bwd(dY.to(DEV), X.to(DEV), w, A.to(DEV), Bm.to(DEV), r, s)
    torch.cuda.synchronize()
    Xf, dYf, Af, Bf = (R.bf16_to_f64(t) for t in (X, dY, A, Bm))
    assert R.err(R.bf16_to_f64(dX), linear.bwd_dx(dYf, _w_hat(W), Af, Bf, s)) <= TOL
    rA, rB = linear.lora_grads(Xf, dYf, Af, Bf, s)
    assert R.err(R.bf16_to_f64(dA), rA) <= TOL
    assert R.err(R.bf16_to_f64(dB), rB) <= TOL


def test_merge_in_the_fp8_format():
    n, k, r, s = 264, 576, 32, 2.0
    W, _, _, A, Bm = _case(n, k, 1, r, 7500)
    w = _quantize(W)
    h, f = B.qlora_merge_adapter(w, A.to(DEV), Bm.to(DEV), r, s, want_bf16=True, want_f32=True)
    h0, _ = B.qlora_merge_adapter(w, None, None, 0, s)
    torch.cuda.synchronize()
    W_hat = _w_hat(W)
    An, Bn = R.bf16_to_f64(A), R.bf16_to_f64(Bm)
    ref = merge.merge_f64(W_hat, An, Bn, s)
    bound = (r + 2) * 2.0 ** -24 * (np.abs(W_hat) + s * (np.abs(Bn) @ np.abs(An))) + 2.0 ** -149
    assert np.all(np.abs(f.double().cpu().numpy() - ref) <= bound)
    assert np.array_equal(R.bf16_to_f64(h0), W_hat)
