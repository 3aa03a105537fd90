"""GPU parity of LoRA dropout (qlora_lora_dropout and the _dropout forms of the
forward and input gradient) against ``oracle/dropout.py``.

* The dropped adapter input Xd is bit-exact: the same Philox4x64-10 draws,
  the same keep threshold round(fp32(p) * 65536), the same fp32 keep scale
  and bf16 rounding; checked at p = 0 (Xd == X), 0.05 (the pages' value) and
  0.5, with 64-bit seeds and offsets that use their high words.
* Y, dX (and dA, dB through qlora_lora_bwd with Xd) within 2e-2 of the
  oracle's fp64 products under the oracle's own mask.  With a zero weight the
  outputs are the (masked) adapter terms alone, so the mask and the keep
  scale are checked where nothing else hides them.
"""
import numpy as np
import pytest
import torch

import oracle_refs as R
from bit_nf4_quantized_qlora_b200 import binding as B
from bit_nf4_quantized_qlora_b200 import workloads as WL
from oracle import dropout, linear

pytestmark = pytest.mark.gpu
TOL = 2e-2
DEV = "cuda:0"
SEED, OFFSET = 0x1234_5678_9ABC_DEF1, 0x0000_0003_0000_0007


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("p", [0.0, 0.05, 0.5])
@pytest.mark.parametrize("mk", [(1, 64), (16, 1024), (300, 1088)], ids=lambda s: f"m{s[0]}_k{s[1]}")
def test_dropout_mask_and_values_bit_exact(mk, p):
    m, k = mk
    X = WL.bf16(WL.normal((m, k), 1.0, 6000 + m))
    Xd = B.qlora_lora_dropout(X.to(DEV), p, SEED, OFFSET)
    torch.cuda.synchronize()
    keep = dropout.keep_mask(m, k, p, SEED, OFFSET)
    want = dropout.dropout_bf16_bits(R.bf16_to_f64(X).astype(np.float32), keep, p)
    assert np.array_equal(_bits(Xd), want)
    if p == 0.0:
        assert np.array_equal(_bits(Xd), _bits(X))


def test_dropout_offsets_and_seeds_give_different_masks():
    X = WL.bf16(WL.normal((8, 512), 1.0, 6100)).to(DEV)
    a = B.qlora_lora_dropout(X, 0.5, SEED, OFFSET)
    b = B.qlora_lora_dropout(X, 0.5, SEED, OFFSET + 1)
    c = B.qlora_lora_dropout(X, 0.5, SEED + 1, OFFSET)
    torch.cuda.synchronize()
    for other in (b, c):
        same = float(((a == 0) == (other == 0)).float().mean())
        assert 0.4 < same < 0.6


def _inputs(n, k, m, r, seed, zero_weight):
    W = torch.zeros(n, k) if zero_weight else WL.weight(n, k, 0.02, seed=seed)
    X = WL.bf16(WL.normal((m, k), 1.0, seed + 1))
    dY = WL.bf16(WL.normal((m, n), 1.0, seed + 2))
    A = WL.bf16(WL.normal((r, k), 0.05, seed + 3))
    Bm = WL.bf16(WL.normal((n, r), 0.05, seed + 4))
    return W, X, dY, A, Bm


@pytest.mark.parametrize("zero_weight", [True, False], ids=["adapter_only", "full"])
@pytest.mark.parametrize("m,r,p", [(16, 16, 0.05), (300, 64, 0.05), (300, 256, 0.5), (1, 16, 0.5)])
def test_forward_input_gradient_and_adapter_grads_with_dropout(m, r, p, zero_weight):
    n, k, s = 776, 1088, 2.0
    W, X, dY, A, Bm = _inputs(n, k, m, r, 6200 + m + r, zero_weight)
    w = B.qlora_quantize_nf4_dq(W.to(DEV))
    Xg, dYg, Ag, Bg = X.to(DEV), dY.to(DEV), A.to(DEV), Bm.to(DEV)
    Y, Xd = B.qlora_linear_fwd_dropout(Xg, w, Ag, Bg, r, s, p, SEED, OFFSET)
    dX = B.qlora_linear_bwd_dx_dropout(dYg, w, Ag, Bg, r, s, p, SEED, OFFSET)
    dA, dB = B.qlora_lora_bwd(Xd, dYg, Ag, Bg, r, s)
    torch.cuda.synchronize()

    keep = dropout.keep_mask(m, k, p, SEED, OFFSET)
    Xf, dYf, Af, Bf = (R.bf16_to_f64(t) for t in (X, dY, A, Bm))
    Xd_ref = dropout.dropout_values(Xf.astype(np.float32), keep, p)
    assert np.array_equal(_bits(Xd), dropout.dropout_bf16_bits(Xf.astype(np.float32), keep, p))
    W_hat = np.zeros((n, k)) if zero_weight else R.dequant_full(W)
    assert R.err(R.bf16_to_f64(Y), dropout.fwd(Xf, W_hat, Af, Bf, s, Xd_ref)) <= TOL
    assert R.err(R.bf16_to_f64(dX), dropout.bwd_dx(dYf, W_hat, Af, Bf, s, keep, p)) <= TOL
    rA, rB = dropout.lora_grads(Xd_ref, dYf, Af, Bf, s)
    assert R.err(R.bf16_to_f64(dA), rA) <= TOL
    assert R.err(R.bf16_to_f64(dB), rB) <= TOL


def test_dropout_at_p_zero_is_the_plain_layer():
    n, k, m, r, s = 520, 640, 200, 16, 2.0
    W, X, dY, A, Bm = _inputs(n, k, m, r, 6300, False)
    w = B.qlora_quantize_nf4_dq(W.to(DEV))
    Xg, dYg, Ag, Bg = X.to(DEV), dY.to(DEV), A.to(DEV), Bm.to(DEV)
    Y0, _ = B.qlora_linear_fwd_dropout(Xg, w, Ag, Bg, r, s, 0.0, SEED, OFFSET)
    dX0 = B.qlora_linear_bwd_dx_dropout(dYg, w, Ag, Bg, r, s, 0.0, SEED, OFFSET)
    torch.cuda.synchronize()
    W_hat = R.dequant_full(W)
    Xf, dYf, Af, Bf = (R.bf16_to_f64(t) for t in (X, dY, A, Bm))
    assert R.err(R.bf16_to_f64(Y0), linear.fwd(Xf, W_hat, Af, Bf, s)) <= TOL
    assert R.err(R.bf16_to_f64(dX0), linear.bwd_dx(dYf, W_hat, Af, Bf, s)) <= TOL
