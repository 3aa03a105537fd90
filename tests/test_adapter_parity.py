"""GPU parity of the adapter terms, on every dispatch path and at every rank.

The whole-output parity tests cannot see a small adapter term: at the 7B MLP
shape s.(X.A^T).B^T is about 1 % of max|Y|, under the 2e-2 bar.  Here the
adapter term is made visible two ways.

* Isolated: the frozen weight is all zeros.  Its blocks quantize to the zero
  code with absmax 0, so W^ = 0 exactly (a pin of the oracle) and the
  library's output is the adapter term alone: Y = bf16(T . B^T) with
  T = bf16(s X A^T), dX = bf16(U . A) with U = bf16(s dY B).  Each is held
  to 2e-2 (max-abs-normalised) against the oracle's s.(X.A^T).B^T and
  s.(dY.B).A, so a dropped or partial adapter k-step, a wrong B tile or a
  wrong scale fails.
* Composed: a real N(0, 0.02) weight with adapters large enough that the
  adapter term is about as large as the base term, so the sum is checked
  where both parts matter.

Dispatch paths of the forward: m <= 4 (per-warp streaming kernel), m = 5..16
(CTA-ring kernel), 16 < m <= 128 (tensor-core kernel, one 128-row tile),
m > 128 (the large-M fused kernel); of the input gradient: m <= 128 and
m > 128.  Ranks 16, 64, 128 and 256 run one to four adapter k-steps of 64.
"""
import numpy as np
import pytest
import torch

import oracle_refs as R
from bit_nf4_quantized_qlora_b200 import binding as B
from bit_nf4_quantized_qlora_b200 import workloads as WL
from oracle import linear

pytestmark = pytest.mark.gpu
TOL = 2e-2
DEV = "cuda:0"

FWD_M = (1, 4, 8, 16, 64, 128, 300, 1024)
BWD_M = (1, 16, 128, 129, 300)
RANKS = (16, 64, 128, 256)


def _zero_weight(n, k):
    w = B.qlora_quantize_nf4_dq(torch.zeros(n, k, dtype=torch.float32, device=DEV))
    torch.cuda.synchronize()
    return w


def _adapters(n, k, r, seed, std=0.05):
    A = WL.bf16(WL.normal((r, k), std, seed))
    Bm = WL.bf16(WL.normal((n, r), std, seed + 1))
    return A, Bm


def test_zero_weight_dequantizes_to_zero_in_the_oracle():
    """The isolation relies on W = 0 giving W^ = 0 exactly."""
    assert np.all(R.dequant_full(torch.zeros(8, 128)) == 0.0)


@pytest.mark.parametrize("r", RANKS)
@pytest.mark.parametrize("m", FWD_M)
def test_fwd_adapter_term_isolated(m, r):
    n, k = 776, 1088                                     # ragged against 256-wide tiles and 4-block chunks
    w = _zero_weight(n, k)
    X = WL.bf16(WL.normal((m, k), 1.0, 4000 + m))
    A, Bm = _adapters(n, k, r, 4100 + r)
    s = 2.0
    Y = B.qlora_linear_fwd(X.to(DEV), w, A.to(DEV), Bm.to(DEV), r, s)
    torch.cuda.synchronize()
    ref = linear.lora_t(R.bf16_to_f64(X), R.bf16_to_f64(A), s) @ R.bf16_to_f64(Bm).T
    e = R.err(R.bf16_to_f64(Y), ref)
    assert e <= TOL, e


@pytest.mark.parametrize("r", RANKS)
@pytest.mark.parametrize("m", BWD_M)
def test_bwd_dx_adapter_term_isolated(m, r):
    n, k = 776, 1088
    w = _zero_weight(n, k)
    dY = WL.bf16(WL.normal((m, n), 1.0, 4200 + m))
    A, Bm = _adapters(n, k, r, 4300 + r)
    s = 0.5
    dX = B.qlora_linear_bwd_dx(dY.to(DEV), w, A.to(DEV), Bm.to(DEV), r, s)
    torch.cuda.synchronize()
    ref = linear.lora_u(R.bf16_to_f64(dY), R.bf16_to_f64(Bm), s) @ R.bf16_to_f64(A)
    e = R.err(R.bf16_to_f64(dX), ref)
    assert e <= TOL, e


@pytest.mark.parametrize("r", (16, 256))
@pytest.mark.parametrize("m", (1, 16, 128, 300))
def test_fwd_and_bwd_dx_with_comparable_adapter_term(m, r):
    """Base and adapter terms of similar size: missing either one is a
    failure of about half the output."""
    n, k = 520, 1024
    W = WL.weight(n, k, 0.02, seed=4400 + m)
    w = B.qlora_quantize_nf4_dq(W.to(DEV))
    X = WL.bf16(WL.normal((m, k), 1.0, 4500 + m))
    dY = WL.bf16(WL.normal((m, n), 1.0, 4600 + m))
    A, Bm = _adapters(n, k, r, 4700 + r, std=0.05 if r == 16 else 0.02)
    s = 2.0
    Xd, Ad, Bd = X.to(DEV), A.to(DEV), Bm.to(DEV)
    Y = B.qlora_linear_fwd(Xd, w, Ad, Bd, r, s)
    dX = B.qlora_linear_bwd_dx(dY.to(DEV), w, Ad, Bd, r, s)
    torch.cuda.synchronize()
    W_hat = R.dequant_full(W)
    Xf, Af, Bf, dYf = (R.bf16_to_f64(t) for t in (X, A, Bm, dY))
    base = Xf @ W_hat.T
    lora = linear.lora_t(Xf, Af, s) @ Bf.T
    assert 0.3 < np.abs(lora).max() / np.abs(base).max() < 3.0
    assert R.err(R.bf16_to_f64(Y), base + lora) <= TOL
    base_dx = dYf @ W_hat
    lora_dx = linear.lora_u(dYf, Bf, s) @ Af
    assert 0.3 < np.abs(lora_dx).max() / np.abs(base_dx).max() < 3.0
    assert R.err(R.bf16_to_f64(dX), base_dx + lora_dx) <= TOL


def test_adapter_term_isolated_at_7b_gate_full_size():
    """7B MLP gate shape (11008 x 4096, m = 4096, r = 64, alpha = 16) with a
    zero weight: Y = bf16(T B^T) and dX = bf16(U A) on sampled rows."""
    case = WL.mlp_7b("gate")
    n, k, m, r = case.n, case.k, case.m, case.r
    w = _zero_weight(n, k)
    X, dY, A, Bm = case.X(), case.dY(), case.A(), case.B()
    Y = B.qlora_linear_fwd(X.to(DEV), w, A.to(DEV), Bm.to(DEV), r, case.scale)
    dX = B.qlora_linear_bwd_dx(dY.to(DEV), w, A.to(DEV), Bm.to(DEV), r, case.scale)
    torch.cuda.synchronize()
    rng = np.random.default_rng(7)
    xs = np.unique(np.concatenate([rng.choice(m, 32, replace=False), [0, m - 1]]))
    Af, Bf = R.bf16_to_f64(A), R.bf16_to_f64(Bm)
    ref_y = linear.lora_t(R.bf16_to_f64(X[xs]), Af, case.scale) @ Bf.T
    assert R.err(R.bf16_to_f64(Y[xs]), ref_y) <= TOL
    ref_dx = linear.lora_u(R.bf16_to_f64(dY[xs]), Bf, case.scale) @ Af
    assert R.err(R.bf16_to_f64(dX[xs]), ref_dx) <= TOL

