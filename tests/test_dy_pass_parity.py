"""GPU parity of the one-pass adapter products (U = bf16(s dY B) and
dB = bf16(dY^T T) from a single read of dY, r <= 64) against the oracle.

qlora_lora_bwd and qlora_linear_bwd take this path for every r <= 64.  dB is
compared directly; U is seen through dA = U^T X and, with a zero weight,
through dX = U . A alone, both pure adapter terms.  Shapes cover:
* r in {16, 32, 48, 64} (N = 64 MMAs whose columns past r are zero);
* ragged m (a last 128-row block with 44 rows, or with one row) and ragged n
  (776 = 6 blocks + 8 rows);
* clusters of 1, 2, 4 and 8 CTAs along m (m = 16, 300, 600, 4096) and up to
  six 128-column blocks per n-range;
* the 7B MLP gate shape at full size (m = 4096, n = 11008, r = 64).
Results are deterministic: the dB partials are added in cluster-rank order
and the U partials in n-range order, so two runs agree bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle_refs as R
from bit_nf4_quantized_qlora_b200 import binding as B
from bit_nf4_quantized_qlora_b200 import workloads as WL

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 2e-2


def _inputs(m, n, k, r, seed):
    X = WL.bf16(WL.normal((m, k), 1.0, seed))
    dY = WL.bf16(WL.normal((m, n), 1.0, seed + 1))
    A = WL.bf16(WL.normal((r, k), 0.05, seed + 2))
    Bm = WL.bf16(WL.normal((n, r), 0.05, seed + 3))
    return X, dY, A, Bm


CASES = [(300, 776, 640, 16), (300, 776, 640, 32), (300, 776, 640, 48), (300, 776, 640, 64),
         (16, 1024, 512, 64), (129, 520, 256, 32), (1, 264, 192, 16), (600, 4104, 1024, 64),
         (4096, 2056, 512, 16)]


@pytest.mark.parametrize("mnkr", CASES, ids=lambda c: "m%d_n%d_k%d_r%d" % c)
def test_lora_bwd_one_pass(mnkr):
    m, n, k, r = mnkr
    s = 2.0
    X, dY, A, Bm = _inputs(m, n, k, r, 8000 + m + r)
    dA, dB = B.qlora_lora_bwd(X.to(DEV), dY.to(DEV), A.to(DEV), Bm.to(DEV), r, s)
    dA2, dB2 = B.qlora_lora_bwd(X.to(DEV), dY.to(DEV), A.to(DEV), Bm.to(DEV), r, s)
    torch.cuda.synchronize()
    rA, rB = R.lora_grads(*(R.bf16_to_f64(t) for t in (X, dY, A, Bm)), s)
    assert R.err(R.bf16_to_f64(dA), rA) <= TOL
    assert R.err(R.bf16_to_f64(dB), rB) <= TOL
    assert torch.equal(dA, dA2) and torch.equal(dB, dB2)


@pytest.mark.parametrize("mr", [(300, 64), (4096, 64), (16, 32)], ids=lambda c: "m%d_r%d" % c)
def test_linear_bwd_adapter_term_through_one_pass(mr):
    """A zero weight: dX = U . A exactly the adapter term, so a wrong U (a
    missing n-range, a wrong scale, a transposed tile) shows in dX."""
    m, r = mr
    n, k, s = 776, 1088, 0.5
    X, dY, A, Bm = _inputs(m, n, k, r, 8100 + m)
    w = B.qlora_quantize_nf4_dq(torch.zeros(n, k, device=DEV))
    dX, dA, dB = B.qlora_linear_bwd(dY.to(DEV), X.to(DEV), w, A.to(DEV), Bm.to(DEV), r, s)
    torch.cuda.synchronize()
    Xf, dYf, Af, Bf = (R.bf16_to_f64(t) for t in (X, dY, A, Bm))
    U = s * dYf @ Bf
    assert R.err(R.bf16_to_f64(dX), U @ Af) <= TOL
    rA, rB = R.lora_grads(Xf, dYf, Af, Bf, s)
    assert R.err(R.bf16_to_f64(dA), rA) <= TOL
    assert R.err(R.bf16_to_f64(dB), rB) <= TOL


def test_7b_gate_full_size():
    m, n, k, r, s = 4096, 11008, 4096, 64, 0.25
    X, dY, A, Bm = _inputs(m, n, k, r, 8200)
    dA, dB = B.qlora_lora_bwd(X.to(DEV), dY.to(DEV), A.to(DEV), Bm.to(DEV), r, s)
    torch.cuda.synchronize()
    rA, rB = R.lora_grads(*(R.bf16_to_f64(t) for t in (X, dY, A, Bm)), s)
    assert R.err(R.bf16_to_f64(dA), rA) <= TOL
    assert R.err(R.bf16_to_f64(dB), rB) <= TOL
    assert B.qlora_poll_device_error() == 0
