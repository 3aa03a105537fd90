"""The device-side guards, exercised without faulting anything.

* A bounded wait that runs out: the self-test kernel waits on an mbarrier
  that nothing arrives at, through the same bounded wait every pipelined
  kernel uses; after its limit it sets its bit in the device error word and
  returns.  The poll reports the bit, the poll clears it, and a normal
  forward afterwards still matches the oracle (the context stays usable).
* fp32(s / 255), computed by Markstein's correctly rounded division where
  the decode and merge kernels form the double-quantization constant, equals
  IEEE division on every fp32 value of whole binades (both result binades of
  each), including the binades just above the switch to IEEE division.
"""
import numpy as np
import pytest
import torch

import oracle_refs as R
from bit_nf4_quantized_qlora_b200 import binding as B
from bit_nf4_quantized_qlora_b200 import workloads as WL

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_bounded_wait_runs_out_sets_its_flag_and_leaves_the_context_usable():
    torch.cuda.set_device(0)
    assert B.qlora_poll_device_error() == 0
    expired = torch.zeros(1, dtype=torch.int32, device=DEV)
    B.qlora_selftest_bounded_wait(1_000_000, expired)          # 1 ms
    torch.cuda.synchronize()
    assert int(expired.item()) == 1
    flags = B.qlora_poll_device_error()
    assert flags == B.QLORA_DEVERR_SELFTEST
    assert B.qlora_poll_device_error() == 0                      # the poll cleared it
    case = WL.single_linear()
    w = B.qlora_quantize_nf4_dq(case.W().to(DEV))
    Y = B.qlora_linear_fwd(case.X().to(DEV), w, case.A().to(DEV), case.B().to(DEV), case.r, case.scale)
    torch.cuda.synchronize()
    ref = R.fwd(R.bf16_to_f64(case.X()), R.dequant_full(case.W()), R.bf16_to_f64(case.A()),
                R.bf16_to_f64(case.B()), case.scale)
    assert R.err(R.bf16_to_f64(Y), ref) <= 2e-2
    assert B.qlora_poll_device_error() == 0


def _binade_bits(e: int):
    """First fp32 bit pattern and count of the binade [2^e, 2^(e+1))."""
    return (e + 127) << 23, 1 << 23


@pytest.mark.parametrize("e", [-100, -99, -60, -8, 0, 7, 8, 60, 126, 127])
def test_div255_equals_ieee_division_on_whole_binades(e):
    first, count = _binade_bits(e)
    if e == 127:
        count -= 1                                             # up to the largest finite value
    mism = torch.zeros(1, dtype=torch.int64, device=DEV)
    B.qlora_selftest_div255(first, count, mism)
    torch.cuda.synchronize()
    assert int(mism.item()) == 0


def test_div255_on_the_subnormal_range():
    mism = torch.zeros(1, dtype=torch.int64, device=DEV)
    B.qlora_selftest_div255(1, (1 << 23) - 1, mism)            # every positive subnormal
    torch.cuda.synchronize()
    assert int(mism.item()) == 0
