"""The forward entry point without a workspace (qlora_linear_fwd_noalloc).

It serves callers that cannot allocate device memory (their host owns every
allocation, or allocation is forbidden on their serving path): the scratch
for the adapter intermediate lives in a fixed device array inside the
library.  Here it is called through the C ABI and compared with the regular
forward (caller workspace) and with the oracle, on two calls in a row with
different shapes, so a second call that read the first call's leftovers
would show.  This file is collected last so a failure here comes after every
other test has run.
"""
import ctypes

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


def _setup(n, k, m, r, seed):
    case = WL.LinearCase(f"noalloc_{n}x{k}_m{m}", n=n, k=k, m=m, r=r, alpha=2.0 * max(r, 1), w_seed=seed,
                         x_seed=seed + 1, a_seed=seed + 2, b_seed=seed + 3)
    w = B.qlora_quantize_nf4_dq(case.W().to(DEV))
    A = case.A().to(DEV) if r else None
    Bm = case.B().to(DEV) if r else None
    return case, w, case.X().to(DEV), A, Bm


def _call_noalloc(X, w, A, Bm, r, scale, Y):
    lib = B.lib()
    wc = w.c_struct()
    stream = torch.cuda.current_stream().cuda_stream
    return lib.qlora_linear_fwd_noalloc(X.data_ptr(), X.shape[0], ctypes.byref(wc),
                                        None if A is None else A.data_ptr(), None if Bm is None else Bm.data_ptr(),
                                        r, scale, Y.data_ptr(), stream)


def _oracle_fwd(case, r):
    W_hat = R.dequant_full(case.W())
    X = R.bf16_to_f64(case.X())
    if not r:
        return linear.fwd(X, W_hat)
    return linear.fwd(X, W_hat, R.bf16_to_f64(case.A()), R.bf16_to_f64(case.B()), case.scale)


def test_noalloc_forward_matches_workspace_forward_and_oracle_on_two_calls():
    torch.cuda.set_device(0)
    # first call: tensor-core path (m > 16); second: weight-streaming path;
    # third: no adapter (the built-in scratch is not used)
    for n, k, m, r, seed in ((1024, 1024, 300, 64, 700), (520, 640, 16, 16, 710), (264, 448, 40, 0, 730)):
        case, w, X, A, Bm = _setup(n, k, m, r, seed)
        ref = B.qlora_linear_fwd(X, w, A, Bm, r, case.scale)
        Y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_noalloc(X, w, A, Bm, r, case.scale, Y) == B.QLORA_OK
        torch.cuda.synchronize()
        assert R.err(R.bf16_to_f64(Y), R.bf16_to_f64(ref)) <= TOL
        assert R.err(R.bf16_to_f64(Y), _oracle_fwd(case, r)) <= TOL


def test_noalloc_rejects_scratch_beyond_its_limit_and_launches_nothing():
    torch.cuda.set_device(0)
    case, w, X, A, Bm = _setup(1024, 1024, 16, 16, 720)
    limit = 1 << 20                                     # QLORA_NOALLOC_SCRATCH_BYTES
    r = 256
    m_big = limit // (2 * r) + 1                        # m*r*2 > limit at r = 256
    Xb = torch.zeros(m_big, 1024, dtype=torch.bfloat16, device=DEV)
    Ab = torch.zeros(r, 1024, dtype=torch.bfloat16, device=DEV)
    Bb = torch.zeros(1024, r, dtype=torch.bfloat16, device=DEV)
    Y = torch.full((m_big, 1024), 7.0, dtype=torch.bfloat16, device=DEV)
    torch.cuda.synchronize()
    launches = B.qlora_launch_count()
    assert _call_noalloc(Xb, w, Ab, Bb, r, 1.0, Y) == B.QLORA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert B.qlora_launch_count() == launches
    assert bool((Y == 7.0).all())
    # the largest m that fits still runs and matches the workspace forward
    m_fit = limit // (2 * r)
    Xf = WL.bf16(WL.normal((m_fit, 1024), 1.0, 740)).to(DEV)
    Af = WL.bf16(WL.normal((r, 1024), 0.01, 741)).to(DEV)
    Bf = WL.bf16(WL.normal((1024, r), 0.01, 742)).to(DEV)
    Yf = torch.empty(m_fit, 1024, dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(Xf, w, Af, Bf, r, 0.125, Yf) == B.QLORA_OK
    ref = B.qlora_linear_fwd(Xf, w, Af, Bf, r, 0.125)
    torch.cuda.synchronize()
    assert R.err(R.bf16_to_f64(Yf), R.bf16_to_f64(ref)) <= TOL
