"""The forward entry point without a workspace (qlora_linear_fwd_noalloc).

It serves callers that cannot allocate device memory (their host owns every
allocation, or allocation is forbidden on their serving path): the scratch
for the adapter intermediate lives in a fixed device array inside the
library.  Here it is called through the C ABI and compared with the regular
forward (caller workspace) on two calls in a row with different shapes, so a
second call that read the first call's leftovers would show.  This file is
collected last so a failure here comes after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantized_qlora_b200 import binding as B
from bit_nf4_quantized_qlora_b200 import workloads as WL

pytestmark = pytest.mark.gpu
TOL = 2e-2
DEV = "cuda:0"


def _err(got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    den = np.max(np.abs(r))
    return float(np.max(np.abs(g - r)) / den) if den > 0 else float(np.max(np.abs(g - r)))


def _setup(n, k, m, r, seed):
    case = WL.LinearCase(f"noalloc_{n}x{k}_m{m}", n=n, k=k, m=m, r=r, alpha=2.0 * r, w_seed=seed,
                         x_seed=seed + 1, a_seed=seed + 2, b_seed=seed + 3)
    w = B.qlora_quantize_nf4_dq(case.W().to(DEV))
    return case, w, case.X().to(DEV), case.A().to(DEV), case.B().to(DEV)


def _call_noalloc(X, w, A, Bm, r, scale, Y):
    lib = B.lib()
    wc = w.c_struct()
    stream = torch.cuda.current_stream().cuda_stream
    return lib.qlora_linear_fwd_noalloc(X.data_ptr(), X.shape[0], ctypes.byref(wc), A.data_ptr(), Bm.data_ptr(),
                                        r, scale, Y.data_ptr(), stream)


def test_noalloc_forward_matches_workspace_forward_on_two_calls():
    torch.cuda.set_device(0)
    # first call: tensor-core path (m > 16); second: weight-streaming path
    for n, k, m, r, seed in ((1024, 1024, 300, 64, 700), (520, 640, 16, 16, 710)):
        case, w, X, A, Bm = _setup(n, k, m, r, seed)
        ref = B.qlora_linear_fwd(X, w, A, Bm, r, case.scale)
        Y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_noalloc(X, w, A, Bm, r, case.scale, Y) == B.QLORA_OK
        torch.cuda.synchronize()
        assert _err(Y, ref) <= TOL


def test_noalloc_rejects_scratch_beyond_its_limit():
    torch.cuda.set_device(0)
    case, w, X, A, Bm = _setup(1024, 1024, 16, 16, 720)
    limit = 1 << 20                                     # QLORA_NOALLOC_SCRATCH_BYTES
    m_big = limit // (2 * 256) + 1                      # m*r*2 > limit at r = 256
    r = 256
    Xb = torch.zeros(m_big, 1024, dtype=torch.bfloat16, device=DEV)
    Ab = torch.zeros(r, 1024, dtype=torch.bfloat16, device=DEV)
    Bb = torch.zeros(1024, r, dtype=torch.bfloat16, device=DEV)
    Y = torch.empty(m_big, 1024, dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(Xb, w, Ab, Bb, r, 1.0, Y) == B.QLORA_ERR_WORKSPACE
