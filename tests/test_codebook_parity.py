"""GPU parity of the FP4 and INT4 baseline codebooks through every kernel.

The codebook is a table the kernels take as a parameter, so the same bars as
NF4 apply: packed codes, absmax codes and group scales bit-exact against the
oracle quantizing with that codebook; the dequantized bf16 weight bit-exact
(FP4's -0 level included); forward and input gradient within 2e-2 of the fp64
oracle on every path (decode streaming m <= 4, CTA ring m <= 16, tcgen05
16 < m <= 128, fused forward m > 128).
"""
import numpy as np
import pytest
import torch

import oracle_refs as R
from bit_nf4_quantized_qlora_b200 import binding as B
from bit_nf4_quantized_qlora_b200 import workloads as WL
from oracle import codebooks, quant

pytestmark = pytest.mark.gpu
TOL = 2e-2
DEV = "cuda:0"
NAMES = ["fp4", "int4"]


def _np(t):
    return t.detach().cpu().numpy()


def _quant(W: torch.Tensor, name: str) -> B.NF4Weight:
    w = B.qlora_quantize_4bit_dq(W.to(DEV), B.CODEBOOKS[name])
    torch.cuda.synchronize()
    return w


@pytest.mark.parametrize("name", NAMES)
@pytest.mark.parametrize("shape", [(1024, 1024), (136, 448), (300, 8192)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_quantize_and_dequant_bit_exact(name, shape):
    n, k = shape
    W = WL.weight(n, k, 0.02, seed=900 + n, outlier_frac=0.001)
    W[0, :64] = 0.0                                   # an all-zero block
    W[1, 5] = -0.0
    W[2, 7] = 0.0
    w = _quant(W, name)
    assert w.codebook == B.CODEBOOKS[name]
    packed, q, S = R.quantize(W, name)
    assert np.array_equal(_np(w.codes), packed)
    assert np.array_equal(_np(w.absmax_q), q)
    assert np.array_equal(_np(w.group_scale).view(np.uint32), S.view(np.uint32))
    got = B.qlora_dequant(w)
    torch.cuda.synchronize()
    ref = quant.dequant_bf16_bits(packed, q, S, name)
    assert np.array_equal(_np(got.view(torch.int16)).view(np.uint16).reshape(-1), ref)


@pytest.mark.parametrize("name", NAMES)
def test_codes_near_midpoints(name):
    """Every midpoint of the codebook times the block absmax and +-1 ulp
    around it, over 512 absmax values spanning 30 binades."""
    rng = np.random.default_rng(77)
    mids = codebooks.midpoints_f32(name)
    nblk = 512
    c = (2.0 ** rng.uniform(-20, 10, nblk)).astype(np.float32)
    W = np.zeros((nblk, 64), dtype=np.float32)
    W[:, 0] = c
    for b in range(nblk):
        vals = []
        for t in mids:
            base = np.float32(t * c[b])
            vals += [np.nextafter(base, np.float32(-np.inf)), base, np.nextafter(base, np.float32(np.inf))]
        vals = np.clip(np.array(vals, dtype=np.float32), -c[b], c[b])
        W[b, 1:1 + vals.size] = vals
    Wt = torch.from_numpy(W.reshape(nblk // 4, 256))
    w = _quant(Wt, name)
    packed, q, S = R.quantize(Wt, name)
    assert np.array_equal(_np(w.codes), packed)
    assert np.array_equal(_np(w.absmax_q), q)


FWD = [(1024, 1024, 1, 16), (264, 1088, 4, 0), (1024, 1024, 16, 16), (520, 640, 96, 16), (1024, 1024, 300, 64)]


@pytest.mark.parametrize("name", NAMES)
@pytest.mark.parametrize("nkmr", FWD, ids=lambda c: "n%d_k%d_m%d_r%d" % c)
def test_fwd_parity(name, nkmr):
    n, k, m, r = nkmr
    case = WL.LinearCase(f"cb_{n}x{k}_m{m}", n=n, k=k, m=m, r=r, alpha=32.0, w_seed=910, x_seed=911, a_seed=912,
                         b_seed=913, dy_seed=914)
    W, X = case.W(), case.X()
    A = case.A() if r else None
    Bm = case.B() if r else None
    w = _quant(W, name)
    Y = B.qlora_linear_fwd(X.to(DEV), w, A.to(DEV) if r else None, Bm.to(DEV) if r else None, r, case.scale)
    torch.cuda.synchronize()
    ref = R.fwd(R.bf16_to_f64(X), R.dequant_full(W, name), R.bf16_to_f64(A) if r else None,
                R.bf16_to_f64(Bm) if r else None, case.scale)
    assert R.err(R.bf16_to_f64(Y), ref) <= TOL


@pytest.mark.parametrize("name", NAMES)
def test_bwd_dx_parity(name):
    case = WL.LinearCase("cb_bwd", n=776, k=512, m=129, r=32, alpha=32.0, w_seed=920, x_seed=921, a_seed=922,
                         b_seed=923, dy_seed=924)
    W, A, Bm, dY = case.W(), case.A(), case.B(), case.dY()
    w = _quant(W, name)
    dX = B.qlora_linear_bwd_dx(dY.to(DEV), w, A.to(DEV), Bm.to(DEV), case.r, case.scale)
    torch.cuda.synchronize()
    ref = R.bwd_dx(R.bf16_to_f64(dY), R.dequant_full(W, name), R.bf16_to_f64(A), R.bf16_to_f64(Bm), case.scale)
    assert R.err(R.bf16_to_f64(dX), ref) <= TOL


def test_nf4_has_the_lowest_error_through_the_library():
    """The pages' claim on the library's own quantize + dequant: on normal
    weights NF4's round-trip error is below both baselines'."""
    W = WL.weight(1024, 4096, 0.02, seed=930)
    Wd = W.to(DEV)
    mse = {}
    for name in ("nf4", "fp4", "int4"):
        w = _quant(W, name)
        back = B.qlora_dequant(w).float()
        mse[name] = float(((back - Wd) ** 2).mean())
    assert mse["nf4"] < 0.85 * mse["fp4"], mse
    assert mse["nf4"] < 0.85 * mse["int4"], mse
