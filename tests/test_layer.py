"""The QLoRA linear as an autograd module, alone and inside a 7B-shaped
decoder block (q, k, v, o, gate, up, down all NF4 + LoRA), against an fp64
CPU reference that uses the oracle's dequantized weights.

The reference runs the same block definition in fp64 with torch autograd on
the CPU; its quantized weights are the oracle's bf16 W^ (bit-identical to the
library's, which the parity tests check), so what is compared is the
library's forward, input gradient and adapter gradients composed through the
block.  The block keeps its activations in bf16 between operations (about a
dozen roundings of at most 2^-9 along the longest gradient path, the
attention softmax included), hence the looser bar on gradients.
"""
import numpy as np
import pytest
import torch

import oracle_refs as R
from bit_nf4_quantized_qlora_b200 import layer as L
from bit_nf4_quantized_qlora_b200 import binding as B
from bit_nf4_quantized_qlora_b200 import workloads as WL

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL_OUT = 2e-2
TOL_GRAD = 5e-2


def _err(got: torch.Tensor, ref: torch.Tensor) -> float:
    g = got.detach().double().cpu()
    r = ref.detach().double().cpu()
    den = r.abs().max().item()
    return (g - r).abs().max().item() / den if den > 0 else (g - r).abs().max().item()


class _RefLinear(torch.nn.Module):
    def __init__(self, W_hat: np.ndarray, A: torch.Tensor, Bm: torch.Tensor, scale: float):
        super().__init__()
        self.W = torch.from_numpy(W_hat)
        self.A = torch.nn.Parameter(A.double())
        self.B = torch.nn.Parameter(Bm.double())
        self.scale = scale

    def forward(self, x):
        return x @ self.W.T + self.scale * (x @ self.A.T) @ self.B.T


def _ref_block(case, lins, x):
    b, t, h = x.shape
    d = h // case.heads

    def rms(v):
        return v * torch.rsqrt(v.pow(2).mean(-1, keepdim=True) + L.RMS_EPS)

    a = rms(x)
    q = lins["q"](a).view(b, t, case.heads, d).transpose(1, 2)
    k = lins["k"](a).view(b, t, case.heads, d).transpose(1, 2)
    v = lins["v"](a).view(b, t, case.heads, d).transpose(1, 2)
    s = (q @ k.transpose(-1, -2)) / np.sqrt(d)
    mask = torch.triu(torch.ones(t, t, dtype=torch.bool), diagonal=1)
    att = torch.softmax(s.masked_fill(mask, float("-inf")), dim=-1) @ v
    x = x + lins["o"](att.transpose(1, 2).reshape(b, t, h))
    m = rms(x)
    g, u = lins["gate"](m), lins["up"](m)
    return x + lins["down"](torch.nn.functional.silu(g) * u)


def test_qlora_linear_module_matches_oracle():
    torch.cuda.set_device(0)
    case = WL.LinearCase("module_520x640", n=520, k=640, m=96, r=16, alpha=32.0, w_seed=900, x_seed=901,
                         a_seed=902, b_seed=903, dy_seed=904)
    lin = L.QLoRALinear.from_float(case.W().to(DEV), case.A().to(DEV), case.B().to(DEV), case.alpha)
    X = case.X().to(DEV).requires_grad_(True)
    Y = lin(X)
    dY = case.dY().to(DEV)
    Y.backward(dY)
    W_hat = R.dequant_full(case.W())
    Xn, An, Bn, dYn = (R.bf16_to_f64(t) for t in (case.X(), case.A(), case.B(), case.dY()))
    assert R.err(R.bf16_to_f64(Y), R.fwd(Xn, W_hat, An, Bn, case.scale)) <= TOL_OUT
    assert R.err(R.bf16_to_f64(X.grad), R.bwd_dx(dYn, W_hat, An, Bn, case.scale)) <= TOL_OUT
    dA, dB = R.lora_grads(Xn, dYn, An, Bn, case.scale)
    assert R.err(R.bf16_to_f64(lin.A.grad), dA) <= TOL_OUT
    assert R.err(R.bf16_to_f64(lin.B.grad), dB) <= TOL_OUT


def test_decoder_block_forward_and_adapter_gradients():
    torch.cuda.set_device(0)
    case = WL.DecoderLayerCase(batch=2, seq=64, hidden=256, heads=4, mlp=704, r=16, alpha=32.0)
    block = L.build_decoder(case, torch.device(DEV))
    x = case.X().to(DEV).requires_grad_(True)
    y = block(x)
    gy = case.grad()
    y.backward(gy.to(DEV))
    torch.cuda.synchronize()

    ref_lins = {name: _RefLinear(R.dequant_full(case.W(name)), case.A(name), case.B(name), case.alpha / case.r)
                for name in L.PROJECTIONS}
    xr = case.X().double().requires_grad_(True)
    yr = _ref_block(case, ref_lins, xr)
    yr.backward(gy.double())

    errs = {"out": _err(y, yr), "dx": _err(x.grad, xr.grad)}
    for name in L.PROJECTIONS:
        errs["dA_" + name] = _err(block.lin[name].A.grad, ref_lins[name].A.grad)
        errs["dB_" + name] = _err(block.lin[name].B.grad, ref_lins[name].B.grad)
    assert errs["out"] <= TOL_OUT, errs
    assert max(errs.values()) <= TOL_GRAD, errs


def test_merged_weight_reproduces_the_forward():
    """Export: the module's merged bf16 weight W' = W^ + s B A, used in a plain
    product, gives the layer's forward (oracle, fp64) within the tolerance;
    the same holds for an FP4 module."""
    torch.cuda.set_device(0)
    for codebook, name in ((B.QLORA_CODEBOOK_NF4, "nf4"), (B.QLORA_CODEBOOK_FP4, "fp4")):
        case = WL.LinearCase("merge_module", n=520, k=640, m=96, r=16, alpha=32.0, w_seed=990, x_seed=991,
                             a_seed=992, b_seed=993, dy_seed=994)
        lin = L.QLoRALinear.from_float(case.W().to(DEV), case.A().to(DEV), case.B().to(DEV), case.alpha,
                                       codebook=codebook)
        assert lin.w.codebook == codebook
        X = case.X().to(DEV)
        Wm = lin.merged_weight()
        Y2 = (X.double() @ Wm.double().t())
        torch.cuda.synchronize()
        ref = R.fwd(R.bf16_to_f64(case.X()), R.dequant_full(case.W(), name), R.bf16_to_f64(case.A()),
                    R.bf16_to_f64(case.B()), case.scale)
        assert R.err(Y2.cpu().numpy(), ref) <= TOL_OUT
        assert lin.merged_weight(torch.float32).dtype == torch.float32
