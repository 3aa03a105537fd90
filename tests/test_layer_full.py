"""The 7B-shaped decoder block at its own size (hidden 4096, 32 heads, MLP
11008, X [2 x 2048 x 4096], LoRA r = 64, alpha = 16), one forward + backward,
with every one of its seven QLoRA projection calls checked against the
oracle on the bf16 tensors that call actually received.

Comparing the block output with an fp64 rendering of the whole block mixes
the library's error with the bf16 roundings of the PyTorch operations between
the projections.  Here each call is isolated instead: its input X, its output
Y, the upstream gradient dY it was given and the dX, dA, dB it returned are
recorded, and the oracle recomputes Y, dX, dA and dB from the same X, dY and
adapters, all at the 2e-2 bar (Y and dX on sampled rows, dA in full, dB on
sampled rows).  At this size the forward takes the large-M fused kernel.
"""
import numpy as np
import pytest
import torch

import oracle_refs as R
from bit_nf4_quantized_qlora_b200 import layer as L
from bit_nf4_quantized_qlora_b200 import workloads as WL
from oracle import linear

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TOL = 2e-2


class _Recorded(torch.autograd.Function):
    """The library's forward and backward, with the call's tensors kept."""

    @staticmethod
    def forward(ctx, X, A, Bm, w, r, scale, rec):
        Y = L.QLoRALinearFunction.forward(ctx, X, A, Bm, w, r, scale)
        rec["X"], rec["Y"] = X.detach().clone(), Y.detach().clone()
        ctx.rec = rec
        return Y

    @staticmethod
    def backward(ctx, dY):
        dX, dA, dB, _, _, _ = L.QLoRALinearFunction.backward(ctx, dY)
        ctx.rec.update(dY=dY.detach().contiguous().clone(), dX=dX.detach().clone(), dA=dA.detach().clone(),
                       dB=dB.detach().clone())
        return dX, dA, dB, None, None, None, None


def test_each_projection_of_the_full_size_block_matches_the_oracle():
    torch.cuda.set_device(0)
    case = WL.DecoderLayerCase()
    block = L.build_decoder(case, DEV)
    recs = {name: {} for name in L.PROJECTIONS}
    for name, lin in block.lin.items():
        def fwd(x, lin=lin, rec=recs[name]):
            lead = x.shape[:-1]
            y = _Recorded.apply(x.reshape(-1, x.shape[-1]).contiguous(), lin.A, lin.B, lin.w, lin.r, lin.scale, rec)
            return y.reshape(*lead, lin.w.n)
        lin.forward = fwd
    x = case.X().to(DEV).requires_grad_(True)
    block(x).backward(case.grad().to(DEV))
    torch.cuda.synchronize()

    rng = np.random.default_rng(5)
    tokens = case.batch * case.seq
    xs = np.unique(np.concatenate([rng.choice(tokens, 16, replace=False), [0, tokens - 1]]))
    for name in L.PROJECTIONS:
        rec, lin = recs[name], block.lin[name]
        n, k = case.proj_shape(name)
        W_hat = R.dequant_full(case.W(name))
        A, Bm = R.bf16_to_f64(lin.A), R.bf16_to_f64(lin.B)
        s = lin.scale
        X = R.bf16_to_f64(rec["X"])
        dY = R.bf16_to_f64(rec["dY"])
        assert X.shape == (tokens, k) and dY.shape == (tokens, n)
        e_y = R.err(R.bf16_to_f64(rec["Y"][xs]), linear.fwd(X[xs], W_hat, A, Bm, s))
        e_dx = R.err(R.bf16_to_f64(rec["dX"][xs]), linear.bwd_dx(dY[xs], W_hat, A, Bm, s))
        rA, _ = linear.lora_grads(X, dY, A, Bm, s)
        cols = np.unique(np.concatenate([rng.choice(n, 64, replace=False), [0, n - 1]]))
        _, rB = linear.lora_grads(X, dY[:, cols], A, Bm[cols], s)
        e_da = R.err(R.bf16_to_f64(rec["dA"]), rA)
        e_db = R.err(R.bf16_to_f64(rec["dB"][cols]), rB)
        assert max(e_y, e_dx, e_da, e_db) <= TOL, (name, e_y, e_dx, e_da, e_db)
        del W_hat, X, dY
