"""The QLoRA linear layer as a torch autograd function, and the 7B-shaped
decoder block used to measure it inside a transformer layer.

The frozen base weight is held only in its NF4 + double-quant form and the
adapters A [r x k], B [n x r] are bf16 parameters ("QLoRA and Quantized
Training", The idea; "QLoRA", Follow one QLoRA training step): the forward is
one ``qlora_linear_fwd`` and the backward one ``qlora_linear_bwd`` (input
gradient and adapter gradients, reusing the forward's rank-r intermediate),
all in libqlora's kernels.  The rest of the decoder block (RMSNorm, causal
attention, SiLU gating, residual adds) is plain PyTorch: it is not part of
the quantized layer, and the pages leave it to the host framework.
"""
from typing import Dict

import torch
import torch.nn.functional as F

from . import binding as B


class QLoRALinearFunction(torch.autograd.Function):
    """Y = X . dequant(W)^T + s (X A^T) B^T for X [m x k] (bf16, contiguous)."""

    @staticmethod
    def forward(ctx, X: torch.Tensor, A: torch.Tensor, Bm: torch.Tensor, w: B.NF4Weight, r: int, scale: float):
        m = X.shape[0]
        ws = torch.empty(max(1, B.qlora_workspace_bytes(B.QLORA_OP_FWD, m, w.n, w.k, r)), dtype=torch.uint8,
                         device=X.device)
        Y = B.qlora_linear_fwd(X, w, A, Bm, r, scale, ws=ws)
        # The forward leaves T = bf16(s X A^T) at the start of its workspace;
        # the backward takes it instead of recomputing it.
        T = ws[:m * r * 2].view(torch.bfloat16).view(m, r) if r > 0 and m > 0 else None
        ctx.save_for_backward(X, A, Bm, T)
        ctx.w, ctx.r, ctx.scale = w, r, scale
        return Y

    @staticmethod
    def backward(ctx, dY: torch.Tensor):
        X, A, Bm, T = ctx.saved_tensors
        dY = dY.contiguous()
        dX, dA, dB = B.qlora_linear_bwd(dY, X, ctx.w, A, Bm, ctx.r, ctx.scale, T=T,
                                        want_dx=ctx.needs_input_grad[0])
        return dX, dA, dB, None, None, None


class QLoRALinear(torch.nn.Module):
    """A frozen NF4 weight [n x k] with trainable bf16 adapters (rank r, s = alpha / r)."""

    def __init__(self, w: B.NF4Weight, A: torch.Tensor, Bm: torch.Tensor, alpha: float):
        super().__init__()
        self.w = w
        self.r = A.shape[0]
        self.scale = alpha / self.r
        self.A = torch.nn.Parameter(A.to(torch.bfloat16).contiguous())
        self.B = torch.nn.Parameter(Bm.to(torch.bfloat16).contiguous())

    @classmethod
    def from_float(cls, W: torch.Tensor, A: torch.Tensor, Bm: torch.Tensor, alpha: float,
                   codebook: int = B.QLORA_CODEBOOK_NF4) -> "QLoRALinear":
        """Quantize an fp32 weight [n x k] on its device (libqlora's quantize
        kernel), NF4 unless another codebook (B.QLORA_CODEBOOK_*) is named."""
        return cls(B.qlora_quantize_4bit_dq(W.float().contiguous(), codebook), A, Bm, alpha)

    @torch.no_grad()
    def merged_weight(self, dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
        """W' = W^ + s . B . A [n x k] (bf16 or fp32) for export or serving
        without the adapter (libqlora's merge kernel)."""
        want_f32 = dtype == torch.float32
        h, f = B.qlora_merge_adapter(self.w, self.A.detach(), self.B.detach(), self.r, self.scale,
                                     want_bf16=not want_f32, want_f32=want_f32)
        return f if want_f32 else h

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        y = QLoRALinearFunction.apply(x.reshape(-1, x.shape[-1]).contiguous(), self.A, self.B, self.w, self.r,
                                      self.scale)
        return y.reshape(*lead, self.w.n)


RMS_EPS = 1e-5
PROJECTIONS = ("q", "k", "v", "o", "gate", "up", "down")


def rms_norm(x: torch.Tensor, eps: float = RMS_EPS) -> torch.Tensor:
    xf = x.float()
    return (xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + eps)).to(x.dtype)


class DecoderLayer(torch.nn.Module):
    """Pre-norm decoder block with seven QLoRA projections: attention
    (q, k, v, o; causal, no positional rotation) and a SwiGLU MLP
    (gate, up, down).  The RMSNorm gains are 1 (frozen)."""

    def __init__(self, heads: int, linears: Dict[str, QLoRALinear]):
        super().__init__()
        self.heads = heads
        self.lin = torch.nn.ModuleDict(linears)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        b, t, h = x.shape
        d = h // self.heads
        a = rms_norm(x)
        q = self.lin["q"](a).view(b, t, self.heads, d).transpose(1, 2)
        k = self.lin["k"](a).view(b, t, self.heads, d).transpose(1, 2)
        v = self.lin["v"](a).view(b, t, self.heads, d).transpose(1, 2)
        att = F.scaled_dot_product_attention(q, k, v, is_causal=True)
        x = x + self.lin["o"](att.transpose(1, 2).reshape(b, t, h))
        m = rms_norm(x)
        g = self.lin["gate"](m)
        u = self.lin["up"](m)
        return x + self.lin["down"](F.silu(g) * u)


def build_decoder(case, device: torch.device) -> DecoderLayer:
    """Quantize the seven fp32 weights of a decoder workload (see
    ``workloads.DecoderLayerCase``) on `device` and attach its adapters."""
    lins = {}
    for name in PROJECTIONS:
        lins[name] = QLoRALinear.from_float(case.W(name).to(device), case.A(name).to(device),
                                            case.B(name).to(device), case.alpha)
    return DecoderLayer(case.heads, lins)


def linear_flops(case, tokens: int) -> Dict[str, float]:
    """Algorithmic FLOPs of the seven quantized projections for `tokens` rows:
    forward 2mnk + 2mr(n+k), input gradient the same, adapter gradients
    2mr(n+2k) + 2mnr."""
    fwd = bwd = grads = 0.0
    for name in PROJECTIONS:
        n, k = case.proj_shape(name)
        m, r = tokens, case.r
        fwd += 2 * m * n * k + 2 * m * r * (n + k)
        bwd += 2 * m * n * k + 2 * m * r * (n + k)
        grads += 2 * m * r * (n + 2 * k) + 2 * m * n * r
    return {"fwd": fwd, "bwd_dx": bwd, "lora_grads": grads, "total": fwd + bwd + grads}
