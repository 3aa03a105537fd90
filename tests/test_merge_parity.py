"""GPU parity of the adapter merge W' = W^ + s . B . A against the oracle.

Bars (the merge is floating point, so not bit-exact; the bounds follow from
its arithmetic): the fp32 export within E = (r + 2) fp32 rounding steps of the
absolute sum |W^| + s Sum|B A| (r exact products summed in fp32, then one fused
multiply-add); the bf16 export, its bf16 rounding, within one bf16 ulp of the
exact merged value plus E (E matters only where W^ and s B A nearly cancel and
the merged value is small); r = 0 returns W^ exactly.  Shapes cover ragged
row tiles (n % 64 != 0), a half column tile (k % 128 == 64), ranks 16 .. 256
and the FP4 and INT4 codebooks; the fp32 export re-quantizes bit-exactly like
the oracle quantizing the same values.
"""
import numpy as np
import pytest
import torch

import oracle_refs as R
from bit_nf4_quantized_qlora_b200 import binding as B
from bit_nf4_quantized_qlora_b200 import workloads as WL
from oracle import merge, quant

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

# Ragged row and column tiles (tiles are 128 x 256), every rank-slab count of
# the tensor-core kernel (ranks 16..64: one slab; 128, 192, 256: two to four
# slabs through the same operand buffers), the three codebooks.
CASES = [(520, 576, 16, "nf4"), (1024, 1024, 64, "nf4"), (136, 448, 32, "fp4"), (64, 128, 256, "int4"),
         (4104, 4096, 64, "nf4"), (300, 704, 128, "nf4"), (264, 320, 192, "fp4")]


def _setup(n, k, r, name, seed=950):
    case = WL.LinearCase(f"merge_{n}x{k}_r{r}", n=n, k=k, m=1, r=r, alpha=2.0 * r, w_seed=seed, x_seed=seed + 1,
                         a_seed=seed + 2, b_seed=seed + 3, dy_seed=seed + 4)
    W = case.W()
    w = B.qlora_quantize_4bit_dq(W.to(DEV), B.CODEBOOKS[name])
    W_hat = R.dequant_full(W, name)
    A = case.A() if r else None
    Bm = case.B() if r else None
    return case, w, W_hat, A, Bm


def _bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (normal range): 2^(floor(log2|x|) - 7)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


@pytest.mark.parametrize("nkr", CASES, ids=lambda c: "n%d_k%d_r%d_%s" % c)
def test_merge_exports_match_the_oracle(nkr):
    n, k, r, name = nkr
    case, w, W_hat, A, Bm = _setup(n, k, r, name)
    got_h, got_f = B.qlora_merge_adapter(w, A.to(DEV), Bm.to(DEV), r, case.scale, want_bf16=True, want_f32=True)
    torch.cuda.synchronize()
    An, Bn = R.bf16_to_f64(A), R.bf16_to_f64(Bm)
    ref = merge.merge_f64(W_hat, An, Bn, case.scale)
    bound = (r + 2) * 2.0 ** -24 * (np.abs(W_hat) + abs(case.scale) * (np.abs(Bn) @ np.abs(An))) + 2.0 ** -149
    gf = got_f.double().cpu().numpy()
    assert np.all(np.abs(gf - ref) <= bound), np.max(np.abs(gf - ref) / bound)
    gh = R.bf16_to_f64(got_h)
    assert np.all(np.abs(gh - ref) <= _bf16_ulp(ref) + bound), np.max(np.abs(gh - ref) / (_bf16_ulp(ref) + bound))
    # the bf16 export is the bf16 rounding of the fp32 export
    assert np.array_equal(quant.bf16_rne_bits(got_f.cpu().numpy()).reshape(-1),
                          got_h.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1))


@pytest.mark.parametrize("only", ["bf16", "f32"])
def test_merge_single_output(only):
    case, w, W_hat, A, Bm = _setup(264, 576, 32, "nf4", seed=960)
    h, f = B.qlora_merge_adapter(w, A.to(DEV), Bm.to(DEV), 32, case.scale, want_bf16=only == "bf16",
                                 want_f32=only == "f32")
    torch.cuda.synchronize()
    An, Bn = R.bf16_to_f64(A), R.bf16_to_f64(Bm)
    ref = merge.merge_f64(W_hat, An, Bn, case.scale)
    bound = 34 * 2.0 ** -24 * (np.abs(W_hat) + abs(case.scale) * (np.abs(Bn) @ np.abs(An))) + 2.0 ** -149
    if only == "bf16":
        assert f is None
        assert np.all(np.abs(R.bf16_to_f64(h) - ref) <= _bf16_ulp(ref) + bound)
    else:
        assert h is None
        assert np.max(np.abs(f.double().cpu().numpy() - ref)) <= 1e-5 * np.max(np.abs(ref))


@pytest.mark.parametrize("name", ["nf4", "fp4"])
def test_zero_rank_returns_the_dequantized_base(name):
    _, w, W_hat, _, _ = _setup(200, 640, 0, name, seed=970)
    h, f = B.qlora_merge_adapter(w, None, None, 0, 0.0, want_bf16=True, want_f32=True)
    deq = B.qlora_dequant(w)
    torch.cuda.synchronize()
    assert torch.equal(h.view(torch.int16), deq.view(torch.int16))
    assert np.array_equal(f.cpu().numpy().astype(np.float64), W_hat)


def test_fp32_export_requantizes_like_the_oracle():
    """Export path: merged fp32 -> a new 4-bit checkpoint with the library's
    quantizer, bit-exact against the oracle quantizing the same fp32 values."""
    case, w, _, A, Bm = _setup(256, 1024, 16, "nf4", seed=980)
    _, f = B.qlora_merge_adapter(w, A.to(DEV), Bm.to(DEV), 16, case.scale, want_bf16=False, want_f32=True)
    w2 = B.qlora_quantize_nf4_dq(f)
    torch.cuda.synchronize()
    packed, q, S, _ = quant.quantize_nf4_dq(f.cpu().numpy().reshape(-1))
    assert np.array_equal(w2.codes.cpu().numpy(), packed)
    assert np.array_equal(w2.absmax_q.cpu().numpy(), q)
    assert np.array_equal(w2.group_scale.cpu().numpy().view(np.uint32), S.view(np.uint32))
