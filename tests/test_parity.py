"""GPU parity: the CUDA path (called through the C ABI) against the oracle.

Bars: packed codes, absmax codes and group scales bit-exact; dequantized bf16
weights bit-exact; forward output, input gradient and adapter gradients within
a max-abs-normalised error of 2e-2 against the fp64 oracle on the same bf16
inputs.  Small cases span several tiles and ragged tails; the full-size
workloads are checked on sampled rows the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle_refs as R
from bit_nf4_quantized_qlora_b200 import binding as B
from bit_nf4_quantized_qlora_b200 import workloads as WL
from oracle import quant

pytestmark = pytest.mark.gpu
TOL = 2e-2
DEV = "cuda:0"


def _gpu_quant(W: torch.Tensor) -> B.NF4Weight:
    w = B.qlora_quantize_nf4_dq(W.to(DEV))
    torch.cuda.synchronize()
    return w


def _case(n, k, m, r, alpha=32.0, seed=100, w_std=0.02, outliers=0.0):
    return WL.LinearCase(f"case_{n}x{k}_m{m}_r{r}", n=n, k=k, m=m, r=r, alpha=alpha, w_std=w_std,
                         w_seed=seed, x_seed=seed + 1, a_seed=seed + 2, b_seed=seed + 3, dy_seed=seed + 4,
                         outlier_frac=outliers)


def _np(t):
    return t.detach().cpu().numpy()


# ---------------------------------------------------------------------------
# quantize / dequant: bit-exact
# ---------------------------------------------------------------------------

QUANT_SHAPES = [(1024, 1024), (72, 64), (8, 128), (136, 448), (300, 8192)]


@pytest.mark.parametrize("shape", QUANT_SHAPES, ids=lambda s: f"{s[0]}x{s[1]}")
def test_quantize_bit_exact(shape):
    n, k = shape
    W = WL.weight(n, k, 0.02, seed=7 + n, outlier_frac=0.001)
    W[0, :64] = 0.0                                   # an all-zero block
    W[1, 5] = -0.0
    w = _gpu_quant(W)
    packed, q, S = R.quantize(W)
    assert np.array_equal(_np(w.codes), packed)
    assert np.array_equal(_np(w.absmax_q), q)
    assert np.array_equal(_np(w.group_scale).view(np.uint32), S.view(np.uint32))


def test_quantize_codes_near_midpoints():
    """Weights on and within +-2 ulps of every midpoint times the block absmax,
    for 2048 random absmax values spanning 40 binades: the codes must equal the
    oracle's, which divides with IEEE round-to-nearest."""
    from oracle import nf4 as onf4
    rng = np.random.default_rng(42)
    mids = onf4.midpoints_f32()
    nblk = 2048
    c = (2.0 ** rng.uniform(-30, 10, nblk)).astype(np.float32)
    W = np.zeros((nblk, 64), dtype=np.float32)
    W[:, 0] = c                                       # the absmax element
    for b in range(nblk):
        vals = []
        for t in mids:
            base = np.float32(t * c[b])
            for d in (-2, -1, 0, 1, 2):
                v = base
                for _ in range(abs(d)):
                    v = np.nextafter(v, np.float32(np.inf if d > 0 else -np.inf))
                vals.append(v)
        vals = np.roll(np.array(vals, dtype=np.float32), -5 * (b % 15))[:63]   # all midpoints over 15 blocks
        vals = np.clip(vals, -c[b], c[b])
        W[b, 1:1 + len(vals)] = vals
    Wt = torch.from_numpy(W.reshape(256, 512))
    w = _gpu_quant(Wt)
    packed, q, S = R.quantize(Wt)
    assert np.array_equal(_np(w.codes), packed)
    assert np.array_equal(_np(w.absmax_q), q)


def test_quantize_absmax_debug_output():
    W = WL.weight(64, 1024, 0.02, seed=3)
    absmax = torch.empty(64 * 1024 // 64, dtype=torch.float32, device=DEV)
    B.qlora_quantize_nf4_dq(W.to(DEV), absmax_fp32=absmax)
    torch.cuda.synchronize()
    ref = quant.block_absmax(W.reshape(-1).numpy())
    assert np.array_equal(_np(absmax).view(np.uint32), ref.view(np.uint32))


def test_quantize_attn_proj_with_outliers_full():
    case = WL.attn_proj_7b()
    W = case.W()
    w = _gpu_quant(W)
    packed, q, S = R.quantize(W)
    assert np.array_equal(_np(w.codes), packed)
    assert np.array_equal(_np(w.absmax_q), q)
    assert np.array_equal(_np(w.group_scale).view(np.uint32), S.view(np.uint32))


def test_quantize_70b_up_proj_sampled_groups():
    case = WL.up_proj_70b()
    W = case.W()
    w = _gpu_quant(W)
    ng = w.group_scale.numel()
    rng = np.random.default_rng(0)
    groups = sorted(set(rng.choice(ng, 6, replace=False).tolist() + [0, ng - 1]))
    ref = R.quantize_groups(W, groups)
    codes = w.codes
    for g, (p, q, S) in ref.items():
        assert np.array_equal(_np(codes[g * 8192:(g + 1) * 8192]), p), g
        assert np.array_equal(_np(w.absmax_q[g * 256:(g + 1) * 256]), q), g
        assert _np(w.group_scale[g:g + 1]).view(np.uint32)[0] == S.view(np.uint32)[0]


@pytest.mark.parametrize("shape", QUANT_SHAPES + [(4096, 4096)], ids=lambda s: f"{s[0]}x{s[1]}")
def test_dequant_bit_exact(shape):
    n, k = shape
    W = WL.weight(n, k, 0.02, seed=11 + k, outlier_frac=0.001)
    w = _gpu_quant(W)
    got = B.qlora_dequant(w)
    torch.cuda.synchronize()
    packed, q, S = R.quantize(W)
    ref_bits = quant.dequant_bf16_bits(packed, q, S)
    assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1), ref_bits)


# ---------------------------------------------------------------------------
# forward, input gradient, adapter gradients on small and ragged shapes
# ---------------------------------------------------------------------------

FWD_CASES = [
    # weight-streaming paths (m <= 16); m <= 4 takes the direct-load kernel: K ragged in chunks of
    # four blocks, groups changing inside a chunk, n % 16 == 8, clusters of 3, 5 and 8 CTAs, and
    # one K beyond a cluster's warps (back on the TMA-ring kernel)
    (1024, 1024, 16, 16), (1024, 1024, 1, 16), (72, 320, 3, 16), (264, 1088, 7, 0), (4096, 1024, 16, 64),
    (264, 1088, 4, 0), (1032, 8256, 2, 32), (136, 16448, 1, 16), (24, 32768, 4, 16), (16, 33024, 1, 16),
    # tcgen05 path: several tiles plus ragged tails in m and n, k a few k-steps
    (520, 640, 200, 16), (264, 192, 17, 0), (1024, 1024, 300, 64), (256, 64, 130, 32), (776, 512, 129, 16),
]


def _inputs(case):
    W = case.W()
    X = case.X()
    A = case.A() if case.r else None
    Bm = case.B() if case.r else None
    return W, X, A, Bm


@pytest.mark.parametrize("nkmr", FWD_CASES, ids=lambda c: "n%d_k%d_m%d_r%d" % c)
def test_fwd_parity(nkmr):
    n, k, m, r = nkmr
    case = _case(n, k, m, r)
    W, X, A, Bm = _inputs(case)
    w = _gpu_quant(W)
    Y = B.qlora_linear_fwd(X.to(DEV), w, A.to(DEV) if r else None, Bm.to(DEV) if r else None, r, case.scale)
    torch.cuda.synchronize()
    W_hat = R.dequant_full(W)
    ref = R.fwd(R.bf16_to_f64(X), W_hat, R.bf16_to_f64(A) if r else None, R.bf16_to_f64(Bm) if r else None,
                case.scale)
    e = R.err(R.bf16_to_f64(Y), ref)
    assert e <= TOL, e


BWD_CASES = [(1024, 1024, 16, 16), (520, 640, 200, 16), (1024, 1024, 300, 64), (264, 192, 5, 0),
             (776, 512, 129, 32)]


@pytest.mark.parametrize("nkmr", BWD_CASES, ids=lambda c: "n%d_k%d_m%d_r%d" % c)
def test_bwd_dx_parity(nkmr):
    n, k, m, r = nkmr
    case = _case(n, k, m, r, seed=300)
    W, _, A, Bm = _inputs(case)
    dY = case.dY()
    w = _gpu_quant(W)
    dX = B.qlora_linear_bwd_dx(dY.to(DEV), w, A.to(DEV) if r else None, Bm.to(DEV) if r else None, r,
                               case.scale)
    torch.cuda.synchronize()
    W_hat = R.dequant_full(W)
    ref = R.bwd_dx(R.bf16_to_f64(dY), W_hat, R.bf16_to_f64(A) if r else None,
                   R.bf16_to_f64(Bm) if r else None, case.scale)
    e = R.err(R.bf16_to_f64(dX), ref)
    assert e <= TOL, e


LORA_CASES = [(1024, 1024, 16, 16), (520, 640, 200, 32), (1024, 1024, 300, 64), (264, 192, 1, 16)]


@pytest.mark.parametrize("nkmr", LORA_CASES, ids=lambda c: "n%d_k%d_m%d_r%d" % c)
def test_lora_grads_parity(nkmr):
    n, k, m, r = nkmr
    case = _case(n, k, m, r, seed=500)
    X, dY, A, Bm = case.X(), case.dY(), case.A(), case.B()
    dA, dB = B.qlora_lora_bwd(X.to(DEV), dY.to(DEV), A.to(DEV), Bm.to(DEV), r, case.scale)
    torch.cuda.synchronize()
    rA, rB = R.lora_grads(R.bf16_to_f64(X), R.bf16_to_f64(dY), R.bf16_to_f64(A), R.bf16_to_f64(Bm), case.scale)
    assert R.err(R.bf16_to_f64(dA), rA) <= TOL
    assert R.err(R.bf16_to_f64(dB), rB) <= TOL


def test_lora_grads_empty_batch_writes_zeros():
    dA = torch.full((16, 128), 3.0, dtype=torch.bfloat16, device=DEV)
    dB = torch.full((64, 16), 3.0, dtype=torch.bfloat16, device=DEV)
    X = torch.empty(0, 128, dtype=torch.bfloat16, device=DEV)
    dY = torch.empty(0, 64, dtype=torch.bfloat16, device=DEV)
    A = torch.zeros(16, 128, dtype=torch.bfloat16, device=DEV)
    Bm = torch.zeros(64, 16, dtype=torch.bfloat16, device=DEV)
    B.qlora_lora_bwd(X, dY, A, Bm, 16, 2.0, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0


def test_fwd_empty_batch_leaves_output_untouched():
    W = WL.weight(64, 128, 0.02, seed=1)
    w = _gpu_quant(W)
    Y = torch.full((0, 64), 1.0, dtype=torch.bfloat16, device=DEV)
    X = torch.empty(0, 128, dtype=torch.bfloat16, device=DEV)
    B.qlora_linear_fwd(X, w, out=Y)
    torch.cuda.synchronize()


def test_single_row_equals_row_of_batch_on_gpu():
    """The weight-streaming path at m=1 and the same row inside an m=16 call
    agree to within the tolerance (both are the same product)."""
    case = _case(1024, 1024, 16, 16, seed=900)
    W, X, A, Bm = _inputs(case)
    w = _gpu_quant(W)
    Xd, Ad, Bd = X.to(DEV), A.to(DEV), Bm.to(DEV)
    Y16 = B.qlora_linear_fwd(Xd, w, Ad, Bd, 16, case.scale)
    Y1 = B.qlora_linear_fwd(Xd[5:6].contiguous(), w, Ad, Bd, 16, case.scale)
    torch.cuda.synchronize()
    assert R.err(R.bf16_to_f64(Y1), R.bf16_to_f64(Y16[5:6])) <= 1e-2


# ---------------------------------------------------------------------------
# full-size workloads, sampled
# ---------------------------------------------------------------------------

def _sampled_check(case, m, rows, xs, check_bwd=True, check_grads=True):
    """Run the full-size launch, compare sampled entries with the oracle.

    Forward: Y[xs, rows] needs only the sampled weight rows.  Input gradient:
    the launch is full size with dY zero outside the sampled columns `rows`,
    so dX[xs, :] again needs only those weight rows.  Adapter gradients: the
    full dA, and the sampled rows of dB."""
    W = case.W()
    w = _gpu_quant(W)
    X = case.X(m)
    A, Bm = case.A(), case.B()
    Xd, Ad, Bd = X.to(DEV), A.to(DEV), Bm.to(DEV)
    Y = B.qlora_linear_fwd(Xd, w, Ad, Bd, case.r, case.scale)
    torch.cuda.synchronize()
    W_rows = R.dequant_rows(W, rows)                      # [len(rows) x k]
    Af, Bf = R.bf16_to_f64(A), R.bf16_to_f64(Bm)
    ref = R.fwd(R.bf16_to_f64(X[xs]), W_rows, Af, Bf[rows], case.scale)
    assert R.err(R.bf16_to_f64(Y[xs][:, rows]), ref) <= TOL
    del Y
    if not check_bwd:
        return
    dY = case.dY(m)
    dY_z = torch.zeros_like(dY)
    dY_z[:, rows] = dY[:, rows]
    dX = B.qlora_linear_bwd_dx(dY_z.to(DEV), w, Ad, Bd, case.r, case.scale)
    torch.cuda.synchronize()
    ref_dx = R.bwd_dx(R.bf16_to_f64(dY_z[xs][:, rows]), W_rows, Af, Bf[rows], case.scale)
    assert R.err(R.bf16_to_f64(dX[xs]), ref_dx) <= TOL
    del dX
    if not check_grads:
        return
    dA, dB = B.qlora_lora_bwd(Xd, dY.to(DEV), Ad, Bd, case.r, case.scale)
    torch.cuda.synchronize()
    Xf, dYf = R.bf16_to_f64(X), R.bf16_to_f64(dY)
    rA, _ = R.lora_grads(Xf, dYf, Af, Bf, case.scale)
    _, rB_rows = R.lora_grads(Xf, dYf[:, rows], Af, Bf[rows], case.scale)
    assert R.err(R.bf16_to_f64(dA), rA) <= TOL
    assert R.err(R.bf16_to_f64(dB)[rows], rB_rows) <= TOL


def _rows(n, count, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.choice(n, count, replace=False), [0, n - 1]]))


@pytest.mark.parametrize("which", ["gate", "down"])
def test_mlp_7b_full_size_sampled(which):
    case = WL.mlp_7b(which)
    rows = _rows(case.n, 48, 1)
    xs = _rows(case.m, 24, 2)
    _sampled_check(case, case.m, rows, xs, check_bwd=True, check_grads=True)


@pytest.mark.parametrize("m", list(WL.M_SWEEP_70B))
def test_up_proj_70b_sampled(m):
    """70B up-projection at every M of its sweep: forward and input gradient
    on sampled rows (adapter gradients at M = 1024)."""
    case = WL.up_proj_70b(m)
    rows = _rows(case.n, 32, 3)
    xs = _rows(m, min(m, 8), 4)
    _sampled_check(case, m, rows, xs, check_bwd=True, check_grads=(m == 1024))


@pytest.mark.parametrize("m", WL.M_SWEEP_ATTN)
def test_attn_proj_7b_decode(m):
    case = WL.attn_proj_7b(m)
    W, X, A, Bm = _inputs(case)
    w = _gpu_quant(W)
    Y = B.qlora_linear_fwd(X.to(DEV), w, A.to(DEV), Bm.to(DEV), case.r, case.scale)
    torch.cuda.synchronize()
    ref = R.fwd(R.bf16_to_f64(X), R.dequant_full(W), R.bf16_to_f64(A), R.bf16_to_f64(Bm), case.scale)
    assert R.err(R.bf16_to_f64(Y), ref) <= TOL


def test_no_device_timeouts_recorded():
    assert B.qlora_poll_device_error() == 0


@pytest.mark.parametrize("nkmr", [(1024, 1024, 16, 16), (520, 640, 200, 32), (776, 1088, 300, 256), (264, 192, 1, 16)],
                         ids=lambda c: "n%d_k%d_m%d_r%d" % c)
@pytest.mark.parametrize("reuse_t", [True, False], ids=["T_from_forward", "T_recomputed"])
def test_linear_bwd_parity(nkmr, reuse_t):
    """qlora_linear_bwd (dX, dA, dB in one call, U formed once, T from the
    forward's workspace or recomputed) against the oracle."""
    n, k, m, r = nkmr
    case = _case(n, k, m, r, seed=1500)
    W, X, A, Bm = _inputs(case)
    dY = case.dY()
    w = _gpu_quant(W)
    Xd, Ad, Bd, dYd = X.to(DEV), A.to(DEV), Bm.to(DEV), dY.to(DEV)
    ws = torch.empty(B.qlora_workspace_bytes(B.QLORA_OP_FWD, m, n, k, r), dtype=torch.uint8, device=DEV)
    B.qlora_linear_fwd(Xd, w, Ad, Bd, r, case.scale, ws=ws)
    T = ws[:m * r * 2].view(torch.bfloat16).view(m, r) if reuse_t else None
    dX, dA, dB = B.qlora_linear_bwd(dYd, Xd, w, Ad, Bd, r, case.scale, T=T)
    _, dA2, dB2 = B.qlora_linear_bwd(dYd, Xd, w, Ad, Bd, r, case.scale, T=T, want_dx=False)
    torch.cuda.synchronize()
    W_hat = R.dequant_full(W)
    Xf, Af, Bf, dYf = (R.bf16_to_f64(t) for t in (X, A, Bm, dY))
    assert R.err(R.bf16_to_f64(dX), R.bwd_dx(dYf, W_hat, Af, Bf, case.scale)) <= TOL
    rA, rB = R.lora_grads(Xf, dYf, Af, Bf, case.scale)
    for a, b in ((dA, dB), (dA2, dB2)):
        assert R.err(R.bf16_to_f64(a), rA) <= TOL
        assert R.err(R.bf16_to_f64(b), rB) <= TOL
