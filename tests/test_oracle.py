"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than its own formula:
invariants of the NF4 construction, a library routine (torch's bf16 cast,
scipy's normal CDF), brute force on tiny inputs, exact special cases, error
bounds, finite differences, and the memory figures the pages print
(``tests/golden/memory_arithmetic.json``).  No GPU is used.
"""
import json
import os

import numpy as np
import pytest
import torch
from scipy import special

from oracle import linear, memory, nf4, quant

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# NF4 levels: "16 levels at the quantiles of a standard normal, equal mass per
# bin, dense near zero" (QLoRA and Quantized Training, 'The idea'; attention.sh
# figure 3), plus an exact zero and the endpoints +-1.
# ---------------------------------------------------------------------------

def test_nf4_sixteen_sorted_levels_with_exact_zero_and_endpoints():
    lv = nf4.levels_f32()
    assert lv.dtype == np.float32 and lv.shape == (16,)
    assert np.all(np.diff(lv.astype(np.float64)) > 0)
    assert lv[7] == np.float32(0.0)
    assert lv[0] == np.float32(-1.0) and lv[15] == np.float32(1.0)
    assert np.sum(lv < 0) == 7 and np.sum(lv > 0) == 8


def test_nf4_equal_normal_mass_within_each_half():
    """Map the levels back through the normal CDF (scipy, an independent
    implementation): above zero the probabilities are equally spaced by
    (o - 1/2)/8, below zero by (o - 1/2)/7, and the extreme sits at o."""
    o = nf4.TAIL_P
    z_top = special.ndtri(o)
    p = special.ndtr(nf4.levels_f64() * z_top)
    pos = np.sort(p[p > 0.5 + 1e-15])
    neg = np.sort(1.0 - p[p < 0.5 - 1e-15])
    assert pos.size == 8 and neg.size == 7
    assert np.allclose(np.diff(pos), (o - 0.5) / 8, rtol=0, atol=1e-12)
    assert np.allclose(np.diff(neg), (o - 0.5) / 7, rtol=0, atol=1e-12)
    assert abs(pos[-1] - o) < 1e-12 and abs(neg[-1] - o) < 1e-12
    assert abs(pos[0] - (0.5 + (o - 0.5) / 8)) < 1e-12


def test_nf4_dense_near_zero_sparse_in_tails():
    lv = nf4.levels_f64()
    gaps = np.diff(lv)
    pos_gaps = gaps[7:]
    neg_gaps = gaps[:7][::-1]
    assert np.all(np.diff(pos_gaps) > 0)
    assert np.all(np.diff(neg_gaps) > 0)


def test_nf4_midpoints_lie_between_levels():
    lv = nf4.levels_f32().astype(np.float64)
    t = nf4.midpoints_f32().astype(np.float64)
    assert t.shape == (15,)
    assert np.all(t > lv[:-1]) and np.all(t < lv[1:])
    assert np.all(np.abs(t - 0.5 * (lv[:-1] + lv[1:])) <= 1e-7)


# ---------------------------------------------------------------------------
# bf16 rounding against torch's cast.
# ---------------------------------------------------------------------------

def test_bf16_rne_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 0.02,
        rng.standard_normal(20000).astype(np.float32) * 1e3,
        np.float32([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40, -1e-40]),
    ])
    # exact halfway cases, both parities of the kept bit
    mant = rng.integers(0, 1 << 7, 4000).astype(np.uint32) << np.uint32(16)
    expo = rng.integers(100, 150, 4000).astype(np.uint32) << np.uint32(23)
    base = mant | expo
    halves = (base | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, halves, -halves])
    ours = quant.bf16_rne_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ---------------------------------------------------------------------------
# Quantize: absmax, codes (brute force nearest level), packing, DQ.
# ---------------------------------------------------------------------------

def _brute_force_codes(w_flat):
    """Per element with pure Python: c = max |w| over its block of 64;
    x = fp32(w / c); the code is the index of the nearest fp32 level (in
    exact arithmetic), except that a value exactly on an fp32 midpoint takes
    the lower index; c == 0 gives code 7."""
    lv = [float(v) for v in nf4.levels_f32()]
    mids = [float(v) for v in nf4.midpoints_f32()]
    w = np.asarray(w_flat, dtype=np.float32)
    out = []
    for b in range(w.size // 64):
        blk = w[b * 64:(b + 1) * 64]
        c = max(abs(float(v)) for v in blk)
        for v in blk:
            if c == 0.0:
                out.append(7)
                continue
            x = float(np.float32(np.float32(v) / np.float32(c)))
            if x in mids:
                out.append(mids.index(x))
                continue
            d = [abs(x - l) for l in lv]
            out.append(int(min(range(16), key=lambda i: (d[i], i))))
    return np.array(out, dtype=np.uint8)


def test_block_absmax_brute_force():
    rng = np.random.default_rng(1)
    w = rng.standard_normal(64 * 37).astype(np.float32)
    ref = [max(abs(float(v)) for v in w[i * 64:(i + 1) * 64]) for i in range(37)]
    assert np.array_equal(quant.block_absmax(w), np.float32(ref))


def test_codes_are_nearest_level_brute_force():
    rng = np.random.default_rng(2)
    w = (rng.standard_normal(64 * 24) * 0.02).astype(np.float32)
    w[5] = 0.0
    w[6] = -0.0
    w[64 * 3:64 * 4] = 0.0                        # an all-zero block
    w[64 * 5 + 7] = 0.2                           # 10-sigma outlier
    w[64 * 6 + 1] = -0.2
    c = quant.block_absmax(w)
    assert np.array_equal(quant.nf4_codes(w, c), _brute_force_codes(w))


def test_codes_on_exact_midpoints_take_lower_index_and_extremes():
    mids = nf4.midpoints_f32()
    blk = np.zeros(64, dtype=np.float32)
    blk[0] = 1.0                                  # absmax 1: x = w exactly
    blk[1:16] = mids
    blk[16] = -1.0
    blk[17] = np.nextafter(mids[3], np.float32(1))
    codes = quant.nf4_codes(blk, quant.block_absmax(blk))
    assert codes[0] == 15 and codes[16] == 0
    assert list(codes[1:16]) == list(range(15))
    assert codes[17] == 4
    assert np.all(codes[18:] == 7)


def test_pack_order_even_element_in_high_nibble():
    codes = np.array([1, 2, 3, 4, 15, 0, 7, 9], dtype=np.uint8)
    packed = quant.pack_codes(codes)
    assert list(packed) == [0x12, 0x34, 0xF0, 0x79]
    assert np.array_equal(quant.unpack_codes(packed), codes)


def test_double_quant_error_within_half_step():
    """Linear unsigned 8-bit codes over [0, S_g]: the reconstructed absmax is
    within half a step S_g/510 of the original (plus fp32 rounding), the group
    maximum maps to 255, and q never exceeds 255."""
    rng = np.random.default_rng(3)
    c = np.abs(rng.standard_normal(256 * 5 + 77)).astype(np.float32) * 0.05
    c[256 * 2:256 * 2 + 256] = 0.0                # an all-zero group
    q, S = quant.double_quantize(c)
    assert S.size == 6
    cp = quant.absmax_dequant(q, S).astype(np.float64)
    for g in range(6):
        sl = slice(g * 256, (g + 1) * 256)
        sg = float(S[g])
        assert sg == float(np.max(c[sl]))
        if sg == 0.0:
            assert np.all(q[sl] == 0) and np.all(cp[sl] == 0.0)
            continue
        assert q[sl].max() == 255
        err = np.abs(cp[sl] - c[sl].astype(np.float64))
        assert np.all(err <= sg / 510.0 * (1 + 1e-6) + 4 * np.finfo(np.float32).eps * sg)


def test_double_quant_codes_brute_force_rounding():
    """q is the integer nearest to 255 * fp32(c / S_g), ties to even."""
    rng = np.random.default_rng(4)
    c = np.abs(rng.standard_normal(700)).astype(np.float32)
    q, S = quant.double_quantize(c)
    for i, ci in enumerate(c):
        sg = np.float32(S[i // 256])
        y = float(np.float32(np.float32(ci / sg) * np.float32(255.0)))
        lo = int(np.floor(y))
        frac = y - lo
        want = lo + 1 if (frac > 0.5 or (frac == 0.5 and lo % 2 == 1)) else lo
        assert q[i] == want


def test_quantize_dequant_lossless_on_levels_times_power_of_two():
    """w = L[i] * 2^e with every block's absmax exactly 2^e: the group scale is
    2^e, every absmax code is 255, c' == c, and quantize -> dequantize returns
    w exactly in fp32 (the bf16 cast is then the only rounding)."""
    rng = np.random.default_rng(5)
    lv = nf4.levels_f32()
    e = -6
    nblk = 256 * 2 + 40
    idx = rng.integers(0, 16, size=(nblk, 64)).astype(np.uint8)
    idx[:, 0] = rng.choice([0, 15], size=nblk)
    w = (lv[idx] * np.float32(2.0 ** e)).astype(np.float32).reshape(-1)
    packed, q, S, c = quant.quantize_nf4_dq(w)
    assert np.all(c == np.float32(2.0 ** e))
    assert np.all(q == 255)
    assert np.array_equal(quant.unpack_codes(packed), idx.reshape(-1))
    back = quant.dequant_f32(packed, q, S)
    assert np.array_equal(back, w)
    assert np.array_equal(quant.dequant_bf16_bits(packed, q, S), quant.bf16_rne_bits(w))


def test_quantize_dequant_error_bound_random_weights():
    """Round trip error on N(0, 0.02) weights with outliers: each weight lands
    within half the local level gap (scaled by its absmax) plus the DQ and
    bf16 rounding."""
    rng = np.random.default_rng(6)
    w = (rng.standard_normal(64 * 512) * 0.02).astype(np.float32)
    w[rng.choice(w.size, 30, replace=False)] = 0.2
    packed, q, S, c = quant.quantize_nf4_dq(w)
    codes = quant.unpack_codes(packed)
    lv = nf4.levels_f64()
    gap_hi = np.append(np.diff(lv), 0.0)
    gap_lo = np.insert(np.diff(lv), 0, 0.0)
    half_gap = 0.5 * np.maximum(gap_hi, gap_lo)[codes]
    cb = np.repeat(c.astype(np.float64), 64)
    cp = np.repeat(quant.absmax_dequant(q, S).astype(np.float64), 64)
    what = quant.dequant_bf16_values(packed, q, S)
    bound = half_gap * cb + np.abs(lv[codes]) * np.abs(cp - cb) + 2.0 ** -8 * np.abs(what) + 1e-12
    assert np.all(np.abs(what - w.astype(np.float64)) <= bound)


def test_dequant_special_codes():
    q = np.array([255, 128], dtype=np.uint8)
    S = np.array([1.0], dtype=np.float32)
    codes = np.zeros(128, dtype=np.uint8)
    codes[0], codes[1], codes[2] = 7, 15, 0
    codes[64], codes[65] = 15, 7
    vals = quant.dequant_bf16_values(quant.pack_codes(codes), q, S)
    cp = quant.absmax_dequant(q, S)
    assert vals[0] == 0.0
    assert vals[1] == float(quant.bf16_bits_to_f32(quant.bf16_rne_bits(np.float32([cp[0]])))[0])
    assert vals[2] == -vals[1]
    assert vals[65] == 0.0
    assert abs(vals[64] - 128.0 / 255.0) <= 128.0 / 255.0 * 2 ** -8


def test_quantize_slice_on_group_boundary_equals_whole():
    rng = np.random.default_rng(7)
    w = (rng.standard_normal(16384 * 3) * 0.02).astype(np.float32)
    p_all, q_all, s_all, _ = quant.quantize_nf4_dq(w)
    p_mid, q_mid, s_mid, _ = quant.quantize_nf4_dq(w[16384:32768])
    assert np.array_equal(p_mid, p_all[8192:16384])
    assert np.array_equal(q_mid, q_all[256:512])
    assert np.array_equal(s_mid, s_all[1:2])


# ---------------------------------------------------------------------------
# Linear algebra: brute force loops and finite differences.
# ---------------------------------------------------------------------------

def _loops_fwd(X, W, A, B, s):
    m, k = X.shape
    n, r = B.shape
    Y = [[0.0] * n for _ in range(m)]
    for i in range(m):
        t = [sum(float(X[i, kk]) * float(A[j, kk]) for kk in range(k)) for j in range(r)]
        for j in range(n):
            base = sum(float(X[i, kk]) * float(W[j, kk]) for kk in range(k))
            Y[i][j] = base + s * sum(t[u] * float(B[j, u]) for u in range(r))
    return np.array(Y)


def _tiny(seed, m=3, n=5, k=64, r=2):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((m, k)), rng.standard_normal((n, k)),
            rng.standard_normal((r, k)), rng.standard_normal((n, r)),
            rng.standard_normal((m, n)))


def test_fwd_matches_index_loops():
    X, W, A, B, _ = _tiny(8)
    assert np.allclose(linear.fwd(X, W, A, B, 1.7), _loops_fwd(X, W, A, B, 1.7), rtol=1e-12, atol=1e-12)


def test_fwd_without_adapter_is_plain_product():
    X, W, A, B, _ = _tiny(9)
    zero_b = np.zeros_like(B)
    assert np.allclose(linear.fwd(X, W, A, zero_b, 2.0), _loops_fwd(X, W, A, zero_b, 0.0), rtol=1e-12, atol=1e-12)
    assert np.allclose(linear.fwd(X, W), linear.fwd(X, W, np.zeros_like(A), B, 2.0), rtol=0, atol=0)


def test_single_row_equals_row_of_batch():
    X, W, A, B, _ = _tiny(10, m=16)
    full = linear.fwd(X, W, A, B, 0.5)
    assert np.allclose(linear.fwd(X[3:4], W, A, B, 0.5), full[3:4], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("s", [2.0, 0.25])
def test_gradients_by_finite_differences(s):
    """L = sum(dY * Y): central differences of L in fp64 give dX, dA, dB
    (Y is linear in each argument, so the differences are exact up to
    rounding)."""
    X, W, A, B, dY = _tiny(11, m=4, n=6, k=64, r=3)

    def loss(X_, A_, B_):
        return float(np.sum(dY * linear.fwd(X_, W, A_, B_, s)))

    h = 1e-3

    def fd(arr, which):
        g = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            p = arr.copy(); p[idx] += h
            mm = arr.copy(); mm[idx] -= h
            args_p = {"X": X, "A": A, "B": B}
            args_m = {"X": X, "A": A, "B": B}
            args_p[which] = p
            args_m[which] = mm
            g[idx] = (loss(args_p["X"], args_p["A"], args_p["B"]) -
                      loss(args_m["X"], args_m["A"], args_m["B"])) / (2 * h)
        return g

    dX = linear.bwd_dx(dY, W, A, B, s)
    dA, dB = linear.lora_grads(X, dY, A, B, s)
    assert np.allclose(dX, fd(X, "X"), rtol=1e-7, atol=1e-7)
    assert np.allclose(dA, fd(A, "A"), rtol=1e-7, atol=1e-7)
    assert np.allclose(dB, fd(B, "B"), rtol=1e-7, atol=1e-7)


def test_error_metric():
    ref = np.array([1.0, -4.0, 2.0])
    assert linear.max_abs_normalised_error(ref + np.array([0.0, 0.04, 0.0]), ref) == pytest.approx(0.01)
    assert linear.max_abs_normalised_error(np.zeros(3), np.zeros(3)) == 0.0


# ---------------------------------------------------------------------------
# Memory arithmetic: the pages' worked figures.
# ---------------------------------------------------------------------------

def _golden_entries():
    with open(os.path.join(GOLDEN, "memory_arithmetic.json")) as f:
        return json.load(f)["entries"]


def test_buffer_sizes_of_the_oracle_give_the_format_rate():
    """Bits per parameter measured from the buffers the oracle actually
    produces for 4096 blocks (16 groups)."""
    rng = np.random.default_rng(12)
    w = (rng.standard_normal(256 * 1024) * 0.02).astype(np.float32)
    packed, q, S, _ = quant.quantize_nf4_dq(w)
    nbytes = packed.nbytes + q.nbytes + S.nbytes
    assert nbytes == memory.total_bytes(w.size)
    assert 8.0 * nbytes / w.size == pytest.approx(memory.RATE_CODES + memory.RATE_SCALE_DQ, abs=0)
    assert 8.0 * (q.nbytes + S.nbytes) / w.size == memory.RATE_SCALE_DQ
    assert memory.RATE_SCALE_FP32 == 0.5
    # 4096 x 4096: the buffers a 7B attention projection needs
    n = 4096 * 4096
    assert memory.code_bytes(n) == 8388608
    assert memory.n_blocks(n) == 262144 and memory.n_groups(n) == 1024


def _quantity(entry):
    p = entry["params"]
    qty = entry["quantity"]
    rate_dq = memory.RATE_SCALE_DQ
    if qty == "bf16_bytes":
        return p * 2 / 1e9
    if qty == "code_bytes":
        return p * memory.RATE_CODES / 8 / 1e9
    if qty == "absmax_fp32_bytes":
        return p * memory.RATE_SCALE_FP32 / 8 / 1e9
    if qty == "absmax_dq_bytes":
        return p * rate_dq / 8 / 1e9
    if qty == "dq_saving_bytes":
        return p * (memory.RATE_SCALE_FP32 - rate_dq) / 8 / 1e9
    if qty in ("total_bytes", "total_bytes_below"):
        return p * (memory.RATE_CODES + rate_dq) / 8 / 1e9
    if qty == "scale_bits_fp32":
        return memory.RATE_SCALE_FP32
    if qty == "scale_bits_dq":
        return rate_dq
    if qty == "dq_saving_bits":
        return memory.RATE_SCALE_FP32 - rate_dq
    if qty == "total_bits":
        return memory.RATE_CODES + rate_dq
    raise KeyError(qty)


@pytest.mark.parametrize("entry", _golden_entries(), ids=lambda e: e["id"])
def test_memory_figures_printed_on_the_pages(entry):
    got = _quantity(entry)
    if entry["quantity"] == "total_bytes_below":
        assert got < entry["value"]
    else:
        assert abs(got - entry["value"]) <= entry["tol"], (entry["id"], got)


def test_exact_rate_matches_large_buffer():
    """The per-parameter rates are the limit of the exact buffer sizes."""
    n = 64 * 256 * 1000
    assert memory.bits_per_param(n) == pytest.approx(4.0 + 0.126953125, abs=0)
    assert memory.scale_bits_per_param(n, double_quant=False) == 0.5
