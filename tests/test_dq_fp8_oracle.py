"""Pins of ``oracle/dq_fp8.py``, the mean-subtracted 8-bit-float double
quantization of the block absmax (CPU).

* E4M3 decoding and round-to-nearest-even encoding against PyTorch's
  float8_e4m3fn (an independent implementation of the same format), on every
  bit pattern and on every tie between neighbouring values.
* The pairwise fp64 sum against its recursive definition and against an
  exact sum (math.fsum).
* The format: c' reproduces the mean exactly where a group is constant,
  round-trips exactly where the offsets are E4M3 values times a power-of-two
  scale, stays within half an E4M3 step of c otherwise, and stores
  0.127 bit per weight.
"""
import math

import numpy as np
import pytest
import torch

from oracle import dq_fp8, quant


def test_e4m3_decode_matches_torch_on_every_pattern():
    codes = np.arange(256, dtype=np.uint8)
    ours = dq_fp8.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2       # 0x7F and 0xFF
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert ours[0x7E] == 448.0 and ours[0x38] == 1.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_e4m3_encode_matches_torch_including_ties():
    pos = dq_fp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    mids = (pos[:-1] + pos[1:]) / 2.0                         # exact in fp32 for this format
    xs = [np.float32(v) for v in np.concatenate([pos, mids])]
    near = []
    for v in xs:
        near += [np.nextafter(v, np.float32(-np.inf)), v, np.nextafter(v, np.float32(np.inf))]
    rng = np.random.default_rng(0)
    x = np.concatenate([np.array(near, dtype=np.float32),
                        rng.uniform(-448, 448, 20000).astype(np.float32),
                        (rng.standard_normal(5000) * 1e-3).astype(np.float32)])
    x = np.clip(x, -448, 448).astype(np.float32)
    x = np.concatenate([x, -x])
    ours = dq_fp8.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def _recursive_sum(v):
    if len(v) == 1:
        return float(v[0])
    half = [v[i] + v[i + 1] for i in range(0, len(v) - 1, 2)] + ([v[-1]] if len(v) % 2 else [])
    return _recursive_sum(half)


def test_pairwise_sum_definition_and_accuracy():
    assert dq_fp8.pairwise_sum([1.0, 2.0, 3.0, 4.0, 5.0]) == ((1.0 + 2.0) + (3.0 + 4.0)) + 5.0
    rng = np.random.default_rng(1)
    for n in (1, 2, 3, 7, 255, 256, 257, 1000):
        v = rng.uniform(0.0, 1.0, n)
        assert dq_fp8.pairwise_sum(v) == _recursive_sum(list(v))
    c = rng.uniform(0.01, 0.2, 100000).astype(np.float32)
    assert abs(dq_fp8.pairwise_sum(c) - math.fsum(c.astype(np.float64))) <= 1e-12 * math.fsum(c.astype(np.float64))


def test_tensor_mean_is_the_group_tree_of_pairwise_sums():
    rng = np.random.default_rng(2)
    c = rng.uniform(0.0, 0.1, 256 * 5 + 37).astype(np.float32)
    sums = [dq_fp8.pairwise_sum(c[i:i + 256]) for i in range(0, c.size, 256)]
    assert dq_fp8.tensor_mean(c) == np.float32(dq_fp8.pairwise_sum(sums) / c.size)
    assert abs(float(dq_fp8.tensor_mean(c)) - float(np.mean(c.astype(np.float64)))) < 1e-7


def test_constant_group_reconstructs_exactly_and_codes_are_zero():
    c = np.full(300, np.float32(0.0375), dtype=np.float32)
    q, gs = dq_fp8.double_quantize_fp8(c)
    assert np.all(q == 0) and gs[-1] == np.float32(0.0375)
    assert np.array_equal(dq_fp8.absmax_dequant_fp8(q, gs), c)


def test_exact_round_trip_when_offsets_are_e4m3_values():
    """mu = 1/4 exactly (values symmetric about it), offsets are E4M3 values
    times 2^-9, the largest offset 448 * 2^-9: every c' equals c."""
    rng = np.random.default_rng(3)
    pos = dq_fp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    off = rng.choice(pos, 127) * np.float32(2.0 ** -9)
    off[0] = np.float32(448.0 * 2.0 ** -9)
    d = np.concatenate([off, -off, [0.0, 0.0]]).astype(np.float32)       # 256 values, mean offset 0
    c = (np.float32(0.25) + d).astype(np.float32)
    q, gs = dq_fp8.double_quantize_fp8(c)
    assert gs[-1] == np.float32(0.25)
    assert np.array_equal(dq_fp8.absmax_dequant_fp8(q, gs), c)


def test_round_trip_error_is_at_most_half_an_e4m3_step():
    rng = np.random.default_rng(4)
    c = np.abs(rng.standard_normal(256 * 9 + 11)).astype(np.float32) * np.float32(0.03)
    q, gs = dq_fp8.double_quantize_fp8(c)
    cp = dq_fp8.absmax_dequant_fp8(q, gs)
    mu = gs[-1]
    for g in range(gs.size - 1):
        sl = slice(g * 256, (g + 1) * 256)
        S = float(np.max(np.abs(c[sl] - mu)))
        d = np.abs(c[sl].astype(np.float64) - mu)
        step = np.maximum(2.0 ** np.floor(np.log2(np.maximum(d / S * 448.0, 2.0 ** -6))) / 8.0, 2.0 ** -9)
        bound = (step / 2.0) * S / 448.0 + 4e-7 * (S + abs(float(mu)))
        assert np.all(np.abs(cp[sl].astype(np.float64) - c[sl]) <= bound)


def test_storage_is_0_127_bit_per_weight():
    n, k = 1024, 1024
    W = np.random.default_rng(5).standard_normal(n * k).astype(np.float32) * np.float32(0.02)
    packed, q, gs, _ = dq_fp8.quantize(W)
    bits = 8.0 * (packed.size + q.size + 4 * gs.size) / (n * k)
    assert abs(bits - 4.0 - (8 / 64 + 32 / (64 * 256) + 32 / (n * k))) < 1e-12
    assert abs(bits - 4.127) < 1e-3
    # The codes do not depend on the double quantization.
    assert np.array_equal(packed, quant.quantize_nf4_dq(W)[0])


def test_decoded_weights_follow_the_reconstructed_constants():
    W = np.random.default_rng(6).standard_normal(64 * 512).astype(np.float32) * np.float32(0.02)
    packed, q, gs, _ = dq_fp8.quantize(W)
    cp = dq_fp8.absmax_dequant_fp8(q, gs)
    codes = quant.unpack_codes(packed)
    from oracle import nf4
    vals = nf4.levels_f32()[codes].reshape(-1, 64) * cp.reshape(-1, 1)
    want = quant.bf16_rne_bits(vals.astype(np.float32).reshape(-1))
    assert np.array_equal(dq_fp8.dequant_bf16_bits(packed, q, gs), want)


def test_rejects_out_of_range_for_the_encoder():
    with pytest.raises(ValueError):
        dq_fp8.e4m3_encode(np.array([449.0], dtype=np.float32))
