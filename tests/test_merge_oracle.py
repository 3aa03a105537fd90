"""Pins of the oracle's adapter merge (``oracle.merge``) on the CPU.

The merged weight must reproduce the layer's forward through a plain product
(``oracle.linear.fwd`` computes (X . A^T) . B^T, a different order of the same
algebra); a zero adapter must return the dequantized base bit for bit; a
rank-1 adapter must match an index-loop brute force.
"""
import numpy as np
import pytest

from oracle import linear, merge, quant


def _base(n, k, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal(n * k) * 0.02).astype(np.float32)
    packed, q, S, _ = quant.quantize_nf4_dq(w)
    return quant.dequant_bf16_values(packed, q, S).reshape(n, k)


def _bf16_vals(a):
    return quant.bf16_bits_to_f32(quant.bf16_rne_bits(np.asarray(a, dtype=np.float32))).astype(np.float64)


@pytest.mark.parametrize("s", [2.0, 0.25])
def test_merged_product_equals_the_layer_forward(s):
    rng = np.random.default_rng(61)
    n, k, r, m = 48, 128, 16, 5
    W_hat = _base(n, k, 62)
    A = _bf16_vals(rng.standard_normal((r, k)) * 0.05)
    B = _bf16_vals(rng.standard_normal((n, r)) * 0.05)
    X = _bf16_vals(rng.standard_normal((m, k)))
    Wm = merge.merge_f64(W_hat, A, B, s)
    got = X @ Wm.T
    ref = linear.fwd(X, W_hat, A, B, s)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_zero_adapter_returns_the_base_bit_for_bit():
    n, k, r = 16, 64, 16
    W_hat = _base(n, k, 63)
    rng = np.random.default_rng(64)
    A = _bf16_vals(rng.standard_normal((r, k)))
    bits = quant.bf16_rne_bits(W_hat.astype(np.float32))
    assert np.array_equal(merge.merge_bf16_bits(W_hat, A, np.zeros((n, r)), 2.0), bits)
    assert np.array_equal(merge.merge_bf16_bits(W_hat, np.zeros((r, k)), np.ones((n, r)), 2.0), bits)


def test_rank_one_adapter_by_index_loops():
    n, k, r = 8, 64, 16
    W_hat = _base(n, k, 65)
    rng = np.random.default_rng(66)
    A = np.zeros((r, k))
    B = np.zeros((n, r))
    A[3] = _bf16_vals(rng.standard_normal(k))
    B[:, 3] = _bf16_vals(rng.standard_normal(n))
    s = 0.5
    got = merge.merge_f64(W_hat, A, B, s)
    for i in range(n):
        for j in range(k):
            assert got[i, j] == W_hat[i, j] + s * (B[i, 3] * A[3, j])


def test_merge_is_linear_in_the_scale():
    n, k, r = 24, 128, 32
    W_hat = _base(n, k, 67)
    rng = np.random.default_rng(68)
    A = _bf16_vals(rng.standard_normal((r, k)) * 0.1)
    B = _bf16_vals(rng.standard_normal((n, r)) * 0.1)
    d1 = merge.merge_f64(W_hat, A, B, 1.0) - W_hat
    d3 = merge.merge_f64(W_hat, A, B, 3.0) - W_hat
    assert np.allclose(d3, 3.0 * d1, rtol=0, atol=1e-15)
