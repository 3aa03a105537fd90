"""Pins of the oracle's LoRA dropout (``oracle.dropout``) on the CPU.

The generator is checked against numpy's own Philox4x64-10 (an independent
implementation; numpy steps its counter before drawing, so its stream at
counter c - 1 is the block of counter c); the mask against the binomial keep
rate, independence across offsets and the uniformity of the 16-bit draws;
inverted dropout against its mean; the layer's gradients under a fixed mask
against central finite differences.
"""
import numpy as np
import pytest

from oracle import dropout, quant


@pytest.mark.parametrize("counter,key", [((1, 0, 0, 0), (7, 0)), ((5, 3, 0, 0), (123456789, 42)),
                                         ((2 ** 40 + 17, 2 ** 63, 9, 1), (2 ** 64 - 1, 2 ** 32))])
def test_philox_matches_numpy(counter, key):
    prev = [counter[0] - 1] + list(counter[1:])
    bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.array(prev, dtype=np.uint64))
    want = [int(v) for v in bg.random_raw(4)]
    assert dropout.philox4x64_10(counter, key) == want


@pytest.mark.parametrize("p", [0.05, 0.5])
def test_keep_rate_is_binomial(p):
    n = 1 << 16
    keep = dropout.keep_mask(64, 1024, p, seed=2024, offset=3)
    rate = 1.0 - dropout.threshold(p) / 65536.0
    sigma = np.sqrt(rate * (1 - rate) / n)
    assert abs(keep.mean() - rate) < 5 * sigma


def test_threshold_resolution():
    assert dropout.threshold(0.0) == 0
    assert dropout.threshold(0.05) == 3277
    assert dropout.threshold(0.5) == 32768
    with pytest.raises(ValueError):
        dropout.threshold(1.0)


def test_p_zero_keeps_everything_unscaled():
    rng = np.random.default_rng(5)
    x = quant.bf16_bits_to_f32(quant.bf16_rne_bits(rng.standard_normal((8, 64)).astype(np.float32)))
    keep = dropout.keep_mask(8, 64, 0.0, seed=1, offset=0)
    assert keep.all()
    assert np.array_equal(dropout.dropout_bf16_bits(x, keep, 0.0), quant.bf16_rne_bits(x))


def test_offsets_and_seeds_give_independent_masks():
    p = 0.5
    a = dropout.keep_mask(32, 1024, p, seed=9, offset=0)
    b = dropout.keep_mask(32, 1024, p, seed=9, offset=1)
    c = dropout.keep_mask(32, 1024, p, seed=10, offset=0)
    n = a.size
    for other in (b, c):
        agree = (a == other).mean()
        assert abs(agree - 0.5) < 5 * np.sqrt(0.25 / n)
    assert np.array_equal(a, dropout.keep_mask(32, 1024, p, seed=9, offset=0))


def test_sixteen_bit_draws_are_uniform():
    u = dropout.uniforms16(1 << 16, seed=77, offset=5)
    counts = np.bincount(u >> 12, minlength=16)
    expected = u.size / 16
    chi2 = float(((counts - expected) ** 2 / expected).sum())
    assert chi2 < 50.0, chi2                      # 15 degrees of freedom: p-value ~ 1e-5
    assert u.max() < 65536


def test_inverted_dropout_keeps_the_mean():
    p = 0.05
    x = np.ones((64, 1024), dtype=np.float32)
    keep = dropout.keep_mask(64, 1024, p, seed=31, offset=7)
    xd = dropout.dropout_values(x, keep, p)
    kept = keep.mean()
    sigma = np.sqrt(kept * (1 - kept) / keep.size)
    assert abs(xd.mean() - 1.0) < 5 * sigma * float(dropout.keep_scale(p)) + 2 ** -8
    assert set(np.unique(xd)) <= {0.0, float(quant.bf16_bits_to_f32(quant.bf16_rne_bits(
        np.float32([dropout.keep_scale(p)])))[0])}


def test_gradients_by_finite_differences():
    """L = sum(dY * Y) with Xd = D * X * c (c = fp32(1 / fp32(1 - p))) taken
    exactly: central differences in X, A and B match bwd_dx and lora_grads."""
    rng = np.random.default_rng(8)
    m, n, k, r, s, p = 3, 8, 64, 16, 2.0, 0.3
    X, W, A, B, dY = (rng.standard_normal(sh) for sh in ((m, k), (n, k), (r, k), (n, r), (m, n)))
    keep = dropout.keep_mask(m, k, p, seed=4, offset=0)
    cks = float(dropout.keep_scale(p))

    def loss(X_, A_, B_):
        Xd = np.where(keep, X_ * cks, 0.0)
        return float((dY * dropout.fwd(X_, W, A_, B_, s, Xd)).sum())

    h = 1e-6
    num = np.zeros_like(X)
    for i in range(m):
        for j in range(k):
            e = np.zeros_like(X)
            e[i, j] = h
            num[i, j] = (loss(X + e, A, B) - loss(X - e, A, B)) / (2 * h)
    assert np.allclose(num, dropout.bwd_dx(dY, W, A, B, s, keep, p), rtol=1e-6, atol=1e-6)
    Xd = np.where(keep, X * cks, 0.0)
    dA, dB = dropout.lora_grads(Xd, dY, A, B, s)
    for M, G, which in ((A, dA, 0), (B, dB, 1)):
        for _ in range(20):
            i, j = rng.integers(0, M.shape[0]), rng.integers(0, M.shape[1])
            e = np.zeros_like(M)
            e[i, j] = h
            if which == 0:
                d = (loss(X, A + e, B) - loss(X, A - e, B)) / (2 * h)
            else:
                d = (loss(X, A, B + e) - loss(X, A, B - e)) / (2 * h)
            assert abs(d - G[i, j]) <= 1e-6 * max(1.0, abs(G[i, j]))
