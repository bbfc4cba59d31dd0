"""Pins for the oracle's W4A16 product (CPU only): exact rational brute force
on tiny inputs, and the post-group algebra of the MixPE page."""

from fractions import Fraction

import numpy as np

from oracle import formats, numerics, products


def _tiny_int4(seed, m, n, k, group):
    rng = np.random.default_rng(seed)
    x = numerics.bf16_round(rng.standard_normal((m, k)).astype(np.float32))
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    q, s, z = formats.int4_quantize(w, group)
    return x, q, s, z


def test_int4_product_brute_force_rational():
    """y = sum_k x (q - z) s computed with exact rationals, K <= 16, N <= 4."""
    for seed, (m, n, k, g) in enumerate([(1, 4, 16, 8), (3, 2, 16, 16), (2, 3, 8, 8)]):
        x, q, s, z = _tiny_int4(seed, m, n, k, g)
        y = products.w4a16_int4(x, q, s, z, g)
        for i in range(m):
            for j in range(n):
                terms = [Fraction(float(x[i, kk])) * (int(q[j, kk]) - Fraction(float(z[j, kk // g])))
                         * Fraction(float(s[j, kk // g])) for kk in range(k)]
                acc = sum(terms)
                # fp64 summation of k exact products: error <= k * 2^-53 * sum |terms|
                bound = k * Fraction(1, 2 ** 53) * sum(abs(t) for t in terms)
                assert abs(Fraction(float(y[i, j])) - acc) <= bound + Fraction(1, 2 ** 1000)


def test_int4_post_group_equals_plain():
    """Applying scale and zero after each group's sum gives the same product."""
    x, q, s, z = _tiny_int4(11, 5, 24, 512, 128)
    a = products.w4a16_int4(x, q, s, z, 128)
    b = products.w4a16_int4_post_group(x, q, s, z, 128)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


def test_nf4_product_brute_force_rational():
    rng = np.random.default_rng(12)
    m, n, k = 2, 2, 64
    x = numerics.bf16_round(rng.standard_normal((m, k)).astype(np.float32))
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    codes, absmax = formats.nf4_quantize(w)
    cb = formats.nf4_codebook()
    y = products.w4a16_nf4(x, codes, absmax, k)
    for i in range(m):
        for j in range(n):
            terms = [Fraction(float(x[i, kk])) * Fraction(float(cb[codes[j * k + kk]]))
                     * Fraction(float(absmax[(j * k + kk) // 64])) for kk in range(k)]
            acc = sum(terms)
            bound = k * Fraction(1, 2 ** 53) * sum(abs(t) for t in terms)
            assert abs(Fraction(float(y[i, j])) - acc) <= bound + Fraction(1, 2 ** 1000)


def test_product_transposition_pin():
    """A transposed operand is caught: y[m, n] pairs row m of x with row n of W."""
    x = np.zeros((2, 8), np.float32)
    x[0, 0] = 1.0
    x[1, 1] = 1.0
    w = np.zeros((3, 8), np.float32)
    w[2, 0] = 0.5
    w[0, 1] = -0.25
    y = products.matmul_exact(x, w)
    assert y.shape == (2, 3)
    assert y[0, 2] == 0.5 and y[1, 0] == -0.25 and np.count_nonzero(y) == 2
