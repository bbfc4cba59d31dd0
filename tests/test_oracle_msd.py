"""Pins for the oracle's Multi-Scale Dequant decomposition and decomposed
product (CPU only): a hand-derived row, the reconstruction bound, the
effective-bits figure the page states for two INT8 passes, and exact rational
equality of the decomposed product with the undecomposed one."""

import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import formats, msd, numerics, products


def test_decompose_golden_row(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "msd_rows.json")))
    x = np.array([g["row"]], dtype=np.float32)
    a, s = msd.decompose(x, g["n_components"])
    assert s[:, 0].tolist() == g["scales"]
    assert a[:, 0, :].tolist() == g["digits"]
    assert np.array_equal(msd.reconstruct(a, s), x.astype(np.float64))


def _acts(seed, m, k, outliers=0.005, scale=50.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((m, k)).astype(np.float32)
    idx = rng.permutation(k)[: max(1, round(outliers * k))]
    x[:, idx] *= np.float32(scale)
    return numerics.bf16_round(x)


@pytest.mark.parametrize("c", [1, 2, 3])
def test_decompose_bound(c):
    x = _acts(21, 48, 1024)
    x[3] = 0.0                       # all-zero row: scale 1, digits 0
    a, s = msd.decompose(x, c)
    assert a.dtype == np.int8
    assert np.abs(a[0]).max() <= 127
    assert np.all(a[0, 3] == 0) and np.all(s[:, 3] == np.float32(1) / np.float32(256) ** np.arange(c))
    err = np.abs(x.astype(np.float64) - msd.reconstruct(a, s))
    bound = s[-1].astype(np.float64)[:, None] / 2 * (1 + 2.0 ** -15)
    assert np.all(err <= bound)
    # scales are exact powers-of-two ratios
    for ci in range(1, c):
        assert np.array_equal(s[ci - 1].astype(np.float64), s[ci].astype(np.float64) * 256)


def test_two_int8_passes_near_16_effective_bits():
    x = _acts(22, 64, 4096)
    a, s = msd.decompose(x, 2)
    bits = msd.effective_bits(x, a, s)
    assert bits >= 15.9
    a1, s1 = msd.decompose(x, 1)
    assert 7.5 <= msd.effective_bits(x, a1, s1) < 8.1


def _tiny_case(seed, m, n, k, group, c):
    rng = np.random.default_rng(seed)
    x = _acts(seed, m, k)
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    q, sw, zw = formats.int4_quantize(w, group)
    a, s = msd.decompose(x, c)
    return x, q, sw, zw, a, s


def test_decomposed_product_equals_undecomposed_rational():
    """sum_c s_c sum_g s (P_c - z R_c) == x_hat . ((q - z) s)^T, exactly."""
    for seed, (m, n, k, g, c) in enumerate([(2, 3, 16, 8, 2), (1, 2, 16, 16, 3), (3, 2, 8, 8, 1)]):
        x, q, sw, zw, a, s = _tiny_case(30 + seed, m, n, k, g, c)
        y = msd.msd_product(a, s, q, sw, zw, g)
        for i in range(m):
            for j in range(n):
                xh = [sum(Fraction(float(s[ci, i])) * int(a[ci, i, kk]) for ci in range(c))
                      for kk in range(k)]
                terms = [xh[kk] * (int(q[j, kk]) - Fraction(float(zw[j, kk // g])))
                         * Fraction(float(sw[j, kk // g])) for kk in range(k)]
                acc = sum(terms)
                bound = 4 * k * c * Fraction(1, 2 ** 53) * sum(abs(t) for t in terms)
                assert abs(Fraction(float(y[i, j])) - acc) <= bound + Fraction(1, 2 ** 1000)


def test_decomposed_product_matches_fp64_and_exact_product():
    x, q, sw, zw, a, s = _tiny_case(40, 8, 32, 512, 128, 2)
    y = msd.msd_product(a, s, q, sw, zw, 128)
    xh = msd.reconstruct(a, s)
    assert np.allclose(y, products.w4a16_int4(xh, q, sw, zw, 128), rtol=1e-12, atol=1e-12)
    # against the undecomposed product: within the 16-bit reconstruction error
    y_exact = products.w4a16_int4(x, q, sw, zw, 128)
    rel, _ = numerics.compare(y, y_exact)
    assert rel < 1e-4


def test_group_sums_and_partials_definition():
    a = np.array([[[1, -2, 3, 4]]], dtype=np.int8)
    q = np.array([[1, 2, 3, 4], [0, 15, 0, 15]], dtype=np.uint8)
    assert msd.group_sums(a, 2).tolist() == [[[-1, 7]]]
    p = msd.int_partials(a, q, 2)
    assert p[0, 0].tolist() == [[-3, 25], [-30, 60]]


# ---------------------------------------------------------------------------
# NF4 weights on the MSD path
# ---------------------------------------------------------------------------

def test_nf4_integer_codebook_digits_and_bound():
    from oracle import formats
    cb = formats.nf4_codebook()
    ci = msd.nf4_int_codebook(cb)
    h, l = msd.nf4_int_digits(cb)
    assert np.all(np.abs(ci / 8192.0 - cb.astype(np.float64)) <= 2.0 ** -14)
    assert np.array_equal(128 * h + l, ci)
    assert l.min() >= -64 and l.max() <= 63 and h.min() >= -64 and h.max() <= 64
    assert ci[0] == -8192 and ci[15] == 8192 and ci[7] == 0      # -1, +1 and the exact zero


def test_msd_nf4_product_is_exact_against_rationals():
    """The product equals x_hat . w_int^T exactly (brute force in rationals on
    a tiny problem), and lies within the weight bound of the exact NF4
    product: |w_int - w| <= absmax 2^-14 per weight."""
    from fractions import Fraction
    from oracle import formats
    rng = np.random.default_rng(11)
    m, n, k = 2, 3, 128
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    codes, absmax = formats.nf4_quantize(w)
    x = rng.standard_normal((m, k)).astype(np.float32)
    a, s = msd.decompose(x, 2)
    cb = formats.nf4_codebook()
    y = msd.msd_nf4_product(a, s, codes, absmax, k, cb)
    h, l = msd.nf4_int_digits(cb)
    q = codes.reshape(n, k).astype(np.int64)
    am = absmax.reshape(n, k // 64)
    for i in range(m):
        for j in range(n):
            tot = Fraction(0)
            for c in range(2):
                for kk in range(k):
                    wij = Fraction(float(am[j, kk // 64])) * (128 * int(h[q[j, kk]]) + int(l[q[j, kk]]))
                    tot += Fraction(float(s[c, i])) * int(a[c, i, kk]) * wij
            tot /= 8192
            # the integer inner sums are exact; the scaled fp64 sums round a few times
            assert abs(Fraction(float(y[i, j])) - tot) <= abs(tot) * Fraction(1, 2 ** 45)
    # against the exact NF4 product of the decomposed activations
    from oracle import products
    x_hat = msd.reconstruct(a, s)
    y_nf4 = products.w4a16_nf4(x_hat, codes, absmax, k)
    bound = np.abs(x_hat) @ np.repeat(am, 64, axis=1).T * 2.0 ** -14
    assert np.all(np.abs(y - y_nf4) <= bound * (1 + 1e-9))
