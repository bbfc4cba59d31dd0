"""Pins for the oracle's salient-channel residual correction (CPU only).

"DecDEC: A Systems Approach to Advancing Low-Bit LLM Quantization", Abstract:
the residual is full precision minus quantized weights, and the residuals of
the channels that the current activations mark as outliers are added back.

The pins use facts from outside the oracle:
- a pure-Python ranking of the channels;
- the full-precision product;
- the exact outer product of a single channel;
- fp16/fp32 rounding bounds computed with np.spacing.
"""

import struct

import numpy as np
import pytest

from oracle import decdec, formats, numerics, products


def _bf16(a):
    return numerics.bf16_round(np.asarray(a, dtype=np.float32))


def _py_select(x, k):
    """Reference ranking written with Python floats and struct: magnitude bits
    (sign cleared) descending, channel index ascending."""
    m, kk = x.shape
    keys = []
    for c in range(kk):
        best = 0
        for i in range(m):
            bits = struct.unpack("<I", struct.pack("<f", float(x[i, c])))[0] & 0x7FFFFFFF
            best = max(best, bits)
        keys.append((-best, c))
    keys.sort()
    return sorted(c for _, c in keys[:max(0, min(k, kk))])


@pytest.mark.parametrize("seed,m,kk", [(0, 1, 7), (1, 3, 33), (2, 2, 64), (3, 16, 40)])
def test_select_matches_python_ranking(seed, m, kk):
    rng = np.random.default_rng(seed)
    x = _bf16(rng.standard_normal((m, kk)))
    # ties: equal magnitudes in several channels, with both signs
    x[:, kk // 3] = -x[:, 1]
    x[:, kk // 2] = x[:, 1]
    x[0, kk - 1] = np.inf
    if m > 1:
        x[1, 2] = np.nan  # NaN ranks above +inf
    for k in (0, 1, 2, 5, kk // 2, kk, kk + 3):
        got = decdec.select_salient(x, k).tolist()
        assert got == _py_select(x, k), (seed, k)


def test_select_picks_the_outlier_channels():
    rng = np.random.default_rng(7)
    x = _bf16(rng.standard_normal((4, 512)))
    outl = [17, 300, 301, 499]
    x[2, outl] = [60.0, -70.0, 80.0, -90.0]  # far above |N(0,1)| draws
    assert set(outl) <= set(decdec.select_salient(x, 4).tolist())
    assert decdec.select_salient(x, 4).tolist() == sorted(outl)


def _int4_case(seed, n=48, k=256, group=64):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    q, s, z = formats.int4_quantize(w, group)
    return w, q, s, z


def test_residual_is_the_rounded_difference():
    """R = fp16(fp32(W - W_hat)): within half an fp16 ulp plus half an fp32 ulp
    of the exact difference, element by element."""
    w, q, s, z = _int4_case(3)
    w_hat = formats.int4_dequant_exact(q, s, z, 64)
    rt = decdec.int4_residual_t(w, q, s, z, 64)
    assert rt.dtype == np.float16 and rt.shape == (w.shape[1], w.shape[0])
    exact = w.astype(np.float64) - w_hat.astype(np.float64)
    got = rt.T.astype(np.float64)
    bound = (0.5 * np.spacing(np.abs(exact).astype(np.float16)).astype(np.float64) +
             0.5 * np.spacing(np.abs(exact).astype(np.float32)).astype(np.float64))
    assert np.all(np.abs(got - exact) <= bound)


def test_residual_of_weights_on_the_grid_is_zero():
    """Weights that are already exactly a dequantized grid value have no residual."""
    w, q, s, z = _int4_case(4)
    w_hat = formats.int4_dequant_exact(q, s, z, 64)
    q2, s2, z2 = formats.int4_quantize(w_hat, 64)
    rt = decdec.int4_residual_t(w_hat, q2, s2, z2, 64)
    assert np.array_equal(formats.int4_dequant_exact(q2, s2, z2, 64), w_hat)
    assert np.count_nonzero(rt) == 0


def test_all_channels_recover_the_full_precision_product():
    """With every channel selected, x . (W_hat + R)^T is the full-precision
    product up to R's fp16 rounding: far closer than the uncorrected one."""
    w, q, s, z = _int4_case(5)
    rng = np.random.default_rng(5)
    x = _bf16(rng.standard_normal((3, w.shape[1])))
    rt = decdec.int4_residual_t(w, q, s, z, 64)
    idx = decdec.select_salient(x, w.shape[1])
    y_full = x.astype(np.float64) @ w.astype(np.float64).T
    y_base = products.w4a16_int4(x, q, s, z, 64)
    y_corr = decdec.int4_corrected(x, q, s, z, 64, rt, idx)
    err_base = np.abs(y_base - y_full).max()
    err_corr = np.abs(y_corr - y_full).max()
    # R's rounding: |R| <= s/2 < 2^-7 here, where half an fp16 ulp is 2^-18
    assert np.abs(rt.astype(np.float64)).max() < 2.0 ** -7
    bound = (np.abs(x).astype(np.float64) @ np.full(w.shape[1], 2.0 ** -18)).max()
    assert err_corr <= bound
    assert err_base > 100 * err_corr


def test_one_channel_adds_its_outer_product():
    w, q, s, z = _int4_case(6)
    rng = np.random.default_rng(6)
    x = _bf16(rng.standard_normal((2, w.shape[1])))
    rt = decdec.int4_residual_t(w, q, s, z, 64)
    c = 77
    diff = (decdec.int4_corrected(x, q, s, z, 64, rt, np.array([c], np.int32)) -
            products.w4a16_int4(x, q, s, z, 64))
    expect = np.outer(x[:, c].astype(np.float64), rt[c].astype(np.float64))
    assert np.array_equal(diff, expect) or np.abs(diff - expect).max() <= 1e-18


def test_no_channels_is_the_plain_product():
    w, q, s, z = _int4_case(8)
    x = _bf16(np.random.default_rng(8).standard_normal((2, w.shape[1])))
    rt = decdec.int4_residual_t(w, q, s, z, 64)
    assert np.array_equal(decdec.int4_corrected(x, q, s, z, 64, rt, decdec.select_salient(x, 0)),
                          products.w4a16_int4(x, q, s, z, 64))


def test_nf4_all_channels_recover_the_full_precision_product():
    rng = np.random.default_rng(9)
    n, k = 32, 256
    w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    codes, absmax = formats.nf4_quantize(w)
    rt = decdec.nf4_residual_t(w, codes, absmax)
    x = _bf16(rng.standard_normal((2, k)))
    y_full = x.astype(np.float64) @ w.astype(np.float64).T
    y_base = products.w4a16_nf4(x, codes, absmax, k)
    y_corr = decdec.nf4_corrected(x, codes, absmax, k, rt, decdec.select_salient(x, k))
    err_corr = np.abs(y_corr - y_full).max()
    assert np.abs(y_base - y_full).max() > 100 * err_corr
