"""Pins for the oracle's rounding helpers and 4-bit formats (CPU only).

Each test checks the oracle against something that does not come from the
oracle: hand-derived golden groups, a library routine, the codebook's defining
property checked through the normal CDF, or exact brute force.
"""

import json
import os

import numpy as np
import pytest
import torch
from scipy.stats import norm

from oracle import formats, numerics


# --------------------------------------------------------------------------
# bf16 rounding: a special case that reduces to a library routine
# --------------------------------------------------------------------------

def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * np.float32(3),
        rng.standard_normal(1000).astype(np.float32) * np.float32(1e-38),   # subnormals
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, -1.00390625, 65504.0,
                  3.3895313892515355e38, np.inf, -np.inf], dtype=np.float32),
    ])
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(numerics.bf16_bits(vals), ref)


def test_bf16_round_keeps_nan():
    out = numerics.bf16_round(np.array([np.nan, -np.nan], dtype=np.float32))
    assert np.isnan(out).all()


def _bf16_spacing_torch(v):
    """Gap between consecutive bf16 numbers in the binade of |v|, from the
    bf16 type itself: the largest bf16 value not above |v| (b), then
    nextafter(b, +inf) - b. Independent of numerics.bf16_ulp."""
    a = torch.from_numpy(np.abs(np.asarray(v, dtype=np.float64)))
    b = a.to(torch.bfloat16)                      # round to nearest even ...
    over = b.double() > a
    b = torch.where(over, torch.nextafter(b, torch.zeros_like(b)), b)   # ... then down
    up = torch.nextafter(b, torch.full_like(b, float("inf")))
    return (up.double() - b.double()).numpy()


def test_bf16_ulp_matches_bf16_type():
    """bf16 keeps 8 significant bits: in the binade [2^e, 2^(e+1)) its numbers
    are 2^(e-7) apart, and below 2^-126 (subnormal) 2^-133 apart. Checked
    against torch.nextafter on bf16 values over every normal binade, on exact
    powers of two and on the fp64 values just below them (where a floating
    log2 can round up into the next binade), negatives and subnormals."""
    rng = np.random.default_rng(7)
    e = np.arange(-140, 127)
    pow2 = np.ldexp(1.0, e)
    vals = np.concatenate([
        pow2, -pow2,
        np.nextafter(pow2, 0.0), -np.nextafter(pow2, 0.0),
        np.nextafter(pow2, np.inf),
        rng.uniform(1.0, 2.0, 4000) * np.ldexp(1.0, rng.integers(-140, 127, 4000)),
        -rng.uniform(1.0, 2.0, 1000) * np.ldexp(1.0, rng.integers(-30, 30, 1000)),
        rng.standard_normal(2000) * 5.6,
        np.array([1e-45, 3.0e-39, 1.1754942e-38, 0.0]),
    ])
    got = numerics.bf16_ulp(vals)
    ref = _bf16_spacing_torch(vals)
    bad = got != ref
    assert not bad.any(), list(zip(vals[bad][:5], got[bad][:5], ref[bad][:5]))
    # spot values by hand: 1 -> 2^-7, 3 -> 2^-6, just below 1 -> 2^-8
    assert numerics.bf16_ulp(np.array([1.0, 3.0, np.nextafter(1.0, 0.0), -0.75])).tolist() == [
        2.0 ** -7, 2.0 ** -6, 2.0 ** -8, 2.0 ** -8]


def test_compare_metrics_closed_form():
    ref = np.array([3.0, 4.0])
    rel, mx = numerics.compare(ref + np.array([0.3, -0.4]), ref)
    assert rel == pytest.approx(0.1)
    assert mx == pytest.approx(0.4 / np.sqrt(12.5))


# --------------------------------------------------------------------------
# NF4 codebook
# --------------------------------------------------------------------------

def test_nf4_codebook_shape_and_endpoints(golden_dir):
    cb = formats.nf4_codebook()
    assert cb.dtype == np.float32 and cb.shape == (16,)
    assert np.all(np.diff(cb) > 0)
    assert cb[0] == -1.0 and cb[15] == 1.0 and cb[7] == 0.0
    assert (cb > 0).sum() == 8 and (cb < 0).sum() == 7
    g = json.load(open(os.path.join(golden_dir, "nf4_blocks.json")))
    assert np.allclose(cb, g["codebook_4dp"], atol=5e-5)


def test_nf4_codebook_quantiles_via_cdf():
    """Defining property, checked with the CDF (not the inverse the oracle uses):
    Phi(c_i * Phi^-1(delta)) are the even splits of [1/2, delta] into 8 steps
    (positive side) and 7 steps (negative side)."""
    cb = formats.nf4_codebook().astype(np.float64)
    d = formats.nf4_offset()
    assert d == pytest.approx(0.5 * ((1 - 1 / 30) + (1 - 1 / 32)), abs=0)
    scale = norm.ppf(d)
    pos = np.sort(cb[cb > 0])
    neg = np.sort(-cb[cb < 0])
    p_pos = norm.cdf(pos * scale)
    p_neg = norm.cdf(neg * scale)
    assert np.allclose(p_pos, 0.5 + (d - 0.5) * np.arange(1, 9) / 8, atol=2e-7)
    assert np.allclose(p_neg, 0.5 + (d - 0.5) * np.arange(1, 8) / 7, atol=2e-7)


# --------------------------------------------------------------------------
# INT4 asymmetric
# --------------------------------------------------------------------------

def _int4_golden(golden_dir):
    return json.load(open(os.path.join(golden_dir, "int4_groups.json")))


def test_int4_quantize_golden_groups(golden_dir):
    g = _int4_golden(golden_dir)
    G = g["group_size"]
    w = np.array([grp["w"] for grp in g["groups"]], dtype=np.float32).reshape(1, -1)
    q, s, z = formats.int4_quantize(w, G)
    for i, grp in enumerate(g["groups"]):
        assert float(s[0, i]) == grp["scale"], grp["note"]
        assert float(z[0, i]) == grp["zero"], grp["note"]
        assert q[0, i * G:(i + 1) * G].tolist() == grp["q"], grp["note"]
    deq = formats.int4_dequant_exact(q, s, z, G)
    want = np.array([grp["dequant"] for grp in g["groups"]], dtype=np.float32).reshape(1, -1)
    assert np.array_equal(deq, want)


def test_int4_pack_golden(golden_dir):
    g = _int4_golden(golden_dir)["pack"]
    words = formats.int4_pack(np.array(g["codes"], dtype=np.uint8))
    assert words.reshape(-1).tolist() == g["words"]


def test_int4_pack_unpack_roundtrip():
    rng = np.random.default_rng(2)
    q = rng.integers(0, 16, size=(37, 256), dtype=np.uint8)
    assert np.array_equal(formats.int4_unpack(formats.int4_pack(q), 256), q)


def test_int4_quantize_properties():
    """Codes in range; zero point is the code of 0; error at most s/2 inside
    the range (round to nearest)."""
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((64, 512)) * 0.02).astype(np.float32)
    w[:, ::37] = 0.0
    q, s, z = formats.int4_quantize(w, 128)
    assert q.max() <= 15
    deq = formats.int4_dequant_exact(q, s, z, 128).astype(np.float64)
    s_full = np.repeat(s.astype(np.float64), 128, axis=1)
    # fp16 rounding of the scale can shrink the covered range by < 15 * ulp16(s)
    slack = 15 * s_full * 2.0 ** -11
    assert np.all(np.abs(deq - w) <= s_full / 2 + slack + 1e-12)
    # the range always includes 0, and 0 quantizes to the zero point exactly
    assert np.all(deq[:, ::37] == 0)


def test_int4_dequant_bf16_is_rne_of_exact():
    rng = np.random.default_rng(4)
    q = rng.integers(0, 16, size=(8, 256), dtype=np.uint8)
    s = (rng.random((8, 2)) * 0.01 + 1e-3).astype(np.float16)
    z = rng.integers(0, 16, size=(8, 2)).astype(np.float16)
    exact = (q.astype(np.float64) - np.repeat(z.astype(np.float64), 128, 1)) * np.repeat(
        s.astype(np.float64), 128, 1)
    want = torch.from_numpy(exact).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(formats.int4_dequant_bf16(q, s, z, 128), want)


# --------------------------------------------------------------------------
# NF4
# --------------------------------------------------------------------------

def _nf4_golden(golden_dir):
    return json.load(open(os.path.join(golden_dir, "nf4_blocks.json")))


def test_nf4_quantize_golden_block(golden_dir):
    g = _nf4_golden(golden_dir)
    head = np.array(g["block"]["w_head"], dtype=np.float32)
    w = np.zeros(128, dtype=np.float32)
    w[:head.size] = head
    codes, absmax = formats.nf4_quantize(w)
    assert float(absmax[0]) == g["block"]["absmax"]
    assert codes[:head.size].tolist() == g["block"]["codes_head"]
    assert np.all(codes[head.size:64] == 7)
    # second block is all zero
    assert float(absmax[1]) == g["zero_block"]["absmax"]
    assert np.all(codes[64:] == g["zero_block"]["codes"])


def test_nf4_quantize_is_nearest_brute_force():
    """Brute force on a small block set: the chosen code minimises the exact
    distance |u - c| over all 16 codes, ties to the lower index."""
    from fractions import Fraction
    cb = formats.nf4_codebook()
    rng = np.random.default_rng(5)
    w = (rng.standard_normal(64 * 6) * 0.02).astype(np.float32)
    # plant exact midpoints (ties) in the last block
    am = np.float32(1.0)
    w[-64:] = 0
    w[-64] = am
    for i in range(15):
        mid = (Fraction(float(cb[i])) + Fraction(float(cb[i + 1]))) / 2
        f = np.float32(float(mid))
        if Fraction(float(f)) == mid:
            w[-63 + i] = f
    codes, absmax = formats.nf4_quantize(w)
    blocks = w.reshape(-1, 64)
    for b in range(blocks.shape[0]):
        a = absmax[b]
        for j in range(64):
            u = Fraction(float(np.float32(blocks[b, j] / a))) if a != 0 else None
            if u is None:
                assert codes[b * 64 + j] == 7
                continue
            d = [abs(u - Fraction(float(c))) for c in cb]
            best = min(range(16), key=lambda i: (d[i], i))
            assert codes[b * 64 + j] == best


def test_nf4_pack_golden_and_roundtrip(golden_dir):
    g = _nf4_golden(golden_dir)["pack"]
    assert formats.nf4_pack(np.array(g["codes"], np.uint8)).tolist() == g["bytes"]
    rng = np.random.default_rng(6)
    c = rng.integers(0, 16, size=4096, dtype=np.uint8)
    assert np.array_equal(formats.nf4_unpack(formats.nf4_pack(c)), c)


def test_nf4_dequant_golden(golden_dir):
    cases = _nf4_golden(golden_dir)["dequant_bf16"]["cases"]
    codes = np.full(64 * len(cases), 7, dtype=np.uint8)
    absmax = np.zeros(len(cases), dtype=np.float32)
    for i, c in enumerate(cases):
        codes[i * 64] = c["code"]
        absmax[i] = c["absmax"]
    out = formats.nf4_dequant_bf16(codes, absmax)
    for i, c in enumerate(cases):
        assert float(out[i * 64]) == c["out"], c
        assert np.all(out[i * 64 + 1:(i + 1) * 64] == 0)


def test_nf4_dequant_fp32_is_single_rounding():
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 16, size=64 * 50, dtype=np.uint8)
    absmax = (rng.random(50) * 0.1).astype(np.float32)
    exact = formats.nf4_dequant_exact(codes, absmax)
    got = formats.nf4_dequant_fp32(codes, absmax)
    assert np.array_equal(got, exact.astype(np.float32))
    want16 = torch.from_numpy(got).to(torch.float16).to(torch.float32).numpy()
    assert np.array_equal(formats.nf4_dequant_fp16(codes, absmax), want16)


def test_nf4_memory_reduction():
    """Four times smaller than 16-bit storage, plus 4 bytes per 64 elements."""
    n = 64 * 1000
    packed = formats.nf4_pack(np.zeros(n, np.uint8))
    assert packed.nbytes * 4 == n * 2
