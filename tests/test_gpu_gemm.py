"""GPU parity of the tcgen05 prefill GEMM (fused INT4 dequantization).

Small cases (several tiles in M, N and K, ragged M, every group size the
kernel supports) compare every output with the fp64 oracle; the full prefill
workloads (M = 512, 2048, 8192 x Llama-3-8B shapes, INT4 g128) compare sampled
rows x columns computed one by one by the oracle. The kernel multiplies in
fp16 (x exact after a per-row power-of-two scaling, each weight rounded once
to fp16), so besides the product tolerance every output must lie within one
bf16 rounding of the exact product (plus 1e-3 of its RMS for the fp16 weight
rounding and fp32 accumulation).
"""

import numpy as np
import pytest
import torch

from oracle import products
from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    import bit_weight_quantized_weights_b200 as pkg
    return pkg.binding


def _x(m, k, seed):
    from bit_weight_quantized_weights_b200 import workloads
    return workloads.activations(m, k, gen=workloads.generator(seed + 2000))


@pytest.mark.parametrize("m,n,k,group", [
    (128, 256, 256, 128),     # one 128x128 tile column pair, 4 k-tiles
    (300, 384, 640, 128),     # ragged M, N not a multiple of 256, ring wraps (10 k-tiles)
    (1, 128, 128, 64),        # one row
    (257, 512, 1024, 1024),   # per-channel groups
    (64, 256, 512, 64),       # M below one tile
    (600, 12800, 256, 128),   # CTA-pair tiles (256 rows x 256 tokens), ragged M
    (384, 9344, 256, 64),     # 128-token tiles (too few 256-token tiles to fill the GPU)
    (600, 12928, 256, 128),   # single-CTA 256-token tiles (N not a multiple of 256)
    (520, 9472, 1024, 64),    # CTA pairs, the 8-stage ring wraps twice, ragged M
    (512, 18944, 512, 512),   # CTA pairs, per-group parameters across several k-tiles
    # the persistent pair kernel (two or more 256 x 256 tiles per pair of CTAs):
    (1100, 8192, 512, 128),   # ragged last token tile, several tiles per pair
    (1024, 9472, 384, 384),   # per-channel groups (three k-tiles per group)
])
def test_gemm_small_every_element(wq, m, n, k, group):
    q, s, z, qweight = helpers.int4_packed(n, k, group, seed=m)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = _x(m, k, m)
    y = wq.wq_w4a16_gemm(x.cuda(), n, wq.WQ_FMT_INT4_ASYM, group, qw, sc, zr)
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)
    y_ref = products.w4a16_int4(helpers.x_f32(x), q, s, z, group)
    helpers.check_product(y, y_ref, "gemm %dx%dx%d g%d" % (m, n, k, group))
    helpers.check_within_bf16_rounding(y, y_ref, "gemm %dx%dx%d g%d" % (m, n, k, group),
                                       slack=EVERY_ELEMENT_SLACK)


# Each dequantized weight is rounded once to fp16, a relative error of at most
# 2^-11 (uniform within that, standard deviation ~2^-11/sqrt(3) = 2.8e-4). Over
# the K products of one output these errors add like independent terms, so
# the output error has a standard deviation of ~2.8e-4 of the output RMS; the
# largest of ~10^7 outputs sits near 5.3 standard deviations, ~1.5e-3 RMS.
# 2e-3 (7 standard deviations) bounds every element of these cases; the bf16
# rounding of the output is the bound's other term.
EVERY_ELEMENT_SLACK = 2e-3


@pytest.mark.parametrize("n,k", [(4096, 4096), (14336, 4096), (4096, 14336)])
@pytest.mark.parametrize("m", [512, 2048, 8192])
def test_gemm_prefill_full_size_sampled(wq, m, n, k):
    q, s, z, qweight = helpers.int4_packed(n, k, 128, seed=0)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = _x(m, k, 0)
    y = wq.wq_w4a16_gemm(x.cuda(), n, wq.WQ_FMT_INT4_ASYM, 128, qw, sc, zr)
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)
    rng = np.random.default_rng(m + n + k)
    rows = np.sort(rng.choice(m, 48, replace=False))
    cols = np.sort(rng.choice(n, 192, replace=False))
    ys = y.cpu()[rows][:, cols]
    y_ref = products.w4a16_int4(helpers.x_f32(x)[rows], q[cols], s[cols], z[cols], 128)
    helpers.check_product(ys, y_ref, "gemm %dx%dx%d sampled" % (m, n, k))
    helpers.check_within_bf16_rounding(ys, y_ref, "gemm %dx%dx%d sampled" % (m, n, k),
                                       slack=1e-3)


def test_gemm_large_activation_range(wq):
    """Rows whose magnitudes span many binades (and one beyond the fp16 range)
    still multiply exactly: the per-row power-of-two scaling keeps them exact."""
    m, n, k, group = 130, 256, 512, 128
    q, s, z, qweight = helpers.int4_packed(n, k, group, seed=77)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = _x(m, k, 77).float()
    x[0] *= 1e5          # beyond fp16's range before scaling
    x[1] *= 1e-6         # far below it
    x[2, ::3] *= 1e-3
    x = x.to(torch.bfloat16)
    y = wq.wq_w4a16_gemm(x.cuda(), n, wq.WQ_FMT_INT4_ASYM, group, qw, sc, zr)
    y_ref = products.w4a16_int4(helpers.x_f32(x), q, s, z, group)
    for r in range(3):
        helpers.check_within_bf16_rounding(y[r:r + 1], y_ref[r:r + 1], "row %d" % r, slack=1e-3)
    helpers.check_within_bf16_rounding(y[3:], y_ref[3:], "rest", slack=1e-3)


def test_dequant_then_cublas_comparator(wq):
    """The dequantize-then-bf16-GEMM comparator: the library's INT4 dequant to
    bf16, then torch.matmul (cuBLAS). Its result matches the oracle's model of
    that baseline (bf16-rounded weights, exact product) within one output
    rounding plus the fp32 accumulation, and the exact product within the
    product tolerance."""
    m, n, k, group = 256, 512, 1024, 128
    q, s, z, qweight = helpers.int4_packed(n, k, group, seed=11)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = _x(m, k, 11)
    wd = wq.wq_int4_dequant(qw, sc, zr, n, k, group)
    y = torch.matmul(x.cuda(), wd.t()).cpu()
    xf = helpers.x_f32(x)
    y_model = products.dequant_then_bf16_matmul_int4(xf, q, s, z, group)
    helpers.check_within_bf16_rounding(y, y_model, "dequant-then-cuBLAS vs its model", slack=1e-3)
    helpers.check_product(y, products.w4a16_int4(xf, q, s, z, group), "dequant-then-cuBLAS")


def _run_nf4_gemm(wq, m, n, k, seed, rows=None, cols=None):
    codes, absmax, packed = helpers.nf4_packed(n, k, seed)
    cw, am = helpers.to_dev_nf4(absmax, packed)
    x = _x(m, k, seed)
    y = wq.wq_w4a16_gemm(x.cuda(), n, wq.WQ_FMT_NF4, 64, cw, am, None)
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)
    xf = helpers.x_f32(x)
    if rows is None:
        rows = np.arange(m)
    if cols is None:
        cols = np.arange(n)
    codes2 = codes.reshape(n, k)
    y_ref = products.w4a16_nf4(xf[rows], codes2[cols], absmax.reshape(n, k // 64)[cols], k)
    ys = y.cpu()[rows][:, cols]
    what = "nf4 gemm %dx%dx%d" % (m, n, k)
    helpers.check_product(ys, y_ref, what)
    # codebook value, absmax and their product each round once to fp16
    # (2^-11 relative): about 2^-10.2 per weight, which spreads over the sum
    helpers.check_within_bf16_rounding(ys, y_ref, what, slack=3e-3)


@pytest.mark.parametrize("m,n,k", [(128, 256, 256), (300, 384, 640), (1, 128, 128),
                                   (600, 12800, 256), (600, 12928, 256), (520, 9472, 1024)])
def test_gemm_nf4_small_every_element(wq, m, n, k):
    """NF4 weights on the fused GEMM: ragged M, several k-tiles, one token,
    and enough tiles for both tile widths and for CTA pairs."""
    _run_nf4_gemm(wq, m, n, k, seed=m)


@pytest.mark.parametrize("m,n,k", [(2048, 14336, 4096), (8192, 4096, 14336)])
def test_gemm_nf4_full_size_sampled(wq, m, n, k):
    rng = np.random.default_rng(m + n + k + 64)
    rows = np.sort(rng.choice(m, 48, replace=False))
    cols = np.sort(rng.choice(n, 192, replace=False))
    _run_nf4_gemm(wq, m, n, k, seed=1, rows=rows, cols=cols)


# NF4 layers whose block absmax spans many orders of magnitude (see the GEMV
# test of the same name): the per-row power of two must keep every row's
# products in fp16's normal range. Rows are checked class by class, every
# output against the dot product's forward error bound.
NF4_RANGE_CASES = {
    "layer_1e-6": dict(factor=1e-6),
    "layer_1e-9": dict(factor=1e-9),
    "layer_1e4": dict(factor=1e4),
    "blocks_1e-8_1e3": dict(block_exp=(-8, 3)),
    "rows_1e-9_1e2": dict(row_exp=(-9, 2)),
}


@pytest.mark.parametrize("case", sorted(NF4_RANGE_CASES))
@pytest.mark.parametrize("m,n,k", [(300, 384, 640), (520, 9472, 1024)])
def test_gemm_nf4_absmax_range(wq, case, m, n, k):
    from bit_weight_quantized_weights_b200 import workloads
    from oracle import formats
    w = workloads.scaled_weights(n, k, seed=12, **NF4_RANGE_CASES[case]).numpy()
    codes, absmax = formats.nf4_quantize(w)
    cw, am = helpers.to_dev_nf4(absmax, formats.nf4_pack(codes))
    x = _x(m, k, 12)
    ws = wq.gemm_workspace(m, n, k, 64)
    y = wq.wq_w4a16_gemm(x.cuda(), n, wq.WQ_FMT_NF4, 64, cw, am, None, workspace=ws)
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)
    xf = helpers.x_f32(x)
    y_ref = products.w4a16_nf4(xf, codes, absmax, k)
    w_abs = np.abs(formats.nf4_dequant_exact(codes, absmax).reshape(n, k))
    y_abs = products.matmul_exact(np.abs(xf), w_abs)
    # per weight: the code value, absmax x 2^e and their product each round
    # once to fp16 (x is exact in fp16); fp32 accumulation adds at most
    # K x 2^-23 relative of the sum of |terms|
    eps = 3 * helpers.FP16_U + k * 2.0 ** -23
    yc = y.cpu()
    classes = [np.arange(n)]
    if "row_exp" in NF4_RANGE_CASES[case]:
        lo, hi = NF4_RANGE_CASES[case]["row_exp"]
        classes = [np.arange(c, n, hi - lo + 1) for c in range(hi - lo + 1)]
    for cols in classes:
        what = "nf4 gemm %s %dx%dx%d rows %d.." % (case, m, n, k, cols[0])
        helpers.check_product(yc[:, cols], y_ref[:, cols], what)
        helpers.check_within_error_bound(yc[:, cols], y_ref[:, cols], y_abs[:, cols], eps, what)


def test_gemm_tiny_activations_beside_large(wq):
    """The fp16 copy of x scales each row so its largest value lands in
    [2^14, 2^15): bf16 values more than 2^28 below it become 0. A row with one
    large value and the rest 2^-29 .. 2^-31 of it (all flushed), a row with
    values spread over 2^-20 .. 1 of its largest, and plain rows all stay
    within the product tolerance and one bf16 rounding."""
    m, n, k, group = 130, 256, 512, 128
    q, s, z, qweight = helpers.int4_packed(n, k, group, seed=21)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = _x(m, k, 21).float()
    g = torch.Generator().manual_seed(21)
    x[0] = 1000.0 * torch.randn(k, generator=g) * 2.0 ** -30
    x[0, 7] = 1000.0
    x[1] = torch.randn(k, generator=g) * torch.pow(2.0, -20.0 * torch.rand(k, generator=g))
    x = x.to(torch.bfloat16)
    y = wq.wq_w4a16_gemm(x.cuda(), n, wq.WQ_FMT_INT4_ASYM, group, qw, sc, zr)
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)
    y_ref = products.w4a16_int4(helpers.x_f32(x), q, s, z, group)
    for rows in (np.array([0]), np.array([1]), np.arange(2, m)):
        what = "gemm tiny-x rows %d.." % rows[0]
        helpers.check_product(y[rows], y_ref[rows], what)
        helpers.check_within_bf16_rounding(y[rows], y_ref[rows], what, slack=EVERY_ELEMENT_SLACK)
