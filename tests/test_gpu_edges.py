"""Degenerate inputs on every product path: empty problems, all-zero
activation rows, all-zero weight groups (the quantizer's +-1 range rule),
NaN activations in the GEMM, and zero-length dequantization."""

import numpy as np
import pytest
import torch

from oracle import formats, msd, numerics, products
from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from bit_weight_quantized_weights_b200 import binding
    return binding


def _degenerate_weights(n, k, group, seed):
    """N(0, 0.02) weights with group 0 of row 0 and the whole of row 1 zero."""
    from bit_weight_quantized_weights_b200 import workloads
    w = workloads.weights(n, k, seed=seed).numpy().copy()
    w[0, :group] = 0.0
    w[1, :] = 0.0
    q, s, z = formats.int4_quantize(w, group)
    return q, s, z, formats.int4_pack(q)


def _x_with_zero_row(m, k, seed):
    from bit_weight_quantized_weights_b200 import workloads
    x = workloads.activations(m, k, gen=workloads.generator(seed)).clone()
    x[0] = 0
    return x


def test_empty_problems_are_noops(wq):
    qw = torch.zeros(128, 32, dtype=torch.int32, device="cuda")
    sc = torch.ones(128, 2, dtype=torch.float16, device="cuda")
    x = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    y = torch.full((0, 128), 3.0, dtype=torch.bfloat16, device="cuda")
    wq.wq_w4a16_gemm(x, 128, wq.WQ_FMT_INT4_ASYM, 128, qw, sc, sc, workspace=None, out=y)
    wq.wq_msd_gemm(x, 128, 2, 128, qw, sc, sc, workspace=None, out=y)
    codes = torch.zeros(0, dtype=torch.uint8, device="cuda")
    absmax = torch.zeros(0, dtype=torch.float32, device="cuda")
    out = torch.empty(0, dtype=torch.bfloat16, device="cuda")
    wq.wq_nf4_dequant(codes, absmax, 0, out=out)
    torch.cuda.synchronize()
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)


@pytest.mark.parametrize("path", ["gemv", "gemm", "msd_decode", "msd_tiles"])
def test_zero_rows_and_zero_groups(wq, path):
    """A zero activation row gives a zero output row; a zero weight group
    dequantizes to exact zeros (range [-1, 1], zero point 8) and adds nothing."""
    m = {"gemv": 5, "gemm": 140, "msd_decode": 7, "msd_tiles": 140}[path]
    n, k, group = 256, 512, 128
    q, s, z, qweight = _degenerate_weights(n, k, group, seed=3)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = _x_with_zero_row(m, k, 3)
    xf = helpers.x_f32(x)
    if path == "gemv":
        y = wq.wq_w4a16_gemv(x.cuda(), n, wq.WQ_FMT_INT4_ASYM, group, qw, sc, zr)
        y_ref = products.w4a16_int4(xf, q, s, z, group)
    elif path == "gemm":
        y = wq.wq_w4a16_gemm(x.cuda(), n, wq.WQ_FMT_INT4_ASYM, group, qw, sc, zr)
        y_ref = products.w4a16_int4(xf, q, s, z, group)
    else:
        y = wq.wq_msd_gemm(x.cuda(), n, 2, group, qw, sc, zr)
        a, sa = msd.decompose(xf, 2)
        y_ref = msd.msd_product(a, sa, q, s, z, group)
    torch.cuda.synchronize()
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)
    y = y.cpu()
    # the oracle's own degenerate-group reading: scale 2/15, zero 8, codes 8
    assert np.all(q[1] == 8) and np.all(q[0, :group] == 8)
    assert torch.count_nonzero(y[0]) == 0, "zero activation row"
    if path == "gemv":
        # post-group form s * (P - (128 + z) * sum(x)): P and sum(x) are fp32
        # sums, so an all-zero weight row leaves a rounding residue of order
        # 2^-24 * (128 + z) * sum|x| instead of an exact zero
        rms = float(np.sqrt(np.mean(y_ref ** 2)))
        assert float(y[:, 1].float().abs().max()) <= 1e-3 * rms, "zero weight row"
    else:
        # the dequantized weight (q - z) * s is exactly zero on these paths
        assert torch.count_nonzero(y[:, 1]) == 0, "zero weight row"
    helpers.check_within_bf16_rounding(y, y_ref, path, slack=1e-3)


def test_gemm_nan_row_stays_in_its_row(wq):
    """A NaN activation makes that token's outputs NaN and leaves the other
    tokens finite (the per-row fp16 scaling ignores it when taking the row's
    largest magnitude)."""
    m, n, k, group = 130, 256, 256, 128
    q, s, z, qweight = helpers.int4_packed(n, k, group, seed=9)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = torch.ones(m, k, dtype=torch.bfloat16)
    x[7, 5] = float("nan")
    y = wq.wq_w4a16_gemm(x.cuda(), n, wq.WQ_FMT_INT4_ASYM, group, qw, sc, zr).cpu()
    assert torch.isnan(y[7]).all()
    rest = torch.cat([y[:7], y[8:]])
    assert torch.isfinite(rest).all()
    y_ref = products.w4a16_int4(np.ones((1, k), np.float32), q, s, z, group)
    helpers.check_within_bf16_rounding(y[:1], y_ref, "gemm ones row", slack=1e-3)


def test_nf4_dequant_zero_blocks(wq):
    """An all-zero block stores absmax 0 and code 7 (the exact zero of the
    codebook); it dequantizes to +0.0 exactly."""
    from bit_weight_quantized_weights_b200 import workloads
    w = workloads.weights(4, 256, seed=2).numpy().copy()
    w[1, 64:128] = 0.0
    codes, absmax = formats.nf4_quantize(w)  # flattened row-major blocks of 64
    assert absmax[1 * 4 + 1] == 0 and np.all(codes[256 + 64:256 + 128] == 7)
    packed = formats.nf4_pack(codes)
    cw, am = helpers.to_dev_nf4(absmax, packed)
    out = wq.wq_nf4_dequant(cw, am, w.size).cpu()
    ref = numerics.bf16_bits(formats.nf4_dequant_exact(codes, absmax))
    got = out.view(torch.int16).numpy().astype(np.uint16).reshape(ref.shape)
    assert np.array_equal(got, ref)
