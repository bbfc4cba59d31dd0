"""GPU parity of the MX path of Multi-Scale Dequant (MXFP4 weights, two MXFP4
passes over the activations, or one MXFP8 pass as the comparator) against the
oracle: the weight codes and scales and the activation passes are bit-exact;
the decode product lies within one bf16 rounding of the oracle's exact
decomposed product (every MMA's block sum is exact; each block's scaled sum
rounds once in fp32), and against the undecomposed product the two-pass
result is reported beside the one-pass MXFP8 comparator."""

import numpy as np
import pytest
import torch

from oracle import mx
from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    import bit_weight_quantized_weights_b200 as pkg
    return pkg.binding


def _w(n, k, seed, scale_exp=None):
    from bit_weight_quantized_weights_b200 import workloads
    if scale_exp is None:
        return workloads.weights(n, k, seed=seed)
    return workloads.scaled_weights(n, k, seed=seed, block_exp=scale_exp)


def _x(m, k, seed):
    from bit_weight_quantized_weights_b200 import workloads
    return workloads.activations(m, k, gen=workloads.generator(seed + 6000), outliers=(0.005, 50.0))


@pytest.mark.parametrize("n,k,scale_exp", [(64, 256, None), (300, 1024, None), (128, 512, (-30, 20)),
                                           (5120, 5120, None)])
def test_mx_quantize_bit_exact(wq, n, k, scale_exp):
    w = _w(n, k, n + k, scale_exp)
    codes, scales = wq.wq_mx_quantize(w.cuda())
    torch.cuda.synchronize()
    c_ref, s_ref = mx.mx_quantize(w.numpy(), "fp4")
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), mx.pack_fp4(c_ref))


@pytest.mark.parametrize("m,k", [(1, 5120), (16, 5120), (3, 25600), (37, 1024)])
@pytest.mark.parametrize("passes", [1, 2])
def test_mx_decompose_bit_exact(wq, m, k, passes):
    x = _x(m, k, m + k)
    if m >= 3:
        x[1] = 0.0                                        # an all-zero row
        x[2, :32] = torch.tensor([6.0, 0.25, 0.75, -1.25, 1.75, 2.5, -3.5, 5.0] * 4)  # every tie
    planes, scales = wq.wq_mx_decompose(x.cuda(), passes)
    torch.cuda.synchronize()
    xf = x.float().numpy().astype(np.float64)
    if passes == 2:
        c_ref, s_ref, _ = mx.mxfp4_two_pass(xf)
        for p in range(2):
            got = mx.e4m3_decode(planes[p].cpu().numpy())
            assert np.array_equal(got, mx.e2m1_decode(c_ref[p]))
            assert np.array_equal(scales[p].cpu().numpy(), s_ref[p])
    else:
        c_ref, s_ref, _ = mx.mxfp8_one_pass(xf)
        assert np.array_equal(planes[0].cpu().numpy(), c_ref)
        assert np.array_equal(scales[0].cpu().numpy(), s_ref)


def _product_case(wq, m, n, k, passes, seed, rows=None, cols=None):
    w = _w(n, k, seed)
    codes, scales = wq.wq_mx_quantize(w.cuda())
    x = _x(m, k, seed)
    y = wq.wq_mx_gemv(x.cuda(), n, passes, codes, scales)
    torch.cuda.synchronize()
    wc, ws = mx.mx_quantize(w.numpy(), "fp4")
    xf = x.float().numpy().astype(np.float64)
    x_hat = mx.mxfp4_two_pass(xf)[2] if passes == 2 else mx.mxfp8_one_pass(xf)[2]
    rows = np.arange(m) if rows is None else rows
    cols = np.arange(n) if cols is None else cols
    y_dec = mx.mx_product(x_hat[rows], wc[cols], ws[cols])
    yg = y.cpu()[rows][:, cols]
    helpers.check_within_bf16_rounding(yg, y_dec, "mx P=%d M=%d %dx%d" % (passes, m, n, k),
                                       slack=1e-4)
    y_exact = xf[rows] @ mx.mx_dequant(wc[cols], ws[cols], "fp4").T
    return yg, y_exact


@pytest.mark.parametrize("m,n,k", [(1, 128, 256), (16, 256, 1024), (5, 1040, 512),
                                   (9, 384, 2560), (16, 2048, 768)])
@pytest.mark.parametrize("passes", [1, 2])
def test_mx_gemv_every_element(wq, m, n, k, passes):
    _product_case(wq, m, n, k, passes, seed=m + n)


@pytest.mark.parametrize("n,k", [(5120, 5120), (25600, 5120), (5120, 25600)])
@pytest.mark.parametrize("m", [1, 16])
def test_mx_gemv_qwen_shapes_sampled(wq, m, n, k):
    rng = np.random.default_rng(m + n + k)
    cols = np.sort(rng.choice(n, 256, replace=False))
    y2, ex = _product_case(wq, m, n, k, 2, seed=1, cols=cols)
    y1, _ = _product_case(wq, m, n, k, 1, seed=1, cols=cols)
    from oracle import numerics
    r2, _ = numerics.compare(y2.float().numpy(), ex)
    r1, _ = numerics.compare(y1.float().numpy(), ex)
    print("relative L2 against the undecomposed product: two MXFP4 passes %.3e, one MXFP8 "
          "pass %.3e" % (r2, r1))


def test_mx_gemv_empty_and_validation(wq):
    x = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    c = torch.zeros(16, 128, dtype=torch.uint8, device="cuda")
    s = torch.zeros(16, 8, dtype=torch.uint8, device="cuda")
    y = wq.wq_mx_gemv(x, 16, 2, c, s, workspace=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert y.shape == (0, 16)
