"""GPU parity of the salient-channel residual correction against the oracle.

"DecDEC: A Systems Approach to Advancing Low-Bit LLM Quantization", Abstract.

- The residual R^T and the selected channel set are integer and bit work, and
  are compared bit for bit.
- The corrected GEMV is compared with the oracle's fp64 corrected product,
  under the product tolerance and the same element bound as the plain GEMV of
  the same format. The correction adds k fp32 products to each output before
  its bf16 rounding.
"""

import numpy as np
import pytest
import torch

from oracle import decdec, formats
from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    import bit_weight_quantized_weights_b200 as pkg
    return pkg.binding


def _w(n, k, seed):
    from bit_weight_quantized_weights_b200 import workloads
    return workloads.weights(n, k, seed=seed).numpy()


def _x(m, k, seed, outliers=(0.01, 20.0)):
    from bit_weight_quantized_weights_b200 import workloads
    return workloads.activations(m, k, gen=workloads.generator(seed + 3000), outliers=outliers)


def _int4(n, k, group, seed):
    w = _w(n, k, seed)
    q, s, z = formats.int4_quantize(w, group)
    return w, q, s, z, formats.int4_pack(q)


def _nf4(n, k, seed):
    w = _w(n, k, seed)
    codes, absmax = formats.nf4_quantize(w)
    return w, codes, absmax, formats.nf4_pack(codes)


def _bits16(t):
    return t.cpu().view(torch.int16).numpy().astype(np.uint16)


@pytest.mark.parametrize("n,k,group", [(1040, 640, 128), (48, 256, 64), (11008, 4096, 128)])
def test_int4_residual_bit_exact(wq, n, k, group):
    w, q, s, z, qweight = _int4(n, k, group, seed=n)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    rt = wq.wq_residual(wq.WQ_FMT_INT4_ASYM, torch.from_numpy(w).cuda(), group, qw, sc, zr)
    ref = decdec.int4_residual_t(w, q, s, z, group)
    assert np.array_equal(_bits16(rt), ref.view(np.uint16))


@pytest.mark.parametrize("n,k", [(1040, 640), (4096, 4096)])
def test_nf4_residual_bit_exact(wq, n, k):
    w, codes, absmax, packed = _nf4(n, k, seed=n)
    cw, am = helpers.to_dev_nf4(absmax, packed)
    rt = wq.wq_residual(wq.WQ_FMT_NF4, torch.from_numpy(w).cuda(), 64, cw, am, None)
    ref = decdec.nf4_residual_t(w, codes, absmax)
    assert np.array_equal(_bits16(rt), ref.view(np.uint16))


@pytest.mark.parametrize("m,k,nsel", [(1, 4096, 1), (1, 4096, 64), (16, 4096, 41),
                                      (5, 11008, 110), (16, 11008, 11008), (3, 640, 600),
                                      (1, 65536, 256)])
def test_select_salient_matches_oracle(wq, m, k, nsel):
    x = _x(m, k, seed=k + m)
    got = wq.wq_select_salient(x.cuda(), nsel).cpu().numpy()
    ref = decdec.select_salient(x.float().numpy(), nsel)
    assert np.array_equal(got, ref)


def test_select_salient_ties_nan_inf(wq):
    """Equal magnitudes of both signs (lower channel wins), an infinite and a
    NaN activation (NaN ranks first), in a channel count that is not a
    multiple of the CTA's threads."""
    m, k = 4, 3001
    x = _x(m, k, seed=9, outliers=None).float()
    x[:, 100:400] = 1.5                # 300 equal keys
    x[2, 150:250] = -1.5
    x[1, 7] = float("inf")
    x[3, 2999] = float("nan")
    x = x.to(torch.bfloat16)
    for nsel in (1, 2, 3, 50, 301, 302, 1000, k):
        got = wq.wq_select_salient(x.cuda(), nsel).cpu().numpy()
        ref = decdec.select_salient(x.float().numpy(), nsel)
        assert np.array_equal(got, ref), nsel


def _corrected_case(wq, fmt, m, n, k, nsel, seed, group=128):
    x = _x(m, k, seed)
    xd = x.cuda()
    xf = helpers.x_f32(x)
    if fmt == "int4":
        w, q, s, z, qweight = _int4(n, k, group, seed)
        qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
        rt = wq.wq_residual(wq.WQ_FMT_INT4_ASYM, torch.from_numpy(w).cuda(), group, qw, sc, zr)
        idx = wq.wq_select_salient(xd, nsel)
        y = wq.wq_w4a16_gemv_corrected(xd, n, wq.WQ_FMT_INT4_ASYM, group, qw, sc, zr, rt, idx)
        ref_rt = decdec.int4_residual_t(w, q, s, z, group)
        ref_idx = decdec.select_salient(xf, nsel)
        y_ref = decdec.int4_corrected(xf, q, s, z, group, ref_rt, ref_idx)
        y_base = decdec.int4_corrected(xf, q, s, z, group, ref_rt, ref_idx[:0])
        slack = 1e-4
    else:
        w, codes, absmax, packed = _nf4(n, k, seed)
        cw, am = helpers.to_dev_nf4(absmax, packed)
        rt = wq.wq_residual(wq.WQ_FMT_NF4, torch.from_numpy(w).cuda(), 64, cw, am, None)
        idx = wq.wq_select_salient(xd, nsel)
        y = wq.wq_w4a16_gemv_corrected(xd, n, wq.WQ_FMT_NF4, 64, cw, am, None, rt, idx)
        ref_rt = decdec.nf4_residual_t(w, codes, absmax)
        ref_idx = decdec.select_salient(xf, nsel)
        y_ref = decdec.nf4_corrected(xf, codes, absmax, k, ref_rt, ref_idx)
        y_base = decdec.nf4_corrected(xf, codes, absmax, k, ref_rt, ref_idx[:0])
        slack = 3e-3
    torch.cuda.synchronize()
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)
    what = "%s corrected gemv M=%d %dx%d k=%d" % (fmt, m, n, k, nsel)
    helpers.check_product(y, y_ref, what)
    helpers.check_within_bf16_rounding(y, y_ref, what, slack=slack)
    return y, y_ref, y_base, w, xf


@pytest.mark.parametrize("fmt", ["int4", "nf4"])
@pytest.mark.parametrize("m,n,k,nsel", [(1, 11008, 4096, 64), (16, 11008, 4096, 64),
                                        (4, 4096, 11008, 110), (3, 1040, 640, 640),
                                        (2, 1040, 640, 0)])
def test_corrected_gemv_matches_oracle(wq, fmt, m, n, k, nsel):
    _corrected_case(wq, fmt, m, n, k, nsel, seed=m + nsel)


@pytest.mark.parametrize("fmt", ["int4", "nf4"])
@pytest.mark.parametrize("m,n,k,nsel", [(1, 11008, 4096, 64), (16, 11008, 4096, 64),
                                        (4, 4096, 11008, 110), (3, 1040, 640, 640)])
def test_salient_step_matches_oracle(wq, fmt, m, n, k, nsel):
    """Selection and corrected GEMV in one call, the GEMV launched to overlap
    the selection: same result as the oracle's corrected product, and the
    channel set written to the scratch equals the oracle's."""
    seed = m + nsel + 5
    x = _x(m, k, seed)
    xd = x.cuda()
    xf = helpers.x_f32(x)
    if fmt == "int4":
        w, q, s, z, qweight = _int4(n, k, 128, seed)
        pk = helpers.to_dev_int4(s, z, qweight)
        f, g = wq.WQ_FMT_INT4_ASYM, 128
        ref_rt = decdec.int4_residual_t(w, q, s, z, 128)
        ref_idx = decdec.select_salient(xf, nsel)
        y_ref = decdec.int4_corrected(xf, q, s, z, 128, ref_rt, ref_idx)
        slack = 1e-4
    else:
        w, codes, absmax, packed = _nf4(n, k, seed)
        cw, am = helpers.to_dev_nf4(absmax, packed)
        pk = (cw, am, None)
        f, g = wq.WQ_FMT_NF4, 64
        ref_rt = decdec.nf4_residual_t(w, codes, absmax)
        ref_idx = decdec.select_salient(xf, nsel)
        y_ref = decdec.nf4_corrected(xf, codes, absmax, k, ref_rt, ref_idx)
        slack = 3e-3
    rt = wq.wq_residual(f, torch.from_numpy(w).cuda(), g, *pk)
    idx = torch.full((nsel,), -1, dtype=torch.int32, device="cuda")
    y = wq.wq_w4a16_gemv_salient(xd, n, f, g, *pk, rt, nsel, idx=idx)
    torch.cuda.synchronize()
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    what = "%s salient step M=%d %dx%d k=%d" % (fmt, m, n, k, nsel)
    helpers.check_product(y, y_ref, what)
    helpers.check_within_bf16_rounding(y, y_ref, what, slack=slack)


@pytest.mark.parametrize("m,n,k,nsel", [(3, 1040, 640, 40), (16, 2064, 1152, 100)])
def test_corrected_gemv_int4_g64(wq, m, n, k, nsel):
    """The 8-byte-load GEMV (INT4 groups of 64) with the correction."""
    _corrected_case(wq, "int4", m, n, k, nsel, seed=m, group=64)


@pytest.mark.parametrize("fmt", ["int4", "nf4"])
def test_correction_moves_toward_full_precision(wq, fmt):
    """With the outlier channels' residuals added back, the GPU result is
    closer to the full-precision product x . W^T than without them. This is
    the property the page claims, measured here on the synthetic outlier
    workload."""
    y, y_ref, y_base, w, xf = _corrected_case(wq, fmt, 1, 11008, 4096, 64, seed=21)
    y_full = xf.astype(np.float64) @ w.astype(np.float64).T
    err_gpu = np.linalg.norm(y.float().cpu().numpy() - y_full)
    err_base = np.linalg.norm(y_base - y_full)
    assert err_gpu < 0.9 * err_base, (err_gpu, err_base)
