"""GPU parity of the decode GEMV against the fp64 oracle product.

All decode workloads (Llama-2-7B linear shapes, M = 1, 4, 8, 16, INT4 g128 and
NF4 b64, 1% outlier channels x20) and the tiny INT4 g64 case are run at full
size, every output compared. INT4 dequantizes exactly inside the kernel, so
besides the product tolerance every INT4 output must lie within one bf16
rounding of the exact product. NF4 multiplies exactly scaled fp16 activations
by the fp16 code values (each rounded once) and applies each block's absmax in
fp32 to the block's partial sum; its element bound keeps the 3e-3 RMS slack of
the GEMM's NF4 cases (the code rounding alone, at most 2^-11 relative per
weight, stays well inside it).
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


def _x(m, k, seed, outliers):
    from bit_weight_quantized_weights_b200 import workloads
    g = workloads.generator(seed + 1000)
    return workloads.activations(m, k, gen=g, outliers=outliers)


def _run_int4(wq, m, n, k, group, outliers=(0.01, 20.0), seed=0, exact_check=True):
    q, s, z, qweight = helpers.int4_packed(n, k, group, seed)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = _x(m, k, seed, outliers)
    y = wq.wq_w4a16_gemv(x.cuda(), n, wq.WQ_FMT_INT4_ASYM, group, qw, sc, zr)
    torch.cuda.synchronize()
    y_ref = products.w4a16_int4(helpers.x_f32(x), q, s, z, group)
    helpers.check_product(y, y_ref, "int4 gemv M=%d %dx%d" % (m, n, k))
    if exact_check:
        helpers.check_within_bf16_rounding(y, y_ref, "int4 gemv M=%d %dx%d" % (m, n, k))


def _run_nf4(wq, m, n, k, outliers=(0.01, 20.0), seed=0):
    codes, absmax, packed = helpers.nf4_packed(n, k, seed)
    cw, am = helpers.to_dev_nf4(absmax, packed)
    x = _x(m, k, seed, outliers)
    y = wq.wq_w4a16_gemv(x.cuda(), n, wq.WQ_FMT_NF4, 64, cw, am, None)
    torch.cuda.synchronize()
    y_ref = products.w4a16_nf4(helpers.x_f32(x), codes, absmax, k)
    # one fp16 rounding per weight (the code value, 2^-11 relative at most),
    # spread over the K-term sum
    helpers.check_within_bf16_rounding(y, y_ref, "nf4 gemv M=%d %dx%d" % (m, n, k), slack=3e-3)
    return helpers.check_product(y, y_ref, "nf4 gemv M=%d %dx%d" % (m, n, k))


def test_gemv_tiny_int4_g64(wq):
    """x [1 x 1024], W [1024 x 1024], INT4 with fp16 scale/zero per 64 inputs."""
    _run_int4(wq, 1, 1024, 1024, 64, outliers=None)


@pytest.mark.parametrize("n,k", [(4096, 4096), (11008, 4096), (4096, 11008)])
@pytest.mark.parametrize("m", [1, 4, 8, 16])
def test_gemv_decode_int4_g128(wq, m, n, k):
    _run_int4(wq, m, n, k, 128)


@pytest.mark.parametrize("n,k", [(4096, 4096), (11008, 4096), (4096, 11008)])
@pytest.mark.parametrize("m", [1, 4, 8, 16])
def test_gemv_decode_nf4(wq, m, n, k):
    _run_nf4(wq, m, n, k)


@pytest.mark.parametrize("m,n,k,group", [(3, 1040, 384, 128), (9, 144, 256, 256),
                                         (16, 16, 128, 128), (5, 2064, 1152, 64),
                                         (2, 528, 640, 640), (7, 1040, 768, 192)])
def test_gemv_ragged_and_groups(wq, m, n, k, group):
    """N not a multiple of the 128-row tile, odd M, groups larger than the
    128-wide unit, groups that straddle two units (G = 192), per-channel
    groups (G = K)."""
    _run_int4(wq, m, n, k, group, seed=m)


def test_gemv_more_tiles_than_resident_ctas(wq):
    """512 row tiles over a short K: more CTAs than fit on the GPU at once,
    so the launch needs several waves."""
    _run_int4(wq, 3, 65536, 256, 128, seed=5)


@pytest.mark.parametrize("m,n,k", [(3, 1040, 384), (13, 272, 1280)])
def test_gemv_ragged_nf4(wq, m, n, k):
    _run_nf4(wq, m, n, k, seed=m)


def _at_16_bytes(t):
    """A copy of t whose data starts 16 bytes past a 256-byte boundary: aligned
    as the ABI requires, but not to 32 or 64 bytes."""
    flat = t.contiguous().view(-1).view(torch.uint8)
    buf = torch.empty(flat.numel() + 256, dtype=torch.uint8, device=t.device)
    off = (16 - buf.data_ptr()) % 256
    out = buf[off:off + flat.numel()]
    out.copy_(flat)
    return out.view(t.dtype).view(t.shape)


@pytest.mark.parametrize("fmt", ["int4", "nf4"])
def test_gemv_operands_only_16_byte_aligned(wq, fmt):
    """Every operand 16 bytes past a 256-byte boundary: the kernel must not
    derive a lane's position (or its NF4 absmax block) from address bits
    above the ABI's 16-byte alignment."""
    m, n, k = 5, 1040, 640
    x = _x(m, k, 3, None)
    xd = _at_16_bytes(x.cuda())
    y = _at_16_bytes(torch.zeros(m, n, dtype=torch.bfloat16, device="cuda"))
    assert xd.data_ptr() % 32 == 16 and y.data_ptr() % 32 == 16
    if fmt == "int4":
        q, s, z, qweight = helpers.int4_packed(n, k, 128, seed=4)
        qw, sc, zr = (_at_16_bytes(t) for t in helpers.to_dev_int4(s, z, qweight))
        assert qw.data_ptr() % 32 == 16
        wq.wq_w4a16_gemv(xd, n, wq.WQ_FMT_INT4_ASYM, 128, qw, sc, zr, out=y)
        y_ref = products.w4a16_int4(helpers.x_f32(x), q, s, z, 128)
        slack = 1e-4
    else:
        codes, absmax, packed = helpers.nf4_packed(n, k, seed=4)
        cw, am = (_at_16_bytes(t) for t in helpers.to_dev_nf4(absmax, packed))
        assert cw.data_ptr() % 32 == 16 and am.data_ptr() % 32 == 16
        wq.wq_w4a16_gemv(xd, n, wq.WQ_FMT_NF4, 64, cw, am, None, out=y)
        y_ref = products.w4a16_nf4(helpers.x_f32(x), codes, absmax, k)
        slack = 3e-3
    torch.cuda.synchronize()
    helpers.check_product(y, y_ref, "%s gemv, 16-byte aligned operands" % fmt)
    helpers.check_within_bf16_rounding(y, y_ref, "%s gemv, 16-byte aligned operands" % fmt,
                                       slack=slack)


def test_gemv_empty_is_noop(wq):
    """M = 0 through the C ABI with real buffers: the call succeeds, writes
    nothing (y points at a sentinel buffer, which must stay untouched) and
    leaves no device error. (torch hands empty tensors a null pointer, so the
    pointers here are those of non-empty buffers.)"""
    xbuf = torch.zeros(1, 256, dtype=torch.bfloat16, device="cuda")
    sentinel = torch.full((4, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    qw = torch.zeros(64, 32, dtype=torch.int32, device="cuda")
    sc = torch.ones(64, 2, dtype=torch.float16, device="cuda")
    st = wq.lib.wq_w4a16_gemv(xbuf.data_ptr(), 0, 64, 256, wq.WQ_FMT_INT4_ASYM, 128,
                              qw.data_ptr(), sc.data_ptr(), sc.data_ptr(), sentinel.data_ptr(),
                              None, 0, None)
    assert st == wq.WQ_OK
    torch.cuda.synchronize()
    assert torch.all(sentinel == 7.0)
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)


def test_gemv_rejects_m17(wq):
    x = torch.zeros(17, 256, dtype=torch.bfloat16, device="cuda")
    qw = torch.zeros(64, 32, dtype=torch.int32, device="cuda")
    sc = torch.ones(64, 2, dtype=torch.float16, device="cuda")
    with pytest.raises(wq.WqError) as e:
        wq.wq_w4a16_gemv(x, 64, wq.WQ_FMT_INT4_ASYM, 128, qw, sc, sc)
    assert e.value.status == wq.WQ_ERR_UNSUPPORTED


def test_gemv_nan_propagates(wq):
    """A NaN activation makes that token's outputs NaN (documented behaviour)."""
    q, s, z, qweight = helpers.int4_packed(128, 256, 128, 9)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = torch.ones(2, 256, dtype=torch.bfloat16)
    x[1, 7] = float("nan")
    y = wq.wq_w4a16_gemv(x.cuda(), 128, wq.WQ_FMT_INT4_ASYM, 128, qw, sc, zr).cpu()
    assert torch.isfinite(y[0].float()).all() and torch.isnan(y[1].float()).all()


# NF4 layers whose block absmax spans many orders of magnitude: the whole
# layer tiny (absmax ~5e-8 and ~5e-11, below fp16's normal range), blocks
# spread over 1e-8 .. 1e3 within every row, and rows of 1e-9 .. 1e2, checked
# class by class so that the tiny rows are held to their own scale, every
# output against the dot product's forward error bound.
NF4_RANGE_CASES = {
    "layer_1e-6": dict(factor=1e-6),
    "layer_1e-9": dict(factor=1e-9),
    "blocks_1e-8_1e3": dict(block_exp=(-8, 3)),
    "rows_1e-9_1e2": dict(row_exp=(-9, 2)),
}


@pytest.mark.parametrize("case", sorted(NF4_RANGE_CASES))
@pytest.mark.parametrize("m", [1, 16])
def test_gemv_nf4_absmax_range(wq, case, m):
    from bit_weight_quantized_weights_b200 import workloads
    from oracle import formats
    n, k = 1024, 4096
    w = workloads.scaled_weights(n, k, seed=11, **NF4_RANGE_CASES[case]).numpy()
    codes, absmax = formats.nf4_quantize(w)
    cw, am = helpers.to_dev_nf4(absmax, formats.nf4_pack(codes))
    x = _x(m, k, 11, (0.01, 20.0))
    y = wq.wq_w4a16_gemv(x.cuda(), n, wq.WQ_FMT_NF4, 64, cw, am, None)
    torch.cuda.synchronize()
    xf = helpers.x_f32(x)
    y_ref = products.w4a16_nf4(xf, codes, absmax, k)
    w_abs = np.abs(formats.nf4_dequant_exact(codes, absmax).reshape(n, k))
    y_abs = products.matmul_exact(np.abs(xf), w_abs)
    # per weight: the code value rounds once to fp16 (x is exact in fp16, the
    # absmax is applied in fp32: one more rounding of a partial sum); fp32
    # accumulation adds at most K x 2^-23 relative of the sum of |terms|
    eps = helpers.FP16_U + k * 2.0 ** -23
    yc = y.cpu()
    classes = [np.arange(n)]
    if "row_exp" in NF4_RANGE_CASES[case]:
        lo, hi = NF4_RANGE_CASES[case]["row_exp"]
        classes = [np.arange(c, n, hi - lo + 1) for c in range(hi - lo + 1)]
    for cols in classes:
        what = "nf4 gemv %s M=%d rows %d.." % (case, m, cols[0])
        helpers.check_product(yc[:, cols], y_ref[:, cols], what)
        helpers.check_within_error_bound(yc[:, cols], y_ref[:, cols], y_abs[:, cols], eps, what)
