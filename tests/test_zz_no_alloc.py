"""The allocation-free Multi-Scale Dequant entry point (wq_msd_gemm_noalloc).

Some callers cannot give the library device memory at call time (a fixed
memory budget carved up at start-up, a plugin interface without a workspace
argument, a loop where allocation is forbidden). The no-allocation variant
keeps its scratch in a fixed device array inside the library. This test calls
it through the C ABI twice in a row (then a third time), with different
problem sizes, so each call runs over the previous call's leftovers in that
array. Each result is checked against the CPU oracle (the decomposed product
within one bf16 rounding, and the exact product under the product
tolerance), and must equal wq_msd_gemm's result bit for bit, since both run
the same kernels on the same data. The cases cover the tcgen05 tile kernel
(M > 16) and the decode kernel (M <= 16, whose digit planes are padded to
128 rows inside the array). The file is named to run last.
"""

import ctypes

import numpy as np
import pytest
import torch

from oracle import msd, products
from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    import bit_weight_quantized_weights_b200 as pkg
    return pkg.binding


def _inputs(m, n, k, group, seed):
    from bit_weight_quantized_weights_b200 import workloads
    q, s, z, qweight = helpers.int4_packed(n, k, group, seed=seed)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = workloads.activations(m, k, gen=workloads.generator(seed + 4000),
                              outliers=(0.005, 50.0))
    return x, (q, s, z), (qw, sc, zr)


def _noalloc(wq, x, n, c, group, qw, sc, zr):
    m, k = x.shape
    y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device=x.device)
    st = wq.lib.wq_msd_gemm_noalloc(
        ctypes.c_void_p(x.data_ptr()), m, n, k, c, group, ctypes.c_void_p(qw.data_ptr()),
        ctypes.c_void_p(sc.data_ptr()), ctypes.c_void_p(zr.data_ptr()),
        ctypes.c_void_p(y.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == wq.WQ_OK, wq.status_string(st)
    return y


def test_noalloc_matches_oracle_and_workspace_entry_point(wq):
    # (M, N, K, group, C, seed): tcgen05 tiles with g128; tcgen05 tiles with a
    # per-channel group and three components; the decode kernel (M = 8)
    cases = [(128, 512, 5120, 128, 2, 1), (37, 384, 2560, 2560, 3, 2), (8, 1024, 5120, 128, 2, 3)]
    for m, n, k, group, c, seed in cases:
        x, (q, s, z), (qw, sc, zr) = _inputs(m, n, k, group, seed)
        xd = x.cuda()
        y = _noalloc(wq, xd, n, c, group, qw, sc, zr)
        y_ws = wq.wq_msd_gemm(xd, n, c, group, qw, sc, zr)
        torch.cuda.synchronize()
        st, detail = wq.wq_device_error()
        assert st == wq.WQ_OK, hex(detail)
        what = "noalloc M=%d N=%d K=%d g%d C=%d" % (m, n, k, group, c)
        assert torch.equal(y.view(torch.int16), y_ws.view(torch.int16)), what + " vs msd_gemm"
        xf = helpers.x_f32(x)
        a, sa = msd.decompose(xf, c)
        y_dec = msd.msd_product(a, sa, q, s, z, group)
        helpers.check_within_bf16_rounding(y.cpu(), y_dec, what + " vs decomposed", slack=1e-4)
        helpers.check_product(y, products.w4a16_int4(xf, q, s, z, group), what + " vs exact")


def test_noalloc_rejects_problems_beyond_its_scratch(wq):
    m, n, k, group = 1024, 128, 5120, 128      # needs ~10.5 MiB of scratch
    _, _, (qw, sc, zr) = _inputs(8, n, k, group, 3)
    big = torch.zeros(m, k, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    st = wq.lib.wq_msd_gemm_noalloc(
        ctypes.c_void_p(big.data_ptr()), m, n, k, 2, group, ctypes.c_void_p(qw.data_ptr()),
        ctypes.c_void_p(sc.data_ptr()), ctypes.c_void_p(zr.data_ptr()),
        ctypes.c_void_p(y.data_ptr()), None)
    assert st == wq.WQ_ERR_UNSUPPORTED
