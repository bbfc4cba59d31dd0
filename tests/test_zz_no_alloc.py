"""The allocation-free Multi-Scale Dequant entry point (wq_msd_gemm_noalloc).

Some callers cannot give the library device memory at call time (a fixed
memory budget carved up at start-up, a plugin interface without a workspace
argument, a loop where allocation is forbidden). The no-allocation variant
keeps its scratch in a fixed device array inside the library. This test calls
it through the C ABI twice in a row, with different problem sizes so the
second call runs over the first call's leftovers, and checks each result
against wq_msd_gemm (which takes a caller workspace) within the tolerance
the other tests use. The file is named to run last.
"""

import ctypes

import numpy as np
import pytest
import torch

from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    import bit_weight_quantized_weights_b200 as pkg
    return pkg.binding


def _inputs(m, n, k, group, seed):
    from bit_weight_quantized_weights_b200 import workloads
    _, s, z, qweight = helpers.int4_packed(n, k, group, seed=seed)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = workloads.activations(m, k, gen=workloads.generator(seed + 4000),
                              outliers=(0.005, 50.0)).cuda()
    return x, qw, sc, zr


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


def test_noalloc_matches_workspace_entry_point_twice(wq):
    cases = [(128, 512, 5120, 128, 2, 1), (37, 384, 2560, 2560, 3, 2)]
    for m, n, k, group, c, seed in cases:
        x, qw, sc, zr = _inputs(m, n, k, group, seed)
        y_ref = wq.wq_msd_gemm(x, n, c, group, qw, sc, zr)
        y = _noalloc(wq, x, n, c, group, qw, sc, zr)
        torch.cuda.synchronize()
        st, detail = wq.wq_device_error()
        assert st == wq.WQ_OK, hex(detail)
        ref = y_ref.float().cpu().numpy().astype(np.float64)
        helpers.check_product(y, ref, "noalloc vs msd_gemm M=%d C=%d" % (m, c))
        helpers.check_within_bf16_rounding(y, ref, "noalloc vs msd_gemm", slack=1e-4)


def test_noalloc_rejects_problems_beyond_its_scratch(wq):
    m, n, k, group = 1024, 128, 5120, 128      # needs ~10.5 MiB of scratch
    x, qw, sc, zr = _inputs(8, n, k, group, 3)
    big = torch.zeros(m, k, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    st = wq.lib.wq_msd_gemm_noalloc(
        ctypes.c_void_p(big.data_ptr()), m, n, k, 2, group, ctypes.c_void_p(qw.data_ptr()),
        ctypes.c_void_p(sc.data_ptr()), ctypes.c_void_p(zr.data_ptr()),
        ctypes.c_void_p(y.data_ptr()), None)
    assert st == wq.WQ_ERR_UNSUPPORTED
