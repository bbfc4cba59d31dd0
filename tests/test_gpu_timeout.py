"""The bounded device waits of the tensor-core kernels expire cleanly.

The failure is made on purpose and without a device fault: through the
library's test hook (wq_test_set_wait) every wait is limited to 1 ms and the
kernel's loader withholds the first k-tile, so the waits on it run out. The
kernel must then record the wait site in the library's error word
(wq_device_error reports WQ_ERR_TIMEOUT), drain what it has in flight, free
its tensor memory and return, leaving the context usable: the next normal call
in the same process must match the oracle. Small grids of each kernel with
bounded waits: the single-CTA fused GEMM (INT4 and NF4), the CTA-pair fused
GEMM (per tile and persistent), and the MSD integer GEMM with and without its
cluster split of K.
"""

import pytest

from oracle import msd, products
from tests import helpers

pytestmark = pytest.mark.gpu

LIMIT_NS = 1_000_000  # 1 ms


@pytest.fixture(scope="module")
def wq():
    import bit_weight_quantized_weights_b200 as pkg
    return pkg.binding


def _x(m, k, seed, outliers=None):
    from bit_weight_quantized_weights_b200 import workloads
    return workloads.activations(m, k, gen=workloads.generator(seed + 5000), outliers=outliers)


def _gemm_int4(wq, m, n, k):
    q, s, z, qweight = helpers.int4_packed(n, k, 128, seed=m + 1)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = _x(m, k, m)
    ws = wq.gemm_workspace(m, n, k, 128)

    def run():
        return wq.wq_w4a16_gemm(x.cuda(), n, wq.WQ_FMT_INT4_ASYM, 128, qw, sc, zr, workspace=ws)

    return run, lambda: products.w4a16_int4(helpers.x_f32(x), q, s, z, 128)


def _gemm_nf4(wq, m, n, k):
    codes, absmax, packed = helpers.nf4_packed(n, k, seed=m + 2)
    cw, am = helpers.to_dev_nf4(absmax, packed)
    x = _x(m, k, m)
    ws = wq.gemm_workspace(m, n, k, 64)

    def run():
        return wq.wq_w4a16_gemm(x.cuda(), n, wq.WQ_FMT_NF4, 64, cw, am, None, workspace=ws)

    return run, lambda: products.w4a16_nf4(helpers.x_f32(x), codes, absmax, k)


def _msd(wq, m, n, k):
    q, s, z, qweight = helpers.int4_packed(n, k, 128, seed=m + 3)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    x = _x(m, k, m, outliers=(0.005, 50.0))

    def run():
        return wq.wq_msd_gemm(x.cuda(), n, 2, 128, qw, sc, zr)

    def ref():
        a, sa = msd.decompose(helpers.x_f32(x), 2)
        return msd.msd_product(a, sa, q, s, z, 128)

    return run, ref


# (name, builder, M, N, K, wait sites of that kernel)
CASES = [
    ("gemm_int4_single_cta", _gemm_int4, 128, 256, 1024, range(0x100, 0x500)),
    ("gemm_nf4_single_cta", _gemm_nf4, 128, 256, 1024, range(0x100, 0x500)),
    ("gemm_int4_cta_pairs", _gemm_int4, 256, 18944, 512, range(0x100, 0x500)),
    ("gemm_int4_persistent_pairs", _gemm_int4, 1024, 9472, 512, range(0x500, 0x600)),
    ("msd_one_rank", _msd, 128, 256, 512, range(0x1100, 0x1500)),
    ("msd_split_k", _msd, 128, 256, 2048, range(0x1100, 0x1500)),
]


@pytest.mark.parametrize("name,build,m,n,k,sites", CASES, ids=[c[0] for c in CASES])
def test_wait_expires_then_next_call_is_clean(wq, name, build, m, n, k, sites):
    run, ref = build(wq, m, n, k)
    st, _ = wq.wq_device_error(clear=True)
    assert st == wq.WQ_OK
    try:
        wq.wq_test_set_wait(LIMIT_NS, stall=1)
        run()
        st, detail = wq.wq_device_error(clear=True)
    finally:
        wq.wq_test_set_wait(0, 0)
    assert st == wq.WQ_ERR_TIMEOUT, name
    assert detail in sites, "%s: wait site 0x%x" % (name, detail)
    # the same call again, normal waits: the context is usable and the result
    # matches the oracle
    y = run()
    st, detail = wq.wq_device_error(clear=True)
    assert st == wq.WQ_OK, "%s: 0x%x" % (name, detail)
    y_ref = ref()
    helpers.check_product(y, y_ref, name + " after the timeout")
    helpers.check_within_bf16_rounding(y, y_ref, name + " after the timeout", slack=3e-3)


def test_test_hook_rejects_unknown_stall(wq):
    assert wq.lib.wq_test_set_wait(0, 2) == wq.WQ_ERR_INVALID_ARG
    assert wq.lib.wq_test_set_wait(0, 0) == wq.WQ_OK
