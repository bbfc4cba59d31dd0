"""GPU parity: quantize/pack, unpack and standalone dequantization are
bit-exact with the oracle (integer, byte and bf16/fp16 bit patterns)."""

import numpy as np
import pytest
import torch

from oracle import formats, numerics
from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    import bit_weight_quantized_weights_b200 as pkg
    return pkg.binding


def _gold_w():
    """Hand-built INT4 groups planted into a seeded matrix (exact-value, tie and
    degenerate groups) plus the seeded normal values."""
    import json
    import os
    from bit_weight_quantized_weights_b200 import workloads
    g = json.load(open(os.path.join(helpers.__file__.rsplit("/", 1)[0], "golden",
                                    "int4_groups.json")))
    w = workloads.weights(37, 512, seed=3).numpy()
    planted = np.array([x for grp in g["groups"] for x in grp["w"]], np.float32)
    w[5, :planted.size] = planted          # groups of 8 inside a 64-group: tests G=8 below
    w[6, :] = 0.0                          # all-zero row -> degenerate groups
    w[7, 64:128] = 1e-9                    # vanishing group (fp16 scale underflows)
    return w


@pytest.mark.parametrize("group", [8, 64, 128, 512])
def test_int4_quantize_pack_bit_exact(wq, group):
    w = _gold_w()
    q, s, z = formats.int4_quantize(w, group)
    qw_ref = formats.int4_pack(q)
    qw, sc, zr = wq.wq_quantize_pack(wq.WQ_FMT_INT4_ASYM, torch.from_numpy(w).cuda(), group)
    torch.cuda.synchronize()
    assert np.array_equal(qw.cpu().numpy().view(np.uint32), qw_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), s.view(np.uint16))
    assert np.array_equal(zr.cpu().numpy().view(np.uint16), z.view(np.uint16))
    codes = wq.wq_unpack(wq.WQ_FMT_INT4_ASYM, qw, w.shape[0], w.shape[1])
    assert np.array_equal(codes.cpu().numpy().reshape(q.shape), q)


def test_nf4_quantize_pack_bit_exact(wq):
    from bit_weight_quantized_weights_b200 import workloads
    w = workloads.weights(64, 1024, seed=4).numpy()
    w[3, :64] = 0.0                                   # zero block
    cb = formats.nf4_codebook()
    # exact ties: midpoints representable in fp32, in a block whose absmax is 1
    w[4, :64] = 0.0
    w[4, 0] = 1.0
    for i in range(15):
        mid = (np.float64(cb[i]) + np.float64(cb[i + 1])) / 2
        if np.float64(np.float32(mid)) == mid:
            w[4, 1 + i] = np.float32(mid)
    codes, absmax = formats.nf4_quantize(w)
    packed = formats.nf4_pack(codes)
    qw, am, _ = wq.wq_quantize_pack(wq.WQ_FMT_NF4, torch.from_numpy(w).cuda(), 64)
    torch.cuda.synchronize()
    assert np.array_equal(qw.cpu().numpy(), packed)
    assert np.array_equal(am.cpu().numpy().view(np.uint32), absmax.view(np.uint32))
    un = wq.wq_unpack(wq.WQ_FMT_NF4, qw, 64, 1024)
    assert np.array_equal(un.cpu().numpy(), codes)


@pytest.mark.parametrize("n,k", [(28672, 8192)])
def test_int4_and_nf4_pack_full_size_sampled_rows(wq, n, k):
    """Full-size pack on the GPU; sampled rows re-quantized by the oracle."""
    from bit_weight_quantized_weights_b200 import workloads
    w = workloads.flat_weights(n, k, seed=0)
    wd = w.cuda()
    rows = np.random.default_rng(0).choice(n, 24, replace=False)
    rows.sort()
    qw, sc, zr = wq.wq_quantize_pack(wq.WQ_FMT_INT4_ASYM, wd, 128)
    cw, am, _ = wq.wq_quantize_pack(wq.WQ_FMT_NF4, wd, 64)
    torch.cuda.synchronize()
    wr = w.numpy()[rows]
    q, s, z = formats.int4_quantize(wr, 128)
    assert np.array_equal(qw[rows].cpu().numpy().view(np.uint32), formats.int4_pack(q))
    assert np.array_equal(sc[rows].cpu().numpy().view(np.uint16), s.view(np.uint16))
    codes, absmax = formats.nf4_quantize(wr)
    cw2 = cw.view(n, k // 2)[rows].cpu().numpy().reshape(-1)
    am2 = am.view(n, k // 64)[rows].cpu().numpy().reshape(-1)
    assert np.array_equal(cw2, formats.nf4_pack(codes))
    assert np.array_equal(am2.view(np.uint32), absmax.view(np.uint32))


def _nf4_case(numel, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 16, size=numel, dtype=np.uint8)
    absmax = (np.abs(rng.standard_normal(numel // 64)) * 0.05).astype(np.float32)
    absmax[::97] = 0.0
    return codes, absmax


@pytest.mark.parametrize("numel", [64, 64 * 7, 64 * 1000 + 64 * 3])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_nf4_dequant_bit_exact_small(wq, numel, dtype):
    codes, absmax = _nf4_case(numel, numel)
    out = wq.wq_nf4_dequant(torch.from_numpy(formats.nf4_pack(codes)).cuda(),
                            torch.from_numpy(absmax).cuda(), numel, out_dtype=dtype)
    torch.cuda.synchronize()
    if dtype == torch.bfloat16:
        ref = numerics.bf16_bits(formats.nf4_dequant_fp32(codes, absmax))
        got = out.cpu().view(torch.int16).numpy().view(np.uint16)
    else:
        ref = formats.nf4_dequant_fp32(codes, absmax).astype(np.float16).view(np.uint16)
        got = out.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("n,k", [(28672, 8192), (8192, 8192), (5120, 25600)])
def test_nf4_dequant_full_size_every_element(wq, n, k):
    """The bench's workload and launch: every output element compared."""
    from bit_weight_quantized_weights_b200 import workloads
    numel = n * k
    g = workloads.generator(1)
    codes = torch.randint(0, 16, (numel,), generator=g, dtype=torch.uint8).numpy()
    absmax = (torch.rand(numel // 64, generator=g) * 0.08).numpy().astype(np.float32)
    out = wq.wq_nf4_dequant(torch.from_numpy(formats.nf4_pack(codes)).cuda(),
                            torch.from_numpy(absmax).cuda(), numel)
    torch.cuda.synchronize()
    got = out.cpu().view(torch.int16).numpy().view(np.uint16)
    ref = numerics.bf16_bits(formats.nf4_dequant_fp32(codes, absmax))
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("n,k,group", [(37, 512, 8), (64, 1024, 64), (300, 4096, 128),
                                       (14336, 4096, 128)])
def test_int4_dequant_bit_exact(wq, n, k, group):
    q, s, z, qweight = helpers.int4_packed(n, k, group, seed=5)
    qw, sc, zr = helpers.to_dev_int4(s, z, qweight)
    out = wq.wq_int4_dequant(qw, sc, zr, n, k, group)
    torch.cuda.synchronize()
    got = out.cpu().view(torch.int16).numpy().view(np.uint16)
    ref = numerics.bf16_bits(formats.int4_dequant_exact(q, s, z, group))
    assert np.array_equal(got, ref)
