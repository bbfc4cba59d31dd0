"""GPU parity of MSD decode attention over an INT4 KV cache.

The cache quantization is bit-exact with the oracle's (codes, scales, zeros).
The attention output is compared element by element with the oracle
(oracle/kvmsd.py) run on the oracle's own quantization of the same seeded
cache. The query digits are the same on both sides (the decomposition is
bit-exact); the scores are fp32 on the GPU and fp64 in the oracle, so the
softmax weights w = e * sv that the value-side decomposition digitizes differ
by a few fp32 ulps, and a digit may round the other way where w sits on a
rounding boundary. The bound written in the tests:

    |out - ref| <= ulp_bf16(ref) + eps * max_l |v_l|

ulp_bf16 covers the output's own bf16 rounding (half an ulp) and the fp32
merge; eps covers the fp32 scores (~2^-20 relative on e) and the rare digit
that rounds the other way: one last-digit step is tau_C = amax(w) / (127 *
256^(C-1)) on one key, divided by E = sum e >= 1, times |v_l|. With C = 2 that
is <= 2^-15 max|v| per flipped key; eps = 2^-12 allows several. With C = 1
(one int8 digit) a flip costs up to amax(w) / 127 / E: the test's softmax is
flat (E in the tens at least), eps = 2^-10.
"""

import numpy as np
import pytest
import torch

from oracle import kvmsd, numerics

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    import bit_weight_quantized_weights_b200 as pkg
    return pkg.binding


def _inputs(b, hq, hkv, length, seed):
    from bit_weight_quantized_weights_b200 import workloads
    return workloads.decode_attention(b, hq, hkv, length, seed=seed)


def _oracle_cache(t):
    return kvmsd.quantize_cache(t.numpy())


def _check(out_gpu, ref, v_deq, eps, what):
    y = out_gpu.float().cpu().numpy().astype(np.float64)
    vmax = np.abs(v_deq).max()
    bound = numerics.bf16_ulp(ref) + eps * vmax
    bad = np.abs(y - ref) > bound
    assert not bad.any(), "%s: %d of %d beyond the bound (worst excess %.3e, vmax %.3f)" % (
        what, int(bad.sum()), bad.size, float((np.abs(y - ref) - bound).max()), vmax)


def _run(wq, q, k, v, c):
    kc = wq.kv_quantize_keys(k.cuda())
    vc = wq.kv_quantize_values(v.cuda())
    out = wq.wq_msd_decode_attention(q.cuda(), kc, vc, n_components=c)
    torch.cuda.synchronize()
    return out, kc, vc


def _pack_rows(codes):
    """Oracle codes [..., L, D] -> uint32 words [..., L, D/8], element d in
    nibble d % 8 of word d / 8 (a plain rearrangement)."""
    c8 = codes.reshape(*codes.shape[:-1], -1, 8).astype(np.uint32)
    out = np.zeros(c8.shape[:-1], dtype=np.uint32)
    for i in range(8):
        out |= c8[..., i] << (4 * i)
    return out


def _pack_blocks(codes):
    """Oracle codes [B, H, L, D] -> uint32 words [B, H, ceil(L/8), D], token
    8 j + t in nibble t of word (j, d), tokens past L zero."""
    b, h, length, d = codes.shape
    nblk = (length + 7) // 8
    padded = np.zeros((b, h, nblk * 8, d), dtype=np.uint32)
    padded[:, :, :length] = codes
    blk = padded.reshape(b, h, nblk, 8, d)
    out = np.zeros((b, h, nblk, d), dtype=np.uint32)
    for t in range(8):
        out |= blk[:, :, :, t, :] << (4 * t)
    return out


@pytest.mark.parametrize("length", [300, 17, 1, 256])
def test_kv_quantize_bit_exact(wq, length):
    q, k, v = _inputs(2, 8, 2, length, seed=length)
    ck, sk, zk = _oracle_cache(k)
    cv, sv, zv = _oracle_cache(v)
    kq, ks, kz = wq.kv_quantize_keys(k.cuda())
    vq, vs, vz = wq.kv_quantize_values(v.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(kq.cpu().numpy().view(np.uint32), _pack_rows(ck))
    assert np.array_equal(vq.cpu().numpy().view(np.uint32), _pack_blocks(cv))
    for got, want in ((ks, sk), (kz, zk), (vs, sv), (vz, zv)):
        assert np.array_equal(got.cpu().numpy().view(np.uint16), want.view(np.uint16))


# (B, Hq, Hkv, L): several 256-key chunks with a ragged tail, a single partial
# chunk, one key, every supported group size R = Hq / Hkv
CASES = [
    (2, 4, 2, 300),     # R = 2, two chunks, tail 44
    (1, 8, 1, 513),     # R = 8, three chunks, tail 1
    (3, 2, 2, 17),      # R = 1, one partial chunk
    (1, 16, 4, 1024),   # R = 4, four full chunks
    (2, 64, 8, 700),    # Qwen3-32B heads
    (1, 8, 8, 1),       # one key: the output is that key's value
]


@pytest.mark.parametrize("b,hq,hkv,length", CASES)
@pytest.mark.parametrize("c", [2, 1])
def test_attention_every_element(wq, b, hq, hkv, length, c):
    q, k, v = _inputs(b, hq, hkv, length, seed=b * 1000 + length + c)
    out, _, _ = _run(wq, q, k, v, c)
    kc, vc = _oracle_cache(k), _oracle_cache(v)
    ref = kvmsd.msd_decode_attention(q.float().numpy(), kc, vc, n_components=c)
    v_deq = kvmsd.dequant_cache(*vc)
    _check(out, ref, v_deq, 2.0 ** -12 if c == 2 else 2.0 ** -10,
           "B=%d Hq=%d Hkv=%d L=%d C=%d" % (b, hq, hkv, length, c))
    st, detail = wq.wq_device_error()
    assert st == wq.WQ_OK, hex(detail)


@pytest.mark.parametrize("b,hq,hkv,length", [(2, 4, 2, 1100), (1, 64, 8, 700),
                                             (3, 8, 1, 2049)])
@pytest.mark.parametrize("ns", [2, 3, 8])
def test_attention_chunks_per_cta(wq, b, hq, hkv, length, ns):
    """Each CTA streaming ns chunks of 256 keys (merged in registers), with a
    ragged last CTA; the same bound against the oracle."""
    q, k, v = _inputs(b, hq, hkv, length, seed=b * 7 + length + ns)
    wq.wq_test_set_attention_split(ns)
    try:
        out, _, _ = _run(wq, q, k, v, 2)
    finally:
        wq.wq_test_set_attention_split(0)
    kc, vc = _oracle_cache(k), _oracle_cache(v)
    ref = kvmsd.msd_decode_attention(q.float().numpy(), kc, vc, n_components=2)
    _check(out, ref, kvmsd.dequant_cache(*vc), 2.0 ** -12,
           "ns=%d B=%d Hq=%d Hkv=%d L=%d" % (ns, b, hq, hkv, length))


def test_one_key_returns_its_value(wq):
    q, k, v = _inputs(2, 4, 2, 1, seed=5)
    out, _, _ = _run(wq, q, k, v, 2)
    vq, vs, vz = _oracle_cache(v)
    vd = kvmsd.dequant_cache(vq, vs, vz)[:, :, 0, :]          # [B, Hkv, D]
    want = np.repeat(vd, 2, axis=1)                            # query head h -> KV head h / 2
    y = out.float().cpu().numpy()
    assert np.all(np.abs(y - want) <= numerics.bf16_ulp(want) + 2.0 ** -12 * np.abs(vd).max())


def test_identical_keys_average_the_values(wq):
    """Every key equal: the softmax is uniform and the output is the mean of
    the dequantized values (within the value-side digits)."""
    q, k, v = _inputs(1, 8, 1, 600, seed=6)
    k[:] = k[:, :, :1, :]
    out, _, _ = _run(wq, q, k, v, 2)
    vd = kvmsd.dequant_cache(*_oracle_cache(v))                # [1, 1, L, D]
    want = np.repeat(vd.mean(axis=2), 8, axis=1)
    y = out.float().cpu().numpy()
    assert np.all(np.abs(y - want) <= numerics.bf16_ulp(want) + 2.0 ** -12 * np.abs(vd).max())


def test_close_to_exact_attention_over_the_dequantized_cache(wq):
    """The property that holds at any size: with C = 2 the result is exact
    softmax attention over the dequantized cache up to ~2^-15 relative and the
    output's bf16 rounding."""
    q, k, v = _inputs(2, 64, 8, 2000, seed=7)
    out, _, _ = _run(wq, q, k, v, 2)
    ref = kvmsd.reference_attention(q.float().numpy(), kvmsd.dequant_cache(*_oracle_cache(k)),
                                    kvmsd.dequant_cache(*_oracle_cache(v)))
    y = out.float().cpu().numpy()
    vmax = float(np.abs(kvmsd.dequant_cache(*_oracle_cache(v))).max())
    assert np.all(np.abs(y - ref) <= numerics.bf16_ulp(ref) + 2.0 ** -11 * vmax)


def test_bench_shape_sampled(wq):
    """The bench's decode-attention configuration (Qwen3-32B heads, B = 32
    sequences of 8192 cached tokens), checked against the oracle on sampled
    sequences (every head of each)."""
    b, hq, hkv, length = 32, 64, 8, 8192
    q, k, v = _inputs(b, hq, hkv, length, seed=11)
    out, _, _ = _run(wq, q, k, v, 2)
    y = out.float().cpu()
    for bi in (0, 17, 31):
        kc, vc = _oracle_cache(k[bi:bi + 1]), _oracle_cache(v[bi:bi + 1])
        ref = kvmsd.msd_decode_attention(q[bi:bi + 1].float().numpy(), kc, vc)
        _check(y[bi:bi + 1], ref, kvmsd.dequant_cache(*vc), 2.0 ** -12, "sequence %d" % bi)


def test_rejections(wq):
    dev = "cuda"
    q = torch.zeros(1, 8, 128, dtype=torch.bfloat16, device=dev)
    kc = wq.kv_quantize_keys(torch.zeros(1, 2, 4, 128, device=dev))
    vc = wq.kv_quantize_values(torch.zeros(1, 2, 4, 128, device=dev))
    with pytest.raises(wq.WqError) as e:      # R = 3
        wq.wq_msd_decode_attention(torch.zeros(1, 6, 128, dtype=torch.bfloat16, device=dev),
                                   kc, vc)
    assert e.value.status == wq.WQ_ERR_UNSUPPORTED
    with pytest.raises(wq.WqError) as e:      # three components
        wq.wq_msd_decode_attention(q, kc, vc, n_components=3)
    assert e.value.status == wq.WQ_ERR_UNSUPPORTED
    ws = torch.empty(16, dtype=torch.uint8, device=dev)
    with pytest.raises(wq.WqError) as e:
        wq.wq_msd_decode_attention(q, kc, vc, workspace=ws)
    assert e.value.status == wq.WQ_ERR_WORKSPACE
