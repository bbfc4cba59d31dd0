"""Pins for the decode-attention MSD oracle (oracle/kvmsd.py).

The MSD attention differs from exact softmax attention over the dequantized
cache only by the two 16-bit digit decompositions (the query rows and, per
chunk, the softmax weights times the value scales), so against plain fp64
attention (a direct definition, no chunking, no digits) it must agree to about
2^-16 relative; a wrong scale, sign, zero term or merge weight is an O(1)
error. Special cases with a known answer: one key (the output is that key's
value), identical keys (the output is the mean of the values).
"""

import numpy as np
import torch

from oracle import kvmsd


def _case(b, hq, hkv, length, d=128, seed=0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(b, hq, d, generator=g).to(torch.bfloat16).float().numpy()
    k = (torch.randn(b, hkv, length, d, generator=g) * 0.5).numpy()
    v = torch.randn(b, hkv, length, d, generator=g).numpy()
    return q, kvmsd.quantize_cache(k), kvmsd.quantize_cache(v)


def _rel(a, b):
    return float(np.abs(a - b).max() / np.abs(b).max())


def test_msd_attention_matches_exact_attention_over_the_dequantized_cache():
    for (b, hq, hkv, length) in [(2, 4, 2, 600), (1, 8, 1, 256), (1, 2, 2, 1000)]:
        q, kc, vc = _case(b, hq, hkv, length, seed=length)
        out = kvmsd.msd_decode_attention(q, kc, vc)
        ref = kvmsd.reference_attention(q, kvmsd.dequant_cache(*kc), kvmsd.dequant_cache(*vc))
        assert _rel(out, ref) < 2e-4, (b, hq, hkv, length, _rel(out, ref))
        # one chunk covering every key gives the same result within the digits
        out1 = kvmsd.msd_decode_attention(q, kc, vc, chunk=length)
        assert _rel(out1, ref) < 2e-4


def test_one_key_returns_its_value():
    q, kc, vc = _case(1, 4, 1, 1, seed=3)
    out = kvmsd.msd_decode_attention(q, kc, vc)
    v = kvmsd.dequant_cache(*vc)[0, 0, 0]
    assert np.abs(out[0] - v[None, :]).max() <= 1e-4 * np.abs(v).max()


def test_identical_keys_average_the_values():
    q, kc, vc = _case(1, 2, 1, 300, seed=4)
    codes, s, z = kc
    codes[:] = codes[:, :, :1, :]
    s[:] = s[:, :, :1]
    z[:] = z[:, :, :1]
    out = kvmsd.msd_decode_attention(q, (codes, s, z), vc)
    mean = kvmsd.dequant_cache(*vc)[0, 0].mean(axis=0)
    assert np.abs(out[0] - mean[None, :]).max() <= 1e-4 * np.abs(mean).max()
