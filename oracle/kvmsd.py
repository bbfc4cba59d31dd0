"""Multi-Scale Dequant in decode attention over a quantized KV cache (test infrastructure).

Source: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
Activation Decomposition for Efficient LLM Inference", Abstract: MSD removes
the KV dequantization from the attention products (the quantized KV cache
multiplies low-precision components of the other operand directly) and so
reduces the KV cache's HBM traffic in attention; the page reports accuracy on
Flash Attention kernels.

The page gives no formulas; the reading (decode: one new query token per
sequence, the plainest setting where the KV cache is read in full):

* cache: K and V [B, Hkv, L, D] quantized per (sequence, head, token) row with
  the INT4 asymmetric group quantizer of the weights (oracle/formats.py) with
  group D (one fp16 scale and one zero per row), codes packed low nibble first;
* query heads: q [B, Hq, D] bf16, Hq = R * Hkv (grouped heads share a KV head);
* scores: each query row is decomposed into C int8 digit planes
  (oracle/msd.py decompose); s[l] = D^-1/2 sum_c sigma_c sk[l]
  (sum_d a_c[d] qk[l, d] - zk[l] sum_d a_c[d]), integer inner sums;
* softmax in chunks of T keys (flash decoding): per chunk j, m_j = max s,
  e[l] = exp(s[l] - m_j), E_j = sum e;
* values: per chunk, w[l] = e[l] sv[l] is decomposed into C int8 digit planes
  over the chunk's keys (the same decomposition, the chunk's keys as one row),
  O_j[d] = sum_c tau_c (sum_l b_c[l] qv[l, d] - sum_l b_c[l] zv[l]), integer
  inner sums;
* merge: with M = max_j m_j, out[d] = sum_j e^(m_j - M) O_j[d] /
  sum_j e^(m_j - M) E_j.

Everything here is fp64 except the decompositions, which follow
oracle/msd.py's fp32 steps (the kernel takes the same decisions in fp32).
"""

import numpy as np

from . import formats, msd

CHUNK = 256


def quantize_cache(kv):
    """INT4 asymmetric, one group per row: kv fp32 [..., L, D] ->
    (codes uint8 [..., L, D], scales fp16 [..., L], zeros fp16 [..., L])."""
    shp = kv.shape
    d = shp[-1]
    q, s, z = formats.int4_quantize(np.asarray(kv, dtype=np.float32).reshape(-1, d), d)
    return q.reshape(shp), s.reshape(shp[:-1]), z.reshape(shp[:-1])


def dequant_cache(codes, scales, zeros):
    """Exact fp64 values (q - z) s of the cache."""
    return (np.asarray(codes, dtype=np.float64) - np.asarray(zeros, np.float64)[..., None]) * \
        np.asarray(scales, np.float64)[..., None]


def msd_decode_attention(q, k_cache, v_cache, n_components=2, chunk=CHUNK):
    """q bf16-valued fp32 [B, Hq, D]; k_cache / v_cache = (codes [B, Hkv, L, D],
    scales [B, Hkv, L], zeros [B, Hkv, L]). Returns out fp64 [B, Hq, D]."""
    qk, sk, zk = k_cache
    qv, sv, zv = v_cache
    b_, hq, d = q.shape
    hkv, length = qk.shape[1], qk.shape[2]
    r = hq // hkv
    out = np.zeros((b_, hq, d), dtype=np.float64)
    a, sig = msd.decompose(q.reshape(b_ * hq, d), n_components)    # [C, B*Hq, D], [C, B*Hq]
    for b in range(b_):
        for h in range(hq):
            kh = h // r
            row = b * hq + h
            qk_h = qk[b, kh].astype(np.float64)
            ad = a[:, row, :].astype(np.float64)                     # [C, D]
            p_int = ad @ qk_h.T                                       # [C, L] exact
            rsum = ad.sum(axis=1)                                     # [C]
            s = np.zeros(length)
            for c in range(n_components):
                s += float(sig[c, row]) * sk[b, kh].astype(np.float64) * \
                    (p_int[c] - zk[b, kh].astype(np.float64) * rsum[c])
            s /= np.sqrt(d)
            ms, es, os_ = [], [], []
            for j0 in range(0, length, chunk):
                sl = slice(j0, min(j0 + chunk, length))
                m_j = s[sl].max()
                e = np.exp(s[sl] - m_j)
                w = (e * sv[b, kh, sl].astype(np.float64)).astype(np.float32)
                bd, tau = msd.decompose(w[None, :], n_components)  # [C, 1, T], [C, 1]
                bd = bd[:, 0, :].astype(np.float64)
                qv_j = qv[b, kh, sl].astype(np.float64)              # [T, D]
                o = np.zeros(d)
                for c in range(n_components):
                    o += float(tau[c, 0]) * (bd[c] @ qv_j - bd[c] @ zv[b, kh, sl].astype(np.float64))
                ms.append(m_j)
                es.append(e.sum())
                os_.append(o)
            big = max(ms)
            wts = np.exp(np.array(ms) - big)
            out[b, h] = (wts[:, None] * np.array(os_)).sum(axis=0) / (wts * np.array(es)).sum()
    return out


def reference_attention(q, k, v):
    """Plain softmax attention in fp64: q [B, Hq, D], k / v [B, Hkv, L, D]."""
    b_, hq, d = q.shape
    r = hq // k.shape[1]
    out = np.zeros((b_, hq, d))
    for b in range(b_):
        for h in range(hq):
            s = k[b, h // r].astype(np.float64) @ q[b, h].astype(np.float64) / np.sqrt(d)
            p = np.exp(s - s.max())
            out[b, h] = (p / p.sum()) @ v[b, h // r].astype(np.float64)
    return out
