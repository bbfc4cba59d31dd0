"""4-bit weight formats: INT4 asymmetric per group, and NF4 (test infrastructure).

Sources
-------
* INT4 asymmetric, per-group scale and zero point: "MixPE: Quantization and
  Hardware Co-design for Efficient LLM Inference", Abstract (the scale and the
  zero point are shared by every weight of one quantization group). The range
  convention (the group range always includes 0) is the one of the GPTQ paper,
  which the "Multi-Scale Dequant" and "Fast NF4 Dequantization Kernels" pages
  cite by title only.
* NF4: "Fast NF4 Dequantization Kernels for Large Language Model Inference",
  Abstract (4-bit NormalFloat codes, a 4x memory reduction against 16-bit, and a
  dequantization to 16-bit before the product). The codebook's construction is
  the one of QLoRA, which "DecDEC: A Systems Approach to Advancing Low-Bit LLM
  Quantization" cites by title; the pages print no codebook values.

Layouts (the library's canonical packed layouts)
------------------------------------------------
* INT4: ``qweight[n, k // 8]`` uint32, the code of column k in bits
  ``4*(k % 8) .. 4*(k % 8) + 3`` (low nibble first). ``scales[n, g]`` and
  ``zeros[n, g]`` are fp16, row-major, g = k // G.
* NF4: elements flattened row-major; byte j holds element 2j in its HIGH nibble
  and element 2j+1 in its low nibble. ``absmax[b]`` (fp32) scales the 64
  consecutive elements of block b.

Readings where the pages are silent (all fixed here and in the CUDA library):
* all divisions are IEEE binary32 divisions, all roundings to integers are
  round-half-to-even, the fp16 scale is binary32 rounded to binary16 (ties even);
* an INT4 group whose fp16 scale would be 0 (an all-zero group, or a group of
  values below ~4.5e-7) is quantized as if its range were [-1, 1];
* an NF4 block whose absmax is 0 stores absmax 0 and the zero code 7;
* NF4 nearest-code ties go to the lower code index.
"""

import numpy as np
from scipy.stats import norm

from .numerics import bf16_round, fp16_round

NF4_BLOCK = 64


# --------------------------------------------------------------------------
# NF4 codebook
# --------------------------------------------------------------------------

def nf4_offset():
    """Outermost quantile probability of the NF4 construction.

    It is the mean of 1 - 1/(2*15) and 1 - 1/(2*16): the midpoints of the last
    bins of a 15-way and a 16-way equal-probability split of (0, 1).
    """
    return 0.5 * ((1.0 - 1.0 / (2 * 15)) + (1.0 - 1.0 / (2 * 16)))


def nf4_codebook():
    """The 16 NF4 code values as float32, sorted ascending.

    Construction (QLoRA's 4-bit NormalFloat, asymmetric variant with an exact 0):
    eight positive values at the standard-normal quantiles of probabilities
    evenly spaced from the offset delta down towards 1/2 (8 of the 9 points of
    the even split of [1/2, delta], 1/2 itself excluded); seven negative values
    the same way with 8 points (7 kept), negated; one exact 0. All 16 are divided
    by the largest (the quantile at delta), so the table spans [-1, 1]. Computed
    in fp64, then rounded once to fp32.
    """
    d = nf4_offset()
    pos_p = np.linspace(d, 0.5, 9)[:-1]
    neg_p = np.linspace(d, 0.5, 8)[:-1]
    pos = norm.ppf(pos_p)
    neg = -norm.ppf(neg_p)
    vals = np.concatenate([neg, [0.0], pos])
    vals = vals / norm.ppf(d)
    vals = np.sort(vals)
    return vals.astype(np.float32)


# --------------------------------------------------------------------------
# INT4 asymmetric, group G along K
# --------------------------------------------------------------------------

def int4_quantize(w, group):
    """Quantize fp32 weights [N, K] to INT4 codes with per-group scale and zero.

    Per row n and group g (columns g*G .. g*G+G-1):
      lo = min(min(w), 0), hi = max(max(w), 0)            (fp32)
      s  = fp16( fp32(hi - lo) / 15 )                    (fp32 sub, fp32 div)
      if s == 0:  lo, hi = -1, 1 and s is recomputed
      z  = clamp(rint(fp32(-lo / s)), 0, 15)              (stored as fp16)
      q  = clamp(rint(fp32(w / s)) + z, 0, 15)
    Returns (q uint8 [N, K], scales float16 [N, K/G], zeros float16 [N, K/G]).
    """
    w = np.ascontiguousarray(w, dtype=np.float32)
    n_rows, k = w.shape
    assert k % group == 0
    ng = k // group
    wg = w.reshape(n_rows, ng, group)
    f0 = np.float32(0)
    lo = np.minimum(wg.min(axis=2), f0)
    hi = np.maximum(wg.max(axis=2), f0)
    fifteen = np.float32(15)
    s = fp16_round(np.float32(hi - lo) / fifteen)
    degenerate = s == 0
    if degenerate.any():
        lo = np.where(degenerate, np.float32(-1), lo).astype(np.float32)
        hi = np.where(degenerate, np.float32(1), hi).astype(np.float32)
        s = fp16_round(np.float32(hi - lo) / fifteen)
    # the zero point is an integer code: stored as +0.0 .. 15.0 (never -0.0)
    z = np.clip(np.rint((-lo) / s), 0, 15).astype(np.int32).astype(np.float32)
    q = np.rint(wg / s[:, :, None]) + z[:, :, None]
    q = np.clip(q, 0, 15).astype(np.uint8).reshape(n_rows, k)
    return q, s.astype(np.float16), z.astype(np.float16)


def int4_pack(q):
    """Pack INT4 codes [N, K] (K % 8 == 0) into uint32 [N, K/8], low nibble first."""
    q = np.asarray(q, dtype=np.uint32)
    n_rows, k = q.shape
    assert k % 8 == 0
    q8 = q.reshape(n_rows, k // 8, 8)
    out = np.zeros((n_rows, k // 8), dtype=np.uint32)
    for i in range(8):
        out |= (q8[:, :, i] & 0xF) << np.uint32(4 * i)
    return out


def int4_unpack(qweight, k):
    """Inverse of int4_pack: uint32 [N, K/8] -> uint8 codes [N, K]."""
    qw = np.asarray(qweight, dtype=np.uint32)
    n_rows = qw.shape[0]
    out = np.empty((n_rows, k // 8, 8), dtype=np.uint8)
    for i in range(8):
        out[:, :, i] = (qw >> np.uint32(4 * i)) & 0xF
    return out.reshape(n_rows, k)


def int4_dequant_exact(q, scales, zeros, group):
    """Exact dequantized weights (q - z) * s as float32 [N, K].

    (q - z) is an integer of at most 4 bits and magnitude and s an fp16 value
    (11 significant bits), so the product is exact in fp32.
    """
    q = np.asarray(q, dtype=np.float32)
    n_rows, k = q.shape
    s = np.repeat(np.asarray(scales, dtype=np.float32), group, axis=1)
    z = np.repeat(np.asarray(zeros, dtype=np.float32), group, axis=1)
    return ((q - z) * s).astype(np.float32)


def int4_dequant_bf16(q, scales, zeros, group):
    """Dequantized INT4 weights rounded once to bf16 (ties even), as float32."""
    return bf16_round(int4_dequant_exact(q, scales, zeros, group))


# --------------------------------------------------------------------------
# NF4, block of 64 consecutive elements
# --------------------------------------------------------------------------

def nf4_quantize(w, codebook=None, block=NF4_BLOCK, chunk=1 << 20):
    """Quantize fp32 weights (any shape, flattened row-major) to NF4.

    Per block of 64: absmax = max|w| (fp32); u = fp32(w / absmax); the code is
    the index of the codebook value nearest to u (exact real distance; ties to
    the lower index). An all-zero block stores absmax 0 and code 7 (the exact 0).
    Returns (codes uint8 [numel], absmax float32 [numel / 64]).
    """
    cb = nf4_codebook() if codebook is None else np.asarray(codebook, np.float32)
    flat = np.ascontiguousarray(w, dtype=np.float32).reshape(-1)
    assert flat.size % block == 0
    blocks = flat.reshape(-1, block)
    absmax = np.abs(blocks).max(axis=1).astype(np.float32)
    codes = np.empty(flat.size, dtype=np.uint8)
    cb64 = cb.astype(np.float64)
    rows_per_chunk = max(1, chunk // block)
    for b0 in range(0, blocks.shape[0], rows_per_chunk):
        bl = blocks[b0:b0 + rows_per_chunk]
        am = absmax[b0:b0 + rows_per_chunk]
        safe = np.where(am == 0, np.float32(1), am)
        u = (bl / safe[:, None]).astype(np.float32)
        # distances of two fp32 numbers of similar size are exact in fp64, and
        # only neighbouring codes compete for the minimum, so argmin over fp64
        # distances is the exact nearest code; argmin returns the first (lower)
        # index on ties.
        dist = np.abs(u.astype(np.float64)[:, :, None] - cb64[None, None, :])
        c = np.argmin(dist, axis=2).astype(np.uint8)
        c[am == 0] = 7
        codes[b0 * block:(b0 + bl.shape[0]) * block] = c.reshape(-1)
    return codes, absmax


def nf4_pack(codes):
    """Two codes per byte: element 2j in the high nibble, 2j+1 in the low one."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    assert c.size % 2 == 0
    return ((c[0::2] << 4) | (c[1::2] & 0xF)).astype(np.uint8)


def nf4_unpack(packed):
    """Inverse of nf4_pack: bytes [numel/2] -> codes [numel]."""
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p >> 4
    out[1::2] = p & 0xF
    return out


def nf4_dequant_fp32(codes, absmax, codebook=None, block=NF4_BLOCK):
    """fp32(codebook[code] * absmax): one binary32 multiply (ties even)."""
    cb = nf4_codebook() if codebook is None else np.asarray(codebook, np.float32)
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    a = np.repeat(np.asarray(absmax, dtype=np.float32), block)
    return (cb[c] * a).astype(np.float32)


def nf4_dequant_bf16(codes, absmax, codebook=None, block=NF4_BLOCK):
    """NF4 dequantization to bf16: the fp32 product rounded to bf16 (ties even)."""
    return bf16_round(nf4_dequant_fp32(codes, absmax, codebook, block))


def nf4_dequant_fp16(codes, absmax, codebook=None, block=NF4_BLOCK):
    """NF4 dequantization to fp16: the fp32 product rounded to fp16 (ties even)."""
    return fp16_round(nf4_dequant_fp32(codes, absmax, codebook, block))


def nf4_dequant_exact(codes, absmax, codebook=None, block=NF4_BLOCK):
    """Exact codebook[code] * absmax in fp64 (a product of two fp32 values)."""
    cb = nf4_codebook() if codebook is None else np.asarray(codebook, np.float32)
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    a = np.repeat(np.asarray(absmax, dtype=np.float64), block)
    return cb[c].astype(np.float64) * a
