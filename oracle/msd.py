"""Multi-Scale Dequant (MSD): activation decomposition and the decomposed
integer product (test infrastructure).

Source: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
Activation Decomposition for Efficient LLM Inference", Abstract. Instead of
lifting the low-bit weights to bf16, the bf16 activations are split into
several low-precision components, each multiplied directly with the quantized
weights by an integer GEMM; two INT8 passes give close to 16 effective bits.
The per-group scale and zero are applied after each group's integer sum
("MixPE: Quantization and Hardware Co-design for Efficient LLM Inference",
Abstract).

The pages print no formulas. The reading used here (the plainest one that
yields "two passes of INT8, near 16 effective bits"):

* per activation row m, component 1 has the scale s_1 = fp32(amax / 127)
  (s_1 = 1 when the row is all zero) and digits
  a_1 = clamp(rint(fp32(x / s_1)), -127, 127);
* each further component c+1 works on the residual r_c = RN32(r_{c-1} - s_c a_c)
  (r_0 = x; one rounding, as a fused multiply-add gives) with the scale
  s_{c+1} = s_c / 256 and the digit d = rint(fp32(r_c / s_{c+1})), which lies
  in [-128, 128];
* a digit of +128 is written as -128 with a carry of +1 into the previous
  component's digit (s_c = 256 s_{c+1}, so the represented value is unchanged);
  the carry never pushes the first digit past 127, because a residual that large
  needs x / s_1 more than 127 - 1/2 away from the first digit;
* x_hat = sum_c s_c a_c. With C = 2 this is a 16-bit fixed-point value made of
  two signed 8-bit digits, and |x - x_hat| <= s_C / 2 up to the binary32
  rounding of the last quotient: log2(127 * 256 * 2), about 16 effective bits.

Weights are the INT4 asymmetric codes q in [0, 15] (per group G along K, G a
divisor of K; G = K is per-channel). With integer
P_c[m, n, g] = sum_{k in g} a_c[m, k] q[n, k] and R_c[m, g] = sum_{k in g} a_c[m, k]:

    y[m, n] = sum_c s_c[m] sum_g s[n, g] (P_c[m, n, g] - z[n, g] R_c[m, g])

which equals x_hat . ((q - z) s)^T exactly.
"""

import numpy as np

RATIO = 256.0  # s_{c+1} = s_c / RATIO, a power of two


def decompose(x, n_components=2):
    """Split activations [M, K] (bf16 values as float32) into digit planes.

    Returns (a int8 [C, M, K], s float32 [C, M]).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    m, k = x.shape
    c_total = int(n_components)
    d = np.zeros((c_total, m, k), dtype=np.int64)
    s = np.zeros((c_total, m), dtype=np.float32)
    amax = np.abs(x).max(axis=1) if k > 0 else np.zeros(m, np.float32)
    s1 = (amax / np.float32(127)).astype(np.float32)
    s1 = np.where(amax == 0, np.float32(1), s1).astype(np.float32)
    r = x
    sc = s1
    for c in range(c_total):
        digit = np.rint((r / sc[:, None]).astype(np.float32))
        if c == 0:
            digit = np.clip(digit, -127, 127)
        d[c] = digit.astype(np.int64)
        s[c] = sc
        # residual with one rounding: the exact r - s*d fits fp64, then RN32
        r = (r.astype(np.float64) - sc.astype(np.float64)[:, None] * digit.astype(np.float64)
             ).astype(np.float32)
        sc = (sc / np.float32(RATIO)).astype(np.float32)
    # digits of +128 become -128 with a carry into the previous component
    for c in range(c_total - 1, 0, -1):
        hit = d[c] == 128
        d[c][hit] = -128
        d[c - 1][hit] += 1
    assert d.min(initial=0) >= -128 and d.max(initial=0) <= 127
    return d.astype(np.int8), s


def reconstruct(a, s):
    """x_hat = sum_c s_c a_c in fp64."""
    a64 = np.asarray(a, dtype=np.float64)
    s64 = np.asarray(s, dtype=np.float64)
    return np.einsum("cm,cmk->mk", s64, a64)


def group_sums(a, group):
    """R_c[m, g] = sum_{k in g} a_c[m, k] (exact integers)."""
    c, m, k = a.shape
    return a.astype(np.int64).reshape(c, m, k // group, group).sum(axis=3)


def int_partials(a, q, group):
    """P_c[m, n, g] = sum_{k in g} a_c[m, k] q[n, k] (exact integers).

    Computed with an fp64 matrix product: every product and partial sum is an
    integer below 2**53, so it is exact.
    """
    c, m, k = a.shape
    n = q.shape[0]
    ng = k // group
    out = np.empty((c, m, n, ng), dtype=np.int64)
    q64 = np.asarray(q, dtype=np.float64)
    for ci in range(c):
        a64 = a[ci].astype(np.float64)
        for g in range(ng):
            sl = slice(g * group, (g + 1) * group)
            out[ci, :, :, g] = np.rint(a64[:, sl] @ q64[:, sl].T).astype(np.int64)
    return out


def msd_product(a, s, q, scales, zeros, group):
    """y[m, n] = sum_c s_c[m] sum_g s[n, g] (P_c - z[n, g] R_c[m, g]) in fp64."""
    p = int_partials(a, q, group)                  # [C, M, N, G]
    r = group_sums(a, group)                       # [C, M, G]
    sw = np.asarray(scales, dtype=np.float64)      # [N, G]
    zw = np.asarray(zeros, dtype=np.float64)       # [N, G]
    c_total, m = s.shape
    n = q.shape[0]
    y = np.zeros((m, n), dtype=np.float64)
    for ci in range(c_total):
        t = p[ci].astype(np.float64) - zw[None, :, :] * r[ci].astype(np.float64)[:, None, :]
        y += np.asarray(s[ci], dtype=np.float64)[:, None] * np.einsum("mng,ng->mn", t, sw)
    return y


def effective_bits(x, a, s):
    """log2(row amax / max reconstruction error), the worst row of x."""
    x64 = np.asarray(x, dtype=np.float64)
    err = np.abs(x64 - reconstruct(a, s)).max(axis=1)
    amax = np.abs(x64).max(axis=1)
    ok = amax > 0
    err = np.maximum(err[ok], np.finfo(np.float64).tiny)
    return float(np.min(np.log2(amax[ok] / err)))


# ---------------------------------------------------------------------------
# NF4 weights on the MSD path
# ---------------------------------------------------------------------------
# The pages give MSD for integer weights; NF4 codes index 16 real codebook
# values ("Fast NF4 Dequantization Kernels for Large Language Model
# Inference", Abstract), which no integer GEMM takes as they are. The reading
# used here keeps MSD's point (integer activation digits times integer
# weights, no weight converted to floating point): the codebook values become
# integers c_int = rint(c * 2^13) in [-8192, 8192] (within 2^-14 of c), split
# into two signed 8-bit digits c_int = 128 h + l with l in [-64, 63] and h in
# [-64, 64]; the block's absmax is applied after the block's integer sum:
#
#   y[m, n] = sum_c s_c[m] sum_blk absmax[n, blk] 2^-13
#             * sum_{k in blk} a_c[m, k] (128 h[q] + l[q])
#
# which equals x_hat . w_int^T exactly, with w_int = absmax * c_int * 2^-13
# (each weight within 2^-14 absmax of the NF4 value codebook[q] * absmax).

NF4_INT_SHIFT = 13


def nf4_int_codebook(codebook):
    """The 16 NF4 code values as integers rint(c * 2^13) (int64 [16])."""
    cb = np.asarray(codebook, dtype=np.float64)
    return np.rint(cb * 2.0 ** NF4_INT_SHIFT).astype(np.int64)


def nf4_int_digits(codebook):
    """(h, l) int64 [16]: c_int = 128 h + l with l in [-64, 63]."""
    ci = nf4_int_codebook(codebook)
    h = np.floor((ci + 64) / 128.0).astype(np.int64)
    return h, ci - 128 * h


def msd_nf4_product(a, s, codes, absmax, k, codebook):
    """y [M, N] in fp64: sum_c s_c sum_blk absmax 2^-13 sum a_c (128 h + l),
    integer inner sums exact. codes: NF4 codes of the row-major [N, K] weight
    (flattened), absmax fp32 [N * K / 64]."""
    h, l = nf4_int_digits(codebook)
    q = np.asarray(codes, dtype=np.int64).reshape(-1, k)
    n = q.shape[0]
    w_int = (128 * h[q] + l[q]).astype(np.float64)          # [N, K], exact integers
    am = np.asarray(absmax, dtype=np.float64).reshape(n, k // 64)
    c_total, m = s.shape
    y = np.zeros((m, n), dtype=np.float64)
    for ci in range(c_total):
        a64 = np.asarray(a[ci], dtype=np.float64)
        for b in range(k // 64):
            sl = slice(64 * b, 64 * (b + 1))
            p = a64[:, sl] @ w_int[:, sl].T                    # exact integers in fp64
            y += np.asarray(s[ci], dtype=np.float64)[:, None] * (am[None, :, b] * p)
    return y * 2.0 ** -NF4_INT_SHIFT
