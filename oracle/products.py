"""The W4A16 product y = x . dequant(W_q)^T in fp64 (test infrastructure).

Sources: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
Activation Decomposition for Efficient LLM Inference", Abstract (the product of
high-precision activations with low-bit weights lifted back to high precision);
"MixPE: Quantization and Hardware Co-design for Efficient LLM Inference",
Abstract (mixed-precision GEMM: low-precision weights times higher-precision
activations; the group's scale and zero can be applied after the per-group sum).

x is [M, K] (bf16 values held as float32), the logical weight is [N, K] and
y is [M, N]. The reference product uses the EXACT dequantized weights (not
rounded to bf16) and accumulates in fp64.
"""

import numpy as np

from . import formats


def matmul_exact(x, w_hat):
    """y[m, n] = sum_k x[m, k] * w_hat[n, k], every product and sum in fp64."""
    x64 = np.asarray(x, dtype=np.float64)
    w64 = np.asarray(w_hat, dtype=np.float64)
    return x64 @ w64.T


def w4a16_int4(x, q, scales, zeros, group):
    """Reference INT4 product: x . ((q - z) * s)^T in fp64."""
    return matmul_exact(x, formats.int4_dequant_exact(q, scales, zeros, group))


def w4a16_int4_post_group(x, q, scales, zeros, group):
    """The same product with the group's scale and zero applied after the sum.

    y[m, n] = sum_g s[n, g] * (sum_{k in g} x[m, k] q[n, k]
                               - z[n, g] * sum_{k in g} x[m, k])
    This is the algebra the MixPE page uses; it must equal w4a16_int4.
    """
    x64 = np.asarray(x, dtype=np.float64)
    q64 = np.asarray(q, dtype=np.float64)
    m, k = x64.shape
    n = q64.shape[0]
    ng = k // group
    y = np.zeros((m, n), dtype=np.float64)
    s = np.asarray(scales, dtype=np.float64)
    z = np.asarray(zeros, dtype=np.float64)
    for g in range(ng):
        sl = slice(g * group, (g + 1) * group)
        p = x64[:, sl] @ q64[:, sl].T            # [M, N]
        sx = x64[:, sl].sum(axis=1)              # [M]
        y += s[None, :, g] * (p - z[None, :, g] * sx[:, None])
    return y


def w4a16_nf4(x, codes, absmax, k, codebook=None):
    """Reference NF4 product: x . (codebook[code] * absmax)^T in fp64.

    ``codes`` and ``absmax`` describe the row-major [N, K] weight flattened.
    """
    w_hat = formats.nf4_dequant_exact(codes, absmax, codebook).reshape(-1, k)
    return matmul_exact(x, w_hat)


def dequant_then_bf16_matmul_int4(x, q, scales, zeros, group):
    """The dequantize-then-multiply baseline's arithmetic: weights rounded to
    bf16 first, product in fp64 (isolates the weight-rounding error)."""
    return matmul_exact(x, formats.int4_dequant_bf16(q, scales, zeros, group))
