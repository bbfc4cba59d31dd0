"""Salient-channel residual correction of a 4-bit product (test infrastructure).

Source: "DecDEC: A Systems Approach to Advancing Low-Bit LLM Quantization",
Abstract. The residual matrix is the difference between the full-precision
weights and the quantized ones. At every decoding step the salient input
channels, which the activation outliers mark, are found from that step's
activations, and the residuals of those channels alone are added back to
correct their quantization error.

The abstract gives no formulas; this module takes the plainest reading of
each step:

* Residual: ``R = fp16(W - W_hat)``, the subtraction done in fp32 on the fp32
  weight and the exactly dequantized weight (INT4: ``(q - z) * s``; NF4:
  ``codebook[q] * absmax`` rounded once to fp32), then rounded once to fp16.
  It is stored channel-major, ``R^T [K, N]``, so that one channel's residuals
  are contiguous.
* Salient channels: the ``k`` input channels with the largest magnitude over
  the step's tokens, ``max_m |x[m, c]|``. Magnitudes are ranked by their
  IEEE-754 bit pattern with the sign cleared, so NaN ranks above +inf; equal
  magnitudes go to the lower channel index. The set is returned in increasing
  channel order.
* Corrected product: ``y = x . W_hat^T + x[:, S] . R[:, S]^T``, every product
  and sum in fp64.
"""

import numpy as np

from . import formats, products


def residual_t(w, w_hat):
    """fp16(w - w_hat) with the subtraction in fp32, transposed to [K, N]."""
    w32 = np.asarray(w, dtype=np.float32)
    d = (w32 - np.asarray(w_hat, dtype=np.float32)).astype(np.float32)
    return np.ascontiguousarray(d.astype(np.float16).T)


def int4_residual_t(w, q, scales, zeros, group):
    """Residual of INT4 weights against their exact dequantization."""
    return residual_t(w, formats.int4_dequant_exact(q, scales, zeros, group))


def nf4_residual_t(w, codes, absmax, codebook=None):
    """Residual of NF4 weights (codes flattened row-major) against
    codebook[q] * absmax in fp32."""
    w32 = np.asarray(w, dtype=np.float32)
    w_hat = formats.nf4_dequant_fp32(codes, absmax, codebook).reshape(w32.shape)
    return residual_t(w32, w_hat)


def magnitude_keys(x):
    """max over tokens of |x[m, c]|, as the uint32 bit pattern of the
    magnitude (sign cleared): an order on magnitudes with NaN above +inf."""
    bits = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32)
    return (bits & np.uint32(0x7FFFFFFF)).max(axis=0)


def select_salient(x, k):
    """The k salient channels of activations x [M, K], in increasing order."""
    keys = magnitude_keys(x)
    kk = keys.shape[0]
    if k <= 0:
        return np.zeros(0, dtype=np.int32)
    # primary key: magnitude, descending; secondary: channel index, ascending
    order = np.lexsort((np.arange(kk), -keys.astype(np.int64)))
    return np.sort(order[:min(k, kk)]).astype(np.int32)


def correction(x, rt, idx):
    """x[:, S] . R[:, S]^T in fp64 (rt is R^T [K, N])."""
    x64 = np.asarray(x, dtype=np.float64)[:, idx]
    r64 = np.asarray(rt, dtype=np.float64)[idx, :]
    return x64 @ r64


def int4_corrected(x, q, scales, zeros, group, rt, idx):
    """INT4 product with the residuals of channels idx added back, in fp64."""
    return products.w4a16_int4(x, q, scales, zeros, group) + correction(x, rt, idx)


def nf4_corrected(x, codes, absmax, k_in, rt, idx, codebook=None):
    """NF4 product with the residuals of channels idx added back, in fp64."""
    return products.w4a16_nf4(x, codes, absmax, k_in, codebook) + correction(x, rt, idx)
