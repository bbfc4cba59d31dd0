"""Shared test helpers: oracle-side preparation of inputs and the tolerance checks.

Every expected value comes from ``oracle/`` on inputs from the seeded
generators in ``bit_weight_quantized_weights_b200.workloads``; nothing here
reads a CUDA result back into an oracle input.
"""

import functools

import numpy as np
import torch

from oracle import formats, numerics

# The product tolerance (relative Frobenius error, max-abs error per unit RMS).
REL_FRO_TOL = 5e-3
MAX_REL_TOL = 2e-2


def check_product(y_gpu, y_ref, what=""):
    """Product tolerance: relative Frobenius error <= 5e-3, and max-abs error
    per unit RMS <= 2e-2 for the error beyond the output's own bf16 rounding.

    y is bf16 by contract, and a bf16 value cannot sit closer to the exact
    result than half a bf16 ulp (2^-8 of |y| at worst); with outlier channels
    the largest outputs reach ~5.6 RMS, where that rounding alone is ~2.2e-2
    RMS. So the max-abs bound is applied to |y - y_ref| - ulp_bf16(y_ref)/2.
    Returns (rel_fro, raw max-abs/RMS)."""
    y = y_gpu.float().cpu().numpy() if isinstance(y_gpu, torch.Tensor) else np.asarray(y_gpu)
    rel, mx = numerics.compare(y, y_ref)
    r = np.asarray(y_ref, dtype=np.float64)
    rms = np.sqrt(np.mean(r * r))
    beyond = np.abs(y.astype(np.float64) - r) - 0.5 * numerics.bf16_ulp(r)
    mx_beyond = float(max(beyond.max(), 0.0) / rms) if rms > 0 else float(beyond.max())
    assert rel <= REL_FRO_TOL and mx_beyond <= MAX_REL_TOL, \
        "%s: rel_fro=%.3e max_rel=%.3e (beyond bf16 rounding %.3e)" % (what, rel, mx, mx_beyond)
    return rel, mx


def check_within_bf16_rounding(y_gpu, y_ref, what="", slack=1e-4):
    """Element-wise: |y - y_ref| <= one bf16 ulp of y_ref + slack * rms(y_ref).

    For kernels whose only rounding beyond fp32 accumulation is the final bf16
    store (exactly dequantized weights)."""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    r = np.asarray(y_ref, dtype=np.float64)
    rms = np.sqrt(np.mean(r * r))
    bound = numerics.bf16_ulp(r) + slack * rms
    bad = np.abs(y - r) > bound
    assert not bad.any(), "%s: %d elements beyond one bf16 ulp (worst %.3e)" % (
        what, int(bad.sum()), float(np.max(np.abs(y - r) - bound)))


# Unit roundoff of binary16 (half the spacing at 1): the largest relative
# error of one round-to-nearest to fp16 in its normal range.
FP16_U = 2.0 ** -11


def check_within_error_bound(y_gpu, y_ref, y_abs, eps, what=""):
    """Element-wise forward error bound of a dot product:
    |y - y_ref| <= one bf16 ulp of y_ref + eps * sum_k |x_k| |w_k|.

    y_abs is sum_k |x_k| |w_k| per output (the oracle's product of |x| and
    |W_hat|); eps is the kernel's relative error per term (its roundings of
    each weight or activation, plus fp32 accumulation), and the bf16 ulp
    covers the output's own rounding. Unlike a slack in units of the output's
    RMS, this bound holds for outputs that cancel inside rows whose terms are
    far larger than the typical output."""
    y = y_gpu.float().cpu().numpy().astype(np.float64) if isinstance(y_gpu, torch.Tensor) \
        else np.asarray(y_gpu, dtype=np.float64)
    r = np.asarray(y_ref, dtype=np.float64)
    bound = numerics.bf16_ulp(r) + eps * np.asarray(y_abs, dtype=np.float64)
    bad = np.abs(y - r) > bound
    assert not bad.any(), "%s: %d elements beyond the error bound (worst %.3e)" % (
        what, int(bad.sum()), float(np.max(np.abs(y - r) - bound)))


@functools.lru_cache(maxsize=16)
def int4_packed(n, k, group, seed=0):
    """Oracle-quantized INT4 weights of the seeded W [N, K]: (q, s, z, qweight)."""
    from bit_weight_quantized_weights_b200 import workloads
    w = workloads.weights(n, k, seed=seed).numpy()
    q, s, z = formats.int4_quantize(w, group)
    return q, s, z, formats.int4_pack(q)


@functools.lru_cache(maxsize=8)
def nf4_packed(n, k, seed=0):
    """Oracle-quantized NF4 weights of the seeded W [N, K]: (codes, absmax, packed)."""
    from bit_weight_quantized_weights_b200 import workloads
    w = workloads.weights(n, k, seed=seed).numpy()
    codes, absmax = formats.nf4_quantize(w)
    return codes, absmax, formats.nf4_pack(codes)


def to_dev_int4(s, z, qweight, device="cuda"):
    qw = torch.from_numpy(qweight.view(np.int32)).to(device)
    sc = torch.from_numpy(s).to(device)
    zr = torch.from_numpy(z).to(device)
    return qw, sc, zr


def to_dev_nf4(absmax, packed, device="cuda"):
    return torch.from_numpy(packed).to(device), torch.from_numpy(absmax).to(device)


def x_f32(x_bf16):
    """bf16 torch tensor -> float32 numpy (exact)."""
    return x_bf16.float().numpy()
