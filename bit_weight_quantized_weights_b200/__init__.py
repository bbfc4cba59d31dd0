"""4-bit weight-only quantized products for NVIDIA B200 (sm_100a).

y = x . dequant(W_q)^T for bf16 activations and INT4-asymmetric or NF4
weights: quantize/pack, standalone dequantization, a decode GEMV, a tcgen05
prefill GEMM with fused dequantization, and the Multi-Scale Dequant path
(int8 activation digit planes times integer weight codes). The kernels live in
libwq.so (C ABI: include/wq.h); ``binding`` is its thin ctypes layer.
"""

from . import binding  # noqa: F401  (fails loudly if libwq.so is missing)
from .binding import (  # noqa: F401
    WQ_FMT_INT4_ASYM, WQ_FMT_NF4, wq_nf4_codebook, wq_packed_sizes, wq_quantize_pack, wq_unpack,
    wq_nf4_dequant, wq_int4_dequant, wq_w4a16_gemv, wq_w4a16_gemm, wq_msd_decompose, wq_msd_gemm,
    wq_workspace_bytes, wq_device_error,
)
