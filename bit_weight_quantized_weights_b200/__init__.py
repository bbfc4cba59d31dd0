"""4-bit weight-only quantized products for NVIDIA B200 (sm_100a).

y = x . dequant(W_q)^T for bf16 activations and INT4-asymmetric or NF4
weights: quantize/pack, standalone dequantization, a decode GEMV, a tcgen05
prefill GEMM with fused dequantization, and the Multi-Scale Dequant path
(int8 activation digit planes times integer weight codes). The kernels live in
libwq.so (C ABI: include/wq.h); ``binding`` is its thin ctypes layer.

Importing the package does not load the library (so ``build_lib`` can run
before it exists); the first use of ``binding`` or of any ``wq_*`` name loads
it and raises ImportError if libwq.so has not been built.
"""

import importlib


def __getattr__(name):
    if name == "binding" or name.startswith("wq_") or name.startswith("WQ_"):
        binding = importlib.import_module(".binding", __name__)
        if name == "binding":
            return binding
        return getattr(binding, name)
    raise AttributeError(name)
