"""Plain CPU oracle for 4-bit weight-only quantized products (test infrastructure).

This package is the reference the CUDA library is checked against. It is test
infrastructure, not product code: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
or run it. It shares no code, table or constant generator with the CUDA path,
and imports nothing from the product package.

Everything is NumPy (and SciPy for the inverse normal CDF), written for
readability rather than speed:

* floating-point steps that the format defines in fp32 / fp16 / bf16 are done
  in exactly that precision (NumPy float32 / float16 arithmetic is IEEE
  round-to-nearest-even, and bf16 rounding is written out bit by bit);
* every product of activations with weights is accumulated in fp64.

Modules
-------
``numerics``   bf16 round-to-nearest-even and the comparison metrics.
``formats``    INT4 asymmetric group quantization and NF4 (codebook, quantize,
               pack, unpack, dequantize).
``products``   the W4A16 product y = x . dequant(W_q)^T in fp64.
``msd``        Multi-Scale Dequant activation decomposition and the
               decomposed integer product.
``decdec``     salient-channel residual correction: the residual matrix,
               the per-step channel selection and the corrected product.
``kvmsd``      decode attention over an INT4 KV cache with MSD on both
               products (query digits times K codes, softmax-weight digits
               times V codes), chunked softmax with the flash-decoding merge.
``mx``         MX block formats (MXFP4 E2M1, MXFP8 E4M3, power-of-two block
               scales), the two-pass MXFP4 activation decomposition, the
               single-pass MXFP8 comparator, and their product with MXFP4
               weights.

Parity pins: every function is pinned by ``tests/test_oracle_*.py`` against
facts that do not come from the oracle itself (hand-computed golden groups,
closed forms, exact rational brute force, library routines, and the
construction's own defining property). Claims that are *parity unpinned*: the
pages' statement that the decomposed product is no less accurate than the
dequantize-then-multiply baseline prints no numbers (it is measured and
reported, never asserted); and the two-pass MXFP4 figures (near 6.6 effective
bits, 1/64 per block), which the plainest MX readings do not reproduce (they
measure 6.15 bits, worst block amax/37, derived bound amax/12; the page's
single-pass MXFP8 figure, 5.24 bits, does reproduce and is pinned).
"""

from . import numerics, formats, products, msd, decdec, mx, kvmsd  # noqa: F401
