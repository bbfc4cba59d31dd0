"""The C-ABI library loads, exports every declared symbol, and validates its
arguments on the host (CPU only: no call here reaches a kernel launch)."""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def wq():
    from bit_weight_quantized_weights_b200 import build_lib
    build_lib.build()
    from bit_weight_quantized_weights_b200 import binding
    return binding


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "wq.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(wq_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    syms = _declared_symbols()
    for name in ["wq_quantize_pack", "wq_nf4_dequant", "wq_w4a16_gemv", "wq_w4a16_gemm",
                 "wq_msd_gemm", "wq_msd_decompose", "wq_workspace_bytes"]:
        assert name in syms


def test_library_exports_every_declared_symbol(wq):
    lib = ctypes.CDLL(wq.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name
    assert sorted(wq.EXPORTED) == _declared_symbols()


def test_status_strings(wq):
    for s in range(7):
        assert wq.status_string(s) and wq.status_string(s) != "unknown status"
    assert wq.status_string(99) == "unknown status"
    assert "sm_100a" in wq.version()


def test_codebook_matches_oracle_bit_exact(wq):
    """The library computes the codebook on its own (bisection + Newton on
    erfc); it must equal the oracle's SciPy construction bit for bit."""
    from oracle import formats
    cb = np.array(wq.wq_nf4_codebook(), dtype=np.float32)
    assert np.array_equal(cb.view(np.uint32), formats.nf4_codebook().view(np.uint32))


def test_packed_sizes(wq):
    assert wq.wq_packed_sizes(wq.WQ_FMT_INT4_ASYM, 1024, 1024, 64) == (512 * 1024, 1024 * 16 * 2,
                                                                        1024 * 16 * 2)
    q, s, z = wq.wq_packed_sizes(wq.WQ_FMT_NF4, 28672, 8192, 64)
    assert q == 28672 * 8192 // 2 and s == 28672 * 8192 // 64 * 4 and z == 0
    with pytest.raises(wq.WqError):
        wq.wq_packed_sizes(wq.WQ_FMT_INT4_ASYM, 16, 100, 64)   # K % G
    with pytest.raises(wq.WqError):
        wq.wq_packed_sizes(wq.WQ_FMT_NF4, 16, 128, 128)        # NF4 block must be 64


def test_workspace_sizes(wq):
    assert wq.wq_workspace_bytes(wq.WQ_OP_GEMV, 16, 4096, 4096, 128) == 0
    assert wq.wq_workspace_bytes(wq.WQ_OP_GEMM, 8192, 4096, 4096, 128) >= 8192 * 4096 * 2 + 8192 * 4
    assert wq.wq_workspace_bytes(wq.WQ_OP_GEMM, 0, 4096, 4096, 128) == 0
    ws = wq.wq_workspace_bytes(wq.WQ_OP_MSD_GEMM, 1024, 5120, 5120, 128, 2)
    assert ws >= 2 * 1024 * 5120 + 2 * 1024 * 4
    assert wq.wq_workspace_bytes(wq.WQ_OP_MSD_GEMM, 0, 5120, 5120, 128, 2) == 0


# Fake device addresses: validation must fail (or finish as a no-op) before
# anything dereferences them or launches.
A16 = 0x10000
MIS = 0x10001


def _gemv(wq, m, n, k, fmt=0, group=128, x=A16, q=A16, s=A16, z=A16, y=A16):
    return wq.lib.wq_w4a16_gemv(x, m, n, k, fmt, group, q, s, z, y, None, 0, None)


def test_gemv_validation(wq):
    assert _gemv(wq, 17, 4096, 4096) == wq.WQ_ERR_UNSUPPORTED        # decode only
    assert _gemv(wq, 1, 4096, 4000) == wq.WQ_ERR_INVALID_ARG          # K % G
    assert _gemv(wq, 1, 4096, 4096, group=96) == wq.WQ_ERR_INVALID_ARG  # K % G (4096 % 96)
    assert _gemv(wq, 1, 4096, 4096, group=32) == wq.WQ_ERR_UNSUPPORTED  # G % 64
    assert _gemv(wq, 1, 4096, 4096, x=0) == wq.WQ_ERR_INVALID_ARG
    assert _gemv(wq, 1, 4096, 4096, y=MIS) == wq.WQ_ERR_ALIGNMENT
    assert _gemv(wq, 1, 4100, 4096) == wq.WQ_ERR_UNSUPPORTED          # N % 16
    assert _gemv(wq, 1, 4096, 4096, fmt=1, group=64) == wq.WQ_ERR_INVALID_ARG  # NF4 w/ zeros
    assert _gemv(wq, 1, 4096, 4096, fmt=7) == wq.WQ_ERR_INVALID_ARG
    assert _gemv(wq, -1, 4096, 4096) == wq.WQ_ERR_INVALID_ARG
    assert _gemv(wq, 0, 4096, 4096) == wq.WQ_OK                      # empty: no-op
    assert _gemv(wq, 4, 0, 4096) == wq.WQ_OK


def test_residual_correction_validation(wq):
    L = wq.lib
    # wq_residual(fmt, W, N, K, group, qweight, scales, zeros, residual_t, stream)
    assert L.wq_residual(0, A16, 64, 100, 64, A16, A16, A16, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_residual(1, A16, 64, 128, 64, A16, A16, A16, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_residual(0, A16, 64, 128, 64, A16, A16, None, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_residual(0, MIS, 64, 128, 64, A16, A16, A16, A16, None) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_residual(0, A16, 0, 128, 64, A16, A16, A16, A16, None) == wq.WQ_OK
    assert L.wq_residual(0, A16, 60, 128, 64, A16, A16, A16, A16, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_residual(0, A16, 64, 96, 32, A16, A16, A16, A16, None) == wq.WQ_ERR_UNSUPPORTED
    # wq_select_salient(x, M, K, k, idx, stream)
    assert L.wq_select_salient(A16, 1, 4096, 4097, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_select_salient(A16, 0, 4096, 8, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_select_salient(A16, 1, 4096, -1, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_select_salient(A16, 1, 4096, 0, A16, None) == wq.WQ_OK
    assert L.wq_select_salient(A16, 1, 4096, 8, MIS, None) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_select_salient(A16, 1, 65552, 8, A16, None) == wq.WQ_ERR_UNSUPPORTED
    # wq_w4a16_gemv_corrected(x, M, N, K, fmt, G, q, s, z, residual_t, idx, k, y, stream)
    cg = L.wq_w4a16_gemv_corrected
    assert cg(A16, 1, 4096, 4096, 0, 128, A16, A16, A16, A16, A16, 4097, A16,
              None) == wq.WQ_ERR_INVALID_ARG
    assert cg(A16, 1, 4096, 4096, 0, 128, A16, A16, A16, None, A16, 8, A16,
              None) == wq.WQ_ERR_INVALID_ARG
    assert cg(A16, 1, 4096, 4096, 0, 128, A16, A16, A16, A16, MIS, 8, A16,
              None) == wq.WQ_ERR_ALIGNMENT
    assert cg(A16, 17, 4096, 4096, 0, 128, A16, A16, A16, A16, A16, 8, A16,
              None) == wq.WQ_ERR_UNSUPPORTED
    assert cg(A16, 0, 4096, 4096, 0, 128, A16, A16, A16, A16, A16, 8, A16, None) == wq.WQ_OK
    # wq_w4a16_gemv_salient(x, M, N, K, fmt, G, q, s, z, residual_t, k, idx, y, stream)
    sg = L.wq_w4a16_gemv_salient
    assert sg(A16, 1, 4096, 4096, 0, 128, A16, A16, A16, A16, 8, None, A16,
              None) == wq.WQ_ERR_INVALID_ARG                        # idx scratch needed
    assert sg(A16, 1, 4096, 4096, 0, 128, A16, A16, A16, A16, 8, MIS, A16,
              None) == wq.WQ_ERR_ALIGNMENT
    assert sg(A16, 1, 4096, 4096, 0, 128, A16, A16, A16, A16, 4097, A16, A16,
              None) == wq.WQ_ERR_INVALID_ARG
    assert sg(A16, 0, 4096, 4096, 0, 128, A16, A16, A16, A16, 8, A16, A16, None) == wq.WQ_OK


def test_gemm_and_msd_validation(wq):
    L = wq.lib
    assert L.wq_w4a16_gemm(A16, 512, 4096, 4096, 1, 64, A16, A16, None, A16, None, 0,
                           None) == wq.WQ_ERR_WORKSPACE                 # NF4 GEMM needs one
    assert L.wq_w4a16_gemm(A16, 512, 4096, 4096, 1, 128, A16, A16, None, A16, None, 0,
                           None) == wq.WQ_ERR_INVALID_ARG               # NF4 block is 64
    assert L.wq_w4a16_gemm(A16, 512, 4160, 4096, 0, 128, A16, A16, A16, A16, None, 0,
                           None) == wq.WQ_ERR_UNSUPPORTED               # N % 128
    assert L.wq_w4a16_gemm(A16, 512, 4096, 4096, 0, 128, A16, A16, A16, MIS, None, 0,
                           None) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_w4a16_gemm(A16, 0, 4096, 4096, 0, 128, A16, A16, A16, A16, None, 0,
                           None) == wq.WQ_OK
    assert L.wq_w4a16_gemm(A16, 512, 4096, 4096, 0, 128, A16, A16, A16, A16, None, 0,
                           None) == wq.WQ_ERR_WORKSPACE
    assert L.wq_w4a16_gemm(A16, 512, 4096, 4096, 0, 128, A16, A16, A16, A16, A16, 1024,
                           None) == wq.WQ_ERR_WORKSPACE
    assert L.wq_msd_gemm(A16, 16, 5120, 5120, 2, 128, A16, A16, A16, A16, None, 0,
                         None) == wq.WQ_ERR_WORKSPACE
    assert L.wq_msd_gemm(A16, 16, 5120, 5120, 4, 128, A16, A16, A16, A16, A16, 1 << 30,
                         None) == wq.WQ_ERR_INVALID_ARG                 # C in 1..3
    assert L.wq_msd_gemm(A16, 16, 5120, 5120, 2, 64, A16, A16, A16, A16, A16, 1 << 30,
                         None) == wq.WQ_ERR_UNSUPPORTED                 # G % 128
    assert L.wq_msd_decompose(A16, 4, 100, 2, A16, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_msd_decompose(A16, 0, 128, 2, A16, A16, None) == wq.WQ_OK


def test_noalloc_validates_like_msd_gemm(wq):
    """wq_msd_gemm_noalloc checks its arguments exactly as wq_msd_gemm does
    before it compares the problem's scratch with its fixed array, so an
    oversized problem with a bad argument reports the bad argument."""
    L = wq.lib
    big = (A16, 4096, 5120, 5120, 2, 128, A16, A16, A16, A16)      # ~40 MiB of scratch
    assert L.wq_msd_gemm_noalloc(*big, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_msd_gemm_noalloc(A16, 4096, 5120, 5000, 2, 125, A16, A16, A16, A16,
                                 None) == wq.WQ_ERR_INVALID_ARG       # group % 8
    assert L.wq_msd_gemm_noalloc(None, 4096, 5120, 5120, 2, 128, A16, A16, A16, A16,
                                 None) == wq.WQ_ERR_INVALID_ARG       # x NULL
    assert L.wq_msd_gemm_noalloc(A16, 4096, 5120, 5120, 2, 128, A16, A16, None, A16,
                                 None) == wq.WQ_ERR_INVALID_ARG       # zeros NULL
    assert L.wq_msd_gemm_noalloc(A16, 4096, 5120, 5120, 2, 128, A16, A16, A16, MIS,
                                 None) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_msd_gemm_noalloc(A16, 4096, 5120, 5120, 4, 128, A16, A16, A16, A16,
                                 None) == wq.WQ_ERR_INVALID_ARG       # C in 1..3
    assert L.wq_msd_gemm_noalloc(A16, 4096, 5120, 5120, 2, 64, A16, A16, A16, A16,
                                 None) == wq.WQ_ERR_UNSUPPORTED       # G % 128
    assert L.wq_msd_gemm_noalloc(A16, 0, 5120, 5120, 2, 128, A16, A16, A16, A16,
                                 None) == wq.WQ_OK                    # empty: no-op


def test_mx_validation(wq):
    L = wq.lib
    assert L.wq_mx_quantize(A16, 16, 100, A16, A16, None) == wq.WQ_ERR_INVALID_ARG   # K % 32
    assert L.wq_mx_quantize(MIS, 16, 128, A16, A16, None) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_mx_quantize(A16, 0, 128, A16, A16, None) == wq.WQ_OK
    assert L.wq_mx_decompose(A16, 4, 128, 3, A16, A16, None) == wq.WQ_ERR_INVALID_ARG  # passes
    assert L.wq_mx_decompose(A16, 4, 100, 2, A16, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_mx_decompose(A16, 0, 128, 2, A16, A16, None) == wq.WQ_OK
    # wq_mx_gemv(x, M, N, K, passes, codes, scales, y, ws, ws_bytes, stream)
    g = L.wq_mx_gemv
    assert g(A16, 17, 256, 512, 2, A16, A16, A16, A16, 1 << 20, None) == wq.WQ_ERR_UNSUPPORTED
    assert g(A16, 4, 256, 480, 2, A16, A16, A16, A16, 1 << 20, None) == wq.WQ_ERR_UNSUPPORTED
    assert g(A16, 4, 250, 512, 2, A16, A16, A16, A16, 1 << 20, None) == wq.WQ_ERR_UNSUPPORTED
    assert g(A16, 4, 256, 512, 0, A16, A16, A16, A16, 1 << 20, None) == wq.WQ_ERR_INVALID_ARG
    assert g(A16, 4, 256, 512, 2, A16, A16, A16, None, 0, None) == wq.WQ_ERR_WORKSPACE
    assert g(A16, 4, 256, 512, 2, A16, A16, MIS, A16, 1 << 20, None) == wq.WQ_ERR_ALIGNMENT
    assert g(A16, 0, 256, 512, 2, A16, A16, A16, None, 0, None) == wq.WQ_OK
    assert wq.wq_workspace_bytes(wq.WQ_OP_MX_GEMV, 16, 256, 512, 0, 2) == 2 * 16 * 512 + 2 * 16 * 16


def test_msd_nf4_validation(wq):
    g = wq.lib.wq_msd_gemm_nf4
    # (x, M, N, K, C, codes, absmax, y, ws, ws_bytes, stream)
    assert g(A16, 17, 256, 512, 2, A16, A16, A16, A16, 1 << 20, None) == wq.WQ_ERR_UNSUPPORTED
    assert g(A16, 4, 256, 640, 2, A16, A16, A16, A16, 1 << 20, None) == wq.WQ_ERR_UNSUPPORTED
    assert g(A16, 4, 250, 512, 2, A16, A16, A16, A16, 1 << 20, None) == wq.WQ_ERR_UNSUPPORTED
    assert g(A16, 4, 256, 512, 4, A16, A16, A16, A16, 1 << 20, None) == wq.WQ_ERR_INVALID_ARG
    assert g(A16, 4, 256, 512, 2, None, A16, A16, A16, 1 << 20, None) == wq.WQ_ERR_INVALID_ARG
    assert g(A16, 4, 256, 512, 2, A16, A16, A16, None, 0, None) == wq.WQ_ERR_WORKSPACE
    assert g(A16, 4, 256, 512, 2, A16, MIS, A16, A16, 1 << 20, None) == wq.WQ_ERR_ALIGNMENT
    assert g(A16, 0, 256, 512, 2, A16, A16, A16, None, 0, None) == wq.WQ_OK


def test_pack_and_dequant_validation(wq):
    L = wq.lib
    assert L.wq_quantize_pack(0, A16, 16, 100, 64, A16, A16, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_pack(1, A16, 16, 128, 64, A16, A16, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_pack(0, MIS, 16, 128, 64, A16, A16, A16, None) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_nf4_dequant(A16, A16, 100, 64, A16, 0, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_nf4_dequant(A16, A16, 128, 32, A16, 0, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_nf4_dequant(A16, A16, 128, 64, A16, 2, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_nf4_dequant(A16, A16, 0, 64, A16, 0, None) == wq.WQ_OK
    assert L.wq_int4_dequant(A16, A16, A16, 16, 128, 12, A16, 0, None) == wq.WQ_ERR_INVALID_ARG


def test_decode_attention_validation(wq):
    g = wq.lib.wq_msd_decode_attention
    ws = wq.lib.wq_msd_decode_attention_workspace
    # (q, B, Hq, Hkv, L, D, C, kq, ks, kz, vq, vs, vz, out, ws, ws_bytes, stream)
    def call(b=2, hq=16, hkv=4, length=300, d=128, c=2, ptr=A16, kq=A16, wsp=A16,
             ws_bytes=1 << 24):
        return g(ptr, b, hq, hkv, length, d, c, kq, A16, A16, A16, A16, A16, A16, wsp, ws_bytes,
                 None)
    assert call(hq=12, hkv=8) == wq.WQ_ERR_INVALID_ARG          # Hq % Hkv
    assert call(hq=48, hkv=16) == wq.WQ_ERR_UNSUPPORTED         # R = 3
    assert call(hq=64, hkv=4) == wq.WQ_ERR_UNSUPPORTED          # R = 16
    assert call(d=64) == wq.WQ_ERR_UNSUPPORTED
    assert call(d=100) == wq.WQ_ERR_INVALID_ARG
    assert call(c=3) == wq.WQ_ERR_UNSUPPORTED
    assert call(c=0) == wq.WQ_ERR_INVALID_ARG
    assert call(length=0) == wq.WQ_ERR_INVALID_ARG
    assert call(b=-1) == wq.WQ_ERR_INVALID_ARG
    assert call(b=70000) == wq.WQ_ERR_UNSUPPORTED
    assert call(kq=None) == wq.WQ_ERR_INVALID_ARG
    assert call(kq=MIS) == wq.WQ_ERR_ALIGNMENT
    assert call(wsp=None, ws_bytes=0) == wq.WQ_ERR_WORKSPACE
    assert call(b=0, ptr=None, kq=None, wsp=None, ws_bytes=0) == wq.WQ_OK
    size = ctypes.c_size_t(0)
    assert ws(2, 16, 4, 300, 128, 2, ctypes.byref(size)) == wq.WQ_OK
    # query digits (2 x 32 rows x 128 bytes), their scales (rounded up to 256
    # bytes), then 2 chunks x (128 + 2) floats per query head
    assert size.value == 2 * 32 * 128 + 256 + 32 * 2 * 130 * 4
    assert call(ws_bytes=size.value - 1) == wq.WQ_ERR_WORKSPACE
    assert ws(2, 16, 4, 300, 128, 3, ctypes.byref(size)) == wq.WQ_ERR_UNSUPPORTED
    assert ws(0, 16, 4, 300, 128, 2, ctypes.byref(size)) == wq.WQ_OK and size.value == 0


def test_attention_split_hook_validation(wq):
    assert wq.lib.wq_test_set_attention_split(-1) == wq.WQ_ERR_INVALID_ARG
    assert wq.lib.wq_test_set_attention_split(65) == wq.WQ_ERR_INVALID_ARG
    assert wq.lib.wq_test_set_attention_split(3) == wq.WQ_OK
    assert wq.lib.wq_test_set_attention_split(0) == wq.WQ_OK


def test_kv_block_values_validation(wq):
    g = wq.lib.wq_kv_block_values
    # (codes, rows, L, D, out, stream)
    assert g(A16, -1, 8, 128, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert g(A16, 4, 0, 128, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert g(A16, 4, 8, 100, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert g(None, 4, 8, 128, A16, None) == wq.WQ_ERR_INVALID_ARG
    assert g(A16, 4, 8, 128, MIS, None) == wq.WQ_ERR_ALIGNMENT
    assert g(None, 0, 8, 128, None, None) == wq.WQ_OK
