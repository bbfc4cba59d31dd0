"""ctypes binding of libwq.so: the C entry points under the same names.

Argument marshalling only: each function checks that tensors are CUDA,
contiguous and of the expected dtype, passes raw pointers and the current
torch CUDA stream, and raises on a non-OK status. Every step of the product
runs in the library's CUDA kernels; there is no CPU or library fallback, and
importing this module fails loudly when libwq.so is missing.
"""

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwq.so")

WQ_OK = 0
WQ_ERR_INVALID_ARG = 1
WQ_ERR_UNSUPPORTED = 2
WQ_ERR_ALIGNMENT = 3
WQ_ERR_CUDA = 4
WQ_ERR_TIMEOUT = 5
WQ_ERR_WORKSPACE = 6

WQ_FMT_INT4_ASYM = 0
WQ_FMT_NF4 = 1
WQ_BF16 = 0
WQ_FP16 = 1
WQ_FP32 = 2
WQ_OP_GEMV = 0
WQ_OP_GEMM = 1
WQ_OP_MSD_GEMM = 2
WQ_OP_MX_GEMV = 3

# every symbol include/wq.h declares
EXPORTED = [
    "wq_status_string", "wq_version", "wq_nf4_codebook", "wq_packed_sizes",
    "wq_quantize_pack", "wq_unpack", "wq_nf4_dequant", "wq_int4_dequant",
    "wq_w4a16_gemv", "wq_w4a16_gemm", "wq_msd_decompose", "wq_msd_gemm",
    "wq_workspace_bytes", "wq_device_error", "wq_msd_gemm_noalloc",
    "wq_residual", "wq_select_salient", "wq_w4a16_gemv_corrected", "wq_w4a16_gemv_salient",
    "wq_test_set_wait", "wq_mx_quantize", "wq_mx_decompose", "wq_mx_gemv", "wq_msd_gemm_nf4",
    "wq_msd_decode_attention", "wq_msd_decode_attention_workspace",
    "wq_test_set_attention_split", "wq_kv_block_values",
]


class WqError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, status_string(status), status))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libwq.so not built at %s; run "
                          "`python -m bit_weight_quantized_weights_b200.build_lib`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32, SZ, U32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t, \
        ctypes.c_uint32
    sig = {
        "wq_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "wq_version": ([], ctypes.c_char_p),
        "wq_nf4_codebook": ([ctypes.POINTER(ctypes.c_float)], ctypes.c_int),
        "wq_packed_sizes": ([ctypes.c_int, I64, I64, I32, ctypes.POINTER(SZ),
                             ctypes.POINTER(SZ), ctypes.POINTER(SZ)], ctypes.c_int),
        "wq_quantize_pack": ([ctypes.c_int, P, I64, I64, I32, P, P, P, P], ctypes.c_int),
        "wq_unpack": ([ctypes.c_int, P, I64, I64, P, P], ctypes.c_int),
        "wq_nf4_dequant": ([P, P, I64, I32, P, ctypes.c_int, P], ctypes.c_int),
        "wq_int4_dequant": ([P, P, P, I64, I64, I32, P, ctypes.c_int, P], ctypes.c_int),
        "wq_w4a16_gemv": ([P, I64, I64, I64, ctypes.c_int, I32, P, P, P, P, P, SZ, P],
                          ctypes.c_int),
        "wq_w4a16_gemm": ([P, I64, I64, I64, ctypes.c_int, I32, P, P, P, P, P, SZ, P],
                          ctypes.c_int),
        "wq_msd_decompose": ([P, I64, I64, I32, P, P, P], ctypes.c_int),
        "wq_msd_gemm": ([P, I64, I64, I64, I32, I32, P, P, P, P, P, SZ, P], ctypes.c_int),
        "wq_workspace_bytes": ([ctypes.c_int, I64, I64, I64, I32, I32, ctypes.POINTER(SZ)],
                               ctypes.c_int),
        "wq_device_error": ([P, ctypes.c_int, ctypes.POINTER(U32)], ctypes.c_int),
        "wq_test_set_wait": ([ctypes.c_uint64, ctypes.c_int], ctypes.c_int),
        "wq_mx_quantize": ([P, I64, I64, P, P, P], ctypes.c_int),
        "wq_mx_decompose": ([P, I64, I64, I32, P, P, P], ctypes.c_int),
        "wq_mx_gemv": ([P, I64, I64, I64, I32, P, P, P, P, SZ, P], ctypes.c_int),
        "wq_msd_gemm_nf4": ([P, I64, I64, I64, I32, P, P, P, P, SZ, P], ctypes.c_int),
        "wq_msd_decode_attention": ([P, I64, I64, I64, I64, I32, I32, P, P, P, P, P, P, P, P, SZ,
                                     P], ctypes.c_int),
        "wq_msd_decode_attention_workspace": ([I64, I64, I64, I64, I32, I32, ctypes.POINTER(SZ)],
                                              ctypes.c_int),
        "wq_test_set_attention_split": ([I32], ctypes.c_int),
        "wq_kv_block_values": ([P, I64, I64, I32, P, P], ctypes.c_int),
        "wq_msd_gemm_noalloc": ([P, I64, I64, I64, I32, I32, P, P, P, P, P], ctypes.c_int),
        "wq_residual": ([ctypes.c_int, P, I64, I64, I32, P, P, P, P, P], ctypes.c_int),
        "wq_select_salient": ([P, I64, I64, I32, P, P], ctypes.c_int),
        "wq_w4a16_gemv_corrected": ([P, I64, I64, I64, ctypes.c_int, I32, P, P, P, P, P, I32, P,
                                     P], ctypes.c_int),
        "wq_w4a16_gemv_salient": ([P, I64, I64, I64, ctypes.c_int, I32, P, P, P, P, I32, P, P,
                                   P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def status_string(status):
    return lib.wq_status_string(int(status)).decode()


def version():
    return lib.wq_version().decode()


def _check(status, where):
    if status != WQ_OK:
        raise WqError(status, where)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(t, dtype, name):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


# ---------------------------------------------------------------------------
# host-only queries
# ---------------------------------------------------------------------------

def wq_nf4_codebook():
    """The 16 NF4 code values the kernels use (host computation)."""
    buf = (ctypes.c_float * 16)()
    _check(lib.wq_nf4_codebook(buf), "wq_nf4_codebook")
    return [float(v) for v in buf]


def wq_packed_sizes(fmt, n, k, group):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.wq_packed_sizes(fmt, n, k, group, ctypes.byref(a), ctypes.byref(b),
                               ctypes.byref(c)), "wq_packed_sizes")
    return a.value, b.value, c.value


def wq_workspace_bytes(op, m, n, k, group, n_components=2):
    out = ctypes.c_size_t()
    _check(lib.wq_workspace_bytes(op, m, n, k, group, n_components, ctypes.byref(out)),
           "wq_workspace_bytes")
    return out.value


# ---------------------------------------------------------------------------
# device entry points
# ---------------------------------------------------------------------------

def alloc_packed(fmt, n, k, group, device="cuda"):
    """Allocate (qweight, scales, zeros) tensors of the canonical packed layout."""
    qb, sb, zb = wq_packed_sizes(fmt, n, k, group)
    if fmt == WQ_FMT_INT4_ASYM:
        qw = torch.empty(n, k // 8, dtype=torch.int32, device=device)
        sc = torch.empty(n, k // group, dtype=torch.float16, device=device)
        zr = torch.empty(n, k // group, dtype=torch.float16, device=device)
    else:
        qw = torch.empty(n * k // 2, dtype=torch.uint8, device=device)
        sc = torch.empty(n * k // 64, dtype=torch.float32, device=device)
        zr = None
    assert qw.numel() * qw.element_size() == qb and sc.numel() * sc.element_size() == sb
    return qw, sc, zr


def wq_quantize_pack(fmt, w, group, qweight=None, scales=None, zeros=None, stream=None):
    """Quantize fp32 W [N, K] on the GPU; returns (qweight, scales, zeros)."""
    _cuda(w, torch.float32, "W")
    n, k = w.shape
    if qweight is None:
        qweight, scales, zeros = alloc_packed(fmt, n, k, group, w.device)
    _check(lib.wq_quantize_pack(fmt, _ptr(w), n, k, group, _ptr(qweight), _ptr(scales),
                                _ptr(zeros), _stream(stream)), "wq_quantize_pack")
    return qweight, scales, zeros


def wq_unpack(fmt, qweight, n, k, out=None, stream=None):
    _cuda(qweight, None, "qweight")
    if out is None:
        out = torch.empty(n * k, dtype=torch.uint8, device=qweight.device)
    _check(lib.wq_unpack(fmt, _ptr(qweight), n, k, _ptr(out), _stream(stream)), "wq_unpack")
    return out


def wq_nf4_dequant(codes, absmax, numel, out=None, out_dtype=torch.bfloat16, stream=None):
    _cuda(codes, torch.uint8, "codes")
    _cuda(absmax, torch.float32, "absmax")
    if out is None:
        out = torch.empty(numel, dtype=out_dtype, device=codes.device)
    dt = WQ_BF16 if out.dtype == torch.bfloat16 else WQ_FP16
    _check(lib.wq_nf4_dequant(_ptr(codes), _ptr(absmax), numel, 64, _ptr(out), dt,
                              _stream(stream)), "wq_nf4_dequant")
    return out


def wq_int4_dequant(qweight, scales, zeros, n, k, group, out=None, out_dtype=torch.bfloat16,
                    stream=None):
    _cuda(qweight, torch.int32, "qweight")
    _cuda(scales, torch.float16, "scales")
    _cuda(zeros, torch.float16, "zeros")
    if out is None:
        out = torch.empty(n, k, dtype=out_dtype, device=qweight.device)
    dt = WQ_BF16 if out.dtype == torch.bfloat16 else WQ_FP16
    _check(lib.wq_int4_dequant(_ptr(qweight), _ptr(scales), _ptr(zeros), n, k, group, _ptr(out),
                               dt, _stream(stream)), "wq_int4_dequant")
    return out


def _product(fn, name, x, n, fmt, group, qweight, scales, zeros, out, workspace, stream):
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    if out is None:
        out = torch.empty(m, n, dtype=torch.bfloat16, device=x.device)
    _cuda(out, torch.bfloat16, "y")
    ws = _ptr(workspace)
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(fn(_ptr(x), m, n, k, fmt, group, _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(out),
              ws, wsb, _stream(stream)), name)
    return out


def wq_w4a16_gemv(x, n, fmt, group, qweight, scales, zeros, out=None, stream=None):
    """Decode GEMV: x bf16 [M<=16, K] -> y bf16 [M, N]."""
    return _product(lib.wq_w4a16_gemv, "wq_w4a16_gemv", x, n, fmt, group, qweight, scales, zeros,
                    out, None, stream)


def wq_residual(fmt, w, group, qweight, scales, zeros, out=None, stream=None):
    """R^T = fp16(W - dequant(W_q)) as fp16 [K, N] from fp32 W [N, K]."""
    _cuda(w, torch.float32, "W")
    n, k = w.shape
    if out is None:
        out = torch.empty(k, n, dtype=torch.float16, device=w.device)
    _cuda(out, torch.float16, "residual_t")
    _check(lib.wq_residual(fmt, _ptr(w), n, k, group, _ptr(qweight), _ptr(scales), _ptr(zeros),
                           _ptr(out), _stream(stream)), "wq_residual")
    return out


def wq_select_salient(x, k, out=None, stream=None):
    """The k salient channels of bf16 x [M, K] as int32 [k], increasing."""
    _cuda(x, torch.bfloat16, "x")
    m, kk = x.shape
    if out is None:
        out = torch.empty(max(k, 0), dtype=torch.int32, device=x.device)
    _cuda(out, torch.int32, "idx")
    _check(lib.wq_select_salient(_ptr(x), m, kk, k, _ptr(out), _stream(stream)),
           "wq_select_salient")
    return out


def wq_w4a16_gemv_corrected(x, n, fmt, group, qweight, scales, zeros, residual_t, idx, out=None,
                            stream=None):
    """Decode GEMV plus the residuals of the channels idx (int32 [k])."""
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    if out is None:
        out = torch.empty(m, n, dtype=torch.bfloat16, device=x.device)
    _cuda(out, torch.bfloat16, "y")
    nsel = 0 if idx is None else idx.numel()
    _check(lib.wq_w4a16_gemv_corrected(_ptr(x), m, n, k, fmt, group, _ptr(qweight), _ptr(scales),
                                       _ptr(zeros), _ptr(residual_t), _ptr(idx), nsel, _ptr(out),
                                       _stream(stream)), "wq_w4a16_gemv_corrected")
    return out


def wq_w4a16_gemv_salient(x, n, fmt, group, qweight, scales, zeros, residual_t, nsel, idx=None,
                          out=None, stream=None):
    """One corrected decode step: select the nsel salient channels into idx
    (int32 scratch, allocated if None), then the corrected GEMV, launched to
    overlap the selection. Returns y."""
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    if out is None:
        out = torch.empty(m, n, dtype=torch.bfloat16, device=x.device)
    _cuda(out, torch.bfloat16, "y")
    if idx is None:
        idx = torch.empty(max(nsel, 1), dtype=torch.int32, device=x.device)
    _cuda(idx, torch.int32, "idx")
    _check(lib.wq_w4a16_gemv_salient(_ptr(x), m, n, k, fmt, group, _ptr(qweight), _ptr(scales),
                                     _ptr(zeros), _ptr(residual_t), nsel, _ptr(idx), _ptr(out),
                                     _stream(stream)), "wq_w4a16_gemv_salient")
    return out


def gemm_workspace(m, n, k, group, device="cuda"):
    nbytes = wq_workspace_bytes(WQ_OP_GEMM, m, n, k, group)
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def wq_w4a16_gemm(x, n, fmt, group, qweight, scales, zeros, workspace=None, out=None,
                  stream=None):
    """Prefill GEMM with fused dequantization on tcgen05: y bf16 [M, N]."""
    _cuda(x, torch.bfloat16, "x")
    if workspace is None:
        workspace = gemm_workspace(x.shape[0], n, x.shape[1], group, x.device)
    return _product(lib.wq_w4a16_gemm, "wq_w4a16_gemm", x, n, fmt, group, qweight, scales, zeros,
                    out, workspace, stream)


def wq_msd_decompose(x, n_components=2, digits=None, comp_scales=None, stream=None):
    """Digit planes int8 [C, M, K] and scales fp32 [C, M] of bf16 x [M, K]."""
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    if digits is None:
        digits = torch.empty(n_components, m, k, dtype=torch.int8, device=x.device)
        comp_scales = torch.empty(n_components, m, dtype=torch.float32, device=x.device)
    _check(lib.wq_msd_decompose(_ptr(x), m, k, n_components, _ptr(digits), _ptr(comp_scales),
                                _stream(stream)), "wq_msd_decompose")
    return digits, comp_scales


def msd_workspace(m, n, k, group, n_components=2, device="cuda"):
    nbytes = wq_workspace_bytes(WQ_OP_MSD_GEMM, m, n, k, group, n_components)
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def wq_msd_gemm(x, n, n_components, group, qweight, scales, zeros, workspace=None, out=None,
                stream=None):
    """Multi-Scale Dequant GEMM: y bf16 [M, N] from int8 digit planes of x."""
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    if workspace is None:
        workspace = msd_workspace(m, n, k, group, n_components, x.device)
    if out is None:
        out = torch.empty(m, n, dtype=torch.bfloat16, device=x.device)
    _check(lib.wq_msd_gemm(_ptr(x), m, n, k, n_components, group, _ptr(qweight), _ptr(scales),
                           _ptr(zeros), _ptr(out), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream)),
           "wq_msd_gemm")
    return out


def wq_msd_gemm_noalloc(x, n, n_components, group, qweight, scales, zeros, out=None,
                        stream=None):
    """wq_msd_gemm without a workspace: the library's fixed device scratch array
    is used, so the call allocates nothing (problem size limited to 8 MiB of
    scratch; calls overlapping on the GPU race on it)."""
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    if out is None:
        out = torch.empty(m, n, dtype=torch.bfloat16, device=x.device)
    _check(lib.wq_msd_gemm_noalloc(_ptr(x), m, n, k, n_components, group, _ptr(qweight),
                                   _ptr(scales), _ptr(zeros), _ptr(out), _stream(stream)),
           "wq_msd_gemm_noalloc")
    return out


def wq_device_error(clear=True, stream=None):
    """Synchronise and read the sticky device error word: (status, detail)."""
    d = ctypes.c_uint32()
    st = lib.wq_device_error(_stream(stream), 1 if clear else 0, ctypes.byref(d))
    return st, d.value


def wq_test_set_wait(limit_ns=0, stall=0):
    """Test hook of the bounded device waits (see include/wq.h): the wait
    limit in ns (0 = the default 2 s) and whether the loader withholds the
    first k-tile of the tensor-core kernels."""
    _check(lib.wq_test_set_wait(int(limit_ns), int(stall)), "wq_test_set_wait")


def wq_mx_quantize(w, codes=None, scales=None, stream=None):
    """MXFP4 weights: w fp32 [N, K] -> (codes uint8 [N, K/2], scale bytes uint8 [N, K/32])."""
    _cuda(w, torch.float32, "w")
    n, k = w.shape
    if codes is None:
        codes = torch.empty(n, k // 2, dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(n, k // 32, dtype=torch.uint8, device=w.device)
    _check(lib.wq_mx_quantize(_ptr(w), n, k, _ptr(codes), _ptr(scales), _stream(stream)),
           "wq_mx_quantize")
    return codes, scales


def wq_mx_decompose(x, n_passes=2, planes=None, scales=None, stream=None):
    """x bf16 [M, K] -> (planes uint8 [P, M, K] E4M3 bytes, scale bytes uint8 [P, M, K/32])."""
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    if planes is None:
        planes = torch.empty(n_passes, m, k, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(n_passes, m, k // 32, dtype=torch.uint8, device=x.device)
    _check(lib.wq_mx_decompose(_ptr(x), m, k, n_passes, _ptr(planes), _ptr(scales),
                               _stream(stream)), "wq_mx_decompose")
    return planes, scales


def mx_workspace(m, n, k, n_passes=2, device="cuda"):
    nbytes = wq_workspace_bytes(WQ_OP_MX_GEMV, m, n, k, 0, n_passes)
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def wq_mx_gemv(x, n, n_passes, codes, scales, workspace=None, out=None, stream=None):
    """y bf16 [M, N] = x_hat . w_hat^T (MXFP4 weights; two MXFP4 passes or one MXFP8 pass)."""
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    if workspace is None:
        workspace = mx_workspace(m, n, k, n_passes, x.device)
    if out is None:
        out = torch.empty(m, n, dtype=torch.bfloat16, device=x.device)
    _check(lib.wq_mx_gemv(_ptr(x), m, n, k, n_passes, _ptr(codes), _ptr(scales), _ptr(out),
                          _ptr(workspace), workspace.numel(), _stream(stream)), "wq_mx_gemv")
    return out


def wq_msd_gemm_nf4(x, n, n_components, codes, absmax, workspace=None, out=None, stream=None):
    """Decode MSD product with NF4 weights (integer codebook digits); M <= 16."""
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    if workspace is None:
        workspace = msd_workspace(m, n, k, 64, n_components, x.device)
    if out is None:
        out = torch.empty(m, n, dtype=torch.bfloat16, device=x.device)
    _check(lib.wq_msd_gemm_nf4(_ptr(x), m, n, k, n_components, _ptr(codes), _ptr(absmax),
                               _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)),
           "wq_msd_gemm_nf4")
    return out


def kv_quantize_keys(k, stream=None):
    """INT4-quantize a key cache fp32 [B, Hkv, L, D] on the GPU, one group per
    (sequence, head, token) row: returns (codes int32 [B, Hkv, L, D/8], scales
    fp16 [B, Hkv, L], zeros fp16 [B, Hkv, L])."""
    _cuda(k, torch.float32, "k")
    b, hkv, length, d = k.shape
    qw, sc, zr = wq_quantize_pack(WQ_FMT_INT4_ASYM, k.reshape(-1, d), d, stream=stream)
    return (qw.view(b, hkv, length, d // 8), sc.view(b, hkv, length), zr.view(b, hkv, length))


def wq_kv_block_values(codes, rows, length, d, out=None, stream=None):
    """V codes from the token layout (int32 [rows * L, D/8]) to blocks of 8
    tokens: int32 [rows, ceil(L/8), D]."""
    _cuda(codes, torch.int32, "codes")
    nblk = (length + 7) // 8
    if out is None:
        out = torch.empty(rows, nblk, d, dtype=torch.int32, device=codes.device)
    _check(lib.wq_kv_block_values(_ptr(codes), rows, length, d, _ptr(out), _stream(stream)),
           "wq_kv_block_values")
    return out


def kv_quantize_values(v, stream=None):
    """INT4-quantize a value cache fp32 [B, Hkv, L, D] on the GPU, one group per
    (sequence, head, token) row: returns (codes int32 [B, Hkv, ceil(L/8), D] in
    blocks of 8 tokens, scales fp16 [B, Hkv, L], zeros fp16 [B, Hkv, L])."""
    _cuda(v, torch.float32, "v")
    b, hkv, length, d = v.shape
    qw, sc, zr = wq_quantize_pack(WQ_FMT_INT4_ASYM, v.reshape(-1, d), d, stream=stream)
    blocked = wq_kv_block_values(qw, b * hkv, length, d, stream=stream)
    return (blocked.view(b, hkv, (length + 7) // 8, d), sc.view(b, hkv, length),
            zr.view(b, hkv, length))


def attention_workspace(b, hq, hkv, length, d, n_components, device):
    size = ctypes.c_size_t(0)
    _check(lib.wq_msd_decode_attention_workspace(b, hq, hkv, length, d, n_components,
                                                 ctypes.byref(size)),
           "wq_msd_decode_attention_workspace")
    return torch.empty(max(int(size.value), 1), dtype=torch.uint8, device=device)


def wq_msd_decode_attention(q, k_cache, v_cache, n_components=2, workspace=None, out=None,
                            stream=None):
    """MSD decode attention: q bf16 [B, Hq, D]; k_cache and v_cache = (codes,
    scales, zeros) as kv_quantize_keys and kv_quantize_values return them.
    Returns out bf16 [B, Hq, D]."""
    _cuda(q, torch.bfloat16, "q")
    b, hq, d = q.shape
    kq, ks, kz = k_cache
    vq, vs, vz = v_cache
    hkv, length = ks.shape[1], ks.shape[2]
    for t, dt, name in ((kq, torch.int32, "k_codes"), (ks, torch.float16, "k_scales"),
                        (kz, torch.float16, "k_zeros"), (vq, torch.int32, "v_codes"),
                        (vs, torch.float16, "v_scales"), (vz, torch.float16, "v_zeros")):
        _cuda(t, dt, name)
    if tuple(kq.shape) != (b, hkv, length, d // 8) or \
            tuple(vq.shape) != (b, hkv, (length + 7) // 8, d) or \
            tuple(vs.shape) != tuple(ks.shape) or tuple(kz.shape) != tuple(ks.shape) or \
            tuple(vz.shape) != tuple(ks.shape) or ks.shape[0] != b:
        raise ValueError("KV cache shapes do not match q")
    if workspace is None:
        workspace = attention_workspace(b, hq, hkv, length, d, n_components, q.device)
    if out is None:
        out = torch.empty(b, hq, d, dtype=torch.bfloat16, device=q.device)
    _check(lib.wq_msd_decode_attention(_ptr(q), b, hq, hkv, length, d, n_components, _ptr(kq),
                                       _ptr(ks), _ptr(kz), _ptr(vq), _ptr(vs), _ptr(vz), _ptr(out),
                                       _ptr(workspace), workspace.numel(), _stream(stream)),
           "wq_msd_decode_attention")
    return out


def wq_test_set_attention_split(chunks_per_cta=0):
    """Fix the attention kernel's chunks per CTA (0: chosen per launch)."""
    _check(lib.wq_test_set_attention_split(chunks_per_cta), "wq_test_set_attention_split")
