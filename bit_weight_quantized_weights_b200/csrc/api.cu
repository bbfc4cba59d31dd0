// C ABI of the library: argument validation and dispatch to the kernels.
// Every check happens before any launch; no C++ exception crosses the ABI.
#include <atomic>
#include <cstring>
#include <exception>

#include "common.cuh"

namespace wq {
wq_status launch_quantize_pack(wq_format, const float*, int64_t, int64_t, int32_t, void*, void*,
                               void*, cudaStream_t);
wq_status launch_unpack(wq_format, const void*, int64_t, int64_t, uint8_t*, cudaStream_t);
wq_status launch_nf4_dequant(const uint8_t*, const float*, int64_t, void*, wq_dtype, cudaStream_t);
wq_status launch_int4_dequant(const uint32_t*, const void*, const void*, int64_t, int64_t, int32_t,
                              void*, wq_dtype, cudaStream_t);
wq_status launch_gemv(const void*, int64_t, int64_t, int64_t, wq_format, int32_t, const void*,
                      const void*, const void*, void*, cudaStream_t,
                      const void* residual_t = nullptr, const int32_t* idx = nullptr,
                      int32_t k = 0, bool early = false);
wq_status launch_residual(wq_format, const float*, int64_t, int64_t, int32_t, const void*,
                          const void*, const void*, void*, cudaStream_t);
wq_status launch_select_salient(const void*, int64_t, int64_t, int32_t, int32_t*, cudaStream_t);
wq_status launch_gemm(const void*, int64_t, int64_t, int64_t, wq_format, int32_t, const void*,
                      const void*, const void*, void*, void*, cudaStream_t);
size_t gemm_workspace_bytes(int64_t M, int64_t K);
wq_status launch_msd_decompose(const void*, int64_t, int64_t, int32_t, int64_t, int8_t*, float*,
                               cudaStream_t);
wq_status launch_msd_gemm(const void*, int64_t, int64_t, int64_t, int32_t, int32_t, const void*,
                          const void*, const void*, void*, void*, cudaStream_t);
size_t msd_workspace_bytes(int64_t M, int64_t K, int32_t C);
wq_status launch_mx_quantize(const float*, int64_t, int64_t, uint8_t*, uint8_t*, cudaStream_t);
wq_status launch_mx_decompose(const void*, int64_t, int64_t, int32_t, uint8_t*, uint8_t*,
                              cudaStream_t);
wq_status launch_mx_gemv(const void*, int64_t, int64_t, int64_t, int32_t, const uint8_t*,
                         const uint8_t*, void*, void*, cudaStream_t);
size_t mx_workspace_bytes(int64_t M, int64_t K, int32_t P);
wq_status launch_msd_nf4(const void*, int64_t, int64_t, int64_t, int32_t, const uint8_t*,
                         const float*, void*, void*, cudaStream_t);
size_t kv_msd_workspace_bytes(int64_t B, int64_t Hq, int64_t L, int32_t C);
wq_status launch_kv_block_values(const uint32_t*, int64_t, int64_t, int32_t, uint32_t*,
                                 cudaStream_t);
extern std::atomic<int> g_kv_chunks_per_cta;
wq_status launch_kv_msd(const void*, int64_t, int64_t, int64_t, int64_t, int32_t, const void*,
                        const void*, const void*, const void*, const void*, const void*, void*,
                        void*, cudaStream_t);
wq_status read_gemm_error(bool clear, uint32_t* v);
wq_status read_msd_error(bool clear, uint32_t* v);
wq_status read_gemv_error(bool clear, uint32_t* v);
}  // namespace wq

namespace wq {
namespace {
std::atomic<uint64_t> g_wait_limit_ns{0};  // 0: the default
std::atomic<int> g_wait_stall{0};
}  // namespace

WaitCtl wait_ctl() {
  const uint64_t l = g_wait_limit_ns.load(std::memory_order_relaxed);
  return WaitCtl{l ? l : sm100_default_wait_ns(), g_wait_stall.load(std::memory_order_relaxed)};
}
}  // namespace wq

using namespace wq;

namespace {

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

template <typename F>
wq_status guarded(F&& f) {
  try {
    return f();
  } catch (...) {
    return WQ_ERR_CUDA;
  }
}

bool all_aligned(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p && !aligned16(p)) return false;
  return true;
}

// INT4: group % 8, K % group; NF4: group == 64 and N*K % 64.
wq_status check_format(wq_format fmt, int64_t N, int64_t K, int32_t group) {
  if (N < 0 || K <= 0) return WQ_ERR_INVALID_ARG;
  if (fmt == WQ_FMT_INT4_ASYM) {
    if (group <= 0 || group % 8 != 0 || K % group != 0) return WQ_ERR_INVALID_ARG;
  } else if (fmt == WQ_FMT_NF4) {
    if (group != 64 || (N * K) % 64 != 0) return WQ_ERR_INVALID_ARG;
  } else {
    return WQ_ERR_INVALID_ARG;
  }
  if (K % 8 != 0) return WQ_ERR_INVALID_ARG;
  return WQ_OK;
}

// Shared checks of the product entry points.
wq_status check_product(const void* x, int64_t M, int64_t N, int64_t K, wq_format fmt,
                        int32_t group, const void* qweight, const void* scales, const void* zeros,
                        const void* y) {
  if (M < 0 || N < 0 || K <= 0) return WQ_ERR_INVALID_ARG;
  wq_status s = check_format(fmt, N, K, group);
  if (s != WQ_OK) return s;
  if (M == 0 || N == 0) return WQ_OK;
  if (!x || !qweight || !scales || !y) return WQ_ERR_INVALID_ARG;
  if (fmt == WQ_FMT_INT4_ASYM && !zeros) return WQ_ERR_INVALID_ARG;
  if (fmt == WQ_FMT_NF4 && zeros) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({x, qweight, scales, zeros, y})) return WQ_ERR_ALIGNMENT;
  if (K % 128 != 0) return WQ_ERR_UNSUPPORTED;
  if (fmt == WQ_FMT_INT4_ASYM && group % 64 != 0) return WQ_ERR_UNSUPPORTED;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return WQ_ERR_UNSUPPORTED;
  return WQ_OK;
}

// Shape checks of the KV-cache attention: WQ_OK, or the status to return.
wq_status check_attention_shape(int64_t B, int64_t Hq, int64_t Hkv, int64_t L, int32_t D,
                                int32_t n_components) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || D <= 0 || D % 8 != 0)
    return WQ_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || n_components < 1 || n_components > 3) return WQ_ERR_INVALID_ARG;
  const int64_t R = Hq / Hkv;
  if (D != 128 || n_components == 3 || (R != 1 && R != 2 && R != 4 && R != 8))
    return WQ_ERR_UNSUPPORTED;
  if (B > 65535 || Hkv > 65535 || L > INT32_MAX - 256 || B * Hq > INT32_MAX)
    return WQ_ERR_UNSUPPORTED;
  return WQ_OK;
}

}  // namespace

extern "C" {

const char* wq_status_string(wq_status s) {
  switch (s) {
    case WQ_OK: return "ok";
    case WQ_ERR_INVALID_ARG: return "invalid argument";
    case WQ_ERR_UNSUPPORTED: return "unsupported shape, group or format";
    case WQ_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case WQ_ERR_CUDA: return "CUDA error";
    case WQ_ERR_TIMEOUT: return "bounded device wait expired";
    case WQ_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char* wq_version(void) { return "wq 0.1 sm_100a"; }

wq_status wq_nf4_codebook(float out[16]) {
  if (!out) return WQ_ERR_INVALID_ARG;
  return guarded([&] {
    std::memcpy(out, nf4_table().v, sizeof(float) * 16);
    return WQ_OK;
  });
}

wq_status wq_packed_sizes(wq_format fmt, int64_t N, int64_t K, int32_t group,
                          size_t* qweight_bytes, size_t* scale_bytes, size_t* zero_bytes) {
  if (!qweight_bytes || !scale_bytes || !zero_bytes) return WQ_ERR_INVALID_ARG;
  wq_status s = check_format(fmt, N, K, group);
  if (s != WQ_OK) return s;
  *qweight_bytes = (size_t)(N * K / 2);
  if (fmt == WQ_FMT_INT4_ASYM) {
    *scale_bytes = (size_t)(N * (K / group) * 2);
    *zero_bytes = *scale_bytes;
  } else {
    *scale_bytes = (size_t)(N * K / 64 * 4);
    *zero_bytes = 0;
  }
  return WQ_OK;
}

wq_status wq_quantize_pack(wq_format fmt, const float* W, int64_t N, int64_t K, int32_t group,
                           void* qweight, void* scales, void* zeros, void* stream) {
  wq_status s = check_format(fmt, N, K, group);
  if (s != WQ_OK) return s;
  if (N == 0) return WQ_OK;
  if (!W || !qweight || !scales) return WQ_ERR_INVALID_ARG;
  if (fmt == WQ_FMT_INT4_ASYM && !zeros) return WQ_ERR_INVALID_ARG;
  if (fmt == WQ_FMT_NF4 && zeros) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({W, qweight, scales, zeros})) return WQ_ERR_ALIGNMENT;
  return guarded(
      [&] { return launch_quantize_pack(fmt, W, N, K, group, qweight, scales, zeros, as_stream(stream)); });
}

wq_status wq_unpack(wq_format fmt, const void* qweight, int64_t N, int64_t K, uint8_t* codes,
                    void* stream) {
  if (N < 0 || K <= 0 || K % 8 != 0) return WQ_ERR_INVALID_ARG;
  if (fmt != WQ_FMT_INT4_ASYM && fmt != WQ_FMT_NF4) return WQ_ERR_INVALID_ARG;
  if (N == 0) return WQ_OK;
  if (!qweight || !codes) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({qweight, codes})) return WQ_ERR_ALIGNMENT;
  return guarded([&] { return launch_unpack(fmt, qweight, N, K, codes, as_stream(stream)); });
}

wq_status wq_nf4_dequant(const uint8_t* codes, const float* absmax, int64_t numel,
                         int32_t blocksize, void* out, wq_dtype out_dtype, void* stream) {
  if (numel < 0 || blocksize != 64 || numel % 64 != 0) return WQ_ERR_INVALID_ARG;
  if (out_dtype != WQ_BF16 && out_dtype != WQ_FP16) return WQ_ERR_UNSUPPORTED;
  if (numel == 0) return WQ_OK;
  if (!codes || !absmax || !out) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({codes, absmax, out})) return WQ_ERR_ALIGNMENT;
  return guarded(
      [&] { return launch_nf4_dequant(codes, absmax, numel, out, out_dtype, as_stream(stream)); });
}

wq_status wq_int4_dequant(const uint32_t* qweight, const void* scales, const void* zeros,
                          int64_t N, int64_t K, int32_t group, void* out, wq_dtype out_dtype,
                          void* stream) {
  wq_status s = check_format(WQ_FMT_INT4_ASYM, N, K, group);
  if (s != WQ_OK) return s;
  if (out_dtype != WQ_BF16 && out_dtype != WQ_FP16) return WQ_ERR_UNSUPPORTED;
  if (N == 0) return WQ_OK;
  if (!qweight || !scales || !zeros || !out) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({qweight, scales, zeros, out})) return WQ_ERR_ALIGNMENT;
  return guarded([&] {
    return launch_int4_dequant(qweight, scales, zeros, N, K, group, out, out_dtype,
                               as_stream(stream));
  });
}

wq_status wq_w4a16_gemv(const void* x, int64_t M, int64_t N, int64_t K, wq_format fmt,
                        int32_t group, const void* qweight, const void* scales, const void* zeros,
                        void* y, void* workspace, size_t ws_bytes, void* stream) {
  (void)workspace;
  (void)ws_bytes;
  wq_status s = check_product(x, M, N, K, fmt, group, qweight, scales, zeros, y);
  if (s != WQ_OK) return s;
  if (M > 16) return WQ_ERR_UNSUPPORTED;
  if (N % 16 != 0) return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  return guarded([&] {
    return launch_gemv(x, M, N, K, fmt, group, qweight, scales, zeros, y, as_stream(stream));
  });
}

wq_status wq_residual(wq_format fmt, const float* W, int64_t N, int64_t K, int32_t group,
                      const void* qweight, const void* scales, const void* zeros,
                      void* residual_t, void* stream) {
  wq_status s = check_format(fmt, N, K, group);
  if (s != WQ_OK) return s;
  if (N == 0) return WQ_OK;
  if (!W || !qweight || !scales || !residual_t) return WQ_ERR_INVALID_ARG;
  if (fmt == WQ_FMT_INT4_ASYM && !zeros) return WQ_ERR_INVALID_ARG;
  if (fmt == WQ_FMT_NF4 && zeros) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({W, qweight, scales, zeros, residual_t})) return WQ_ERR_ALIGNMENT;
  if (K % 64 != 0 || N % 8 != 0) return WQ_ERR_UNSUPPORTED;
  if (N > INT32_MAX || K > INT32_MAX || (N + 63) / 64 > 65535) return WQ_ERR_UNSUPPORTED;
  return guarded([&] {
    return launch_residual(fmt, W, N, K, group, qweight, scales, zeros, residual_t,
                           as_stream(stream));
  });
}

wq_status wq_select_salient(const void* x, int64_t M, int64_t K, int32_t k, int32_t* idx,
                            void* stream) {
  if (M <= 0 || K <= 0 || k < 0 || k > K) return WQ_ERR_INVALID_ARG;
  if (k == 0) return WQ_OK;
  if (!x || !idx) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({x, idx})) return WQ_ERR_ALIGNMENT;
  if (K > 65536 || M > INT32_MAX) return WQ_ERR_UNSUPPORTED;
  return guarded([&] { return launch_select_salient(x, M, K, k, idx, as_stream(stream)); });
}

wq_status wq_w4a16_gemv_corrected(const void* x, int64_t M, int64_t N, int64_t K, wq_format fmt,
                                  int32_t group, const void* qweight, const void* scales,
                                  const void* zeros, const void* residual_t, const int32_t* idx,
                                  int32_t k, void* y, void* stream) {
  wq_status s = check_product(x, M, N, K, fmt, group, qweight, scales, zeros, y);
  if (s != WQ_OK) return s;
  if (k < 0 || k > K) return WQ_ERR_INVALID_ARG;
  if (M > 16) return WQ_ERR_UNSUPPORTED;
  if (N % 16 != 0) return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  if (k > 0) {
    if (!residual_t || !idx) return WQ_ERR_INVALID_ARG;
    if (!all_aligned({residual_t, idx})) return WQ_ERR_ALIGNMENT;
  }
  return guarded([&] {
    return launch_gemv(x, M, N, K, fmt, group, qweight, scales, zeros, y, as_stream(stream),
                       residual_t, idx, k);
  });
}

wq_status wq_w4a16_gemv_salient(const void* x, int64_t M, int64_t N, int64_t K, wq_format fmt,
                                int32_t group, const void* qweight, const void* scales,
                                const void* zeros, const void* residual_t, int32_t k,
                                int32_t* idx, void* y, void* stream) {
  wq_status s = check_product(x, M, N, K, fmt, group, qweight, scales, zeros, y);
  if (s != WQ_OK) return s;
  if (k < 0 || k > K) return WQ_ERR_INVALID_ARG;
  if (M > 16) return WQ_ERR_UNSUPPORTED;
  if (N % 16 != 0) return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  if (k > 0) {
    if (!residual_t || !idx) return WQ_ERR_INVALID_ARG;
    if (!all_aligned({residual_t, idx})) return WQ_ERR_ALIGNMENT;
    if (K > 65536) return WQ_ERR_UNSUPPORTED;
  }
  return guarded([&] {
    if (k > 0) {
      const wq_status r = launch_select_salient(x, M, K, k, idx, as_stream(stream));
      if (r != WQ_OK) return r;
    }
    return launch_gemv(x, M, N, K, fmt, group, qweight, scales, zeros, y, as_stream(stream),
                       residual_t, idx, k, /*early=*/true);
  });
}

wq_status wq_w4a16_gemm(const void* x, int64_t M, int64_t N, int64_t K, wq_format fmt,
                        int32_t group, const void* qweight, const void* scales, const void* zeros,
                        void* y, void* workspace, size_t ws_bytes, void* stream) {
  wq_status s = check_product(x, M, N, K, fmt, group, qweight, scales, zeros, y);
  if (s != WQ_OK) return s;
  if (N % 128 != 0) return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  if (!workspace || ws_bytes < gemm_workspace_bytes(M, K)) return WQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return WQ_ERR_ALIGNMENT;
  return guarded([&] {
    return launch_gemm(x, M, N, K, fmt, group, qweight, scales, zeros, y, workspace,
                       as_stream(stream));
  });
}

wq_status wq_msd_decompose(const void* x, int64_t M, int64_t K, int32_t n_components,
                           int8_t* digits, float* comp_scales, void* stream) {
  if (M < 0 || K <= 0 || K % 16 != 0) return WQ_ERR_INVALID_ARG;
  if (n_components < 1 || n_components > 3) return WQ_ERR_INVALID_ARG;
  if (M == 0) return WQ_OK;
  if (!x || !digits || !comp_scales) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({x, digits, comp_scales})) return WQ_ERR_ALIGNMENT;
  if (M > INT32_MAX || K > INT32_MAX) return WQ_ERR_UNSUPPORTED;
  return guarded([&] {
    return launch_msd_decompose(x, M, K, n_components, M, digits, comp_scales, as_stream(stream));
  });
}

wq_status wq_msd_gemm(const void* x, int64_t M, int64_t N, int64_t K, int32_t n_components,
                      int32_t group, const void* qweight, const void* scales, const void* zeros,
                      void* y, void* workspace, size_t ws_bytes, void* stream) {
  wq_status s = check_product(x, M, N, K, WQ_FMT_INT4_ASYM, group, qweight, scales, zeros, y);
  if (s != WQ_OK) return s;
  if (n_components < 1 || n_components > 3) return WQ_ERR_INVALID_ARG;
  if (group % 128 != 0 || N % 128 != 0) return WQ_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return WQ_OK;
  const size_t need = msd_workspace_bytes(M, K, n_components);
  if (!workspace || ws_bytes < need) return WQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return WQ_ERR_ALIGNMENT;
  return guarded([&] {
    return launch_msd_gemm(x, M, N, K, n_components, group, qweight, scales, zeros, y, workspace,
                           as_stream(stream));
  });
}

wq_status wq_msd_gemm_nf4(const void* x, int64_t M, int64_t N, int64_t K, int32_t n_components,
                          const uint8_t* codes, const float* absmax, void* y, void* workspace,
                          size_t ws_bytes, void* stream) {
  wq_status s = check_product(x, M, N, K, WQ_FMT_NF4, 64, codes, absmax, nullptr, y);
  if (s != WQ_OK) return s;
  if (n_components < 1 || n_components > 3) return WQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return WQ_OK;
  if (M > 16 || K % 256 != 0 || N % 16 != 0) return WQ_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < msd_workspace_bytes(M, K, n_components)) return WQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return WQ_ERR_ALIGNMENT;
  return guarded([&] {
    return launch_msd_nf4(x, M, N, K, n_components, codes, absmax, y, workspace,
                          as_stream(stream));
  });
}

wq_status wq_mx_quantize(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* scales,
                         void* stream) {
  if (N < 0 || K <= 0 || K % 32 != 0) return WQ_ERR_INVALID_ARG;
  if (N == 0) return WQ_OK;
  if (!W || !codes || !scales) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({W, codes, scales})) return WQ_ERR_ALIGNMENT;
  return guarded([&] { return launch_mx_quantize(W, N, K, codes, scales, as_stream(stream)); });
}

wq_status wq_mx_decompose(const void* x, int64_t M, int64_t K, int32_t n_passes, uint8_t* planes,
                          uint8_t* scales, void* stream) {
  if (M < 0 || K <= 0 || K % 32 != 0) return WQ_ERR_INVALID_ARG;
  if (n_passes != 1 && n_passes != 2) return WQ_ERR_INVALID_ARG;
  if (M == 0) return WQ_OK;
  if (!x || !planes || !scales) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({x, planes, scales})) return WQ_ERR_ALIGNMENT;
  if (M > INT32_MAX || K > INT32_MAX) return WQ_ERR_UNSUPPORTED;
  return guarded(
      [&] { return launch_mx_decompose(x, M, K, n_passes, planes, scales, as_stream(stream)); });
}

wq_status wq_mx_gemv(const void* x, int64_t M, int64_t N, int64_t K, int32_t n_passes,
                     const uint8_t* codes, const uint8_t* scales, void* y, void* workspace,
                     size_t ws_bytes, void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % 32 != 0) return WQ_ERR_INVALID_ARG;
  if (n_passes != 1 && n_passes != 2) return WQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return WQ_OK;
  if (!x || !codes || !scales || !y) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({x, codes, scales, y})) return WQ_ERR_ALIGNMENT;
  if (M > 16 || K % 256 != 0 || N % 16 != 0) return WQ_ERR_UNSUPPORTED;
  if (N > INT32_MAX || K > INT32_MAX) return WQ_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < mx_workspace_bytes(M, K, n_passes)) return WQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return WQ_ERR_ALIGNMENT;
  return guarded([&] {
    return launch_mx_gemv(x, M, N, K, n_passes, codes, scales, y, workspace, as_stream(stream));
  });
}

wq_status wq_kv_block_values(const uint32_t* codes, int64_t rows, int64_t L, int32_t D,
                             uint32_t* out, void* stream) {
  if (rows < 0 || L <= 0 || D <= 0 || D % 8 != 0) return WQ_ERR_INVALID_ARG;
  if (rows == 0) return WQ_OK;
  if (!codes || !out) return WQ_ERR_INVALID_ARG;
  if (!all_aligned({codes, out})) return WQ_ERR_ALIGNMENT;
  if (L > INT32_MAX - 8 || D > 65536) return WQ_ERR_UNSUPPORTED;
  return guarded([&] { return launch_kv_block_values(codes, rows, L, D, out, as_stream(stream)); });
}

wq_status wq_msd_decode_attention_workspace(int64_t B, int64_t Hq, int64_t Hkv, int64_t L,
                                            int32_t D, int32_t n_components, size_t* bytes) {
  if (!bytes) return WQ_ERR_INVALID_ARG;
  wq_status s = check_attention_shape(B, Hq, Hkv, L, D, n_components);
  if (s != WQ_OK) return s;
  *bytes = B == 0 ? 0 : kv_msd_workspace_bytes(B, Hq, L, n_components);
  return WQ_OK;
}

wq_status wq_msd_decode_attention(const void* q, int64_t B, int64_t Hq, int64_t Hkv, int64_t L,
                                  int32_t D, int32_t n_components, const void* k_codes,
                                  const void* k_scales, const void* k_zeros, const void* v_codes,
                                  const void* v_scales, const void* v_zeros, void* out,
                                  void* workspace, size_t ws_bytes, void* stream) {
  wq_status s = check_attention_shape(B, Hq, Hkv, L, D, n_components);
  if (s != WQ_OK) return s;
  if (B == 0) return WQ_OK;
  if (!q || !k_codes || !k_scales || !k_zeros || !v_codes || !v_scales || !v_zeros || !out)
    return WQ_ERR_INVALID_ARG;
  if (!all_aligned({q, k_codes, k_scales, k_zeros, v_codes, v_scales, v_zeros, out}))
    return WQ_ERR_ALIGNMENT;
  if (!workspace || ws_bytes < kv_msd_workspace_bytes(B, Hq, L, n_components))
    return WQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return WQ_ERR_ALIGNMENT;
  return guarded([&] {
    return launch_kv_msd(q, B, Hq, Hkv, L, n_components, k_codes, k_scales, k_zeros, v_codes,
                         v_scales, v_zeros, out, workspace, as_stream(stream));
  });
}

wq_status wq_workspace_bytes(wq_op op, int64_t M, int64_t N, int64_t K, int32_t group,
                             int32_t n_components, size_t* bytes) {
  (void)N;
  (void)group;
  if (!bytes || M < 0 || K < 0) return WQ_ERR_INVALID_ARG;
  switch (op) {
    case WQ_OP_GEMV:
      *bytes = 0;
      return WQ_OK;
    case WQ_OP_GEMM:
      *bytes = M == 0 ? 0 : gemm_workspace_bytes(M, K);
      return WQ_OK;
    case WQ_OP_MSD_GEMM:
      if (n_components < 1 || n_components > 3) return WQ_ERR_INVALID_ARG;
      *bytes = M == 0 ? 0 : msd_workspace_bytes(M, K, n_components);
      return WQ_OK;
    case WQ_OP_MX_GEMV:
      if (n_components != 1 && n_components != 2) return WQ_ERR_INVALID_ARG;
      *bytes = M == 0 ? 0 : mx_workspace_bytes(M, K, n_components);
      return WQ_OK;
  }
  return WQ_ERR_INVALID_ARG;
}

wq_status wq_test_set_wait(uint64_t limit_ns, int stall) {
  if (stall != 0 && stall != 1) return WQ_ERR_INVALID_ARG;
  g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
  g_wait_stall.store(stall, std::memory_order_relaxed);
  return WQ_OK;
}

wq_status wq_test_set_attention_split(int32_t chunks_per_cta) {
  if (chunks_per_cta < 0 || chunks_per_cta > 64) return WQ_ERR_INVALID_ARG;
  g_kv_chunks_per_cta.store(chunks_per_cta, std::memory_order_relaxed);
  return WQ_OK;
}

wq_status wq_device_error(void* stream, int clear, uint32_t* detail) {
  return guarded([&] {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return WQ_ERR_CUDA;
    uint32_t a = 0, b = 0, c = 0;
    wq_status s = read_gemm_error(clear != 0, &a);
    if (s != WQ_OK) return s;
    s = read_msd_error(clear != 0, &b);
    if (s != WQ_OK) return s;
    s = read_gemv_error(clear != 0, &c);
    if (s != WQ_OK) return s;
    if (detail) *detail = a ? a : (b ? b : c);
    return (a || b || c) ? WQ_ERR_TIMEOUT : WQ_OK;
  });
}

}  // extern "C"
