// Multi-Scale Dequant GEMM without caller workspace and without allocation.
//
// wq_msd_gemm needs scratch memory for the activation digit planes and their
// scales, and asks the caller for it. Some callers cannot provide or obtain
// device memory at call time: an engine whose memory is carved up once at
// start-up and which must not grow, a host application embedding the library
// behind a fixed-signature plugin API with no workspace argument, or a
// latency-critical loop where a device allocation (which can synchronise the
// device) is not allowed. For them this file keeps the scratch in a
// file-scope device array of fixed size, so every call runs with no
// cudaMalloc, no cudaFree and no allocating library routine.
#include <mutex>

#include "common.cuh"

namespace wq {
wq_status launch_msd_gemm(const void*, int64_t, int64_t, int64_t, int32_t, int32_t, const void*,
                          const void*, const void*, void*, void*, cudaStream_t);
size_t msd_workspace_bytes(int64_t M, int64_t K, int32_t C);
}  // namespace wq

namespace {

// 8 MiB of device memory, reserved on every GPU that loads the library until
// the process exits. Enough for M up to 128 tokens at K = 25600 with two
// components (all decode and small-prefill shapes of the Qwen3-32B layers).
constexpr size_t kScratchBytes = size_t(8) << 20;
static __device__ __align__(256) uint8_t g_msd_noalloc_scratch[kScratchBytes];

// The array's name is only a host-side stand-in in host code; its device
// address is looked up once per device (with that device current).
constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

wq_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return WQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_msd_noalloc_scratch) != cudaSuccess || !p)
      return WQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return WQ_OK;
}

}  // namespace

extern "C" {

wq_status wq_msd_gemm_noalloc(const void* x, int64_t M, int64_t N, int64_t K,
                              int32_t n_components, int32_t group, const void* qweight,
                              const void* scales, const void* zeros, void* y, void* stream) {
  // Same argument rules as wq_msd_gemm, checked first and by wq_msd_gemm
  // itself: with no workspace it validates every argument and returns
  // WQ_ERR_WORKSPACE only when they are all valid (WQ_OK for the empty
  // problems it leaves untouched), so a bad argument gets the status it
  // would get there. Only then is the scratch size compared with the array.
  const wq_status v = wq_msd_gemm(x, M, N, K, n_components, group, qweight, scales, zeros, y,
                                  nullptr, 0, stream);
  if (v != WQ_ERR_WORKSPACE) return v;
  const size_t need = wq::msd_workspace_bytes(M, K, n_components);
  if (need > kScratchBytes) return WQ_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  try {
    wq_status s = scratch_for_current_device(&scratch);
    if (s != WQ_OK) return s;
  } catch (...) {
    return WQ_ERR_CUDA;
  }
  // The digit planes and scales are rewritten by every call before they are
  // read, so nothing in the array has to start at zero.
  return wq_msd_gemm(x, M, N, K, n_components, group, qweight, scales, zeros, y, scratch,
                     kScratchBytes, stream);
}

}  // extern "C"
