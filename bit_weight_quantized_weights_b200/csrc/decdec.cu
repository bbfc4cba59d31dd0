// Salient-channel residual correction for the decode GEMV: the residual
// matrix and the per-step selection of salient channels. The correction itself
// is added inside the GEMV's epilogue (gemv.cu, splitk_common.cuh).
//
// Source: "DecDEC: A Systems Approach to Advancing Low-Bit LLM Quantization",
// Abstract. The residual is the difference between the full-precision and the
// quantized weights. At every decoding step the salient channels, which the
// activation outliers mark, are found from the step's activations, and only
// their residuals are fetched to correct the quantization error.
//
// Readings, the same in the CPU oracle:
// * R = fp16(W - W_hat): W_hat is (q - z) * s (exact in fp32) for INT4 and
//   fp32(codebook[q] * absmax) for NF4, the subtraction is one fp32 rounding
//   and the result one fp16 rounding. It is stored channel-major, R^T [K, N],
//   so that a channel's residuals are one contiguous row.
// * Salient channels: the k largest max_m |x[m, c]|, compared as the bf16 bit
//   pattern with the sign cleared (NaN ranks above +inf), ties to the lower
//   channel; the k indices are written in increasing order.
// The host-memory placement of the residuals on the page's laptop GPU is not
// reproduced: R^T lives in device memory and only the k selected rows are read.
#include "common.cuh"
#include "salient.cuh"

namespace wq {
namespace {

// One 64 (k) x 64 (n) tile of R^T per 256-thread CTA. Each thread reads 4
// consecutive weights of a row as one float4 (16 threads per 256-byte row
// segment) and stores their residuals transposed into shared memory; the tile
// then leaves as 16-byte rows of 8 consecutive n (8 threads per 128-byte k row).
// K % 64 == 0; rows beyond N are skipped.
template <bool kNF4>
__global__ void __launch_bounds__(256) residual_kernel(
    const float* __restrict__ W, int N, int K, int G, const uint32_t* __restrict__ qw,
    const uint8_t* __restrict__ codes, const __half* __restrict__ scales,
    const __half* __restrict__ zeros, const float* __restrict__ absmax, Nf4Table tab,
    __half* __restrict__ rt) {
  constexpr int kPitch = 64 + 8;  // halves per k row of the tile (16-byte rows stay aligned)
  __shared__ __align__(16) __half tile[64 * kPitch];
  const int k0 = blockIdx.x * 64, n0 = blockIdx.y * 64;
  const int tid = threadIdx.x;
  const int kq = (tid & 15) * 4;  // this thread's 4 consecutive k of the segment
  for (int r = tid >> 4; r < 64; r += 16) {
    const int n = n0 + r;
    float4 w4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    float wh[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (n < N) {
      const int64_t e = (int64_t)n * K + k0 + kq;  // multiple of 4
      w4 = __ldg(reinterpret_cast<const float4*>(W + e));
      if (kNF4) {
        const uint16_t b2 = __ldg(reinterpret_cast<const uint16_t*>(codes + (e >> 1)));
        const float am = __ldg(absmax + (e >> 6));
        // bytes j, j + 1 = elements (e, e+1), (e+2, e+3); element 2j: high nibble
        const int q[4] = {(b2 >> 4) & 0xF, b2 & 0xF, (b2 >> 12) & 0xF, (b2 >> 8) & 0xF};
#pragma unroll
        for (int i = 0; i < 4; ++i) wh[i] = __fmul_rn(tab.v[q[i]], am);  // one fp32 rounding
      } else {
        const uint32_t word = __ldg(qw + (e >> 3));
        const int sh = (int)(e & 7) * 4;  // 0 or 16: the word's low or high four codes
        const int64_t gi = (int64_t)n * (K / G) + (k0 + kq) / G;
        const float sc = __half2float(scales[gi]), z = __half2float(zeros[gi]);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          wh[i] = __fmul_rn((float)((word >> (sh + 4 * i)) & 0xFu) - z, sc);  // exact
      }
    }
    const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      tile[(kq + i) * kPitch + r] = __float2half_rn(__fsub_rn(wv[i], wh[i]));
  }
  __syncthreads();
  const int nc = (tid & 7) * 8;  // 8 consecutive n
  for (int kr = tid >> 3; kr < 64; kr += 32) {
    const int n = n0 + nc;
    if (n + 8 <= N) {
      *reinterpret_cast<uint4*>(rt + (int64_t)(k0 + kr) * N + n) =
          *reinterpret_cast<const uint4*>(tile + kr * kPitch + nc);
    } else {
      for (int i = 0; i < 8 && n + i < N; ++i)
        rt[(int64_t)(k0 + kr) * N + n + i] = tile[kr * kPitch + nc + i];
    }
  }
}

constexpr int kSelThreads = 1024;

// One CTA selects for the whole step.
__global__ void __launch_bounds__(kSelThreads) select_kernel(const uint16_t* __restrict__ x, int M,
                                                             int K, int k, int* __restrict__ idx) {
  extern __shared__ uint16_t keys[];
  __shared__ salient::Scratch sc;
  // a GEMV launched after this one with programmatic stream serialization
  // may start now; it waits (griddepcontrol.wait) before it reads idx
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  salient::select_block(x, M, K, k, keys, sc, idx);
}

}  // namespace

wq_status launch_residual(wq_format fmt, const float* W, int64_t N, int64_t K, int32_t G,
                          const void* qweight, const void* scales, const void* zeros, void* rt,
                          cudaStream_t st) {
  const dim3 grid((unsigned)(K / 64), (unsigned)((N + 63) / 64));
  if (fmt == WQ_FMT_NF4)
    residual_kernel<true><<<grid, 256, 0, st>>>(
        W, (int)N, (int)K, G, nullptr, static_cast<const uint8_t*>(qweight), nullptr, nullptr,
        static_cast<const float*>(scales), nf4_table(), static_cast<__half*>(rt));
  else
    residual_kernel<false><<<grid, 256, 0, st>>>(
        W, (int)N, (int)K, G, static_cast<const uint32_t*>(qweight), nullptr,
        static_cast<const __half*>(scales), static_cast<const __half*>(zeros), nullptr,
        nf4_table(), static_cast<__half*>(rt));
  return launch_status();
}

wq_status launch_select_salient(const void* x, int64_t M, int64_t K, int32_t k, int32_t* idx,
                                cudaStream_t st) {
  const size_t smem = (size_t)K * 2;
  if (cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return WQ_ERR_CUDA;
  select_kernel<<<1, kSelThreads, smem, st>>>(static_cast<const uint16_t*>(x), (int)M, (int)K, k,
                                              idx);
  return launch_status();
}

}  // namespace wq
