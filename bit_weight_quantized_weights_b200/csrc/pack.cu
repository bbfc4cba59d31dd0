// Quantize + pack (INT4 asymmetric per group, NF4 per block of 64) and unpack.
//
// INT4: "MixPE: Quantization and Hardware Co-design for Efficient LLM
// Inference", Abstract -- one scale and one zero point per quantization group.
// NF4: "Fast NF4 Dequantization Kernels for Large Language Model Inference",
// Abstract -- 4-bit NormalFloat codes with a per-block absmax.
//
// Offline steps, written for exact agreement with the oracle rather than for
// speed: IEEE divisions (__fdiv_rn), round-half-even (rintf), fp16 by RNE.
#include <math.h>

#include "common.cuh"

namespace wq {
namespace {

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// One warp per (row, group). G % 8 == 0; rows are K floats apart.
__global__ void __launch_bounds__(256) int4_quantize_kernel(const float* __restrict__ W,
                                                            int64_t n_rows, int64_t K, int G,
                                                            uint32_t* __restrict__ qweight,
                                                            __half* __restrict__ scales,
                                                            __half* __restrict__ zeros) {
  const int lane = threadIdx.x & 31;
  const int64_t ng = K / G;
  const int64_t item = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (item >= n_rows * ng) return;
  const int64_t n = item / ng, g = item % ng;
  const float* wr = W + n * K + g * G;

  float mn = INFINITY, mx = -INFINITY;
  for (int i = lane; i < G; i += 32) {
    float v = wr[i];
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  mn = warp_min(mn);
  mx = warp_max(mx);
  float lo = fminf(mn, 0.0f), hi = fmaxf(mx, 0.0f);
  __half sh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
  float s = __half2float(sh);
  if (s == 0.0f) {  // all-zero (or vanishing) group: range [-1, 1]
    lo = -1.0f;
    hi = 1.0f;
    sh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
    s = __half2float(sh);
  }
  const int z = (int)fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.0f), 15.0f);

  uint32_t* qrow = qweight + n * (K / 8) + g * (G / 8);
  for (int wi = lane; wi < G / 8; wi += 32) {
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float qf = rintf(__fdiv_rn(wr[wi * 8 + i], s)) + (float)z;
      int q = (int)fminf(fmaxf(qf, 0.0f), 15.0f);
      word |= (uint32_t)q << (4 * i);
    }
    qrow[wi] = word;
  }
  if (lane == 0) {
    scales[n * ng + g] = sh;
    zeros[n * ng + g] = __int2half_rn(z);
  }
}

// One warp per block of 64 elements; lane l owns elements 2l and 2l+1 and
// writes byte l (element 2l in the high nibble).
__global__ void __launch_bounds__(256) nf4_quantize_kernel(const float* __restrict__ W,
                                                           int64_t n_blocks, Nf4Table tab,
                                                           uint8_t* __restrict__ codes,
                                                           float* __restrict__ absmax) {
  const int lane = threadIdx.x & 31;
  const int64_t b = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (b >= n_blocks) return;
  // decision points between neighbouring code values, exact in double
  double mid[15];
#pragma unroll
  for (int j = 0; j < 15; ++j) mid[j] = 0.5 * ((double)tab.v[j] + (double)tab.v[j + 1]);

  const float2 v = reinterpret_cast<const float2*>(W + b * 64)[lane];
  const float am = warp_max(fmaxf(fabsf(v.x), fabsf(v.y)));
  int c0 = 7, c1 = 7;
  if (am != 0.0f) {
    const double u0 = (double)__fdiv_rn(v.x, am);
    const double u1 = (double)__fdiv_rn(v.y, am);
    c0 = 0;
    c1 = 0;
#pragma unroll
    for (int j = 0; j < 15; ++j) {
      c0 += (u0 > mid[j]) ? 1 : 0;  // ties (u == midpoint) keep the lower code
      c1 += (u1 > mid[j]) ? 1 : 0;
    }
  }
  codes[b * 32 + lane] = (uint8_t)((c0 << 4) | c1);
  if (lane == 0) absmax[b] = am;
}

__global__ void int4_unpack_kernel(const uint32_t* __restrict__ qweight, int64_t n_words,
                                   uint8_t* __restrict__ out) {
  const int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= n_words) return;
  const uint32_t v = qweight[w];
  uint2 r;
  r.x = (v & 0xFu) | ((v >> 4 & 0xFu) << 8) | ((v >> 8 & 0xFu) << 16) | ((v >> 12 & 0xFu) << 24);
  r.y = (v >> 16 & 0xFu) | ((v >> 20 & 0xFu) << 8) | ((v >> 24 & 0xFu) << 16) |
        ((v >> 28 & 0xFu) << 24);
  reinterpret_cast<uint2*>(out)[w] = r;
}

__global__ void nf4_unpack_kernel(const uint8_t* __restrict__ packed, int64_t n_bytes,
                                  uint8_t* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_bytes) return;
  const uint32_t v = packed[i];
  out[2 * i] = (uint8_t)(v >> 4);
  out[2 * i + 1] = (uint8_t)(v & 0xFu);
}

}  // namespace

wq_status launch_quantize_pack(wq_format fmt, const float* W, int64_t N, int64_t K, int32_t group,
                               void* qweight, void* scales, void* zeros, cudaStream_t st) {
  if (fmt == WQ_FMT_INT4_ASYM) {
    const int64_t items = N * (K / group);
    const int64_t blocks = (items + 7) / 8;
    int4_quantize_kernel<<<(unsigned)blocks, 256, 0, st>>>(
        W, N, K, group, static_cast<uint32_t*>(qweight), static_cast<__half*>(scales),
        static_cast<__half*>(zeros));
  } else {
    const int64_t nb = N * K / 64;
    const int64_t blocks = (nb + 7) / 8;
    nf4_quantize_kernel<<<(unsigned)blocks, 256, 0, st>>>(W, nb, nf4_table(),
                                                          static_cast<uint8_t*>(qweight),
                                                          static_cast<float*>(scales));
  }
  return launch_status();
}

wq_status launch_unpack(wq_format fmt, const void* qweight, int64_t N, int64_t K, uint8_t* codes,
                        cudaStream_t st) {
  if (fmt == WQ_FMT_INT4_ASYM) {
    const int64_t nw = N * K / 8;
    int4_unpack_kernel<<<(unsigned)((nw + 255) / 256), 256, 0, st>>>(
        static_cast<const uint32_t*>(qweight), nw, codes);
  } else {
    const int64_t nb = N * K / 2;
    nf4_unpack_kernel<<<(unsigned)((nb + 255) / 256), 256, 0, st>>>(
        static_cast<const uint8_t*>(qweight), nb, codes);
  }
  return launch_status();
}

}  // namespace wq
