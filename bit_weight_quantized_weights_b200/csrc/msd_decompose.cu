// Multi-Scale Dequant activation decomposition.
//
// Source: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
// Activation Decomposition for Efficient LLM Inference", Abstract: the bf16
// activations are split into several low-precision components that multiply
// the quantized weights directly; two INT8 passes give close to 16 effective
// bits. Reading (per activation row): s_1 = amax / 127, s_{c+1} = s_c / 256;
// digit c is the round-half-even quotient of the running residual by s_c; the
// residual update rounds once (fused multiply-add); a +128 digit is written as
// -128 with a carry into the previous digit.
//
// One CTA per activation row: a max-reduction pass, then one pass that emits
// all C digit planes (16 elements per thread step, 16-byte stores per plane).
// The planes are written in k order, or (for the tensor-core MSD GEMM) with
// each run of 8 k permuted to the order of its INT4 weight nibbles after a
// mask and a shift: k = 0, 2, 4, 6, 1, 3, 5, 7. The digits are the same; an
// integer dot product over the permuted k is the same sum.
#include "common.cuh"

namespace wq {
namespace {

// byte position of element e (0..15) of a thread's 16-element step
template <bool kNibbleOrder>
__device__ __forceinline__ constexpr int digit_pos(int e) {
  return kNibbleOrder ? (e & 8) | ((e & 1) << 2) | ((e >> 1) & 3) : e;
}

template <bool kNibbleOrder>
__global__ void __launch_bounds__(256) msd_decompose_kernel(const uint16_t* __restrict__ x, int M,
                                                            int K, int C, int64_t plane_rows,
                                                            int8_t* __restrict__ digits,
                                                            float* __restrict__ comp_scales) {
  __shared__ float red[8];
  // a grid launched after this one as a programmatic dependent (the decode
  // GEMV) may start at once: it waits for this grid before it reads the
  // planes and scales
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int m = blockIdx.x;
  const uint16_t* row = x + (int64_t)m * K;
  const int chunks = K / 16;

  float amax = 0.0f;
  for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
    const uint4 a = *reinterpret_cast<const uint4*>(row + c * 16);
    const uint4 b = *reinterpret_cast<const uint4*>(row + c * 16 + 8);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      amax = fmaxf(amax, fabsf(bf16_lo_to_f32(w[i])));
      amax = fmaxf(amax, fabsf(bf16_hi_to_f32(w[i])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);

  float sc[3];
  sc[0] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 1.0f;
  sc[1] = __fdiv_rn(sc[0], 256.0f);
  sc[2] = __fdiv_rn(sc[1], 256.0f);
  if (threadIdx.x < C) comp_scales[(int64_t)threadIdx.x * M + m] = sc[threadIdx.x];

  for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
    const uint4 a = *reinterpret_cast<const uint4*>(row + c * 16);
    const uint4 b = *reinterpret_cast<const uint4*>(row + c * 16 + 8);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[3][4];
#pragma unroll
    for (int p = 0; p < 3; ++p)
#pragma unroll
      for (int q = 0; q < 4; ++q) out[p][q] = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float xv = (e & 1) ? bf16_hi_to_f32(w[e >> 1]) : bf16_lo_to_f32(w[e >> 1]);
      int d[3] = {0, 0, 0};
      float r = xv;
      d[0] = (int)fminf(fmaxf(rintf(__fdiv_rn(r, sc[0])), -127.0f), 127.0f);
      r = __fmaf_rn(-sc[0], (float)d[0], r);
      if (C > 1) {
        d[1] = (int)rintf(__fdiv_rn(r, sc[1]));
        r = __fmaf_rn(-sc[1], (float)d[1], r);
      }
      if (C > 2) {
        d[2] = (int)rintf(__fdiv_rn(r, sc[2]));
      }
      if (C > 2 && d[2] == 128) { d[2] = -128; d[1] += 1; }
      if (C > 1 && d[1] == 128) { d[1] = -128; d[0] += 1; }
#pragma unroll
      for (int p = 0; p < 3; ++p)
        out[p][digit_pos<kNibbleOrder>(e) >> 2] |= ((uint32_t)(d[p] & 0xFF))
                                                   << (8 * (digit_pos<kNibbleOrder>(e) & 3));
    }
    for (int p = 0; p < C; ++p) {
      int8_t* dst = digits + ((int64_t)p * plane_rows + m) * K + c * 16;
      *reinterpret_cast<uint4*>(dst) = make_uint4(out[p][0], out[p][1], out[p][2], out[p][3]);
    }
  }
}

}  // namespace

wq_status launch_msd_decompose(const void* x, int64_t M, int64_t K, int32_t C, int64_t plane_rows,
                               int8_t* digits, float* comp_scales, cudaStream_t st) {
  msd_decompose_kernel<false><<<(unsigned)M, 256, 0, st>>>(
      static_cast<const uint16_t*>(x), (int)M, (int)K, C, plane_rows, digits, comp_scales);
  return launch_status();
}

wq_status launch_msd_decompose_nibble_order(const void* x, int64_t M, int64_t K, int32_t C,
                                            int64_t plane_rows, int8_t* digits,
                                            float* comp_scales, cudaStream_t st) {
  msd_decompose_kernel<true><<<(unsigned)M, 256, 0, st>>>(
      static_cast<const uint16_t*>(x), (int)M, (int)K, C, plane_rows, digits, comp_scales);
  return launch_status();
}

}  // namespace wq
