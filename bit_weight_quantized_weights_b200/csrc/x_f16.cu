// Activations bf16 -> fp16 with a per-row power-of-two scale.
//
// The fused GEMM multiplies in fp16 (11 significant bits, so the dequantized
// weight (q - z) * s rounds 16x more finely than in bf16). bf16 activations
// have 8 significant bits, so x * 2^e is exact in fp16 as long as it lies in
// fp16's normal range. Per row, e puts the row's largest magnitude in
// [2^14, 2^15): every element down to amax * 2^-28 converts exactly, none can
// overflow, and the GEMM epilogue multiplies by 2^-e (exact) before rounding
// to bf16.
//
// For INT4 weights the copy stores every 8-element chunk in the order
// x0 x4 x1 x5 x2 x6 x3 x7: the order in which the GEMM's dequantization
// produces the weights of one packed INT4 word (nibbles e and e + 4 share a
// 32-bit register). A product over k is the same under any permutation of k
// applied to both operands. For NF4 weights (codes already in k order) the
// copy keeps the natural order.
#include "common.cuh"

namespace wq {
namespace {

// One warp per row. Rows of up to 32 x kRegChunks 8-element chunks (K <= 4096)
// stay in registers between the amax and the conversion, so every load of
// the row is issued at once and the row is read once; longer rows read it
// twice (the second read mostly hits L1).
constexpr int kRegChunks = 16;
constexpr int kRowsPerBlock = 8;

__device__ __forceinline__ float chunk_amax(const uint4& a) {
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    m = fmaxf(m, fmaxf(fabsf(bf16_lo_to_f32(w[i])), fabsf(bf16_hi_to_f32(w[i]))));
  return m;
}

template <bool kPermute>
__device__ __forceinline__ uint4 chunk_to_f16(const uint4& a, float sc) {
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
  uint32_t o[4];
  if (kPermute) {  // x0 x4 x1 x5 x2 x6 x3 x7 (see the header)
    o[0] = pack_f16x2(bf16_lo_to_f32(w[0]) * sc, bf16_lo_to_f32(w[2]) * sc);
    o[1] = pack_f16x2(bf16_hi_to_f32(w[0]) * sc, bf16_hi_to_f32(w[2]) * sc);
    o[2] = pack_f16x2(bf16_lo_to_f32(w[1]) * sc, bf16_lo_to_f32(w[3]) * sc);
    o[3] = pack_f16x2(bf16_hi_to_f32(w[1]) * sc, bf16_hi_to_f32(w[3]) * sc);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o[i] = pack_f16x2(bf16_lo_to_f32(w[i]) * sc, bf16_hi_to_f32(w[i]) * sc);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <bool kPermute, bool kInRegisters>
__global__ void __launch_bounds__(32 * kRowsPerBlock) x_to_f16_kernel(
    const uint16_t* __restrict__ x, int64_t M, int K, uint16_t* __restrict__ x16,
    float* __restrict__ inv_scale) {
  const int lane = threadIdx.x & 31;
  const int64_t m = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  if (m >= M) return;
  const uint4* row = reinterpret_cast<const uint4*>(x + m * K);
  uint4* out = reinterpret_cast<uint4*>(x16 + m * K);
  const int chunks = K / 8;
  uint4 v[kInRegisters ? kRegChunks : 1];
  float amax = 0.0f;
  if (kInRegisters) {
#pragma unroll
    for (int j = 0; j < kRegChunks; ++j) {
      const int c = lane + 32 * j;
      v[j] = c < chunks ? row[c] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < kRegChunks; ++j) amax = fmaxf(amax, chunk_amax(v[j]));
  } else {
    for (int c = lane; c < chunks; c += 32) amax = fmaxf(amax, chunk_amax(row[c]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  // exponent of amax (amax finite and > 0): amax in [2^ex, 2^(ex+1))
  int e = 0;
  if (amax > 0.0f && amax <= 3.0e38f) {
    const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
    e = 14 - ex;
    e = e > 100 ? 100 : (e < -100 ? -100 : e);
  }
  const float sc = __uint_as_float((uint32_t)(127 + e) << 23);       // 2^e
  if (lane == 0) inv_scale[m] = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e
  if (kInRegisters) {
#pragma unroll
    for (int j = 0; j < kRegChunks; ++j) {
      const int c = lane + 32 * j;
      if (c < chunks) out[c] = chunk_to_f16<kPermute>(v[j], sc);
    }
  } else {
    for (int c = lane; c < chunks; c += 32) out[c] = chunk_to_f16<kPermute>(row[c], sc);
  }
}

}  // namespace

wq_status launch_x_to_f16(const void* x, int64_t M, int64_t K, void* x16, float* inv_scale,
                          bool permute, cudaStream_t st) {
  if (M == 0) return WQ_OK;
  const bool regs = K <= 32 * kRegChunks * 8;
  auto kern = permute ? (regs ? x_to_f16_kernel<true, true> : x_to_f16_kernel<true, false>)
                      : (regs ? x_to_f16_kernel<false, true> : x_to_f16_kernel<false, false>);
  const unsigned blocks = (unsigned)((M + kRowsPerBlock - 1) / kRowsPerBlock);
  kern<<<blocks, 32 * kRowsPerBlock, 0, st>>>(static_cast<const uint16_t*>(x), M, (int)K,
                                              static_cast<uint16_t*>(x16), inv_scale);
  return launch_status();
}

}  // namespace wq
