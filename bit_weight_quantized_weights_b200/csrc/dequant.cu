// Standalone dequantization kernels (HBM-bound streaming).
//
// NF4 -> bf16/fp16: "Fast NF4 Dequantization Kernels for Large Language Model
// Inference", Abstract (lifting NF4 back to 16-bit before the product is the
// bottleneck that page speeds up on A100 with a 64-byte shared-memory codebook).
// INT4 -> bf16/fp16: the weight lifting that "Multi-Scale Dequant: Eliminating
// Dequantization Bottleneck via Activation Decomposition for Efficient LLM
// Inference", Abstract, removes from the GEMM path; here it feeds the
// dequantize-then-GEMM baseline.
//
// B200 design: a grid-stride stream over 16-byte chunks of packed codes; each
// thread turns one chunk into 64 (NF4) or 32 (INT4) output elements and writes
// them with 16-byte evict-first stores. The 16-entry codebook sits in shared
// memory (all lanes reading one of 16 words never conflict: equal words
// broadcast, distinct words sit in distinct banks).
#include "common.cuh"

namespace wq {
namespace {

template <bool kBf16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  return kBf16 ? pack_bf16x2(lo, hi) : pack_f16x2(lo, hi);
}

// Each thread: 16 code bytes (32 elements, half of one 64-element block).
template <bool kBf16>
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint8_t* __restrict__ codes,
                                                          const float* __restrict__ absmax,
                                                          int64_t n_chunks, Nf4Table tab,
                                                          uint16_t* __restrict__ out) {
  __shared__ float cb[16];
  if (threadIdx.x < 16) cb[threadIdx.x] = tab.v[threadIdx.x];
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < n_chunks; c += stride) {
    const uint4 v = ld_stream_u4(codes + c * 16);
    const float a = __ldg(absmax + (c >> 1));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t byte = (w[i] >> (8 * j)) & 0xFFu;
        // element 2j of the byte pair is the high nibble
        const float e0 = __fmul_rn(cb[byte >> 4], a);
        const float e1 = __fmul_rn(cb[byte & 0xFu], a);
        o[i * 4 + j] = pack2<kBf16>(e0, e1);
      }
    }
    uint16_t* dst = out + c * 32;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      st_stream_u4(dst + i * 8, make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]));
  }
}

// Each thread: one packed word (8 elements of one row, one group).
template <bool kBf16>
__global__ void __launch_bounds__(256) int4_dequant_kernel(const uint32_t* __restrict__ qweight,
                                                           const __half* __restrict__ scales,
                                                           const __half* __restrict__ zeros,
                                                           int64_t n_words, int64_t words_per_row,
                                                           int words_per_group,
                                                           uint16_t* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t groups_per_row = words_per_row / words_per_group;
  for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < n_words; w += stride) {
    const uint32_t v = __ldg(qweight + w);
    const int64_t n = w / words_per_row;
    const int64_t g = (w - n * words_per_row) / words_per_group;
    const float s = __half2float(scales[n * groups_per_row + g]);
    const float z = __half2float(zeros[n * groups_per_row + g]);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // (q - z) is exact in fp32, and so is its product with the fp16 scale
      const float e0 = __fmul_rn(__fsub_rn((float)((v >> (8 * i)) & 0xFu), z), s);
      const float e1 = __fmul_rn(__fsub_rn((float)((v >> (8 * i + 4)) & 0xFu), z), s);
      o[i] = pack2<kBf16>(e0, e1);
    }
    st_stream_u4(out + w * 8, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

inline unsigned stream_grid(int64_t items) {
  const int64_t cap = (int64_t)num_sms() * 8;  // 8 CTAs of 256 threads fill an SM
  const int64_t need = (items + 255) / 256;
  return (unsigned)(need < cap ? (need > 0 ? need : 1) : cap);
}

}  // namespace

wq_status launch_nf4_dequant(const uint8_t* codes, const float* absmax, int64_t numel, void* out,
                             wq_dtype dt, cudaStream_t st) {
  const int64_t chunks = numel / 32;
  const unsigned grid = stream_grid(chunks);
  if (dt == WQ_BF16)
    nf4_dequant_kernel<true><<<grid, 256, 0, st>>>(codes, absmax, chunks, nf4_table(),
                                                   static_cast<uint16_t*>(out));
  else
    nf4_dequant_kernel<false><<<grid, 256, 0, st>>>(codes, absmax, chunks, nf4_table(),
                                                    static_cast<uint16_t*>(out));
  return launch_status();
}

wq_status launch_int4_dequant(const uint32_t* qweight, const void* scales, const void* zeros,
                              int64_t N, int64_t K, int32_t group, void* out, wq_dtype dt,
                              cudaStream_t st) {
  const int64_t n_words = N * K / 8;
  const unsigned grid = stream_grid(n_words);
  const __half* s = static_cast<const __half*>(scales);
  const __half* z = static_cast<const __half*>(zeros);
  if (dt == WQ_BF16)
    int4_dequant_kernel<true><<<grid, 256, 0, st>>>(qweight, s, z, n_words, K / 8, group / 8,
                                                    static_cast<uint16_t*>(out));
  else
    int4_dequant_kernel<false><<<grid, 256, 0, st>>>(qweight, s, z, n_words, K / 8, group / 8,
                                                     static_cast<uint16_t*>(out));
  return launch_status();
}

}  // namespace wq
