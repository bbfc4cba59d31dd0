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
// B200 design: a grid-stride stream sized to fill every SM; loads and 16-byte
// evict-first stores are laid out so each warp instruction covers contiguous
// full sectors. The 16-entry codebook sits in shared memory (all lanes reading
// one of 16 words never conflict: equal words broadcast, distinct words sit in
// distinct banks).
#include "common.cuh"

namespace wq {
namespace {

template <bool kBf16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  return kBf16 ? pack_bf16x2(lo, hi) : pack_f16x2(lo, hi);
}

// One warp step covers 1024 elements (512 code bytes). Lane l takes 4 code
// bytes (8 elements) from each of four 128-byte slices, so every load
// instruction of the warp reads 128 contiguous bytes and every 16-byte store
// instruction writes 512 contiguous bytes (full sectors). Two warp steps are
// issued per loop trip to keep eight independent loads in flight per thread.
template <bool kBf16>
__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint8_t* __restrict__ codes,
                                                          const float* __restrict__ absmax,
                                                          int64_t numel, Nf4Table tab,
                                                          uint16_t* __restrict__ out) {
  __shared__ float cb[16];
  if (threadIdx.x < 16) cb[threadIdx.x] = tab.v[threadIdx.x];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t steps = numel / 1024;   // full warp steps
  constexpr int U = 2;                  // warp steps per loop trip
  for (int64_t s0 = warp * U; s0 < steps; s0 += nwarps * U) {
    uint32_t w[U][4];
    float a[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t st = s0 + u;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (st < steps) {
          const int64_t e0 = st * 1024 + 256 * j + 8 * lane;  // first element of this lane
          w[u][j] = __ldcs(reinterpret_cast<const unsigned int*>(codes + (e0 >> 1)));
          a[u][j] = __ldg(absmax + (e0 >> 6));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t st = s0 + u;
      if (st < steps) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t o[4];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t byte = (w[u][j] >> (8 * b)) & 0xFFu;
            // element 2b of the pair is the high nibble
            o[b] = pack2<kBf16>(__fmul_rn(cb[byte >> 4], a[u][j]),
                                __fmul_rn(cb[byte & 0xFu], a[u][j]));
          }
          st_stream_u4(out + st * 1024 + 256 * j + 8 * lane, make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
    }
  }
  // tail: elements past the last full 1024 (a multiple of 64), one lane per 8
  const int64_t tail0 = steps * 1024;
  for (int64_t e0 = tail0 + 8 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); e0 < numel;
       e0 += 8 * (int64_t)gridDim.x * blockDim.x) {
    const uint32_t wv = *reinterpret_cast<const uint32_t*>(codes + (e0 >> 1));
    const float av = absmax[e0 >> 6];
    uint32_t o[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t byte = (wv >> (8 * b)) & 0xFFu;
      o[b] = pack2<kBf16>(__fmul_rn(cb[byte >> 4], av), __fmul_rn(cb[byte & 0xFu], av));
    }
    *reinterpret_cast<uint4*>(out + e0) = make_uint4(o[0], o[1], o[2], o[3]);
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
  const unsigned grid = stream_grid(numel / 32);
  if (dt == WQ_BF16)
    nf4_dequant_kernel<true><<<grid, 256, 0, st>>>(codes, absmax, numel, nf4_table(),
                                                   static_cast<uint16_t*>(out));
  else
    nf4_dequant_kernel<false><<<grid, 256, 0, st>>>(codes, absmax, numel, nf4_table(),
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
