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
    for (int i = 0; i < 4; ++i) tile[(kq + i) * kPitch + r] = __float2half_rn(__fsub_rn(wv[i], wh[i]));
  }
  __syncthreads();
  const int nc = (tid & 7) * 8;  // 8 consecutive n
  for (int kr = tid >> 3; kr < 64; kr += 32) {
    const int n = n0 + nc;
    if (n + 8 <= N) {
      *reinterpret_cast<uint4*>(rt + (int64_t)(k0 + kr) * N + n) =
          *reinterpret_cast<const uint4*>(tile + kr * kPitch + nc);
    } else {
      for (int i = 0; i < 8 && n + i < N; ++i) rt[(int64_t)(k0 + kr) * N + n + i] = tile[kr * kPitch + nc + i];
    }
  }
}

constexpr int kSelThreads = 1024;

// Exclusive prefix sum over the CTA's threads; *total gets the sum.
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned v, unsigned* warp_sums,
                                                         unsigned* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    unsigned w = warp_sums[lane];
    unsigned wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    warp_sums[lane] = wi - w;  // exclusive over warps
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const unsigned r = warp_sums[warp] + inc - v;
  __syncthreads();
  return r;
}

// The histogram bin holding the want-th largest key, and how many keys lie in
// higher bins: thread t takes bin nbins - 1 - t, an exclusive scan over the
// threads counts the keys above it, and the one thread whose bin contains
// the want-th key writes the answer. All threads call it.
__device__ __forceinline__ void find_bin(const unsigned* hist, int nbins, unsigned want,
                                         unsigned* warp_sums, unsigned* total, unsigned* bin,
                                         unsigned* above) {
  const int t = threadIdx.x;
  const unsigned h = t < nbins ? hist[nbins - 1 - t] : 0u;
  const unsigned before = block_exclusive_scan(h, warp_sums, total);
  if (t < nbins && h > 0 && before < want && want <= before + h) {
    *bin = (unsigned)(nbins - 1 - t);
    *above = before;
  }
  __syncthreads();
}

// hist[bin] += 1 for every calling lane, one shared-memory atomic per
// distinct bin among the warp's active lanes.
__device__ __forceinline__ void hist_add(unsigned* hist, unsigned bin) {
  const unsigned peers = __match_any_sync(__activemask(), bin);
  if ((__ffs(peers) - 1) == (int)(threadIdx.x & 31)) atomicAdd(&hist[bin], __popc(peers));
}

// The k salient channels of x [M, K] (1 <= k <= K), one CTA: 15-bit keys in
// shared memory, a two-pass radix select of the k-th largest key T (high 8
// bits, then low 7), then an order-preserving compaction that takes every key
// above T and the lowest-index keys equal to T.
__global__ void __launch_bounds__(kSelThreads) select_kernel(const uint16_t* __restrict__ x, int M,
                                                             int K, int k, int* __restrict__ idx) {
  extern __shared__ uint16_t keys[];
  __shared__ unsigned hist[256];
  __shared__ unsigned warp_sums[32];
  __shared__ unsigned s_bin, s_above, s_T, s_need, s_total;
  const int tid = threadIdx.x;
  for (int c = tid; c < K; c += kSelThreads) {
    unsigned best = 0;
    for (int m = 0; m < M; ++m) best = max(best, (unsigned)(x[(size_t)m * K + c] & 0x7FFFu));
    keys[c] = (uint16_t)best;
  }
  if (tid < 256) hist[tid] = 0;
  __syncthreads();
  for (int c = tid; c < K; c += kSelThreads) hist_add(hist, keys[c] >> 7);
  __syncthreads();
  find_bin(hist, 256, (unsigned)k, warp_sums, &s_total, &s_bin, &s_above);
  const unsigned hi = s_bin, above_hi = s_above;
  if (tid < 256) hist[tid] = 0;
  __syncthreads();
  for (int c = tid; c < K; c += kSelThreads)
    if ((unsigned)(keys[c] >> 7) == hi) hist_add(hist, keys[c] & 0x7Fu);
  __syncthreads();
  find_bin(hist, 128, (unsigned)k - above_hi, warp_sums, &s_total, &s_bin, &s_above);
  if (tid == 0) {
    s_T = (hi << 7) | s_bin;
    s_need = (unsigned)k - above_hi - s_above;  // keys equal to T to take, >= 1
  }
  __syncthreads();
  const unsigned T = s_T, need = s_need;
  // this thread's contiguous range of channels
  const int per = (K + kSelThreads - 1) / kSelThreads;
  const int c0 = min(K, tid * per), c1 = min(K, c0 + per);
  unsigned n_gt = 0, n_eq = 0;
  for (int c = c0; c < c1; ++c) {
    n_gt += keys[c] > T;
    n_eq += keys[c] == T;
  }
  const unsigned eq_before = block_exclusive_scan(n_eq, warp_sums, &s_total);
  const unsigned take_eq = eq_before >= need ? 0u : min(n_eq, need - eq_before);
  unsigned pos = block_exclusive_scan(n_gt + take_eq, warp_sums, &s_total);
  unsigned taken = 0;
  for (int c = c0; c < c1; ++c) {
    const unsigned key = keys[c];
    if (key > T || (key == T && taken < take_eq)) {
      idx[pos++] = c;
      if (key == T) ++taken;
    }
  }
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
