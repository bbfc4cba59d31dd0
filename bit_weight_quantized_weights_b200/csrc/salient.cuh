// Selection of the salient channels of a decode step: the k largest
// max_m |x[m, c]| of bf16 x [M, K], ranked by the bit pattern with the sign
// cleared (NaN above +inf), ties to the lower channel, written in increasing
// channel order. Used by the one-CTA selection kernel and, inside the decode
// GEMV, by every CTA for itself.
// Source: "DecDEC: A Systems Approach to Advancing Low-Bit LLM Quantization",
// Abstract (salient channels found from the step's activation outliers).
#pragma once

#include "common.cuh"

namespace wq {
namespace salient {

// Exclusive prefix sum over the CTA's threads (a multiple of 32, at most
// 1024); *total gets the sum. All threads call it.
__device__ __forceinline__ unsigned block_exclusive_scan(unsigned v, unsigned* warp_sums,
                                                         unsigned* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (int)(blockDim.x >> 5);
  unsigned inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const unsigned w = lane < nwarps ? warp_sums[lane] : 0u;
    unsigned wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    if (lane < nwarps) warp_sums[lane] = wi - w;  // exclusive over warps
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const unsigned r = warp_sums[warp] + inc - v;
  __syncthreads();
  return r;
}

// The histogram bin holding the want-th largest key, and how many keys lie
// in higher bins: with nbins <= threads, thread t takes bin nbins - 1 - t, an
// exclusive scan counts the keys above it, and the one thread whose bin holds
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

// Shared-memory scratch of select_block (besides the K keys).
struct Scratch {
  unsigned hist[256];
  unsigned warp_sums[32];
  unsigned bin, above, T, need, total;
};

// The k salient channels (1 <= k <= K) into idx (global or shared memory),
// by all threads of the CTA (blockDim.x >= 256, a multiple of 32): 15-bit
// keys in keys[K], a two-pass radix select of the k-th largest key T (high 8
// bits, then low 7), then an order-preserving compaction that takes every key
// above T and the lowest-index keys equal to T. Ends with a barrier.
__device__ __forceinline__ void select_block(const uint16_t* __restrict__ x, int M, int K, int k,
                                             uint16_t* keys, Scratch& sc, int* idx) {
  const int tid = threadIdx.x, nt = (int)blockDim.x;
  for (int c = tid; c < K; c += nt) {
    unsigned best = 0;
    for (int m = 0; m < M; ++m) best = max(best, (unsigned)(x[(size_t)m * K + c] & 0x7FFFu));
    keys[c] = (uint16_t)best;
  }
  for (int b = tid; b < 256; b += nt) sc.hist[b] = 0;
  __syncthreads();
  for (int c = tid; c < K; c += nt) hist_add(sc.hist, keys[c] >> 7);
  __syncthreads();
  find_bin(sc.hist, 256, (unsigned)k, sc.warp_sums, &sc.total, &sc.bin, &sc.above);
  const unsigned hi = sc.bin, above_hi = sc.above;
  for (int b = tid; b < 256; b += nt) sc.hist[b] = 0;
  __syncthreads();
  for (int c = tid; c < K; c += nt)
    if ((unsigned)(keys[c] >> 7) == hi) hist_add(sc.hist, keys[c] & 0x7Fu);
  __syncthreads();
  find_bin(sc.hist, 128, (unsigned)k - above_hi, sc.warp_sums, &sc.total, &sc.bin, &sc.above);
  if (tid == 0) {
    sc.T = (hi << 7) | sc.bin;
    sc.need = (unsigned)k - above_hi - sc.above;  // keys equal to T to take, >= 1
  }
  __syncthreads();
  const unsigned T = sc.T, need = sc.need;
  // this thread's contiguous range of channels
  const int per = (K + nt - 1) / nt;
  const int c0 = min(K, tid * per), c1 = min(K, c0 + per);
  unsigned n_gt = 0, n_eq = 0;
  for (int c = c0; c < c1; ++c) {
    n_gt += keys[c] > T;
    n_eq += keys[c] == T;
  }
  const unsigned eq_before = block_exclusive_scan(n_eq, sc.warp_sums, &sc.total);
  const unsigned take_eq = eq_before >= need ? 0u : min(n_eq, need - eq_before);
  unsigned pos = block_exclusive_scan(n_gt + take_eq, sc.warp_sums, &sc.total);
  unsigned taken = 0;
  for (int c = c0; c < c1; ++c) {
    const unsigned key = keys[c];
    if (key > T || (key == T && taken < take_eq)) {
      idx[pos++] = c;
      if (key == T) ++taken;
    }
  }
  __syncthreads();
}

}  // namespace salient
}  // namespace wq
