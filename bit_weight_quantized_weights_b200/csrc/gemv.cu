// Decode W4A16 GEMV (1 <= M <= 16): y = x . dequant(W_q)^T.
//
// Sources: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
// Activation Decomposition for Efficient LLM Inference", Abstract (the
// low-bit-weight product and its dequantization cost); "MixPE: Quantization
// and Hardware Co-design for Efficient LLM Inference", Abstract (scale and
// zero are shared per group, so they are applied after the group's sum);
// "Fast NF4 Dequantization Kernels for Large Language Model Inference",
// Abstract (NF4 codes with a per-block absmax; a small shared-memory codebook).
//
// B200 design
// -----------
// * The weight stream is the whole cost (0.53 byte per weight against 2*M
//   flops). Weights are read with plain 8-byte loads that do not allocate in
//   L1, by many small CTAs (up to three per SM), each warp keeping the next
//   128-k unit of its 16 rows (and that unit's group parameters) in flight
//   while it computes the current one. Measured on B200, plain coalesced loads
//   stream HBM far better than a TMA ring of small boxes for this work.
// * At M = 16 the multiply-adds alone (2*16 flops per weight at ~12 Tweights/s)
//   exceed what the CUDA cores can issue, so the product runs on the tensor
//   cores with warp-level mma.m16n8k16 (fp32 accumulate): weight rows form
//   the 16-row A operand, tokens the 8-column B operand. The tensor pipe stays
//   far from busy; HBM is the bound.
// * INT4 codes become bf16 in registers without arithmetic: OR-ing a nibble
//   into the mantissa of 128.0 (bit pattern 0x4300) gives exactly 128 + q, two
//   per 32-bit LOP3. The MMA sums (128 + q) x over a 64-wide sub-group, a
//   second MMA with an all-ones A operand sums x itself, and the epilogue
//   applies s * (P - (128 + z) * sum(x)), the MixPE post-group form.
// * NF4 codes go through a 256-entry table indexed by a whole packed byte that
//   yields the two fp16 code values already paired as one A-operand register.
//   The table is replicated per lane (lane l reads column l, so bank l): every
//   lookup is conflict-free. The block's absmax is applied after the block's
//   sum. The NF4 product runs in fp16 (the code values keep 11 significant
//   bits): the staged x chunk is converted to fp16 scaled per token by a power
//   of two that puts its largest magnitude in [2^14, 2^15) (exact for bf16
//   values down to 2^-28 of it); the power is divided back out of the partial.
// * Split-K across a thread-block cluster: the S CTAs of a cluster share one
//   128-row tile and split K; their fp32 partials are summed through
//   distributed shared memory, in a fixed rank order, and written once as
//   bf16. No workspace, no atomics.
//
// Data placement per CTA (dynamic shared memory):
//   xs   [8*NT tokens][Kc] bf16 (fp16 for NF4), the CTA's K-chunk of x
//        (zero-padded tokens); odd tokens have bit 3 of k flipped (a 16-byte
//        swizzle that keeps the fragment loads conflict-free)
//   lut  [256 entries][32 lanes] u32 (NF4 only)
//   red  [128 rows][16 tokens] fp32, the partials the cluster reads
#include "common.cuh"

namespace wq {
namespace {

__device__ unsigned int g_gemv_error;  // this kernel has no waits; kept for the ABI

constexpr int kRowsPerCta = 128;

struct GemvArgs {
  const uint16_t* x;
  const uint8_t* qw;      // INT4: uint32 words viewed as bytes; NF4: code bytes
  const void* scales;     // INT4: fp16 [N, K/G]; NF4: fp32 absmax [N*K/64]
  const __half* zeros;    // INT4 only
  uint16_t* y;
  int M, N, K, G;
  int units;              // K / 128
  int S;                  // cluster size along K
  int kc;                 // shared-memory K-chunk length (max over ranks)
};

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ uint32_t map_rank(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// (128 + nibble) as bf16 for nibbles e and e + 4 of w -> one bf16x2 register.
__device__ __forceinline__ uint32_t int4_pair(uint32_t w, int e) {
  return lop3_and_or(w >> (4 * e), 0x000F000Fu, 0x43004300u);
}

// One 128-k unit of this lane's two weight rows, with its group parameters.
struct Unit {
  uint2 w[4];       // [row g h0, row g h1, row g+8 h0, row g+8 h1] (8 bytes each)
  uint32_t prm[4];  // INT4: (scale, zero) fp16 pairs [h][row]; NF4: absmax [h][row]
};

template <bool kNF4>
__device__ __forceinline__ void load_unit(Unit& U, const uint8_t* wA, const uint8_t* wB, int u,
                                          int nA, int nB, const GemvArgs& p, int ng) {
  const int64_t off = (int64_t)u * 64;
  U.w[0] = ld_stream_u2(wA + off);
  U.w[1] = ld_stream_u2(wA + off + 32);
  U.w[2] = ld_stream_u2(wB + off);
  U.w[3] = ld_stream_u2(wB + off + 32);
  if (kNF4) {
    const float* am = static_cast<const float*>(p.scales);
    const float2 aA =
        __ldg(reinterpret_cast<const float2*>(am + (int64_t)nA * (p.K / 64) + 2 * u));
    const float2 aB =
        __ldg(reinterpret_cast<const float2*>(am + (int64_t)nB * (p.K / 64) + 2 * u));
    U.prm[0] = __float_as_uint(aA.x);
    U.prm[1] = __float_as_uint(aB.x);
    U.prm[2] = __float_as_uint(aA.y);
    U.prm[3] = __float_as_uint(aB.y);
  } else {
    const unsigned short* s16 = reinterpret_cast<const unsigned short*>(p.scales);
    const unsigned short* z16 = reinterpret_cast<const unsigned short*>(p.zeros);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gi = (u * 128 + h * 64) / p.G;
      const int64_t iA = (int64_t)nA * ng + gi, iB = (int64_t)nB * ng + gi;
      U.prm[2 * h + 0] = (uint32_t)__ldg(s16 + iA) | ((uint32_t)__ldg(z16 + iA) << 16);
      U.prm[2 * h + 1] = (uint32_t)__ldg(s16 + iB) | ((uint32_t)__ldg(z16 + iB) << 16);
    }
  }
}

template <int NT, bool kNF4>
__global__ void __launch_bounds__(256, 3) gemv_kernel(GemvArgs p, Nf4Table tab) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int kTok = 8 * NT;
  const int kc = p.kc;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);
  uint8_t* cursor = smem + (size_t)kTok * kc * 2;
  uint32_t* lut = nullptr;
  if (kNF4) {
    lut = reinterpret_cast<uint32_t*>(cursor);
    cursor += 256 * 32 * 4;
  }
  float* red = reinterpret_cast<float*>(cursor);
  __shared__ float tok_inv[16];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)blockIdx.x;  // == cluster rank (the cluster spans gridDim.x)
  const int u0 = (int)((int64_t)rank * p.units / p.S);
  const int u1 = (int)((int64_t)(rank + 1) * p.units / p.S);
  const int k0 = u0 * 128;
  const int klen = (u1 - u0) * 128;
  const int row_tile = (int)blockIdx.y * kRowsPerCta;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = row_tile + warp * 16;
  const bool active = n0 < p.N;
  const int nA = n0 + g, nB = n0 + g + 8;
  const int ng = p.K / p.G;

  // the first unit's loads go out before anything else
  const int64_t row_bytes = (int64_t)p.K / 2;
  const uint8_t* wrowA = p.qw + (int64_t)(active ? nA : 0) * row_bytes + 8 * t;
  const uint8_t* wrowB = wrowA + 8 * row_bytes;
  Unit cur, nxt;
  if (active && u0 < u1) load_unit<kNF4>(cur, wrowA, wrowB, u0, nA, nB, p, ng);

  // ---- stage x[:, k0 : k0+klen) into shared memory (16-byte chunks) -------
  {
    const int chunks_per_row = kc / 8;
    for (int c = tid; c < kTok * chunks_per_row; c += blockDim.x) {
      const int gt = c / chunks_per_row;
      const int kl = (c - gt * chunks_per_row) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (gt < p.M && kl < klen)
        v = *reinterpret_cast<const uint4*>(p.x + (size_t)gt * p.K + k0 + kl);
      *reinterpret_cast<uint4*>(xs + (size_t)gt * kc + (kl ^ ((gt & 1) << 3))) = v;
    }
  }
  if (kNF4) {
    // four lanes' copies of one entry per 16-byte store
    for (int i = tid; i < 256 * 8; i += blockDim.x) {
      const int e = i >> 3;
      // low half: element 2j (high nibble); high half: element 2j+1
      const uint32_t v = pack_f16x2(tab.v[e >> 4], tab.v[e & 15]);
      reinterpret_cast<uint4*>(lut)[i] = make_uint4(v, v, v, v);
    }
  }
  __syncthreads();
  if (kNF4) {
    // per token: x chunk -> fp16 * 2^e in place (the swizzle moves whole chunks)
    constexpr int tpt = 256 / kTok;  // threads per token: 32 or 16
    const int gt = tid / tpt, j = tid % tpt;
    uint16_t* row = xs + (size_t)gt * kc;
    float mx = 0.0f;
    for (int c = j; c < kc / 8; c += tpt) {
      const uint4 v = *reinterpret_cast<const uint4*>(row + c * 8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        mx = fmaxf(mx, fmaxf(fabsf(bf16_lo_to_f32(w[i])), fabsf(bf16_hi_to_f32(w[i]))));
    }
#pragma unroll
    for (int o = tpt / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    int e = 0;
    if (mx > 0.0f && mx <= 3.0e38f) {
      e = 14 - ((int)((__float_as_uint(mx) >> 23) & 0xFF) - 127);
      e = e > 100 ? 100 : (e < -100 ? -100 : e);
    }
    const float sc = __uint_as_float((uint32_t)(127 + e) << 23);
    if (j == 0) tok_inv[gt] = __uint_as_float((uint32_t)(127 - e) << 23);
    for (int c = j; c < kc / 8; c += tpt) {
      uint4 v = *reinterpret_cast<const uint4*>(row + c * 8);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        w[i] = pack_f16x2(bf16_lo_to_f32(w[i]) * sc, bf16_hi_to_f32(w[i]) * sc);
      *reinterpret_cast<uint4*>(row + c * 8) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    __syncthreads();
  }

  // ---- main loop: warp owns 16 weight rows over this CTA's K-chunk --------
  float acc[NT][4];
#pragma unroll
  for (int a = 0; a < NT; ++a)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[a][r] = 0.0f;

  if (active) {
    const uint32_t lut_lane = kNF4 ? smem_u32(lut) + 4u * lane : 0u;
    constexpr uint32_t kOnes = 0x3F803F80u;  // bf16x2 (1, 1)
    for (int u = u0; u < u1; ++u) {
      if (u + 1 < u1) load_unit<kNF4>(nxt, wrowA, wrowB, u + 1, nA, nB, p, ng);
      const int lu = u - u0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint2 wa = cur.w[h], wb = cur.w[2 + h];
        uint32_t X[NT][8];
#pragma unroll
        for (int a = 0; a < NT; ++a) {
          const int tok = g + 8 * a;
          const uint16_t* base = xs + (size_t)tok * kc;
          const int kk = lu * 128 + h * 64 + 16 * t;
          const uint4 c0 = *reinterpret_cast<const uint4*>(base + (kk ^ ((tok & 1) << 3)));
          const uint4 c1 = *reinterpret_cast<const uint4*>(base + ((kk + 8) ^ ((tok & 1) << 3)));
          X[a][0] = c0.x; X[a][1] = c0.y; X[a][2] = c0.z; X[a][3] = c0.w;
          X[a][4] = c1.x; X[a][5] = c1.y; X[a][6] = c1.z; X[a][7] = c1.w;
        }
        float cp[NT][4], cs[NT][4];
#pragma unroll
        for (int a = 0; a < NT; ++a)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            cp[a][r] = 0.0f;
            cs[a][r] = 0.0f;
          }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          uint32_t a0, a1, a2, a3, bs0, bs1;
          if (!kNF4) {
            const int jw = ks >> 1, hh = ks & 1;
            const uint32_t WA = jw ? wa.y : wa.x, WB = jw ? wb.y : wb.x;
            a0 = int4_pair(WA, 2 * hh);
            a1 = int4_pair(WB, 2 * hh);
            a2 = int4_pair(WA, 2 * hh + 1);
            a3 = int4_pair(WB, 2 * hh + 1);
            bs0 = 4 * jw + hh;
            bs1 = 4 * jw + hh + 2;
          } else {
            // bytes 2ks and 2ks+1 of this lane's 8-byte slice
            const uint32_t WA = (ks >> 1) ? wa.y : wa.x, WB = (ks >> 1) ? wb.y : wb.x;
            const int sh0 = 16 * (ks & 1), sh1 = sh0 + 8;
            const uint32_t eA0 = (WA >> sh0) & 0xFFu, eA1 = (WA >> sh1) & 0xFFu;
            const uint32_t eB0 = (WB >> sh0) & 0xFFu, eB1 = (WB >> sh1) & 0xFFu;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a0) : "r"(lut_lane + eA0 * 128u));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a1) : "r"(lut_lane + eB0 * 128u));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a2) : "r"(lut_lane + eA1 * 128u));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a3) : "r"(lut_lane + eB1 * 128u));
            bs0 = 2 * ks;
            bs1 = 2 * ks + 1;
          }
#pragma unroll
          for (int a = 0; a < NT; ++a) {
            if (!kNF4) {
              // (x[2i], x[2i+4]) and (x[2i+1], x[2i+5]) from consecutive pairs
              const uint32_t b0 = prmt(X[a][bs0], X[a][bs1], 0x5410u);
              const uint32_t b1 = prmt(X[a][bs0], X[a][bs1], 0x7632u);
              mma16816(cp[a], a0, a1, a2, a3, b0, b1);
              mma16816(cs[a], kOnes, kOnes, kOnes, kOnes, b0, b1);  // sum of x
            } else {
              mma16816_f16(cp[a], a0, a1, a2, a3, X[a][bs0], X[a][bs1]);
            }
          }
        }
        // post-group (INT4) / post-block (NF4) scaling
#pragma unroll
        for (int a = 0; a < NT; ++a) {
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const uint32_t pv = cur.prm[2 * h + (r >> 1)];  // row g for r < 2, g+8 else
            if (kNF4) {
              acc[a][r] = fmaf(__uint_as_float(pv), cp[a][r], acc[a][r]);
            } else {
              const float s = __half2float(__ushort_as_half((unsigned short)(pv & 0xFFFFu)));
              const float zb =
                  128.0f + __half2float(__ushort_as_half((unsigned short)(pv >> 16)));
              acc[a][r] = fmaf(s, fmaf(-zb, cs[a][r], cp[a][r]), acc[a][r]);
            }
          }
        }
      }
      cur = nxt;
    }
  }

  // ---- cluster split-K reduction through distributed shared memory --------
#pragma unroll
  for (int a = 0; a < NT; ++a)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = warp * 16 + g + 8 * (r >> 1);
      const int tok = 8 * a + 2 * t + (r & 1);
      red[row * 16 + tok] = kNF4 ? acc[a][r] * tok_inv[tok] : acc[a][r];
    }
  if (p.S > 1) {
    cluster_sync_all();
  } else {
    __syncthreads();
  }
  {
    const int rows_per_rank = kRowsPerCta / p.S;  // S divides 128 (S is 1, 2, 4 or 8)
    const int r_begin = rank * rows_per_rank;
    const int items = rows_per_rank * p.M;
    for (int i = tid; i < items; i += blockDim.x) {
      const int tok = i / rows_per_rank;
      const int row = r_begin + (i - tok * rows_per_rank);
      const int n = row_tile + row;
      const float* src = &red[row * 16 + tok];
      float parts[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)  // all remote loads in flight before the sum
        parts[q] =
            (q < p.S) ? (p.S > 1 ? ld_cluster_f32(map_rank(src, (uint32_t)q)) : *src) : 0.0f;
      float v = 0.0f;
#pragma unroll
      for (int q = 0; q < 8; ++q) v += parts[q];
      if (n < p.N) p.y[(int64_t)tok * p.N + n] = (uint16_t)(pack_bf16x2(v, 0.0f) & 0xFFFFu);
    }
  }
  if (p.S > 1) cluster_sync_all();  // keep shared memory alive until all ranks have read it
}

template <int NT, bool kNF4>
size_t gemv_smem(int kc) {
  return (size_t)8 * NT * kc * 2 + (size_t)kRowsPerCta * 16 * 4 + (kNF4 ? 256 * 32 * 4 : 0);
}

// Cluster size S (K split): every CTA holds one 128-row tile over one K-chunk.
// S is chosen among {1, 2, 4, 8} (S <= 128-wide units, x chunk <= 48 KB) to
// fill the resident CTA slots of the GPU with the fewest partial waves.
template <int NT, bool kNF4>
int gemv_split(int64_t N, int64_t K) {
  const int64_t tiles = (N + kRowsPerCta - 1) / kRowsPerCta;
  const int64_t units = K / 128;
  double best = -1.0;
  int bS = 0;
  for (int S = 1; S <= 8; S *= 2) {
    if (S > units) break;
    const int kc = (int)((units + S - 1) / S) * 128;
    if ((int64_t)8 * NT * kc * 2 > 48 * 1024) continue;
    const size_t smem = gemv_smem<NT, kNF4>(kc);
    auto kern = gemv_kernel<NT, kNF4>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      continue;
    int slots = 0;
    if (S == 1) {
      int per_sm = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem) != cudaSuccess)
        continue;
      slots = per_sm * num_sms();
    } else {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)S, (unsigned)tiles, 1);
      cfg.blockDim = dim3(256, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)S;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        continue;
      }
      slots = clusters * S;
    }
    if (slots < 1) continue;
    const int64_t grid = tiles * S;
    const int64_t waves = (grid + slots - 1) / slots;
    // share of the resident slots kept busy, discounted per extra wave
    const double score = (double)grid / ((double)waves * slots) - 0.02 * (double)(waves - 1);
    if (score > best + 1e-9) {
      best = score;
      bS = S;
    }
  }
  return bS;
}

template <int NT, bool kNF4>
wq_status launch_t(GemvArgs a, cudaStream_t st) {
  a.S = gemv_split<NT, kNF4>(a.N, a.K);
  if (a.S < 1) return WQ_ERR_UNSUPPORTED;
  a.kc = ((a.units + a.S - 1) / a.S) * 128;
  const size_t smem = gemv_smem<NT, kNF4>(a.kc);
  auto kern = gemv_kernel<NT, kNF4>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return WQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.S, (unsigned)((a.N + kRowsPerCta - 1) / kRowsPerCta), 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)a.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, a, nf4_table()) != cudaSuccess) return WQ_ERR_CUDA;
  return launch_status();
}

}  // namespace

wq_status launch_gemv(const void* x, int64_t M, int64_t N, int64_t K, wq_format fmt, int32_t group,
                      const void* qweight, const void* scales, const void* zeros, void* y,
                      cudaStream_t st) {
  const int NT = M <= 8 ? 1 : 2;
  GemvArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.qw = static_cast<const uint8_t*>(qweight);
  a.scales = scales;
  a.zeros = static_cast<const __half*>(zeros);
  a.y = static_cast<uint16_t*>(y);
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.G = group;
  a.units = (int)(K / 128);
  a.S = 1;
  a.kc = 0;
  if (fmt == WQ_FMT_NF4) return NT == 1 ? launch_t<1, true>(a, st) : launch_t<2, true>(a, st);
  return NT == 1 ? launch_t<1, false>(a, st) : launch_t<2, false>(a, st);
}

wq_status read_gemv_error(bool clear, uint32_t* v) {
  uint32_t h = 0;
  if (cudaMemcpyFromSymbol(&h, g_gemv_error, sizeof(h)) != cudaSuccess) return WQ_ERR_CUDA;
  if (clear && h) {
    const uint32_t z = 0;
    if (cudaMemcpyToSymbol(g_gemv_error, &z, sizeof(z)) != cudaSuccess) return WQ_ERR_CUDA;
  }
  *v = h;
  return WQ_OK;
}

}  // namespace wq
