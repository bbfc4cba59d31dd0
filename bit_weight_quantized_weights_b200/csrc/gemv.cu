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
//   flops), so the kernel is built to keep HBM busy: 16-byte-aligned 8-byte
//   loads that do not allocate in L1, many independent warps, and no
//   workspace traffic.
// * At M = 16 the multiply-adds alone (2*16 flops per weight at ~12 Tweights/s)
//   exceed what the CUDA cores can issue, so the product runs on the tensor
//   cores with warp-level mma.m16n8k16 (bf16 in, fp32 accumulate): weight rows
//   form the 16-row A operand, tokens the 8-column B operand. This is an
//   HBM-bound kernel; the tensor pipe is far from busy.
// * INT4 codes become bf16 in registers without any arithmetic: OR-ing a nibble
//   into the mantissa of 128.0 (bit pattern 0x4300) gives exactly 128 + q, two
//   per 32-bit LOP3. The MMA then sums (128 + q) x over a 64-wide sub-group and
//   the epilogue applies s * (P - (128 + z) * sum(x)), the MixPE post-group
//   form, with sum(x) computed once per CTA from shared memory.
// * NF4 codes go through a 256-entry table indexed by a whole packed byte that
//   yields the two fp16 code values already paired as one A-operand register.
//   The table is replicated per lane (lane l reads column l, so bank l), which
//   makes every lookup conflict-free. The block's absmax is applied after the
//   block's sum. The NF4 product runs in fp16 (the code values keep 11
//   significant bits): each CTA converts its x chunk to fp16 in shared memory,
//   scaled per token by a power of two that puts the chunk's largest magnitude
//   in [2^14, 2^15) (exact for bf16 inputs down to 2^-28 of it), and divides
//   the power back out of its partial sums.
// * Split-K across a thread-block cluster: the S CTAs of a cluster share one
//   128-row tile and split K; their fp32 partials are summed through
//   distributed shared memory, in a fixed order, and written once as bf16.
//
// Data placement per CTA (dynamic shared memory):
//   xs   [8*NT tokens][Kc] bf16, the CTA's K-chunk of x (zero-padded tokens);
//        a token row of odd index has bit 3 of k flipped (16-byte swizzle)
//   xsum [8*NT tokens][Kc/64] fp32 (INT4 only)
//   lut  [256 entries][32 lanes] u32 (NF4 only)
//   red  [128 rows][16 tokens] fp32, the partials read by the cluster
#include "common.cuh"

namespace wq {
namespace {

constexpr int kRowsPerCta = 128;
constexpr int kWarps = 8;

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

__device__ __forceinline__ uint2 ld_w64(const uint8_t* p) { return ld_stream_u2(p); }

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(const float* local, uint32_t rank) {
  uint32_t a = smem_u32(local), r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(r) : "memory");
  return v;
}

// (128 + nibble) as bf16 for nibbles e and e + 4 of w -> one bf16x2 register.
__device__ __forceinline__ uint32_t int4_pair(uint32_t w, int e) {
  return lop3_and_or(w >> (4 * e), 0x000F000Fu, 0x43004300u);
}

template <int NT, bool kNF4>
__global__ void __launch_bounds__(256) gemv_kernel(GemvArgs p, Nf4Table tab) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int kTok = 8 * NT;
  const int kc = p.kc;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);
  uint8_t* cursor = smem + (size_t)kTok * kc * 2;
  float* xsum = nullptr;
  uint32_t* lut = nullptr;
  if (!kNF4) {
    xsum = reinterpret_cast<float*>(cursor);
    cursor += (size_t)kTok * (kc / 64) * 4;
  } else {
    lut = reinterpret_cast<uint32_t*>(cursor);
    cursor += 256 * 32 * 4;
  }
  float* red = reinterpret_cast<float*>(cursor);
  __shared__ float tok_inv[16];  // NF4: 2^-e per token of this CTA's chunk

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)blockIdx.x;  // == cluster rank (cluster spans gridDim.x)
  const int u0 = (int)((int64_t)rank * p.units / p.S);
  const int u1 = (int)((int64_t)(rank + 1) * p.units / p.S);
  const int k0 = u0 * 128;
  const int klen = (u1 - u0) * 128;
  const int row_tile = (int)blockIdx.y * kRowsPerCta;

  // ---- stage x[:, k0 : k0+klen) into shared memory (16-byte chunks) -------
  {
    const int chunks_per_row = kc / 8;
    for (int c = tid; c < kTok * chunks_per_row; c += blockDim.x) {
      const int g = c / chunks_per_row;
      const int kl = (c - g * chunks_per_row) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (g < p.M && kl < klen)
        v = *reinterpret_cast<const uint4*>(p.x + (size_t)g * p.K + k0 + kl);
      const int ks = kl ^ ((g & 1) << 3);
      *reinterpret_cast<uint4*>(xs + (size_t)g * kc + ks) = v;
    }
  }
  if (kNF4) {
    __shared__ float cb[16];
    if (tid < 16) cb[tid] = tab.v[tid];
    __syncthreads();
    for (int i = tid; i < 256 * 32; i += blockDim.x) {
      const int e = i >> 5;
      // low half: element 2j (high nibble); high half: element 2j+1
      lut[i] = pack_f16x2(cb[e >> 4], cb[e & 15]);
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
  if (!kNF4) {
    const int subs = kc / 64;
    for (int i = tid; i < kTok * subs; i += blockDim.x) {
      const int g = i / subs, su = i - g * subs;
      float s = 0.0f;
      const uint16_t* row = xs + (size_t)g * kc;
      for (int k = su * 64; k < su * 64 + 64; ++k) {
        const int ks = k ^ ((g & 1) << 3);
        s += __uint_as_float((uint32_t)row[ks] << 16);
      }
      xsum[i] = s;
    }
    __syncthreads();
  }

  // ---- main loop: warp owns 16 weight rows, all of this CTA's K-chunk ------
  const int g = lane >> 2, t = lane & 3;
  const int n0 = row_tile + warp * 16;
  const bool active = n0 < p.N;
  float acc[NT][4];
#pragma unroll
  for (int a = 0; a < NT; ++a)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[a][r] = 0.0f;

  if (active) {
    // byte offsets of this lane's 8-byte slice of rows n0+g and n0+g+8
    const int64_t row_bytes = (int64_t)p.K / 2;
    const uint8_t* wrowA = p.qw + (int64_t)(n0 + g) * row_bytes + 8 * t;
    const uint8_t* wrowB = wrowA + 8 * row_bytes;
    const uint32_t lut_lane = kNF4 ? smem_u32(lut) + 4u * lane : 0u;
    const int ng = p.K / p.G;

    constexpr int UB = 4;  // units per load batch
    for (int ub = u0; ub < u1; ub += UB) {
      uint2 wv[UB][4];     // [unit][rowA h0, rowA h1, rowB h0, rowB h1]
      float sc[UB][2][2];  // [unit][h][row]  scale (INT4) or absmax (NF4)
      float zb[UB][2][2];  // [unit][h][row]  128 + zero (INT4)
#pragma unroll
      for (int b = 0; b < UB; ++b) {
        const int u = ub + b;
        if (u < u1) {
          const int64_t off = (int64_t)u * 64;
          wv[b][0] = ld_w64(wrowA + off);
          wv[b][1] = ld_w64(wrowA + off + 32);
          wv[b][2] = ld_w64(wrowB + off);
          wv[b][3] = ld_w64(wrowB + off + 32);
          if (kNF4) {
            const float* am = static_cast<const float*>(p.scales);
            const float2 aA = __ldg(reinterpret_cast<const float2*>(
                am + (int64_t)(n0 + g) * (p.K / 64) + 2 * u));
            const float2 aB = __ldg(reinterpret_cast<const float2*>(
                am + (int64_t)(n0 + g + 8) * (p.K / 64) + 2 * u));
            sc[b][0][0] = aA.x; sc[b][1][0] = aA.y;
            sc[b][0][1] = aB.x; sc[b][1][1] = aB.y;
          } else {
            const __half* s16 = static_cast<const __half*>(p.scales);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int gi = (u * 128 + h * 64) / p.G;
              const int64_t iA = (int64_t)(n0 + g) * ng + gi;
              const int64_t iB = (int64_t)(n0 + g + 8) * ng + gi;
              sc[b][h][0] = __half2float(s16[iA]);
              sc[b][h][1] = __half2float(s16[iB]);
              zb[b][h][0] = 128.0f + __half2float(p.zeros[iA]);
              zb[b][h][1] = 128.0f + __half2float(p.zeros[iB]);
            }
          }
        }
      }
#pragma unroll
      for (int b = 0; b < UB; ++b) {
        const int u = ub + b;
        if (u < u1) {
          const int lu = u - u0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint2 wa = wv[b][h], wb = wv[b][2 + h];
            // x fragments: 16 consecutive k of this lane, two 16-byte chunks
            uint32_t X[NT][8];
#pragma unroll
            for (int a = 0; a < NT; ++a) {
              const int tok = g + 8 * a;
              const uint16_t* base = xs + (size_t)tok * kc;
              const int kk = lu * 128 + h * 64 + 16 * t;
              const uint4 c0 = *reinterpret_cast<const uint4*>(base + (kk ^ ((tok & 1) << 3)));
              const uint4 c1 =
                  *reinterpret_cast<const uint4*>(base + ((kk + 8) ^ ((tok & 1) << 3)));
              X[a][0] = c0.x; X[a][1] = c0.y; X[a][2] = c0.z; X[a][3] = c0.w;
              X[a][4] = c1.x; X[a][5] = c1.y; X[a][6] = c1.z; X[a][7] = c1.w;
            }
            float cp[NT][4];
#pragma unroll
            for (int a = 0; a < NT; ++a)
#pragma unroll
              for (int r = 0; r < 4; ++r) cp[a][r] = 0.0f;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              uint32_t a0, a1, a2, a3;
              uint32_t bsel0, bsel1;  // x register indices (INT4 needs a pair permute)
              if (!kNF4) {
                const int j = s >> 1, hh = s & 1;
                const uint32_t WA = j ? wa.y : wa.x, WB = j ? wb.y : wb.x;
                a0 = int4_pair(WA, 2 * hh);
                a1 = int4_pair(WB, 2 * hh);
                a2 = int4_pair(WA, 2 * hh + 1);
                a3 = int4_pair(WB, 2 * hh + 1);
                bsel0 = 4 * j + hh;
                bsel1 = 4 * j + hh + 2;
              } else {
                // bytes 2s and 2s+1 of this lane's 8-byte slice
                const uint32_t WA = (s >> 1) ? wa.y : wa.x, WB = (s >> 1) ? wb.y : wb.x;
                const int sh0 = 16 * (s & 1), sh1 = sh0 + 8;
                const uint32_t eA0 = (WA >> sh0) & 0xFFu, eA1 = (WA >> sh1) & 0xFFu;
                const uint32_t eB0 = (WB >> sh0) & 0xFFu, eB1 = (WB >> sh1) & 0xFFu;
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a0) : "r"(lut_lane + eA0 * 128u));
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a1) : "r"(lut_lane + eB0 * 128u));
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a2) : "r"(lut_lane + eA1 * 128u));
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a3) : "r"(lut_lane + eB1 * 128u));
                bsel0 = 2 * s;
                bsel1 = 2 * s + 1;
              }
#pragma unroll
              for (int a = 0; a < NT; ++a) {
                uint32_t b0, b1;
                if (!kNF4) {
                  // (x[2i], x[2i+4]) and (x[2i+1], x[2i+5]) from consecutive pairs
                  b0 = prmt(X[a][bsel0], X[a][bsel1], 0x5410u);
                  b1 = prmt(X[a][bsel0], X[a][bsel1], 0x7632u);
                } else {
                  b0 = X[a][bsel0];
                  b1 = X[a][bsel1];
                }
                if (kNF4) mma16816_f16(cp[a], a0, a1, a2, a3, b0, b1);
                else mma16816(cp[a], a0, a1, a2, a3, b0, b1);
              }
            }
            // post-group (INT4) / post-block (NF4) scaling
            const int su = lu * 2 + h;
#pragma unroll
            for (int a = 0; a < NT; ++a) {
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const int row = r >> 1;  // 0: row g, 1: row g+8
                if (kNF4) {
                  acc[a][r] = fmaf(sc[b][h][row], cp[a][r], acc[a][r]);
                } else {
                  const int tok = 8 * a + 2 * t + (r & 1);
                  const float sx = xsum[tok * (kc / 64) + su];
                  acc[a][r] = fmaf(sc[b][h][row], fmaf(-zb[b][h][row], sx, cp[a][r]), acc[a][r]);
                }
              }
            }
          }
        }
      }
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
      float v = 0.0f;
      for (int q = 0; q < p.S; ++q)
        v += (p.S > 1) ? ld_dsmem_f32(&red[row * 16 + tok], (uint32_t)q) : red[row * 16 + tok];
      if (n < p.N) {
        const uint32_t b = pack_bf16x2(v, 0.0f) & 0xFFFFu;
        p.y[(int64_t)tok * p.N + n] = (uint16_t)b;
      }
    }
  }
  if (p.S > 1) cluster_sync_all();  // keep shared memory alive until all ranks have read it
}

template <int NT, bool kNF4>
wq_status launch_t(const GemvArgs& a, cudaStream_t st) {
  size_t smem = (size_t)8 * NT * a.kc * 2 + (size_t)kRowsPerCta * 16 * 4;
  smem += kNF4 ? 256 * 32 * 4 : (size_t)8 * NT * (a.kc / 64) * 4;
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

// Cluster size along K: enough CTAs for about two per SM, at most 8 (the
// portable cluster limit), a power of two dividing 128 rows, no more than the
// number of 128-wide K units, and few enough K per CTA for x to fit on chip.
int gemv_split(int64_t N, int64_t K, int NT) {
  const int64_t tiles = (N + kRowsPerCta - 1) / kRowsPerCta;
  const int64_t units = K / 128;
  int S = 1;
  while (S < 8 && tiles * S < 2 * (int64_t)num_sms() && 2 * S <= units) S *= 2;
  // x chunk: 8*NT tokens * kc * 2 bytes <= 96 KB
  while (S < 8 && 2 * S <= units && (int64_t)8 * NT * ((units + S - 1) / S) * 128 * 2 > 96 * 1024)
    S *= 2;
  return S;
}

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
  a.S = gemv_split(N, K, NT);
  a.kc = ((a.units + a.S - 1) / a.S) * 128;
  if ((int64_t)8 * NT * a.kc * 2 > 96 * 1024) return WQ_ERR_UNSUPPORTED;
  if (fmt == WQ_FMT_NF4)
    return NT == 1 ? launch_t<1, true>(a, st) : launch_t<2, true>(a, st);
  return NT == 1 ? launch_t<1, false>(a, st) : launch_t<2, false>(a, st);
}

}  // namespace wq
