// MX (microscaling) path of Multi-Scale Dequant: MXFP4 weights, activations
// decomposed into two MXFP4 passes (or one MXFP8 pass, the comparator).
//
// Source: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
// Activation Decomposition for Efficient LLM Inference", Abstract: for MXFP4
// weights, two MXFP4 passes over the bf16 activations multiply the weights
// directly, against one MXFP8 pass. Group (here block) scales are applied after
// each block's sum ("MixPE: Quantization and Hardware Co-design for Efficient
// LLM Inference", Abstract).
//
// Format (the plainest reading of the page's MXFP4 / MXFP8): blocks of 32
// consecutive elements along K share one power-of-two scale X = 2^e, stored as
// the byte e + 127 (the smallest e with amax <= 6 * 2^e for E2M1, 448 * 2^e for
// E4M3: no element saturates); elements E2M1 (magnitudes 0, 0.5, 1, 1.5, 2, 3,
// 4, 6; sign bit 3) or E4M3, rounded to nearest with ties to the even code; a
// value that rounds to zero is the positive zero code. MXFP4 weights pack two
// codes per byte, element 2j in the low nibble.
//
// B200 design. Every E2M1 value is exact in E4M3, so the product runs on the
// FP8 tensor cores: warp-level mma.m16n8k32 e4m3 x e4m3 with fp32
// accumulation (FP4 inputs to mma.sync do not exist on sm_100a). One MMA's
// k = 32 is exactly one MX block of both operands, and its sum is exact (at
// most 32 products of 13-bit dyadics), so each MMA's partial takes the two
// block scales 2^(e_w + e_x) in fp32 (two exact power-of-two multiplies and one
// rounding add). The decomposition writes the activation passes as E4M3 bytes
// (their MXFP4 values re-encoded exactly), so they are the B operand as
// stored; the weights' E2M1 nibbles become E4M3 bytes in registers with two
// byte permutes. The decode kernel is the split-K cluster GEMV structure of
// the INT4/NF4 decode path: 128 weight rows per CTA, K split over the
// cluster, each warp's 16 rows streamed through a cp.async ring of 128-byte
// row segments (8 blocks), partials reduced through distributed shared
// memory.
#include <cuda_fp8.h>

#include "splitk_common.cuh"

namespace wq {
namespace {

using namespace splitk;

constexpr int kMxStages = 3;
constexpr int kMaxMxChunkBytes = 64 * 1024;  // activation passes of one CTA's K-chunk

// E2M1 magnitude code of a scaled value |v| <= 6, nearest with ties to the
// even code: the decision points are the midpoints 0.25 .. 5, a tie going to
// the even side.
__device__ __forceinline__ uint32_t e2m1_code(float v) {
  const float a = fabsf(v);
  uint32_t c = a <= 0.25f ? 0u : a < 0.75f ? 1u : a <= 1.25f ? 2u : a < 1.75f ? 3u
             : a <= 2.5f ? 4u : a < 3.5f ? 5u : a <= 5.0f ? 6u : 7u;
  if (v < 0.0f && c != 0u) c |= 8u;
  return c;
}

__device__ __forceinline__ float e2m1_value(uint32_t c) {
  const float m[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  const float v = m[c & 7u];
  return (c & 8u) ? -v : v;
}

// E4M3 byte of the same value: magnitude codes 0..7 -> 0x00 0x30 0x38 0x3C
// 0x40 0x44 0x48 0x4C, sign bit 7.
__device__ __forceinline__ uint32_t e2m1_to_e4m3(uint32_t c) {
  const uint32_t m = prmt(0x3C383000u, 0x4C484440u, c & 7u) & 0xFFu;
  return m | ((c & 8u) << 4);
}

// Four E2M1 codes (nibbles of the low 16 bits of h) -> four E4M3 bytes. The
// magnitudes come from one byte permute (selectors = the nibbles' low 3
// bits); the second permute, with the sign bits left in the selectors,
// returns 0x01 for a non-negative nibble and 0x00 for a negative one (sign
// replication of 0x01), which becomes the 0x80 sign bit.
__device__ __forceinline__ uint32_t e2m1x4_to_e4m3x4(uint32_t h) {
  const uint32_t mag = prmt(0x3C383000u, 0x4C484440u, h & 0x7777u);
  const uint32_t pos = prmt(0x01010101u, 0x01010101u, h & 0xFFFFu);
  return mag | ((pos ^ 0x01010101u) << 7);
}

// Smallest e in [-127, 127] with a <= maxv * 2^e, maxv = 1.5 * 2^2 (E2M1) or
// 1.75 * 2^8 (E4M3); 0 for a = 0. For a in [2^F, 2^(F+1)): e = F - 2 + (a >
// 1.5 * 2^F) for E2M1 and F - 8 + (a > 1.75 * 2^F) for E4M3.
template <bool kFp8>
__device__ __forceinline__ int mx_exponent(float a) {
  if (!(a > 0.0f)) return 0;
  const int F = ilogbf(a);
  const float top = ldexpf(kFp8 ? 1.75f : 1.5f, F);
  int e = F - (kFp8 ? 8 : 2) + (a > top ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

__device__ __forceinline__ float pow2f(int e) {  // exact for e in [-127, 127]
  return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// ---------------------------------------------------------------------------
// Weight quantization: one warp per 32-element block (lane = element).
// ---------------------------------------------------------------------------
__global__ void mx_quantize_kernel(const float* __restrict__ w, int64_t nblocks,
                                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  for (int64_t b = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / 32; b < nblocks;
       b += (int64_t)gridDim.x * blockDim.x / 32) {
    const float v = w[b * 32 + lane];
    float a = fabsf(v);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const int e = mx_exponent<false>(a);
    const uint32_t c = e2m1_code(v * pow2f(-e));
    const uint32_t hi = __shfl_down_sync(0xffffffffu, c, 1);
    if ((lane & 1) == 0) codes[b * 16 + lane / 2] = (uint8_t)(c | (hi << 4));
    if (lane == 0) scales[b] = (uint8_t)(e + 127);
  }
}

// ---------------------------------------------------------------------------
// Activation decomposition: one warp per (row, block). Two MXFP4 passes
// (x1 = MXFP4(x), r = x - x1 exact in fp32, x2 = MXFP4(r)) or one MXFP8 pass,
// each written as E4M3 bytes planes[p][m][k] and scale bytes scales[p][m][blk].
// ---------------------------------------------------------------------------
template <int P>
__global__ void mx_decompose_kernel(const uint16_t* __restrict__ x, int M, int K,
                                    uint8_t* __restrict__ planes, uint8_t* __restrict__ scales) {
  // a dependent grid (the decode product) may start at once; it waits for
  // this grid before reading the planes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int nblk = K / 32;
  const int64_t total = (int64_t)M * nblk;
  for (int64_t wb = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) / 32; wb < total;
       wb += (int64_t)gridDim.x * blockDim.x / 32) {
    const int m = (int)(wb / nblk), b = (int)(wb - (int64_t)m * nblk);
    const int64_t idx = (int64_t)m * K + b * 32 + lane;
    float v = __uint_as_float((uint32_t)x[idx] << 16);
#pragma unroll
    for (int p = 0; p < P; ++p) {
      float a = fabsf(v);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      uint32_t byte;
      int e;
      if (P == 1) {
        e = mx_exponent<true>(a);
        byte = __nv_cvt_float_to_fp8(v * pow2f(-e), __NV_SATFINITE, __NV_E4M3);
        if ((byte & 0x7Fu) == 0u) byte = 0u;  // a value rounding to zero: +0
      } else {
        e = mx_exponent<false>(a);
        const uint32_t c = e2m1_code(v * pow2f(-e));
        byte = e2m1_to_e4m3(c);
        v = v - e2m1_value(c) * pow2f(e);  // the residual, exact in fp32
      }
      planes[(int64_t)p * M * K + idx] = (uint8_t)byte;
      if (lane == 0) scales[((int64_t)p * M + m) * nblk + b] = (uint8_t)(e + 127);
    }
  }
}

// ---------------------------------------------------------------------------
// Decode product (M <= 16).
// ---------------------------------------------------------------------------
struct MxArgs {
  const uint8_t* planes;  // [P][M][K] E4M3 bytes
  const uint8_t* xs;      // [P][M][K/32] scale bytes
  const uint8_t* qw;      // [N][K/2] E2M1 codes
  const uint8_t* ws;      // [N][K/32] scale bytes
  uint16_t* y;
  int M, N, K;
  int units;              // K / 256 (one weight stage each)
  int S, kc;
};

__device__ __forceinline__ void mma_e4m3(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Weight stage: the warp's 16 rows x 128 bytes (8 blocks = 256 k); 16-byte
// chunk c (one block) of row r stored at chunk c ^ (r & 7), so that the four
// lanes reading word t of one block in eight different rows hit distinct
// banks.
__device__ __forceinline__ void mx_issue_stage(uint8_t* slot, const uint8_t* wtile,
                                               int64_t row_bytes, int stage, int lane) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q = 32 * i + lane, r = q >> 3, c = q & 7;
    cp_async16(slot + r * kStageRowBytes + ((c ^ (r & 7)) << 4),
               wtile + (int64_t)r * row_bytes + (int64_t)stage * 128 + 16 * c);
  }
}

// Data placement per CTA (dynamic shared memory):
//   ring [8 warps][kMxStages][16 rows][128 B]  weight stages
//   xp   [P][M][Kc] E4M3 bytes, 16-byte chunk c of token m at c ^ 2(m & 3)
//   xsc  [P][M][Kc/32] activation block scales as fp32 powers of two
//   red  [S ranks][ceil(128/S)][16] fp32
template <int NT, int P>
__global__ void __launch_bounds__(256, 2) mx_gemv_kernel(MxArgs p, Nf4Table) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int kc = p.kc, M = p.M;
  uint8_t* rings = smem;
  uint8_t* xp = smem + (size_t)8 * kMxStages * kStageBytes;
  float* xsc = reinterpret_cast<float*>(xp + (size_t)P * M * kc);
  float* red = xsc + (size_t)P * M * (kc / 32);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)blockIdx.x;
  const int u0 = (int)((int64_t)rank * p.units / p.S);
  const int u1 = (int)((int64_t)(rank + 1) * p.units / p.S);
  const int nst = u1 - u0;                 // weight stages (256 k each)
  const int k0 = u0 * 256, klen = nst * 256;
  const int row_tile = (int)blockIdx.y * kRowsPerCta;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = row_tile + warp * 16;
  const bool active = n0 < p.N;
  const int64_t row_bytes = p.K / 2;
  const int nblk = p.K / 32;

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- the first stages of this warp's weights and their scale bytes
  // (8 blocks of rows g and g + 8: two 8-byte loads per stage)
  uint8_t* wring = rings + (size_t)warp * kMxStages * kStageBytes;
  const uint8_t* wtile = p.qw + (int64_t)(active ? n0 : 0) * row_bytes;
  const uint8_t* wsA = p.ws + (int64_t)(active ? n0 + g : 0) * nblk;
  const uint8_t* wsB = wsA + 8 * (int64_t)nblk;
  uint2 wsc[kMxStages][2];
  auto issue = [&](int j, uint2 (&sc)[2], uint8_t* slot) {
    mx_issue_stage(slot, wtile, row_bytes, u0 + j, lane);
    sc[0] = __ldg(reinterpret_cast<const uint2*>(wsA + (u0 + j) * 8));
    sc[1] = __ldg(reinterpret_cast<const uint2*>(wsB + (u0 + j) * 8));
  };
#pragma unroll
  for (int i = 0; i < kMxStages - 1; ++i) {
    if (active && i < nst) issue(i, wsc[i], wring + i * kStageBytes);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  // ---- the activation passes of this K-chunk, once the decomposition is done
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int kch = klen / 16;
  for (int c = tid; c < P * M * kch; c += blockDim.x) {
    const int pm = c / kch, cl = c - pm * kch;
    const int m = pm % M;
    cp_async16(xp + (size_t)pm * kc + ((cl ^ (2 * (m & 3))) << 4),
               p.planes + (int64_t)pm * p.K + k0 + cl * 16);
  }
  for (int c = tid; c < P * M * (klen / 32); c += blockDim.x) {
    const int pm = c / (klen / 32), b = c - pm * (klen / 32);
    xsc[(size_t)pm * (kc / 32) + b] = pow2f((int)p.xs[(int64_t)pm * nblk + k0 / 32 + b] - 127);
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  // the lane's B rows (padding tokens read token 0: their columns never reach
  // an output) and the tokens of its accumulator columns
  int brow[NT], tokc[NT][2];
#pragma unroll
  for (int a = 0; a < NT; ++a) {
    brow[a] = (g + 8 * a < M) ? g + 8 * a : 0;
#pragma unroll
    for (int e = 0; e < 2; ++e) tokc[a][e] = min(8 * a + 2 * t + e, M - 1);
  }

  float acc[NT][4];
#pragma unroll
  for (int a = 0; a < NT; ++a)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[a][r] = 0.0f;

  for (int jb = 0; jb < nst; jb += kMxStages) {
#pragma unroll
    for (int i = 0; i < kMxStages; ++i) {
      const int j = jb + i;
      if (j < nst) {
        const int kNext = (i + kMxStages - 1) % kMxStages;  // a constant once unrolled
        if (active && j + kMxStages - 1 < nst)
          issue(j + kMxStages - 1, wsc[kNext], wring + kNext * kStageBytes);
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group %0;" ::"n"(kMxStages - 1) : "memory");
        __syncwarp();
        if (active) {
          const uint8_t* slot = wring + i * kStageBytes;
          const uint32_t swA[2] = {wsc[i][0].x, wsc[i][0].y}, swB[2] = {wsc[i][1].x, wsc[i][1].y};
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            // this lane's 8 codes (word t of block b) of rows g and g + 8:
            // block-local k = 8t .. 8t + 7 in the MMA's k slots 4t .. 4t + 3
            // and 16 + 4t .. 16 + 4t + 3 (the activations use the same slots)
            const uint32_t wa = *reinterpret_cast<const uint32_t*>(
                slot + g * kStageRowBytes + ((b ^ (g & 7)) << 4) + 4 * t);
            const uint32_t wb = *reinterpret_cast<const uint32_t*>(
                slot + (g + 8) * kStageRowBytes + ((b ^ (g & 7)) << 4) + 4 * t);
            const uint32_t a0 = e2m1x4_to_e4m3x4(wa), a2 = e2m1x4_to_e4m3x4(wa >> 16);
            const uint32_t a1 = e2m1x4_to_e4m3x4(wb), a3 = e2m1x4_to_e4m3x4(wb >> 16);
            const float fwA = pow2f((int)((swA[b >> 2] >> (8 * (b & 3))) & 0xFFu) - 127);
            const float fwB = pow2f((int)((swB[b >> 2] >> (8 * (b & 3))) & 0xFFu) - 127);
            const int lb = j * 8 + b;  // block index within the K-chunk
#pragma unroll
            for (int pp = 0; pp < P; ++pp)
#pragma unroll
              for (int a = 0; a < NT; ++a) {
                const int bt = brow[a];
                const uint2 xv = *reinterpret_cast<const uint2*>(
                    xp + ((size_t)pp * M + bt) * kc + (((2 * lb + (t >> 1)) ^ (2 * (bt & 3))) << 4) +
                    8 * (t & 1));
                float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                mma_e4m3(d, a0, a1, a2, a3, xv.x, xv.y);
                const float fx0 = xsc[((size_t)pp * M + tokc[a][0]) * (kc / 32) + lb];
                const float fx1 = xsc[((size_t)pp * M + tokc[a][1]) * (kc / 32) + lb];
                acc[a][0] = fmaf(d[0] * fwA, fx0, acc[a][0]);
                acc[a][1] = fmaf(d[1] * fwA, fx1, acc[a][1]);
                acc[a][2] = fmaf(d[2] * fwB, fx0, acc[a][2]);
                acc[a][3] = fmaf(d[3] * fwB, fx1, acc[a][3]);
              }
          }
        }
        __syncwarp();
      }
    }
  }

  reduce_and_store<NT>(acc, nullptr, red, p.S, rank, row_tile, M, p.N, p.y);
}

template <int NT, int P>
size_t mx_smem(int kc, int S, int M) {
  return (size_t)8 * kMxStages * kStageBytes + (size_t)P * M * kc +
         (size_t)P * M * (kc / 32) * 4 + red_bytes(S);
}

template <int NT, int P>
wq_status launch_mx_t(MxArgs a, cudaStream_t st) {
  auto kern = mx_gemv_kernel<NT, P>;
  // the planner splits K in units of 128; this kernel's stages are 256 k,
  // so it plans on K / 2 and doubles the chunk
  const Plan pl = cached_plan(reinterpret_cast<const void*>(kern), a.M, a.N, a.K, P, [&] {
    return make_plan(
        kern, 256, a.N, a.K / 2, [&](int kc) { return (int64_t)P * a.M * 2 * kc <= kMaxMxChunkBytes; },
        [&](int kc, int S) { return mx_smem<NT, P>(2 * kc, S, a.M); });
  });
  if (pl.S < 1) return WQ_ERR_UNSUPPORTED;
  a.S = pl.S;
  a.kc = 2 * pl.kc;
  Plan pl2 = pl;
  pl2.smem = mx_smem<NT, P>(a.kc, pl.S, a.M);
  return launch_split(kern, pl2, 256, a.N, st, a, nf4_table(), false, /*early=*/true);
}

}  // namespace

wq_status launch_mx_quantize(const float* w, int64_t N, int64_t K, uint8_t* codes,
                             uint8_t* scales, cudaStream_t st) {
  const int64_t nblocks = N * K / 32;
  const int64_t grid = std::min<int64_t>((nblocks + 7) / 8, (int64_t)num_sms() * 16);
  mx_quantize_kernel<<<(unsigned)grid, 256, 0, st>>>(w, nblocks, codes, scales);
  return launch_status();
}

wq_status launch_mx_decompose(const void* x, int64_t M, int64_t K, int32_t P, uint8_t* planes,
                              uint8_t* scales, cudaStream_t st) {
  const int64_t warps = M * (K / 32);
  const int64_t grid = std::min<int64_t>((warps + 7) / 8, (int64_t)num_sms() * 16);
  if (P == 2)
    mx_decompose_kernel<2><<<(unsigned)grid, 256, 0, st>>>(static_cast<const uint16_t*>(x),
                                                           (int)M, (int)K, planes, scales);
  else
    mx_decompose_kernel<1><<<(unsigned)grid, 256, 0, st>>>(static_cast<const uint16_t*>(x),
                                                           (int)M, (int)K, planes, scales);
  return launch_status();
}

// Workspace: the activation passes [P][M][K] (256-byte aligned), then their
// scale bytes [P][M][K/32].
size_t mx_workspace_bytes(int64_t M, int64_t K, int32_t P) {
  return ((size_t)P * M * K + 255) / 256 * 256 + (size_t)P * M * (K / 32);
}

wq_status launch_mx_gemv(const void* x, int64_t M, int64_t N, int64_t K, int32_t P,
                         const uint8_t* codes, const uint8_t* scales, void* y, void* workspace,
                         cudaStream_t st) {
  uint8_t* planes = static_cast<uint8_t*>(workspace);
  uint8_t* xs = planes + ((size_t)P * M * K + 255) / 256 * 256;
  wq_status s = launch_mx_decompose(x, M, K, P, planes, xs, st);
  if (s != WQ_OK) return s;
  MxArgs a;
  a.planes = planes;
  a.xs = xs;
  a.qw = codes;
  a.ws = scales;
  a.y = static_cast<uint16_t*>(y);
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.units = (int)(K / 256);
  a.S = 1;
  a.kc = 0;
  if (P == 2) return M <= 8 ? launch_mx_t<1, 2>(a, st) : launch_mx_t<2, 2>(a, st);
  return M <= 8 ? launch_mx_t<1, 1>(a, st) : launch_mx_t<2, 1>(a, st);
}

}  // namespace wq
