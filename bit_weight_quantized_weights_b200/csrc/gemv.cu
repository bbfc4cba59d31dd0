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
//   flops). Weights are read with plain 16-byte (8-byte for NF4 and INT4
//   groups of 64) loads that do not allocate in L1, by two 256-thread CTAs per SM,
//   each warp keeping three or four 128-k units of its 16 rows (with their
//   group parameters) in flight while it computes the oldest. Measured on
//   B200, plain coalesced loads stream HBM far better than a TMA ring of
//   small boxes for this work.
// * At M = 16 the multiply-adds alone (2*16 flops per weight at ~12 Tweights/s)
//   exceed what the CUDA cores can issue, so the product runs on the tensor
//   cores with warp-level mma.m16n8k16 (fp32 accumulate): weight rows form
//   the 16-row A operand, tokens the 8-column B operand. Measured on B200,
//   one such MMA issues every ~8.3 cycles per SM sub-partition, so even at
//   M = 16 (16 MMAs per KB of weights) the pipe keeps up with ~8 TB/s.
// * INT4 codes become bf16 in registers without arithmetic: OR-ing a nibble
//   into the mantissa of 128.0 (bit pattern 0x4300) gives exactly 128 + q, two
//   per 32-bit LOP3, paired as (k, k + 4). x is staged in that same pairing,
//   so its fragments load straight from shared memory. The MMA sums
//   (128 + q) x over the group's part of a 128-wide unit and the epilogue
//   applies s * (P - (128 + z) * sum(x)), the MixPE post-group form, with the
//   sums of x per 64-wide sub-group computed once per CTA while x is staged.
// * NF4 codes go through a 256-entry table indexed by a whole packed byte that
//   yields the two fp16 code values already paired as one A-operand register.
//   The table is replicated per lane (lane l reads column l, so bank l): every
//   lookup is conflict-free. NF4 uses the 8-byte layout: half h of a unit is
//   one 64-element absmax block, so every MMA stays inside one block and the
//   block's fp32 absmax multiplies the MMA's partial sum in fp32 (only the
//   code value is rounded, once, to fp16; a block of any absmax, however
//   small, keeps full precision). The NF4 product runs in fp16: the staged x
//   chunk is converted to fp16 scaled per token by a power of two that puts
//   its largest magnitude in [2^14, 2^15) (exact for bf16 values down to
//   2^-28 of it); the power is divided back out of the partial.
// * Optional salient-channel residual correction (kRes, "DecDEC: A Systems
//   Approach to Advancing Low-Bit LLM Quantization", Abstract): the owners add
//   sum_j x[m, c_j] R^T[c_j, n] to each output in fp32 before its rounding.
// * Split-K across a thread-block cluster: the S CTAs of a cluster share one
//   128-row tile and split K. Each CTA pushes its fp32 partials into the
//   shared memory of the rank that owns those rows (remote stores, no round
//   trip); after one cluster barrier each owner sums its rows in rank order
//   and writes them once as bf16. No workspace, no atomics.
// * x reaches shared memory by 16-byte asynchronous copies issued before the
//   first weight loads, so the whole CTA waits on one round trip for it.
//
// Data placement per CTA (dynamic shared memory):
//   xs   [8*NT tokens][Kc] bf16 (fp16 for NF4), the CTA's K-chunk of x, in
//        16-byte chunks. Only the M real tokens are written: a padding
//        token's MMA column never reaches an output. Chunk c of token m sits
//        at chunk c ^ (m & 1), and for the 16-byte layout (INT4 groups that
//        are multiples of 128) also ^ (bit 3 of c moved to bit 1), so that
//        the fragment loads of a warp hit distinct banks. For INT4 each chunk
//        holds the pairs (x0,x4)(x1,x5)(x2,x6)(x3,x7), the nibble pairing.
//   xsum [Kc/64 or Kc/128][8*NT tokens] fp32, sums of x per group part (INT4)
//   lut  [256 entries][32 lanes] u32 (NF4 only)
//   red  [S ranks][ceil(128/S) rows][16 tokens] fp32, the partials of the
//        rows this rank owns, as pushed by every rank of the cluster
#include "splitk_common.cuh"

namespace wq {
namespace {

__device__ unsigned int g_gemv_error;  // this kernel has no waits; kept for the ABI

using namespace splitk;

constexpr size_t kMaxSmemBytes = 227 * 1024;  // dynamic shared memory of one CTA

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
  uint32_t gmagic;        // h / (G / 64) == umulhi(h, gmagic) for 64-wide part h; 0 if G == 64
  Residual rc;            // salient-channel correction (k == 0: none)
};

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// (128 + nibble) as bf16 for nibbles e and e + 4 of w -> one bf16x2 register.
__device__ __forceinline__ uint32_t int4_pair(uint32_t w, int e) {
  return lop3_and_or(w >> (4 * e), 0x000F000Fu, 0x43004300u);
}

// One 128-k unit of this lane's two weight rows (g and g + 8), with its
// group parameters, as the MMA loop takes it.
//   wide  : w[0..3] = 16 bytes of row g at byte 16t, w[4..7] the same of row
//           g + 8 (k = 32t .. 32t + 31); INT4: prm[0..1] = the scale bits of
//           rows g, g + 8 and prm[2..3] their zero bits (one group spans the
//           unit).
//   narrow: w[0..1] row g, half 0 (byte 8t), w[2..3] row g, half 1 (byte
//           32 + 8t), w[4..7] the same of row g + 8; prm[2h + i] = the scale
//           bits of half h for row g (i = 0) or g + 8 (i = 1), zz[2h + i] the
//           zero bits.
// NF4 (narrow): prm[2h + i] = the fp32 absmax bits of block 2u + h of row g
// (i = 0) or g + 8 (i = 1).
struct Unit {
  uint32_t w[8];
  uint32_t prm[4];
  uint32_t zz[4];  // narrow INT4 only
};

// Group parameters of unit u (see Unit) into prm[0..3], zz[0..3].
template <bool kNF4, bool kWide>
__device__ __forceinline__ void load_unit_prm(uint32_t* prm, uint32_t* zz, int u, int nA, int nB,
                                              const GemvArgs& p, int ng) {
  if (kNF4) {
    // half h of the unit (bytes 32h .. 32h + 31 of each row) is block 2u + h
    const float* am = static_cast<const float*>(p.scales);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      prm[2 * h + 0] = __float_as_uint(__ldg(am + (int64_t)nA * (p.K / 64) + 2 * u + h));
      prm[2 * h + 1] = __float_as_uint(__ldg(am + (int64_t)nB * (p.K / 64) + 2 * u + h));
    }
  } else {
    const unsigned short* s16 = reinterpret_cast<const unsigned short*>(p.scales);
    const unsigned short* z16 = reinterpret_cast<const unsigned short*>(p.zeros);
#pragma unroll
    for (int h = 0; h < (kWide ? 1 : 2); ++h) {
      const int gi = div_by_magic(2 * u + h, p.gmagic);
      const int64_t iA = (int64_t)nA * ng + gi, iB = (int64_t)nB * ng + gi;
      prm[2 * h + 0] = __ldg(s16 + iA);
      prm[2 * h + 1] = __ldg(s16 + iB);
      if (kWide) {
        prm[2] = __ldg(z16 + iA);
        prm[3] = __ldg(z16 + iB);
      } else {
        zz[2 * h + 0] = __ldg(z16 + iA);
        zz[2 * h + 1] = __ldg(z16 + iB);
      }
    }
  }
}

// The parameters of the two units of one stage.
struct StagePrm {
  uint32_t prm[2][4];
  uint32_t zz[2][4];
};

// Unit h of a stage slot into U.w (see Unit).
template <bool kWide>
__device__ __forceinline__ void read_unit(Unit& U, const uint8_t* slot, int h, int g, int t) {
  read_stage_unit<kWide>(U.w, slot, h, g, t);
}

// acc += s * (P - (128 + z) * sum(x)) for the four accumulator slots of one
// token tile; s_*, z_* hold the fp16 bits of rows g and g + 8, sx the two
// tokens' sums of x.
__device__ __forceinline__ void int4_post(float (&acc)[4], const float (&cp)[4], uint32_t s_g,
                                          uint32_t s_g8, uint32_t z_g, uint32_t z_g8,
                                          float2 sx) {
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const bool hi = (r >> 1) != 0;  // row g for r < 2, g + 8 else
    const float s = __half2float(__ushort_as_half((unsigned short)(hi ? s_g8 : s_g)));
    const float zb = 128.0f + __half2float(__ushort_as_half((unsigned short)(hi ? z_g8 : z_g)));
    acc[r] = fmaf(s, fmaf(-zb, (r & 1) ? sx.y : sx.x, cp[r]), acc[r]);
  }
}

// The products of one 128-k unit, accumulated into acc (see the data
// placement above for the shared-memory layouts read here).
// Token rows of xs above `mlast` are not staged; their lanes read row mlast
// instead (those MMA columns never reach an output).
template <int NT, bool kNF4, bool kWide>
__device__ __forceinline__ void compute_unit(const Unit& U, int lu, const uint16_t* xs, int kc,
                                             const float* xsum, const uint32_t* lut_lane, int g,
                                             int t, float (&acc)[NT][4], int mlast = 15) {
  constexpr int kTok = 8 * NT;
  if (kNF4) {
    // Narrow layout: half h of the unit is one 64-element absmax block, so
    // every MMA below stays inside one block. The table gives the fp16 code
    // values (each rounded once); the MMA sums them against the fp16 x
    // (exact) in fp32, and the block's fp32 absmax multiplies that partial
    // sum in fp32. Step ks = (jw, hh) of half h uses bytes 4jw + 2hh and
    // 4jw + 2hh + 1 of word 2h + jw: codes 64h + 16t + 8jw + 4hh + {0..3};
    // x is staged in natural order, so chunk 8h + 2t + jw holds them.
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float cp[2][NT][4];
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int a = 0; a < NT; ++a)
#pragma unroll
          for (int r = 0; r < 4; ++r) cp[c][a][r] = 0.0f;
      uint4 X[NT][2];
#pragma unroll
      for (int a = 0; a < NT; ++a) {
        const int tok = min(g + 8 * a, mlast);
        const int c0 = 16 * lu + 8 * h + 2 * t;
        const uint16_t* base = xs + (size_t)tok * kc;
        X[a][0] = *reinterpret_cast<const uint4*>(base + (c0 ^ (tok & 1)) * 8);
        X[a][1] = *reinterpret_cast<const uint4*>(base + ((c0 + 1) ^ (tok & 1)) * 8);
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int jw = ks >> 1, hh = ks & 1;
        const uint32_t WA = U.w[2 * h + jw], WB = U.w[4 + 2 * h + jw];
        const int sh0 = 16 * hh, sh1 = sh0 + 8;
        const uint32_t a0 = lut_lane[((WA >> sh0) & 0xFFu) * 32];
        const uint32_t a1 = lut_lane[((WB >> sh0) & 0xFFu) * 32];
        const uint32_t a2 = lut_lane[((WA >> sh1) & 0xFFu) * 32];
        const uint32_t a3 = lut_lane[((WB >> sh1) & 0xFFu) * 32];
#pragma unroll
        for (int a = 0; a < NT; ++a) {
          const uint32_t b0 = hh ? X[a][jw].z : X[a][jw].x;
          const uint32_t b1 = hh ? X[a][jw].w : X[a][jw].y;
          mma16816_f16(cp[hh][a], a0, a1, a2, a3, b0, b1);
        }
      }
      const float amA = __uint_as_float(U.prm[2 * h]), amB = __uint_as_float(U.prm[2 * h + 1]);
#pragma unroll
      for (int a = 0; a < NT; ++a) {
        acc[a][0] = fmaf(amA, cp[0][a][0] + cp[1][a][0], acc[a][0]);
        acc[a][1] = fmaf(amA, cp[0][a][1] + cp[1][a][1], acc[a][1]);
        acc[a][2] = fmaf(amB, cp[0][a][2] + cp[1][a][2], acc[a][2]);
        acc[a][3] = fmaf(amB, cp[0][a][3] + cp[1][a][3], acc[a][3]);
      }
    }
  } else if (kWide) {
    // two accumulator chains (even and odd k-steps) halve the MMA dependency chain
    float cp[2][NT][4];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int a = 0; a < NT; ++a)
#pragma unroll
        for (int r = 0; r < 4; ++r) cp[c][a][r] = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 X[NT];
#pragma unroll
      for (int a = 0; a < NT; ++a) {
        const int tok = min(g + 8 * a, mlast);
        const int pc = (16 * lu + 4 * t + j) ^ (t & 2) ^ (tok & 1);
        X[a] = *reinterpret_cast<const uint4*>(xs + (size_t)tok * kc + pc * 8);
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t a0 = int4_pair(U.w[j], 2 * hh), a1 = int4_pair(U.w[4 + j], 2 * hh);
        const uint32_t a2 = int4_pair(U.w[j], 2 * hh + 1), a3 = int4_pair(U.w[4 + j], 2 * hh + 1);
#pragma unroll
        for (int a = 0; a < NT; ++a)
          mma16816(cp[hh][a], a0, a1, a2, a3, hh ? X[a].z : X[a].x, hh ? X[a].w : X[a].y);
      }
    }
#pragma unroll
    for (int a = 0; a < NT; ++a) {
      float cs[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) cs[r] = cp[0][a][r] + cp[1][a][r];
      const float2 sx = *reinterpret_cast<const float2*>(xsum + lu * kTok + 8 * a + 2 * t);
      int4_post(acc[a], cs, U.prm[0], U.prm[1], U.prm[2], U.prm[3], sx);
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float cp[2][NT][4];  // even and odd k-steps
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int a = 0; a < NT; ++a)
#pragma unroll
          for (int r = 0; r < 4; ++r) cp[c][a][r] = 0.0f;
      uint4 X[NT][2];
#pragma unroll
      for (int a = 0; a < NT; ++a) {
        const int tok = g + 8 * a;
        const int c0 = 16 * lu + 8 * h + 2 * t;
        const uint16_t* base = xs + (size_t)tok * kc;
        X[a][0] = *reinterpret_cast<const uint4*>(base + (c0 ^ (tok & 1)) * 8);
        X[a][1] = *reinterpret_cast<const uint4*>(base + ((c0 + 1) ^ (tok & 1)) * 8);
      }
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int jw = ks >> 1, hh = ks & 1;
        const uint32_t WA = U.w[2 * h + jw], WB = U.w[4 + 2 * h + jw];
        const uint32_t a0 = int4_pair(WA, 2 * hh), a1 = int4_pair(WB, 2 * hh);
        const uint32_t a2 = int4_pair(WA, 2 * hh + 1), a3 = int4_pair(WB, 2 * hh + 1);
#pragma unroll
        for (int a = 0; a < NT; ++a) {
          const uint32_t b0 = hh ? X[a][jw].z : X[a][jw].x;
          const uint32_t b1 = hh ? X[a][jw].w : X[a][jw].y;
          mma16816(cp[hh][a], a0, a1, a2, a3, b0, b1);
        }
      }
#pragma unroll
      for (int a = 0; a < NT; ++a) {
        float cs[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) cs[r] = cp[0][a][r] + cp[1][a][r];
        const float2 sx =
            *reinterpret_cast<const float2*>(xsum + (2 * lu + h) * kTok + 8 * a + 2 * t);
        int4_post(acc[a], cs, U.prm[2 * h], U.prm[2 * h + 1], U.zz[2 * h], U.zz[2 * h + 1], sx);
      }
    }
  }
}

// The CTA: 16 warps of 16 rows (a 256-row tile), one CTA per SM, each warp
// with its own ring of kStages stages.
constexpr int kGemvRows = 256;
constexpr int kGemvThreads = 2 * kGemvRows;
constexpr int kStages = 3;

template <int NT, bool kNF4>
__host__ __device__ constexpr size_t gemv_fixed_smem() {
  return (size_t)(kGemvThreads / 32) * kStages * kStageBytes + (kNF4 ? 256 * 32 * 4 : 0);
}

template <int NT, bool kNF4, bool kWide, bool kRes>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_kernel(GemvArgs p, Nf4Table tab) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int kTok = 8 * NT;
  const int kc = p.kc;
  // weight rings first (16-byte copies need 16-byte slots), then the
  // lookup table (NF4), x, its group sums (INT4), the reduction buffer
  uint8_t* rings = smem;
  uint8_t* cursor = smem + (size_t)(kGemvThreads / 32) * kStages * kStageBytes;
  uint32_t* lut = nullptr;
  if (kNF4) {
    lut = reinterpret_cast<uint32_t*>(cursor);
    cursor += 256 * 32 * 4;
  }
  uint16_t* xs = reinterpret_cast<uint16_t*>(cursor);
  cursor += (size_t)kTok * kc * 2;
  float* xsum = nullptr;
  if (!kNF4) {
    xsum = reinterpret_cast<float*>(cursor);
    cursor += (size_t)kTok * (kc / 64) * 4;
  }
  float* red = reinterpret_cast<float*>(cursor);
  __shared__ float tok_inv[16];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)blockIdx.x;  // == cluster rank (the cluster spans gridDim.x)
  const int u0 = (int)((int64_t)rank * p.units / p.S);
  const int u1 = (int)((int64_t)(rank + 1) * p.units / p.S);
  const int k0 = u0 * 128;
  const int klen = (u1 - u0) * 128;
  const int row_tile = (int)blockIdx.y * kGemvRows;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = row_tile + warp * 16;
  const bool active = n0 < p.N;
  const int nA = n0 + g, nB = n0 + g + 8;
  const int ng = p.K / p.G;

  // Programmatic dependent launch: a following kernel launched with the
  // attribute may start its own weight stream while this one finishes (it
  // waits for this grid before it reads x); this grid in turn starts its
  // weight stream before waiting for the preceding kernel, whose output may
  // be x. (The correction variants keep their own order: they may run as the
  // dependent of the channel selection, which only reads x, and wait before
  // their epilogue reads the selected channels.)
  if constexpr (!kRes) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- the first kStages - 1 weight stages of this warp (and their
  // parameters): one copy group per stage, committed by every thread (empty
  // for inactive warps and beyond the last stage) so that group counts agree
  const int64_t row_bytes = (int64_t)p.K / 2;
  const int nunits = u1 - u0;
  const int nst = (nunits + 1) / 2;
  uint8_t* wring = rings + (size_t)warp * kStages * kStageBytes;
  const uint8_t* wtile = p.qw + (int64_t)(active ? n0 : 0) * row_bytes;
  StagePrm sp[kStages];
  auto issue = [&](int j, StagePrm& prm, uint8_t* slot) {
    const bool one = 2 * j + 1 >= nunits;
    issue_stage<kWide>(slot, wtile, row_bytes, u0 + 2 * j, one, lane);
    load_unit_prm<kNF4, kWide>(prm.prm[0], prm.zz[0], u0 + 2 * j, nA, nB, p, ng);
    if (!one) load_unit_prm<kNF4, kWide>(prm.prm[1], prm.zz[1], u0 + 2 * j + 1, nA, nB, p, ng);
  };
#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (active && i < nst) issue(i, sp[i], wring + i * kStageBytes);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  // ---- x[:, k0 : k0+klen) -> shared memory, as 16-byte asynchronous copies
  // (after the preceding grid, which may have written x, has completed). Only
  // the M real tokens are copied: a padding token's MMA column never reaches
  // an output.
  if constexpr (!kRes) asm volatile("griddepcontrol.wait;" ::: "memory");
  const int kchunks = klen / 8;  // a multiple of 16
  const uint32_t cmagic = div_magic((uint32_t)kchunks);
  for (int c = tid; c < p.M * kchunks; c += blockDim.x) {
    const int gt = div_by_magic(c, cmagic), cl = c - gt * kchunks;
    int pc = cl ^ (gt & 1);
    if (kWide) pc ^= (cl >> 2) & 2;
    cp_async16(xs + (size_t)gt * kc + pc * 8, p.x + (size_t)gt * p.K + k0 + cl * 8);
  }
  // every copy issued so far (x and the first weight stages) has landed
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  if (!kNF4) {
    // In place, chunk by chunk: sums of x per 64- (8-byte layout) or 128-wide (16-byte layout)
    // sub-group, and the (k, k + 4) pairing of the INT4 nibbles. The chunks of
    // one sub-group sit in 8 or 16 consecutive lanes; the loop runs whole
    // warps (bound rounded up to 32) for the shuffles.
    const int nchunks = p.M * kchunks;
    for (int c = tid; c < ((nchunks + 31) & ~31); c += blockDim.x) {
      const bool real = c < nchunks;
      const int gt = div_by_magic(c, cmagic), cl = c - gt * kchunks;
      int pc = cl ^ (gt & 1);
      if (kWide) pc ^= (cl >> 2) & 2;
      uint4* slot = reinterpret_cast<uint4*>(xs + (size_t)gt * kc + pc * 8);
      uint4 v = real ? *slot : make_uint4(0, 0, 0, 0);
      float sm = 0.0f;
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) sm += bf16_lo_to_f32(w[q]) + bf16_hi_to_f32(w[q]);
      sm += __shfl_xor_sync(0xffffffffu, sm, 1);
      sm += __shfl_xor_sync(0xffffffffu, sm, 2);
      sm += __shfl_xor_sync(0xffffffffu, sm, 4);
      if (kWide) {
        sm += __shfl_xor_sync(0xffffffffu, sm, 8);
        if (real && (cl & 15) == 0) xsum[(cl >> 4) * kTok + gt] = sm;
      } else {
        if (real && (cl & 7) == 0) xsum[(cl >> 3) * kTok + gt] = sm;
      }
      if (real)
        *slot = make_uint4(prmt(v.x, v.z, 0x5410u), prmt(v.x, v.z, 0x7632u),
                           prmt(v.y, v.w, 0x5410u), prmt(v.y, v.w, 0x7632u));
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
    // per token: x chunk -> fp16 * 2^e in place (the swizzle moves whole
    // chunks); warp gt converts token gt (the max is a warp reduction)
    if (warp < kTok) {
      const int gt = warp, j = lane;
      uint16_t* row = xs + (size_t)gt * kc;
      float mx = 0.0f;
      for (int c = j; c < kchunks; c += 32) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + c * 8);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          mx = fmaxf(mx, fmaxf(fabsf(bf16_lo_to_f32(w[i])), fabsf(bf16_hi_to_f32(w[i]))));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      int e = 0;
      if (mx > 0.0f && mx <= 3.0e38f) {
        e = 14 - ((int)((__float_as_uint(mx) >> 23) & 0xFF) - 127);
        e = e > 100 ? 100 : (e < -100 ? -100 : e);
      }
      const float sc = __uint_as_float((uint32_t)(127 + e) << 23);
      if (j == 0) tok_inv[gt] = __uint_as_float((uint32_t)(127 - e) << 23);
      for (int c = j; c < kchunks; c += 32) {
        uint4 v = *reinterpret_cast<const uint4*>(row + c * 8);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          w[i] = pack_f16x2(bf16_lo_to_f32(w[i]) * sc, bf16_hi_to_f32(w[i]) * sc);
        *reinterpret_cast<uint4*>(row + c * 8) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    __syncthreads();
  }

  // ---- main loop: warp owns 16 weight rows over this CTA's K-chunk --------
  float acc[NT][4];
#pragma unroll
  for (int a = 0; a < NT; ++a)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[a][r] = 0.0f;

  const uint32_t* lut_lane = kNF4 ? lut + lane : nullptr;
  for (int jb = 0; jb < nst; jb += kStages) {
#pragma unroll
    for (int i = 0; i < kStages; ++i) {
      const int j = jb + i;
      if (j < nst) {
        // stage j + kStages - 1 goes into the slot stage j - 1 left
        const int kNext = (i + kStages - 1) % kStages;  // a constant once unrolled
        if (active && j + kStages - 1 < nst)
          issue(j + kStages - 1, sp[kNext], wring + kNext * kStageBytes);
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group %0;" ::"n"(kStages - 1) : "memory");
        __syncwarp();  // every lane's copies of stage j are visible to the warp
        if (active) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int lu = 2 * j + h;
            if (lu < nunits) {
              Unit U;
              read_unit<kWide>(U, wring + i * kStageBytes, h, g, t);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                U.prm[q] = sp[i].prm[h][q];
                U.zz[q] = sp[i].zz[h][q];
              }
              compute_unit<NT, kNF4, kWide>(U, lu, xs, kc, xsum, lut_lane, g, t, acc);
            }
          }
        }
        __syncwarp();  // stage j's slot is refilled in the next iteration
      }
    }
  }

  // ---- cluster split-K reduction (through distributed shared memory) -----
  reduce_and_store<NT, kRes, kGemvRows>(acc, kNF4 ? tok_inv : nullptr, red, p.S, rank, row_tile,
                                        p.M, p.N, p.y, p.rc);
}

template <int NT, bool kNF4>
size_t gemv_smem(int kc, int S) {
  return gemv_fixed_smem<NT, kNF4>() + (size_t)8 * NT * kc * 2 + red_bytes<kGemvRows>(S) +
         (kNF4 ? 0 : (size_t)8 * NT * (kc / 64) * 4);
}

template <int NT, bool kNF4, bool kWide, bool kRes>
wq_status launch_t(GemvArgs a, cudaStream_t st, bool early = false) {
  auto kern = gemv_kernel<NT, kNF4, kWide, kRes>;
  const int M = a.M;
  const Plan pl = cached_plan(reinterpret_cast<const void*>(kern), M, a.N, a.K, 0, [&] {
    return make_plan(
        kern, kGemvThreads, a.N, a.K,
        [&](int kc) { return gemv_smem<NT, kNF4>(kc, kMaxSplit) <= kMaxSmemBytes; },
        [&](int kc, int S) { return gemv_smem<NT, kNF4>(kc, S); }, false, kGemvRows);
  });
  if (pl.S < 1) return WQ_ERR_UNSUPPORTED;
  a.S = pl.S;
  a.kc = pl.kc;
  // the plain GEMV is always launched as a programmatic dependent (see the
  // kernel); the correction variants only when asked (after the selection)
  return launch_split(kern, pl, kGemvThreads, a.N, st, a, nf4_table(), false, kRes ? early : true,
                      kGemvRows);
}

}  // namespace

wq_status launch_gemv(const void* x, int64_t M, int64_t N, int64_t K, wq_format fmt, int32_t group,
                      const void* qweight, const void* scales, const void* zeros, void* y,
                      cudaStream_t st, const void* residual_t, const int32_t* idx, int32_t k,
                      bool early) {
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
  a.gmagic = div_magic((uint32_t)(group / 64));
  if (k > 0) {
    a.rc.rt = static_cast<const uint16_t*>(residual_t);
    a.rc.idx = idx;
    a.rc.x = a.x;
    a.rc.k = k;
    a.rc.K = (int)K;
  }
  const bool res = k > 0;
  if (fmt == WQ_FMT_NF4) {
    if (res)
      return NT == 1 ? launch_t<1, true, false, true>(a, st, early)
                     : launch_t<2, true, false, true>(a, st, early);
    return NT == 1 ? launch_t<1, true, false, false>(a, st)
                   : launch_t<2, true, false, false>(a, st);
  }
  if (group % 128 == 0) {
    if (res)
      return NT == 1 ? launch_t<1, false, true, true>(a, st, early)
                     : launch_t<2, false, true, true>(a, st, early);
    return NT == 1 ? launch_t<1, false, true, false>(a, st) : launch_t<2, false, true, false>(a, st);
  }
  if (res)
    return NT == 1 ? launch_t<1, false, false, true>(a, st, early)
                   : launch_t<2, false, false, true>(a, st, early);
  return NT == 1 ? launch_t<1, false, false, false>(a, st) : launch_t<2, false, false, false>(a, st);
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
