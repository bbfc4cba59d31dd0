// NF4 weights on the Multi-Scale Dequant path (decode, 1 <= M <= 16).
//
// Sources: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
// Activation Decomposition for Efficient LLM Inference", Abstract (integer
// activation digits multiply the quantized weights directly); "Fast NF4
// Dequantization Kernels for Large Language Model Inference", Abstract (NF4:
// 4-bit codes into a 16-value codebook, one fp32 absmax per 64-element block).
//
// The pages give MSD for integer weights; NF4 codes index real codebook
// values. Reading: the 16 code values become integers c_int = rint(c * 2^13)
// (within 2^-14 of c), split into two signed 8-bit digits c_int = 128 h + l
// (l in [-64, 63], h in [-64, 64]). Then, with the MSD activation digits
// a_c and scales s_c,
//   y[m, n] = sum_c s_c[m] sum_blk absmax[n, blk] 2^-13
//             * sum_{k in blk} a_c[m, k] (128 h[q] + l[q])
// where the inner sums are exact int32 tensor-core sums (s8 x s8) and each
// 64-element block's absmax is applied after its sum (as MixPE applies group
// scales: "MixPE: Quantization and Hardware Co-design for Efficient LLM
// Inference", Abstract). No weight is converted to floating point.
//
// B200 design: the split-K cluster GEMV structure of the other decode
// kernels (128 weight rows per CTA, K split over the cluster, each warp's 16
// rows streamed through a cp.async ring of 128-byte row segments, partials
// reduced through distributed shared memory), with warp-level
// mma.m16n8k32 s8 x s8 -> s32. Each MMA's k = 32 lies in one absmax block.
// Four NF4 nibbles become their four h bytes and four l bytes with byte
// permutes from register-held tables (no memory lookups): one permute per
// table half indexed by the nibbles' low 3 bits, one more choosing the half
// by bit 3. NF4 packs element 2j in the HIGH nibble, so a 16-bit group of
// codes yields the elements in the order 1, 0, 3, 2; the staged activation
// digits are swapped pairwise to the same order (the MMA only needs both
// operands in the same k order).
#include "splitk_common.cuh"

namespace wq {
namespace {

using namespace splitk;

constexpr int kNf4Stages = 3;
constexpr int kMaxNf4ChunkBytes = 64 * 1024;  // digit planes of one CTA's K-chunk

struct MsdNf4Args {
  const int8_t* planes;  // [C][plane_rows][K]
  int64_t plane_rows;
  const float* cs;       // [C][M]
  const uint8_t* codes;  // [N][K/2] NF4 codes, element 2j in the high nibble
  const float* absmax;   // [N][K/64]
  uint16_t* y;
  int M, N, K;
  int units;             // K / 256 (one weight stage each)
  int S, kc;
  uint32_t h_tab[4], l_tab[4];  // the h and l digit bytes of codes 0..15
};

__device__ __forceinline__ void mma_s8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 4-bit codes (nibbles of the low 16 bits of n) -> their four digit
// bytes from the 16-byte table t[0..3] (byte i of the result = entry of
// nibble i).
__device__ __forceinline__ uint32_t nib_lookup(uint32_t n, const uint32_t (&t)[4], uint32_t lo3,
                                               uint32_t sel) {
  const uint32_t a = prmt(t[0], t[1], lo3);   // entries 0..7
  const uint32_t b = prmt(t[2], t[3], lo3);   // entries 8..15
  return prmt(a, b, sel);                     // byte i from a or b by bit 3 of nibble i
}

// Weight stage: the warp's 16 rows x 128 bytes (256 codes, 4 absmax blocks);
// 16-byte chunk c of row r stored at chunk c ^ (r & 7).
__device__ __forceinline__ void nf4_issue_stage(uint8_t* slot, const uint8_t* wtile,
                                                int64_t row_bytes, int stage, int lane) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q = 32 * i + lane, r = q >> 3, c = q & 7;
    cp_async16(slot + r * kStageRowBytes + ((c ^ (r & 7)) << 4),
               wtile + (int64_t)r * row_bytes + (int64_t)stage * 128 + 16 * c);
  }
}

// Data placement per CTA (dynamic shared memory):
//   ring [8 warps][kNf4Stages][16 rows][128 B]  weight stages
//   pl   [C][M][Kc] int8 digits, adjacent bytes swapped; 16-byte chunk c of
//        token m at c ^ 2(m & 3)
//   red  [S ranks][ceil(128/S)][16] fp32
template <int NT, int C>
__global__ void __launch_bounds__(256, 2) msd_nf4_gemv_kernel(MsdNf4Args p, Nf4Table) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int kc = p.kc, M = p.M;
  uint8_t* rings = smem;
  uint8_t* pl = smem + (size_t)8 * kNf4Stages * kStageBytes;
  float* red = reinterpret_cast<float*>(pl + (size_t)C * M * kc);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)blockIdx.x;
  const int u0 = (int)((int64_t)rank * p.units / p.S);
  const int u1 = (int)((int64_t)(rank + 1) * p.units / p.S);
  const int nst = u1 - u0;
  const int k0 = u0 * 256, klen = nst * 256;
  const int row_tile = (int)blockIdx.y * kRowsPerCta;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = row_tile + warp * 16;
  const bool active = n0 < p.N;
  const int64_t row_bytes = p.K / 2;
  const int nblk = p.K / 64;

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- the first weight stages and their absmax (4 blocks of rows g, g + 8)
  uint8_t* wring = rings + (size_t)warp * kNf4Stages * kStageBytes;
  const uint8_t* wtile = p.codes + (int64_t)(active ? n0 : 0) * row_bytes;
  const float* amA = p.absmax + (int64_t)(active ? n0 + g : 0) * nblk;
  const float* amB = amA + 8 * (int64_t)nblk;
  float4 am[kNf4Stages][2];
  auto issue = [&](int j, float4 (&a)[2], uint8_t* slot) {
    nf4_issue_stage(slot, wtile, row_bytes, u0 + j, lane);
    a[0] = __ldg(reinterpret_cast<const float4*>(amA + (u0 + j) * 4));
    a[1] = __ldg(reinterpret_cast<const float4*>(amB + (u0 + j) * 4));
  };
#pragma unroll
  for (int i = 0; i < kNf4Stages - 1; ++i) {
    if (active && i < nst) issue(i, am[i], wring + i * kStageBytes);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  // ---- the digit planes of this K-chunk, once the decomposition is done
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int kch = klen / 16;
  for (int c = tid; c < C * M * kch; c += blockDim.x) {
    const int cm = c / kch, cl = c - cm * kch;
    const int m = cm % M;
    cp_async16(pl + (size_t)cm * kc + ((cl ^ (2 * (m & 3))) << 4),
               p.planes + ((int64_t)(cm / M) * p.plane_rows + m) * p.K + k0 + cl * 16);
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  // swap adjacent digit bytes (the order four NF4 nibbles decode in)
  for (int c = tid; c < C * M * kch * 4; c += blockDim.x) {
    const int cm = c / (kch * 4), wi = c - cm * (kch * 4);
    uint32_t* wp = reinterpret_cast<uint32_t*>(pl + (size_t)cm * kc) + wi;
    *wp = prmt(*wp, 0u, 0x2301u);
  }
  __syncthreads();

  int brow[NT], tokc[NT][2];
  float sc[C][NT][2];
#pragma unroll
  for (int a = 0; a < NT; ++a) {
    brow[a] = (g + 8 * a < M) ? g + 8 * a : 0;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      tokc[a][e] = min(8 * a + 2 * t + e, M - 1);
#pragma unroll
      for (int c = 0; c < C; ++c) sc[c][a][e] = p.cs[c * M + tokc[a][e]];
    }
  }
  const uint32_t h_tab[4] = {p.h_tab[0], p.h_tab[1], p.h_tab[2], p.h_tab[3]};
  const uint32_t l_tab[4] = {p.l_tab[0], p.l_tab[1], p.l_tab[2], p.l_tab[3]};

  float acc[NT][4];
#pragma unroll
  for (int a = 0; a < NT; ++a)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[a][r] = 0.0f;

  for (int jb = 0; jb < nst; jb += kNf4Stages) {
#pragma unroll
    for (int i = 0; i < kNf4Stages; ++i) {
      const int j = jb + i;
      if (j < nst) {
        const int kNext = (i + kNf4Stages - 1) % kNf4Stages;  // a constant once unrolled
        if (active && j + kNf4Stages - 1 < nst)
          issue(j + kNf4Stages - 1, am[kNext], wring + kNext * kStageBytes);
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group %0;" ::"n"(kNf4Stages - 1) : "memory");
        __syncwarp();
        if (active) {
          const uint8_t* slot = wring + i * kStageBytes;
          const float amA4[4] = {am[i][0].x, am[i][0].y, am[i][0].z, am[i][0].w};
          const float amB4[4] = {am[i][1].x, am[i][1].y, am[i][1].z, am[i][1].w};
#pragma unroll
          for (int blk = 0; blk < 4; ++blk) {
            int P[C][NT][2][4];  // [plane][token tile][h, l][entry]
#pragma unroll
            for (int c = 0; c < C; ++c)
#pragma unroll
              for (int a = 0; a < NT; ++a)
#pragma unroll
                for (int d = 0; d < 2; ++d)
#pragma unroll
                  for (int r = 0; r < 4; ++r) P[c][a][d][r] = 0;
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) {
              const int ks = 2 * blk + hs;  // 32-code k-step within the stage
              // this lane's 8 codes (word t of chunk ks) of rows g and g + 8
              const uint32_t wa = *reinterpret_cast<const uint32_t*>(
                  slot + g * kStageRowBytes + ((ks ^ (g & 7)) << 4) + 4 * t);
              const uint32_t wb = *reinterpret_cast<const uint32_t*>(
                  slot + (g + 8) * kStageRowBytes + ((ks ^ (g & 7)) << 4) + 4 * t);
              uint32_t ah[4], al[4];
              const uint32_t src[4] = {wa, wb, wa >> 16, wb >> 16};  // a0 a1 a2 a3
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint32_t n16 = src[q] & 0xFFFFu;
                const uint32_t lo3 = n16 & 0x7777u;
                const uint32_t sel = 0x3210u | ((n16 >> 1) & 0x4444u);
                ah[q] = nib_lookup(n16, h_tab, lo3, sel);
                al[q] = nib_lookup(n16, l_tab, lo3, sel);
              }
              const int lk = j * 256 + ks * 32;  // k within the chunk
#pragma unroll
              for (int c = 0; c < C; ++c)
#pragma unroll
                for (int a = 0; a < NT; ++a) {
                  const int bt = brow[a];
                  const uint2 xv = *reinterpret_cast<const uint2*>(
                      pl + ((size_t)c * M + bt) * kc +
                      ((((lk >> 4) + (t >> 1)) ^ (2 * (bt & 3))) << 4) + 8 * (t & 1));
                  mma_s8s8(P[c][a][0], ah[0], ah[1], ah[2], ah[3], xv.x, xv.y);
                  mma_s8s8(P[c][a][1], al[0], al[1], al[2], al[3], xv.x, xv.y);
                }
            }
            // the block's integer sums, scaled by its absmax and the planes'
            // scales (2^-13 is applied at the end)
#pragma unroll
            for (int a = 0; a < NT; ++a)
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                float v = 0.0f;
#pragma unroll
                for (int c = 0; c < C; ++c)
                  v = fmaf(sc[c][a][r & 1], (float)(128 * P[c][a][0][r] + P[c][a][1][r]), v);
                acc[a][r] = fmaf((r < 2 ? amA4 : amB4)[blk], v, acc[a][r]);
              }
          }
        }
        __syncwarp();
      }
    }
  }
#pragma unroll
  for (int a = 0; a < NT; ++a)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[a][r] *= 1.0f / 8192.0f;

  reduce_and_store<NT>(acc, nullptr, red, p.S, rank, row_tile, M, p.N, p.y);
}

template <int NT, int C>
size_t nf4_smem(int kc, int S, int M) {
  return (size_t)8 * kNf4Stages * kStageBytes + (size_t)C * M * kc + red_bytes(S);
}

template <int NT, int C>
wq_status launch_nf4_t(MsdNf4Args a, cudaStream_t st) {
  auto kern = msd_nf4_gemv_kernel<NT, C>;
  // the planner splits K in units of 128; this kernel's stages are 256 k
  const Plan pl = cached_plan(reinterpret_cast<const void*>(kern), a.M, a.N, a.K, 16 + C, [&] {
    return make_plan(
        kern, 256, a.N, a.K / 2,
        [&](int kc) { return (int64_t)C * a.M * 2 * kc <= kMaxNf4ChunkBytes; },
        [&](int kc, int S) { return nf4_smem<NT, C>(2 * kc, S, a.M); });
  });
  if (pl.S < 1) return WQ_ERR_UNSUPPORTED;
  a.S = pl.S;
  a.kc = 2 * pl.kc;
  return launch_split(kern, pl, 256, a.N, st, a, nf4_table(), false, /*early=*/true);
}

template <int NT>
wq_status launch_nf4_nt(const MsdNf4Args& a, int C, cudaStream_t st) {
  switch (C) {
    case 1: return launch_nf4_t<NT, 1>(a, st);
    case 2: return launch_nf4_t<NT, 2>(a, st);
    default: return launch_nf4_t<NT, 3>(a, st);
  }
}

// The h and l digit bytes of the 16 NF4 code values: c_int = rint(c 2^13) =
// 128 h + l, l in [-64, 63] (host; from the library's own codebook).
void nf4_digit_tables(uint32_t (&h)[4], uint32_t (&l)[4]) {
  const Nf4Table& tb = nf4_table();
  for (int w = 0; w < 4; ++w) h[w] = l[w] = 0u;
  for (int i = 0; i < 16; ++i) {
    const long ci = lrint((double)tb.v[i] * 8192.0);
    const long hi = (long)floor((double)(ci + 64) / 128.0);
    const long lo = ci - 128 * hi;
    h[i / 4] |= ((uint32_t)(uint8_t)(int8_t)hi) << (8 * (i % 4));
    l[i / 4] |= ((uint32_t)(uint8_t)(int8_t)lo) << (8 * (i % 4));
  }
}

}  // namespace

wq_status launch_msd_decompose(const void*, int64_t, int64_t, int32_t, int64_t, int8_t*, float*,
                               cudaStream_t);
size_t msd_workspace_bytes(int64_t M, int64_t K, int32_t C);

wq_status launch_msd_nf4(const void* x, int64_t M, int64_t N, int64_t K, int32_t C,
                         const uint8_t* codes, const float* absmax, void* y, void* workspace,
                         cudaStream_t st) {
  int8_t* planes = static_cast<int8_t*>(workspace);
  // the digit planes hold M rows (the layout the decomposition writes with
  // plane_rows = M); the scales follow the padded size the workspace has
  const size_t planes_bytes = ((size_t)C * ((M + 127) / 128 * 128) * K + 255) / 256 * 256;
  float* cs = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + planes_bytes);
  wq_status s = launch_msd_decompose(x, M, K, C, M, planes, cs, st);
  if (s != WQ_OK) return s;
  MsdNf4Args a;
  a.planes = planes;
  a.plane_rows = M;
  a.cs = cs;
  a.codes = codes;
  a.absmax = absmax;
  a.y = static_cast<uint16_t*>(y);
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.units = (int)(K / 256);
  a.S = 1;
  a.kc = 0;
  nf4_digit_tables(a.h_tab, a.l_tab);
  return M <= 8 ? launch_nf4_nt<1>(a, C, st) : launch_nf4_nt<2>(a, C, st);
}

}  // namespace wq
