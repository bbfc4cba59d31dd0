// Multi-Scale Dequant GEMV for decode (1 <= M <= 16).
//
// Source: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
// Activation Decomposition for Efficient LLM Inference", Abstract: the
// activations are split into C int8 components so that the integer weights
// enter the multiply directly; group scale and zero per "MixPE: Quantization
// and Hardware Co-design for Efficient LLM Inference", Abstract (applied after
// the group's integer sum).
//
// Per 128-k unit u (the groups are multiples of 128, so one group spans the
// unit), row n, token m and component c:
//   P_c = sum_k a_c[m, k] * q[n, k]            (u8 x s8 -> s32, exact)
//   R_c = sum_k a_c[m, k]                      (s32, per token and unit)
//   y[m, n] += s[n, g] * sum_c s_c[m] * (P_c - z[n, g] * R_c)
// For C = 2 the components combine exactly in int32 first: s_1 d_1 + s_2 d_2
// = s_2 (256 d_1 + d_2) with d_c = P_c - z R_c (s_2 = s_1 / 256 exactly), and
// |256 d_1 + d_2| <= 257 * 127 * 15 * 128 < 2^31.
//
// B200 design: the split-K cluster structure of the W4A16 GEMV (one 128-row
// weight tile per CTA, K split over the cluster, partials reduced through
// distributed shared memory), with the product on warp-level
// mma.m16n8k32.u8.s8: weight rows are the A operand (nibbles -> u8 by one
// AND, no zero subtraction), digit planes the B operand. Each lane reads 16
// bytes of each of its two rows per unit (k = 32t .. 32t + 31); its AND-ed
// low nibbles are k + {0,2,4,6} and high nibbles k + {1,3,5,7} of every
// 8-element group, so the planes are staged with the even-k bytes of each
// group first, then the odd-k bytes.
//
// It is launched as a programmatic dependent of the decomposition kernel: its
// first weight loads overlap the decomposition, and it waits for it only
// before it reads the digit planes.
//
// Data placement per CTA (dynamic shared memory):
//   pl   [C][M][Kc] int8, the CTA's K-chunk of the digit planes; 16-byte chunk
//        c of token m at chunk c ^ (m & 1) (conflict-free fragment loads)
//   rs   [C][Kc/128][8*NT] int32, R_c per unit and token
//   red  [S ranks][ceil(128/S) rows][16 tokens] fp32, the split-K partials
#include "splitk_common.cuh"

namespace wq {
namespace {

using namespace splitk;

constexpr int kMaxPlaneChunkBytes = 64 * 1024;

struct MsdArgs {
  const int8_t* planes;  // [C][plane_rows][K]
  int64_t plane_rows;
  const float* cs;       // [C][M] component scales
  const uint8_t* qw;     // INT4 words viewed as bytes, [N][K/2]
  const __half* scales;  // [N][K/G]
  const __half* zeros;   // [N][K/G]
  uint16_t* y;
  int M, N, K, G, C;
  int units;             // K / 128
  int S;                 // cluster size along K
  int kc;                // shared-memory K-chunk length (max over ranks)
  uint32_t umagic;       // u / (G / 128) == umulhi(u, umagic); 0 if G == 128
};

__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 128-k unit of this lane's rows g and g + 8: w[0..3] = 16 bytes of row g
// at byte 16t, w[4..7] the same of row g + 8; prm[0..1] = the fp16 scale bits
// of rows g, g + 8 and prm[2..3] their zero bits, kept as loaded (no
// arithmetic on them before the unit is computed, so their loads never stall
// a warp still issuing its first units).
struct MsdUnit {
  uint32_t w[8];
  uint32_t prm[4];
};

__device__ __forceinline__ void msd_load_unit(MsdUnit& U, const uint8_t* wA, const uint8_t* wB,
                                              int u, int nA, int nB, const MsdArgs& p, int ng) {
  const int64_t off = (int64_t)u * 64;
  const uint4 a = ld_stream_u4(wA + off), b = ld_stream_u4(wB + off);
  U.w[0] = a.x; U.w[1] = a.y; U.w[2] = a.z; U.w[3] = a.w;
  U.w[4] = b.x; U.w[5] = b.y; U.w[6] = b.z; U.w[7] = b.w;
  const int gi = div_by_magic(u, p.umagic);
  const unsigned short* s16 = reinterpret_cast<const unsigned short*>(p.scales);
  const unsigned short* z16 = reinterpret_cast<const unsigned short*>(p.zeros);
  const int64_t iA = (int64_t)nA * ng + gi, iB = (int64_t)nB * ng + gi;
  U.prm[0] = __ldg(s16 + iA);
  U.prm[1] = __ldg(s16 + iB);
  U.prm[2] = __ldg(z16 + iA);
  U.prm[3] = __ldg(z16 + iB);
}

template <int NT>
struct MsdTraits {
  static constexpr int D = NT == 1 ? 4 : 3;  // units in flight per warp
};

template <int NT>
size_t msd_smem(int kc, int S, int M, int C) {
  // planes, digit sums, two partial buffers (alternating row tiles)
  return (size_t)C * M * kc + (size_t)C * (kc / 128) * 8 * NT * 4 + 2 * red_bytes(S);
}

template <int NT, int C>
__global__ void __launch_bounds__(256, 2) msd_gemv_kernel(MsdArgs p, Nf4Table) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int kTok = 8 * NT;
  constexpr int D = MsdTraits<NT>::D;
  const int kc = p.kc, M = p.M;
  const int upc = kc / 128;  // units per K-chunk
  int8_t* pl = reinterpret_cast<int8_t*>(smem);
  int* rs = reinterpret_cast<int*>(smem + (size_t)C * M * kc);
  float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(rs) + (size_t)C * upc * kTok * 4);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)blockIdx.x;  // == cluster rank (the cluster spans gridDim.x)
  const int u0 = (int)((int64_t)rank * p.units / p.S);
  const int u1 = (int)((int64_t)(rank + 1) * p.units / p.S);
  const int k0 = u0 * 128;
  const int klen = (u1 - u0) * 128;
  const int g = lane >> 2, t = lane & 3;
  const int ng = p.K / p.G;
  const int tiles = (p.N + kRowsPerCta - 1) / kRowsPerCta;
  // Persistent over row tiles: this cluster takes tiles blockIdx.y,
  // blockIdx.y + gridDim.y, ...; the digit planes of its K-chunk are staged
  // and prepared once. Per tile: the warp's 16 rows and their weight rows.
  int tile = (int)blockIdx.y;
  int row_tile = tile * kRowsPerCta;
  int n0 = row_tile + warp * 16;
  bool active = n0 < p.N;
  int nA = n0 + g, nB = n0 + g + 8;

  // Programmatic dependent launch: this grid starts while the decomposition
  // that writes the digit planes and their scales may still run (its CTAs
  // release this grid at once); it issues its first weight units, then waits
  // for that grid before it reads the planes. It releases its own dependents
  // at once in turn.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- the first D units of weights of this warp
  const int64_t row_bytes = (int64_t)p.K / 2;
  const uint8_t* wrowA = p.qw + (int64_t)(active ? nA : 0) * row_bytes + 16 * t;
  const uint8_t* wrowB = wrowA + 8 * row_bytes;
  const float* red_buf[2] = {red, red + red_bytes(p.S) / 4};
  MsdUnit ring[D];
  if (active) {
#pragma unroll
    for (int i = 0; i < D; ++i)
      if (u0 + i < u1) msd_load_unit(ring[i], wrowA, wrowB, u0 + i, nA, nB, p, ng);
  }

  // ---- then the digit planes [C][M][k0 : k0+klen) -> shared memory
  // (16-byte copies), once the decomposition has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int kchunks = klen / 16;  // a multiple of 8
  const int per_plane = M * kchunks;
  const uint32_t mag_plane = div_magic((uint32_t)per_plane), mag_row = div_magic((uint32_t)kchunks);
  for (int i = tid; i < C * per_plane; i += blockDim.x) {
    const int c = div_by_magic(i, mag_plane), rem = i - c * per_plane;
    const int gt = div_by_magic(rem, mag_row), cl = rem - gt * kchunks;
    cp_async16(pl + ((size_t)c * M + gt) * kc + (cl ^ (gt & 1)) * 16,
               p.planes + ((int64_t)c * p.plane_rows + gt) * p.K + k0 + cl * 16);
  }
  cp_async_wait_all();
  __syncthreads();

  // In place, chunk by chunk: R_c per unit and token, and the even-k /
  // odd-k byte order within every 8-byte group. The 8 chunks of one unit sit
  // in 8 consecutive lanes; the loop runs whole warps for the shuffles.
  {
    const int total = C * per_plane;
    for (int i = tid; i < ((total + 31) & ~31); i += blockDim.x) {
      const bool real = i < total;
      const int c = real ? div_by_magic(i, mag_plane) : 0;
      const int rem = i - c * per_plane;
      const int gt = real ? div_by_magic(rem, mag_row) : 0;
      const int cl = rem - gt * kchunks;
      uint4* slot = reinterpret_cast<uint4*>(pl + ((size_t)c * M + gt) * kc + (cl ^ (gt & 1)) * 16);
      const uint4 v = real ? *slot : make_uint4(0, 0, 0, 0);
      int sm = __dp4a((int)v.x, 0x01010101, 0);
      sm = __dp4a((int)v.y, 0x01010101, sm);
      sm = __dp4a((int)v.z, 0x01010101, sm);
      sm = __dp4a((int)v.w, 0x01010101, sm);
      sm += __shfl_xor_sync(0xffffffffu, sm, 1);
      sm += __shfl_xor_sync(0xffffffffu, sm, 2);
      sm += __shfl_xor_sync(0xffffffffu, sm, 4);
      if (real && (cl & 7) == 0) rs[(c * upc + (cl >> 3)) * kTok + gt] = sm;
      if (real)
        *slot = make_uint4(prmt(v.x, v.y, 0x6420u), prmt(v.x, v.y, 0x7531u),
                           prmt(v.z, v.w, 0x6420u), prmt(v.z, v.w, 0x7531u));
    }
  }
  __syncthreads();

  // plane rows of this lane's B tokens (padding tokens read token 0's row:
  // their MMA columns never reach an output) and the component scales of its
  // accumulator tokens 8a + 2t + {0, 1}
  const int8_t* prow[C][NT];
  int psw[NT];
  float scl[C][NT][2];
#pragma unroll
  for (int a = 0; a < NT; ++a) {
    const int tr = (g + 8 * a < M) ? g + 8 * a : 0;
    psw[a] = tr & 1;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      prow[c][a] = pl + ((size_t)c * M + tr) * kc;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = 8 * a + 2 * t + e;
        scl[c][a][e] = tok < M ? p.cs[c * M + tok] : 0.0f;
      }
    }
  }

  for (int it = 0; tile < tiles; ++it) {
  // ---- main loop: warp owns 16 weight rows over this CTA's K-chunk --------
  float acc[NT][4];
#pragma unroll
  for (int a = 0; a < NT; ++a)
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[a][r] = 0.0f;

  if (active) {
    for (int ub = u0; ub < u1; ub += D) {
#pragma unroll
      for (int i = 0; i < D; ++i) {
        const int u = ub + i;
        if (u >= u1) continue;
        const int lu = u - u0;
        const MsdUnit& U = ring[i];
        int P[C][NT][4];
        uint4 X[C][NT][2];
#pragma unroll
        for (int c = 0; c < C; ++c)
#pragma unroll
          for (int a = 0; a < NT; ++a) {
#pragma unroll
            for (int r = 0; r < 4; ++r) P[c][a][r] = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h)
              X[c][a][h] = *reinterpret_cast<const uint4*>(
                  prow[c][a] + ((lu * 8 + 2 * t + h) ^ psw[a]) * 16);
          }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t a0 = U.w[ks] & 0x0F0F0F0Fu, a2 = (U.w[ks] >> 4) & 0x0F0F0F0Fu;
          const uint32_t a1 = U.w[4 + ks] & 0x0F0F0F0Fu, a3 = (U.w[4 + ks] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
          for (int c = 0; c < C; ++c)
#pragma unroll
            for (int a = 0; a < NT; ++a) {
              const uint4& xv = X[c][a][ks >> 1];
              const uint32_t b0 = (ks & 1) ? xv.z : xv.x;
              const uint32_t b1 = (ks & 1) ? xv.w : xv.y;
              mma_u8s8(P[c][a], a0, a1, a2, a3, b0, b1);
            }
        }
        // post-group scaling of this unit
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const float s = __half2float(__ushort_as_half((unsigned short)U.prm[hr]));
          const int z = (int)__half2float(__ushort_as_half((unsigned short)U.prm[2 + hr]));
#pragma unroll
          for (int a = 0; a < NT; ++a) {
            int2 R[C];
#pragma unroll
            for (int c = 0; c < C; ++c)
              R[c] = *reinterpret_cast<const int2*>(rs + (c * upc + lu) * kTok + 8 * a + 2 * t);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int r = 2 * hr + e;
              int d[C];
#pragma unroll
              for (int c = 0; c < C; ++c) d[c] = P[c][a][r] - z * (e ? R[c].y : R[c].x);
              if (C == 1) {
                acc[a][r] = fmaf(s * scl[0][a][e], (float)d[0], acc[a][r]);
              } else if (C == 2) {
                // s_1 d_1 + s_2 d_2 = s_2 (256 d_1 + d_2), with s_2 = s_1 / 256
                acc[a][r] = fmaf(s * scl[C - 1][a][e], (float)(256 * d[0] + d[1]), acc[a][r]);
              } else {
                float v = scl[0][a][e] * (float)d[0];
#pragma unroll
                for (int c = 1; c < C; ++c) v = fmaf(scl[c][a][e], (float)d[c], v);
                acc[a][r] = fmaf(s, v, acc[a][r]);
              }
            }
          }
        }
        // this slot's unit is consumed: refill it
        if (u + D < u1) msd_load_unit(ring[i], wrowA, wrowB, u + D, nA, nB, p, ng);
      }
    }
  }

  // every slot of the ring is consumed: start the next tile's weight stream
  // before this tile's reduction
  const int cur_row_tile = row_tile;
  tile += (int)gridDim.y;
  if (tile < tiles) {
    row_tile = tile * kRowsPerCta;
    n0 = row_tile + warp * 16;
    active = n0 < p.N;
    nA = n0 + g;
    nB = n0 + g + 8;
    wrowA = p.qw + (int64_t)(active ? nA : 0) * row_bytes + 16 * t;
    wrowB = wrowA + 8 * row_bytes;
    if (active) {
#pragma unroll
      for (int i = 0; i < D; ++i)
        if (u0 + i < u1) msd_load_unit(ring[i], wrowA, wrowB, u0 + i, nA, nB, p, ng);
    }
  }

  // ---- cluster split-K reduction (through distributed shared memory) -----
  // (the partial buffers alternate between tiles: the next tile's pushes
  // follow this tile's barrier, which the owner passes only after reading)
  reduce_and_store<NT>(acc, nullptr, const_cast<float*>(red_buf[it & 1]), p.S, rank,
                       cur_row_tile, M, p.N, p.y);
  }
}

template <int NT, int C>
wq_status launch_msd_t(MsdArgs a, cudaStream_t st) {
  auto kern = msd_gemv_kernel<NT, C>;
  const Plan pl = cached_plan(reinterpret_cast<const void*>(kern), a.M, a.N, a.K, C, [&] {
    return make_plan(
        kern, 256, a.N, a.K,
        [&](int kc) { return (int64_t)C * a.M * kc <= kMaxPlaneChunkBytes; },
        [&](int kc, int S) { return msd_smem<NT>(kc, S, a.M, C); }, /*persistent=*/true);
  });
  if (pl.S < 1) return WQ_ERR_UNSUPPORTED;
  a.S = pl.S;
  a.kc = pl.kc;
  // a programmatic dependent of the decomposition (see the kernel)
  return launch_split(kern, pl, 256, a.N, st, a, nf4_table(), /*persistent=*/true,
                      /*early=*/true);
}

template <int NT>
wq_status launch_msd_nt(const MsdArgs& a, cudaStream_t st) {
  switch (a.C) {
    case 1: return launch_msd_t<NT, 1>(a, st);
    case 2: return launch_msd_t<NT, 2>(a, st);
    default: return launch_msd_t<NT, 3>(a, st);
  }
}

}  // namespace

// Digit planes [C][plane_rows][K] int8 and component scales [C][M] fp32 as
// written by the decomposition; requires 1 <= M <= 16, G % 128 == 0.
wq_status launch_msd_gemv(const int8_t* planes, int64_t plane_rows, const float* comp_scales,
                          int64_t M, int64_t N, int64_t K, int32_t C, int32_t G,
                          const void* qweight, const void* scales, const void* zeros, void* y,
                          cudaStream_t st) {
  if (M < 1 || M > 16 || G % 128 != 0 || C < 1 || C > 3) return WQ_ERR_UNSUPPORTED;
  MsdArgs a;
  a.planes = planes;
  a.plane_rows = plane_rows;
  a.cs = comp_scales;
  a.qw = static_cast<const uint8_t*>(qweight);
  a.scales = static_cast<const __half*>(scales);
  a.zeros = static_cast<const __half*>(zeros);
  a.y = static_cast<uint16_t*>(y);
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.G = G;
  a.C = C;
  a.units = (int)(K / 128);
  a.S = 1;
  a.kc = 0;
  a.umagic = div_magic((uint32_t)(G / 128));
  return M <= 8 ? launch_msd_nt<1>(a, st) : launch_msd_nt<2>(a, st);
}

}  // namespace wq
