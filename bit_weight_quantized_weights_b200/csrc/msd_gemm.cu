// Multi-Scale Dequant GEMM on the int8 tensor cores (tcgen05.mma kind::i8).
//
// Source: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
// Activation Decomposition for Efficient LLM Inference", Abstract: instead of
// lifting the low-bit weights to bf16, the bf16 activations are decomposed
// into low-precision components that multiply the quantized weights directly
// on the native integer GEMM hardware. The group's scale is applied after the
// group's integer sum ("MixPE: Quantization and Hardware Co-design for
// Efficient LLM Inference", Abstract).
//
//   y[m, n] = s_C[m] * sum_g s[n, g] * sum_c 256^(C-c) * P_c[m, n, g]
//   P_c[m, n, g] = sum_{k in g} a_c[m, k] * (q[n, k] - z[n, g])     (exact int32)
//
// (s_c = s_C * 256^(C-c) exactly, so the components combine as integers.)
// The zero point is folded into the 8-bit weight operand: q - z lies in
// [-15, 15], an exact signed byte; no weight is ever converted to floating
// point. The group sums of the digits are therefore not needed.
//
// B200 design (one 128-token x 128-feature tile per CTA, BK = 128 = one group
// of 128):
//   warp 0       TMA producer: the C digit-plane tiles (int8, 128-byte
//                swizzled) and the packed weight tile, STAGES-deep ring.
//   warp 1       TMEM owner; one lane issues C x 4 tcgen05.mma.kind::i8
//                (128 x 128 x 32, s8 x s8 -> s32) per k-tile into the group's
//                TMEM accumulators (C x 128 columns, double-buffered when they
//                fit), commits stages and finished groups. The unpacked
//                weights are the MMA's A operand (M = 128 features) and a
//                digit plane its B operand (N = 128 tokens), so a TMEM lane is
//                one feature and a column one token.
//   warps 2-5    unpack: low and high nibbles -> bytes (a mask and a shift
//                per 8 codes), minus the group's zero point per byte (one add
//                and one xor per 4 codes), into the UMMA K-major
//                128-byte-swizzled weight tile. The digit planes are written
//                in the same permuted k order (0, 2, 4, 6, 1, 3, 5, 7 in each
//                run of 8), so no byte permute is needed.
//   warps 6-13   drain each finished group from TMEM: combine the components
//                in int32, convert, scale by the group's s[n, g] (one value
//                per thread: its feature), accumulate in fp32 registers; the
//                last group scales by the tokens' s_C[m] and writes bf16 y
//                through a shared-memory transpose.
#include "sm100.cuh"
#include "splitk_common.cuh"

namespace wq {

__device__ unsigned int g_msd_error;

wq_status launch_msd_decompose(const void*, int64_t, int64_t, int32_t, int64_t, int8_t*, float*,
                               cudaStream_t);
wq_status launch_msd_decompose_nibble_order(const void*, int64_t, int64_t, int32_t, int64_t,
                                            int8_t*, float*, cudaStream_t);

namespace {

constexpr int BM = 128, BN = 128, BK = 128;
#ifndef MSD_DRAIN_WARPS
#define MSD_DRAIN_WARPS 8
#endif
constexpr int kUnpackWarps = 4;
// group-drain warps: kEpiWarps / 4 per TMEM lane quarter, each with an
// equal share of the 128 token columns. 8 (64 columns each) measured 4-6 %
// faster than 16 on B200: the drain is bound by issue slots it shares with
// the unpack warps, not by each warp's chain of TMEM loads.
constexpr int kEpiWarps = MSD_DRAIN_WARPS;
constexpr int kThreads = 64 + 32 * kUnpackWarps + 32 * kEpiWarps;
constexpr int kDrainCols = BM / (kEpiWarps / 4);  // token columns per drain warp
constexpr int kPlaneBytes = BM * BK;      // 16 KB per digit plane tile
constexpr int kBBytes = BN * BK;          // 16 KB
constexpr int kWBytes = BN * BK / 2;      // 8 KB packed
constexpr int kOutPitch = BN + 8;         // bf16 transpose tile row (16-byte rows, banks shifted)
constexpr int kRedPitch = BM + 4;         // fp32 split-K partial row (16-byte aligned)

inline int64_t m_padded(int64_t M) { return (M + 127) / 128 * 128; }

inline size_t planes_bytes(int64_t M, int64_t K, int C) {
  size_t b = (size_t)C * m_padded(M) * K;
  return (b + 255) / 256 * 256;
}

template <int C>
struct MsdCfg {
  static constexpr int kNB = (2 * C * BN <= 512) ? 2 : 1;  // TMEM accumulator buffers
  static constexpr int kTmemCols = (C * BN * kNB <= 256) ? 256 : 512;
  static constexpr int kStageBytes = C * kPlaneBytes + kBBytes + kWBytes;
  // 4 stages where they fit (C <= 2: 224 KB), else 3
  static constexpr int kStages = (4 * kStageBytes + 256 + 1024 <= 232448) ? 4 : 3;
  static constexpr int kSmem = kStages * kStageBytes + 256 + 1024;
  // the transpose tile and the split-K partials reuse the stage ring
  static_assert(kStages >= 2 && 3 * kStages + 2 * kNB + 1 <= 31, "stages and barriers");
  static_assert(kStages * kStageBytes >= BM * kOutPitch * 2, "transpose tile");
  // S ranks of ceil(128 / S) rows, S <= 8
  static_assert(kStages * kStageBytes >= (BN + 7) * kRedPitch * 4, "split-K partials");
};

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Packed fp32 pair arithmetic (sm_100 f32x2: each lane rounds as the scalar
// operation would).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// 8 INT4 codes of one packed word -> 8 signed bytes q - z, in the order the
// digit planes of this kernel use (codes 0, 2, 4, 6, then 1, 3, 5, 7: the low
// and the high nibbles of each byte). zc holds 128 - z in every byte: per
// byte 128 + q - z lies in [113, 143], so the add carries across no byte,
// and ^ 128 turns it into q - z as a two's-complement byte.
__device__ __forceinline__ uint2 unpack_word_minus_zero(uint32_t w, uint32_t zc) {
  return make_uint2(((w & 0x0F0F0F0Fu) + zc) ^ 0x80808080u,
                    (((w >> 4) & 0x0F0F0F0Fu) + zc) ^ 0x80808080u);
}

template <int C, bool kIntCombine, bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
    msd_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_w, const __half* __restrict__ scales,
                    const __half* __restrict__ zeros, const float* __restrict__ comp_scales,
                    uint16_t* __restrict__ y, int M, int N, int K, int G, int m_pad, int S,
                    WaitCtl wc) {
  using Cfg = MsdCfg<C>;
  constexpr int NB = Cfg::kNB;
  constexpr int kStages = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;                                  // [stage][plane] 16 KB
  uint8_t* sB = sA + kStages * C * kPlaneBytes;        // [stage] 16 KB
  uint8_t* sW = sB + kStages * kBBytes;                // [stage] 8 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sW + kStages * kWBytes);
  uint64_t* full = bars;
  uint64_t* deq = bars + kStages;
  uint64_t* empty = bars + 2 * kStages;
  uint64_t* acc_full = bars + 3 * kStages;
  uint64_t* acc_empty = acc_full + NB;
  uint64_t* mma_done = acc_empty + NB;  // the MMA issuer's final commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // split-K: cluster rank `rank` (of S along grid x) owns k-tiles [kt0, kt1)
  // (without kSplit the launch has S == 1; the constants let the compiler
  // keep the single-rank loops as simple as a kernel without the split)
  const int rank = kSplit ? (int)blockIdx.x : 0;
  // grid: (S, feature tiles, token tiles) with kSplit, else (feature tiles,
  // token tiles)
  const int n0 = (kSplit ? blockIdx.y : blockIdx.x) * BN;
  const int m0 = (kSplit ? blockIdx.z : blockIdx.y) * BM;
  const int KTA = K / BK;
  const int kt0 = kSplit ? (int)((int64_t)rank * KTA / S) : 0;
  const int kt1 = kSplit ? (int)((int64_t)(rank + 1) * KTA / S) : KTA;
  const int KT = kt1 - kt0;  // k-tiles of this rank
  const int TPG = G / BK;    // k-tiles per group
  const int NG = K / G;
  // the rank's k-tiles cut its groups into sub-groups g_first .. g_last
  const int g_first = kSplit ? kt0 / TPG : 0;
  const int NSG = kSplit ? (kt1 - 1) / TPG - g_first + 1 : NG;

  if (threadIdx.x == 0) {
    sm100::tma_prefetch_desc(&tmap_a);
    sm100::tma_prefetch_desc(&tmap_w);
    for (int s = 0; s < kStages; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&deq[s], kUnpackWarps);
      sm100::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NB; ++b) {
      sm100::mbar_init(&acc_full[b], 1);
      sm100::mbar_init(&acc_empty[b], kEpiWarps);
    }
    sm100::mbar_init(mma_done, 1);
    *abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc(tmem_slot, Cfg::kTmemCols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int last_issued = -1;  // producer: the last k-tile (of this rank) whose loads it issued
  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < KT; ++i) {
        const int kt = kt0 + i;
        const int s = i % kStages;
        const uint32_t ph = (uint32_t)(i / kStages) & 1u;
        if (i >= kStages &&
            !sm100::mbar_wait(&empty[s], ph ^ 1u, &g_msd_error, 0x1101u, abort_flag, wc.limit_ns))
          break;
        if (wc.stall && i == 0) continue;  // test hook: the first k-tile never arrives
        last_issued = i;
        sm100::mbar_arrive_expect_tx(&full[s], C * kPlaneBytes + kWBytes);
#pragma unroll
        for (int c = 0; c < C; ++c)
          sm100::tma_load_2d(sA + (s * C + c) * kPlaneBytes, &tmap_a, &full[s], kt * BK,
                             c * m_pad + m0);
        sm100::tma_load_2d(sW + s * kWBytes, &tmap_w, &full[s], kt * (BK / 8), n0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // the C plane tiles of a stage are adjacent 128-row K-major tiles, so
      // up to two planes form one N = 256 B operand: one MMA then reads the
      // weight tile for both (a 128-wide MMA costs ~85 % of a 256-wide one)
      constexpr int kPair = C >= 2 ? 2 : 1;
      constexpr uint32_t idesc_pair = sm100::idesc_s8_s32(BN, kPair * BM);
      constexpr uint32_t idesc_one = sm100::idesc_s8_s32(BN, BM);
      int i = 0;  // k-tiles consumed by this rank
      bool ok = true;
      for (int gi = 0; gi < NSG && ok; ++gi) {
        const int b = gi % NB;
        if (gi >= NB) {
          if (!sm100::mbar_wait(&acc_empty[b], (uint32_t)((gi / NB) - 1) & 1u, &g_msd_error,
                                0x1201u, abort_flag, wc.limit_ns)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
        }
        const int g = g_first + gi;
        const int sg0 = kSplit ? max(kt0, g * TPG) : g * TPG;
        const int sg1 = kSplit ? min(kt1, (g + 1) * TPG) : (g + 1) * TPG;
        for (int t = 0; t < sg1 - sg0; ++t, ++i) {
          const int s = i % kStages;
          const uint32_t ph = (uint32_t)(i / kStages) & 1u;
          if (!sm100::mbar_wait(&full[s], ph, &g_msd_error, 0x1202u, abort_flag, wc.limit_ns) ||
              !sm100::mbar_wait(&deq[s], ph, &g_msd_error, 0x1203u, abort_flag, wc.limit_ns)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint32_t b_base = smem_u32(sB + s * kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // A = weights (features x k), B = digit planes (tokens x k);
            // accumulator columns c * 128 + token hold plane c
            const uint32_t acc_in = (t | kk) != 0 ? 1u : 0u;
            const uint64_t adesc = sm100::sdesc_sw128_kmajor(b_base + kk * 32);
            sm100::mma_i8(tmem + (uint32_t)(b * C * BN),
                          adesc,
                          sm100::sdesc_sw128_kmajor(smem_u32(sA + s * C * kPlaneBytes) + kk * 32),
                          idesc_pair, acc_in);
#pragma unroll
            for (int c = kPair; c < C; ++c)
              sm100::mma_i8(tmem + (uint32_t)((b * C + c) * BN), adesc,
                            sm100::sdesc_sw128_kmajor(smem_u32(sA + (s * C + c) * kPlaneBytes) +
                                                      kk * 32),
                            idesc_one, acc_in);
          }
          sm100::mma_commit(&empty[s]);
        }
        if (ok) sm100::mma_commit(&acc_full[b]);
      }
      sm100::mma_commit(mma_done);
    }
  } else if (warp < 2 + kUnpackWarps) {
    // ---------------- unpack: B row r = feature n0 + r ----------------
    const int r = threadIdx.x - 64;
    const __half* zrow = zeros + (int64_t)(n0 + r) * NG;
    // the zero point of the rank's first group (its k-tiles may start inside it)
    // and the next group's, loaded one group ahead (at 128-wide groups a
    // zero-point load at the top of each k-tile sat on the critical path)
    const int g0 = kt0 / TPG;
    uint32_t zc = (128u - (uint32_t)__half2float(zrow[g0])) * 0x01010101u;
    __half z_next = zrow[(kt0 % TPG == 0) ? g0 : min(g0 + 1, NG - 1)];
    for (int i = 0; i < KT; ++i) {
      const int kt = kt0 + i;
      const int s = i % kStages;
      const uint32_t ph = (uint32_t)(i / kStages) & 1u;
      if (kt % TPG == 0) {
        zc = (128u - (uint32_t)__half2float(z_next)) * 0x01010101u;
        z_next = zrow[min(kt / TPG + 1, NG - 1)];
      }
      bool got = sm100::mbar_wait(&full[s], ph, &g_msd_error, 0x1301u, abort_flag, wc.limit_ns);
      if (!__all_sync(0xffffffffu, got)) break;
      const uint4* wsrc = reinterpret_cast<const uint4*>(sW + s * kWBytes + r * 64);
      uint8_t* bdst = sB + s * kBBytes + r * 128;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        // rows are 64 bytes apart: rotating the chunk order by r / 2 puts
        // the 16-byte reads of a warp on distinct banks
        const int j4 = (jj + (r >> 1)) & 3;
        const uint4 wv = wsrc[j4];  // words 4*j4 .. 4*j4+3 -> chunks 2*j4, 2*j4+1
        const uint2 b0 = unpack_word_minus_zero(wv.x, zc);
        const uint2 b1 = unpack_word_minus_zero(wv.y, zc);
        const uint2 b2 = unpack_word_minus_zero(wv.z, zc);
        const uint2 b3 = unpack_word_minus_zero(wv.w, zc);
        const int c0 = 2 * j4, c1 = 2 * j4 + 1;
        *reinterpret_cast<uint4*>(bdst + ((c0 ^ (r & 7)) << 4)) = make_uint4(b0.x, b0.y, b1.x, b1.y);
        *reinterpret_cast<uint4*>(bdst + ((c1 ^ (r & 7)) << 4)) = make_uint4(b2.x, b2.y, b3.x, b3.y);
      }
      sm100::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&deq[s]);
    }
  } else {
    // ---------------- drain / epilogue ----------------
    // thread = TMEM lane = feature n0 + row; its kDrainCols columns are the
    // tokens m0 + c0 + j
    const int q = warp & 3;                              // TMEM lane quarter
    const int c0 = ((warp - 2 - kUnpackWarps) >> 2) * kDrainCols;
    const int row = 32 * q + lane;
    // acc2[i] holds the tokens c0 + 2i, c0 + 2i + 1 (packed pairs)
    uint64_t acc2[kDrainCols / 2];
#pragma unroll
    for (int j = 0; j < kDrainCols / 2; ++j) acc2[j] = 0ull;
    const __half* srow = scales + (int64_t)(n0 + row) * NG + g_first;
    float scl = __half2float(srow[0]);
    bool ok = true;
    for (int gi = 0; gi < NSG; ++gi) {
      const int b = gi % NB;
      const float scl_next = gi + 1 < NSG ? __half2float(srow[gi + 1]) : 0.0f;
      if (ok) {
        bool got = sm100::mbar_wait(&acc_full[b], (uint32_t)(gi / NB) & 1u, &g_msd_error,
                                    0x1401u, abort_flag, wc.limit_ns);
        ok = __all_sync(0xffffffffu, got);
      }
      if (!ok) break;
      sm100::tc_fence_after();
      const uint64_t scl2 = f2_pack(scl, scl);
#pragma unroll
      for (int cc = 0; cc < kDrainCols / 16; ++cc) {
        const int col = c0 + 16 * cc;
        const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * C * BN + col);
        uint32_t p[C][16];
#pragma unroll
        for (int c = 0; c < C; ++c) tmem_ld16(base + (uint32_t)(c * BN), p[c]);
        sm100::tmem_ld_wait();
        float t[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (kIntCombine) {
            int32_t v = (int32_t)p[0][j];
#pragma unroll
            for (int c = 1; c < C; ++c) v = v * 256 + (int32_t)p[c][j];
            t[j] = (float)v;
          } else {
            t[j] = (float)(int32_t)p[0][j];
#pragma unroll
            for (int c = 1; c < C; ++c) t[j] = fmaf(t[j], 256.0f, (float)(int32_t)p[c][j]);
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
          acc2[8 * cc + j] = f2_fma(scl2, f2_pack(t[2 * j], t[2 * j + 1]), acc2[8 * cc + j]);
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&acc_empty[b]);
      scl = scl_next;
    }
    float acc[kDrainCols];
#pragma unroll
    for (int j = 0; j < kDrainCols / 2; ++j) {
      const float2 v = f2_unpack(acc2[j]);
      acc[2 * j] = v.x;
      acc[2 * j + 1] = v.y;
    }
    if (!kSplit) {
      // transpose through shared memory (the stage ring is idle once the
      // last group is drained: every TMA load has been consumed), then write
      // whole 256-byte rows of y
      uint16_t* out_s = reinterpret_cast<uint16_t*>(smem);  // [128 tokens][kOutPitch]
      if (ok) {
#pragma unroll
        for (int j = 0; j < kDrainCols; ++j) {
          const int m = m0 + c0 + j;
          const float sC = m < M ? comp_scales[(int64_t)(C - 1) * M + m] : 0.0f;
          out_s[(c0 + j) * kOutPitch + row] = bf16_bits(acc[j] * sC);
        }
      }
      named_bar_sync(1, 32 * kEpiWarps);
      if (ok) {
        const int e = threadIdx.x - 64 - 32 * kUnpackWarps;  // 0 .. 32 * kEpiWarps - 1
        for (int it = e; it < BM * (BN / 8); it += 32 * kEpiWarps) {
          const int t = it / (BN / 8), ch = it % (BN / 8);
          const int m = m0 + t;
          if (m < M)
            *reinterpret_cast<uint4*>(y + (int64_t)m * N + n0 + 8 * ch) =
                *reinterpret_cast<const uint4*>(out_s + t * kOutPitch + 8 * ch);
        }
      }
    } else {
      // push this rank's partials to the rank that owns the feature row
      splitk::cluster_sync_all();  // every rank is past its main loop
      const int rows_max = (BN + S - 1) / S;
      const int owner = splitk::row_owner(row, S);
      const int lr = row - splitk::rank_row_begin(owner, S);
      float* dst = reinterpret_cast<float*>(smem) + ((size_t)rank * rows_max + lr) * kRedPitch +
                   c0;
      const uint32_t rdst = splitk::map_rank(dst, (uint32_t)owner);
#pragma unroll
      for (int i = 0; i < kDrainCols / 4; ++i)
        asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(rdst + 16u * i),
                     "f"(acc[4 * i]), "f"(acc[4 * i + 1]), "f"(acc[4 * i + 2]),
                     "f"(acc[4 * i + 3])
                     : "memory");
      splitk::cluster_sync_all();  // all partials have landed
    }
  }
  if (kSplit) {
    // Split-K over the cluster: once every rank has finished its main loop
    // (first cluster barrier; the stage ring is then free everywhere), the
    // drain warps pushed their partials into the ring of the rank that owns
    // those token rows (red[src rank][local row][128 features] there, remote
    // stores); after the second barrier each owner sums its rows in rank
    // order and writes them once as bf16. Every thread of every rank passes
    // both barriers, also after an abort.
    if (warp < 2 + kUnpackWarps) {
      __syncwarp();
      splitk::cluster_sync_all();
      splitk::cluster_sync_all();
    }
    // red[src rank][local feature row][token]; the owner of feature rows
    // [r_begin, r_begin + nrows) sums them in rank order and writes y, each
    // thread one (token, feature) with consecutive threads on consecutive
    // features
    const float* red = reinterpret_cast<const float*>(smem);
    const int rows_max = (BN + S - 1) / S;
    const int r_begin = splitk::rank_row_begin(rank, S);
    const int nrows = splitk::rank_row_begin(rank + 1, S) - r_begin;
    for (int it = threadIdx.x; it < nrows * BM; it += blockDim.x) {
      const int t = it / nrows, lr = it - t * nrows;
      const int m = m0 + t;
      if (m >= M) continue;
      float v = 0.0f;
      for (int qq = 0; qq < S; ++qq) v += red[((size_t)qq * rows_max + lr) * kRedPitch + t];
      const float sC = comp_scales[(int64_t)(C - 1) * M + m];
      y[(int64_t)m * N + n0 + r_begin + lr] = bf16_bits(v * sC);
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  // After an abort (every role has left its loop): the producer waits until
  // each load it issued has landed (only its last kStages can be in flight:
  // k-tile i was issued after k-tile i - kStages had been consumed), and the
  // MMA issuer until its final commit reports every MMA done, before TMEM is
  // freed and the CTA exits.
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int i = max(0, last_issued - kStages + 1); i <= last_issued; ++i)
        if (!(wc.stall && i == 0))
          sm100::mbar_wait_drain(&full[i % kStages], (uint32_t)(i / kStages) & 1u, wc.limit_ns);
    } else if (warp == 1 && lane == 0) {
      sm100::mbar_wait_drain(mma_done, 0, wc.limit_ns);
    }
    __syncthreads();
  }
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// K split (cluster size). Each rank of an S-CTA cluster takes a contiguous
// run of k-tiles (at least one) and the partials meet through distributed
// shared memory. S minimises (waves of clusters) x (k-tiles per rank + the
// fixed cost of a CTA + the cost of the reduction when split), both costs in
// k-tile times as measured on B200 (about 6 each): it fills the GPU when
// there are fewer output tiles than SMs and evens out a last wave that would
// run mostly empty when K is long (1024 x 5120 x 25600: 3 unsplit waves of
// 200 k-tiles take 652 us, 4-way split 595 us). Clusters per wave come from
// the occupancy API; the choice is cached per shape.
template <class Kern>
int msd_split(Kern kern, int smem, int64_t tiles, int64_t ktiles) {
  const splitk::Plan pl = splitk::cached_plan(
      reinterpret_cast<const void*>(kern), (int)tiles, 0, ktiles, smem, [&] {
        int best_s = 1;
        double best = -1.0;
        for (int S = 1; S <= 8 && S <= ktiles; ++S) {
          int per_wave = 0;
          if (S == 1) {
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem) !=
                cudaSuccess) {
              cudaGetLastError();
              continue;
            }
            per_wave = per_sm * num_sms();
          } else {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)S, (unsigned)tiles, 1);
            cfg.blockDim = dim3(kThreads, 1, 1);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = (unsigned)S;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&per_wave, kern, &cfg) != cudaSuccess) {
              cudaGetLastError();
              continue;
            }
          }
          if (per_wave < 1) continue;
          const int64_t waves = (tiles + per_wave - 1) / per_wave;
          constexpr int kCtaCost = 6, kReduceCost = 6;  // in k-tile times
          const double cost =
              (double)waves * (double)((ktiles + S - 1) / S + kCtaCost + (S > 1 ? kReduceCost : 0));
          if (best < 0.0 || cost < best) {
            best = cost;
            best_s = S;
          }
        }
        return splitk::Plan{best_s, 0, (size_t)smem};
      });
  return pl.S < 1 ? 1 : pl.S;
}

template <int C, bool kInt>
wq_status launch_c(const CUtensorMap& ta, const CUtensorMap& tw, const void* scales,
                   const void* zeros, const float* cs, void* y, int64_t M, int64_t N, int64_t K,
                   int32_t G, cudaStream_t st) {
  using Cfg = MsdCfg<C>;
  const int64_t mp = m_padded(M);
  const int64_t tiles = (N / BN) * (mp / BM);
  auto kern_split = msd_gemm_kernel<C, kInt, true>;
  auto kern_one = msd_gemm_kernel<C, kInt, false>;
  for (auto kf : {kern_split, kern_one})
    if (cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem) !=
        cudaSuccess)
      return WQ_ERR_CUDA;
  const int S = msd_split(kern_split, Cfg::kSmem, tiles, K / BK);
  auto kern = S > 1 ? kern_split : kern_one;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = S > 1 ? dim3((unsigned)S, (unsigned)(N / BN), (unsigned)(mp / BM))
                      : dim3((unsigned)(N / BN), (unsigned)(mp / BM), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = S > 1 ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, ta, tw, static_cast<const __half*>(scales),
                         static_cast<const __half*>(zeros), cs, static_cast<uint16_t*>(y), (int)M,
                         (int)N, (int)K, G, (int)mp, S, wait_ctl()) != cudaSuccess)
    return WQ_ERR_CUDA;
  return launch_status();
}

}  // namespace

// Workspace: digit planes [C][M_pad][K] int8 (M_pad = M rounded up to 128;
// in k order for the decode kernel, k permuted within runs of 8 for the
// tensor-core kernel), then the component scales [C][M] fp32, 256-byte
// aligned.
size_t msd_workspace_bytes(int64_t M, int64_t K, int32_t C) {
  return planes_bytes(M, K, C) + (size_t)C * M * 4;
}

wq_status launch_msd_gemv(const int8_t* planes, int64_t plane_rows, const float* comp_scales,
                          int64_t M, int64_t N, int64_t K, int32_t C, int32_t G,
                          const void* qweight, const void* scales, const void* zeros, void* y,
                          cudaStream_t st);

wq_status launch_msd_gemm(const void* x, int64_t M, int64_t N, int64_t K, int32_t C, int32_t G,
                          const void* qweight, const void* scales, const void* zeros, void* y,
                          void* workspace, cudaStream_t st) {
  int8_t* planes = static_cast<int8_t*>(workspace);
  float* cs = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + planes_bytes(M, K, C));
  const int64_t mp = m_padded(M);
  // decode sizes: the weight stream is the cost, so the split-K GEMV with
  // integer warp MMAs replaces the 128-token tcgen05 tiles (it stages the
  // planes in k order itself; the tensor-core kernel reads them permuted)
  if (M <= 16 && G % 128 == 0) {
    wq_status s = launch_msd_decompose(x, M, K, C, mp, planes, cs, st);
    if (s != WQ_OK) return s;
    return launch_msd_gemv(planes, mp, cs, M, N, K, C, G, qweight, scales, zeros, y, st);
  }
  wq_status s = launch_msd_decompose_nibble_order(x, M, K, C, mp, planes, cs, st);
  if (s != WQ_OK) return s;
  CUtensorMap ta, tw;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, planes, (uint64_t)K, (uint64_t)(C * mp),
                    (uint64_t)K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return WQ_ERR_CUDA;
  if (!make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight, (uint64_t)K / 8, (uint64_t)N,
                    (uint64_t)K / 2, BK / 8, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return WQ_ERR_CUDA;
  // integer combination of the components while it cannot overflow int32:
  // |P_1| <= 127 * 15 * G and 256 * |P_1| + |P_2| must stay below 2^31
  const bool int_ok = (int64_t)G * 127 * 15 * 257 < ((int64_t)1 << 31);
  switch (C) {
    case 1: return launch_c<1, true>(ta, tw, scales, zeros, cs, y, M, N, K, G, st);
    case 2:
      return int_ok ? launch_c<2, true>(ta, tw, scales, zeros, cs, y, M, N, K, G, st)
                    : launch_c<2, false>(ta, tw, scales, zeros, cs, y, M, N, K, G, st);
    default: return launch_c<3, false>(ta, tw, scales, zeros, cs, y, M, N, K, G, st);
  }
}

wq_status read_msd_error(bool clear, uint32_t* v) {
  uint32_t h = 0;
  if (cudaMemcpyFromSymbol(&h, g_msd_error, sizeof(h)) != cudaSuccess) return WQ_ERR_CUDA;
  if (clear && h) {
    const uint32_t z = 0;
    if (cudaMemcpyToSymbol(g_msd_error, &z, sizeof(z)) != cudaSuccess) return WQ_ERR_CUDA;
  }
  *v = h;
  return WQ_OK;
}

}  // namespace wq
