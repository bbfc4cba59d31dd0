// Prefill W4A16 GEMM with the INT4 dequantization fused into a tcgen05 GEMM.
//
// Source: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
// Activation Decomposition for Efficient LLM Inference", Abstract: lifting the
// low-bit weights to bf16 before the multiply can cost more cycles than the
// multiply and leave the tensor cores idle. Group scale/zero per "MixPE:
// Quantization and Hardware Co-design for Efficient LLM Inference", Abstract.
//
// B200 design. The CTA computes the transposed tile D = W_tile . x_tile^T:
// 128 weight rows (the MMA's M) by BT tokens (its N, 256 or 128), BK = 64.
//   * The dequantized weights are the A operand and live in tensor memory:
//     dequantization warps write them with tcgen05.st straight from
//     registers, so they never touch shared memory. Shared memory carries
//     only the TMA traffic (x tiles and packed weight tiles) and the tensor
//     core's reads of x.
//   * Putting the 256-wide side on the tokens halves the dequantization work
//     per MMA flop compared with a 256-wide weight tile.
//   warp 0      TMA producer: x tile (fp16, 128-byte swizzled, BT rows) and
//               the packed weight tile (128 rows x 8 words) into an ST-deep
//               shared ring.
//   warp 1      allocates TMEM; one lane issues tcgen05.mma.kind::f16
//               (128 x BT x 16, A from TMEM, B = x from shared memory, fp32
//               accumulator in TMEM).
//   warps 2-9   dequantize one k-tile per TMEM A stage (SA stages of 32
//   (2-17 NF4)  columns); NF4 has two groups of 8 taking alternate k-tiles. Warp w
//               owns TMEM lanes 32 (w % 4) .. +31, i.e. one weight row per
//               thread, and half of its k-tile's 64 k. After the main loop
//               they are the epilogue: TMEM -> x 2^-e per token -> bf16 ->
//               shared staging tile [BT tokens][128 rows] -> one TMA store
//               into y.
// NF4 weights (block 64 = one k-tile) take the same path: a 256-entry
// per-lane table turns each code byte into the fp16 pair of its two codebook
// values, and one fp16 multiply applies the block's absmax, prescaled in
// fp32 by a power of two per weight row (the row's largest absmax lands in
// [2^14, 2^15), so the product stays in fp16's normal range for any absmax;
// the epilogue divides it back out).
// Operands are fp16, not bf16: the activations arrive as fp16 copies scaled
// by a power of two per row (exact), and the dequantized weight is
// fp16_rn((q - z) * s): the nibble becomes fp16 1024 + q or 64 + q by one
// AND-OR, subtracting 1024 + z or 64 + z is exact, and one multiply by the
// fp16 scale rounds once (2^-12 relative, against 2^-9 for a bf16 weight).
// Within every 8-element chunk of k both operands use the order
// k0 k4 k1 k5 k2 k6 k3 k7 (the order one packed word dequantizes into).
#include <algorithm>

#include "sm100.cuh"

namespace wq {

wq_status launch_x_to_f16(const void* x, int64_t M, int64_t K, void* x16, float* inv_scale,
                          bool permute, cudaStream_t st);

namespace {

__device__ unsigned int g_gemm_error;

constexpr int BW = 128;          // weight rows per CTA (MMA M)
constexpr int kRowMaxBytes = 4 * BW * 4;  // NF4: per-row partial absmax maxima [4][BW]
constexpr int BK = 64;           // k per stage
constexpr int kDeqWarps = 8;     // per k-tile: two per TMEM lane quarter
// Dequantization warp groups, each taking every kGroups-th k-tile: a warp
// handles one k-tile at a time through a chain of dependent steps (wait, load,
// convert, TMEM store, wait for it, arrive). NF4's table lookups make that
// chain long enough that two groups overlapping two k-tiles pay (+6 to +19 %
// measured); for INT4 a second group measured 3-5 % slower.
template <bool kNF4>
struct Deq {
  static constexpr int kGroups = kNF4 ? 2 : 1;
  static constexpr int kThreads = 64 + 32 * kDeqWarps * kGroups;
};
constexpr int SA = 4;            // TMEM A stages (32 columns each)

// KB: k per stage, 64 or 128 (two 64-wide swizzled x blocks; half the
// barrier round trips per MMA).
template <int BT, bool kNF4, int KB>
struct GemmCfg {
  static constexpr int kXBlocks = KB / 64;
  static constexpr int kACols = KB / 2;           // TMEM columns of one A stage
  // A multiple of the dequantization groups, so that every ring stage and A
  // stage is always waited on by the same group, one phase at a time (a
  // parity wait must never run two phases ahead of its barrier). NF4 needs
  // room for its lookup table.
  static constexpr int kStages =
      KB == 64 ? ((BT == 256) ? (kNF4 ? 4 : 5) : 8) : ((BT == 256) ? 3 : 4);
  static constexpr int kXBytes = BT * KB * 2;     // 16-64 KB
  static constexpr int kWBytes = BW * KB / 2;     // 4 or 8 KB
  static constexpr int kStageBytes = kXBytes + kWBytes;
  static constexpr int kOutBytes = BT * BW * 2;   // epilogue staging (reuses the ring)
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kRingOrOut = kRing > kOutBytes ? kRing : kOutBytes;
  static constexpr int kLutBytes = 256 * 32 * 4;  // NF4: byte -> fp16 pair, one copy per lane
  // ring or staging, 2^-e per token, barriers (512 B), alignment slack; NF4
  // adds the lookup table and the per-row partial absmax maxima after the
  // barriers
  static constexpr int kSmem = kRingOrOut + BT * 4 + 512 + 1024;
  static constexpr int smem(bool nf4) { return kSmem + (nf4 ? kLutBytes + kRowMaxBytes : 0); }
  static constexpr uint32_t kAccCols = BT;
  static constexpr uint32_t kTmemCols = (BT + SA * kACols <= 256) ? 256 : 512;
  static_assert(BT + SA * kACols <= 512, "A stages fit in TMEM");
  static_assert(kStages % Deq<kNF4>::kGroups == 0 && SA % Deq<kNF4>::kGroups == 0,
                "stages per group");
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned for the swizzle");
};

__device__ __forceinline__ uint32_t f16x2_sub(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// 8 INT4 codes (one packed word, k..k+7) -> 8 fp16 rn((q - z) * s), in the
// order k0 k4 k1 k5 k2 k6 k3 k7. A nibble OR-ed into the fp16 mantissa reads
// as 1024 + q (bits 0-3, pattern 0x6400) or 64 + q (bits 4-7, pattern
// 0x5400), two per register with no shift; subtracting 1024 + z or 64 + z is
// exact, and the multiply by the fp16 scale rounds once.
// zb_hi / zb_lo: fp16x2 (1024 + z) and (64 + z).
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t zb_hi, uint32_t zb_lo,
                                             uint32_t s2, uint32_t* out) {
  const uint32_t w8 = w >> 8;
  out[0] = f16x2_mul(f16x2_sub(lop3_and_or(w, 0x000F000Fu, 0x64006400u), zb_hi), s2);
  out[1] = f16x2_mul(f16x2_sub(lop3_and_or(w, 0x00F000F0u, 0x54005400u), zb_lo), s2);
  out[2] = f16x2_mul(f16x2_sub(lop3_and_or(w8, 0x000F000Fu, 0x64006400u), zb_hi), s2);
  out[3] = f16x2_mul(f16x2_sub(lop3_and_or(w8, 0x00F000F0u, 0x54005400u), zb_lo), s2);
}

// NF4: per weight row a power of two 2^e that puts the row's largest block
// absmax in [2^14, 2^15), so that codebook value x absmax x 2^e rounds to
// fp16 in its normal range (never above 2^15) whatever the absmax; the
// epilogue multiplies by 2^-e. Blocks more than 2^28 below the row's largest
// underflow toward zero, a negligible part of the row's products. The four
// dequantization threads of a row (two groups x two k halves) each take the
// max over every fourth block; `part` (0..3) names this thread's share and
// rmax[part][128] collects them. All 32 * kDeqWarps * 2 dequantization
// threads call this; returns (2^e, 2^-e).
__device__ __forceinline__ float2 nf4_row_pow2(const float* arow, int nblk, int part, int r,
                                               float* rmax, int nthreads) {
  float mx = 0.0f;
  for (int j = part; j < nblk; j += 4) mx = fmaxf(mx, __ldg(arow + j));
  rmax[part * BW + r] = mx;
  sm100::named_barrier(2, (uint32_t)nthreads);
  mx = fmaxf(fmaxf(rmax[r], rmax[BW + r]), fmaxf(rmax[2 * BW + r], rmax[3 * BW + r]));
  int e = 0;
  if (mx > 0.0f && mx <= 3.4028235e38f) {
    e = 14 - ((int)((__float_as_uint(mx) >> 23) & 0xFF) - 127);
    e = e > 126 ? 126 : (e < -126 ? -126 : e);
  }
  return make_float2(__uint_as_float((uint32_t)(127 + e) << 23),
                     __uint_as_float((uint32_t)(127 - e) << 23));
}

template <int BT, bool kNF4, int KB>
__global__ void __launch_bounds__(Deq<kNF4>::kThreads, 1)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_y, const void* __restrict__ scales,
                      const __half* __restrict__ zeros, const float* __restrict__ inv_scale, int M,
                      int N, int K, int G, Nf4Table tab, WaitCtl wc) {
  using C = GemmCfg<BT, kNF4, KB>;
  constexpr int ST = C::kStages;
  constexpr int kDeqGroups = Deq<kNF4>::kGroups;
  constexpr int kThreads = Deq<kNF4>::kThreads;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;                                    // ST x (x tile, packed W tile)
  uint16_t* out_s = reinterpret_cast<uint16_t*>(smem);     // epilogue: [BT][BW] bf16
  float* s_inv = reinterpret_cast<float*>(smem + C::kRingOrOut);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_inv + BT);
  uint64_t* full = bars;
  uint64_t* empty = bars + ST;
  uint64_t* aready = bars + 2 * ST;
  uint64_t* afree = aready + SA;
  uint64_t* accf = afree + SA;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // NF4 only: lut[byte][lane] = fp16 pair (codebook[high nibble], codebook[low
  // nibble]) = elements (2j, 2j + 1); lane l reads column l, so bank l; then
  // the per-row partial absmax maxima
  uint32_t* lut = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(bars) + 512);
  float* rmax = reinterpret_cast<float*>(lut + 256 * 32);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BW;
  const int m0 = blockIdx.y * BT;
  const int KT = K / KB;

  if (threadIdx.x == 0) {
    sm100::tma_prefetch_desc(&tmap_x);
    sm100::tma_prefetch_desc(&tmap_w);
    sm100::tma_prefetch_desc(&tmap_y);
    for (int s = 0; s < ST; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < SA; ++a) {
      sm100::mbar_init(&aready[a], kDeqWarps);
      sm100::mbar_init(&afree[a], 1);
    }
    sm100::mbar_init(accf, 1);
    *abort_flag = 0;
    sm100::fence_mbar_init();
  }
  for (int j = (int)threadIdx.x - 64; j >= 0 && j < BT; j += kThreads - 64)
    s_inv[j] = (m0 + j < M) ? inv_scale[m0 + j] : 0.0f;
  if (kNF4) {
    // four lanes' copies of one entry per 16-byte store
    for (int i = threadIdx.x; i < 256 * 8; i += kThreads) {
      const int e = i >> 3;
      const uint32_t v = pack_f16x2(tab.v[e >> 4], tab.v[e & 15]);
      reinterpret_cast<uint4*>(lut)[i] = make_uint4(v, v, v, v);
    }
  }
  if (warp == 1) {
    sm100::tmem_alloc(tmem_slot, C::kTmemCols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int last_issued = -1;  // producer: the last k-tile whose loads it issued
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % ST;
        const uint32_t ph = (uint32_t)(kt / ST) & 1u;
        if (kt >= ST && !sm100::mbar_wait(&empty[s], ph ^ 1u, &g_gemm_error, 0x101u, abort_flag,
                                          wc.limit_ns))
          break;
        if (wc.stall && kt == 0) continue;  // test hook: the first k-tile never arrives
        last_issued = kt;
        uint8_t* st = ring + s * C::kStageBytes;
        sm100::mbar_arrive_expect_tx(&full[s], C::kStageBytes);
#pragma unroll
        for (int blk = 0; blk < C::kXBlocks; ++blk)
          sm100::tma_load_2d(st + blk * (BT * 64 * 2), &tmap_x, &full[s], kt * KB + 64 * blk, m0);
        // packed tile: KB / 8 uint32 words (INT4) or KB / 2 code bytes (NF4) per row
        sm100::tma_load_2d(st + C::kXBytes, &tmap_w, &full[s], kt * (kNF4 ? KB / 2 : KB / 8), n0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = sm100::idesc_f16_f32(BW, BT);
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % ST, a = kt % SA;
        const uint32_t ph = (uint32_t)(kt / ST) & 1u, pa = (uint32_t)(kt / SA) & 1u;
        if (!sm100::mbar_wait(&full[s], ph, &g_gemm_error, 0x201u, abort_flag, wc.limit_ns)) break;
        if (!sm100::mbar_wait(&aready[a], pa, &g_gemm_error, 0x202u, abort_flag, wc.limit_ns)) break;
        sm100::tc_fence_after();
        const uint32_t x_base = smem_u32(ring + s * C::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < KB / 16; ++kk) {
          const uint64_t bd =
              sm100::sdesc_sw128_kmajor(x_base + (kk / 4) * (BT * 64 * 2) + (kk % 4) * 32);
          const uint32_t at = tmem + C::kAccCols + (uint32_t)(a * C::kACols + kk * 8);
          sm100::mma_f16_tmem_a(tmem, at, bd, idesc, (kt | kk) != 0 ? 1u : 0u);
        }
        sm100::mma_commit(&empty[s]);
        sm100::mma_commit(&afree[a]);
      }
      sm100::mma_commit(accf);
    }
  } else {
    // ---------------- dequantize (warps 2..9), then epilogue ----------------
    const int dq = warp - 2;            // 0 .. 8 * kDeqGroups - 1
    const int grp = dq / kDeqWarps;     // this warp's k-tiles: kt = grp (mod kDeqGroups)
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int hk = (dq % kDeqWarps) >> 2;  // which half of the k-tile (32 k, 4 words)
    const int r = 32 * q + lane;        // weight row within the tile = TMEM lane
    const int n = n0 + r;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const int ng = K / G;
    // this thread's half of each k-tile is KB / 2 wide and lies in one group
    // (G a multiple of KB, or G == KB / 2); its groups advance by gstep every
    // tiles_per_group of its k-tiles
    const int tiles_per_group = G >= KB ? G / KB : 1;
    const int gstep = G >= KB ? 1 : KB / G;
    const int g_start = G >= KB ? 0 : hk;
    const __half* srow = static_cast<const __half*>(scales) + (int64_t)n * ng;
    const __half* zrow = kNF4 ? nullptr : zeros + (int64_t)n * ng;
    // INT4 runs one dequantization group: the group parameters are loaded
    // one group ahead of their use and converted once per group
    static_assert(kNF4 || kDeqGroups == 1, "INT4 parameter stepping assumes one group");
    __half s_next = kNF4 ? __ushort_as_half(0) : srow[g_start];
    __half z_next = kNF4 ? __ushort_as_half(0) : zrow[g_start];
    uint32_t zb_hi = 0, zb_lo = 0, s2 = 0;
    int gi = g_start, left = 0;  // group whose parameters are loaded, k-tiles left
    const bool any = grp < KT;
    // NF4: the absmax of (row n, 64-element block kt) is one per k-tile
    const float* arow = static_cast<const float*>(scales) + (int64_t)n * (K / 64);
    // NF4: the absmax block of this thread's half of k-tile kt
    auto am_block = [&](int kt) { return (kt * KB + hk * (KB / 2)) / 64; };
    float am_next = (kNF4 && any) ? arow[am_block(grp)] : 0.0f;
    const uint32_t* lut_lane = lut + lane;
    // NF4: the row's power of two (2^e, 2^-e); 1 for INT4
    const float2 rpow = kNF4 ? nf4_row_pow2(arow, K / 64, 2 * grp + hk, r, rmax,
                                            32 * kDeqWarps * kDeqGroups)
                             : make_float2(1.0f, 1.0f);
    bool ok = true;
    for (int kt = grp; kt < KT && ok; kt += kDeqGroups) {
      const int s = kt % ST, a = kt % SA;
      const uint32_t ph = (uint32_t)(kt / ST) & 1u, pa = (uint32_t)(kt / SA) & 1u;
      const bool more = kt + kDeqGroups < KT;
      uint32_t am2 = 0;
      if (kNF4) {
        // fp16x2 (absmax 2^e, absmax 2^e), rounded once; this warp's next
        // one is loaded now
        am2 = pack_f16x2(am_next * rpow.x, am_next * rpow.x);
        if (more) am_next = arow[am_block(kt + kDeqGroups)];
      } else if (left == 0) {
        const uint32_t sb = __half_as_ushort(s_next);
        const uint32_t zq = (uint32_t)__half2float(z_next);
        s2 = sb | (sb << 16);
        zb_hi = (0x6400u | zq) * 0x00010001u;         // fp16x2 (1024 + z, 1024 + z)
        zb_lo = (0x5400u | (zq << 4)) * 0x00010001u;  // fp16x2 (64 + z, 64 + z)
        if (gi + gstep < ng) {
          s_next = srow[gi + gstep];
          z_next = zrow[gi + gstep];
        }
        gi += gstep;
        left = tiles_per_group;
      }
      if (!kNF4) --left;
      bool got = sm100::mbar_wait(&full[s], ph, &g_gemm_error, 0x301u, abort_flag, wc.limit_ns);
      if (got && kt >= SA)
        got = sm100::mbar_wait(&afree[a], pa ^ 1u, &g_gemm_error, 0x302u, abort_flag, wc.limit_ns);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      // this thread's KB / 4 packed bytes: its row r, half hk of the k-tile
      const uint4* wsrc = reinterpret_cast<const uint4*>(ring + s * C::kStageBytes + C::kXBytes +
                                                         r * (KB / 2) + hk * (KB / 4));
#pragma unroll
      for (int h16 = 0; h16 < KB / 64; ++h16) {
        const uint4 wv = wsrc[h16];
        uint32_t cols[16];
        if (kNF4) {
          // 16 code bytes = elements (2j, 2j + 1) in k order: one table read
          // gives the fp16 code pair, one multiply applies the block's absmax
          const uint32_t wb[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int j = 0; j < 16; ++j)
            cols[j] = f16x2_mul(lut_lane[((wb[j >> 2] >> (8 * (j & 3))) & 0xFFu) * 32], am2);
        } else {
          dequant_word(wv.x, zb_hi, zb_lo, s2, cols + 0);
          dequant_word(wv.y, zb_hi, zb_lo, s2, cols + 4);
          dequant_word(wv.z, zb_hi, zb_lo, s2, cols + 8);
          dequant_word(wv.w, zb_hi, zb_lo, s2, cols + 12);
        }
        sm100::tmem_st16(tmem + lane_base + C::kAccCols +
                             (uint32_t)(a * C::kACols + hk * (KB / 4) + h16 * 16),
                         cols);
      }
      sm100::tmem_st_wait();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&aready[a]);
    }
    // ---------------- epilogue ----------------
    if (ok) ok = sm100::mbar_wait(accf, 0, &g_gemm_error, 0x401u, abort_flag, wc.limit_ns);
    const bool all_ok = __all_sync(0xffffffffu, ok);
    if (all_ok) {
      sm100::tc_fence_after();
      // this warp: TMEM lanes of quarter q, token columns
      // [(dq / 4) * kEpiCols, (dq / 4 + 1) * kEpiCols)
      constexpr int kEpiCols = BT / (2 * kDeqGroups);
#pragma unroll 1
      for (int c0 = (dq / 4) * kEpiCols; c0 < (dq / 4 + 1) * kEpiCols; c0 += 32) {
        uint32_t v[32];
        sm100::tmem_ld32(tmem + lane_base + (uint32_t)c0, v);
        sm100::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float val = __uint_as_float(v[j]) * s_inv[c0 + j] * rpow.y;
          out_s[(c0 + j) * BW + r] = (uint16_t)(pack_bf16x2(val, 0.0f) & 0xFFFFu);
        }
      }
      sm100::fence_proxy_async_smem();
    }
    sm100::named_barrier(1, 32 * kDeqWarps * kDeqGroups);
    if (threadIdx.x == 64 && *abort_flag == 0) {
      sm100::tma_store_2d(&tmap_y, out_s, n0, m0);
      sm100::bulk_commit();
      sm100::bulk_wait_read_all();
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  // After an abort (every role has left its loop, so nothing new is issued):
  // the producer waits until each load it issued has landed (only its last
  // ST can be in flight: k-tile kt was issued after k-tile kt - ST had been
  // consumed), and the MMA issuer until its final commit reports every MMA
  // done, so that no copy or MMA touches this CTA's shared memory or TMEM
  // after it frees them and exits.
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int kt = max(0, last_issued - ST + 1); kt <= last_issued; ++kt)
        if (!(wc.stall && kt == 0))
          sm100::mbar_wait_drain(&full[kt % ST], (uint32_t)(kt / ST) & 1u, wc.limit_ns);
    } else if (warp == 1 && lane == 0) {
      sm100::mbar_wait_drain(accf, 0, wc.limit_ns);
    }
    __syncthreads();
  }
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// CTA-pair version (cta_group::2). A 2-CTA cluster computes 256 weight rows
// by 256 tokens with one 256 x 256 x 16 MMA per k step, issued by the even
// CTA. Each CTA dequantizes its own 128 weight rows into its own TMEM (the
// A rows it contributes) and loads only its 128-token half of the x tile (the
// B columns it contributes); its TMEM accumulator holds its 128 rows by all
// 256 tokens. Per SM the x bytes per k-tile halve (16 KB instead of 32 KB).
// Measured on B200 (per-role clock stamps and A/B builds):
//   * the ring's round trip (MMA done -> slot free -> next load -> landed ->
//     dequantized -> MMA issued) over the slots in flight sets the pace, with
//     the loads themselves far from any bandwidth limit;
//   * the stage ring and the TMEM A stages have the same depth (8), so one
//     MMA commit per k-tile frees both (each commit costs the issuing thread
//     time; two per k-tile were 7 % slower);
//   * the odd CTA's dequantization warps arrive on the even CTA's barrier
//     with the default CTA-scope release (a cluster-scope release costs about
//     a microsecond per arrive and halved the kernel's speed);
//   * a separate, deeper ring for the packed weights, loaded 8 k-tiles ahead,
//     measured no faster.
// Synchronisation (stage s = kt % 8 holds this CTA's x half and its packed
// weight tile):
//   xfull[s]   (even CTA's) both CTAs' x halves landed (their TMA loads count
//              bytes on it; the even CTA's producer sets the expected total)
//   wfull[s]   (each CTA's) its packed weight tile landed
//   done[s]    the MMAs of k-tile kt completed: stage s and A stage s are
//              free (the even CTA's commit arrives on both CTAs)
//   aready[s]  (even CTA's) all 16 dequantization warps of the pair wrote A
//              stage s (the odd CTA's arrive remotely)
//   accf       all MMAs done (the even CTA's commit arrives on both CTAs)
// All waits are bounded; every thread of both CTAs reaches the final cluster
// barriers on every path.
// KB: k per stage, 64 or 128 (two 64-wide 128-byte-swizzled x blocks). The
// wider stage halves the barrier round trips per MMA.
template <int KB>
struct Gemm2Cfg {
  static constexpr int BT = 256;                  // tokens per pair tile (MMA N)
  static constexpr int kXBlocks = KB / 64;        // 64-wide swizzled x blocks per stage
  static constexpr int kACols = KB / 2;           // TMEM columns of one A stage (fp16 pairs)
  static constexpr int kStages = KB == 64 ? 8 : 4;  // stages = TMEM A stages
  static constexpr int kXBytes = 128 * KB * 2;    // this CTA's x half: 16 or 32 KB
  static constexpr int kWBytes = BW * KB / 2;     // 4 or 8 KB
  static constexpr int kStageBytes = kXBytes + kWBytes;
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kOutBytes = BT * BW * 2;   // epilogue staging (reuses the ring)
  static constexpr int kLutBytes = 256 * 32 * 4;
  static constexpr int kSmem = kRing + BT * 4 + 512 + 1024;
  static constexpr int smem(bool nf4) { return kSmem + (nf4 ? kLutBytes + kRowMaxBytes : 0); }
  static constexpr uint32_t kAccCols = BT;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kAccCols + kStages * kACols <= kTmemCols, "A stages fit in TMEM");
  static_assert(kOutBytes <= kRing, "the staging tile fits in the ring");
  static_assert(kStages % 2 == 0, "every stage is waited on by one group (up to two)");
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned for the swizzle");
  // xfull, wfull, done, aready, accf, then the TMEM slot, the abort flag and
  // the two words the other CTA writes at the end
  static_assert(8 * (4 * kStages + 1) + 16 <= 512, "barriers fit their 512 bytes");
};

template <bool kNF4, int KB>
__global__ void __launch_bounds__(Deq<kNF4>::kThreads, 1)
    w4a16_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_x,
                           const __grid_constant__ CUtensorMap tmap_w,
                           const __grid_constant__ CUtensorMap tmap_y,
                           const void* __restrict__ scales, const __half* __restrict__ zeros,
                           const float* __restrict__ inv_scale, int M, int N, int K, int G,
                           Nf4Table tab, WaitCtl wc) {
  using C = Gemm2Cfg<KB>;
  constexpr int BT = C::BT;
  constexpr int ST = C::kStages;
  constexpr int kDeqGroups = Deq<kNF4>::kGroups;
  constexpr int kThreads = Deq<kNF4>::kThreads;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;                                    // ST x (x half, packed W tile)
  uint16_t* out_s = reinterpret_cast<uint16_t*>(smem);     // epilogue: [BT][BW] bf16
  float* s_inv = reinterpret_cast<float*>(smem + C::kRing);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_inv + BT);
  uint64_t* xfull = bars;
  uint64_t* wfull = bars + ST;
  uint64_t* done = bars + 2 * ST;
  uint64_t* aready = bars + 3 * ST;
  uint64_t* accf = aready + ST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // written by the other CTA's producer at the end: its last issued k-tile
  // and whether it gave up
  volatile int* peer_info = reinterpret_cast<volatile int*>(tmem_slot + 2);
  uint32_t* lut = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(bars) + 512);
  float* rmax = reinterpret_cast<float*>(lut + 256 * 32);  // NF4 per-row partial maxima

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = sm100::cluster_ctarank();  // 0: issues the MMAs
  const bool leader = rank == 0;
  const int n0 = (int)(blockIdx.x >> 1) * (2 * BW) + BW * (int)rank;
  const int m0 = blockIdx.y * BT;                  // the pair's first token
  const int KT = K / KB;

  if (threadIdx.x == 0) {
    sm100::tma_prefetch_desc(&tmap_x);
    sm100::tma_prefetch_desc(&tmap_w);
    sm100::tma_prefetch_desc(&tmap_y);
    for (int s = 0; s < ST; ++s) {
      sm100::mbar_init(&xfull[s], 1);
      sm100::mbar_init(&wfull[s], 1);
      sm100::mbar_init(&done[s], 1);
      sm100::mbar_init(&aready[s], 2 * kDeqWarps);
    }
    sm100::mbar_init(accf, 1);
    *abort_flag = 0;
    sm100::fence_mbar_init();
  }
  for (int j = (int)threadIdx.x - 64; j >= 0 && j < BT; j += kThreads - 64)
    s_inv[j] = (m0 + j < M) ? inv_scale[m0 + j] : 0.0f;
  if (kNF4) {
    for (int i = threadIdx.x; i < 256 * 8; i += kThreads) {
      const int e = i >> 3;
      const uint32_t v = pack_f16x2(tab.v[e >> 4], tab.v[e & 15]);
      reinterpret_cast<uint4*>(lut)[i] = make_uint4(v, v, v, v);
    }
  }
  if (warp == 1) {
    sm100::tmem_alloc_pair(tmem_slot, C::kTmemCols);
    sm100::tmem_relinquish_pair();
  }
  sm100::tc_fence_before();
  __syncthreads();
  // both CTAs' barriers are initialised before any load or remote arrive
  // can target them
  sm100::cluster_sync();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int last_issued = -1;  // producer: the last k-tile whose loads it issued
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % ST;
        const uint32_t ph = (uint32_t)(kt / ST) & 1u;
        if (kt >= ST && !sm100::mbar_wait(&done[s], ph ^ 1u, &g_gemm_error, 0x111u, abort_flag,
                                          wc.limit_ns))
          break;
        if (wc.stall && kt == 0) continue;  // test hook: the first k-tile never arrives
        last_issued = kt;
        uint8_t* st = ring + s * C::kStageBytes;
        sm100::mbar_arrive_expect_tx(&wfull[s], C::kWBytes);
        sm100::tma_load_2d(st + C::kXBytes, &tmap_w, &wfull[s], kt * (kNF4 ? KB / 2 : KB / 8),
                           n0);
        if (leader) sm100::mbar_arrive_expect_tx(&xfull[s], 2 * C::kXBytes);
#pragma unroll
        for (int blk = 0; blk < C::kXBlocks; ++blk)
          sm100::tma_load_2d_pair(st + blk * (128 * 64 * 2), &tmap_x,
                                  sm100::cluster_addr(&xfull[s], 0), kt * KB + 64 * blk,
                                  m0 + 128 * (int)rank);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- pair MMA issuer (even CTA) ----------------
      constexpr uint32_t idesc = sm100::idesc_f16_f32(2 * BW, BT);
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % ST;
        const uint32_t ph = (uint32_t)(kt / ST) & 1u;
        if (!sm100::mbar_wait(&xfull[s], ph, &g_gemm_error, 0x211u, abort_flag, wc.limit_ns)) break;
        if (!sm100::mbar_wait(&aready[s], ph, &g_gemm_error, 0x212u, abort_flag, wc.limit_ns)) break;
        sm100::tc_fence_after();
        const uint32_t x_base = smem_u32(ring + s * C::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < KB / 16; ++kk) {
          const uint64_t bd =
              sm100::sdesc_sw128_kmajor(x_base + (kk / 4) * (128 * 64 * 2) + (kk % 4) * 32);
          const uint32_t at = tmem + C::kAccCols + (uint32_t)(s * C::kACols + kk * 8);
          sm100::mma_f16_tmem_a_pair(tmem, at, bd, idesc, (kt | kk) != 0 ? 1u : 0u);
        }
        sm100::mma_commit_pair(&done[s], 0x3);
      }
      sm100::mma_commit_pair(accf, 0x3);
    }
  } else {
    // ---------------- dequantize (warps 2..9), then epilogue ----------------
    const int dq = warp - 2;
    const int grp = dq / kDeqWarps;
    const int q = warp & 3;
    const int hk = (dq % kDeqWarps) >> 2;
    const int r = 32 * q + lane;
    const int n = n0 + r;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const int ng = K / G;
    // this thread's half of each k-tile is KB / 2 wide and lies in one group
    // (G a multiple of KB, or G == KB / 2); its groups advance by gstep every
    // tiles_per_group of its k-tiles
    const int tiles_per_group = G >= KB ? G / KB : 1;
    const int gstep = G >= KB ? 1 : KB / G;
    const __half* srow = static_cast<const __half*>(scales) + (int64_t)n * ng;
    const __half* zrow = kNF4 ? nullptr : zeros + (int64_t)n * ng;
    // INT4 runs one dequantization group: the group parameters are loaded
    // one group ahead of their use and converted once per group
    static_assert(kNF4 || kDeqGroups == 1, "INT4 parameter stepping assumes one group");
    const int g_start = G >= KB ? 0 : hk;
    __half s_next = kNF4 ? __ushort_as_half(0) : srow[g_start];
    __half z_next = kNF4 ? __ushort_as_half(0) : zrow[g_start];
    uint32_t zb_hi = 0, zb_lo = 0, s2 = 0;
    int gi = g_start, left = 0;  // group whose parameters are loaded, k-tiles left
    const bool any = grp < KT;
    const float* arow = static_cast<const float*>(scales) + (int64_t)n * (K / 64);
    // NF4: the absmax block of this thread's half of k-tile kt
    auto am_block = [&](int kt) { return (kt * KB + hk * (KB / 2)) / 64; };
    float am_next = (kNF4 && any) ? arow[am_block(grp)] : 0.0f;
    const uint32_t* lut_lane = lut + lane;
    // NF4: the row's power of two (2^e, 2^-e); 1 for INT4
    const float2 rpow = kNF4 ? nf4_row_pow2(arow, K / 64, 2 * grp + hk, r, rmax,
                                            32 * kDeqWarps * kDeqGroups)
                             : make_float2(1.0f, 1.0f);
    bool ok = true;
    for (int kt = grp; kt < KT && ok; kt += kDeqGroups) {
      const int s = kt % ST;
      const uint32_t ph = (uint32_t)(kt / ST) & 1u;
      const bool more = kt + kDeqGroups < KT;
      uint32_t am2 = 0;
      if (kNF4) {
        am2 = pack_f16x2(am_next * rpow.x, am_next * rpow.x);
        if (more) am_next = arow[am_block(kt + kDeqGroups)];
      } else if (left == 0) {
        const uint32_t sb = __half_as_ushort(s_next);
        const uint32_t zq = (uint32_t)__half2float(z_next);
        s2 = sb | (sb << 16);
        zb_hi = (0x6400u | zq) * 0x00010001u;
        zb_lo = (0x5400u | (zq << 4)) * 0x00010001u;
        if (gi + gstep < ng) {
          s_next = srow[gi + gstep];
          z_next = zrow[gi + gstep];
        }
        gi += gstep;
        left = tiles_per_group;
      }
      if (!kNF4) --left;
      // the weight tile landed; A stage s is free once the MMAs of k-tile
      // kt - ST completed (they also freed the stage this tile landed in)
      bool got = sm100::mbar_wait(&wfull[s], ph, &g_gemm_error, 0x311u, abort_flag, wc.limit_ns);
      if (got && kt >= ST)
        got = sm100::mbar_wait(&done[s], ph ^ 1u, &g_gemm_error, 0x312u, abort_flag, wc.limit_ns);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      // this thread's KB / 4 packed bytes: its row r, half hk of the k-tile
      const uint4* wsrc = reinterpret_cast<const uint4*>(ring + s * C::kStageBytes + C::kXBytes +
                                                         r * (KB / 2) + hk * (KB / 4));
#pragma unroll
      for (int h16 = 0; h16 < KB / 64; ++h16) {
        const uint4 wv = wsrc[h16];
        uint32_t cols[16];
        if (kNF4) {
          const uint32_t wb[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int j = 0; j < 16; ++j)
            cols[j] = f16x2_mul(lut_lane[((wb[j >> 2] >> (8 * (j & 3))) & 0xFFu) * 32], am2);
        } else {
          dequant_word(wv.x, zb_hi, zb_lo, s2, cols + 0);
          dequant_word(wv.y, zb_hi, zb_lo, s2, cols + 4);
          dequant_word(wv.z, zb_hi, zb_lo, s2, cols + 8);
          dequant_word(wv.w, zb_hi, zb_lo, s2, cols + 12);
        }
        sm100::tmem_st16(tmem + lane_base + C::kAccCols +
                             (uint32_t)(s * C::kACols + hk * (KB / 4) + h16 * 16),
                         cols);
      }
      sm100::tmem_st_wait();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          sm100::mbar_arrive(&aready[s]);
        else
          sm100::mbar_arrive_cluster(sm100::cluster_addr(&aready[s], 0));
      }
    }
    // ---------------- epilogue: this CTA's 128 rows x 256 tokens ----------------
    if (ok) ok = sm100::mbar_wait(accf, 0, &g_gemm_error, 0x411u, abort_flag, wc.limit_ns);
    const bool all_ok = __all_sync(0xffffffffu, ok);
    if (all_ok) {
      sm100::tc_fence_after();
      constexpr int kEpiCols = BT / (2 * kDeqGroups);
#pragma unroll 1
      for (int c0 = (dq / 4) * kEpiCols; c0 < (dq / 4 + 1) * kEpiCols; c0 += 32) {
        uint32_t v[32];
        sm100::tmem_ld32(tmem + lane_base + (uint32_t)c0, v);
        sm100::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float val = __uint_as_float(v[j]) * s_inv[c0 + j] * rpow.y;
          out_s[(c0 + j) * BW + r] = (uint16_t)(pack_bf16x2(val, 0.0f) & 0xFFFFu);
        }
      }
      sm100::fence_proxy_async_smem();
    }
    sm100::named_barrier(1, 32 * kDeqWarps * kDeqGroups);
    if (threadIdx.x == 64 && *abort_flag == 0) {
      sm100::tma_store_2d(&tmap_y, out_s, n0, m0);
      sm100::bulk_commit();
      sm100::bulk_wait_read_all();
    }
  }

  // neither CTA frees its TMEM or exits while the pair may still use it
  sm100::tc_fence_before();
  __syncthreads();
  // Every role of this CTA has left its loop. Each producer tells the other
  // which k-tile it issued last and whether this CTA gave up (remote stores,
  // published by the cluster barrier), so both CTAs take the same path.
  if (warp == 0 && lane == 0) {
    const uint32_t peer = sm100::cluster_addr((const void*)peer_info, rank ^ 1u);
    asm volatile("st.shared::cluster.v2.s32 [%0], {%1, %2};" ::"r"(peer), "r"(last_issued),
                 "r"(*abort_flag)
                 : "memory");
  }
  sm100::cluster_sync();
  if (*abort_flag || peer_info[1]) {
    // The drain after an abort. A CTA's x half lands on the even CTA's
    // barrier, which completes a phase only once the even CTA armed it and
    // both halves landed. A producer issues k-tile kt only after the MMAs of
    // kt - ST completed, so either producer is at most ST - 1 k-tiles ahead
    // of the other, and the stages of the k-tiles it is ahead by are free in
    // the other CTA. The producer that is behind issues its x half of those
    // k-tiles (the even CTA arming each first); then every x phase either
    // producer started completes, and the even CTA waits for the last ST of
    // them (covering both CTAs' halves), each producer for its own weight
    // loads, and the MMA issuer for its final commit.
    if (warp == 0 && lane == 0) {
      const int other_last = peer_info[0];
      for (int kt = last_issued + 1; kt <= other_last; ++kt) {
        if (wc.stall && kt == 0) continue;
        const int s = kt % ST;
        uint8_t* st = ring + s * C::kStageBytes;
        if (leader) sm100::mbar_arrive_expect_tx(&xfull[s], 2 * C::kXBytes);
#pragma unroll
        for (int blk = 0; blk < C::kXBlocks; ++blk)
          sm100::tma_load_2d_pair(st + blk * (128 * 64 * 2), &tmap_x,
                                  sm100::cluster_addr(&xfull[s], 0), kt * KB + 64 * blk,
                                  m0 + 128 * (int)rank);
      }
      const int last_x = max(last_issued, other_last);
      if (leader)
        for (int kt = max(0, last_x - ST + 1); kt <= last_x; ++kt)
          if (!(wc.stall && kt == 0))
            sm100::mbar_wait_drain(&xfull[kt % ST], (uint32_t)(kt / ST) & 1u, wc.limit_ns);
      for (int kt = max(0, last_issued - ST + 1); kt <= last_issued; ++kt)
        if (!(wc.stall && kt == 0))
          sm100::mbar_wait_drain(&wfull[kt % ST], (uint32_t)(kt / ST) & 1u, wc.limit_ns);
    } else if (warp == 1 && lane == 0 && leader) {
      sm100::mbar_wait_drain(accf, 0, wc.limit_ns);
    }
    sm100::cluster_sync();
  }
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc_pair(tmem, C::kTmemCols);
  }
  sm100::cluster_sync();
}

// Epilogue of 32 accumulator columns of one TMEM lane (one weight row):
// column j times the token scale si[j], rounded once to bf16, into the
// [token][row] staging tile at dst[j * BW]. The scales are read four at a
// time (si is 16-byte aligned) and the values converted two at a time.
__device__ __forceinline__ void epi_store32(const uint32_t (&v)[32], const float* si,
                                            uint16_t* dst) {
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 s4 = *reinterpret_cast<const float4*>(si + j);
    const uint32_t p0 = pack_bf16x2(__uint_as_float(v[j]) * s4.x, __uint_as_float(v[j + 1]) * s4.y);
    const uint32_t p1 =
        pack_bf16x2(__uint_as_float(v[j + 2]) * s4.z, __uint_as_float(v[j + 3]) * s4.w);
    dst[(j + 0) * BW] = (uint16_t)(p0 & 0xFFFFu);
    dst[(j + 1) * BW] = (uint16_t)(p0 >> 16);
    dst[(j + 2) * BW] = (uint16_t)(p1 & 0xFFFFu);
    dst[(j + 3) * BW] = (uint16_t)(p1 >> 16);
  }
}

// Persistent CTA-pair kernel (INT4, 128-wide k stages, G a multiple of 128).
// The pair kernel above pays, for every 256 x 256 tile, its prologue, the
// fill of its stage ring and its epilogue one after the other; here each pair
// of CTAs loops over the tiles t = pair, pair + pairs, ... (features fastest),
// and the producer, the MMA issuer and the dequantization warps run one
// flattened sequence of (tile, k-tile) steps, so the ring's phases continue
// from tile to tile and the next tile's loads and dequantization overlap the
// current tile's epilogue. Sixteen epilogue warps of their own drain each tile
// (four per TMEM lane quarter, 64 token columns each, so the accumulator is
// free again after two TMEM loads per thread):
//   accf       (both CTAs) the tile's MMAs completed (one phase per tile)
//   acc_empty  (even CTA's) both CTAs' epilogue warps read the accumulator:
//              the tile after may start its MMAs (one phase per tile)
// The staging tile of the output has its own 64 KB (the ring is busy with the
// next tile). The other barriers are those of the pair kernel.
struct Gemm2PCfg {
  static constexpr int KB = 128;
  static constexpr int BT = 256;                  // tokens per pair tile (MMA N)
  static constexpr int kACols = KB / 2;           // TMEM columns of one A stage
  static constexpr int kStages = 4;
  static constexpr int kXBytes = 128 * KB * 2;    // this CTA's x half: 32 KB
  static constexpr int kWBytes = BW * KB / 2;     // 8 KB
  static constexpr int kStageBytes = kXBytes + kWBytes;
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kOutBytes = BT * BW * 2;   // [BT tokens][BW rows] bf16
  static constexpr int kEpiWarps = 16;            // four per TMEM lane quarter, 64 columns each
  static constexpr int kEpiFirst = 64 + 32 * kDeqWarps;  // first epilogue thread
  static constexpr int kThreads = kEpiFirst + 32 * kEpiWarps;
  static constexpr int kSmem = kRing + kOutBytes + BT * 4 + 512 + 1024;
  static constexpr uint32_t kAccCols = BT;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kAccCols + kStages * kACols <= kTmemCols, "A stages fit in TMEM");
  static_assert(kSmem <= 232448, "shared memory");
  static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned for the swizzle");
};

__global__ void __launch_bounds__(Gemm2PCfg::kThreads, 1)
    w4a16_gemm_pair_persistent_kernel(const __grid_constant__ CUtensorMap tmap_x,
                                      const __grid_constant__ CUtensorMap tmap_w,
                                      const __grid_constant__ CUtensorMap tmap_y,
                                      const __half* __restrict__ scales,
                                      const __half* __restrict__ zeros,
                                      const float* __restrict__ inv_scale, int M, int N, int K,
                                      int G, WaitCtl wc) {
  using C = Gemm2PCfg;
  constexpr int BT = C::BT, ST = C::kStages, KB = C::KB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint16_t* out_s = reinterpret_cast<uint16_t*>(smem + C::kRing);          // [BT][BW] bf16
  float* s_inv = reinterpret_cast<float*>(smem + C::kRing + C::kOutBytes);  // [BT]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_inv + BT);
  uint64_t* xfull = bars;
  uint64_t* wfull = bars + ST;
  uint64_t* done = bars + 2 * ST;
  uint64_t* aready = bars + 3 * ST;
  uint64_t* accf = bars + 4 * ST;
  uint64_t* acc_empty = accf + 1;
  uint64_t* mma_done = accf + 2;  // the MMA issuer's final commit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* peer_info = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [2]
  volatile int* epi_ok = reinterpret_cast<volatile int*>(tmem_slot + 4);     // [kEpiWarps]
  static_assert(4 * (4 + Gemm2PCfg::kEpiWarps) + 8 * (4 * Gemm2PCfg::kStages + 3) <= 512,
                "barriers and flags fit their 512 bytes");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = sm100::cluster_ctarank();  // 0: issues the MMAs
  const bool leader = rank == 0;
  const int npairs = (int)(gridDim.x >> 1);
  const int pair = (int)(blockIdx.x >> 1);
  const int ntn = N / (2 * BW);  // pair tiles along the features
  const int ntiles = ntn * ((M + BT - 1) / BT);
  const int nlocal = pair < ntiles ? (ntiles - pair + npairs - 1) / npairs : 0;
  const int KT = K / KB;
  const int total = nlocal * KT;  // this pair's (tile, k-tile) steps
  auto tile_of = [&](int j) { return pair + j * npairs; };
  auto n0_of = [&](int t) { return (t % ntn) * (2 * BW) + BW * (int)rank; };
  auto m0_of = [&](int t) { return (t / ntn) * BT; };

  if (threadIdx.x == 0) {
    sm100::tma_prefetch_desc(&tmap_x);
    sm100::tma_prefetch_desc(&tmap_w);
    sm100::tma_prefetch_desc(&tmap_y);
    for (int s = 0; s < ST; ++s) {
      sm100::mbar_init(&xfull[s], 1);
      sm100::mbar_init(&wfull[s], 1);
      sm100::mbar_init(&done[s], 1);
      sm100::mbar_init(&aready[s], 2 * kDeqWarps);
    }
    sm100::mbar_init(accf, 1);
    sm100::mbar_init(acc_empty, 2 * C::kEpiWarps);
    sm100::mbar_init(mma_done, 1);
    *abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc_pair(tmem_slot, C::kTmemCols);
    sm100::tmem_relinquish_pair();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::cluster_sync();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int last_issued = -1;  // producer: the last step whose loads it issued
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      // (k-tile, tile and its coordinates advance incrementally: no division per step)
      int kt = 0, j = 0, n0 = n0_of(tile_of(0)), m0 = m0_of(tile_of(0));
      for (int it = 0; it < total; ++it, ++kt) {
        if (kt == KT) {
          kt = 0;
          ++j;
          n0 = n0_of(tile_of(j));
          m0 = m0_of(tile_of(j));
        }
        const int s = it % ST;
        const uint32_t ph = (uint32_t)(it / ST) & 1u;
        if (it >= ST && !sm100::mbar_wait(&done[s], ph ^ 1u, &g_gemm_error, 0x511u, abort_flag,
                                          wc.limit_ns))
          break;
        if (wc.stall && it == 0) continue;  // test hook: the first step never arrives
        last_issued = it;
        uint8_t* st = ring + s * C::kStageBytes;
        sm100::mbar_arrive_expect_tx(&wfull[s], C::kWBytes);
        sm100::tma_load_2d(st + C::kXBytes, &tmap_w, &wfull[s], kt * (KB / 8), n0);
        if (leader) sm100::mbar_arrive_expect_tx(&xfull[s], 2 * C::kXBytes);
#pragma unroll
        for (int blk = 0; blk < KB / 64; ++blk)
          sm100::tma_load_2d_pair(st + blk * (128 * 64 * 2), &tmap_x,
                                  sm100::cluster_addr(&xfull[s], 0), kt * KB + 64 * blk,
                                  m0 + 128 * (int)rank);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- pair MMA issuer (even CTA) ----------------
      constexpr uint32_t idesc = sm100::idesc_f16_f32(2 * BW, BT);
      int kt = 0, j = 0;
      for (int it = 0; it < total; ++it, ++kt) {
        if (kt == KT) {
          kt = 0;
          ++j;
        }
        const int s = it % ST;
        const uint32_t ph = (uint32_t)(it / ST) & 1u;
        if (kt == 0 && j > 0) {
          // both CTAs' epilogues have read the previous tile's accumulator
          if (!sm100::mbar_wait(acc_empty, (uint32_t)(j - 1) & 1u, &g_gemm_error, 0x521u,
                                abort_flag, wc.limit_ns))
            break;
          sm100::tc_fence_after();
        }
        if (!sm100::mbar_wait(&xfull[s], ph, &g_gemm_error, 0x522u, abort_flag, wc.limit_ns)) break;
        if (!sm100::mbar_wait(&aready[s], ph, &g_gemm_error, 0x523u, abort_flag, wc.limit_ns)) break;
        sm100::tc_fence_after();
        const uint32_t x_base = smem_u32(ring + s * C::kStageBytes);
#pragma unroll
        for (int kk = 0; kk < KB / 16; ++kk) {
          const uint64_t bd =
              sm100::sdesc_sw128_kmajor(x_base + (kk / 4) * (128 * 64 * 2) + (kk % 4) * 32);
          const uint32_t at = tmem + C::kAccCols + (uint32_t)(s * C::kACols + kk * 8);
          sm100::mma_f16_tmem_a_pair(tmem, at, bd, idesc, (kt | kk) != 0 ? 1u : 0u);
        }
        sm100::mma_commit_pair(&done[s], 0x3);
        if (kt == KT - 1) sm100::mma_commit_pair(accf, 0x3);
      }
      sm100::mma_commit_pair(mma_done, 0x3);
    }
  } else if (warp < 2 + kDeqWarps) {
    // ---------------- dequantize (warps 2..9) ----------------
    const int dq = warp - 2;
    const int q = warp & 3;
    const int hk = dq >> 2;  // which 64-k half of each k-tile
    const int r = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const int ng = K / G;
    const int tpg = G / KB;  // k-tiles per group
    // group parameters of row n, group g
    auto load_prm = [&](int n, int g, __half& sv, __half& zv) {
      const int64_t idx = (int64_t)n * ng + g;
      sv = scales[idx];
      zv = zeros[idx];
    };
    // the step's k-tile, its group and k-tile within the group, and this
    // thread's weight row in the step's tile and in the next tile advance
    // incrementally (no division per step); a group's parameters are loaded
    // one group ahead
    int kt = 0, j = 0, gi = 0, gk = 0;
    int nrow = n0_of(tile_of(0)) + r;
    int nrow_next = nlocal > 1 ? n0_of(tile_of(1)) + r : nrow;
    __half s_next = __ushort_as_half(0), z_next = __ushort_as_half(0);
    if (total > 0) load_prm(nrow, 0, s_next, z_next);
    uint32_t zb_hi = 0, zb_lo = 0, s2 = 0;
    for (int it = 0; it < total; ++it) {
      const int s = it % ST;
      const uint32_t ph = (uint32_t)(it / ST) & 1u;
      if (gk == 0) {
        // a group starts: its parameters were loaded a group ahead
        const uint32_t sb = __half_as_ushort(s_next);
        const uint32_t zq = (uint32_t)__half2float(z_next);
        s2 = sb | (sb << 16);
        zb_hi = (0x6400u | zq) * 0x00010001u;
        zb_lo = (0x5400u | (zq << 4)) * 0x00010001u;
        if (kt + tpg < KT)
          load_prm(nrow, gi + 1, s_next, z_next);
        else if (j + 1 < nlocal)
          load_prm(nrow_next, 0, s_next, z_next);
      }
      // the weight tile landed; A stage s is free once the MMAs of step it - ST completed
      bool got = sm100::mbar_wait(&wfull[s], ph, &g_gemm_error, 0x531u, abort_flag, wc.limit_ns);
      if (got && it >= ST)
        got = sm100::mbar_wait(&done[s], ph ^ 1u, &g_gemm_error, 0x532u, abort_flag, wc.limit_ns);
      if (!__all_sync(0xffffffffu, got)) break;
      // the packed tile arrives in the TMA 64-byte swizzle: 16-byte chunk c of
      // row r at chunk c ^ ((r >> 1) & 3), so a warp's 16-byte reads (rows
      // 64 bytes apart) spread over every bank
      const uint8_t* wrow = ring + s * C::kStageBytes + C::kXBytes + r * (KB / 2);
#pragma unroll
      for (int h16 = 0; h16 < KB / 64; ++h16) {
        const uint4 wv = *reinterpret_cast<const uint4*>(
            wrow + (((2 * hk + h16) ^ ((r >> 1) & 3)) << 4));
        uint32_t cols[16];
        dequant_word(wv.x, zb_hi, zb_lo, s2, cols + 0);
        dequant_word(wv.y, zb_hi, zb_lo, s2, cols + 4);
        dequant_word(wv.z, zb_hi, zb_lo, s2, cols + 8);
        dequant_word(wv.w, zb_hi, zb_lo, s2, cols + 12);
        sm100::tmem_st16(tmem + lane_base + C::kAccCols +
                             (uint32_t)(s * C::kACols + hk * (KB / 4) + h16 * 16),
                         cols);
      }
      sm100::tmem_st_wait();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          sm100::mbar_arrive(&aready[s]);
        else
          sm100::mbar_arrive_cluster(sm100::cluster_addr(&aready[s], 0));
      }
      if (++gk == tpg) {
        gk = 0;
        ++gi;
      }
      if (++kt == KT) {
        kt = 0;
        gi = 0;
        gk = 0;
        ++j;
        nrow = nrow_next;
        if (j + 1 < nlocal) nrow_next = n0_of(tile_of(j + 1)) + r;
      }
    }
  } else {
    // ---------------- epilogue (warps 10..25): one tile at a time ----------------
    const int eq = warp - (2 + kDeqWarps);  // 0 .. 15
    const int q = warp & 3;                 // TMEM lane quarter
    const int cbase = 64 * (eq >> 2);       // this warp's 64 token columns
    const int r = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const int e = (int)threadIdx.x - C::kEpiFirst;  // 0 .. 511
    constexpr uint32_t kEpiThreads = 32 * C::kEpiWarps;
    // the token scales of the next tile travel in a register (threads e <
    // BT hold one each) and reach shared memory before its wait, so no
    // global load and no extra barrier sit between a finished accumulator
    // and its release
    float si_next = 0.0f;
    if (nlocal > 0 && e < BT) {
      const int m = m0_of(tile_of(0)) + e;
      si_next = m < M ? inv_scale[m] : 0.0f;
    }
    for (int j = 0; j < nlocal; ++j) {
      const int t = tile_of(j);
      const int m0 = m0_of(t);
      // every epilogue thread passed the previous tile's last barrier, so
      // its conversion no longer reads s_inv
      if (e < BT) s_inv[e] = si_next;
      if (j + 1 < nlocal && e < BT) {
        const int m = m0_of(tile_of(j + 1)) + e;
        si_next = m < M ? inv_scale[m] : 0.0f;
      }
      // (a tile's mainloop is long: the warps wait suspended in hardware,
      // off the issue slots of the dequantization warps and the MMA issuer,
      // and resume as soon as the accumulator is complete)
      bool got = sm100::mbar_wait_hint(accf, (uint32_t)j & 1u, &g_gemm_error, 0x541u,
                                       abort_flag, wc.limit_ns, 1000000u);
      got = __all_sync(0xffffffffu, got);
      // the previous tile's store has read the staging tile (issued a whole
      // mainloop ago)
      if (e == 0) sm100::bulk_wait_read_all();
      // the epilogue warps decide together whether to go on; the barrier
      // also publishes s_inv and the staging tile's release
      if (lane == 0) epi_ok[eq] = got ? 1 : 0;
      sm100::named_barrier(3, kEpiThreads);
      bool go = true;
#pragma unroll
      for (int w = 0; w < C::kEpiWarps; ++w) go = go && epi_ok[w] != 0;
      if (!go) break;
      sm100::tc_fence_after();
      uint32_t v[32];
      sm100::tmem_ld32(tmem + lane_base + (uint32_t)cbase, v);
      sm100::tmem_ld_wait();
      epi_store32(v, s_inv + cbase, out_s + cbase * BW + r);
      sm100::tmem_ld32(tmem + lane_base + (uint32_t)(cbase + 32), v);
      sm100::tmem_ld_wait();
      // the accumulator is read: the next tile's MMAs may start while this
      // warp converts its second half
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          sm100::mbar_arrive(acc_empty);
        else
          sm100::mbar_arrive_cluster(sm100::cluster_addr(acc_empty, 0));
      }
      epi_store32(v, s_inv + cbase + 32, out_s + (cbase + 32) * BW + r);
      sm100::fence_proxy_async_smem();
      sm100::named_barrier(3, kEpiThreads);
      if (e == 0) {
        sm100::tma_store_2d(&tmap_y, out_s, n0_of(t), m0);
        sm100::bulk_commit();
      }
    }
    if (e == 0) sm100::bulk_wait_all();
  }

  // neither CTA frees its TMEM or exits while the pair may still use it
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0) {
    const uint32_t peer = sm100::cluster_addr((const void*)peer_info, rank ^ 1u);
    asm volatile("st.shared::cluster.v2.s32 [%0], {%1, %2};" ::"r"(peer), "r"(last_issued),
                 "r"(*abort_flag)
                 : "memory");
  }
  sm100::cluster_sync();
  if (*abort_flag || peer_info[1]) {
    // The drain after an abort, as in the pair kernel, over the steps of the
    // flattened sequence: the producer that is behind issues its x half of
    // the steps the other issued (the even CTA arming each first), then the
    // even CTA waits for the last ST x phases, each producer for its own
    // weight loads, and the MMA issuer for its final commit.
    if (warp == 0 && lane == 0) {
      const int other_last = peer_info[0];
      for (int it = last_issued + 1; it <= other_last; ++it) {
        if (wc.stall && it == 0) continue;
        const int j = it / KT, kt = it - j * KT;
        const int t = tile_of(j);
        const int s = it % ST;
        uint8_t* st = ring + s * C::kStageBytes;
        if (leader) sm100::mbar_arrive_expect_tx(&xfull[s], 2 * C::kXBytes);
#pragma unroll
        for (int blk = 0; blk < KB / 64; ++blk)
          sm100::tma_load_2d_pair(st + blk * (128 * 64 * 2), &tmap_x,
                                  sm100::cluster_addr(&xfull[s], 0), kt * KB + 64 * blk,
                                  m0_of(t) + 128 * (int)rank);
      }
      const int last_x = max(last_issued, other_last);
      if (leader)
        for (int it = max(0, last_x - ST + 1); it <= last_x; ++it)
          if (!(wc.stall && it == 0))
            sm100::mbar_wait_drain(&xfull[it % ST], (uint32_t)(it / ST) & 1u, wc.limit_ns);
      for (int it = max(0, last_issued - ST + 1); it <= last_issued; ++it)
        if (!(wc.stall && it == 0))
          sm100::mbar_wait_drain(&wfull[it % ST], (uint32_t)(it / ST) & 1u, wc.limit_ns);
    } else if (warp == 1 && lane == 0 && leader) {
      sm100::mbar_wait_drain(mma_done, 0, wc.limit_ns);
    }
    sm100::cluster_sync();
  }
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc_pair(tmem, C::kTmemCols);
  }
  sm100::cluster_sync();
}

wq_status launch_pair_persistent(const void* x16, const float* inv_scale, int64_t M, int64_t N,
                                 int64_t K, int32_t G, const void* qweight, const void* scales,
                                 const void* zeros, void* y, cudaStream_t st) {
  using C = Gemm2PCfg;
  CUtensorMap tx, tw, ty;
  if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x16, (uint64_t)K, (uint64_t)M,
                    (uint64_t)K * 2, BK, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight, (uint64_t)K / 8, (uint64_t)N,
                    (uint64_t)K / 2, C::KB / 8, BW, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                    (uint64_t)N * 2, BW, C::BT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return WQ_ERR_CUDA;
  auto kern = w4a16_gemm_pair_persistent_kernel;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
      cudaSuccess)
    return WQ_ERR_CUDA;
  const int64_t ntiles = (N / (2 * BW)) * ((M + C::BT - 1) / C::BT);
  const int64_t pairs = std::min<int64_t>(ntiles, num_sms() / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tx, tw, ty, static_cast<const __half*>(scales),
                         static_cast<const __half*>(zeros), inv_scale, (int)M, (int)N, (int)K,
                         G, wait_ctl()) != cudaSuccess)
    return WQ_ERR_CUDA;
  return launch_status();
}

template <bool kNF4, int KB>
wq_status launch_pair(const void* x16, const float* inv_scale, int64_t M, int64_t N, int64_t K,
                      int32_t G, const void* qweight, const void* scales, const void* zeros,
                      void* y, cudaStream_t st) {
  using C = Gemm2Cfg<KB>;
  CUtensorMap tx, tw, ty;
  // x: this CTA's 128-token half of the pair's tile
  if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x16, (uint64_t)K, (uint64_t)M,
                    (uint64_t)K * 2, BK, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return WQ_ERR_CUDA;
  const bool wmap = kNF4 ? make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, qweight,
                                        (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, KB / 2, BW,
                                        CU_TENSOR_MAP_SWIZZLE_NONE)
                         : make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight,
                                        (uint64_t)K / 8, (uint64_t)N, (uint64_t)K / 2, KB / 8, BW,
                                        CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!wmap) return WQ_ERR_CUDA;
  if (!make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                    (uint64_t)N * 2, BW, C::BT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return WQ_ERR_CUDA;
  auto kern = w4a16_gemm_pair_kernel<kNF4, KB>;
  const int smem = C::smem(kNF4);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return WQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(N / BW), (unsigned)((M + C::BT - 1) / C::BT), 1);
  cfg.blockDim = dim3(Deq<kNF4>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tx, tw, ty, scales, static_cast<const __half*>(zeros),
                         inv_scale, (int)M, (int)N, (int)K, G, nf4_table(), wait_ctl()) !=
      cudaSuccess)
    return WQ_ERR_CUDA;
  return launch_status();
}

template <int BT, bool kNF4, int KB>
wq_status launch_bt(const void* x16, const float* inv_scale, int64_t M, int64_t N, int64_t K,
                    int32_t G, const void* qweight, const void* scales, const void* zeros, void* y,
                    cudaStream_t st) {
  CUtensorMap tx, tw, ty;
  if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x16, (uint64_t)K, (uint64_t)M,
                    (uint64_t)K * 2, BK, BT, CU_TENSOR_MAP_SWIZZLE_128B))
    return WQ_ERR_CUDA;
  // the packed tile is 32 bytes of each of 128 rows in both formats
  const bool wmap = kNF4 ? make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, qweight,
                                        (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, KB / 2, BW,
                                        CU_TENSOR_MAP_SWIZZLE_NONE)
                         : make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight,
                                        (uint64_t)K / 8, (uint64_t)N, (uint64_t)K / 2, KB / 8, BW,
                                        CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!wmap) return WQ_ERR_CUDA;
  if (!make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                    (uint64_t)N * 2, BW, BT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return WQ_ERR_CUDA;
  using C = GemmCfg<BT, kNF4, KB>;
  auto kern = w4a16_gemm_kernel<BT, kNF4, KB>;
  const int smem = C::smem(kNF4);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return WQ_ERR_CUDA;
  dim3 grid((unsigned)(N / BW), (unsigned)((M + BT - 1) / BT));
  kern<<<grid, Deq<kNF4>::kThreads, smem, st>>>(tx, tw, ty, scales,
                                                 static_cast<const __half*>(zeros), inv_scale,
                                                 (int)M, (int)N, (int)K, G, nf4_table(),
                                                 wait_ctl());
  return launch_status();
}

}  // namespace

// The CTA-pair kernel is the default for wide tiles; WQ_GEMM_PAIRS=0 in the
// environment selects the single-CTA kernel (kept as the reference design
// and for comparison).
bool gemm_pairs_enabled() {
  static const bool on = [] {
    const char* e = getenv("WQ_GEMM_PAIRS");
    return !(e && e[0] == '0');
  }();
  return on;
}

// The persistent pair kernel is the default where it applies (INT4, G a
// multiple of 128, two or more tiles per pair); WQ_GEMM_PERSIST=0 in the
// environment selects the per-tile pair kernel instead (for comparison).
bool gemm_persistent_enabled() {
  static const bool on = [] {
    const char* e = getenv("WQ_GEMM_PERSIST");
    return !(e && e[0] == '0');
  }();
  return on;
}

bool gemm_kb128_enabled() {
  static const bool on = [] {
    const char* e = getenv("WQ_GEMM_KB");
    return !(e && e[0] == '6');
  }();
  return on;
}

// Workspace: the fp16 copy of x [M, K] (256-byte aligned), then 2^-e per row.
size_t gemm_workspace_bytes(int64_t M, int64_t K) {
  return ((size_t)M * K * 2 + 255) / 256 * 256 + (size_t)M * 4;
}

wq_status launch_gemm(const void* x, int64_t M, int64_t N, int64_t K, wq_format fmt, int32_t G,
                      const void* qweight, const void* scales, const void* zeros, void* y,
                      void* workspace, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* x16 = ws;
  float* inv_scale = reinterpret_cast<float*>(ws + ((size_t)M * K * 2 + 255) / 256 * 256);
  const bool nf4 = fmt == WQ_FMT_NF4;
  wq_status s = launch_x_to_f16(x, M, K, x16, inv_scale, /*permute=*/!nf4, st);
  if (s != WQ_OK) return s;
  // 256-token tiles when they alone fill the machine, else 128-token ones.
  const int64_t tiles256 = (N / BW) * ((M + 255) / 256);
  const bool wide = tiles256 >= (int64_t)num_sms();
  // CTA pairs (256 weight rows x 256 tokens per pair) where the rows pair up
  const bool pair = wide && N % (2 * BW) == 0 && gemm_pairs_enabled();
  // 128-wide k stages where every thread's half stage lies in one group
  const bool wide_k = K % 128 == 0 && (G % 128 == 0 || G == 64) && gemm_kb128_enabled();
  if (nf4) {
    if (pair)
      return wide_k
                 ? launch_pair<true, 128>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st)
                 : launch_pair<true, 64>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st);
    // 256-token NF4 tiles keep 64-k stages: with the lookup table only two
    // 128-k stages would fit
    if (wide) return launch_bt<256, true, 64>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st);
    return wide_k
               ? launch_bt<128, true, 128>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st)
               : launch_bt<128, true, 64>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st);
  }
  // persistent pairs where every pair has at least two tiles to loop over
  if (pair && K % 128 == 0 && G % 128 == 0 && gemm_persistent_enabled() &&
      (N / (2 * BW)) * ((M + 255) / 256) >= 2 * (int64_t)(num_sms() / 2))
    return launch_pair_persistent(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st);
  if (pair)
    return wide_k
               ? launch_pair<false, 128>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st)
               : launch_pair<false, 64>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st);
  if (wide)
    return wide_k
               ? launch_bt<256, false, 128>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st)
               : launch_bt<256, false, 64>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st);
  return wide_k
             ? launch_bt<128, false, 128>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st)
             : launch_bt<128, false, 64>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st);
}

wq_status read_gemm_error(bool clear, uint32_t* v) {
  uint32_t h = 0;
  if (cudaMemcpyFromSymbol(&h, g_gemm_error, sizeof(h)) != cudaSuccess) return WQ_ERR_CUDA;
  if (clear && h) {
    const uint32_t z = 0;
    if (cudaMemcpyToSymbol(g_gemm_error, &z, sizeof(z)) != cudaSuccess) return WQ_ERR_CUDA;
  }
  *v = h;
  return WQ_OK;
}

}  // namespace wq
