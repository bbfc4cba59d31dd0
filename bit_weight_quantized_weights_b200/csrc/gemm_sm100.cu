// Prefill W4A16 GEMM with the INT4 dequantization fused into a tcgen05 GEMM.
//
// Source: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
// Activation Decomposition for Efficient LLM Inference", Abstract: lifting the
// low-bit weights to bf16 before the multiply can cost more cycles than the
// multiply and leave the tensor cores idle. Group scale/zero per "MixPE:
// Quantization and Hardware Co-design for Efficient LLM Inference", Abstract.
//
// B200 design (one 128 x BN output tile per CTA, BN = 256 or 128, BK = 64):
//   warp 0      TMA producer: x tile (fp16, 128-byte swizzled) and the packed
//               weight tile (uint32 words) into a STAGES-deep shared ring.
//   warp 1      allocates TMEM; one lane issues tcgen05.mma.kind::f16
//               (128 x BN x 16, fp16 operands, fp32 accumulator in TMEM) and
//               commits each stage back to the producer.
//   warps 2-17  dequantize the packed tile into the fp16 B operand, written
//               straight into the UMMA K-major 128-byte-swizzled layout, then
//               serve as the epilogue (tcgen05.ld -> x 2^-e -> bf16 -> global).
// Operands are fp16, not bf16: the activations arrive as fp16 copies scaled
// by a power of two per row (exact), and the dequantized weight is
// fp16_rn((q - z) * s): the nibble becomes fp16 1024 + q by byte permutes
// alone, (1024 + q) - (1024 + z) is exact, and one multiply by the fp16 scale
// rounds once (2^-12 relative, against 2^-9 for a bf16 weight).
#include "sm100.cuh"

namespace wq {

wq_status launch_x_to_f16(const void* x, int64_t M, int64_t K, void* x16, float* inv_scale,
                          cudaStream_t st);

namespace {

__device__ unsigned int g_gemm_error;

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kDeqWarps = 16;
constexpr int kThreads = 64 + 32 * kDeqWarps;

template <int BN>
struct GemmCfg {
  static constexpr int kStages = (BN == 256) ? 3 : 5;
  static constexpr int kABytes = BM * BK * 2;   // 16 KB
  static constexpr int kBBytes = BN * BK * 2;   // 32 / 16 KB
  static constexpr int kWBytes = BN * BK / 2;   // 8 / 4 KB
  static constexpr int kSmem = kStages * (kABytes + kBBytes + kWBytes) + 1024 /*align*/ + 256;
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

// 8 INT4 codes (one packed word, k..k+7) -> 8 fp16 rn((q - z) * s), in k order.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t zb2, uint32_t s2) {
  const uint32_t v = w & 0x0F0F0F0Fu;         // codes 0, 2, 4, 6
  const uint32_t u = (w >> 4) & 0x0F0F0F0Fu;  // codes 1, 3, 5, 7
  const uint32_t i01 = prmt(v, u, 0x5140u);   // bytes: c0 c1 c2 c3
  const uint32_t i23 = prmt(v, u, 0x7362u);   // bytes: c4 c5 c6 c7
  const uint32_t M64 = 0x64646464u;
  uint32_t p[4];
  p[0] = prmt(i01, M64, 0x4140u);  // fp16x2 (1024 + c0, 1024 + c1)
  p[1] = prmt(i01, M64, 0x4342u);
  p[2] = prmt(i23, M64, 0x4140u);
  p[3] = prmt(i23, M64, 0x4342u);
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = f16x2_mul(f16x2_sub(p[i], zb2), s2);  // (q - z) exact, x s
  return make_uint4(p[0], p[1], p[2], p[3]);
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_w, const __half* __restrict__ scales,
                      const __half* __restrict__ zeros, const float* __restrict__ inv_scale,
                      uint16_t* __restrict__ y, int M, int N, int K, int G) {
  using C = GemmCfg<BN>;
  constexpr int ST = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + ST * C::kABytes;
  uint8_t* sW = sB + ST * C::kBBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sW + ST * C::kWBytes);
  uint64_t* full = bars;
  uint64_t* deq = bars + ST;
  uint64_t* empty = bars + 2 * ST;
  uint64_t* accf = bars + 3 * ST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int m0 = blockIdx.y * BM;
  const int KT = K / BK;

  if (threadIdx.x == 0) {
    sm100::tma_prefetch_desc(&tmap_x);
    sm100::tma_prefetch_desc(&tmap_w);
    for (int s = 0; s < ST; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&deq[s], kDeqWarps);
      sm100::mbar_init(&empty[s], 1);
    }
    sm100::mbar_init(accf, 1);
    *abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc(tmem_slot, BN);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % ST;
        const uint32_t ph = (uint32_t)(kt / ST) & 1u;
        if (kt >= ST && !sm100::mbar_wait(&empty[s], ph ^ 1u, &g_gemm_error, 0x101u, abort_flag))
          break;
        sm100::mbar_arrive_expect_tx(&full[s], C::kABytes + C::kWBytes);
        sm100::tma_load_2d(sA + s * C::kABytes, &tmap_x, &full[s], kt * BK, m0);
        sm100::tma_load_2d(sW + s * C::kWBytes, &tmap_w, &full[s], kt * (BK / 8), n0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = sm100::idesc_f16_f32(BM, BN);
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % ST;
        const uint32_t ph = (uint32_t)(kt / ST) & 1u;
        if (!sm100::mbar_wait(&full[s], ph, &g_gemm_error, 0x201u, abort_flag)) break;
        if (!sm100::mbar_wait(&deq[s], ph, &g_gemm_error, 0x202u, abort_flag)) break;
        sm100::tc_fence_after();
        const uint32_t a_base = smem_u32(sA + s * C::kABytes);
        const uint32_t b_base = smem_u32(sB + s * C::kBBytes);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = sm100::sdesc_sw128_kmajor(a_base + kk * 32);
          const uint64_t bd = sm100::sdesc_sw128_kmajor(b_base + kk * 32);
          sm100::mma_f16(tmem, ad, bd, idesc, (kt | kk) != 0 ? 1u : 0u);
        }
        sm100::mma_commit(&empty[s]);
      }
      sm100::mma_commit(accf);
    }
  } else {
    // ---------------- dequantize (warps 2..17), then epilogue ----------------
    const int dq = threadIdx.x - 64;            // 0..511
    constexpr int kTPR = 32 * kDeqWarps / BN;   // threads per B row: 2 or 4
    constexpr int kWords = 8 / kTPR;            // packed words per thread per k-tile
    const int r = dq / kTPR;
    const int w0 = (dq % kTPR) * kWords;
    const int n = n0 + r;
    const int ng = K / G;
    const int tiles_per_group = G / BK;
    // group parameters are loaded one group ahead of their use
    const __half* srow = scales + (int64_t)n * ng;
    const __half* zrow = zeros + (int64_t)n * ng;
    __half s_next = srow[0], z_next = zrow[0];
    uint32_t zb2 = 0, s2 = 0;
    bool ok = true;
    for (int kt = 0; kt < KT && ok; ++kt) {
      const int s = kt % ST;
      const uint32_t ph = (uint32_t)(kt / ST) & 1u;
      if (kt % tiles_per_group == 0) {
        const int gi = kt / tiles_per_group;
        const uint32_t sb = __half_as_ushort(s_next);
        const uint32_t zq = (uint32_t)__half2float(z_next);
        s2 = sb | (sb << 16);
        zb2 = (0x6400u | zq) * 0x00010001u;  // fp16x2 (1024 + z, 1024 + z)
        if (gi + 1 < ng) {
          s_next = srow[gi + 1];
          z_next = zrow[gi + 1];
        }
      }
      const bool got = sm100::mbar_wait(&full[s], ph, &g_gemm_error, 0x301u, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      const uint32_t* wsrc =
          reinterpret_cast<const uint32_t*>(sW + s * C::kWBytes) + r * 8 + w0;
      uint8_t* bdst = sB + s * C::kBBytes + r * 128;
      uint32_t ws[kWords];
      if (kWords == 4) {
        const uint4 wv = *reinterpret_cast<const uint4*>(wsrc);
        ws[0] = wv.x; ws[1] = wv.y; ws[2 % kWords] = wv.z; ws[3 % kWords] = wv.w;
      } else {
        const uint2 wv = *reinterpret_cast<const uint2*>(wsrc);
        ws[0] = wv.x; ws[1] = wv.y;
      }
#pragma unroll
      for (int j = 0; j < kWords; ++j) {
        const int c = w0 + j;  // 16-byte chunk index within the 128-byte row
        const uint4 o = dequant_word(ws[j], zb2, s2);
        *reinterpret_cast<uint4*>(bdst + ((c ^ (r & 7)) << 4)) = o;
      }
      sm100::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(&deq[s]);
    }
    // ---------------- epilogue ----------------
    if (ok) ok = sm100::mbar_wait(accf, 0, &g_gemm_error, 0x401u, abort_flag);
    if (__all_sync(0xffffffffu, ok)) {
      sm100::tc_fence_after();
      const int q = warp & 3;              // TMEM lane quarter this warp may read
      const int slice = (warp - 2) >> 2;   // which quarter of the columns
      const int row = 32 * q + lane;
      const int m = m0 + row;
      const float rs = m < M ? inv_scale[m] : 0.0f;  // 2^-e of this row
#pragma unroll
      for (int c = 0; c < BN / 128; ++c) {
        const int col0 = slice * (BN / 4) + 32 * c;
        uint32_t v[32];
        sm100::tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)col0, v);
        sm100::tmem_ld_wait();
        if (m < M) {
          uint16_t* dst = y + (int64_t)m * N + n0 + col0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]) * rs, __uint_as_float(v[8 * i + 1]) * rs);
            o.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]) * rs, __uint_as_float(v[8 * i + 3]) * rs);
            o.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]) * rs, __uint_as_float(v[8 * i + 5]) * rs);
            o.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]) * rs, __uint_as_float(v[8 * i + 7]) * rs);
            *reinterpret_cast<uint4*>(dst + 8 * i) = o;
          }
        }
      }
    }
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, BN);
  }
}

template <int BN>
wq_status launch_bn(const void* x16, const float* inv_scale, int64_t M, int64_t N, int64_t K,
                    int32_t G, const void* qweight, const void* scales, const void* zeros, void* y,
                    cudaStream_t st) {
  CUtensorMap tx, tw;
  if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x16, (uint64_t)K, (uint64_t)M,
                    (uint64_t)K * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B))
    return WQ_ERR_CUDA;
  if (!make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight, (uint64_t)K / 8, (uint64_t)N,
                    (uint64_t)K / 2, BK / 8, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return WQ_ERR_CUDA;
  using C = GemmCfg<BN>;
  auto kern = w4a16_gemm_kernel<BN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
      cudaSuccess)
    return WQ_ERR_CUDA;
  dim3 grid((unsigned)(N / BN), (unsigned)((M + BM - 1) / BM));
  kern<<<grid, kThreads, C::kSmem, st>>>(tx, tw, static_cast<const __half*>(scales),
                                         static_cast<const __half*>(zeros), inv_scale,
                                         static_cast<uint16_t*>(y), (int)M, (int)N, (int)K, G);
  return launch_status();
}

}  // namespace

// Workspace: the fp16 copy of x [M, K] (256-byte aligned), then 2^-e per row.
size_t gemm_workspace_bytes(int64_t M, int64_t K) {
  return ((size_t)M * K * 2 + 255) / 256 * 256 + (size_t)M * 4;
}

wq_status launch_gemm(const void* x, int64_t M, int64_t N, int64_t K, int32_t G,
                      const void* qweight, const void* scales, const void* zeros, void* y,
                      void* workspace, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* x16 = ws;
  float* inv_scale = reinterpret_cast<float*>(ws + ((size_t)M * K * 2 + 255) / 256 * 256);
  wq_status s = launch_x_to_f16(x, M, K, x16, inv_scale, st);
  if (s != WQ_OK) return s;
  // 256-wide tiles when they alone fill the machine, else 128-wide ones.
  const int64_t mt = (M + BM - 1) / BM;
  const bool wide = (N % 256 == 0) && (mt * (N / 256) >= (int64_t)num_sms());
  return wide ? launch_bn<256>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st)
              : launch_bn<128>(x16, inv_scale, M, N, K, G, qweight, scales, zeros, y, st);
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
