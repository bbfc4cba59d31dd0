// Shared pieces of the decode (M <= 16) kernels: the W4A16 GEMV and the
// Multi-Scale Dequant GEMV. Both give every CTA one weight tile of ROWS rows
// (16 per warp: 256 for the GEMV, 128 for the MSD GEMV) over one K-chunk,
// split K across a thread-block cluster, and reduce the fp32 partials through
// distributed shared memory.
#pragma once

#include <mutex>

#include "common.cuh"

namespace wq {
namespace splitk {

constexpr int kRowsPerCta = 128;  // default tile: 8 warps x 16 rows
constexpr int kMaxSplit = 16;  // cluster size limit (non-portable above 8)

// n / d without a divide: umulhi(n, floor(2^32 / d) + 1) is exact whenever
// n * d < 2^32 (d >= 2).
__host__ __device__ __forceinline__ uint32_t div_magic(uint32_t d) {
  return d < 2 ? 0u : (uint32_t)(0xFFFFFFFFu / d) + 1u;
}
__device__ __forceinline__ int div_by_magic(int n, uint32_t magic) {
  return magic ? (int)__umulhi((uint32_t)n, magic) : n;
}

// Cluster barrier that publishes this CTA's shared-memory writes to the others.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ uint32_t map_rank(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_f32x2(uint32_t addr, float a, float b) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}

// 16-byte asynchronous global -> shared copy (L2 only), and its completion.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// The weight stream. Each warp owns 16 rows and streams them through a ring
// of kStages shared-memory stages of 256 k: 16 rows x 128 contiguous bytes
// (two 128-k units). Measured on B200, 128 or more contiguous bytes per row
// and request stream a row-strided matrix at 6 TB/s, where 64-byte pieces
// (one unit per request) reach far less. A stage is copied by 16-byte
// cp.async (one warp instruction covers 4 rows x 128 bytes), issued
// kStages - 1 stages ahead of the one computed and awaited with
// cp.async.wait_group, so the copies of later stages stay in flight while a
// stage is computed whatever the compute costs. Chunk c (16 bytes) of row r
// is stored at chunk c ^ swz(r): the fragment reads of a warp then hit
// distinct banks (wide: each 8-lane phase reads two rows of different parity;
// narrow: each 16-lane phase reads four rows 0..3 mod 4).
// The group parameters of a stage are loaded into registers when its copies
// are issued.
// ---------------------------------------------------------------------------
constexpr int kStageRowBytes = 128;            // per row per stage (256 k)
constexpr int kStageBytes = 16 * kStageRowBytes;  // per warp per stage

template <bool kWide>
__device__ __forceinline__ int swz(int r) {
  return kWide ? 4 * (r & 1) : 2 * (r & 3);
}

// Copies of stage (units ub, ub + 1; only ub when one = true) of the warp's
// 16 rows starting at wtile into slot.
template <bool kWide>
__device__ __forceinline__ void issue_stage(uint8_t* slot, const uint8_t* wtile,
                                            int64_t row_bytes, int ub, bool one, int lane) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q = 32 * i + lane, r = q >> 3, c = q & 7;
    if (!one || c < 4)
      cp_async16(slot + r * kStageRowBytes + ((c ^ swz<kWide>(r)) << 4),
                 wtile + (int64_t)r * row_bytes + (int64_t)ub * 64 + 16 * c);
  }
}

// Unit h (128 k) of a stage slot: this lane's bytes of rows g and g + 8.
//   wide  : w[0..3] = 16 bytes of row g at byte 16t of the unit, w[4..7] the
//           same of row g + 8;
//   narrow: w[0..1] row g, bytes 8t .. 8t + 7, w[2..3] row g, bytes
//           32 + 8t .., w[4..7] the same of row g + 8.
template <bool kWide>
__device__ __forceinline__ void read_stage_unit(uint32_t (&w)[8], const uint8_t* slot, int h, int g,
                                                int t) {
  const uint8_t* ra = slot + g * kStageRowBytes;
  const uint8_t* rb = slot + (g + 8) * kStageRowBytes;
  const int sw = swz<kWide>(g);  // rows g and g + 8 share it
  if (kWide) {
    const int c = ((4 * h + t) ^ sw) << 4;
    const uint4 a = *reinterpret_cast<const uint4*>(ra + c);
    const uint4 b = *reinterpret_cast<const uint4*>(rb + c);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
    const int c0 = (((4 * h + (t >> 1)) ^ sw) << 4) + 8 * (t & 1);
    const int c1 = (((4 * h + 2 + (t >> 1)) ^ sw) << 4) + 8 * (t & 1);
    const uint2 a0 = *reinterpret_cast<const uint2*>(ra + c0);
    const uint2 a1 = *reinterpret_cast<const uint2*>(ra + c1);
    const uint2 b0 = *reinterpret_cast<const uint2*>(rb + c0);
    const uint2 b1 = *reinterpret_cast<const uint2*>(rb + c1);
    w[0] = a0.x; w[1] = a0.y; w[2] = a1.x; w[3] = a1.y;
    w[4] = b0.x; w[5] = b0.y; w[6] = b1.x; w[7] = b1.y;
  }
}

// Rows of a ROWS-row tile are split over the S ranks of a cluster as
// [b(r), b(r + 1)) with b(r) = floor(ROWS r / S); the owner of row is the r
// with b(r) <= row < b(r + 1).
template <int ROWS = kRowsPerCta>
__host__ __device__ __forceinline__ int rank_row_begin(int r, int S) { return r * ROWS / S; }
template <int ROWS = kRowsPerCta>
__device__ __forceinline__ int row_owner(int row, int S) {
  return ((row + 1) * S + ROWS - 1) / ROWS - 1;
}

// Shared-memory bytes of the reduction buffer red[S ranks][ceil(ROWS/S)][16].
template <int ROWS = kRowsPerCta>
__host__ __device__ __forceinline__ size_t red_bytes(int S) {
  return (size_t)S * ((ROWS + S - 1) / S) * 16 * 4;
}

// Optional salient-channel residual correction ("DecDEC: A Systems Approach
// to Advancing Low-Bit LLM Quantization", Abstract), added to an output in
// fp32 before its bf16 rounding: y[m, n] += sum_j x[m, idx[j]] * R^T[idx[j], n]
// with R^T fp16 [K, N] (a selected channel's residuals are one contiguous
// row, so the owners' loads of consecutive n coalesce). k == 0 adds nothing.
struct Residual {
  const uint16_t* rt = nullptr;  // fp16 bits of R^T [K, N]
  const int* idx = nullptr;      // k channel indices
  const uint16_t* x = nullptr;   // bf16 bits of x [M, K]
  int k = 0;
  int K = 0;
};

// Items (token, owned row) per thread in the owners' epilogue: nrows * M is
// at most ROWS * 16 over 2 * ROWS threads (8 warps per 128 rows).
constexpr int kMaxItemsPerThread = 8;

// This thread's part of the correction of its items (token tok[it], row
// n[it]; n < 0 for none): channels j = j0, j0 + L, j0 + 2L, ... in batches
// of 8, the 8 indices loaded once per batch for all items, then every item's
// x and residual loads, all independent.
__device__ __forceinline__ void residual_parts(const Residual& rc, const int (&tok)[kMaxItemsPerThread],
                                               const int (&n)[kMaxItemsPerThread], int N, int j0,
                                               int L, float (&out)[kMaxItemsPerThread]) {
  int j = j0;
  for (; j + 7 * L < rc.k; j += 8 * L) {
    int c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = __ldg(rc.idx + j + i * L);
#pragma unroll
    for (int it = 0; it < kMaxItemsPerThread; ++it) {
      if (n[it] < 0) continue;
      const uint16_t* xr = rc.x + (size_t)tok[it] * rc.K;
      float xv[8], r[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        xv[i] = __uint_as_float((uint32_t)__ldg(xr + c[i]) << 16);
        r[i] = __half2float(__ushort_as_half(__ldg(rc.rt + (size_t)c[i] * N + n[it])));
      }
      float v = out[it];
#pragma unroll
      for (int i = 0; i < 8; ++i) v = fmaf(xv[i], r[i], v);
      out[it] = v;
    }
  }
  for (; j < rc.k; j += L) {
    const int c = __ldg(rc.idx + j);
#pragma unroll
    for (int it = 0; it < kMaxItemsPerThread; ++it) {
      if (n[it] < 0) continue;
      out[it] = fmaf(__uint_as_float((uint32_t)__ldg(rc.x + (size_t)tok[it] * rc.K + c) << 16),
                     __half2float(__ushort_as_half(__ldg(rc.rt + (size_t)c * N + n[it]))),
                     out[it]);
    }
  }
}


// The cluster split-K reduction. acc[a][r] of this lane holds rows
// warp*16 + g + 8 (r >> 1), tokens 8a + 2t + (r & 1) (the m16n8 accumulator
// layout); tok_scale (optional, per token) multiplies it first. Each CTA
// pushes its partials into the shared memory of the rank that owns the rows
// (red[src rank][local row][token] there), one cluster barrier, then each
// owner sums its rows in rank order and writes them once as bf16. Remote
// stores need no round trip, and no CTA touches another's shared memory after
// the barrier. With kRes the owners add the residual correction rc (k >= 1)
// before the rounding. All threads of the CTA must call this.
template <int NT, bool kRes = false, int ROWS = kRowsPerCta>
__device__ __forceinline__ void reduce_and_store(const float (&acc)[NT][4], const float* tok_scale,
                                                 float* red, int S, int rank, int row_tile, int M,
                                                 int N, uint16_t* y,
                                                 const Residual& rc = Residual()) {
  static_assert(ROWS * 16 <= 2 * ROWS * kMaxItemsPerThread, "items per thread");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int rows_max = (ROWS + S - 1) / S;
#pragma unroll
  for (int a = 0; a < NT; ++a)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int row = warp * 16 + g + 8 * hr;
      const int owner = row_owner<ROWS>(row, S);
      const int lr = row - rank_row_begin<ROWS>(owner, S);
      const int tok = 8 * a + 2 * t;
      float v0 = acc[a][2 * hr], v1 = acc[a][2 * hr + 1];
      if (tok_scale) {
        v0 *= tok_scale[tok];
        v1 *= tok_scale[tok + 1];
      }
      float* dst = red + ((size_t)rank * rows_max + lr) * 16 + tok;
      if (S > 1) {
        st_cluster_f32x2(map_rank(dst, (uint32_t)owner), v0, v1);
      } else {
        dst[0] = v0;
        dst[1] = v1;
      }
    }
  const int r_begin = rank_row_begin<ROWS>(rank, S);
  const int nrows = rank_row_begin<ROWS>(rank + 1, S) - r_begin;
  const int items = nrows * M;
  if constexpr (!kRes) {
    if (S > 1) {
      cluster_sync_all();
    } else {
      __syncthreads();
    }
    for (int i = tid; i < items; i += blockDim.x) {
      const int tok = i / nrows;
      const int lr = i - tok * nrows;
      const int n = row_tile + r_begin + lr;
      float v = 0.0f;
      for (int q = 0; q < S; ++q) v += red[((size_t)q * rows_max + lr) * 16 + tok];
      if (n < N) y[(int64_t)tok * N + n] = (uint16_t)(pack_bf16x2(v, 0.0f) & 0xFFFFu);
    }
  } else {
    // When this grid was launched early after the channel selection
    // (programmatic dependent launch), wait for it before reading idx; a no-op
    // otherwise.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // Item (token, owned row) i is handled by the L consecutive lanes of slot
    // i mod slots: with fewer items than threads, each item's k channels are
    // split over L lanes (a power of two up to 32) and summed by shuffles.
    // The correction is computed before the cluster barrier, while the other
    // ranks may still be pushing their partials.
    int L = 1;
    while (L < 32 && items * (2 * L) <= (int)blockDim.x) L *= 2;
    const int slots = (int)blockDim.x / L, slot = tid / L, sub = tid % L;
    float corr[kMaxItemsPerThread];
    int c_tok[kMaxItemsPerThread], c_n[kMaxItemsPerThread];
#pragma unroll
    for (int it = 0; it < kMaxItemsPerThread; ++it) {
      corr[it] = 0.0f;
      const int i = slot + it * slots;
      c_tok[it] = 0;
      c_n[it] = -1;
      if (i < items) {
        const int tok = i / nrows;
        const int n = row_tile + r_begin + (i - tok * nrows);
        if (n < N) {
          c_tok[it] = tok;
          c_n[it] = n;
        }
      }
    }
    residual_parts(rc, c_tok, c_n, N, sub, L, corr);
    if (L > 1) {
#pragma unroll
      for (int it = 0; it < kMaxItemsPerThread; ++it)
        for (int o = L / 2; o > 0; o >>= 1) corr[it] += __shfl_xor_sync(0xffffffffu, corr[it], o);
    }
    if (S > 1) {
      cluster_sync_all();
    } else {
      __syncthreads();
    }
#pragma unroll
    for (int it = 0; it < kMaxItemsPerThread; ++it) {
      const int i = slot + it * slots;
      if (sub != 0 || i >= items) break;
      const int tok = i / nrows;
      const int lr = i - tok * nrows;
      const int n = row_tile + r_begin + lr;
      float v = corr[it];
      for (int q = 0; q < S; ++q) v += red[((size_t)q * rows_max + lr) * 16 + tok];
      if (n < N) y[(int64_t)tok * N + n] = (uint16_t)(pack_bf16x2(v, 0.0f) & 0xFFFFu);
    }
  }
}

struct Plan {
  int S = 0;
  int kc = 0;
  size_t smem = 0;
  int resident = 0;  // S-CTA clusters resident at once (persistent launches)
};

// Cluster size S (K split): every CTA holds one 128-row tile over one K-chunk
// of kc = ceil(units / S) * 128. S (1..16, at most one 128-k unit per CTA,
// fits(kc) true) minimises the K streamed per CTA slot plus fixed costs, in
// k: waves x (kc + 512 for staging x and the reduction), since a wave lasts
// as long as its CTAs' K-chunks (two waves of half-K CTAs beat two waves of
// full-K ones). A persistent kernel (each resident cluster loops over row
// tiles and stages its x chunk once) pays the staging once: 512 once plus
// waves x (kc + 256). Ties go to the fuller GPU. smem_of(kc, S) gives the
// CTA's dynamic shared memory.
template <class Kern, class Fits, class SmemOf>
Plan make_plan(Kern kern, int threads, int64_t N, int64_t K, Fits fits, SmemOf smem_of,
               bool persistent = false, int rows = kRowsPerCta) {
  const int64_t tiles = (N + rows - 1) / rows;
  const int64_t units = K / 128;
  cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaGetLastError();
  double best = -1e30;
  Plan bp;
  for (int S = 1; S <= kMaxSplit; ++S) {
    if (S > units) break;
    const int kc = (int)((units + S - 1) / S) * 128;
    if (!fits(kc)) continue;
    const size_t smem = smem_of(kc, S);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
      cudaGetLastError();
      continue;
    }
    int slots = 0;
    if (S == 1) {
      int per_sm = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) !=
          cudaSuccess) {
        cudaGetLastError();
        continue;
      }
      slots = per_sm * num_sms();
    } else {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)S, (unsigned)tiles, 1);
      cfg.blockDim = dim3((unsigned)threads, 1, 1);
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
    const double per_wave = persistent ? 256.0 : 512.0, once = persistent ? 512.0 : 0.0;
    const double fill = (double)grid / ((double)waves * slots);
    const double score = -((double)waves * ((double)kc + per_wave) + once) + 1e-3 * fill;
    if (score > best + 1e-9) {
      best = score;
      bp.S = S;
      bp.kc = kc;
      bp.smem = smem;
      bp.resident = slots / S;
    }
  }
  return bp;
}

// Plans are cached per (kernel, device, M, N, K, extra): the occupancy
// queries cost far more host time than the launch itself.
template <class MakeFn>
Plan cached_plan(const void* kern, int M, int64_t N, int64_t K, int extra, MakeFn make) {
  struct Entry {
    const void* kern;
    int dev, M, extra;
    int64_t N, K;
    Plan plan;
  };
  constexpr int kEntries = 128;
  static Entry cache[kEntries];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return Plan{};
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].kern == kern && cache[i].dev == dev && cache[i].M == M && cache[i].N == N &&
        cache[i].K == K && cache[i].extra == extra)
      return cache[i].plan;
  const Plan pl = make();
  if (pl.S > 0 && used < kEntries) cache[used++] = Entry{kern, dev, M, extra, N, K, pl};
  return pl;
}

// Launch `kern` on the plan's (S x row tiles) grid with S-CTA clusters.
// persistent: the grid has at most pl.resident clusters along y, each looping
// over the row tiles y, y + gridDim.y, ...
template <class Kern, class Args>
wq_status launch_split(Kern kern, const Plan& pl, int threads, int64_t N, cudaStream_t st,
                       const Args& args, const Nf4Table& tab, bool persistent = false,
                       bool early = false, int rows = kRowsPerCta) {
  // the attribute is a per-function maximum; plans of other shapes may have
  // set a smaller one since
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem) !=
      cudaSuccess)
    return WQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  const int64_t tiles = (N + rows - 1) / rows;
  const int64_t gy = persistent && pl.resident > 0 && pl.resident < tiles ? pl.resident : tiles;
  cfg.gridDim = dim3((unsigned)pl.S, (unsigned)gy, 1);
  cfg.blockDim = dim3((unsigned)threads, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)pl.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // early: programmatic dependent launch after the preceding kernel, which
  // must only read what this kernel reads before its griddepcontrol.wait
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = early ? 2 : 1;
  if (cudaLaunchKernelEx(&cfg, kern, args, tab) != cudaSuccess) return WQ_ERR_CUDA;
  return launch_status();
}

}  // namespace splitk
}  // namespace wq
