// Multi-Scale Dequant in decode attention over an INT4 KV cache.
//
// Source: "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
// Activation Decomposition for Efficient LLM Inference", Abstract: MSD removes
// the KV dequantization from the attention products (the quantized cache
// multiplies low-precision components of the other operand directly), which
// cuts the cache's HBM traffic in attention.
//
// Per sequence b, KV head kh and its R query heads (decode: one query token):
//   scores  s[l] = D^-1/2 sk[l] sum_c sig_c (sum_d a_c[d] qk[l, d] - zk[l] sum_d a_c[d])
//           with a_c the int8 digit planes of the query row (the activation
//           decomposition) and qk the K codes: exact integer dot products;
//   softmax in chunks of 256 keys: m_j = max s, e = exp(s - m_j), E_j = sum e;
//   values  w[l] = e[l] sv[l] decomposed per chunk into int8 digits b_c (the
//           same decomposition, the chunk's keys as one row);
//           O_j[d] = sum_c tau_c (sum_l b_c[l] qv[l, d] - sum_l b_c[l] zv[l]),
//           exact integer sums;
//   merge   out = sum_j e^(m_j - M) O_j / sum_j e^(m_j - M) E_j.
// The cache rows use the INT4 asymmetric quantizer with one group per row
// (group = D = 128): codes uint32 [B, Hkv, L, 16] (low nibble first), fp16
// scales and integer zeros [B, Hkv, L].
//
// B200 design. Decode attention reads the cache once, so the kernel is bound
// by HBM and the products only have to keep up: both are integer tensor-core
// products (mma.m16n8k32, s8 digits x u8 codes). One CTA per (256-key chunk,
// KV head, sequence) copies its K and V code rows into shared memory with
// 16-byte cp.async, issued before it waits for the query decomposition (a
// programmatic dependent launch). The R x C digit rows of the query are the
// A operand (M = 16 rows, the unused ones zero):
//   scores: N = keys, K = d. A K code word unpacks to two u8 words (even d,
//           odd d); the query digits are stored in that order, so the
//           contraction order matches without moving the codes;
//   values: N = d, K = keys. The B fragment wants four keys of one d in a
//           register: three byte permutes gather them from four code rows.
//           The keys of a 32-key step are taken in the order that makes those
//           row reads conflict-free, and the value digits are stored in the
//           same order.
// Each warp owns 16 output elements over all 256 keys, so no cross-warp
// reduction is needed; the chunk's partial O_j and (m_j, E_j) go to the
// workspace and a second kernel merges the chunks.
#include "splitk_common.cuh"

namespace wq {
namespace {

using namespace splitk;

constexpr int kD = 128;                  // head dimension
constexpr int kT = 256;                  // keys per chunk
constexpr int kRowBytes = kD / 2;        // 64 bytes of codes per key
constexpr int kQwStride = kD / 4 + 4;    // words per query digit row (padded)
constexpr int kBdStride = kT + 16;       // bytes per value digit row (padded)

// shared memory carve-up (bytes)
constexpr int kOffK = 0;                                  // K codes, later P
constexpr int kOffV = kOffK + kT * kRowBytes;             // V codes
constexpr int kOffBd = kOffV + kT * kRowBytes;            // value digits [16][kBdStride]
constexpr int kOffSc = kOffBd + 16 * kBdStride;           // sk, sv (fp32), zk, zv (int)
constexpr int kOffQw = kOffSc + 4 * kT * 4;               // query digits [16][kQwStride]
constexpr int kOffQm = kOffQw + 16 * kQwStride * 4;       // qsig, qsum, tau, zt: [16] each
constexpr int kOffRed = kOffQm + 4 * 16 * 4;              // [8 warps][16]
constexpr int kSmemBytes = kOffRed + 8 * 16 * 4;
static_assert(kSmemBytes <= 48 * 1024, "static shared memory");
static_assert(16 * kT * 4 <= kT * kRowBytes, "P fits the K buffer");

// 16-byte chunk c (0..3) of key row l is stored at chunk c ^ ((l >> 1) & 3).
__device__ __forceinline__ int kv_off(int l, int c) {
  return l * kRowBytes + ((c ^ ((l >> 1) & 3)) << 4);
}
// P[hc][l] (int) at word hc * kT + (l ^ ((hc & 3) << 3)).
__device__ __forceinline__ int p_idx(int hc, int l) { return hc * kT + (l ^ ((hc & 3) << 3)); }
// Column of key kk (0..255) in the value digit rows: within each 16-key half
// of a 32-key step, key t + 4 i sits at slot 4 t + i (t, i in 0..3).
__device__ __forceinline__ int bd_col(int kk) {
  return (kk & ~15) + 4 * (kk & 3) + ((kk >> 2) & 3);
}

__device__ __forceinline__ void mma_s8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct KvArgs {
  const int8_t* qd;       // [C][B*Hq][D] query digits
  const float* qs;        // [C][B*Hq] their scales
  const uint8_t* kq;      // K codes [B, Hkv, L, D/2]
  const __half* ks;       // [B, Hkv, L]
  const __half* kz;
  const uint8_t* vq;      // V codes
  const __half* vs;
  const __half* vz;
  float* part;            // [B, Hkv, nch, R, D] chunk outputs O_j
  float* stat;            // [B, Hkv, nch, R, 2] (m_j, E_j)
  int B, Hq, Hkv, L, nch;
  float inv_sqrt_d;
};

// v[i] combined over the CTA (256 threads); red holds [8][N] values; every
// thread receives the result.
template <int N, typename T, typename Op>
__device__ __forceinline__ void block_all(T (&v)[N], T* red, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[i] = op(v[i], __shfl_xor_sync(0xffffffffu, v[i], o));
  __syncthreads();
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < N; ++i) red[warp * N + i] = v[i];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < N; ++i) {
    T a = red[i];
#pragma unroll
    for (int w = 1; w < 8; ++w) a = op(a, red[w * N + i]);
    v[i] = a;
  }
}

template <int R, int C>
__global__ void __launch_bounds__(256, 3) kv_msd_chunk_kernel(KvArgs p) {
  constexpr int RC = R * C;
  static_assert(RC <= 16, "at most 16 digit rows");
  __shared__ __align__(16) uint8_t sm[kSmemBytes];
  uint8_t* kc = sm + kOffK;
  uint8_t* vc = sm + kOffV;
  int* P = reinterpret_cast<int*>(sm + kOffK);
  int8_t* bd = reinterpret_cast<int8_t*>(sm + kOffBd);
  float* skf = reinterpret_cast<float*>(sm + kOffSc);
  float* svf = skf + kT;
  int* zki = reinterpret_cast<int*>(svf + kT);
  int* zvi = zki + kT;
  uint32_t* qw = reinterpret_cast<uint32_t*>(sm + kOffQw);
  float* qsig = reinterpret_cast<float*>(sm + kOffQm);
  int* qsum = reinterpret_cast<int*>(qsig + 16);
  float* tau = reinterpret_cast<float*>(qsum + 16);
  int* zt = reinterpret_cast<int*>(tau + 16);
  float* redf = reinterpret_cast<float*>(sm + kOffRed);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int j = blockIdx.x, kh = blockIdx.y, b = blockIdx.z;
  const int l0 = j * kT;
  const int nk = min(kT, p.L - l0);
  const int64_t row0 = ((int64_t)b * p.Hkv + kh) * p.L + l0;  // first cache row of the chunk

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // ---- the chunk's K and V code rows; the cache is not written by the grid
  // this one may overlap, so the copies go before the wait
  for (int i = tid; i < nk * 4; i += 256) {
    const int l = i >> 2, c = i & 3;
    cp_async16(kc + kv_off(l, c), p.kq + (row0 + l) * kRowBytes + 16 * c);
    cp_async16(vc + kv_off(l, c), p.vq + (row0 + l) * kRowBytes + 16 * c);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  if (tid < nk) {
    skf[tid] = __half2float(p.ks[row0 + tid]);
    svf[tid] = __half2float(p.vs[row0 + tid]);
    zki[tid] = (int)__half2float(p.kz[row0 + tid]);
    zvi[tid] = (int)__half2float(p.vz[row0 + tid]);
  }
  // ---- the query digits of this KV head's R query heads (rows hc = h C + c)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int qrow0 = b * p.Hq + kh * R;
  const int64_t plane = (int64_t)p.B * p.Hq;
  if (tid < RC * (kD / 8)) {
    const int hc = tid >> 4, g8 = tid & 15;
    const int h = hc / C, c = hc - h * C;
    const uint2 v =
        *reinterpret_cast<const uint2*>(p.qd + ((int64_t)c * plane + qrow0 + h) * kD + 8 * g8);
    qw[hc * kQwStride + 2 * g8] = prmt(v.x, v.y, 0x6420u);      // d = 8 g8 + 0, 2, 4, 6
    qw[hc * kQwStride + 2 * g8 + 1] = prmt(v.x, v.y, 0x7531u);  // d = 8 g8 + 1, 3, 5, 7
  }
  if (tid < RC) {
    const int h = tid / C, c = tid - h * C;
    qsig[tid] = p.qs[(int64_t)c * plane + qrow0 + h];
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  if (tid < RC) {
    int s = 0;
    for (int i = 0; i < kD / 4; ++i) s = __dp4a((int)qw[tid * kQwStride + i], 0x01010101, s);
    qsum[tid] = s;
  }

  // ---- scores: warp w takes keys 32 w .. 32 w + 31 (four n-tiles of 8 keys)
  int sacc[4][4];
  {
    uint32_t a[4][4];  // [k-step][fragment register]
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      a[s][0] = g < RC ? qw[g * kQwStride + 8 * s + t4] : 0u;
      a[s][1] = g + 8 < RC ? qw[(g + 8) * kQwStride + 8 * s + t4] : 0u;
      a[s][2] = g < RC ? qw[g * kQwStride + 8 * s + 4 + t4] : 0u;
      a[s][3] = g + 8 < RC ? qw[(g + 8) * kQwStride + 8 * s + 4 + t4] : 0u;
    }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) sacc[nt][i] = 0;
      const int l = 32 * warp + 8 * nt + g;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint32_t* ch = reinterpret_cast<const uint32_t*>(kc + kv_off(l, s));
        const uint32_t w0 = ch[t4 >> 1], w1 = ch[2 + (t4 >> 1)];
        const int sh = 4 * (t4 & 1);
        mma_s8u8(sacc[nt], a[s][0], a[s][1], a[s][2], a[s][3], (w0 >> sh) & 0x0F0F0F0Fu,
                 (w1 >> sh) & 0x0F0F0F0Fu);
      }
    }
  }
  __syncthreads();  // every warp is done with the K codes: P takes their place
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    const int l = 32 * warp + 8 * nt + 2 * t4;
    *reinterpret_cast<int2*>(P + p_idx(g, l)) = make_int2(sacc[nt][0], sacc[nt][1]);
    *reinterpret_cast<int2*>(P + p_idx(g + 8, l)) = make_int2(sacc[nt][2], sacc[nt][3]);
  }
  __syncthreads();

  // ---- softmax statistics of the chunk; thread tid takes key tid
  const bool valid = tid < nk;
  float m[R], es[R], am[R], w[R];
#pragma unroll
  for (int h = 0; h < R; ++h) {
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const int hc = h * C + c;
      const int dint = P[p_idx(hc, tid)] - (valid ? zki[tid] : 0) * qsum[hc];  // |.| < 2^24
      s = fmaf(qsig[hc], (float)dint, s);
    }
    m[h] = valid ? s * skf[tid] * p.inv_sqrt_d : -INFINITY;
    w[h] = m[h];
  }
  block_all<R>(m, redf, [](float x, float y) { return fmaxf(x, y); });
#pragma unroll
  for (int h = 0; h < R; ++h) {
    const float e = valid ? expf(w[h] - m[h]) : 0.0f;
    es[h] = e;
    w[h] = e * (valid ? svf[tid] : 0.0f);
    am[h] = fabsf(w[h]);
  }
  block_all<R>(es, redf, [](float x, float y) { return x + y; });
  const int64_t base = (((int64_t)b * p.Hkv + kh) * p.nch + j) * R;
#pragma unroll
  for (int h = 0; h < R; ++h)
    if (tid == h) *reinterpret_cast<float2*>(p.stat + (base + h) * 2) = make_float2(m[h], es[h]);
  block_all<R>(am, redf, [](float x, float y) { return fmaxf(x, y); });
  // the decomposition of w over the chunk's keys, as for an activation row:
  // s_1 = amax / 127, s_{c+1} = s_c / 256, digit rint(r / s_c) (the first
  // clamped to +-127), residual r - s_c a_c rounded once, and a digit of +128
  // becomes -128 with a carry into the digit before it. Thread h computes
  // head h's scales once.
#pragma unroll
  for (int h = 0; h < R; ++h)
    if (tid == h) {
      float sc = am[h] > 0.0f ? __fdiv_rn(am[h], 127.0f) : 1.0f;
#pragma unroll
      for (int c = 0; c < C; ++c, sc *= (1.0f / 256.0f)) tau[h * C + c] = sc;
    }
  __syncthreads();
  {
    const int col = bd_col(tid);
#pragma unroll
    for (int h = 0; h < R; ++h) {
      int dg[C];
      float r = w[h];
#pragma unroll
      for (int c = 0; c < C; ++c) {
        const float sc = tau[h * C + c];
        float q = rintf(__fdiv_rn(r, sc));
        if (c == 0) q = fminf(fmaxf(q, -127.0f), 127.0f);
        dg[c] = (int)q;
        r = __fmaf_rn(-sc, q, r);
      }
#pragma unroll
      for (int c = C - 1; c > 0; --c)
        if (dg[c] == 128) {
          dg[c] = -128;
          dg[c - 1] += 1;
        }
#pragma unroll
      for (int c = 0; c < C; ++c) bd[(h * C + c) * kBdStride + col] = (int8_t)dg[c];
    }
  }
  __syncthreads();
  // the zero terms zt[hc] = sum_l b_c[l] zv[l]: warp w takes digit rows 2 w, 2 w + 1
#pragma unroll
  for (int r2 = 0; r2 < 2; ++r2) {
    const int hc = 2 * warp + r2;
    if (hc < RC) {
      int acc = 0;
#pragma unroll
      for (int i = 0; i < kT / 32; ++i) {
        const int l = lane + 32 * i;
        acc += (int)bd[hc * kBdStride + bd_col(l)] * (l < nk ? zvi[l] : 0);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) zt[hc] = acc;
    }
  }
  __syncthreads();

  // ---- values: warp w owns d in [16 w, 16 w + 16), words wi = 2 w, 2 w + 1
  // of each code row. MMA jm, column n: d = 8 (2 w + (n >> 2)) + (n & 3) + 4 jm.
  int vacc[2][4];
#pragma unroll
  for (int jm = 0; jm < 2; ++jm)
#pragma unroll
    for (int i = 0; i < 4; ++i) vacc[jm][i] = 0;
  {
    const int wi = 2 * warp + (g >> 2);
    const int q = g & 3;
    const int sh = 4 * (q & 1);
    // byte (q >> 1) of two rows into bytes 0, 1 (jm = 0); byte 2 + (q >> 1) (jm = 1)
    const uint32_t sel0 = (uint32_t)((q >> 1) | ((4 + (q >> 1)) << 4));
    const uint32_t sel1 = sel0 + 0x22u;
    const uint32_t* arow0 = reinterpret_cast<const uint32_t*>(bd + g * kBdStride);
    const uint32_t* arow1 = reinterpret_cast<const uint32_t*>(bd + (g + 8) * kBdStride);
#pragma unroll 2
    for (int ks = 0; ks < kT / 32; ++ks) {
      const int k0 = 32 * ks;
      const uint32_t a0 = g < RC ? arow0[(k0 >> 2) + t4] : 0u;
      const uint32_t a1 = g + 8 < RC ? arow1[(k0 >> 2) + t4] : 0u;
      const uint32_t a2 = g < RC ? arow0[(k0 >> 2) + 4 + t4] : 0u;
      const uint32_t a3 = g + 8 < RC ? arow1[(k0 >> 2) + 4 + t4] : 0u;
      uint32_t bb[2][2];  // [jm][key half]
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        uint32_t rw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int l = k0 + 16 * hb + t4 + 4 * i;
          rw[i] = *reinterpret_cast<const uint32_t*>(vc + kv_off(l, wi >> 2) + 4 * (wi & 3));
        }
        const uint32_t x0 = prmt(rw[0], rw[1], sel0), y0 = prmt(rw[2], rw[3], sel0);
        const uint32_t x1 = prmt(rw[0], rw[1], sel1), y1 = prmt(rw[2], rw[3], sel1);
        bb[0][hb] = (prmt(x0, y0, 0x5410u) >> sh) & 0x0F0F0F0Fu;
        bb[1][hb] = (prmt(x1, y1, 0x5410u) >> sh) & 0x0F0F0F0Fu;
      }
      mma_s8u8(vacc[0], a0, a1, a2, a3, bb[0][0], bb[0][1]);
      mma_s8u8(vacc[1], a0, a1, a2, a3, bb[1][0], bb[1][1]);
    }
  }
  // ---- epilogue: O_j[h][d] = sum_c tau_c (acc - zt); the components of a
  // head sit in C consecutive rows, held by lanes 4 apart
#pragma unroll
  for (int jm = 0; jm < 2; ++jm) {
    const int d = 8 * (2 * warp + (t4 >> 1)) + 2 * (t4 & 1) + 4 * jm;  // columns 2 t4, 2 t4 + 1
#pragma unroll
    for (int rh = 0; rh < 2; ++rh) {
      const int hc = g + 8 * rh;
      const int hcs = hc < RC ? hc : 0;
      float o0 = tau[hcs] * (float)(vacc[jm][2 * rh] - zt[hcs]);
      float o1 = tau[hcs] * (float)(vacc[jm][2 * rh + 1] - zt[hcs]);
      if (C == 2) {
        o0 += __shfl_xor_sync(0xffffffffu, o0, 4);
        o1 += __shfl_xor_sync(0xffffffffu, o1, 4);
      }
      if (hc < RC && hc % C == 0)
        *reinterpret_cast<float2*>(p.part + (base + hc / C) * kD + d) = make_float2(o0, o1);
    }
  }
}

// Merge the chunks of each (sequence, query head): out = sum_j e^(m_j - M)
// O_j / sum_j e^(m_j - M) E_j, one CTA of 128 threads (one per element).
template <int R>
__global__ void __launch_bounds__(kD) kv_msd_merge_kernel(KvArgs p, uint16_t* __restrict__ out) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int bh = blockIdx.x;  // b * Hq + hq
  const int b = bh / p.Hq, hq = bh - b * p.Hq;
  const int kh = hq / R, h = hq - kh * R;
  const int d = threadIdx.x;
  const int64_t base = ((int64_t)b * p.Hkv + kh) * p.nch;
  float big = -INFINITY;
  for (int j = 0; j < p.nch; ++j) big = fmaxf(big, p.stat[((base + j) * R + h) * 2]);
  float num = 0.0f, den = 0.0f;
  for (int j = 0; j < p.nch; ++j) {
    const int64_t ri = (base + j) * R + h;
    const float f = expf(p.stat[ri * 2] - big);
    num = fmaf(f, p.part[ri * kD + d], num);
    den = fmaf(f, p.stat[ri * 2 + 1], den);
  }
  out[(int64_t)bh * kD + d] = bf16_bits(num / den);
}

template <int R, int C>
wq_status launch_kv_rc(const KvArgs& a, void* out, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.stream = st;
  cfg.gridDim = dim3((unsigned)a.nch, (unsigned)a.Hkv, (unsigned)a.B);
  cfg.blockDim = dim3(256, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kv_msd_chunk_kernel<R, C>, a) != cudaSuccess) return WQ_ERR_CUDA;
  cfg.gridDim = dim3((unsigned)(a.B * a.Hq), 1, 1);
  cfg.blockDim = dim3(kD, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kv_msd_merge_kernel<R>, a, static_cast<uint16_t*>(out)) !=
      cudaSuccess)
    return WQ_ERR_CUDA;
  return launch_status();
}

template <int C>
wq_status launch_kv_c(const KvArgs& a, int R, void* out, cudaStream_t st) {
  switch (R) {
    case 1: return launch_kv_rc<1, C>(a, out, st);
    case 2: return launch_kv_rc<2, C>(a, out, st);
    case 4: return launch_kv_rc<4, C>(a, out, st);
    default: return launch_kv_rc<8, C>(a, out, st);
  }
}

}  // namespace

wq_status launch_msd_decompose(const void*, int64_t, int64_t, int32_t, int64_t, int8_t*, float*,
                               cudaStream_t);

// Workspace: query digits [C][B*Hq][D] and their scales [C][B*Hq] fp32 (each
// rounded up to 256 bytes), then the chunk outputs [B, Hkv, nch, R, D] and
// statistics [B, Hkv, nch, R, 2] fp32.
size_t kv_msd_workspace_bytes(int64_t B, int64_t Hq, int64_t L, int32_t C) {
  const int64_t nch = (L + kT - 1) / kT;
  const size_t dig = ((size_t)C * B * Hq * kD + 255) / 256 * 256;
  const size_t sc = ((size_t)C * B * Hq * 4 + 255) / 256 * 256;
  return dig + sc + (size_t)B * Hq * nch * (kD + 2) * 4;
}

wq_status launch_kv_msd(const void* q, int64_t B, int64_t Hq, int64_t Hkv, int64_t L, int32_t C,
                        const void* kq, const void* ks, const void* kz, const void* vq,
                        const void* vs, const void* vz, void* out, void* workspace,
                        cudaStream_t st) {
  uint8_t* w = static_cast<uint8_t*>(workspace);
  const int64_t nch = (L + kT - 1) / kT;
  const size_t dig = ((size_t)C * B * Hq * kD + 255) / 256 * 256;
  const size_t sc = ((size_t)C * B * Hq * 4 + 255) / 256 * 256;
  int8_t* qd = reinterpret_cast<int8_t*>(w);
  float* qs = reinterpret_cast<float*>(w + dig);
  float* part = reinterpret_cast<float*>(w + dig + sc);
  float* stat = part + (size_t)B * Hq * nch * kD;
  wq_status s = launch_msd_decompose(q, B * Hq, kD, C, B * Hq, qd, qs, st);
  if (s != WQ_OK) return s;
  KvArgs a;
  a.qd = qd;
  a.qs = qs;
  a.kq = static_cast<const uint8_t*>(kq);
  a.ks = static_cast<const __half*>(ks);
  a.kz = static_cast<const __half*>(kz);
  a.vq = static_cast<const uint8_t*>(vq);
  a.vs = static_cast<const __half*>(vs);
  a.vz = static_cast<const __half*>(vz);
  a.part = part;
  a.stat = stat;
  a.B = (int)B;
  a.Hq = (int)Hq;
  a.Hkv = (int)Hkv;
  a.L = (int)L;
  a.nch = (int)nch;
  a.inv_sqrt_d = 1.0f / sqrtf((float)kD);
  const int R = (int)(Hq / Hkv);
  return C == 1 ? launch_kv_c<1>(a, R, out, st) : launch_kv_c<2>(a, R, out, st);
}

}  // namespace wq
