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
// (group = D = 128), fp16 scales and integer zeros [B, Hkv, L]. K codes are
// stored by token: uint32 [B, Hkv, L, 16], element d in nibble d % 8 of word
// d / 8. V codes are stored in blocks of 8 tokens: uint32 [B, Hkv, ceil(L/8),
// 128], token 8 j + t of dimension d in nibble t of word (j, d) (tokens past
// L zero), so that one word holds 4 keys of one d in its low nibbles and 4 in
// its high nibbles: the operand layout of the value product.
//
// B200 design. Decode attention reads the cache once, so the kernel is bound
// by HBM when its per-key work keeps up. Both products are integer
// tensor-core MMAs (mma.m16n8k32, s8 digits x u8 codes) with the R x C query
// digit rows as the A operand (M = 16, unused rows zero):
//   scores: N = keys, K = d. One K code word (8 d of one key) gives both B
//           registers of a lane: its low nibbles (even d) and high nibbles
//           (odd d); the query digits are stored in that k order. Column n of
//           n-tile t of warp w is key 32 w + 8 (n >> 1) + 2 t + (n & 1), so
//           the accumulator fragment gives each lane the 8 keys of one V
//           block, whose value digits pack into two 32-bit words per digit
//           row;
//   values: N = d, K = keys. One V code word (8 keys of one d) gives both B
//           registers of a lane, low and high nibbles, and the value digits
//           are stored in that k order; the digit rows (A) come in by
//           ldmatrix. The zero terms sum_l b_c[l] zv[l] are one more MMA per
//           step, with the zero bytes as every column of B.
// The chunk softmax runs on the score fragments: the lanes holding the two
// components of a head swap halves (one shuffle), each lane takes one head
// for its 8 keys, and the chunk statistics need one warp reduction and one
// cross-warp step through shared memory. A CTA streams ns consecutive chunks
// of one (sequence, KV head) through a two-stage ring: every thread copies
// its share of a chunk's K and V code rows (2 x 16 KB) with 16-byte cp.async
// into the stage freed by the chunk two back, so a chunk is in flight while
// the one before is computed. (Measured on B200: 256-row TMA tiles of these
// 64-byte rows streamed slower than the cp.async copies.) The chunks merge in
// registers (flash-decoding rescaling); a second kernel merges the CTAs'
// partials.
#include <algorithm>
#include <atomic>
#include <cmath>

#include "splitk_common.cuh"

namespace wq {

namespace {

using namespace splitk;

constexpr int kD = 128;                  // head dimension
constexpr int kT = 256;                  // keys per chunk
constexpr int kRowBytes = kD / 2;        // 64 bytes of codes per key
constexpr int kQwStride = kD / 4 + 4;    // words per query digit row (padded)
constexpr int kBdStride = kT + 16;       // bytes per value digit row (padded)
constexpr int kStages = 2;               // chunks of K and V codes in the ring
constexpr int kMinBlocks = 3;            // CTAs per SM the kernel is sized for
constexpr uint32_t kStageBytes = 2 * kT * kRowBytes;  // K codes, then V codes

// dynamic shared memory carve-up (bytes)
constexpr int kOffBd = kStages * kStageBytes;             // value digits [16][kBdStride]
constexpr int kOffQw = kOffBd;                            // query digits (prologue only)
constexpr int kVRowWords = kD;                            // V tile: 32 rows of 8-token blocks
constexpr int kOffKi = kOffBd + 16 * kBdStride;           // per key: sk, zk, sv (float4)
constexpr int kOffZv = kOffKi + kT * 16;                  // zv bytes in digit-slot order, x2
constexpr int kOffQm = kOffZv + 2 * kT;                   // qsig[16], qsum[16]
constexpr int kOffCo = kOffQm + 2 * 16 * 4;               // coefA[16], coefB[16] per digit row
constexpr int kOffRun = kOffCo + 2 * 16 * 4;              // running M[8], E[8] per head
constexpr int kOffRed = kOffRun + 2 * 8 * 4;              // [3][8 warps][8 heads]
constexpr int kSmemBytes = kOffRed + 3 * 8 * 8 * 4;
static_assert(16 * kQwStride * 4 <= 16 * kBdStride, "query digits fit the digit rows");
// kMinBlocks CTAs per SM (228 KB, 1 KB reserved per CTA)
static_assert(kMinBlocks * (kSmemBytes + 1024) <= 228 * 1024, "CTAs per SM");

// Shared-memory tiles. K: 16-byte piece c of key row l at byte
// l * 64 + ((c ^ ((l >> 3) & 3)) << 4); the score B reads (rows 8 (g >> 1) +
// 2 t + (g & 1), one word of one piece each) then hit distinct banks. V: word
// (block j, d) at word j * 128 + (d ^ 8 (j & 3)); the value B reads (blocks
// 4 s + t4, 8 consecutive d) then hit distinct banks.
// Value digits: within each 32-key step, key 8 b + 2 j + p (b, j in 0..3, p
// in 0..1, the low (p = 0) or high nibble j of V block b) sits at k slot
// 16 p + 4 b + j. The zero bytes are kept per step in the order 8 b + 4 p + j,
// so one 8-byte read gives a lane both B registers of the zero-term MMA.
__device__ __forceinline__ int zv_pos(int kk) {
  return (kk & ~31) + 8 * ((kk >> 3) & 3) + 4 * (kk & 1) + ((kk >> 1) & 3);
}

// Slot of key kk in the per-key table (float4): bits 1-2 of kk XOR-ed with
// bits 3-4, so the four lanes t4 of a lane group, whose keys are 8 apart,
// read distinct banks.
__device__ __forceinline__ int ki_pos(int kk) { return kk ^ (((kk >> 3) & 3) << 1); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma_s8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// a / b rounded to nearest from y = RN(1 / b): one correction step on the
// product a y (Markstein's theorem: with y the correctly rounded reciprocal
// and the residual a - b q formed exactly by a fused multiply-add, the
// corrected quotient is the correctly rounded a / b, barring overflow and
// underflow).
__device__ __forceinline__ float div_by(float a, float b, float y) {
  const float q = a * y;
  return __fmaf_rn(__fmaf_rn(-q, b, a), y, q);
}

// 2^x (ex2.approx: relative error about 2^-22; 2^-inf = 0).
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct KvArgs {
  const int8_t* qd;       // [C][B*Hq][D] query digits
  const float* qs;        // [C][B*Hq] their scales
  const __half* ks;       // [B, Hkv, L]
  const __half* kz;
  const __half* vs;
  const __half* vz;
  float* part;            // [B, Hkv, nsplit, R, D] partial outputs
  float* stat;            // [B, Hkv, nsplit, R, 2] (M, E) of each partial, M in log2 units
  int B, Hq, Hkv, L, nch, ns, nsplit;
  const uint8_t* kq;      // K codes [B, Hkv, L, D/2]
  const uint8_t* vq;      // V codes [B, Hkv, nblk, D] words (8-token blocks)
  int nblk;               // ceil(L / 8)
  float score_scale;      // log2(e) / sqrt(D): scores in log2 units
};

template <int R, int C>
__global__ void __launch_bounds__(256, kMinBlocks)
    kv_msd_split_kernel(KvArgs p) {
  constexpr int RC = R * C;
  static_assert(RC <= 16 && (C == 1 || C == 2), "digit rows");
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23 (see below)
  extern __shared__ __align__(16) uint8_t sm[];
  int8_t* bd = reinterpret_cast<int8_t*>(sm + kOffBd);
  uint32_t* qw = reinterpret_cast<uint32_t*>(sm + kOffQw);
  float4* ki = reinterpret_cast<float4*>(sm + kOffKi);
  uint8_t* zvb = sm + kOffZv;
  float* qsig = reinterpret_cast<float*>(sm + kOffQm);
  int* qsum = reinterpret_cast<int*>(qsig + 16);
  float* coefA = reinterpret_cast<float*>(sm + kOffCo);
  float* coefB = coefA + 16;
  float* Mrun = reinterpret_cast<float*>(sm + kOffRun);
  float* Erun = Mrun + 8;
  float* redm = reinterpret_cast<float*>(sm + kOffRed);
  float* rede = redm + 64;
  float* reda = rede + 64;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int split = blockIdx.x, kh = blockIdx.y, b = blockIdx.z;
  const int j0 = split * p.ns;
  const int nsub = min(p.ns, p.nch - j0);
  const int64_t seq0 = ((int64_t)b * p.Hkv + kh) * p.L;  // cache row of token 0
  // the head this lane takes in the softmax: rows (2h, 2h + 1) are held by
  // lanes g = 2h (h < 4, as row g and, after the swap, g + 1) and g = 2h - 7
  // (h >= 4, as rows g + 7 and g + 8)
  const int hl = C == 2 ? ((g & 1) ? (g + 7) >> 1 : g >> 1) : g;
  const bool hv = hl < R;

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // chunk jc's K rows and V blocks into stage st (the caller commits the
  // cp.async group). Thread tid copies 16-byte piece tid & 3 of K rows
  // tid / 4 + 64 r and piece tid & 31 of V block rows tid / 32 + 8 r (r < 4),
  // so its swizzles ((row >> 3) & 3 = (tid >> 5) & 3 for both) and its
  // offsets are fixed.
  const int sw_cp = (tid >> 5) & 3;
  const int k_dst = (tid >> 2) * kRowBytes + (((tid & 3) ^ sw_cp) << 4);
  const int k_src = (tid >> 2) * kRowBytes + 16 * (tid & 3);
  const int v_dst = kT * kRowBytes + (tid >> 5) * (kVRowWords * 4) + (((tid & 31) ^ (2 * sw_cp)) << 4);
  const int v_src = (tid >> 5) * (kVRowWords * 4) + 16 * (tid & 31);
  const int64_t vseq = ((int64_t)b * p.Hkv + kh) * p.nblk;  // V block row of token 0
  auto issue = [&](int st, int jc) {
    uint8_t* dst = sm + st * kStageBytes;
    const int64_t koff = (seq0 + (int64_t)jc * kT) * kRowBytes + k_src;
    const int nk = min(kT, p.L - jc * kT);
    const int64_t voff = (vseq + (int64_t)jc * (kT / 8)) * (kVRowWords * 4) + v_src;
    const int nb = min(kT / 8, p.nblk - jc * (kT / 8));
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      if ((tid >> 2) + 64 * r < nk)
        cp_async16(dst + k_dst + r * 64 * kRowBytes, p.kq + koff + r * 64 * kRowBytes);
      if ((tid >> 5) + 8 * r < nb)
        cp_async16(dst + v_dst + r * 8 * kVRowWords * 4,
                   p.vq + voff + r * 8 * kVRowWords * 4);
    }
  };
  // key tid's (sk, zk, sv, zv) of chunk jc, zeros past the end of the cache
  auto load_info = [&](int jc, __half (&h)[4]) {
    const int l = jc * kT + tid;
    const __half z = __float2half(0.0f);
    h[0] = h[1] = h[2] = h[3] = z;
    if (l < p.L) {
      h[0] = p.ks[seq0 + l];
      h[1] = p.kz[seq0 + l];
      h[2] = p.vs[seq0 + l];
      h[3] = p.vz[seq0 + l];
    }
  };
  auto store_info = [&](const __half (&h)[4], int buf) {
    ki[ki_pos(tid)] = make_float4(__half2float(h[0]), __int_as_float((int)__half2float(h[1])),
                          __half2float(h[2]), 0.0f);
    zvb[buf * kT + zv_pos(tid)] = (uint8_t)__half2float(h[3]);
  };

  // ---- prologue: the first two chunks' codes and the first key data (the
  // cache is not written by the grid this one may overlap, so they go before
  // the wait)
#pragma unroll
  for (int st = 0; st < kStages; ++st) {
    if (st < nsub) issue(st, j0 + st);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  if (tid < R) {
    Mrun[tid] = -INFINITY;
    Erun[tid] = 0.0f;
  }
  {
    __half h[4];
    load_info(j0, h);
    store_info(h, 0);
  }
  // the query digits of this KV head's R query heads (rows hc = h C + c), in
  // the even-d / odd-d order of the unpacked K code words, and their sums
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int qrow0 = b * p.Hq + kh * R;
  const int64_t plane = (int64_t)p.B * p.Hq;
  {
    int part = 0;
    if (tid < RC * (kD / 8)) {
      const int hc = tid >> 4, g8 = tid & 15;
      const int h = hc / C, c = hc - h * C;
      const uint2 v = *reinterpret_cast<const uint2*>(
          p.qd + ((int64_t)c * plane + qrow0 + h) * kD + 8 * g8);
      const uint32_t ev = prmt(v.x, v.y, 0x6420u), od = prmt(v.x, v.y, 0x7531u);
      // k-step s = g8 / 4 holds the even-d words of its four K code words
      // first, then the odd-d words
      qw[hc * kQwStride + 8 * (g8 >> 2) + (g8 & 3)] = ev;      // d = 8 g8 + 0, 2, 4, 6
      qw[hc * kQwStride + 8 * (g8 >> 2) + 4 + (g8 & 3)] = od;  // d = 8 g8 + 1, 3, 5, 7
      part = __dp4a((int)ev, 0x01010101, __dp4a((int)od, 0x01010101, 0));
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (tid < RC * (kD / 8) && (tid & 15) == 0) qsum[tid >> 4] = part;
    if (tid < RC) {
      const int h = tid / C, c = tid - h * C;
      qsig[tid] = p.qs[(int64_t)c * plane + qrow0 + h];
    }
  }
  __syncthreads();
  uint32_t a[4][4];  // score A fragments, [k-step][register]
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    a[s][0] = g < RC ? qw[g * kQwStride + 8 * s + t4] : 0u;
    a[s][1] = g + 8 < RC ? qw[(g + 8) * kQwStride + 8 * s + t4] : 0u;
    a[s][2] = g < RC ? qw[g * kQwStride + 8 * s + 4 + t4] : 0u;
    a[s][3] = g + 8 < RC ? qw[(g + 8) * kQwStride + 8 * s + 4 + t4] : 0u;
  }
  // Scores in log2 units. With C = 2 the component scales satisfy
  // sig_1 = 256 sig_2 exactly (a power-of-two ratio), so the two integer
  // partial sums combine exactly as 256 (P_1 - zk R_1) + (P_2 - zk R_2)
  // = 256 P_1 + P_2 - zk (256 R_1 + R_2) (|.| < 2^31) before one conversion.
  const int r0 = hv ? hl * C : 0;
  const float cs = qsig[r0 + C - 1] * p.score_scale;
  const int qsc = C == 2 ? 256 * qsum[r0] + qsum[r0 + 1] : qsum[r0];
  __syncthreads();  // the query digits' space becomes the value digit rows
  for (int i = RC * kBdStride / 4 + tid; i < 16 * kBdStride / 4; i += 256)
    reinterpret_cast<uint32_t*>(bd)[i] = 0u;  // the unused A rows of the value MMA

  // lane-constant parts of the shared-memory offsets within a stage (the
  // swizzle of every row a lane reads depends on the lane only):
  //   score B: K row 32 w + 8 (g >> 1) + 2 nt + (g & 1), word t4 of piece s;
  //            (row >> 3) & 3 = (g >> 1) & 3;
  //   value B: V block 4 ks + t4, word d = 16 w + 8 jm + g; (block & 3) = t4.
  int koff[4];
#pragma unroll
  for (int s = 0; s < 4; ++s)
    koff[s] = (32 * warp + 8 * (g >> 1) + (g & 1)) * kRowBytes + ((s ^ ((g >> 1) & 3)) << 4) +
              4 * t4;
  int voff[2];
#pragma unroll
  for (int jm = 0; jm < 2; ++jm)
    voff[jm] = kT * kRowBytes + 4 * (t4 * kVRowWords + ((16 * warp + 8 * jm + g) ^ (8 * t4)));
  // the lane's keys 32 w + 8 t4 + 2 nt + e sit at slots 32 w + 8 t4 +
  // 2 (nt ^ t4) + e
  const float4* kinf = ki + 32 * warp + 8 * t4;
  // ldmatrix row addresses of the value digit rows (A): lanes 0-7 rows 0-7,
  // 8-15 rows 8-15, at k bytes 0-15; lanes 16-31 the same rows at 16-31
  const int8_t* arow = bd + ((lane & 7) + 8 * ((lane >> 3) & 1)) * kBdStride + 16 * (lane >> 4);

  float O[2][4];
#pragma unroll
  for (int jm = 0; jm < 2; ++jm)
#pragma unroll
    for (int i = 0; i < 4; ++i) O[jm][i] = 0.0f;

  for (int i = 0; i < nsub; ++i) {
    const int jc = j0 + i;
    const int nk = min(kT, p.L - jc * kT);
    const bool more = i + 1 < nsub;
    const int st = i % kStages;
    // this chunk's group (the next chunk's may still be in flight)
    asm volatile("cp.async.wait_group %0;" ::"n"(kStages - 1) : "memory");
    __syncthreads();
    const uint8_t* kc = sm + st * kStageBytes;
    __half nxt[4];
    if (more) load_info(jc + 1, nxt);
    // ---- scores: warp w takes keys 32 w .. 32 w + 31; column n of n-tile nt
    // is key 32 w + 8 (n >> 1) + 2 nt + (n & 1)
    int sacc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int r = 0; r < 4; ++r) sacc[nt][r] = 0;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(kc + koff[s] + nt * 2 * kRowBytes);
        mma_s8u8(sacc[nt], a[s][0], a[s][1], a[s][2], a[s][3], w & 0x0F0F0F0Fu,
                 (w >> 4) & 0x0F0F0F0Fu);
      }
    }
    // the lane's head for its keys 32 w + 8 t4 + 2 nt + e
    float sc[4][2];
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        int dint;
        if (C == 2) {
          const int send = (g & 1) ? sacc[nt][e] : sacc[nt][2 + e];
          const int recv = __shfl_xor_sync(0xffffffffu, send, 4);
          const int p0 = (g & 1) ? recv : sacc[nt][e];
          const int p1 = (g & 1) ? sacc[nt][2 + e] : recv;
          dint = 256 * p0 + p1;
        } else {
          dint = sacc[nt][e];
        }
        const float4 inf = kinf[2 * (nt ^ t4) + e];
        dint -= __float_as_int(inf.y) * qsc;
        const float s = (float)dint * (inf.x * cs);
        sc[nt][e] = hv ? s : -INFINITY;
      }
    if (nk < kT)  // the cache's last chunk: keys past its end do not count
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          if (32 * warp + 8 * t4 + 2 * nt + e >= nk) sc[nt][e] = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) mx = fmaxf(mx, fmaxf(sc[nt][0], sc[nt][1]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    // Softmax statistics in one cross-warp step: each warp exponentiates
    // against its own maximum m_w; with M the chunk's maximum and
    // f_w = 2^(m_w - M), E = sum_w f_w E_w, amax = max_w f_w amax_w, and a
    // key's weight is f_own 2^(s - m_w) sv. (Rounding is monotonic, so no
    // weight exceeds the amax computed this way.)
    float wv[4][2], es = 0.0f, am = 0.0f;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        // sc = -inf: 0; a warp whose keys are all past the end (mx = -inf): 0
        const float ex = (hv && mx != -INFINITY) ? exp2_approx(sc[nt][e] - mx) : 0.0f;
        es += ex;
        wv[nt][e] = ex * kinf[2 * (nt ^ t4) + e].z;  // >= 0: sv > 0
        am = fmaxf(am, wv[nt][e]);
      }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      es += __shfl_xor_sync(0xffffffffu, es, o);
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    }
    if (t4 == 0 && hv) {
      redm[warp * 8 + hl] = mx;
      rede[warp * 8 + hl] = es;
      reda[warp * 8 + hl] = am;
    }
    __syncthreads();
    float m = -INFINITY, E = 0.0f, A = 0.0f, fown = 0.0f;
    if (hv) {
#pragma unroll
      for (int w = 0; w < 8; ++w) m = fmaxf(m, redm[w * 8 + hl]);
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float f = exp2_approx(redm[w * 8 + hl] - m);  // a warp without keys: 0
        E = fmaf(f, rede[w * 8 + hl], E);
        A = fmaxf(A, f * reda[w * 8 + hl]);
      }
      fown = exp2_approx(mx - m);
    }
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) wv[nt][e] *= fown;
    // The decomposition of w over the chunk's keys, as for an activation row:
    // s_1 = amax / 127, s_{c+1} = s_c / 256, digit rint(r / s_c) (the first
    // clamped to +-127), residual r - s_c a_c rounded once, and a digit of
    // +128 becomes -128 with a carry into the digit before it. Here
    // 0 <= w <= amax, and RN(w / s_1) <= RN(127 (1 + 2^-24)) < 127.5, so the
    // first digit needs no clamp. Rounding to an integer: t = x + 1.5 * 2^23
    // lies in [2^23, 2^24), where the spacing is 1, so the add rounds x to
    // nearest-even and t's low mantissa byte is the digit's two's-complement
    // byte (|x| <= 128.5).
    const float tau0 = A > 0.0f ? __fdiv_rn(A, 127.0f) : 1.0f;
    const float y0 = __frcp_rn(tau0);
    const float tau1 = tau0 * (1.0f / 256.0f), y1 = y0 * 256.0f;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      uint32_t tb[C][4];  // the digits' float bit patterns, keys nt = 0..3
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const float r = wv[nt][e];
        float t0 = div_by(r, tau0, y0) + kRound;
        if (C == 2) {
          const float r1 = __fmaf_rn(-tau0, t0 - kRound, r);
          const float t1 = div_by(r1, tau1, y1) + kRound;
          if (t1 == kRound + 128.0f) t0 += 1.0f;  // the byte of +128 already reads -128
          tb[C - 1][nt] = __float_as_uint(t1);
        }
        tb[0][nt] = __float_as_uint(t0);
      }
      if (hv)
#pragma unroll
        for (int c = 0; c < C; ++c)
          *reinterpret_cast<uint32_t*>(bd + (hl * C + c) * kBdStride + 32 * warp + 16 * e +
                                       4 * t4) =
              prmt(prmt(tb[c][0], tb[c][1], 0x0040u), prmt(tb[c][2], tb[c][3], 0x0040u), 0x5410u);
    }
    // merge weights of this chunk into the CTA's running sums (log2 units)
    if (warp == 0 && t4 == 0 && hv) {
      const float M0 = Mrun[hl], Mn = fmaxf(M0, m);
      const float al = exp2_approx(M0 - Mn), be = exp2_approx(m - Mn);  // M0 = -inf: al = 0
      Erun[hl] = fmaf(Erun[hl], al, E * be);
      Mrun[hl] = Mn;
#pragma unroll
      for (int c = 0; c < C; ++c) {
        coefA[hl * C + c] = al;
        coefB[hl * C + c] = be * (c == 0 ? tau0 : tau1);
      }
    }
    __syncthreads();
    // the next chunk's key data (this chunk's is no longer read; its zero
    // bytes go to the other buffer)
    if (more) store_info(nxt, (i + 1) & 1);

    // ---- values: warp w owns d in [16 w, 16 w + 16); MMA jm, column n:
    // d = 16 w + 8 jm + n
    int vacc[2][4], zacc[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) vacc[0][r] = vacc[1][r] = zacc[r] = 0;
    {
      const uint8_t* zb = zvb + (i & 1) * kT + 8 * t4;
#pragma unroll
      for (int ks = 0; ks < kT / 32; ++ks) {
        uint32_t af[4];
        ldsm_x4(af, arow + 32 * ks);
#pragma unroll
        for (int jm = 0; jm < 2; ++jm) {
          const uint32_t w =
              *reinterpret_cast<const uint32_t*>(kc + voff[jm] + 4 * (4 * ks * kVRowWords));
          mma_s8u8(vacc[jm], af[0], af[1], af[2], af[3], w & 0x0F0F0F0Fu, (w >> 4) & 0x0F0F0F0Fu);
        }
        const uint2 z = *reinterpret_cast<const uint2*>(zb + 32 * ks);
        mma_s8u8(zacc, af[0], af[1], af[2], af[3], z.x, z.y);
      }
    }
    // O = O alpha + beta tau_c (acc - zt) for the lane's rows g and g + 8
#pragma unroll
    for (int rh = 0; rh < 2; ++rh) {
      const int row = g + 8 * rh;
      const float cA = row < RC ? coefA[row] : 0.0f, cB = row < RC ? coefB[row] : 0.0f;
#pragma unroll
      for (int jm = 0; jm < 2; ++jm)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          O[jm][2 * rh + e] =
              fmaf(O[jm][2 * rh + e], cA, cB * (float)(vacc[jm][2 * rh + e] - zacc[2 * rh]));
    }
    __syncthreads();  // the stage, the digits and the weights of this chunk are consumed
    if (i + kStages < nsub) issue(st, jc + kStages);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  // ---- the CTA's partial: the components of a head sit in C consecutive
  // rows, held by lanes 4 apart
  const int64_t base = (((int64_t)b * p.Hkv + kh) * p.nsplit + split) * R;
#pragma unroll
  for (int jm = 0; jm < 2; ++jm) {
    const int d = 16 * warp + 8 * jm + 2 * t4;  // columns 2 t4, 2 t4 + 1
#pragma unroll
    for (int rh = 0; rh < 2; ++rh) {
      const int row = g + 8 * rh;
      float o0 = O[jm][2 * rh], o1 = O[jm][2 * rh + 1];
      if (C == 2) {
        o0 += __shfl_xor_sync(0xffffffffu, o0, 4);
        o1 += __shfl_xor_sync(0xffffffffu, o1, 4);
      }
      if (row < RC && row % C == 0)
        *reinterpret_cast<float2*>(p.part + (base + row / C) * kD + d) = make_float2(o0, o1);
    }
  }
  if (tid < R)
    *reinterpret_cast<float2*>(p.stat + (base + tid) * 2) = make_float2(Mrun[tid], Erun[tid]);
}

// Merge the CTAs' partials of each (sequence, query head): out = sum_j
// 2^(M_j - M) O_j / sum_j 2^(M_j - M) E_j, one CTA of 128 threads (one per element).
template <int R>
__global__ void __launch_bounds__(kD) kv_msd_merge_kernel(KvArgs p, uint16_t* __restrict__ out) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int bh = blockIdx.x;  // b * Hq + hq
  const int b = bh / p.Hq, hq = bh - b * p.Hq;
  const int kh = hq / R, h = hq - kh * R;
  const int d = threadIdx.x;
  const int64_t base = ((int64_t)b * p.Hkv + kh) * p.nsplit;
  float big = -INFINITY;
  for (int j = 0; j < p.nsplit; ++j) big = fmaxf(big, p.stat[((base + j) * R + h) * 2]);
  float num = 0.0f, den = 0.0f;
  for (int j = 0; j < p.nsplit; ++j) {
    const int64_t ri = (base + j) * R + h;
    const float f = exp2_approx(p.stat[ri * 2] - big);
    num = fmaf(f, p.part[ri * kD + d], num);
    den = fmaf(f, p.stat[ri * 2 + 1], den);
  }
  out[(int64_t)bh * kD + d] = bf16_bits(num / den);
}

// V codes from the token layout (uint32 [rows * L, D / 8], element d in
// nibble d % 8 of word d / 8) to blocks of 8 tokens (uint32 [rows, nblk, D],
// token 8 j + t in nibble t of word (j, d), tokens past L zero): one thread
// per output word.
__global__ void __launch_bounds__(256) kv_block_values_kernel(const uint32_t* __restrict__ in,
                                                              int64_t rows, int L, int D,
                                                              int nblk,
                                                              uint32_t* __restrict__ out) {
  const int64_t total = rows * nblk * D;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int d = (int)(idx % D);
    const int64_t rb = idx / D;  // row * nblk + block
    const int blk = (int)(rb % nblk);
    const int64_t row = rb / nblk;
    uint32_t w = 0;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int l = 8 * blk + t;
      if (l < L) w |= ((in[(row * L + l) * (D / 8) + d / 8] >> (4 * (d % 8))) & 15u) << (4 * t);
    }
    out[idx] = w;
  }
}

template <int R, int C>
wq_status launch_kv_rc(const KvArgs& a, void* out, cudaStream_t st) {
  static bool attr_set = [] {
    return cudaFuncSetAttribute(kv_msd_split_kernel<R, C>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemBytes) == cudaSuccess;
  }();
  if (!attr_set) return WQ_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.stream = st;
  cfg.gridDim = dim3((unsigned)a.nsplit, (unsigned)a.Hkv, (unsigned)a.B);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  if (cudaLaunchKernelEx(&cfg, kv_msd_split_kernel<R, C>, a) != cudaSuccess)
    return WQ_ERR_CUDA;
  cfg.gridDim = dim3((unsigned)(a.B * a.Hq), 1, 1);
  cfg.blockDim = dim3(kD, 1, 1);
  cfg.dynamicSmemBytes = 0;
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

std::atomic<int> g_kv_chunks_per_cta{0};  // 0: chosen per launch

// Workspace: query digits [C][B*Hq][D] and their scales [C][B*Hq] fp32 (each
// rounded up to 256 bytes), then the partial outputs [B, Hkv, nsplit, R, D]
// and statistics [B, Hkv, nsplit, R, 2] fp32, sized for nsplit = nch (one
// chunk per CTA, the most partials any launch writes).
size_t kv_msd_workspace_bytes(int64_t B, int64_t Hq, int64_t L, int32_t C) {
  const int64_t nch = (L + kT - 1) / kT;
  const size_t dig = ((size_t)C * B * Hq * kD + 255) / 256 * 256;
  const size_t sc = ((size_t)C * B * Hq * 4 + 255) / 256 * 256;
  return dig + sc + (size_t)B * Hq * nch * (kD + 2) * 4;
}

wq_status launch_kv_block_values(const uint32_t* codes, int64_t rows, int64_t L, int32_t D,
                                 uint32_t* out, cudaStream_t st) {
  const int nblk = (int)((L + 7) / 8);
  const int64_t total = rows * nblk * D;
  const int64_t grid = std::min<int64_t>((total + 255) / 256, (int64_t)num_sms() * 16);
  kv_block_values_kernel<<<(unsigned)grid, 256, 0, st>>>(codes, rows, (int)L, D, nblk, out);
  return launch_status();
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
  wq_status s = launch_msd_decompose(q, B * Hq, kD, C, B * Hq, qd, qs, st);
  if (s != WQ_OK) return s;
  KvArgs a;
  a.qd = qd;
  a.qs = qs;
  a.kq = static_cast<const uint8_t*>(kq);
  a.vq = static_cast<const uint8_t*>(vq);
  a.nblk = (int)((L + 7) / 8);
  a.ks = static_cast<const __half*>(ks);
  a.kz = static_cast<const __half*>(kz);
  a.vs = static_cast<const __half*>(vs);
  a.vz = static_cast<const __half*>(vz);
  a.part = part;
  a.B = (int)B;
  a.Hq = (int)Hq;
  a.Hkv = (int)Hkv;
  a.L = (int)L;
  a.nch = (int)nch;
  // chunks per CTA: enough CTAs for about four waves of kMinBlocks per SM, at
  // most 8 (or the count the test hook fixed)
  const int64_t total = B * Hkv * nch;
  const int forced = g_kv_chunks_per_cta.load(std::memory_order_relaxed);
  a.ns = forced > 0 ? forced
                    : (int)std::max<int64_t>(
                          1, std::min<int64_t>(8, total / ((int64_t)num_sms() * kMinBlocks * 4)));
  a.nsplit = (int)((nch + a.ns - 1) / a.ns);
  a.stat = part + (size_t)B * Hkv * a.nsplit * (Hq / Hkv) * kD;
  a.score_scale = (float)(1.4426950408889634 / std::sqrt((double)kD));
  const int R = (int)(Hq / Hkv);
  return C == 1 ? launch_kv_c<1>(a, R, out, st) : launch_kv_c<2>(a, R, out, st);
}

}  // namespace wq
