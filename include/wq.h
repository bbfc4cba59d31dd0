/*
 * wq.h -- C ABI of the 4-bit weight-only quantized product library for
 * NVIDIA B200 (sm_100a).
 *
 * The library computes y = x . dequant(W_q)^T for bf16 activations x [M, K]
 * and 4-bit weights W [N, K] (N output features, K input features), with the
 * dequantization fused into the product, plus the Multi-Scale Dequant path in
 * which the activations are split into int8 digit planes that multiply the
 * integer weight codes directly.
 *
 * Sources (each entry point names the passage that defines it):
 *  [MSD]   "Multi-Scale Dequant: Eliminating Dequantization Bottleneck via
 *          Activation Decomposition for Efficient LLM Inference", Abstract.
 *  [MIXPE] "MixPE: Quantization and Hardware Co-design for Efficient LLM
 *          Inference", Abstract.
 *  [NF4]   "Fast NF4 Dequantization Kernels for Large Language Model
 *          Inference", Abstract.
 *  [QLORA] "QLoRA: Efficient Finetuning of Quantized LLMs" (cited by title on
 *          "DecDEC: A Systems Approach to Advancing Low-Bit LLM Quantization"):
 *          the NF4 codebook construction.
 *  [DECDEC] "DecDEC: A Systems Approach to Advancing Low-Bit LLM
 *          Quantization", Abstract: salient-channel residual correction.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor argument is a DEVICE pointer owned by the caller unless the
 *    comment says "host". The library never allocates, frees or retains
 *    caller memory. Workspace, where an entry point takes one, is caller
 *    provided and sized by wq_workspace_bytes().
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream). Every device call is asynchronous on that stream; the library
 *    never synchronises, except wq_device_error(), which says so.
 *  - Device pointers must be 16-byte aligned (WQ_ERR_ALIGNMENT otherwise).
 *  - All arguments are validated before anything is launched; a failed
 *    validation returns a status and launches nothing. No C++ exception
 *    crosses this boundary. A launch failure returns WQ_ERR_CUDA (the CUDA
 *    error is left for cudaGetLastError to report as usual).
 *  - Rounding: every float -> integer rounding is round-half-to-even, every
 *    division is an IEEE binary32 division, every narrowing is
 *    round-to-nearest-even. No fast-math.
 *  - The current CUDA device is the one every pointer must live on.
 *
 * Canonical packed layouts (the only layouts that cross this ABI)
 * ---------------------------------------------------------------
 *  INT4 asymmetric, group size G along K ([MIXPE]):
 *    qweight  uint32 [N, K/8]  code of column k in bits 4*(k%8) .. +3
 *    scales   fp16   [N, K/G]  s, row-major
 *    zeros    fp16   [N, K/G]  z (an exact integer 0..15), row-major
 *    dequant: w = (q - z) * s  (exact in fp32)
 *    quantize (per row n, group g): lo = min(min w, 0), hi = max(max w, 0);
 *    s = fp16(fp32(hi - lo) / 15), recomputed with lo=-1, hi=1 if that is 0;
 *    z = clamp(rint(-lo / s), 0, 15); q = clamp(rint(w / s) + z, 0, 15).
 *  NF4, block of 64 consecutive elements of the row-major [N, K] weight
 *  ([NF4], [QLORA]):
 *    codes    uint8  [N*K/2]   element 2j in the HIGH nibble of byte j,
 *                              element 2j+1 in the low nibble
 *    absmax   fp32   [N*K/64]
 *    dequant: w = fp32(codebook[code] * absmax)
 *    quantize: absmax = max|w|; code = index of the codebook value nearest to
 *    fp32(w / absmax), ties to the lower index; an all-zero block stores
 *    absmax 0 and code 7 (the exact zero).
 */
#ifndef WQ_H_
#define WQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WQ_OK = 0,
  WQ_ERR_INVALID_ARG = 1,   /* NULL pointer, negative or inconsistent size  */
  WQ_ERR_UNSUPPORTED = 2,   /* valid request outside what the kernels cover */
  WQ_ERR_ALIGNMENT = 3,     /* a device pointer is not 16-byte aligned      */
  WQ_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed         */
  WQ_ERR_TIMEOUT = 5,       /* a bounded device-side wait expired           */
  WQ_ERR_WORKSPACE = 6      /* workspace NULL or smaller than required      */
} wq_status;

typedef enum { WQ_FMT_INT4_ASYM = 0, WQ_FMT_NF4 = 1 } wq_format;
typedef enum { WQ_BF16 = 0, WQ_FP16 = 1, WQ_FP32 = 2 } wq_dtype;
typedef enum { WQ_OP_GEMV = 0, WQ_OP_GEMM = 1, WQ_OP_MSD_GEMM = 2, WQ_OP_MX_GEMV = 3 } wq_op;

/* Human-readable name of a status. Never NULL. Host only. */
const char* wq_status_string(wq_status status);

/* Library version string, e.g. "wq 0.1 sm_100a". Host only. */
const char* wq_version(void);

/*
 * The 16 NF4 code values (fp32, ascending) the device kernels use. Host only;
 * `out` is a host array of 16 floats. The library computes them once from the
 * QLoRA construction ([QLORA], used by [NF4]): quantiles of the standard
 * normal at probabilities evenly spaced from delta = (1 - 1/30 + 1 - 1/32)/2
 * towards 1/2 (8 positive, 7 negative), an exact 0, normalised by the largest,
 * each rounded once to fp32.
 */
wq_status wq_nf4_codebook(float out[16]);

/*
 * Byte sizes of the caller-allocated packed buffers for `fmt` and an [N, K]
 * weight. INT4: group G (G % 8 == 0, K % G == 0); qweight N*K/2, scales and
 * zeros N*(K/G)*2 each. NF4: group must be 64 (the block size), N*K % 64 == 0;
 * qweight N*K/2, scales = absmax N*K/64*4, zeros 0. This is the 4x memory
 * reduction of [NF4]. Host only; output pointers are host pointers.
 */
wq_status wq_packed_sizes(wq_format fmt, int64_t N, int64_t K, int32_t group,
                          size_t* qweight_bytes, size_t* scale_bytes,
                          size_t* zero_bytes);

/*
 * Quantize and pack fp32 weights W [N, K] (device, row-major) into the
 * canonical layout above ([MIXPE] group scale/zero; [NF4] codes + absmax).
 * INT4: `scales`/`zeros` are fp16 [N, K/G]. NF4: group == 64, `scales` is the
 * fp32 absmax [N*K/64] and `zeros` must be NULL. Requires K % 8 == 0.
 * Bit-exact with the CPU oracle for finite weights whose group ranges fit
 * fp16 (|hi - lo| / 15 <= 65504). Non-finite weights give unspecified codes.
 */
wq_status wq_quantize_pack(wq_format fmt, const float* W, int64_t N, int64_t K,
                           int32_t group, void* qweight, void* scales,
                           void* zeros, void* stream);

/*
 * Unpack codes to one byte per element: codes[n*K + k] in 0..15, for either
 * format (NF4: numel = N*K, flattened). For checking packed data.
 */
wq_status wq_unpack(wq_format fmt, const void* qweight, int64_t N, int64_t K,
                    uint8_t* codes, void* stream);

/*
 * Standalone NF4 dequantization ([NF4]: lifting NF4 back to 16-bit before the
 * product, the kernel that page accelerates):
 *   out[i] = RN_dtype( fp32(codebook[code_i] * absmax[i / 64]) )
 * codes: packed NF4 [numel/2]; absmax fp32 [numel/64]; out bf16 or fp16
 * [numel]. blocksize must be 64, numel % 64 == 0. Bit-exact with the oracle.
 */
wq_status wq_nf4_dequant(const uint8_t* codes, const float* absmax,
                         int64_t numel, int32_t blocksize, void* out,
                         wq_dtype out_dtype, void* stream);

/*
 * Standalone INT4 dequantization ([MSD]: lifting the low-bit weights to bf16,
 * the step MSD removes; used by the dequantize-then-GEMM baseline):
 *   out[n, k] = RN_dtype( (q - z) * s )   (the product is exact in fp32)
 * out bf16 or fp16 [N, K]. K % 8 == 0, K % group == 0, group % 8 == 0.
 */
wq_status wq_int4_dequant(const uint32_t* qweight, const void* scales,
                          const void* zeros, int64_t N, int64_t K,
                          int32_t group, void* out, wq_dtype out_dtype,
                          void* stream);

/*
 * Decode W4A16 GEMV ([MSD], [MIXPE], [NF4]): y[m, n] = sum_k x[m, k] w[n, k]
 * for 1 <= M <= 16, fp32 accumulation, bf16 output.
 *   x bf16 [M, K] row-major; y bf16 [M, N] row-major.
 *   INT4: scales/zeros fp16 [N, K/G], G % 64 == 0, K % G == 0. The group's
 *         scale and zero are applied after the group's sum ([MIXPE]).
 *   NF4 : group == 64, scales = fp32 absmax [N*K/64], zeros NULL. The code
 *         values are rounded once to fp16 and multiply an fp16 copy of x
 *         (scaled per token by a power of two: exact for bf16 values down to
 *         2^-28 of the token's largest) with fp32 accumulation; each 64-element
 *         block's partial sum is then multiplied by its fp32 absmax in fp32, so
 *         blocks of any finite absmax, however small, keep full precision.
 * Requires K % 128 == 0 and N % 16 == 0. M == 0 or N == 0 is a no-op.
 * Workspace: none needed (pass NULL, 0); split-K partials are reduced on chip
 * through thread-block-cluster shared memory.
 */
wq_status wq_w4a16_gemv(const void* x, int64_t M, int64_t N, int64_t K,
                        wq_format fmt, int32_t group, const void* qweight,
                        const void* scales, const void* zeros, void* y,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * Salient-channel residual correction ([DECDEC]: the residual matrix is the
 * full-precision weights minus the quantized ones; the residuals of the
 * channels that the current activations mark as outliers are added back).
 *
 * wq_residual: R^T = fp16(W - W_hat) as fp16 [K, N] (channel-major: one
 *   channel's residuals are contiguous). W fp32 [N, K] row-major; the packed
 *   weights and parameters as for wq_w4a16_gemv. W_hat is (q - z) * s (exact
 *   in fp32) for INT4 and fp32(codebook[q] * absmax) for NF4; the subtraction
 *   rounds once in fp32, the result once to fp16. Bit-exact with the oracle.
 *   Requires K % 64 == 0 and N % 8 == 0; N == 0 is a no-op.
 *
 * wq_select_salient: the k salient channels of x bf16 [M, K] (M >= 1,
 *   0 <= k <= K <= 65536): the k largest max_m |x[m, c]|, ranked by the bf16
 *   bit pattern with the sign cleared (NaN above +inf), ties to the lower
 *   channel. idx int32 [k] receives them in increasing order. k == 0 is a
 *   no-op. One CTA.
 *
 * wq_w4a16_gemv_corrected: wq_w4a16_gemv plus, for every output,
 *   sum_j x[m, idx[j]] * R^T[idx[j], n], added in fp32 before the bf16
 *   rounding. idx holds k channels (0 <= k <= K; k == 0 is wq_w4a16_gemv);
 *   residual_t is fp16 [K, N] as written by wq_residual. Only the k selected
 *   rows of R^T are read.
 * All three are asynchronous on `stream`; buffers are caller-owned.
 */
wq_status wq_residual(wq_format fmt, const float* W, int64_t N, int64_t K,
                      int32_t group, const void* qweight, const void* scales,
                      const void* zeros, void* residual_t, void* stream);
wq_status wq_select_salient(const void* x, int64_t M, int64_t K, int32_t k,
                            int32_t* idx, void* stream);
wq_status wq_w4a16_gemv_corrected(const void* x, int64_t M, int64_t N, int64_t K,
                                  wq_format fmt, int32_t group,
                                  const void* qweight, const void* scales,
                                  const void* zeros, const void* residual_t,
                                  const int32_t* idx, int32_t k, void* y,
                                  void* stream);

/*
 * wq_w4a16_gemv_salient: one decode step of the correction, selection
 * included: wq_select_salient into idx (caller-owned int32 [k] scratch,
 * written), then wq_w4a16_gemv_corrected. The GEMV is launched as a
 * programmatic dependent of the selection: it starts while the selection
 * runs and waits for it only before its epilogue reads idx. Requires
 * K <= 65536 when k > 0; k == 0 is wq_w4a16_gemv.
 */
wq_status wq_w4a16_gemv_salient(const void* x, int64_t M, int64_t N, int64_t K,
                                wq_format fmt, int32_t group,
                                const void* qweight, const void* scales,
                                const void* zeros, const void* residual_t,
                                int32_t k, int32_t* idx, void* y, void* stream);

/*
 * Prefill W4A16 GEMM with fused dequantization on the tensor cores ([MSD]:
 * the dequantize-then-multiply product; here the dequantized tile is written
 * straight into tensor memory and never leaves the SM). Same arguments and
 * layouts as wq_w4a16_gemv, any
 * M >= 1, INT4 or NF4. Requires K % 128 == 0, N % 128 == 0, G % 64 == 0,
 * K % G == 0, and INT4 group scales with 15 * s <= 65504.
 * NF4 ([NF4]: codebook value x block absmax): per weight row n a power of two
 * 2^e_n puts the row's largest absmax in [2^14, 2^15); each weight is
 * fp16_rn(fp16(code) * fp16_rn(absmax * 2^e_n)) and the epilogue divides 2^e_n
 * back out. Any finite absmax works; a block more than 2^28 below its row's
 * largest absmax loses relative precision, a negligible part of that row's
 * outputs.
 * The product runs in fp16 with fp32 accumulation: x is first copied to fp16
 * scaled per row by a power of two (exact for bf16 values down to 2^-28 of the
 * row's largest), each weight is fp16_rn((q - z) * s), and the epilogue
 * removes the power of two before rounding y to bf16.
 * Workspace: at least wq_workspace_bytes(WQ_OP_GEMM, ...) bytes (the fp16
 * copy of x and the per-row scales); contents on entry do not matter.
 * May return WQ_ERR_TIMEOUT through wq_device_error if an internal bounded
 * wait expires.
 */
wq_status wq_w4a16_gemm(const void* x, int64_t M, int64_t N, int64_t K,
                        wq_format fmt, int32_t group, const void* qweight,
                        const void* scales, const void* zeros, void* y,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * Multi-Scale Dequant activation decomposition ([MSD]): per row m of x
 * (bf16 [M, K]), n_components (C, 1..3) int8 digit planes a [C, M, K] and
 * fp32 scales s [C, M] with x ~= sum_c s[c, m] a[c, m, :]:
 *   s[0] = fp32(amax / 127) (1 for an all-zero row), a[0] = clamp(rint(x /
 *   s[0]), -127, 127); s[c] = s[c-1] / 256; the residual after c components is
 *   r = RN32(r - s[c] a[c]) (one rounding); a[c] = rint(r / s[c]) in [-128,
 *   128], a +128 written as -128 with +1 carried into a[c-1].
 *   Two components give |x - x_hat| <= s[1] / 2: close to 16 effective bits.
 * Bit-exact with the oracle. M == 0 is a no-op; K % 16 == 0.
 */
wq_status wq_msd_decompose(const void* x, int64_t M, int64_t K,
                           int32_t n_components, int8_t* digits,
                           float* comp_scales, void* stream);

/*
 * Multi-Scale Dequant GEMM ([MSD], with [MIXPE]'s post-group scaling):
 *   y[m, n] = sum_c s_c[m] sum_g s[n, g] (sum_{k in g} a_c[m, k] (q[n, k] - z[n, g]))
 * i.e. x_hat . dequant(W)^T, with x_hat the C-component decomposition of x
 * (wq_msd_decompose). The integer weight codes enter int8 tensor-core MMAs
 * directly; no weight is converted to a floating-point type.
 * INT4 asymmetric weights only; group G % 128 == 0 (G == K is per-channel),
 * K % G == 0, K % 128 == 0, N % 128 == 0, 1 <= n_components <= 3.
 * Workspace: at least wq_workspace_bytes(WQ_OP_MSD_GEMM, ...) bytes (it holds
 * the digit planes and scales); its contents on entry do not matter.
 */
wq_status wq_msd_gemm(const void* x, int64_t M, int64_t N, int64_t K,
                      int32_t n_components, int32_t group, const void* qweight,
                      const void* scales, const void* zeros, void* y,
                      void* workspace, size_t ws_bytes, void* stream);

/*
 * Multi-Scale Dequant with NF4 weights, decode (1 <= M <= 16) ([MSD] with
 * [NF4]). The pages give MSD for integer weights; NF4 codes index real
 * codebook values, so the library reads NF4-MSD as: the 16 code values become
 * integers c_int = rint(c * 2^13) (within 2^-14 of c), split into two signed
 * 8-bit digits c_int = 128 h + l; the activation digits of wq_msd_decompose
 * multiply them on the int8 tensor cores and each 64-element block's absmax
 * is applied after the block's integer sum:
 *   y[m, n] = sum_c s_c[m] sum_blk absmax[n, blk] 2^-13
 *             sum_{k in blk} a_c[m, k] (128 h[q] + l[q])
 * (each weight within 2^-14 absmax of codebook[q] * absmax). No weight is
 * converted to floating point. codes/absmax: the canonical NF4 layout. M == 0
 * or N == 0 is a no-op; requires K % 256 == 0, N % 16 == 0, 1 <= n_components
 * <= 3. Workspace: at least wq_workspace_bytes(WQ_OP_MSD_GEMM, ...) bytes.
 */
wq_status wq_msd_gemm_nf4(const void* x, int64_t M, int64_t N, int64_t K, int32_t n_components,
                          const uint8_t* codes, const float* absmax, void* y, void* workspace,
                          size_t ws_bytes, void* stream);

/*
 * wq_msd_gemm for callers that cannot allocate device memory. The library's
 * pages have no counterpart to this call; it exists for deployment. Some
 * callers cannot hand the library a workspace: an engine that carves up all
 * device memory once at start-up and must not grow, a plugin host whose fixed
 * call signature has no workspace argument, or a latency-critical loop in
 * which a device allocation (which may synchronise the GPU) is forbidden.
 * This entry point takes the same arguments as wq_msd_gemm minus the
 * workspace and computes the same result with the same kernels, using a
 * fixed 8 MiB scratch array that the library reserves in device memory on
 * every GPU that loads it (held until the process exits). It allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *  - Limit: wq_workspace_bytes(WQ_OP_MSD_GEMM, M, N, K, group, C) must not
 *    exceed 8 MiB (C * roundup(M, 128) * K + C * M * 4 bytes, e.g. M <= 128
 *    at K = 25600 with C = 2); larger problems return WQ_ERR_UNSUPPORTED and
 *    launch nothing.
 *  - The first call on a device looks up the scratch array's device address
 *    (once per device, with that device current); make that first call
 *    before any stream capture.
 *  - Every call shares the one array, and each call overwrites what it reads
 *    before reading it (nothing has to start at zero). Calls that overlap on
 *    the GPU (other streams, or other threads' streams) race on it: order
 *    them on one stream.
 */
wq_status wq_msd_gemm_noalloc(const void* x, int64_t M, int64_t N, int64_t K,
                              int32_t n_components, int32_t group, const void* qweight,
                              const void* scales, const void* zeros, void* y, void* stream);

/*
 * MX path of Multi-Scale Dequant ([MSD]: for MXFP4 weights, two MXFP4 passes
 * over the bf16 activations multiply the weights directly, against one MXFP8
 * pass). The page names the formats without defining them; the library reads
 * them as microscaling blocks:
 *   - 32 consecutive elements along K share one power-of-two scale 2^e, stored
 *     as the byte e + 127 (e in -127..127): the smallest e such that no
 *     element saturates (amax <= 6 * 2^e for E2M1, 448 * 2^e for E4M3);
 *   - MXFP4 elements are FP4 E2M1 codes (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4,
 *     6; bit 3 = sign), MXFP8 elements FP8 E4M3 bytes; both round to nearest
 *     with ties to the even code, and a value that rounds to zero is +0.
 *
 * wq_mx_quantize: MXFP4 weights W fp32 [N, K] (device) -> codes uint8
 *   [N, K/2] (element 2j in the low nibble of byte j) and scale bytes uint8
 *   [N, K/32]. K % 32 == 0. Bit-exact with the oracle.
 * wq_mx_decompose: activations x bf16 [M, K] -> n_passes planes uint8
 *   [n_passes][M][K] and scale bytes uint8 [n_passes][M][K/32].
 *   n_passes == 2: x1 = MXFP4(x), r = x - x1 (exact), x2 = MXFP4(r) with its
 *     own block scales; the planes hold the MXFP4 values as E4M3 bytes (every
 *     E2M1 value is exact in E4M3).
 *   n_passes == 1: one MXFP8 pass (the comparator).
 *   K % 32 == 0. Bit-exact with the oracle.
 * wq_mx_gemv: decode product y bf16 [M, N] = x_hat . w_hat^T for 1 <= M <= 16
 *   (M == 0 or N == 0: no-op), with x_hat the n_passes decomposition of x and
 *   w_hat the MXFP4 weights; every MMA covers one 32-element block of both
 *   operands exactly and its partial sum takes the two block scales in fp32.
 *   Requires K % 256 == 0 and N % 16 == 0. Workspace: at least
 *   wq_workspace_bytes(WQ_OP_MX_GEMV, M, N, K, 0, n_passes) bytes (it holds
 *   the decomposition); contents on entry do not matter.
 * All are asynchronous on `stream`; every buffer is caller-owned.
 */
wq_status wq_mx_quantize(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* scales,
                         void* stream);
wq_status wq_mx_decompose(const void* x, int64_t M, int64_t K, int32_t n_passes, uint8_t* planes,
                          uint8_t* scales, void* stream);
wq_status wq_mx_gemv(const void* x, int64_t M, int64_t N, int64_t K, int32_t n_passes,
                     const uint8_t* codes, const uint8_t* scales, void* y, void* workspace,
                     size_t ws_bytes, void* stream);

/*
 * Multi-Scale Dequant in decode attention over an INT4 KV cache ([MSD],
 * Abstract: the quantized KV cache multiplies low-precision components of
 * the other operand directly, so the cache is never dequantized and its HBM
 * traffic in attention shrinks). One new query token per sequence:
 *   q        bf16 [B, Hq, D] (device); Hq = R * Hkv, query head h reads KV
 *            head h / R (grouped heads), R in {1, 2, 4, 8}; D == 128;
 *   K and V  each INT4 asymmetric with one group per (sequence, head, token)
 *            row, as wq_quantize_pack(WQ_FMT_INT4_ASYM, group = D) computes it
 *            for the [B * Hkv * L, D] rows: scales fp16 [B, Hkv, L], zeros
 *            fp16 [B, Hkv, L] holding integers 0..15, and
 *            K codes uint32 [B, Hkv, L, D/8], that call's layout (element d in
 *            nibble d % 8 of word d / 8);
 *            V codes uint32 [B, Hkv, ceil(L/8), D], blocks of 8 tokens (token
 *            8 j + t of dimension d in nibble t of word (j, d), tokens past L
 *            zero), which wq_kv_block_values makes from that call's layout;
 *   out      bf16 [B, Hq, D] = softmax(q . k^T / sqrt(D)) . v over the L
 *            cached tokens, computed as follows (the page gives no formulas;
 *            this is the library's reading):
 *   - the query row is split into n_components int8 digit planes a_c with
 *     scales sigma_c (the rules of wq_msd_decompose); the scores are
 *     s[l] = sk[l] sum_c sigma_c (sum_d a_c[d] qk[l][d] - zk[l] sum_d a_c[d])
 *     / sqrt(D), with exact integer inner sums;
 *   - per chunk j of 256 tokens: m_j = max s, e = exp(s - m_j), E_j = sum e,
 *     and w = e * sv (fp32) split into digit planes b_c with scales tau_c by
 *     the same rules, the chunk's tokens taken as one row; then
 *     O_j[d] = sum_c tau_c (sum_l b_c[l] qv[l][d] - sum_l b_c[l] zv[l]), exact
 *     integer inner sums;
 *   - out = sum_j e^(m_j - M) O_j / sum_j e^(m_j - M) E_j, M = max_j m_j.
 * With n_components == 2 both products carry ~16-bit operands, so out agrees
 * with fp32 attention over the dequantized cache to bf16 rounding plus the
 * fp32 error of the softmax. B == 0 is a no-op; L == 0, Hq % Hkv != 0, or
 * n_components outside 1..3 return WQ_ERR_INVALID_ARG; D != 128,
 * n_components == 3, an R outside {1, 2, 4, 8}, B or Hkv > 65535, L >
 * 2^31 - 257 or B * Hq > 2^31 - 1 return WQ_ERR_UNSUPPORTED. Workspace: at
 * least wq_msd_decode_attention_workspace(...) bytes; contents on entry do
 * not matter. Asynchronous on `stream`; every buffer is caller-owned.
 */
wq_status wq_msd_decode_attention(const void* q, int64_t B, int64_t Hq, int64_t Hkv, int64_t L,
                                  int32_t D, int32_t n_components, const void* k_codes,
                                  const void* k_scales, const void* k_zeros, const void* v_codes,
                                  const void* v_scales, const void* v_zeros, void* out,
                                  void* workspace, size_t ws_bytes, void* stream);

/*
 * The value-cache layout of wq_msd_decode_attention: V codes from the token
 * layout of wq_quantize_pack (uint32 [rows * L, D / 8], element d in nibble
 * d % 8 of word d / 8) to blocks of 8 tokens, out uint32 [rows, ceil(L/8), D]
 * (token 8 j + t of dimension d in nibble t of word (j, d); nibbles of tokens
 * past L are 0). rows is the number of (sequence, head) pairs. One word then
 * holds 4 tokens of one dimension in its low nibbles and 4 in its high
 * nibbles, the operand layout of the attention's value product. rows == 0 is
 * a no-op; L <= 0 or D not a positive multiple of 8 return
 * WQ_ERR_INVALID_ARG. Bit-exact rearrangement; asynchronous on `stream`.
 */
wq_status wq_kv_block_values(const uint32_t* codes, int64_t rows, int64_t L, int32_t D,
                             uint32_t* out, void* stream);

/*
 * Workspace bytes of wq_msd_decode_attention (0 for B == 0); the same shape
 * checks and status codes. Host only; `bytes` is a host pointer.
 */
wq_status wq_msd_decode_attention_workspace(int64_t B, int64_t Hq, int64_t Hkv, int64_t L,
                                            int32_t D, int32_t n_components, size_t* bytes);

/*
 * Workspace bytes an entry point needs for the given problem (0 if none);
 * for WQ_OP_MX_GEMV, n_components is the number of passes (1 or 2).
 * Host only; `bytes` is a host pointer.
 */
wq_status wq_workspace_bytes(wq_op op, int64_t M, int64_t N, int64_t K,
                             int32_t group, int32_t n_components,
                             size_t* bytes);

/*
 * Test hook for the bounded device waits. The pages have no counterpart: it
 * exists so that the timeout path can be exercised without a device fault.
 * It applies to every later launch, in this process, of the kernels with
 * bounded waits (the tensor-core kernels of wq_w4a16_gemm, and of
 * wq_msd_gemm for M > 16):
 *   limit_ns  how long any one device wait may last before the kernel gives
 *             up; 0 restores the default of 2 s;
 *   stall     1: the kernel's loader withholds the first k-tile, so the first
 *             waits on it expire after limit_ns; 0: normal operation.
 * A kernel that gives up records its wait site for wq_device_error
 * (WQ_ERR_TIMEOUT), waits (bounded by limit_ns) for the copies and
 * tensor-core operations it has in flight, frees its tensor memory and
 * returns; its output is then unspecified. Host only; process-wide; change it
 * only while no such kernel is being launched from another thread.
 * Returns WQ_ERR_INVALID_ARG for a stall other than 0 or 1.
 */
wq_status wq_test_set_wait(uint64_t limit_ns, int stall);

/*
 * Test hook for wq_msd_decode_attention. The pages have no counterpart: it
 * exists so that tests can reach, at small sizes, the chunk-streaming path
 * that large problems take. Each CTA of the attention kernel streams
 * chunks_per_cta consecutive 256-token chunks of one (sequence, KV head) and
 * merges them in registers; by default (0) the count is chosen per launch
 * (1..8, from the problem size and the SM count). 1..64 fixes it for every
 * later launch in this process; the result differs only by fp32 rounding.
 * Host only; process-wide; change it only while no attention call is being
 * made from another thread. Returns WQ_ERR_INVALID_ARG outside 0..64.
 */
wq_status wq_test_set_attention_split(int32_t chunks_per_cta);

/*
 * Read (and, if `clear` != 0, reset) the library's sticky device error word,
 * which kernels with bounded waits set when a wait expires. SYNCHRONISES
 * `stream` first. Returns WQ_ERR_TIMEOUT if the word was set, WQ_OK if not.
 * `detail` (host, may be NULL) receives the raw word: the id of the kernel
 * role and wait site that gave up.
 */
wq_status wq_device_error(void* stream, int clear, uint32_t* detail);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* WQ_H_ */
