/*
 * fp8mm.h -- C ABI of the B200 (sm_100a) scaled FP8 GEMM library (libfp8mm.so).
 *
 * The library computes the scaled FP8 GEMM at the core of FP8 LLM inference,
 *     C_bf16 = (A_e4m3 * scale_a) x (B_e4m3 * scale_b),
 * in the two scale modes of the source pages, together with the bf16 -> E4M3
 * quantizer of each mode:
 *   mode 1, per-token / per-channel fp32 scales -- the deep_gemm.fp8_gemm call
 *           of page "FP8 推理基础设施（五）：从 DeepGEMM 到 vLLM", listing 1
 *           (A, B, m, n, k, scale_a[m], scale_b[n]); scale = max|x| / 448 as
 *           in listing 3 (_calibrate_scales).
 *   mode 2, MXFP8 1x32 block scales along K with UE8M0 exponents -- the
 *           mm_mxfp8 path of page "[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합"
 *           (section 1: one uint8 scale per 32 elements of K, [n, k // 32];
 *           section 2: the GEMM call on the quantized activation and the
 *           pre-processed weight).
 * Around them: a per-tensor calibration scale, a static-scale quantizer and
 * an fp8_gemm with E4M3 output (listing 3 as printed; listing 1's C_fp8); a
 * decode GEMM from a bf16 activation that quantizes it in the kernel
 * (mxfp8_quantize_gemm); and the FP8 key assembly of multi-head latent
 * attention (concat_mla_k, page "[flashinfer] FlashInfer, FP8 지원으로 장문
 * 컨텍스트 추론 성능을 극적으로 향상시키다").
 *
 * Conventions shared by every entry point
 *   - Pointers named *_bf16, *_e4m3, c, scale*, sf* are DEVICE pointers owned
 *     by the caller.  The library never allocates, frees or retains device
 *     memory; it keeps only per-device launch settings.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued asynchronously on it.  No call syncs the
 *     host, except fp8mm_last_device_error and fp8mm_selftest_wait_timeout.
 *   - Every kernel is launched with programmatic stream serialisation: it may
 *     begin (set-up, and for the small-M kernel under
 *     FP8MM_FLAG_WEIGHTS_READY the weight stream) while the preceding kernel
 *     on the stream finishes, and waits for it in-kernel
 *     (griddepcontrol.wait) before it reads an input or writes an output
 *     that kernel may use.  Stream order is therefore kept as for ordinary
 *     launches.
 *   - Matrices are row-major.  A is [m, k] and B is given as [n, k] (the
 *     transpose of the pages' logical [k, n], K contiguous -- the "weight_t"
 *     layout of the mm_mxfp8 call).  C is [m, n] bf16 with row stride ldc
 *     elements.
 *   - E4M3 is the OCP "fn" variant (max finite 448, no infinities).  Encoding
 *     rounds to nearest even and saturates to +-448.  bf16 output rounds to
 *     nearest even.
 *   - Inputs must be finite; NaN/Inf inputs give unspecified results.
 *   - Argument errors are returned synchronously, before any CUDA call, so
 *     they can be checked without a GPU.  A device that is not sm_100 gives
 *     FP8MM_ERR_UNSUPPORTED.
 *   - Every wait inside a kernel is bounded.  On expiry the kernel records a
 *     device error word, frees what it holds and returns.  The host reads the
 *     word with fp8mm_last_device_error().
 */
#ifndef FP8MM_H
#define FP8MM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int fp8mm_status;

#define FP8MM_OK 0
#define FP8MM_ERR_NULL 1          /* a required pointer is NULL */
#define FP8MM_ERR_SHAPE 2         /* negative size, or k not a multiple of the mode's granule */
#define FP8MM_ERR_ALIGN 3         /* pointer or leading dimension breaks the 16-byte rules */
#define FP8MM_ERR_UNSUPPORTED 4   /* no sm_100 device current */
#define FP8MM_ERR_LAUNCH 5        /* a CUDA call failed (the CUDA error is in fp8mm_last_cuda_error) */
#define FP8MM_ERR_WORKSPACE 6     /* split-K requested without a large enough workspace */
#define FP8MM_ERR_DEVICE 7        /* a kernel recorded a device-side error (bounded wait expired) */

/* Optional knobs of the GEMM calls (pass NULL for defaults). */
typedef struct fp8mm_opts {
  /* Device scratch for split K: fp32 partial tiles plus 32-bit arrival
   * counters, fp8mm_workspace_bytes(m, n, k, small_m_ctas) bytes, 256-byte
   * aligned.  Used by the small-M kernel (mxfp8_gemm, m <= 64) and, for
   * m > 64 and K >= 8192, by the paired-SM kernel: the 256 x 256 tiles of its
   * last, partly filled wave of SM pairs (all tiles, where they fill less than
   * one wave) have their K range split over several pairs, so that the wave
   * keeps every pair busy (fp8mm_workspace_bytes is 0 for shapes that are
   * never split).
   * Caller-owned.  It must be zeroed once before first use (e.g.
   * cudaMemsetAsync); every successful call leaves the counters zero again.
   * After a call that reported FP8MM_ERR_DEVICE it must be zeroed again.
   * Calls sharing one workspace must not overlap on the GPU.  NULL disables
   * split K.  A workspace too small for the split the shape takes is
   * FP8MM_ERR_WORKSPACE. */
  void* workspace;
  size_t workspace_bytes;
  /* Kernel choice: FP8MM_KERNEL_AUTO (small-M kernel for mxfp8_gemm with
   * m <= 64, paired-SM tiles for m >= 256, single-SM tiles otherwise, and
   * single-SM 128x128 tiles where the 256-wide tiles would need more waves:
   * shapes that leave most SMs idle, such as 2048 x 1024),
   * FP8MM_KERNEL_TILED (tiled, chosen by size as for AUTO),
   * FP8MM_KERNEL_SMALL_M (weights on the MMA M side, tokens on N; mxfp8_gemm
   * only, m <= 64), FP8MM_KERNEL_TILED_1SM (persistent 128x256 tiles, one CTA
   * per SM), FP8MM_KERNEL_TILED_2SM (256x256 tiles on 2-CTA clusters with
   * cta_group::2 MMAs; each CTA loads its own halves of A and B) or
   * FP8MM_KERNEL_TILED_1SM_N128 (persistent 128x128 tiles, one CTA per SM,
   * two accumulators in both scale modes). */
  int32_t kernel;
  /* Number of CTAs for the small-M kernel's stream-K split (0 = automatic:
   * one or two per SM, at least 4 K slabs of 128 per CTA, replaced by a
   * tile-aligned count with s dividing the K slabs where one comes close). */
  int32_t small_m_ctas;
  /* FP8MM_FLAG_* bits. */
  uint32_t flags;
} fp8mm_opts;

/* The small-M kernel is launched with programmatic dependent launch: it may
 * start while the preceding kernel on the stream is still running, and waits
 * for it before reading a, sf_a or writing c / the workspace.  With this flag
 * it also starts streaming b and sf_b (the weights) before that wait, which
 * hides its start-up behind the preceding kernel.  Set it only when b and
 * sf_b were complete before the preceding kernel started (e.g. weights
 * quantized at load time); never when the preceding kernel writes them. */
#define FP8MM_FLAG_WEIGHTS_READY 1u
/* The small-M kernel reduces a split whose CTA count is tile-aligned (s CTAs
 * per 128-row weight tile, 2 <= s <= min(8, ceil(k / 128)); CTA r of a tile
 * takes K slabs [floor(r * nk / s), floor((r + 1) * nk / s)), nk = ceil(k /
 * 128)) inside
 * thread-block clusters of s CTAs, through distributed shared memory, and
 * then needs no workspace.  With this flag it reduces such splits through
 * the workspace instead (identical results; for comparison and testing). */
#define FP8MM_FLAG_SPLIT_VIA_WORKSPACE 2u
/* mxfp8_gemm / small-M kernel only (m <= 64; FP8MM_ERR_SHAPE otherwise):
 * sf_a is in the small-M scale layout written by mxfp8_quantize_8x4 instead
 * of the 128-row chunk layout. */
#define FP8MM_FLAG_SF_A_8X4 4u

#define FP8MM_KERNEL_AUTO 0
#define FP8MM_KERNEL_TILED 1
#define FP8MM_KERNEL_SMALL_M 2
#define FP8MM_KERNEL_TILED_1SM 3
#define FP8MM_KERNEL_TILED_2SM 4
#define FP8MM_KERNEL_TILED_1SM_N128 5

/* ---------------------------------------------------------------- mode 1 */

/* Per-row E4M3 quantizer (mode 1) -- page "从 DeepGEMM 到 vLLM", listing 3
 * (scale = max|x| / 448) applied per row, feeding listing 1's per-token
 * scale_a (rows of A) and per-channel scale_b (rows of B^T).
 *   x_bf16  [rows, k] bf16, row stride ld_x elements
 *   q_e4m3  [rows, k] E4M3 bytes out, row stride ld_q bytes
 *   scale   [rows] fp32 out: s[r] = amax_r / 448 (IEEE fp32 division), 1.0 for
 *           an all-zero row
 *   q[r, j] = E4M3_RNE_sat(x[r, j] / s[r]) with an IEEE fp32 quotient.
 * Requires k % 8 == 0, ld_x % 8 == 0, ld_q % 8 == 0, ld_x >= k, ld_q >= k,
 * x 16-byte aligned, q 8-byte aligned, scale 4-byte aligned.
 * rows == 0 is a no-op; k == 0 writes scale = 1. */
fp8mm_status fp8_quantize_rowwise(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x,
                                  void* q_e4m3, int64_t ld_q, float* scale, void* stream);

/* Per-token / per-channel scaled FP8 GEMM (mode 1) -- deep_gemm.fp8_gemm of
 * page "从 DeepGEMM 到 vLLM", listing 1.
 *   c[i, j] = bf16_RNE( scale_a[i] * scale_b[j] * sum_k dec(a[i,k]) dec(b[j,k]) )
 * with fp32 accumulation on the tensor cores.
 *   a [m, k] E4M3 (row stride k bytes), b [n, k] E4M3 (row stride k bytes),
 *   scale_a [m] fp32, scale_b [n] fp32, c [m, n] bf16 with row stride ldc.
 * Requires k % 16 == 0, a/b 16-byte aligned, c 2-byte aligned, ldc >= n (rows
 * whose address is 16-byte aligned are written with 16-byte stores).
 * m == 0 or n == 0 is a no-op; k == 0 writes zeros.  opt may be NULL; with
 * opt->workspace, m > 64 shapes split the K range of the tiles of their last
 * wave of SM pairs over the pairs (see fp8mm_opts.workspace). */
fp8mm_status fp8_gemm(const void* a_e4m3, const void* b_e4m3, int64_t m, int64_t n, int64_t k,
                      const float* scale_a, const float* scale_b, void* c_bf16, int64_t ldc,
                      const fp8mm_opts* opt, void* stream);

/* ------------------------------------------------ per-tensor scale, FP8 out */

/* Per-tensor scale -- page "FP8 推理基础设施（五）：从 DeepGEMM 到 vLLM",
 * listing 3 (_calibrate_scales as printed: one scale per tensor):
 *   *scale = fp32(max |x| / 448) over the whole [rows, k] bf16 tensor (row
 *   stride ld_x elements), 1.0 for an all-zero tensor.
 * *scale is a device fp32 that the call overwrites (it is also the work word
 * of the reduction).  Requires k % 8 == 0, x 16-byte aligned, ld_x % 8 == 0,
 * rows * k / 8 < 2^32.  Three kernels on the stream (zero the word, fold
 * the maximum into it, divide).  rows == 0 or k == 0 writes 1.0. */
fp8mm_status fp8_tensor_scale(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, float* scale,
                              void* stream);

/* Static-scale quantizer (a calibrated per-tensor scale, as the same listing
 * uses it at inference; also the FP8 KV-cache quantizer):
 *   q[r, j] = E4M3_RNE_sat(fp32(x[r, j] / *scale))   (IEEE fp32 quotient)
 * scale: device fp32 > 0, read once by the kernel.  Layout and alignment
 * rules as fp8_quantize_rowwise; rows * k / 8 < 2^32. */
fp8mm_status fp8_quantize_static(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, const float* scale,
                                 void* q_e4m3, int64_t ld_q, void* stream);

/* fp8_gemm with an E4M3 output (listing 1's C_fp8), scaled for the next
 * layer:  c[m, n] = E4M3_RNE_sat( fp32(scale_a[m] scale_b[n] acc[m, n]) / *scale_out )
 * where acc is the fp32 tensor-core sum over K; scale_out is a device fp32
 * (e.g. from fp8_tensor_scale on calibration data).  c_e4m3 [m, n] bytes with
 * row stride ldc >= n, any alignment; other arguments and rules as fp8_gemm.
 * The quotient is within one fp32 step of the IEEE quotient (exact tensor-
 * core accumulation order is not defined anyway); outputs past +-448 saturate. */
fp8mm_status fp8_gemm_e4m3_out(const void* a_e4m3, const void* b_e4m3, int64_t m, int64_t n, int64_t k,
                               const float* scale_a, const float* scale_b, const float* scale_out, void* c_e4m3,
                               int64_t ldc, const fp8mm_opts* opt, void* stream);

/* ---------------------------------------------------------------- mode 2 */

/* Scale-factor (SF) layout of this library.  Rows are padded to a multiple of
 * 128 and K-blocks (32 elements each) to a multiple of 4.  The buffer is made
 * of 512-byte chunks, one per (128-row tile rt, group of 4 K-blocks kc),
 * ordered rt-major: chunk (rt, kc) starts at (rt * n_kc + kc) * 512 with
 * n_kc = ceil(k / 128).  Inside a chunk, the byte of row r and block b is
 *     (r % 32) * 16 + ((r % 128) / 32) * 4 + (b % 4),
 * i.e. each 32-bit word holds the 4 block exponents of one row and each 16-byte
 * line holds rows r, r+32, r+64, r+96 -- the shape one tcgen05.cp (32x128b,
 * warpx4) moves into tensor memory.  Padding bytes are written as 0.
 * Byte value e encodes the scale 2^(e - 127) (UE8M0). */
size_t fp8mm_sf_bytes(int64_t rows, int64_t k);
/* Byte offset of (row, block) in that layout; -1 when out of range. */
int64_t fp8mm_sf_offset(int64_t rows, int64_t k, int64_t row, int64_t block);
/* Host-memory permutations between that layout and the canonical row-major
 * [rows, k/32] scale tensor of the pages ([n, k // 32]).  Both pointers are
 * HOST pointers; nothing is launched. */
fp8mm_status fp8mm_sf_to_canonical(const uint8_t* sf, int64_t rows, int64_t k, uint8_t* canonical);
fp8mm_status fp8mm_sf_from_canonical(const uint8_t* canonical, int64_t rows, int64_t k, uint8_t* sf);

/* MXFP8 quantizer (mode 2) -- one UE8M0 exponent per 32 elements of K as in
 * page "[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합", section 1, with the
 * amax/448 rule of page "从 DeepGEMM 到 vLLM", listing 3, restricted to powers
 * of two:  e = clamp(ceil(log2(amax / 448)) + 127, 0, 254)  (e = 127 for an
 * all-zero block), q = E4M3_RNE_sat(x * 2^(127 - e)) (the scaling is exact).
 *   x_bf16 [rows, k] bf16, row stride ld_x; q_e4m3 [rows, k], row stride ld_q;
 *   sf     fp8mm_sf_bytes(rows, k) bytes in the layout above (written whole,
 *          padding included).
 * Requires k % 32 == 0, ld_x % 8 == 0, ld_q % 8 == 0, x 16-byte aligned,
 * q 8-byte aligned, sf 16-byte aligned.  rows == 0 or k == 0 is a no-op. */
fp8mm_status mxfp8_quantize(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, void* q_e4m3,
                            int64_t ld_q, uint8_t* sf, void* stream);

/* Small-M scale layout, for activations of a few token rows -- the
 * use_8x4_sf_layout option of the mm_mxfp8 call on page "[sglang] FlashInfer
 * v0.6.7 MXFP8 Gemm 통합", section 2, in this library's own form: rows are
 * padded to a multiple of 8 (not 128) and K-blocks to a multiple of 4.  The
 * buffer is made of 32-byte atoms of 8 rows x 4 K-blocks; atom (r8, g) sits at
 * (g * ceil(rows / 8) + r8) * 32, and inside it the byte of row r and block b
 * is (r % 8) * 4 + (b % 4).  So for each 128-wide K slab g the 32-bit scale
 * words of all rows are contiguous: byte ((b / 4) * rows_pad8 + r) * 4 + b % 4.
 * Padding bytes are written as 0.  Byte value e encodes 2^(e - 127). */
size_t fp8mm_sf8x4_bytes(int64_t rows, int64_t k);
/* Byte offset of (row, block) in the small-M layout; -1 when out of range. */
int64_t fp8mm_sf8x4_offset(int64_t rows, int64_t k, int64_t row, int64_t block);
/* mxfp8_quantize with the scales in the small-M layout (sf:
 * fp8mm_sf8x4_bytes(rows, k) bytes, written whole, padding included); the
 * codes and exponents are those of mxfp8_quantize.  Same arguments and rules. */
fp8mm_status mxfp8_quantize_8x4(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, void* q_e4m3,
                                int64_t ld_q, uint8_t* sf, void* stream);

/* MXFP8 block-scaled GEMM (mode 2) -- the mm_mxfp8(a, b_t, a_sf, b_sf,
 * out_dtype=bf16) call of page "[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합",
 * section 2, with the scales consumed inside the tensor-core MMA:
 *   c[i, j] = bf16_RNE( sum_b 2^(ea[i,b]-127) 2^(eb[j,b]-127) sum_{k in b} dec(a) dec(b) )
 *   a [m, k], sf_a fp8mm_sf_bytes(m, k); b [n, k], sf_b fp8mm_sf_bytes(n, k);
 *   c [m, n] bf16, row stride ldc.
 * Requires k % 32 == 0, a/b/sf 16-byte aligned, c 2-byte aligned, ldc >= n.
 * With m <= 64 the small-M (decode) kernel runs: weights b fill the MMA's
 * 128-row side, tokens the N side, and K is split stream-K style over the SMs
 * when opt->workspace is given (see fp8mm_workspace_bytes); partial sums are
 * reduced deterministically (fixed order) by the last CTA of each tile.  With
 * m > 64 and a workspace, the 256 x 256 tiles of the last, partly filled
 * wave of SM pairs (all tiles, where they fill less than one wave) split
 * their K range over pairs the same way. */
fp8mm_status mxfp8_gemm(const void* a_e4m3, const uint8_t* sf_a, const void* b_e4m3, const uint8_t* sf_b,
                        int64_t m, int64_t n, int64_t k, void* c_bf16, int64_t ldc, const fp8mm_opts* opt,
                        void* stream);

/* Decode-shape MXFP8 GEMM from a bf16 activation: the result equals
 * mxfp8_quantize(a) followed by mxfp8_gemm(...) with the small-M kernel and
 * the same options, bit for bit (page "[sglang] FlashInfer v0.6.7 MXFP8 Gemm
 * 통합", section 2: the activation is quantized per call, the weights once).
 * For m <= 8 the activation is quantized inside the GEMM kernel: one launch
 * and no intermediate E4M3 activation in memory.  For 8 < m <= 64 the
 * quantizer runs as its own launch into the tail of the workspace, which is
 * then required.
 *   a_bf16  [m, k] bf16 activation, row stride lda elements (16-byte aligned,
 *           lda % 8 == 0, lda >= k)
 *   b_e4m3, sf_b, c_bf16, ldc, opt, stream: as for mxfp8_gemm (opt->kernel
 *           must be FP8MM_KERNEL_AUTO or FP8MM_KERNEL_SMALL_M; small_m_ctas
 *           and FP8MM_FLAG_WEIGHTS_READY act as there)
 *   opt->workspace: optional for m <= 8 (as for mxfp8_gemm); for m > 8 at
 *           least fp8mm_quantize_gemm_workspace_bytes(m, n, k, small_m_ctas)
 *           bytes, 256-byte aligned (FP8MM_ERR_WORKSPACE otherwise)
 * Requires 0 <= m <= 64 and k % 32 == 0 (FP8MM_ERR_SHAPE otherwise).
 * m == 0 or n == 0 is a no-op; k == 0 writes zeros. */
fp8mm_status mxfp8_quantize_gemm(const void* a_bf16, int64_t lda, const void* b_e4m3, const uint8_t* sf_b,
                                 int64_t m, int64_t n, int64_t k, void* c_bf16, int64_t ldc, const fp8mm_opts* opt,
                                 void* stream);
/* Workspace bytes mxfp8_quantize_gemm needs: fp8mm_workspace_bytes(m, n, k,
 * ctas), plus for m > 8 room for the quantized activation and its scales
 * (each 256-byte aligned).  0 for m outside [1, 64]. */
size_t fp8mm_quantize_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k, int32_t ctas);

/* Workspace bytes a GEMM of this shape uses: for m <= 64 those of the
 * small-M kernel with `ctas` CTAs (0 = its automatic choice); for m > 64 those
 * of the paired-SM kernel's K split (`ctas` ignored): room for one split part
 * per SM pair, (SMs / 2) x 256 KiB of partials plus the counters, whatever
 * the tile count, for K >= 8192, and 0 below (never split).  The current
 * device's SM count decides; on a host without a GPU, 148. */
size_t fp8mm_workspace_bytes(int64_t m, int64_t n, int64_t k, int32_t ctas);

/* The paired-SM kernel's K split for an m > 64 call with a workspace when
 * `pairs` SM pairs run at once: returns the K parts of each split tile (1: no
 * split) and stores in *dp_tiles (if not NULL) how many of the ceil(m/256) x
 * ceil(n/256) tiles, taken in raster order, run whole; the rest, the last
 * partly filled wave, are split.  Parts: the most that fit the pairs that
 * wave leaves, each of at least 16 K slabs of 128, at most 8; none for
 * m <= 64, K < 8192, or tiles that fill whole waves.  Host-only; a planning
 * query with no device work (invalid sizes give 1 and 0). */
int32_t fp8mm_pair_split_plan(int64_t m, int64_t n, int64_t k, int32_t pairs, int32_t* dp_tiles);

/* ---------------------------------------------------------------- KV cache */

/* Key assembly for multi-head latent attention, for FP8 (E4M3 / E5M2) or
 * 16-bit elements -- page "[flashinfer] FlashInfer, FP8 지원으로 장문 컨텍스트
 * 추론 성능을 극적으로 향상시키다", 코드 분석 items 1 and 3:
 *   k_out[t, h, 0:nope_dim]                   = k_nope[t, h, :]
 *   k_out[t, h, nope_dim:nope_dim + rope_dim] = k_rope[t, h, :]
 * for t < num_tokens, h < num_heads.  A copy: the output bytes are the input
 * bytes.  rope_stride_h = 0 broadcasts one rope vector per token to every
 * head.  All strides are in elements of elem_bytes (1 or 2) bytes; every
 * pointer is 16-byte aligned and every stride, nope_dim and rope_dim times
 * elem_bytes is a multiple of 16 (FP8MM_ERR_ALIGN otherwise);
 * num_tokens * num_heads * (nope_dim + rope_dim) * elem_bytes / 16 < 2^32.
 * num_tokens == 0 or num_heads == 0 is a no-op. */
fp8mm_status concat_mla_k(const void* k_nope, const void* k_rope, void* k_out, int64_t num_tokens,
                          int64_t num_heads, int64_t nope_dim, int64_t rope_dim, int64_t elem_bytes,
                          int64_t nope_stride_t, int64_t nope_stride_h, int64_t rope_stride_t,
                          int64_t rope_stride_h, int64_t out_stride_t, int64_t out_stride_h, void* stream);

/* ---------------------------------------------------------------- misc */

const char* fp8mm_status_str(fp8mm_status status);
/* CUDA error code of the last failed CUDA call made by the library (0 if none). */
int fp8mm_last_cuda_error(void);
/* Synchronizes the current device, returns the device error word (0 = none;
 * bits 0-7 kind (1 = bounded wait expired), 8-15 wait site, 16-31 CTA) and
 * clears it. */
unsigned int fp8mm_last_device_error(void);
/* Self-test of the bounded wait: launches one CTA that waits on an mbarrier
 * nothing will ever arrive at, with a limit of timeout_us microseconds, and
 * returns after it.  Returns FP8MM_ERR_DEVICE when the wait expired and was
 * reported as it should be (and clears the word), FP8MM_OK if it unexpectedly
 * completed. */
fp8mm_status fp8mm_selftest_wait_timeout(uint32_t timeout_us, void* stream);
/* ABI version of this header: major * 10000 + minor * 100 + patch. */
int fp8mm_version(void);


/* ------------------------------------------------- no-allocation variant */

/* Small-M MXFP8 GEMM (the same arithmetic and kernel as mxfp8_gemm with
 * m <= 64) for callers that cannot allocate device memory.  The source pages
 * have no counterpart: this entry point exists for how the library is called,
 * not for what it computes.
 *
 * Who needs it: a caller whose device memory is fully reserved up front by
 * its own pool (a serving engine that hands nearly all HBM to its KV cache),
 * a caller on a latency-critical path where cudaMalloc's implicit device
 * synchronisation is not acceptable, or a plain-C host with no allocator for
 * the split-K workspace that mxfp8_gemm needs.  Such a caller still passes
 * its inputs and output; the split-K partial sums and arrival counters live
 * in a fixed 8 MiB array inside the library (FP8MM_NOALLOC_SCRATCH_BYTES),
 * which every GPU that loads the library holds until the process exits.
 *
 *   a [m, k], sf_a, b [n, k], sf_b, c [m, n] (row stride ldc): as in
 *   mxfp8_gemm.  Requires 1 <= m <= 64 (else FP8MM_ERR_SHAPE), k % 32 == 0,
 *   and at most 16384 weight tiles, i.e. n <= 2097152 (else
 *   FP8MM_ERR_WORKSPACE: the request does not fit the fixed scratch).  The
 *   stream-K split uses the CTA count mxfp8_gemm would choose, capped at what
 *   the scratch holds (508 CTAs for up to 16 tokens, 127 for 49..64).
 *
 * Allocates nothing: no cudaMalloc / cudaFree and no allocating library
 * call.  The first call on each device looks up the scratch array's device
 * address (cudaGetSymbolAddress, with that device current) and caches it;
 * make that first call before any stream capture.  Every call clears the
 * counters it uses (an async memset on `stream`) before its kernel runs.
 * All calls share the one array, which keeps the last call's contents, so
 * calls that overlap on the GPU (e.g. on two streams) race: serialise them. */
#define FP8MM_NOALLOC_SCRATCH_BYTES (8u << 20)
fp8mm_status mxfp8_gemm_small_m_noalloc(const void* a_e4m3, const uint8_t* sf_a, const void* b_e4m3,
                                        const uint8_t* sf_b, int64_t m, int64_t n, int64_t k, void* c_bf16,
                                        int64_t ldc, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FP8MM_H */
