/*
 * oracle.h -- plain, slow, obviously correct CPU oracle for the scaled FP8 GEMM
 * and its bf16 -> E4M3 quantizers, in both scale modes.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
 * baseline of the benchmark may load this library.  The product path (the
 * CUDA library and its Python binding) never calls it, and the two share no
 * code, header, table or constant.
 *
 * Sources (web pages on FP8 / MXFP8 inference; cited by title and section):
 *  [DG]  "FP8 推理基础设施（五）：从 DeepGEMM 到 vLLM" -- listing 1 (the
 *        deep_gemm.fp8_gemm call with per-token scale_a[m] and per-channel
 *        scale_b[n], fp32), listing 3 (_calibrate_scales: scale = max|x| / 448,
 *        "E4M3 max is 448").
 *  [MX]  "[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합" -- section 1 (weight
 *        preprocessing: one uint8 scale per 32 elements of K, scale tensor
 *        shaped [n, k // 32], num_elts_per_sf = 32) and section 2 (the
 *        mm_mxfp8 call on the quantized activation and its x_scale_u8).
 *  [ROCm] "为什么在 Instinct GPU 上死磕 FP8？" -- fp8 means E4M3.
 *
 * Where the pages leave a step open, the reading taken is stated beside the
 * function (formats: OCP 8-bit float E4M3 "fn" variant; UE8M0 = 2^(e-127)).
 *
 * Floating point is fp64 except where the data itself is fp32 (the scale
 * vectors are fp32 tensors in [DG] listing 1, and the scaled activation is
 * formed in fp32 before the cast, as the kernel does).
 */
#ifndef FP8_ORACLE_H
#define FP8_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* E4M3 decode of one code byte, from the bit definition: sign s = b>>7,
 * exponent E = (b>>3)&15 (bias 7), mantissa m = b&7.  E=0: (-1)^s m 2^-9
 * (subnormal); E=15,m=7: NaN (0x7F, 0xFF); else (-1)^s (1+m/8) 2^(E-7).
 * Max finite 0x7E = 448 ([DG] listing 3).  Returns NaN for the two NaN codes. */
double orc_e4m3_decode(uint8_t code);

/* E4M3 encode of a finite value: nearest of the 127 non-negative finite
 * magnitudes (codes 0x00..0x7E), ties to the even code, |v| >= 448 saturates
 * to 448 (0x7E), sign bit kept (so -0 and negatives that round to zero give
 * 0x80).  The search is a plain binary search over the decoded magnitudes. */
uint8_t orc_e4m3_encode(double v);

/* MX block exponent of a block maximum a >= 0:
 * e = ceil(log2(a / 448)) + 127, clamped to [0, 254]; a == 0 gives 127
 * (scale 1).  The smallest power-of-two scale 2^(e-127) with a / scale <= 448,
 * i.e. the amax/448 rule of [DG] listing 3 restricted to UE8M0 scales ([MX]). */
int orc_mx_exponent(double amax);

/* Per-tensor scale ([DG] listing 3, _calibrate_scales as printed: one scale
 * per tensor, max |x| over all of it / 448): s = fp32(amax / 448), 1 when the
 * tensor is all zero.  x: bf16 bit patterns, rows x k, row stride ld_x. */
float orc_tensor_scale(const uint16_t* x, int64_t rows, int64_t k, int64_t ld_x);

/* Static-scale quantizer: q[r, j] = encode(fp32(x[r, j] / s)) with one given
 * fp32 scale s > 0 for the whole tensor (a calibrated per-tensor scale, as
 * [DG] listing 3 computes once and then uses for inference). */
void orc_quantize_static(const uint16_t* x, int64_t rows, int64_t k, int64_t ld_x, float s,
                         uint8_t* q, int64_t ld_q, int nthreads);

/* Per-row quantizer (mode 1).  For each row r of x (bf16 bit patterns,
 * row stride ld_x elements): amax = max |x|; s[r] = fp32(amax / 448)
 * (s = 1 when amax == 0); q[r, j] = encode(fp32(x[r, j] / s[r])).
 * q has row stride ld_q bytes.  The same call quantizes B per channel when
 * given B^T (rows = output channels). */
void orc_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t k, int64_t ld_x,
                          uint8_t* q, int64_t ld_q, float* s, int nthreads);

/* MX quantizer (mode 2).  k % 32 == 0.  For each row r and block b of 32
 * consecutive elements along K: e = orc_mx_exponent(max |x|) and
 * q = encode(x * 2^(127 - e)) (exact in fp64).  sf is canonical row-major
 * [rows, k/32] uint8 -- the [n, k // 32] shape of [MX] section 1. */
void orc_mx_quantize(const uint16_t* x, int64_t rows, int64_t k, int64_t ld_x,
                     uint8_t* q, int64_t ld_q, uint8_t* sf, int nthreads);

/* Mode-1 GEMM reference.  qa [m,k], qb [n,k] E4M3 codes (row-major, K
 * contiguous; B is given as B^T), sa [m], sb [n] fp32.
 *   c_ref[i,j] = sa[i] * sb[j] * sum_k dec(qa[i,k]) dec(qb[j,k])
 *   bound[i,j] = sum_k |sa[i] dec(qa[i,k])| |sb[j] dec(qb[j,k])|
 * Every product is a multiple of 2^-18 below 2^18 in magnitude, so the fp64
 * sum is exact for k < 2^17 (any order).  Outputs are fp64 [m,n] row-major;
 * bound may be NULL. */
void orc_gemm_rowwise(const uint8_t* qa, const uint8_t* qb, int64_t m, int64_t n, int64_t k,
                      const float* sa, const float* sb, double* c_ref, double* bound,
                      int nthreads);

/* Mode-2 GEMM reference.  sfa [m, k/32], sfb [n, k/32] canonical UE8M0.
 *   c_ref[i,j] = sum_b 2^(sfa[i,b]-127) 2^(sfb[j,b]-127) sum_{k in b} dec(qa) dec(qb)
 *   bound[i,j] = sum_b 2^(..) 2^(..) sum_{k in b} |dec(qa)| |dec(qb)|
 * The per-block sums are exact; only the cross-block fp64 sum rounds. */
void orc_gemm_mx(const uint8_t* qa, const uint8_t* sfa, const uint8_t* qb, const uint8_t* sfb,
                 int64_t m, int64_t n, int64_t k, double* c_ref, double* bound, int nthreads);

#ifdef __cplusplus
}
#endif
#endif
