// quant.cuh -- bf16 -> E4M3 quantizers for both scale modes (HBM-bound).
//
// Mode 1 (per row):  s = amax / 448 (IEEE fp32 division, 1 for a zero row),
//   q = E4M3_RNE_sat(x / s), x / s the correctly rounded fp32 quotient.  Page "从 DeepGEMM 到 vLLM", listing 3
//   (_calibrate_scales) applied per row; listing 1 takes per-token scale_a
//   and per-channel scale_b.
// Mode 2 (MX, 1x32 blocks along K):  e = clamp(ceil(log2(amax/448)) + 127,
//   0, 254), 127 for a zero block; q = E4M3_RNE_sat(x * 2^(127-e)).  Page
//   "[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합", section 1 (one uint8 scale
//   per 32 elements).
//
// Both kernels read bf16 with 16-byte vector loads; a warp always covers a
// contiguous run of one row.  They are
// launched with programmatic dependent launch and wait for the preceding
// kernel before touching memory, so only their launch overlaps it.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "ptx.cuh"

namespace fp8mm {

// 16-byte streaming load (not kept in L1).  Coherent (no .nc): the kernels
// read inputs that the preceding kernel, overlapping them through
// programmatic dependent launch, may still be writing before their
// griddepcontrol.wait.
__device__ __forceinline__ uint4 ld_stream_16(const void* p) {
  uint4 v;
  asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// The 8 bf16 values of a 16-byte vector as fp32 (exact).
__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float absmax8(const float (&f)[8]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
  return m;
}

// 8 fp32 -> 8 E4M3 bytes (round to nearest even, saturate to +-448), element 0
// in the lowest byte.
__device__ __forceinline__ uint2 f32x8_to_e4m3(const float (&y)[8]) {
  uint32_t b[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    b[i] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(y[2 * i], y[2 * i + 1]),
                                                          __NV_SATFINITE, __NV_E4M3));
  return make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
}

// ------------------------------------------------------------------ mode 1

// x / s correctly rounded to fp32 without a division per element, by
// Markstein's residual correction (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): with r = RN(1/s) and q = RN(x r), the residual e = q s - x is exact
// (one fma) and RN(q - e r) is RN(x / s).  For x with 8 significant bits (any
// bf16 value) this holds for every pair of significands, which a host-side
// test checks exhaustively with IEEE fp32 arithmetic; scaling by powers of two
// keeps it while q, e and r stay in the normal range, which
// quotient_fast_ok() ensures for every element that can give a nonzero code
// (|x| >= 2^-102); smaller |x| give |x / s| < 2^-22 and the code 0 with the
// sign of x either way.  The signs in the two fmas make x = -0 give -0.
__device__ __forceinline__ float quotient_rn(float x, float s, float r) {
  const float q = x * r;
  const float e = __fmaf_rn(q, s, -x);
  return __fmaf_rn(-e, r, q);
}
// Row scales for which quotient_rn() is exact: s in [2^-80, 2^126] (so r is
// normal and every |x| >= 448 s 2^-11 exceeds 2^-102); other rows divide.
__device__ __forceinline__ bool quotient_fast_ok(float s) {
  return s >= 0x1p-80f && s <= 0x1p126f;
}

// x / s where x / s may lie far beyond the E4M3 range (a static scale, a GEMM
// output): an approximation x * r above 1024 means the quotient is past 464
// and saturates to 448 whatever its exact value, so +-1024 is returned (this
// also covers x * r overflowing, where the correction would give NaN);
// otherwise quotient_rn.  For bf16 x the result is the IEEE quotient or
// saturates like it; for fp32 x (GEMM outputs) it is within one fp32 step.
__device__ __forceinline__ float quotient_sat(float x, float s, float r) {
  const float q0 = x * r;
  return fabsf(q0) > 1024.f ? copysignf(1024.f, q0) : quotient_rn(x, s, r);
}

constexpr int kQ1Threads = 256;

// One CTA per row (grid-stride over rows).  The row is held in registers
// (NV 16-byte vectors per thread), so x is read once; rows longer than
// NV * blockDim * 8 elements use the two-pass variant below.
template <int NV>
__global__ void __launch_bounds__(kQ1Threads) quant_rowwise_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                                   int64_t k, int64_t ld_x, uint8_t* __restrict__ q,
                                                                   int64_t ld_q, float* __restrict__ scale) {
  __shared__ float red[kQ1Threads / 32];
  const int nvec = static_cast<int>(k / 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_launch_dependents();
  griddep_wait();  // x and the outputs may belong to the preceding kernel
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const __nv_bfloat16* xr = x + row * ld_x;
    uint4 v[NV];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int idx = threadIdx.x + i * blockDim.x;
      if (idx < nvec) {
        v[i] = ld_stream_16(xr + static_cast<int64_t>(idx) * 8);
        float f[8];
        bf16x8_to_f32(v[i], f);
        amax = fmaxf(amax, absmax8(f));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    float m = 0.f;
    const int nw = blockDim.x >> 5;
    for (int w = 0; w < nw; ++w) m = fmaxf(m, red[w]);
    __syncthreads();  // red[] is rewritten by the next row
    const float s = (m == 0.f) ? 1.f : __fdiv_rn(m, 448.f);
    if (threadIdx.x == 0) scale[row] = s;
    uint8_t* qr = q + row * ld_q;
    if (quotient_fast_ok(s)) {
      const float r = __frcp_rn(s);
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int idx = threadIdx.x + i * blockDim.x;
        if (idx < nvec) {
          float f[8];
          bf16x8_to_f32(v[i], f);
#pragma unroll
          for (int j = 0; j < 8; ++j) f[j] = quotient_rn(f[j], s, r);
          *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(idx) * 8) = f32x8_to_e4m3(f);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int idx = threadIdx.x + i * blockDim.x;
        if (idx < nvec) {
          float f[8];
          bf16x8_to_f32(v[i], f);
#pragma unroll
          for (int j = 0; j < 8; ++j) f[j] = __fdiv_rn(f[j], s);
          *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(idx) * 8) = f32x8_to_e4m3(f);
        }
      }
    }
  }
}

// Long rows: one pass for the maximum, a second pass (mostly from L2) to
// quantize.
__global__ void __launch_bounds__(kQ1Threads) quant_rowwise_2pass_kernel(const __nv_bfloat16* __restrict__ x,
                                                                         int64_t rows, int64_t k, int64_t ld_x,
                                                                         uint8_t* __restrict__ q, int64_t ld_q,
                                                                         float* __restrict__ scale) {
  __shared__ float red[kQ1Threads / 32];
  const int64_t nvec = k / 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_launch_dependents();
  griddep_wait();
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const __nv_bfloat16* xr = x + row * ld_x;
    float amax = 0.f;
    for (int64_t idx = threadIdx.x; idx < nvec; idx += blockDim.x) {
      float f[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(xr + idx * 8), f);
      amax = fmaxf(amax, absmax8(f));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    float m = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
    __syncthreads();
    const float s = (m == 0.f) ? 1.f : __fdiv_rn(m, 448.f);
    if (threadIdx.x == 0) scale[row] = s;
    uint8_t* qr = q + row * ld_q;
    const bool fast = quotient_fast_ok(s);
    const float r = __frcp_rn(s);
    for (int64_t idx = threadIdx.x; idx < nvec; idx += blockDim.x) {
      float f[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(xr + idx * 8), f);
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = fast ? quotient_rn(f[j], s, r) : __fdiv_rn(f[j], s);
      *reinterpret_cast<uint2*>(qr + idx * 8) = f32x8_to_e4m3(f);
    }
  }
}

// ------------------------------------------------------------------ per tensor

// Per-tensor scale (page "FP8 推理基础设施（五）：从 DeepGEMM 到 vLLM", listing 3:
// one scale per tensor, max|x| / 448), in three kernels chained by
// programmatic dependent launch: one thread zeroes the output word (a kernel
// rather than a memset, which cost ~3 us more between the neighbouring
// kernels in a CUDA graph on B200), then every block takes the exact maximum of |x| over its
// share (an unsigned 16-bit max over the sign-cleared bf16 bits, four 16-byte
// loads in flight per thread: one flat run for a contiguous tensor, row by
// row otherwise) and folds it into the word with one atomicMax (bf16 bits
// << 16 are the fp32 bits of the maximum, whose integer order is their value
// order); then one thread turns it into s = amax / 448 (IEEE division), 1 for
// an all-zero tensor.  A single-kernel form that finalized in the last block
// to arrive (a compare-and-swap loop on the same word carrying an arrival
// count in its low half) measured 16 times slower on B200: the blocks finish
// together and their compare-and-swaps serialise.
constexpr int kTensorThreads = 256;
constexpr int kAmaxUnroll = 4;

__global__ void __launch_bounds__(kTensorThreads) tensor_amax_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                                    int64_t k, int64_t ld_x, unsigned* word) {
  griddep_launch_dependents();
  griddep_wait();
  const int vpr = static_cast<int>(k / 8);  // 16-byte vectors per row
  uint32_t m = 0;
  auto fold = [&m](const uint4& w) {
    m = __vmaxu2(__vmaxu2(m, w.x & 0x7FFF7FFFu), __vmaxu2(w.y & 0x7FFF7FFFu, __vmaxu2(w.z & 0x7FFF7FFFu, w.w & 0x7FFF7FFFu)));
  };
  if (ld_x == k) {  // contiguous: one flat run of rows * k / 8 vectors
    const int64_t total = rows * vpr;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kTensorThreads * kAmaxUnroll;
    for (int64_t v0 = static_cast<int64_t>(blockIdx.x) * kTensorThreads * kAmaxUnroll + threadIdx.x; v0 < total;
         v0 += stride) {
      uint4 w[kAmaxUnroll];
#pragma unroll
      for (int u = 0; u < kAmaxUnroll; ++u) {
        const int64_t v = v0 + u * kTensorThreads;
        w[u] = v < total ? ld_stream_16(x + v * 8) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kAmaxUnroll; ++u) fold(w[u]);
    }
  } else {
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const __nv_bfloat16* xr = x + row * ld_x;
    for (int v0 = threadIdx.x; v0 < vpr; v0 += kTensorThreads * kAmaxUnroll) {
      uint4 w[kAmaxUnroll];
#pragma unroll
      for (int u = 0; u < kAmaxUnroll; ++u) {
        const int v = v0 + u * kTensorThreads;
        w[u] = v < vpr ? ld_stream_16(xr + static_cast<int64_t>(v) * 8) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kAmaxUnroll; ++u) fold(w[u]);
    }
  }
  }
  m = max(m & 0xFFFFu, m >> 16) << 16;
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(word, m);
}

__global__ void tensor_scale_zero_kernel(unsigned* word) {
  griddep_launch_dependents();
  griddep_wait();  // the word may still be read by the preceding kernel
  *word = 0u;
}

__global__ void tensor_scale_finalize_kernel(float* scale) {
  griddep_wait();
  const float amax = *scale;  // the maximum's bits, left by tensor_amax_kernel
  *scale = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 448.f);
}

// Static-scale quantizer: q = E4M3_RNE_sat(fp32(x / s)) with one fp32 scale
// for the whole tensor (a calibrated per-tensor scale; also the FP8 KV-cache
// quantizer).  Grid-stride over 16-byte vectors; the quotient is quotient_sat
// (the IEEE quotient, or saturated like it) when quotient_fast_ok(s), else
// an IEEE division.
__global__ void __launch_bounds__(kTensorThreads) quant_static_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                                     int64_t k, int64_t ld_x,
                                                                     const float* __restrict__ scale,
                                                                     uint8_t* __restrict__ q, int64_t ld_q) {
  griddep_launch_dependents();
  griddep_wait();  // the scale and x may be written by the preceding kernel
  const float s = *scale;
  const float r = __frcp_rn(s);
  const bool fast = quotient_fast_ok(s);
  const uint32_t vpr = static_cast<uint32_t>(k / 8);
  const uint32_t total = static_cast<uint32_t>(rows) * vpr;  // < 2^32 (checked by the host)
  for (uint32_t v = blockIdx.x * kTensorThreads + threadIdx.x; v < total; v += gridDim.x * kTensorThreads) {
    const uint32_t row = v / vpr;
    const uint32_t c8 = v - row * vpr;
    float f[8];
    bf16x8_to_f32(ld_stream_16(x + static_cast<int64_t>(row) * ld_x + c8 * 8), f);
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = fast ? quotient_sat(f[j], s, r) : __fdiv_rn(f[j], s);
    *reinterpret_cast<uint2*>(q + static_cast<int64_t>(row) * ld_q + c8 * 8) = f32x8_to_e4m3(f);
  }
}

// ------------------------------------------------------------------ mode 2

// UE8M0 exponent of a block maximum a (an exact bf16 value held in fp32):
// a = (1 + m/128) 2^(Ea-127) and 448 = 1.75 * 2^8, so
// ceil(log2(a/448)) + 127 = Ea - 8 + (m > 96); clamped to [0, 254];
// a bf16 subnormal gives 0 and a == 0 gives 127.
__device__ __forceinline__ int mx_exponent(float a) {
  const uint32_t bits = __float_as_uint(a);
  const int Ea = static_cast<int>(bits >> 23);
  const int m7 = static_cast<int>((bits >> 16) & 0x7Fu);
  if (Ea == 0) return (a == 0.f) ? 127 : 0;
  const int e = Ea - 8 + (m7 > 96 ? 1 : 0);
  return e < 0 ? 0 : (e > 254 ? 254 : e);
}

// 2^(127 - e) as fp32, exactly (e in [0, 254]).
__device__ __forceinline__ float mx_inv_scale(int e) {
  return (e < 254) ? __uint_as_float(static_cast<uint32_t>(254 - e) << 23) : __uint_as_float(0x00400000u);
}

constexpr int kQ2Threads = 256;

// Exact maximum of |x| over the 32 bf16 values of four 16-byte vectors, as
// fp32: for finite bf16 the order of magnitudes is the order of the
// sign-cleared bit patterns, so it is a 16-bit unsigned maximum.
__device__ __forceinline__ float bf16x32_absmax(const uint4 (&v)[4]) {
  uint32_t m = 0;
#pragma unroll
  for (int t = 0; t < 4; ++t)
    m = __vmaxu2(__vmaxu2(m, v[t].x & 0x7FFF7FFFu),
                 __vmaxu2(v[t].y & 0x7FFF7FFFu, __vmaxu2(v[t].z & 0x7FFF7FFFu, v[t].w & 0x7FFF7FFFu)));
  return __uint_as_float(max(m & 0xFFFFu, m >> 16) << 16);
}

// One warp per segment of 32 consecutive K blocks (1024 elements) of one
// padded row, grid-stride over the rows_pad x ceil(n_kc*4 / 32) segments;
// lane L owns block kb = 32*seg + L: four 16-byte loads, its maximum, the
// exponent, 32 E4M3 bytes, and the lanes L % 4 == 0 gather the four
// exponents of one scale word.  The next segment's loads are in flight
// while the current one is converted.  Rows >= rows and blocks >= k/32
// (padding) get exponent 0 and no codes.  k8x4: the scales go to the small-M
// layout (rows padded to 8; the word of row r and K group g at
// (g * rows_pad + r) * 4) instead of the 128-row chunks.
template <bool k8x4 = false>
__global__ void __launch_bounds__(kQ2Threads) quant_mx_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                              int64_t k, int64_t ld_x, uint8_t* __restrict__ q,
                                                              int64_t ld_q, uint8_t* __restrict__ sf, int n_kc,
                                                              int64_t rows_pad) {
  const int lane = threadIdx.x & 31;
  const int nkb = static_cast<int>(k / 32);
  const int nkb4 = n_kc * 4;
  const int segs = (nkb4 + 31) / 32;
  const int64_t total = rows_pad * segs;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * (kQ2Threads / 32);
  int64_t w = static_cast<int64_t>(blockIdx.x) * (kQ2Threads / 32) + (threadIdx.x >> 5);
  // (row, seg) of w, advanced without division
  int64_t row = w / segs;
  int seg = static_cast<int>(w - row * segs);
  const int64_t drow = wstride / segs;
  const int dseg = static_cast<int>(wstride - drow * segs);
  const bool q16 = (reinterpret_cast<uintptr_t>(q) % 16 == 0) && (ld_q % 16 == 0);
  griddep_launch_dependents();  // a following GEMM may start prefetching its weights
  griddep_wait();               // x and the outputs may belong to the preceding kernel
  auto load = [&](int64_t r, int sg, uint4 (&v)[4]) {
    const int kb = sg * 32 + lane;
    const bool real = r < rows && kb < nkb;
    const __nv_bfloat16* src = x + (real ? r : 0) * ld_x + static_cast<int64_t>(kb) * 32;
#pragma unroll
    for (int t = 0; t < 4; ++t) v[t] = real ? ld_stream_16(src + 8 * t) : make_uint4(0u, 0u, 0u, 0u);
  };
  uint4 cur[4], nxt[4];
  if (w < total) load(row, seg, cur);
  for (; w < total; w += wstride) {
    int64_t nrow = row + drow;
    int nseg = seg + dseg;
    if (nseg >= segs) {
      nseg -= segs;
      ++nrow;
    }
    if (w + wstride < total) load(nrow, nseg, nxt);
    const int kb = seg * 32 + lane;
    const bool real = row < rows && kb < nkb;
    const int e = real ? mx_exponent(bf16x32_absmax(cur)) : 0;
    if (real) {
      const float inv = mx_inv_scale(e);  // exact: power-of-two scaling
      uint2 c[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float f[8];
        bf16x8_to_f32(cur[t], f);
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] *= inv;
        c[t] = f32x8_to_e4m3(f);
      }
      uint8_t* dst = q + row * ld_q + static_cast<int64_t>(kb) * 32;
      if (q16) {
        reinterpret_cast<uint4*>(dst)[0] = make_uint4(c[0].x, c[0].y, c[1].x, c[1].y);
        reinterpret_cast<uint4*>(dst)[1] = make_uint4(c[2].x, c[2].y, c[3].x, c[3].y);
      } else {
#pragma unroll
        for (int t = 0; t < 4; ++t) reinterpret_cast<uint2*>(dst)[t] = c[t];
      }
    }
    // scale word of blocks kb..kb+3 (lanes L..L+3, L % 4 == 0)
    const uint32_t e1 = __shfl_down_sync(0xFFFFFFFFu, static_cast<uint32_t>(e), 1);
    const uint32_t e2 = __shfl_down_sync(0xFFFFFFFFu, static_cast<uint32_t>(e), 2);
    const uint32_t e3 = __shfl_down_sync(0xFFFFFFFFu, static_cast<uint32_t>(e), 3);
    if ((lane & 3) == 0 && kb < nkb4) {
      const int64_t off = k8x4 ? (static_cast<int64_t>(kb / 4) * rows_pad + row) * 4
                               : ((row / 128) * n_kc + kb / 4) * 512 + (row % 32) * 16 + ((row % 128) / 32) * 4;
      *reinterpret_cast<uint32_t*>(sf + off) = static_cast<uint32_t>(e) | (e1 << 8) | (e2 << 16) | (e3 << 24);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) cur[t] = nxt[t];
    row = nrow;
    seg = nseg;
  }
}

// Activations of at most 128 rows (one row tile; the launcher uses it for
// decode activations of up to 32 rows with a long K): one warp per (scale
// line L, segment of 32 K blocks).  Line L of a 512-byte
// chunk holds the words of rows L, L + 32, L + 64 and L + 96, so the warp
// quantizes those of its rows that exist -- lane l owns block 32 seg + l of
// each, with every row's four loads in flight at once -- and writes the whole
// 16-byte line (zero words for rows past the last).  32 x segments warps
// instead of 128 x segments, none of them for padding rows only, and the same
// codes, exponents and padding bytes as quant_mx_kernel.
__global__ void __launch_bounds__(kQ2Threads) quant_mx_lines_kernel(const __nv_bfloat16* __restrict__ x, int rows,
                                                                    int64_t k, int64_t ld_x, uint8_t* __restrict__ q,
                                                                    int64_t ld_q, uint8_t* __restrict__ sf, int n_kc) {
  const int lane = threadIdx.x & 31;
  const int nkb = static_cast<int>(k / 32);
  const int nkb4 = n_kc * 4;
  const int segs = (nkb4 + 31) / 32;
  const int task = blockIdx.x * (kQ2Threads / 32) + (threadIdx.x >> 5);
  const int L = task % 32, seg = task / 32;
  const bool q16 = (reinterpret_cast<uintptr_t>(q) % 16 == 0) && (ld_q % 16 == 0);
  griddep_launch_dependents();  // a following GEMM may start prefetching its weights
  griddep_wait();               // x and the outputs may belong to the preceding kernel
  if (seg >= segs) return;
  const int kb = seg * 32 + lane;
  uint4 v[4][4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int row = L + 32 * g;
    const bool real = row < rows && kb < nkb;
    const __nv_bfloat16* src = x + static_cast<int64_t>(real ? row : 0) * ld_x + static_cast<int64_t>(kb) * 32;
#pragma unroll
    for (int t = 0; t < 4; ++t) v[g][t] = real ? ld_stream_16(src + 8 * t) : make_uint4(0u, 0u, 0u, 0u);
  }
  uint32_t word[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int row = L + 32 * g;
    const bool real = row < rows && kb < nkb;
    const int e = real ? mx_exponent(bf16x32_absmax(v[g])) : 0;
    if (real) {
      const float inv = mx_inv_scale(e);  // exact: power-of-two scaling
      uint2 c[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float f[8];
        bf16x8_to_f32(v[g][t], f);
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] *= inv;
        c[t] = f32x8_to_e4m3(f);
      }
      uint8_t* dst = q + static_cast<int64_t>(row) * ld_q + static_cast<int64_t>(kb) * 32;
      if (q16) {
        reinterpret_cast<uint4*>(dst)[0] = make_uint4(c[0].x, c[0].y, c[1].x, c[1].y);
        reinterpret_cast<uint4*>(dst)[1] = make_uint4(c[2].x, c[2].y, c[3].x, c[3].y);
      } else {
#pragma unroll
        for (int t = 0; t < 4; ++t) reinterpret_cast<uint2*>(dst)[t] = c[t];
      }
    }
    // the word of blocks kb..kb+3 of this row (lanes L..L+3, L % 4 == 0)
    const uint32_t e1 = __shfl_down_sync(0xFFFFFFFFu, static_cast<uint32_t>(e), 1);
    const uint32_t e2 = __shfl_down_sync(0xFFFFFFFFu, static_cast<uint32_t>(e), 2);
    const uint32_t e3 = __shfl_down_sync(0xFFFFFFFFu, static_cast<uint32_t>(e), 3);
    word[g] = static_cast<uint32_t>(e) | (e1 << 8) | (e2 << 16) | (e3 << 24);
  }
  if ((lane & 3) == 0 && kb < nkb4)
    *reinterpret_cast<uint4*>(sf + static_cast<int64_t>(kb / 4) * 512 + L * 16) =
        make_uint4(word[0], word[1], word[2], word[3]);
}

}  // namespace fp8mm
