// gemm.cuh -- persistent, warp-specialised tcgen05 GEMM for both scale modes.
//
//   mode 1: C = diag(scale_a) (A x B^T) diag(scale_b)  (page "从 DeepGEMM 到
//           vLLM", listing 1: fp8_gemm with per-token scale_a[m] and
//           per-channel scale_b[n]); kind::f8f6f4, scales applied in the
//           epilogue in fp32.
//   mode 2: C = sum over 32-wide K blocks of 2^(ea-127) 2^(eb-127) A_b B_b^T
//           (page "[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합", section 2,
//           mm_mxfp8); kind::mxf8f6f4.block_scale, scales consumed by the MMA
//           from TMEM.
//
// One CTA per SM loops over 128 x kBN output tiles, kBN = 256 or 128 (grouped
// raster: kGroupM M-tiles share each B tile while it is hot in L2).  The
// 128-wide tiles, with two accumulators also in mode 2, serve shapes whose
// 256-wide tiles would leave most SMs idle.  Warp roles:
//   warp 0      TMA producer: A/B tiles (128-byte swizzle) and, in mode 2,
//               the 512-byte scale chunks, into a kStages-deep ring.
//   warp 1      allocates TMEM; one elected lane of the converged warp issues
//               tcgen05.mma (and tcgen05.cp of the scale chunks) per 128-byte K
//               slab, commits to free the slab.
//   warps 2..9  epilogue: each drains half a tile row-block of the fp32
//               accumulator into registers (tcgen05.ld, one wait), frees the
//               accumulator, then scales, converts to bf16 RNE and stores
//               (or, with kOut8 in mode 1, E4M3 codes of C / scale_out: the
//               FP8 output of listing 1's C_fp8 for the next layer).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "quant.cuh"

namespace fp8mm {

constexpr int kBM = 128;            // tile rows (A / M side of the MMA)
constexpr int kBK = 128;            // K elements (= bytes) per pipeline slab
constexpr int kMmaK = 32;           // K per tcgen05.mma for 8-bit operands
constexpr int kGemmThreads = 320;   // 10 warps: producer, MMA, 8 epilogue
constexpr int kGroupM = 16;

struct GemmArgs {
  int m, n, k;
  int num_k;                 // ceil(k / kBK)
  int tiles_m, tiles_n, num_tiles;
  __nv_bfloat16* c;
  int64_t ldc;
  uint8_t* c8;               // kOut8: E4M3 output (row stride ldc bytes)
  const float* s_out;        // kOut8: output scale (device scalar)
  const float* sa;           // mode 1
  const float* sb;
  const uint8_t* sfa;        // mode 2 (library scale layout)
  const uint8_t* sfb;
  int n_kc;                  // scale chunks per 128-row tile = ceil(k / 128)
  int sfb_row_tiles;         // ceil(n / 128): 128-row tiles present in sfb
  uint64_t timeout_ns;
  int group_m;               // paired-SM kernel: 256-row tiles per raster group
  int split;                 // paired-SM kernel: K parts per split tile (1 = whole K, no partials)
  int dp_tiles;              // paired-SM kernel: tiles [0, dp_tiles) run whole, the rest in split parts
  float* partials;           // split > 1: fp32 partials [(num_tiles - dp_tiles) * split][2][128 * 256]
  unsigned* tickets;         // split > 1: arrivals per (split tile, CTA rank), zero between calls
  int tma_c;                 // paired MX kernel: whole tiles' C goes out by TMA stores through shared memory
};

// Per-token / per-channel scaling of an fp32 accumulator, sa * sb * acc
// (page "从 DeepGEMM 到 vLLM", listing 1: scale_a[m] and scale_b[n]).  The
// scale product is rounded once and applied where it is a normal fp32; where
// it is not (a subnormal row or column scale, or sa * sb past the fp32 range)
// the accumulator is scaled by each in turn, so that neither a huge row scale
// meeting a tiny column scale overflows on the way nor a subnormal product
// loses its significand.
__device__ __forceinline__ float scale_acc(float acc, float sa, float sb) {
  const float sab = sa * sb;
  const float m = fabsf(sab);
  return (m >= 0x1p-126f && m <= 0x1.fffffep127f) ? acc * sab : (acc * sa) * sb;
}

// Epilogue store of one thread's 32 consecutive outputs v[0..31] of row `row`
// from column col0: bf16 round-to-nearest-even into p.c, or with kOut8 the
// E4M3 codes of v / s_out (quotient_sat, IEEE division when !fast) into p.c8.
// Full 32-column runs store 32 bytes at a time where the address is 32-byte
// aligned (bf16: each store fills a whole 32-byte sector), else 16 bytes at a
// time where it is 16-byte aligned; ragged or unaligned runs store element by
// element.
template <bool kOut8>
__device__ __forceinline__ void store_out32(const GemmArgs& p, int row, int col0, const float (&v)[32], float s_out,
                                            float r_out, bool fast) {
  if (row >= p.m || col0 >= p.n) return;
  if constexpr (kOut8) {
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float y[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) y[u] = fast ? quotient_sat(v[4 * j + u], s_out, r_out) : __fdiv_rn(v[4 * j + u], s_out);
      w[j] = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(y[0], y[1]), __NV_SATFINITE, __NV_E4M3)) |
             (static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(y[2], y[3]), __NV_SATFINITE, __NV_E4M3)) << 16);
    }
    uint8_t* dst = p.c8 + static_cast<int64_t>(row) * p.ldc + col0;
    if (col0 + 32 <= p.n && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < p.n) dst[j] = static_cast<uint8_t>(w[j >> 2] >> (8 * (j & 3)));
    }
  } else {
    uint32_t packed[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
      packed[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    __nv_bfloat16* dst = p.c + static_cast<int64_t>(row) * p.ldc + col0;
    if (col0 + 32 <= p.n && (reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
      st_global_v8(dst, packed[0], packed[1], packed[2], packed[3], packed[4], packed[5], packed[6], packed[7]);
      st_global_v8(dst + 16, packed[8], packed[9], packed[10], packed[11], packed[12], packed[13], packed[14],
                   packed[15]);
    } else if (col0 + 32 <= p.n && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        *reinterpret_cast<uint4*>(dst + q4 * 8) =
            make_uint4(packed[4 * q4], packed[4 * q4 + 1], packed[4 * q4 + 2], packed[4 * q4 + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (col0 + j < p.n) {
          const uint32_t w = packed[j >> 1];
          *reinterpret_cast<uint16_t*>(dst + j) = static_cast<uint16_t>((j & 1) ? (w >> 16) : (w & 0xFFFFu));
        }
      }
    }
  }
}

template <bool kMX, int kBN, int kStages, int kAccStages>
struct GemmCfg {
  static_assert(kBN % 128 == 0 && kBN <= 256, "B tile rows");
  static constexpr int kABytes = kBM * kBK;
  static constexpr int kBBytes = kBN * kBK;
  static constexpr int kSfaBytes = kMX ? 512 : 0;
  static constexpr int kSfbChunks = kBN / 128;
  static constexpr int kSfbBytes = kMX ? kSfbChunks * 512 : 0;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kABytes;
  static constexpr int kOffSfa = kOffB + kStages * kBBytes;
  static constexpr int kOffSfb = kOffSfa + kStages * kSfaBytes;
  static constexpr int kOffBar = kOffSfb + kStages * kSfbBytes;
  static constexpr int kNumBars = 2 * kStages + 2 * kAccStages + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack to align the base to 1024
  // TMEM columns: accumulators, then (mode 2) per-stage scale columns:
  // 4 for the A chunk, 4 per 128 rows of B.
  static constexpr int kSfColsPerStage = 4 + 4 * kSfbChunks;
  static constexpr int kSfCol0 = kAccStages * kBN;
  static constexpr int kColsUsed = kSfCol0 + (kMX ? kStages * kSfColsPerStage : 0);
  static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
  static_assert(kColsUsed <= 512, "TMEM budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ void tile_coords(int t, const GemmArgs& p, int& mb, int& nb) {
  const int per_group = kGroupM * p.tiles_n;
  const int g = t / per_group;
  const int first_m = g * kGroupM;
  const int gm = min(p.tiles_m - first_m, kGroupM);
  const int r = t - g * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

template <bool kMX, int kBN, int kStages, int kAccStages, bool kOut8 = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tiled_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const GemmArgs p) {
  using Cfg = GemmCfg<kMX, kBN, kStages, kAccStages>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + kAccStages;
  uint64_t* drain = acc_empty + kAccStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Launched with programmatic stream serialisation: the set-up below may
  // overlap the preceding kernel; the producer and the epilogue wait for it
  // before their first global access.
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kAccStages; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    // The whole warp runs the loop; one elected lane issues (see elect_one_sync).
    griddep_wait();  // A, B and their scales may be written by the preceding kernel
    {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        int sfb_chunks = 0;
        if constexpr (kMX) sfb_chunks = min(Cfg::kSfbChunks, p.sfb_row_tiles - nb * Cfg::kSfbChunks);
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!warp_wait(&empty[stage], phase ^ 1u, p.timeout_ns, abort_flag, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          if (elect_one_sync()) {
            uint32_t bytes = Cfg::kABytes + Cfg::kBBytes;
            if constexpr (kMX) bytes += 512u + 512u * sfb_chunks;
            mbar_arrive_expect_tx(&full[stage], bytes);
            tma_load_2d(smem + Cfg::kOffA + stage * Cfg::kABytes, &tmA, &full[stage], kb * kBK, mb * kBM);
            tma_load_2d(smem + Cfg::kOffB + stage * Cfg::kBBytes, &tmB, &full[stage], kb * kBK, nb * kBN);
            if constexpr (kMX) {
              bulk_load(smem + Cfg::kOffSfa + stage * 512, p.sfa + (static_cast<int64_t>(mb) * p.n_kc + kb) * 512,
                        512u, &full[stage]);
              for (int i = 0; i < sfb_chunks; ++i)
                bulk_load(smem + Cfg::kOffSfb + stage * Cfg::kSfbBytes + i * 512,
                          p.sfb + (static_cast<int64_t>(nb * Cfg::kSfbChunks + i) * p.n_kc + kb) * 512, 512u,
                          &full[stage]);
            }
          }
          __syncwarp();
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Let every copy the warp started land before the CTA can exit.
      for (int s = 0; s < kStages; ++s)
        if (issued_mask & (1u << s))
          mbar_wait(&full[s], (issued_parity >> s) & 1u, p.timeout_ns, nullptr, kSiteProducerDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    // The whole warp runs the loop; one elected lane issues (see elect_one_sync).
    {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
        if (!warp_wait(&acc_empty[acc], acc_phase ^ 1u, p.timeout_ns, abort_flag, kSiteMmaAccEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        for (int kb = 0; kb < p.num_k; ++kb) {
          if (!warp_wait(&full[stage], phase, p.timeout_ns, abort_flag, kSiteMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one_sync()) {
            const uint64_t adesc = sw128_kmajor_desc(smem_u32(smem + Cfg::kOffA + stage * Cfg::kABytes));
            const uint64_t bdesc = sw128_kmajor_desc(smem_u32(smem + Cfg::kOffB + stage * Cfg::kBBytes));
            if constexpr (kMX) {
              const uint32_t sfa_t = tmem_base + static_cast<uint32_t>(Cfg::kSfCol0 + stage * Cfg::kSfColsPerStage);
              const uint32_t sfb_t = sfa_t + 4u;
              tmem_cp_32x128b_warpx4(sfa_t, sf_chunk_desc(smem_u32(smem + Cfg::kOffSfa + stage * 512)));
#pragma unroll
              for (int i = 0; i < Cfg::kSfbChunks; ++i)
                tmem_cp_32x128b_warpx4(
                    sfb_t + 4u * i, sf_chunk_desc(smem_u32(smem + Cfg::kOffSfb + stage * Cfg::kSfbBytes + i * 512)));
#pragma unroll
              for (int kk = 0; kk < kBK / kMmaK; ++kk)
                mma_mxf8f6f4(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc_mxf8f6f4(kBM, kBN, kk, kk), sfa_t,
                             sfb_t, (kb | kk) != 0);
            } else {
#pragma unroll
              for (int kk = 0; kk < kBK / kMmaK; ++kk)
                mma_f8f6f4(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc_f8f6f4(kBM, kBN), (kb | kk) != 0);
            }
            tc_commit(&empty[stage]);
          }
          __syncwarp();
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (elect_one_sync()) tc_commit(&acc_full[acc]);
        __syncwarp();
        if (++acc == kAccStages) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // Every MMA / copy the warp issued must finish before TMEM is freed.
      if (elect_one_sync()) tc_commit(drain);
      __syncwarp();
      mbar_wait(drain, 0, p.timeout_ns, nullptr, kSiteDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ epilogue
    // Eight warps: warp w reads TMEM sub-partition (w % 4), i.e. tile rows
    // 32*(w%4) .. +31, and one half of the tile's columns.  Each thread pulls
    // its kBN/2 accumulator values into registers with kBN/64 loads and a
    // single wait, then releases the accumulator at once, so the next tile's
    // MMAs overlap the scaling, conversion and stores below.
    griddep_wait();  // C and the scales may belong to the preceding kernel
    const int sp = warp & 3;
    const int col_half = (warp - 2) >> 2;
    constexpr int kHalf = kBN / 2;
    constexpr int kChunks = kHalf / 32;
    float s_out = 1.f, r_out = 1.f;
    bool out_fast = true;
    if constexpr (kOut8) {
      s_out = __ldg(p.s_out);
      r_out = __frcp_rn(s_out);
      out_fast = quotient_fast_ok(s_out);
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      if (!mbar_wait(&acc_full[acc], acc_phase, p.timeout_ns, abort_flag, kSiteEpiAccFull)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sp * 32) << 16) +
                             static_cast<uint32_t>(acc * kBN + col_half * kHalf);
      uint32_t r[kChunks][32];
#pragma unroll
      for (int ch = 0; ch < kChunks; ++ch) tmem_ld_32x32b_x32(t_row + ch * 32, r[ch]);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int ch = 0; ch < kChunks; ++ch) asm volatile("" : FP8MM_RW32(r[ch]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == kAccStages) {
        acc = 0;
        acc_phase ^= 1u;
      }

      const int row = mb * kBM + sp * 32 + lane;
      float s_row = 1.f;
      if constexpr (!kMX) s_row = (row < p.m) ? __ldg(p.sa + row) : 0.f;
#pragma unroll
      for (int ch = 0; ch < kChunks; ++ch) {
        const int col0 = nb * kBN + col_half * kHalf + ch * 32;
        float sbv = 1.f;
        if constexpr (!kMX) sbv = (col0 + lane < p.n) ? __ldg(p.sb + col0 + lane) : 0.f;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] = __uint_as_float(r[ch][j]);
          if constexpr (!kMX) v[j] = scale_acc(v[j], s_row, __shfl_sync(0xFFFFFFFFu, sbv, j));
        }
        store_out32<kOut8>(p, row, col0, v, s_out, r_out, out_fast);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace fp8mm
