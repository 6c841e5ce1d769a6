// decode.cuh -- small-M (decode) MXFP8 GEMM: C[m, n] for m <= 64 tokens.
//
// The arithmetic is the block-scaled GEMM of page "[sglang] FlashInfer v0.6.7
// MXFP8 Gemm 통합", section 2, with the operand roles swapped: the weight B
// ([n, k], pre-quantized with its scales) fills the MMA's 128-row M side and
// the m tokens the N side (padded to kNM = 16..64), so D = B_tile x A^T lands
// in TMEM as 128 weight rows x kNM tokens.  At these sizes the call is bound
// by streaming the weight bytes from HBM, so the K range of the n/128 weight
// tiles is split stream-K style over up to two CTAs per SM: CTA b owns units
// [b*U/G, (b+1)*U/G) of the U = n_tiles * num_k (tile, 128-wide K slab)
// units.  A tile covered by one CTA is written directly; otherwise each
// contributor stores its fp32 partial in the workspace, bumps the tile's
// arrival counter, and the last to arrive sums the partials in CTA order
// (a fixed order, so results do not depend on timing), writes bf16 and
// resets the counter.  No CTA ever waits for another.
//
// With kCR (cluster reduction) the CTA count is tile-aligned: s = G / n_tiles
// CTAs per weight tile (s need not divide the tile's K slabs: CTA b = t*s + r
// owns slabs [floor(r*num_k/s), floor((r+1)*num_k/s)) of tile t), so CTA b
// runs the one segment b % s of tile b / s, and the s contributors of a tile
// are launched as one thread-block cluster.  Each writes its fp32 partial into its own
// (idle) weight ring, signals every peer's mbarrier, and then sums the slice
// of weight rows [r*128/s, (r+1)*128/s) that its rank r owns over all s
// partials, read through distributed shared memory in rank order (the same
// order as the workspace reduction, so the two give identical bits).  No
// workspace and no global round trip; the cluster meets once more before
// exit so that no CTA leaves while a peer may still read its shared memory.
//
// With kSF8 the activation's scales come in the small-M ("8x4") layout of
// mxfp8_quantize_8x4: per 128-wide K slab one 32-bit word per token row
// (rows padded to 8), rows_pad8 * 4 contiguous bytes, instead of the 512-byte
// chunk of 128 rows.  One more warp reads each slab's words (L2-resident) and
// writes them into the stage's scale image in the chunk form tcgen05.cp
// takes (row r at byte (r % 32) * 16 + (r / 32) * 4), then arrives on the
// stage's full barrier next to the TMA bytes.
//
// With kQX (m <= 8) the activation arrives as bf16 and is quantized inside
// the kernel (the per-call activation quantization of page "[sglang]
// FlashInfer v0.6.7 MXFP8 Gemm 통합", section 2, fused into the GEMM): two
// more warps take the CTA's K slabs in turn (warp q the slabs q, q+2, ...).
// Each reads its slab of the activation (m rows x 128, zero past k) straight
// from global memory -- it is small and shared by all CTAs, so it stays in L2
// -- holding the next slab's loads in registers while it quantizes the
// current one, one 32-element block per lane, with the 1x32 UE8M0 rule of
// mxfp8_quantize (the same exponent and conversion functions, and the exact
// block maximum, so codes and exponents are identical).  It writes the E4M3 tile
// in the 128-byte-swizzled K-major layout the MMA reads plus the exponents as
// the stage's scale chunk, and arrives on the stage's full barrier next to
// the weight bytes.  The tile rows m..kNM-1 are zeroed once and never
// written; K blocks past k quantize to zero with exponent 127 and meet zero
// weights, so the output equals that of mxfp8_quantize followed by the
// unfused kernel with the same CTA count.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "quant.cuh"

namespace fp8mm {

struct DecodeArgs {
  int m, n, k;
  int num_k;          // ceil(k / 128)
  int n_tiles;        // ceil(n / 128)
  int64_t units;      // n_tiles * num_k
  int ctas;           // G
  __nv_bfloat16* c;
  int64_t ldc;
  const uint8_t* sfw;  // scales of the weight b (rows = n)
  const uint8_t* sfx;  // scales of the activation a (rows = m)
  int n_kc;            // ceil(k / 128)
  float* partials;     // [2 * G][kNM][128] fp32
  unsigned* tickets;   // [n_tiles], zero between calls
  uint64_t timeout_ns;
  int prefetch_w;      // weights may be read before the preceding kernel ends
  int l2_ahead;        // slabs past the staged ones whose weights are prefetched into L2 at the start
  const __nv_bfloat16* x;  // kQX: bf16 activation [m, k]
  int64_t ldx;             // kQX: its row stride in elements
  int cluster_s;           // kCR: CTAs per weight tile (= the cluster size)
};

template <int kNM, int kStages, bool kQX = false, bool kSF8 = false>
struct DecodeCfg {
  static_assert(kNM % 16 == 0 && kNM >= 16 && kNM <= 64, "token tile");
  static_assert(!(kQX && kSF8), "the in-kernel quantizer writes the scale image itself");
  // warps: producer, MMA, four epilogue warps (+ two activation-quantizer
  // warps, or one warp that lays out 8x4 activation scales)
  static constexpr int kQuantWarps = kQX ? 2 : (kSF8 ? 1 : 0);
  static constexpr int kThreads = 192 + 32 * kQuantWarps;
  static constexpr int kQuantWarp0 = 6;
  // Shared memory and registers within half an SM, so two CTAs share an SM
  // and the next kernel on the stream (launched early, programmatically) can
  // hold a CTA on each SM and start streaming while this one finishes.  (The
  // 8x4-scale variant with 48/64-token tiles keeps one per SM: its extra warp
  // would not fit the registers.)
  static constexpr int kMinBlocksPerSm = (kNM <= 32 || !kSF8) ? 2 : 1;
  static constexpr int kWBytes = 128 * 128;
  static constexpr int kXBytes = kNM * 128;
  static_assert(!kQX || kNM == 16, "activation quantized in the kernel for m <= 8 (16-token tile)");
  static constexpr int kOffW = 0;
  static constexpr int kOffX = kOffW + kStages * kWBytes;
  static constexpr int kOffSfw = kOffX + kStages * kXBytes;
  static constexpr int kOffSfx = kOffSfw + kStages * 512;
  static constexpr int kOffBar = kOffSfx + kStages * 512;
  // full, empty per stage; acc_full, acc_empty x2; drain; epi_sync; red_ready (kCR)
  static constexpr int kNumBars = 2 * kStages + 2 * 2 + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static constexpr int kSfCol0 = 2 * kNM;
  static constexpr int kColsUsed = kSfCol0 + 8 * kStages;
  static constexpr int kTmemCols = kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128 : kColsUsed <= 256 ? 256 : 512;
  static_assert(kSmemBytes * kMinBlocksPerSm + 1024 * (kMinBlocksPerSm - 1) <= 232448, "shared memory budget");
  // kCR: a CTA's fp32 partial tile [kNM][128] lives in its weight ring
  static_assert(kNM * 128 * 4 <= kStages * kWBytes, "partial tile fits the weight ring");
};

__device__ __forceinline__ int64_t dec_unit_start(int b, const DecodeArgs& p) {
  return static_cast<int64_t>(b) * p.units / p.ctas;
}
// CTA that owns unit u: the largest b with floor(b*U/G) <= u.
__device__ __forceinline__ int dec_owner(int64_t u, const DecodeArgs& p) {
  return static_cast<int>(((u + 1) * p.ctas - 1) / p.units);
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void regs_fence_16(uint32_t* r) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]));
}

__device__ __forceinline__ float4 ld_shared_cluster_v4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}

// Cluster reduction of split tile t (kCR): the CTA of rank `rank` sums weight
// rows [4 q0, 4 q1) -- its share of the tile's 32 row quads -- over the S
// partials red[token][row] of the cluster's CTAs, in rank order, and writes
// the m tokens' bf16 outputs.  tid is 0..127 (the four epilogue warps).  All
// of a thread's distributed-shared-memory loads (ITEMS x S 16-byte vectors)
// are issued before the first sum, so the reduction costs about one remote
// round trip.  S = 3 stands for every split this kernel is not specialised
// for (the loop bounds then use the runtime count).
template <int S, int kNM>
__device__ __forceinline__ void cluster_reduce_slice(const float* red, int rank, int t, int tid, const DecodeArgs& p) {
  const int s = (S == 3) ? p.cluster_s : S;
  constexpr int kMaxQuads = (S == 3) ? 11 : (32 + S - 1) / S;   // S == 3: any s in 3..6
  constexpr int kItems = (kMaxQuads * kNM + 127) / 128;
  constexpr int kSrc = (S == 3) ? 6 : S;
  // specialised splits hold every load of the thread at once (<= 84 floats);
  // the generic one item at a time
  constexpr int kBatch = (S == 3) ? 1 : kItems;
  const int q0 = rank * 32 / s, nq = (rank + 1) * 32 / s - q0;
  const int total = nq * p.m;
  const uint32_t base = smem_u32(red);
#pragma unroll
  for (int it0 = 0; it0 < kItems; it0 += kBatch) {
    float4 v[kBatch][kSrc];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int idx = tid + (it0 + b) * 128;
      const int j = idx / nq;
      const uint32_t a = base + static_cast<uint32_t>((j * 128 + (q0 + idx - j * nq) * 4) * 4);
#pragma unroll
      for (int q = 0; q < kSrc; ++q)
        v[b][q] = (idx < total && q < s) ? ld_shared_cluster_v4(mapa_shared(a, static_cast<uint32_t>(q)))
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int idx = tid + (it0 + b) * 128;
      if (idx >= total) continue;
      const int j = idx / nq;
      const int quad = q0 + (idx - j * nq);
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < kSrc; ++q) {
        if (q >= s) break;
        sum.x += v[b][q].x;
        sum.y += v[b][q].y;
        sum.z += v[b][q].z;
        sum.w += v[b][q].w;
      }
      const float o[4] = {sum.x, sum.y, sum.z, sum.w};
      const int n0 = t * 128 + quad * 4;
      __nv_bfloat16* dst = p.c + static_cast<int64_t>(j) * p.ldc + n0;
      if (n0 + 4 <= p.n && (reinterpret_cast<uintptr_t>(dst) & 7u) == 0) {
        // four outputs in one 8-byte store (a warp writes 256 contiguous bytes)
        const __nv_bfloat162 lo = __floats2bfloat162_rn(o[0], o[1]);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(o[2], o[3]);
        *reinterpret_cast<uint2*>(dst) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (n0 + e < p.n) dst[e] = __float2bfloat16_rn(o[e]);
      }
    }
  }
}

// tmX: the quantized activation (E4M3 [m, k], 128-byte swizzle, box 128 x
// kNM); unused with kQX (the activation comes as p.x).
template <int kNM, int kStages, bool kQX, bool kCR = false, bool kSF8 = false>
__global__ void __launch_bounds__(DecodeCfg<kNM, kStages, kQX, kSF8>::kThreads,
                                  DecodeCfg<kNM, kStages, kQX, kSF8>::kMinBlocksPerSm)
    gemm_small_m_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                        const DecodeArgs p) {
  using Cfg = DecodeCfg<kNM, kStages, kQX, kSF8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* epi_sync = drain + 1;  // the four epilogue warps meet here (bounded)
  uint64_t* red_ready = epi_sync + 1;  // kCR: every peer's four epilogue warps have written their partial
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int64_t u_begin = dec_unit_start(b, p);
  const int64_t u_end = dec_unit_start(b + 1, p);
  const int first_tile = static_cast<int>(u_begin / p.num_k);
  griddep_launch_dependents();  // a following kernel launched the same way may start its prologue

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], (kQX || kSF8) ? 2 : 1);  // + the quantizer (kQX) or scale (kSF8) warp
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(drain, 1);
    mbar_init(epi_sync, 4);
    if (kCR) mbar_init(red_ready, 4 * p.cluster_s);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    if (!kQX) prefetch_tmap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  if constexpr (kCR)
    cluster_sync_all();  // every peer's red_ready is initialised before anyone can arrive on it
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    // The CTA's slabs in order: slab i is unit u_begin + i = (tile t, K slab
    // kb).  When the caller vouches that the weights do not depend on the
    // preceding kernel (prefetch_w), the weights of the first stages are
    // requested before griddepcontrol.wait; the activation always after it.
    // The whole warp runs the loops; one elected lane issues (see
    // elect_one_sync).
    {
      if (!p.prefetch_w) griddep_wait();
      const int64_t nslabs = u_end - u_begin;
      const int npre = static_cast<int>(nslabs < kStages ? nslabs : kStages);
      const int t0 = static_cast<int>(u_begin / p.num_k);
      const int kb0 = static_cast<int>(u_begin % p.num_k);
      constexpr uint32_t kTx = kQX    ? Cfg::kWBytes + 512u
                               : kSF8 ? Cfg::kWBytes + Cfg::kXBytes + 512u
                                      : Cfg::kWBytes + Cfg::kXBytes + 1024u;
      int t = t0, kb = kb0;
      for (int i = 0; i < npre; ++i) {  // fresh stages: nothing to wait for
        if (elect_one_sync()) {
          mbar_arrive_expect_tx(&full[i], kTx);
          tma_load_2d(smem + Cfg::kOffW + i * Cfg::kWBytes, &tmW, &full[i], kb * 128, t * 128);
          bulk_load(smem + Cfg::kOffSfw + i * 512, p.sfw + (static_cast<int64_t>(t) * p.n_kc + kb) * 512, 512u,
                    &full[i]);
        }
        __syncwarp();
        if (++kb == p.num_k) {
          kb = 0;
          ++t;
        }
      }
      // The weights of the next l2_ahead slabs go to L2 now, so that HBM keeps
      // streaming while the stages wait for the activation (and, under
      // programmatic launch, for the preceding kernel).
      const int64_t l2_end = npre + p.l2_ahead < nslabs ? npre + p.l2_ahead : nslabs;
      for (int64_t i = npre; i < l2_end; ++i) {
        if (elect_one_sync()) {
          tma_prefetch_l2_2d(&tmW, kb * 128, t * 128);
          bulk_prefetch_l2(p.sfw + (static_cast<int64_t>(t) * p.n_kc + kb) * 512, 512u);
        }
        __syncwarp();
        if (++kb == p.num_k) {
          kb = 0;
          ++t;
        }
      }
      griddep_wait();
      t = t0;
      kb = kb0;
      for (int i = 0; i < npre; ++i) {
        if (!kQX) {
          if (elect_one_sync()) {
            tma_load_2d(smem + Cfg::kOffX + i * Cfg::kXBytes, &tmX, &full[i], kb * 128, 0);
            if (!kSF8)
              bulk_load(smem + Cfg::kOffSfx + i * 512, p.sfx + static_cast<int64_t>(kb) * 512, 512u, &full[i]);
          }
          __syncwarp();
        }
        if (++kb == p.num_k) {
          kb = 0;
          ++t;
        }
      }
      int stage = npre % kStages;
      uint32_t phase = (npre == kStages) ? 1u : 0u;
      uint32_t issued_mask = (npre == kStages) ? ((1u << kStages) - 1u) : ((1u << npre) - 1u);
      uint32_t issued_parity = 0;
      for (int64_t i = npre; i < nslabs; ++i) {
        if (!warp_wait(&empty[stage], phase ^ 1u, p.timeout_ns, abort_flag, kSiteProducerEmpty)) break;
        if (elect_one_sync()) {
          mbar_arrive_expect_tx(&full[stage], kTx);
          tma_load_2d(smem + Cfg::kOffW + stage * Cfg::kWBytes, &tmW, &full[stage], kb * 128, t * 128);
          bulk_load(smem + Cfg::kOffSfw + stage * 512, p.sfw + (static_cast<int64_t>(t) * p.n_kc + kb) * 512, 512u,
                    &full[stage]);
          if (!kQX) {
            tma_load_2d(smem + Cfg::kOffX + stage * Cfg::kXBytes, &tmX, &full[stage], kb * 128, 0);
            if (!kSF8)
              bulk_load(smem + Cfg::kOffSfx + stage * 512, p.sfx + static_cast<int64_t>(kb) * 512, 512u,
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
        if (++kb == p.num_k) {
          kb = 0;
          ++t;
        }
      }
      for (int s = 0; s < kStages; ++s)
        if (issued_mask & (1u << s))
          mbar_wait(&full[s], (issued_parity >> s) & 1u, p.timeout_ns, nullptr, kSiteProducerDrain);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer
    // The whole warp runs the loop; one elected lane issues (see elect_one_sync).
    {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t u = u_begin; ok && u < u_end;) {
        const int kb0 = static_cast<int>(u % p.num_k);
        const int kb1 = static_cast<int>(kb0 + (u_end - u) < p.num_k ? kb0 + (u_end - u) : p.num_k);
        if (!warp_wait(&acc_empty[acc], acc_phase ^ 1u, p.timeout_ns, abort_flag, kSiteMmaAccEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kNM);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!warp_wait(&full[stage], phase, p.timeout_ns, abort_flag, kSiteMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one_sync()) {
            const uint32_t sfw_t = tmem_base + static_cast<uint32_t>(Cfg::kSfCol0 + stage * 8);
            const uint32_t sfx_t = sfw_t + 4u;
            tmem_cp_32x128b_warpx4(sfw_t, sf_chunk_desc(smem_u32(smem + Cfg::kOffSfw + stage * 512)));
            tmem_cp_32x128b_warpx4(sfx_t, sf_chunk_desc(smem_u32(smem + Cfg::kOffSfx + stage * 512)));
            const uint64_t wdesc = sw128_kmajor_desc(smem_u32(smem + Cfg::kOffW + stage * Cfg::kWBytes));
            const uint64_t xdesc = sw128_kmajor_desc(smem_u32(smem + Cfg::kOffX + stage * Cfg::kXBytes));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_mxf8f6f4(d_tmem, wdesc + 2u * kk, xdesc + 2u * kk, idesc_mxf8f6f4(128, kNM, kk, kk), sfw_t, sfx_t,
                           (kb != kb0) || (kk != 0));
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
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
        u += kb1 - kb0;
      }
      if (elect_one_sync()) tc_commit(drain);
      __syncwarp();
      mbar_wait(drain, 0, p.timeout_ns, nullptr, kSiteDrain);
    }
    __syncwarp();
  } else if (kCR && warp < Cfg::kQuantWarp0) {
    // ------------------------------------------------------ epilogue, cluster reduction
    griddep_wait();  // C may still be in use by the preceding kernel
    const int sp = warp & 3;
    const int nl = sp * 32 + lane;  // weight row inside the tile
    const int ns = p.cluster_s;
    const int rank = static_cast<int>(cluster_ctarank());
    bool ok = mbar_wait(&acc_full[0], 0, p.timeout_ns, abort_flag, kSiteEpiAccFull);
    uint32_t r[kNM];
#pragma unroll
    for (int j = 0; j < kNM; ++j) r[j] = 0u;
    if (ok) {
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sp * 32) << 16);
#pragma unroll
      for (int ch = 0; ch < kNM / 16; ++ch) tmem_ld_32x32b_x16(t_row + ch * 16, r + ch * 16);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int ch = 0; ch < kNM / 16; ++ch) regs_fence_16(r + ch * 16);
    }
    // The weight ring is idle: every TMA write into it was consumed by an MMA
    // that completed before acc_full.  Partial [token j][row] as fp32.
    float* red = reinterpret_cast<float*>(smem + Cfg::kOffW);
    fence_proxy_async_smem();
#pragma unroll
    for (int j = 0; j < kNM; ++j) red[j * 128 + nl] = __uint_as_float(r[j]);
    // The warp's stores are ordered before lane 0's release arrivals (the
    // warp barrier orders them; release is cumulative); each peer's acquiring
    // wait then sees them.  A CTA that failed above still arrives, so its
    // peers finish; the error word reports the call.
    __syncwarp();
    if (lane == 0)
      for (int q = 0; q < ns; ++q) mbar_arrive_cluster(mapa_shared(smem_u32(red_ready), static_cast<uint32_t>(q)));
    ok = mbar_wait_cluster(red_ready, 0, p.timeout_ns, abort_flag, kSiteClusterReduce) && ok;
    if (ok) {
      switch (ns) {
        case 2: cluster_reduce_slice<2, kNM>(red, rank, first_tile, threadIdx.x - 64, p); break;
        case 4: cluster_reduce_slice<4, kNM>(red, rank, first_tile, threadIdx.x - 64, p); break;
        case 7: cluster_reduce_slice<7, kNM>(red, rank, first_tile, threadIdx.x - 64, p); break;
        case 8: cluster_reduce_slice<8, kNM>(red, rank, first_tile, threadIdx.x - 64, p); break;
        default: cluster_reduce_slice<3, kNM>(red, rank, first_tile, threadIdx.x - 64, p); break;  // 3, 5, 6
      }
    }
  } else if (warp < Cfg::kQuantWarp0) {
    // ------------------------------------------------------ epilogue
    griddep_wait();  // the workspace and C may still be in use by the preceding kernel
    const int sp = warp & 3;
    const int nl = sp * 32 + lane;  // weight row inside the tile = output column
    int acc = 0;
    uint32_t acc_phase = 0, sync_phase = 0;
    // All four epilogue warps meet; false if the wait expired or the CTA aborted.
    auto epi_meet = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_sync);
      const bool ok = mbar_wait(epi_sync, sync_phase, p.timeout_ns, abort_flag, kSiteEpiSync);
      sync_phase ^= 1u;
      return ok;
    };
    for (int64_t u = u_begin; u < u_end;) {
      const int t = static_cast<int>(u / p.num_k);
      const int kb0 = static_cast<int>(u % p.num_k);
      const int kb1 = static_cast<int>(kb0 + (u_end - u) < p.num_k ? kb0 + (u_end - u) : p.num_k);
      u += kb1 - kb0;
      if (!mbar_wait(&acc_full[acc], acc_phase, p.timeout_ns, abort_flag, kSiteEpiAccFull)) break;
      tc_fence_after();
      uint32_t r[kNM];
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(sp * 32) << 16) + static_cast<uint32_t>(acc * kNM);
#pragma unroll
      for (int ch = 0; ch < kNM / 16; ++ch) tmem_ld_32x32b_x16(t_row + ch * 16, r + ch * 16);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
      for (int ch = 0; ch < kNM / 16; ++ch) regs_fence_16(r + ch * 16);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }

      const int n_col = t * 128 + nl;
      if (kb0 == 0 && kb1 == p.num_k) {
        if (n_col < p.n) {
#pragma unroll
          for (int j = 0; j < kNM; ++j)
            if (j < p.m) p.c[static_cast<int64_t>(j) * p.ldc + n_col] = __float2bfloat16_rn(__uint_as_float(r[j]));
        }
        continue;
      }
      // partial tile: publish, count, and let the last contributor reduce
      const int slot = 2 * b + (t == first_tile ? 0 : 1);
      float* mine = p.partials + static_cast<int64_t>(slot) * kNM * 128;
#pragma unroll
      for (int j = 0; j < kNM; ++j)
        if (j < p.m) mine[j * 128 + nl] = __uint_as_float(r[j]);
      // The four warps' partial stores are ordered before one thread's
      // acquire-release ticket increment at GPU scope (the barrier between
      // them is CTA-scope release/acquire and release is cumulative); the
      // last contributor's increment acquires every earlier contributor's
      // stores, and the barrier after it hands them to its other threads.
      if (!epi_meet()) break;
      const int b_first = dec_owner(static_cast<int64_t>(t) * p.num_k, p);
      const int b_last = dec_owner(static_cast<int64_t>(t + 1) * p.num_k - 1, p);
      if (threadIdx.x == 64) {
        unsigned prev;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(&p.tickets[t]) : "memory");
        *last_flag = (prev == static_cast<unsigned>(b_last - b_first)) ? 1 : 0;
      }
      if (!epi_meet()) break;
      if (*last_flag) {
        // Sum the contributors' partials in CTA order (fixed, so the result
        // does not depend on arrival order); kU contributors' loads are in
        // flight at a time.
        constexpr int kU = kNM <= 16 ? 4 : (kNM <= 32 ? 2 : 1);
        float sum[kNM];
#pragma unroll
        for (int j = 0; j < kNM; ++j) sum[j] = 0.f;
        for (int bb = b_first; bb <= b_last; bb += kU) {
          float v[kU][kNM];
#pragma unroll
          for (int q = 0; q < kU; ++q) {
            const int b2 = bb + q;
            const float* src = nullptr;
            if (b2 <= b_last) {
              const int first_b2 = static_cast<int>(dec_unit_start(b2, p) / p.num_k);
              src = p.partials + static_cast<int64_t>(2 * b2 + (t == first_b2 ? 0 : 1)) * kNM * 128;
            }
#pragma unroll
            for (int j = 0; j < kNM; ++j) v[q][j] = (src != nullptr && j < p.m) ? __ldcg(src + j * 128 + nl) : 0.f;
          }
#pragma unroll
          for (int q = 0; q < kU; ++q)
#pragma unroll
            for (int j = 0; j < kNM; ++j) sum[j] += v[q][j];
        }
        if (n_col < p.n) {
#pragma unroll
          for (int j = 0; j < kNM; ++j)
            if (j < p.m) p.c[static_cast<int64_t>(j) * p.ldc + n_col] = __float2bfloat16_rn(sum[j]);
        }
        if (threadIdx.x == 64) p.tickets[t] = 0u;
      }
    }
  } else if (kQX) {
    // ------------------------------------------------------ activation quantizer
    // Warp qw takes slabs qw, qw + Q, ... (Q quantizer warps).  Lane L owns the
    // 32-element K block b = L % 4 of row L/4 < m (m <= 8) of each slab: four
    // 16-byte loads, the block maximum, one exponent, and 32 E4M3 bytes = two
    // 16-byte chunks of the swizzled tile row.  The loads of the warp's next
    // two slabs are in flight while it quantizes the current one.
    constexpr int Q = Cfg::kQuantWarps;
    constexpr int kP = 1;
    const int qw = warp - Cfg::kQuantWarp0;
    const int b = lane & 3;
    const int rsub = lane >> 2;
    const int64_t nslabs = u_end - u_begin;
    // Tile rows m..kNM-1 (and their scale words, with the words of rows
    // kNM..127 that the MMA never reads) are zeroed once; the loop below
    // writes only rows < m.  Word (L, g) of a scale chunk holds row 32g + L.
    const int qt = threadIdx.x - Cfg::kQuantWarp0 * 32;
    for (int o = qt; o < kStages * (kNM - p.m) * 8; o += 32 * Q) {
      const int st = o / ((kNM - p.m) * 8), rem = o % ((kNM - p.m) * 8);
      reinterpret_cast<uint4*>(smem + Cfg::kOffX + st * Cfg::kXBytes + (p.m + rem / 8) * 128)[rem % 8] =
          make_uint4(0u, 0u, 0u, 0u);
    }
    for (int w = qt; w < kStages * 128; w += 32 * Q) {
      const int L = (w & 127) >> 2, g = w & 3;
      if (32 * g + L >= p.m) reinterpret_cast<uint32_t*>(smem + Cfg::kOffSfx)[(w >> 7) * 128 + L * 4 + g] = 0u;
    }
    // The zeroed rows are read by the tensor core: each thread fences its
    // stores to the async proxy, and the quantizer warps meet before any of
    // them arrives on a stage's full barrier.
    fence_proxy_async_smem();
    asm volatile("bar.sync 1, %0;" ::"n"(32 * Q) : "memory");
    griddep_wait();  // the activation may be written by the preceding kernel
    // this lane's block of slab i in each pass (zero past m rows and past k)
    auto load_slab = [&](int64_t i, uint4 (&v)[kP][4]) {
      const int64_t col = static_cast<int64_t>((u_begin + i) % p.num_k) * 128 + b * 32;
#pragma unroll
      for (int q = 0; q < kP; ++q) {
        const int r = rsub + 8 * q;
        const bool in = r < p.m && col < p.k;
        const __nv_bfloat16* src = p.x + static_cast<int64_t>(r) * p.ldx + col;
#pragma unroll
        for (int t = 0; t < 4; ++t) v[q][t] = in ? ld_stream_16(src + 8 * t) : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    uint4 cur[kP][4], nxt[kP][4], nxt2[kP][4];
    if (qw < nslabs) load_slab(qw, cur);
    if (qw + Q < nslabs) load_slab(qw + Q, nxt);
    bool ok = true;
    for (int64_t i = qw; i < nslabs; i += Q) {
      if (i + 2 * Q < nslabs) load_slab(i + 2 * Q, nxt2);
      const int stage = static_cast<int>(i % kStages);
      ok = ok && mbar_wait(&empty[stage], static_cast<uint32_t>(((i / kStages) & 1) ^ 1), p.timeout_ns, abort_flag,
                           kSiteQuantStage);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      uint8_t* xq = smem + Cfg::kOffX + stage * Cfg::kXBytes;
      uint8_t* sfx = smem + Cfg::kOffSfx + stage * 512;
#pragma unroll
      for (int q = 0; q < kP; ++q) {
        const int r = rsub + 8 * q;
        if (8 * q >= p.m) break;  // no row of this pass is real
        // block maximum of |x|: for finite bf16 the magnitude order is the
        // order of the sign-cleared bit patterns, so a 16-bit unsigned max
        uint32_t mx = 0;
#pragma unroll
        for (int t = 0; t < 4; ++t)
          mx = __vmaxu2(__vmaxu2(mx, cur[q][t].x & 0x7FFF7FFFu), __vmaxu2(cur[q][t].y & 0x7FFF7FFFu,
               __vmaxu2(cur[q][t].z & 0x7FFF7FFFu, cur[q][t].w & 0x7FFF7FFFu)));
        const float a = __uint_as_float(max(mx & 0xFFFFu, mx >> 16) << 16);
        const int e = mx_exponent(a);
        const float inv = mx_inv_scale(e);
        uint2 c[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          float f[8];
          bf16x8_to_f32(cur[q][t], f);
#pragma unroll
          for (int u = 0; u < 8; ++u) f[u] *= inv;
          c[t] = f32x8_to_e4m3(f);
        }
        if (r < p.m) {
          // bytes 32b..32b+31 of row r: chunks 2b and 2b+1, stored at chunk c ^ (r % 8)
          uint8_t* row = xq + r * 128;
          *reinterpret_cast<uint4*>(row + (((2 * b) ^ (r & 7)) << 4)) = make_uint4(c[0].x, c[0].y, c[1].x, c[1].y);
          *reinterpret_cast<uint4*>(row + (((2 * b + 1) ^ (r & 7)) << 4)) = make_uint4(c[2].x, c[2].y, c[3].x, c[3].y);
          sfx[(r & 31) * 16 + ((r & 127) >> 5) * 4 + b] = static_cast<uint8_t>(e);
        }
      }
      fence_proxy_async_smem();  // the tile and scales are read by the tensor core (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[stage]);
#pragma unroll
      for (int q = 0; q < kP; ++q)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          cur[q][t] = nxt[q][t];
          nxt[q][t] = nxt2[q][t];
        }
    }
  }

  if constexpr (kSF8) {
    if (warp == Cfg::kQuantWarp0) {
      // ---------------------------------------------------- 8x4 activation scales
      // Lane L owns token rows L and L + 32: its word of each slab goes to
      // the image at byte L * 16 (row L) and L * 16 + 4 (row L + 32).  Words
      // of rows past m are zero in the 8x4 layout up to rows_pad8, and zero
      // here beyond it; rows >= kNM are never read.  The next two slabs'
      // words are in flight while the current one is placed.
      constexpr int kW = kNM > 32 ? 2 : 1;
      const int rows8 = (p.m + 7) & ~7;
      const int64_t nslabs = u_end - u_begin;
      griddep_wait();  // the scales may be written by the preceding kernel
      auto load = [&](int64_t i, uint32_t (&w)[kW]) {
        const int kb = static_cast<int>((u_begin + i) % p.num_k);
        const uint32_t* src = reinterpret_cast<const uint32_t*>(p.sfx) + static_cast<int64_t>(kb) * rows8;
#pragma unroll
        for (int h = 0; h < kW; ++h) w[h] = (lane + 32 * h < rows8) ? __ldcg(src + lane + 32 * h) : 0u;
      };
      uint32_t cur[kW], nxt[kW], nxt2[kW];
      if (nslabs > 0) load(0, cur);
      if (nslabs > 1) load(1, nxt);
      bool ok = true;
      for (int64_t i = 0; i < nslabs; ++i) {
        if (i + 2 < nslabs) load(i + 2, nxt2);
        const int stage = static_cast<int>(i % kStages);
        ok = ok && mbar_wait(&empty[stage], static_cast<uint32_t>(((i / kStages) & 1) ^ 1), p.timeout_ns,
                             abort_flag, kSiteQuantStage);
        if (!__all_sync(0xFFFFFFFFu, ok)) break;
        uint32_t* img = reinterpret_cast<uint32_t*>(smem + Cfg::kOffSfx + stage * 512);
#pragma unroll
        for (int h = 0; h < kW; ++h) img[lane * 4 + h] = cur[h];
        fence_proxy_async_smem();  // the image is read by tcgen05.cp (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
#pragma unroll
        for (int h = 0; h < kW; ++h) {
          cur[h] = nxt[h];
          nxt[h] = nxt2[h];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (kCR) cluster_sync_all();  // no CTA leaves while a peer may still read its partial
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace fp8mm
