// gemm2.cuh -- paired-SM tcgen05 GEMM (cta_group::2) for both scale modes.
//
// Same arithmetic as gemm.cuh (page "从 DeepGEMM 到 vLLM", listing 1 for the
// per-token mode, with its bf16 or E4M3 output; page "[sglang] FlashInfer v0.6.7 MXFP8 Gemm 통합", section 2
// for the block-scaled mode), computed by 2-CTA clusters on 256 x 256 output
// tiles.  Each CTA of a pair loads its own 128-row half of the A tile and its
// own 128-row half of the B tile; nothing is multicast.  Those loads complete
// on the rank-0 CTA's barrier, whose MMA warp issues (from one elected lane)
// the cta_group::2 MMAs (M = 256, N = 256, K = 32) that read A and B from both
// CTAs' shared memory
// and accumulate 128 rows in each CTA's TMEM.  Per 128-byte K slab a CTA moves
// 32 KiB into shared memory for 128x256x128 MACs, two thirds of what the
// single-CTA 128x256 tile needs.
//
// Block scales (mode 2): each CTA loads its A scale chunk and both B scale
// chunks (every CTA needs all 256 B rows' scales in its own TMEM) with the
// same pair-completed TMA loads; the MMA warp copies them into the stage's
// TMEM columns right before that stage's MMAs, three 32x128b.warpx4 copies
// (A, B rows 0-127, B rows 128-255).  Issued from a converged warp the copies
// cost little (see elect_one_sync); from a lone lane each stalled the tensor
// pipe, and B's two chunks then went as four replicas each through one
// 128x256b copy.  Measured on B200 (8192 x 22016 x 8192, converged issue):
// plain chunks and 5 stages are 1.3 % faster than replicas and 6 stages.
// Moving the copies to other warps (tcgen05.st from four scale warps, or the
// copies issued by a second thread) measured no faster, and cluster-scope
// release arrivals from those warps made the kernel ~45 % slower.
//
// Warp roles per CTA: warp 0 TMA producer; warp 1 TMEM owner and, on rank 0,
// MMA issuer (the whole warp, one elected lane issuing); warps 2..17
// epilogue (four per TMEM sub-partition, 64 accumulator columns each,
// drained into registers with one wait so the accumulator is free again at
// once).
//
// Split K (split > 1): tiles [0, dp_tiles) are whole work units; each later
// tile is `split` units (tile, K part), part j covering K slabs
// [floor(j*num_k/split), floor((j+1)*num_k/split)).  Pairs take units in
// turn, so with dp_tiles a multiple of the pair count the split tiles form
// the last round: where the tiles fill less than one wave all are split
// (dp_tiles = 0), else only those of the last, partly filled wave.  Each CTA
// of a split unit stores its fp32 partial (its 128 rows x 256 columns) in the
// workspace, bumps the (tile, rank) arrival counter, and the last to arrive
// sums the parts in part order (fixed, so the result does not depend on
// timing), applies the scales, writes C and resets the counter.  No CTA waits
// for another.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "gemm.cuh"
#include "ptx.cuh"

namespace fp8mm {

constexpr int kPairGroupM = 8;     // 256-row tiles per raster group (doubled for B larger than 64 MiB)

template <bool kMX, int kStages, int kAccStages>
struct PairCfg {
  // Warps: producer, MMA, 16 epilogue warps.
  static constexpr int kEpiWarp0 = 2;
  static constexpr int kThreads = (kEpiWarp0 + 16) * 32;
  static constexpr int kABytes = 128 * kBK;          // this CTA's half of A
  static constexpr int kBBytes = 128 * kBK;          // this CTA's half of B
  static constexpr int kSfaBytes = kMX ? 512 : 0;    // this CTA's 128 A rows x 4 blocks
  static constexpr int kSfbBytes = kMX ? 1024 : 0;   // all 256 B rows x 4 blocks: two 512-byte chunks
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kABytes;
  static constexpr int kOffSfa = kOffB + kStages * kBBytes;
  static constexpr int kOffSfb = kOffSfa + kStages * kSfaBytes;
  static constexpr int kOffBar = kOffSfb + kStages * kSfbBytes;
  // full, empty per stage; acc_full, acc_empty per accumulator; drain; epi_sync
  static constexpr int kNumBars = 2 * kStages + 2 * kAccStages + 2;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // MX: one 2 KiB staging buffer per epilogue warp (32 rows x 32 bf16 with the
  // 64-byte swizzle) for the TMA stores of C.
  static constexpr int kEpiBufBytes = 2048;
  static constexpr int kOffEpi = kMX ? ((kOffMisc + 16 + 1023) / 1024) * 1024 : kOffMisc + 16;
  static constexpr int kSmemBytes = kOffEpi + (kMX ? 16 * kEpiBufBytes : 0) + 1024;
  // bytes of both CTAs' loads, all completing on the leader's barrier
  static constexpr uint32_t kTxPair = 2u * (kABytes + kBBytes + kSfaBytes + kSfbBytes);
  static constexpr int kSfColsPerStage = 16;                       // A: columns 0-3, B: 8-15
  static constexpr int kSfCol0 = kAccStages * 256;
  static constexpr int kColsUsed = kSfCol0 + (kMX ? kStages * kSfColsPerStage : 0);
  static constexpr int kTmemCols = kColsUsed <= 256 ? 256 : 512;
  static_assert(kColsUsed <= 512, "TMEM budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ void pair_tile_coords(int t, const GemmArgs& p, int& mb, int& nb) {
  const int per_group = p.group_m * p.tiles_n;
  const int g = t / per_group;
  const int first_m = g * p.group_m;
  const int gm = min(p.tiles_m - first_m, p.group_m);
  const int r = t - g * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

// Work unit u: tile t and its K slabs [kb0, kb1).
__device__ __forceinline__ void pair_unit(int u, const GemmArgs& p, int& t, int& kb0, int& kb1) {
  if (u < p.dp_tiles) {
    t = u;
    kb0 = 0;
    kb1 = p.num_k;
    return;
  }
  const int v = u - p.dp_tiles;
  const int q = v / p.split;
  t = p.dp_tiles + q;
  const int j = v - q * p.split;
  kb0 = static_cast<int>(static_cast<int64_t>(j) * p.num_k / p.split);
  kb1 = static_cast<int>(static_cast<int64_t>(j + 1) * p.num_k / p.split);
}

// Floats of one CTA's partial tile: 16 epilogue warps x 2 chunks x 32
// columns x 32 lanes (= 128 rows x 256 columns), stored so that each warp's
// 32 lanes write 128 contiguous bytes per column.
constexpr int kPairPartFloats = 16 * 2 * 32 * 32;

// GemmArgs fields as in gemm.cuh, with tiles_m = ceil(m/256), tiles_n =
// ceil(n/256).  tmSFA, tmSFB: 3-D maps over the scale layout viewed as uint32
// [n_rt][n_kc][128], boxes of one and two 128-row chunks (both unused in
// per-token mode).  tmC (MX mode with p.tma_c): C as bf16 [m][n] with row
// stride ldc, box 32 x 32, 64-byte swizzle; stores past m or n are clipped.
template <bool kMX, int kStages, int kAccStages, bool kOut8 = false>
__global__ void __launch_bounds__(PairCfg<kMX, kStages, kAccStages>::kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                     const __grid_constant__ CUtensorMap tmC, const GemmArgs p) {
  using Cfg = PairCfg<kMX, kStages, kAccStages>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + kAccStages;
  uint64_t* drain = acc_empty + kAccStages;
  uint64_t* epi_sync = drain + 1;  // the 16 epilogue warps meet here (split K; bounded)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 8);
  const int num_units = p.dp_tiles + (p.num_tiles - p.dp_tiles) * p.split;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());
  // Launched with programmatic stream serialisation: the set-up below may
  // overlap the preceding kernel; the producer and the epilogue wait for it
  // before their first global access, and a following kernel may start its own
  // set-up as SMs free up.
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kAccStages; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 32);  // 16 epilogue warps in each CTA of the pair
    }
    mbar_init(drain, 1);
    mbar_init(epi_sync, 16);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if constexpr (kMX) {
      prefetch_tmap(&tmSFA);
      prefetch_tmap(&tmSFB);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer (both CTAs)
    // The whole warp runs the loop; one elected lane issues (see elect_one_sync).
    griddep_wait();  // A, B and their scales may be written by the preceding kernel
    {
      int stage = 0;
      uint32_t phase = 0, issued_mask = 0, issued_parity = 0;
      bool ok = true;
      for (int u = pair; ok && u < num_units; u += npairs) {
        int t, kb0, kb1, mb, nb;
        pair_unit(u, p, t, kb0, kb1);
        pair_tile_coords(t, p, mb, nb);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!warp_wait_cluster(&empty[stage], phase ^ 1u, p.timeout_ns, abort_flag, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          if (elect_one_sync()) {
            if (leader) mbar_arrive_expect_tx(&full[stage], Cfg::kTxPair);
            const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
            tma_load_2d_pair(smem + Cfg::kOffA + stage * Cfg::kABytes, &tmA, fb, kb * kBK, mb * 256 + rank * 128);
            tma_load_2d_pair(smem + Cfg::kOffB + stage * Cfg::kBBytes, &tmB, fb, kb * kBK, nb * 256 + rank * 128);
            if constexpr (kMX) {
              tma_load_3d_pair(smem + Cfg::kOffSfa + stage * Cfg::kSfaBytes, &tmSFA, fb, 0, kb, mb * 2 + rank);
              // both 128-row chunks of B's scales for this K slab in one load
              tma_load_3d_pair(smem + Cfg::kOffSfb + stage * Cfg::kSfbBytes, &tmSFB, fb, 0, kb, nb * 2);
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
      // Every copy of both CTAs completes on the leader's barriers: the leader
      // waits for the last phase issued on each stage before the pair may exit.
      if (leader)
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s))
            mbar_wait_cluster(&full[s], (issued_parity >> s) & 1u, p.timeout_ns, nullptr, kSiteProducerDrain);
      if (!leader && !ok) {
        // A/B loads of this CTA that the leader never waited for may still be
        // in flight; give them time to land before the final cluster barrier.
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------ MMA issuer (rank 0 only)
    // The whole warp runs the loop; one elected lane issues (see elect_one_sync).
    if (leader) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int u = pair; ok && u < num_units; u += npairs) {
        int t, kb0, kb1;
        pair_unit(u, p, t, kb0, kb1);
        if (!warp_wait_cluster(&acc_empty[acc], acc_phase ^ 1u, p.timeout_ns, abort_flag, kSiteMmaAccEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!warp_wait_cluster(&full[stage], phase, p.timeout_ns, abort_flag, kSiteMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one_sync()) {
            const uint64_t adesc = sw128_kmajor_desc(smem_u32(smem + Cfg::kOffA + stage * Cfg::kABytes));
            const uint64_t bdesc = sw128_kmajor_desc(smem_u32(smem + Cfg::kOffB + stage * Cfg::kBBytes));
            if constexpr (kMX) {
              const uint32_t sfa_t = tmem_base + static_cast<uint32_t>(Cfg::kSfCol0 + stage * Cfg::kSfColsPerStage);
              tmem_cp_32x128b_warpx4_pair(sfa_t,
                                          sf_chunk_desc(smem_u32(smem + Cfg::kOffSfa + stage * Cfg::kSfaBytes)));
              tmem_cp_32x128b_warpx4_pair(sfa_t + 8u,
                                          sf_chunk_desc(smem_u32(smem + Cfg::kOffSfb + stage * Cfg::kSfbBytes)));
              tmem_cp_32x128b_warpx4_pair(sfa_t + 12u,
                                          sf_chunk_desc(smem_u32(smem + Cfg::kOffSfb + stage * Cfg::kSfbBytes + 512)));
#pragma unroll
              for (int kk = 0; kk < kBK / kMmaK; ++kk)
                mma_mxf8f6f4_pair(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc_mxf8f6f4(256, 256, kk, kk), sfa_t,
                                  sfa_t + 8u, kb != kb0 || kk != 0);
            } else {
#pragma unroll
              for (int kk = 0; kk < kBK / kMmaK; ++kk)
                mma_f8f6f4_pair(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc_f8f6f4(256, 256),
                                kb != kb0 || kk != 0);
            }
            tc_commit_pair_mc(&empty[stage], 0x3);
          }
          __syncwarp();
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (elect_one_sync()) tc_commit_pair_mc(&acc_full[acc], 0x3);
        __syncwarp();
        if (++acc == kAccStages) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (elect_one_sync()) tc_commit_pair_mc(drain, 0x1);
      __syncwarp();
      mbar_wait(drain, 0, p.timeout_ns, nullptr, kSiteDrain);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ epilogue (both CTAs)
    griddep_wait();  // C, the workspace and the scales may belong to the preceding kernel
    const int sp = warp & 3;
    const int quarter = (warp - Cfg::kEpiWarp0) >> 2;  // 64-column slice of the 256-column tile
    float s_out = 1.f, r_out = 1.f;
    bool out_fast = true;
    if constexpr (kOut8) {
      s_out = __ldg(p.s_out);
      r_out = __frcp_rn(s_out);
      out_fast = quotient_fast_ok(s_out);
    }
    int acc = 0;
    uint32_t acc_phase = 0, sync_phase = 0;
    const int wl = warp - Cfg::kEpiWarp0;  // 0..15
    // The 16 epilogue warps meet (split K); false if the wait expired or the CTA aborted.
    auto epi_meet = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_sync);
      const bool ok = mbar_wait(epi_sync, sync_phase, p.timeout_ns, abort_flag, kSiteEpiSync);
      sync_phase ^= 1u;
      return ok;
    };
    for (int u = pair; u < num_units; u += npairs) {
      int t, kb0, kb1, mb, nb;
      pair_unit(u, p, t, kb0, kb1);
      pair_tile_coords(t, p, mb, nb);
      if (!mbar_wait_cluster(&acc_full[acc], acc_phase, p.timeout_ns, abort_flag, kSiteEpiAccFull)) break;
      tc_fence_after();
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(sp * 32) << 16) + static_cast<uint32_t>(acc * 256 + quarter * 64);
      uint32_t r[2][32];
      tmem_ld_32x32b_x32(t_row, r[0]);
      tmem_ld_32x32b_x32(t_row + 32, r[1]);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      asm volatile("" : FP8MM_RW32(r[0]));
      asm volatile("" : FP8MM_RW32(r[1]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[acc]), 0));
      if (++acc == kAccStages) {
        acc = 0;
        acc_phase ^= 1u;
      }

      const int row = mb * 256 + static_cast<int>(rank) * 128 + sp * 32 + lane;
      float s_row = 1.f;
      if constexpr (!kMX) s_row = (row < p.m) ? __ldg(p.sa + row) : 0.f;
      if (u >= p.dp_tiles) {
        // Publish this part, count it; the last part to arrive reduces.
        float* mine =
            p.partials + (static_cast<int64_t>(u - p.dp_tiles) * 2 + rank) * kPairPartFloats + wl * 2048 + lane;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch)
#pragma unroll
          for (int j = 0; j < 32; ++j) mine[ch * 1024 + j * 32] = __uint_as_float(r[ch][j]);
        // The 16 warps' partial stores are ordered before one thread's
        // acquire-release counter increment at GPU scope (the barrier between
        // them is CTA-scope release/acquire and release is cumulative); the
        // last part's increment acquires every earlier part's stores, and the
        // barrier after it hands them to its other threads.
        if (!epi_meet()) break;
        unsigned* ticket = p.tickets + static_cast<int64_t>(t - p.dp_tiles) * 2 + rank;
        if (threadIdx.x == Cfg::kEpiWarp0 * 32) {
          unsigned prev;
          asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(ticket) : "memory");
          *last_flag = (prev == static_cast<unsigned>(p.split - 1)) ? 1 : 0;
        }
        if (!epi_meet()) break;
        if (*last_flag == 0) continue;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          const int col0 = nb * 256 + quarter * 64 + ch * 32;
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
          for (int part = 0; part < p.split; ++part) {
            const float* src =
                p.partials + (static_cast<int64_t>((t - p.dp_tiles) * p.split + part) * 2 + rank) * kPairPartFloats +
                wl * 2048 + ch * 1024 + lane;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += __ldcg(src + j * 32);
          }
          if constexpr (!kMX) {
            const float sbv = (col0 + lane < p.n) ? __ldg(p.sb + col0 + lane) : 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = scale_acc(v[j], s_row, __shfl_sync(0xFFFFFFFFu, sbv, j));
          }
          store_out32<kOut8>(p, row, col0, v, s_out, r_out, out_fast);
        }
        if (threadIdx.x == Cfg::kEpiWarp0 * 32) *ticket = 0u;
        continue;
      }
      if (kMX && p.tma_c) {
        // bf16 rows into the warp's staging buffer (lane = row; 16-byte chunk q
        // of a 64-byte row lands at chunk q ^ ((row >> 1) & 3), the 64-byte
        // swizzle, so each 16-byte store of the warp takes four wavefronts),
        // then one TMA store of the 32 x 32 block.  Measured on B200 (ffn_up):
        // 0.8 % faster than the 32-byte stores from registers, bit-identical.
        uint8_t* buf = smem + Cfg::kOffEpi + wl * Cfg::kEpiBufBytes;
        const int row0 = mb * 256 + static_cast<int>(rank) * 128 + sp * 32;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t packed[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[ch][2 * j]), __uint_as_float(r[ch][2 * j + 1]));
            packed[j] = *reinterpret_cast<uint32_t*>(&h);
          }
          if (lane == 0) bulk_wait_read0();  // the previous store from this buffer has read it
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(buf + lane * 64 + ((q ^ ((lane >> 1) & 3)) * 16)) =
                make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmC, buf, nb * 256 + quarter * 64 + ch * 32, row0);
            bulk_commit();
          }
        }
        continue;
      }
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const int col0 = nb * 256 + quarter * 64 + ch * 32;
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
    if (kMX && p.tma_c && lane == 0) bulk_wait_all0();  // this warp's stores of C are complete
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still signal or read it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace fp8mm
