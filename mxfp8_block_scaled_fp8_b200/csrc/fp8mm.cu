// fp8mm.cu -- the C ABI of include/fp8mm.h: argument checks, TMA descriptors,
// launch geometry, and the kernels of quant.cuh / gemm.cuh / decode.cuh
// (one translation unit, so the device error word is a single symbol).
#include "fp8mm.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <utility>

#include "decode.cuh"
#include "kvcache.cuh"
#include "gemm.cuh"
#include "gemm2.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace fp8mm {

// ------------------------------------------------------------------ host state
static thread_local int t_last_cuda_error = 0;

static fp8mm_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return FP8MM_ERR_LAUNCH;
}

struct DeviceInfo {
  int device = -1;
  int sms = 0;
  bool sm100 = false;
};

static std::mutex g_mu;

static fp8mm_status current_device(DeviceInfo* info) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  static DeviceInfo cache[64];
  if (dev < 0 || dev >= 64) return FP8MM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (cache[dev].device != dev) {
    int major = 0, sms = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    cache[dev].device = dev;
    cache[dev].sms = sms;
    cache[dev].sm100 = (major == 10);
  }
  *info = cache[dev];
  return info->sm100 ? FP8MM_OK : FP8MM_ERR_UNSUPPORTED;
}

// Opt a kernel into its dynamic shared memory size, once per device.
static fp8mm_status ensure_smem(const void* kernel, int bytes, int dev) {
  static std::set<std::pair<const void*, int>> done;
  std::lock_guard<std::mutex> lock(g_mu);
  if (done.count({kernel, dev})) return FP8MM_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e);
  done.insert({kernel, dev});
  return FP8MM_OK;
}

static uint64_t wait_timeout_ns() {
  static uint64_t ns = [] {
    const char* s = std::getenv("FP8MM_WAIT_TIMEOUT_MS");
    long long ms = s ? std::atoll(s) : 0;
    return static_cast<uint64_t>(ms > 0 ? ms : 2000) * 1000000ull;
  }();
  return ns;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a row-major uint8 matrix [rows, k] (row stride k bytes),
// box = 128 bytes of K x box_rows rows, 128-byte swizzle, zero fill outside.
static fp8mm_status make_map(CUtensorMap* map, const void* base, int64_t k, int64_t rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k)};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return FP8MM_OK;
}

// 3-D map over a library scale buffer viewed as uint32 [n_rt][n_kc][128]
// (one 512-byte chunk per 128-row tile and 4-block group); box = box_rt chunks
// of consecutive row tiles at one K group; zero fill past the last row tile.
static fp8mm_status make_sf_map(CUtensorMap* map, const void* sf, int64_t k, int64_t rows, int box_rt) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cuda_fail(cudaErrorNotSupported);
  const int64_t n_kc = (k + 127) / 128, n_rt = (rows + 127) / 128;
  cuuint64_t dims[3] = {128u, static_cast<cuuint64_t>(n_kc), static_cast<cuuint64_t>(n_rt)};
  cuuint64_t strides[2] = {512u, static_cast<cuuint64_t>(n_kc) * 512u};
  cuuint32_t box[3] = {128u, 1u, static_cast<cuuint32_t>(box_rt)};
  cuuint32_t es[3] = {1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(sf), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return FP8MM_OK;
}

// 2-D map over a bf16 output C [m][n] with row stride ldc elements, for the
// paired MX kernel's TMA stores: box 32 columns x 32 rows, 64-byte swizzle.
// Needs a 16-byte aligned base and ldc * 2 a multiple of 16.  An optional
// fast path: false (and no error recorded) when the map cannot be made.
static bool make_c_map(CUtensorMap* map, void* c, int64_t m, int64_t n, int64_t ldc) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(m)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldc) * 2u};
  cuuint32_t box[2] = {32u, 32u};
  cuuint32_t es[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Launch with programmatic stream serialisation (the kernel may begin while
// the preceding kernel on the stream finishes; it waits for it in-kernel).
template <typename... KArgs, typename... Args>
static fp8mm_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                               Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) {
    t_last_cuda_error = static_cast<int>(e);
    return FP8MM_ERR_LAUNCH;
  }
  return FP8MM_OK;
}

static fp8mm_status launched() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FP8MM_OK : cuda_fail(e);
}

// ------------------------------------------------------------------ kernels' configs
using G1 = GemmCfg<false, 256, 4, 2>;
using G2 = GemmCfg<true, 256, 4, 1>;
using G1n = GemmCfg<false, 128, 6, 2>;  // 128 x 128 tiles
using G2n = GemmCfg<true, 128, 6, 2>;
// Small-M ring depth: as many stages as half an SM's shared memory holds, so
// that two CTAs share each SM.  For 48- and 64-token tiles that is 4 stages
// (one CTA per SM with 9 / 8 stages was 6-16 % slower on the decode shapes at
// m = 33..64, level on down-projection m = 64).
constexpr int dec_stages(int nm) { return nm <= 32 ? 5 : 4; }
// With the activation quantized in the kernel (m <= 8).
constexpr int dec_stages_qx(int nm) { return nm <= 16 ? 5 : 0; }

__global__ void selftest_wait_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must expire and report.
  if (threadIdx.x == 0) mbar_wait(&bar, 0, timeout_ns, &abort_flag, kSiteSelfTest);
}

// ------------------------------------------------------------------ launchers
template <typename Cfg, typename Kern>
static fp8mm_status launch_tiled_kernel(Kern kern, int grid, const CUtensorMap& ta, const CUtensorMap& tb,
                                        const GemmArgs& p, cudaStream_t stream, int dev) {
  fp8mm_status st = ensure_smem(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, dev);
  if (st != FP8MM_OK) return st;
  return launch_pdl(kern, dim3(grid), dim3(kGemmThreads), Cfg::kSmemBytes, stream, ta, tb, p);
}

// Single-SM tiled kernel, 128 x 256 tiles or (n128) 128 x 128 tiles.
// c8 != nullptr (mode 1 only): E4M3 output c8 = E4M3(C / *s_out) instead of bf16 c.
static fp8mm_status launch_tiled(bool mx, const void* a, const void* b, const uint8_t* sfa, const uint8_t* sfb,
                                 int64_t m, int64_t n, int64_t k, const float* sa, const float* sb, void* c,
                                 int64_t ldc, cudaStream_t stream, const DeviceInfo& dev, uint8_t* c8 = nullptr,
                                 const float* s_out = nullptr, bool n128 = false) {
  const int bn = n128 ? 128 : 256;
  CUtensorMap ta, tb;
  fp8mm_status st = make_map(&ta, a, k, m, kBM);
  if (st != FP8MM_OK) return st;
  st = make_map(&tb, b, k, n, bn);
  if (st != FP8MM_OK) return st;
  GemmArgs p{};
  p.m = static_cast<int>(m);
  p.n = static_cast<int>(n);
  p.k = static_cast<int>(k);
  p.num_k = static_cast<int>(cdiv(k, kBK));
  p.tiles_m = static_cast<int>(cdiv(m, kBM));
  p.tiles_n = static_cast<int>(cdiv(n, bn));
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.c = static_cast<__nv_bfloat16*>(c);
  p.ldc = ldc;
  p.sa = sa;
  p.sb = sb;
  p.sfa = sfa;
  p.sfb = sfb;
  p.n_kc = static_cast<int>(cdiv(k, 128));
  p.sfb_row_tiles = static_cast<int>(cdiv(n, 128));
  p.timeout_ns = wait_timeout_ns();
  p.c8 = c8;
  p.s_out = s_out;
  p.split = 1;
  const int grid = std::min(p.num_tiles, dev.sms);
  if (n128) {
    if (c8 != nullptr) return launch_tiled_kernel<G1n>(gemm_tiled_kernel<false, 128, 6, 2, true>, grid, ta, tb, p, stream, dev.device);
    if (mx) return launch_tiled_kernel<G2n>(gemm_tiled_kernel<true, 128, 6, 2>, grid, ta, tb, p, stream, dev.device);
    return launch_tiled_kernel<G1n>(gemm_tiled_kernel<false, 128, 6, 2>, grid, ta, tb, p, stream, dev.device);
  }
  if (c8 != nullptr) return launch_tiled_kernel<G1>(gemm_tiled_kernel<false, 256, 4, 2, true>, grid, ta, tb, p, stream, dev.device);
  if (mx) return launch_tiled_kernel<G2>(gemm_tiled_kernel<true, 256, 4, 1>, grid, ta, tb, p, stream, dev.device);
  return launch_tiled_kernel<G1>(gemm_tiled_kernel<false, 256, 4, 2>, grid, ta, tb, p, stream, dev.device);
}

// Tiled kernel for a call: the requested one, or (AUTO / TILED) paired-SM
// 256 x 256 tiles from m >= 256 and single-SM 128 x 256 tiles below -- unless
// single-SM 128 x 128 tiles need fewer waves, a 128 x 128 wave counted as
// three quarters of a 256-wide one (half the work per SM, with relatively
// more fixed cost: scale copies, start-up, epilogue).  That picks 128 x 128
// where the 256-wide tiles leave most SMs idle, e.g. M 2048 x N 1024: 32
// paired tiles on 74 SM pairs, or 128 single-SM tiles on 148 SMs.
enum class Tiled { kPair, k1Sm, k1SmN128 };
static Tiled tiled_kind(int kind, int64_t m, int64_t n, int64_t sms) {
  if (kind == FP8MM_KERNEL_TILED_2SM) return Tiled::kPair;
  if (kind == FP8MM_KERNEL_TILED_1SM) return Tiled::k1Sm;
  if (kind == FP8MM_KERNEL_TILED_1SM_N128) return Tiled::k1SmN128;
  const bool pair = m >= 256;
  const int64_t big = pair ? cdiv(m, 256) * cdiv(n, 256) : cdiv(m, kBM) * cdiv(n, 256);
  const int64_t waves_big = cdiv(big, pair ? std::max<int64_t>(1, sms / 2) : sms);
  const int64_t waves_small = cdiv(cdiv(m, kBM) * cdiv(n, 128), sms);
  if (3 * waves_small < 4 * waves_big) return Tiled::k1SmN128;
  return pair ? Tiled::kPair : Tiled::k1Sm;
}

using P1 = PairCfg<false, 6, 2>;
using P2 = PairCfg<true, 5, 1>;

// Largest number of co-resident 2-CTA clusters of a pair kernel (cached per
// kernel and device).
static fp8mm_status max_pairs(const void* kern, int smem, int threads, const DeviceInfo& dev, int* out) {
  static std::map<std::pair<const void*, int>, int> cached;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = cached.find({kern, dev.device});
    if (it != cached.end()) {
      *out = it->second;
      return FP8MM_OK;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * (dev.sms / 2), 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
  if (e != cudaSuccess) return cuda_fail(e);
  if (n <= 0) n = 1;
  std::lock_guard<std::mutex> lock(g_mu);
  cached[{kern, dev.device}] = n;
  *out = n;
  return FP8MM_OK;
}

// 256-row output tiles per raster group of the paired-SM kernel.  Within a
// group the tiles run down M, then across N, so B is read from DRAM once per
// group and the group's A rows are reused from L2.  Where B is too large to
// stay in L2 between groups, taller groups read it fewer times: measured on
// B200 with the 8192 x 22016 x 8192 MX GEMM, 16 rows of tiles are 1.3 %
// faster than 8 (32 slower: the 67 MB of A no longer stays in L2), while on
// 8192 x 2048 x 8192 (B 16 MB, L2-resident) 16 are 1.6 % slower than 8.
static int pair_group_m(int64_t n, int64_t k) { return n * k > (int64_t{64} << 20) ? 2 * kPairGroupM : kPairGroupM; }

// Split K of the paired-SM kernel over `pairs` co-resident SM pairs: the
// tiles of the last, partly filled wave (all tiles, where they fill less
// than one wave) run as `split` K parts each -- the most parts that still fit
// in that wave, each of at least 16 slabs of 128, at most 8 -- so that the
// wave keeps every pair busy; the other tiles run whole.  Only for m > 64
// (below that mxfp8_gemm runs the small-M kernel) and K of at least 64 slabs:
// the fp32 partials cost a write and a read of 256 KB per part and tile
// through L2, so short K gains nothing.  Measured on B200: 512 x 2048 x 8192
// (16 tiles, 4 parts of 16 slabs) takes 23.2 us against 29.5 us unsplit
// (MX), but 2048 x 1024 x 4096 with 2 parts of 16 slabs 21.4 us against 18.3
// us on 128 x 128 single-SM tiles.
struct PairPlan {
  int split;     // K parts per split tile (1: no split)
  int dp_tiles;  // tiles run whole; the rest are split
};
static PairPlan pair_plan(int64_t m, int64_t n, int64_t k, int64_t pairs) {
  const int64_t num_k = cdiv(k, kBK);
  const int64_t tiles = cdiv(m, 256) * cdiv(n, 256);
  if (m <= 64 || num_k < 64 || pairs < 2) return {1, static_cast<int>(tiles)};
  const int64_t rem = tiles % pairs;
  if (rem == 0) return {1, static_cast<int>(tiles)};
  const int64_t s = std::min<int64_t>(std::min<int64_t>(pairs / rem, num_k / 16), 8);
  if (s < 2) return {1, static_cast<int>(tiles)};
  return {static_cast<int>(s), static_cast<int>(tiles - rem)};
}
static size_t round256(size_t b) { return (b + 255) & ~size_t(255); }
// Workspace of a split paired launch on a device with `sms` SMs: at most one
// split part per co-resident pair (<= sms / 2), each with both CTAs'
// partials, then one arrival counter per (split tile, rank).  Shapes the plan
// never splits need none.
static size_t pair_partials_bytes(int64_t sms) {
  return round256(static_cast<size_t>(std::max<int64_t>(1, sms / 2)) * 2 * kPairPartFloats * sizeof(float));
}
static size_t pair_split_bytes(int64_t m, int64_t k, int64_t sms) {
  if (m <= 64 || cdiv(k, kBK) < 64) return 0;
  return pair_partials_bytes(sms) + round256(static_cast<size_t>(std::max<int64_t>(1, sms / 2)) * 2 * 4);
}
// Whether a tiled call may split: a workspace is given and the kernel choice
// allows the paired kernel (AUTO, TILED, TILED_2SM); 1 if so, 0 if not, -1
// when the shape may split and that workspace is too small or misaligned.
static int tiled_split(const fp8mm_opts* opt, int kind, int64_t m, int64_t n, int64_t k, int64_t sms) {
  (void)n;
  if (opt == nullptr || opt->workspace == nullptr) return 0;
  if (kind != FP8MM_KERNEL_AUTO && kind != FP8MM_KERNEL_TILED && kind != FP8MM_KERNEL_TILED_2SM) return 0;
  const size_t need = pair_split_bytes(m, k, sms);
  if (need == 0) return 0;
  if (opt->workspace_bytes < need || !aligned(opt->workspace, 256)) return -1;
  return 1;
}
// Tiled kernel of a call that has passed tiled_split (ws: a usable
// workspace): tiled_kind's choice, except that a shape whose tiles all split
// (fewer than one wave of pairs) takes the paired kernel whenever there is a
// workspace.
static Tiled tiled_choice(int kind, int64_t m, int64_t n, int64_t k, bool ws, int64_t sms) {
  const Tiled tk = tiled_kind(kind, m, n, sms);
  if (ws) {
    const PairPlan plan = pair_plan(m, n, k, std::max<int64_t>(1, sms / 2));
    if (plan.split > 1 && plan.dp_tiles == 0) return Tiled::kPair;
  }
  return tk;
}

// Paired-SM kernel.  c8 != nullptr (mode 1 only): E4M3 output c8 =
// E4M3(C / *s_out) instead of bf16 c.  workspace != nullptr
// (pair_split_bytes(m, k, sms) bytes, counters zero): K split as pair_plan
// says, partials and counters there.
static fp8mm_status launch_pair(bool mx, const void* a, const void* b, const uint8_t* sfa, const uint8_t* sfb,
                                int64_t m, int64_t n, int64_t k, const float* sa, const float* sb, void* c,
                                int64_t ldc, cudaStream_t stream, const DeviceInfo& dev, uint8_t* c8 = nullptr,
                                const float* s_out = nullptr, void* workspace = nullptr) {
  CUtensorMap ta, tb, tsa, tsb, tc;
  fp8mm_status st = make_map(&ta, a, k, m, 128);
  if (st != FP8MM_OK) return st;
  if ((st = make_map(&tb, b, k, n, 128)) != FP8MM_OK) return st;
  if (mx) {
    if ((st = make_sf_map(&tsa, sfa, k, m, 1)) != FP8MM_OK) return st;
    if ((st = make_sf_map(&tsb, sfb, k, n, 2)) != FP8MM_OK) return st;
  } else {
    tsa = ta;  // unused in per-token mode
    tsb = tb;
  }
  GemmArgs p{};
  p.m = static_cast<int>(m);
  p.n = static_cast<int>(n);
  p.k = static_cast<int>(k);
  p.num_k = static_cast<int>(cdiv(k, kBK));
  p.tiles_m = static_cast<int>(cdiv(m, 256));
  p.tiles_n = static_cast<int>(cdiv(n, 256));
  p.num_tiles = p.tiles_m * p.tiles_n;
  p.c = static_cast<__nv_bfloat16*>(c);
  p.ldc = ldc;
  p.sa = sa;
  p.sb = sb;
  p.sfa = sfa;
  p.sfb = sfb;
  p.n_kc = static_cast<int>(cdiv(k, 128));
  p.sfb_row_tiles = static_cast<int>(cdiv(n, 128));
  p.timeout_ns = wait_timeout_ns();
  p.c8 = c8;
  p.s_out = s_out;
  p.group_m = pair_group_m(n, k);
  p.split = 1;
  p.dp_tiles = p.num_tiles;
  // MX mode writes whole tiles of C by TMA stores where C allows a tensor map
  // (16-byte aligned base and row stride); otherwise, and for split tiles, by
  // stores from registers.
  tc = ta;  // unused unless p.tma_c
  p.tma_c = (mx && c != nullptr && aligned(c, 16) && (ldc * 2) % 16 == 0 && make_c_map(&tc, c, m, n, ldc)) ? 1 : 0;
  const void* kern = mx ? reinterpret_cast<const void*>(gemm_pair_kernel<true, 5, 1>)
                     : c8 ? reinterpret_cast<const void*>(gemm_pair_kernel<false, 6, 2, true>)
                          : reinterpret_cast<const void*>(gemm_pair_kernel<false, 6, 2>);
  const int smem = mx ? P2::kSmemBytes : P1::kSmemBytes;
  const int threads = mx ? P2::kThreads : P1::kThreads;
  if ((st = ensure_smem(kern, smem, dev.device)) != FP8MM_OK) return st;
  int pairs = 0;
  if ((st = max_pairs(kern, smem, threads, dev, &pairs)) != FP8MM_OK) return st;
  if (workspace != nullptr) {
    const PairPlan plan = pair_plan(m, n, k, std::min<int64_t>(pairs, std::max(1, dev.sms / 2)));
    if (plan.split > 1) {
      p.split = plan.split;
      p.dp_tiles = plan.dp_tiles;
      p.partials = static_cast<float*>(workspace);
      p.tickets = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(workspace) + pair_partials_bytes(dev.sms));
    }
  }
  pairs = std::min(pairs, p.dp_tiles + (p.num_tiles - p.dp_tiles) * p.split);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see the kernel's griddep calls
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = mx   ? cudaLaunchKernelEx(&cfg, gemm_pair_kernel<true, 5, 1>, ta, tb, tsa, tsb, tc, p)
                  : c8 ? cudaLaunchKernelEx(&cfg, gemm_pair_kernel<false, 6, 2, true>, ta, tb, tsa, tsb, tc, p)
                       : cudaLaunchKernelEx(&cfg, gemm_pair_kernel<false, 6, 2>, ta, tb, tsa, tsb, tc, p);
  if (e != cudaSuccess) return cuda_fail(e);
  return launched();
}

static int small_m_tile(int64_t m) { return m <= 16 ? 16 : m <= 32 ? 32 : m <= 48 ? 48 : 64; }

static size_t small_m_partials_bytes(int ctas, int nm) {
  size_t b = static_cast<size_t>(2) * ctas * nm * 128 * sizeof(float);
  return (b + 255) & ~size_t(255);
}

// Launched with programmatic stream serialisation: the kernel may start while
// the preceding kernel on the stream (normally the activation quantizer) is
// still running; it prefetches weights and then waits for it in-kernel.
// With p.cluster_s > 1 the kernel reduces split tiles inside clusters of
// p.cluster_s CTAs (one cluster per weight tile) instead of the workspace.
// kSF8: the activation's scales are in the small-M (8x4) layout.
template <int kNM, bool kQX = false, bool kSF8 = false>
static fp8mm_status launch_small_m_t(const CUtensorMap& tw, const CUtensorMap& tx, const DecodeArgs& p,
                                     cudaStream_t stream, int dev) {
  constexpr int kStages = kQX ? dec_stages_qx(kNM) : dec_stages(kNM);
  using Cfg = DecodeCfg<kNM, kStages, kQX, kSF8>;
  const bool cr = p.cluster_s > 1;
  auto kern = cr ? gemm_small_m_kernel<kNM, kStages, kQX, true, kSF8>
                 : gemm_small_m_kernel<kNM, kStages, kQX, false, kSF8>;
  fp8mm_status st = ensure_smem(reinterpret_cast<const void*>(kern), Cfg::kSmemBytes, dev);
  if (st != FP8MM_OK) return st;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cr ? static_cast<unsigned>(p.cluster_s) : 1u;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.gridDim = dim3(p.ctas, 1, 1);
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = cr ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tw, tx, p);
  if (e != cudaSuccess) return cuda_fail(e);
  return launched();
}

// Largest cluster the small-M kernel reduces in (portable cluster size).
constexpr int64_t kMaxClusterSplit = 8;

// CTAs per weight tile when `ctas` is a tile-aligned split that the kernel can
// reduce inside clusters (2..8 CTAs per tile, each with at least one K slab);
// 0 otherwise.  CTA b = t*s + r owns slabs [floor(b*U/G), floor((b+1)*U/G))
// = t*num_k + [floor(r*num_k/s), floor((r+1)*num_k/s)): always inside tile t,
// whether or not s divides num_k.
static int cluster_split(int64_t ctas, int64_t n_tiles, int64_t num_k) {
  if (ctas % n_tiles != 0) return 0;
  const int64_t s = ctas / n_tiles;
  return (s >= 2 && s <= kMaxClusterSplit && s <= num_k) ? static_cast<int>(s) : 0;
}

// Largest tile-aligned CTA count (s CTAs per tile, 2 <= s <= 8, s dividing
// the K slabs, at least kMinSlabsPerCta slabs each) within `slots`; 0 if none.
static int64_t best_cluster_ctas(int64_t n_tiles, int64_t num_k, int64_t slots);

// Slabs per CTA (past the staged ones) whose weights the small-M kernel
// prefetches into L2 when it starts.  Only where two CTAs share an SM: the
// next call's CTAs then start as this call's finish, and the prefetch keeps
// HBM busy through this call's tail.  Measured on B200 (14336 x 4096, m <= 32,
// back-to-back calls): 2 slabs ahead makes a call 2-5 % faster, 4 and more
// slower.  With one CTA per SM the next call's CTAs sit beside this call's
// from its start, and any prefetch only takes bandwidth from it.
constexpr int64_t kL2AheadSlabs = 2;
static int small_m_l2_ahead(int64_t units, int64_t ctas, int64_t sms) {
  if (ctas <= sms) return 0;
  return static_cast<int>(std::min<int64_t>(kL2AheadSlabs, cdiv(units, ctas)));
}

// CTAs of the small-M kernel: the requested number; else one per SM, or two
// per SM when the weight tiles are short (<= 48 K slabs, so the finer split
// adds at most about one contributor per tile) and every CTA keeps >= 8
// slabs; in every case no fewer than 4 slabs per CTA, never more CTAs than
// slabs, never fewer than the tiles.
//
// That count is replaced by a tile-aligned one -- s CTAs per weight tile,
// with s dividing the tile's K slabs, so every CTA runs one segment inside
// one tile and all contributors of a tile are equal (and reduce inside a
// cluster) -- when the largest such count that fits two CTAs per SM comes
// within 75 % of it (16-token tiles) or 60 % (larger tiles, whose split-tile
// partials cost more).  Measured on B200 with back-to-back calls (GEMM alone,
// before 48- and 64-token tiles ran two per SM): 6144 x
// 4096 at m <= 32 with 192 CTAs instead of 148 is 12-17 % faster and at m = 64
// with 96 instead of 148 10 %, 4096 x 14336 at m <= 8 with 256 instead of 148
// 8 % and at m = 64 with 128 instead of 148 6 %, 14336 x 4096 at m = 32 with
// 224 instead of 296 5 % and at m = 64 with 112 instead of 148 9 %.  With
// converged issue (see elect_one_sync), 14336 x 4096 at m <= 16 with 224
// instead of 296 is 4-5 % faster (13.3 against 13.9 us; it was 3 % slower
// before).  Splits that do not divide the K slabs (cluster_split allows them)
// measured slower than the dividing ones next to them (6144 x 4096: 144 and
// 240 CTAs 8.8 us against 7.9 us at 192; 4096 x 14336: 160-224 against 128
// and 256).  Counts between the aligned ones are slower than both neighbours
// (e.g. 6144 x 4096, m = 1: 8.5 us at 192 CTAs, 9.6-10.4 us at 160-240).
constexpr int64_t kMinSlabsPerCta = 4;
static int64_t best_cluster_ctas(int64_t n_tiles, int64_t num_k, int64_t slots) {
  int64_t best = 0;
  for (int64_t s = 2; s <= kMaxClusterSplit && s <= num_k / kMinSlabsPerCta; ++s)
    if (num_k % s == 0 && n_tiles * s <= slots) best = n_tiles * s;
  return best;
}
static int small_m_ctas(int64_t units, int64_t n_tiles, int64_t num_k, int nm, int64_t requested, int64_t sms) {
  int64_t g = requested;
  if (g <= 0) {
    const bool two_per_sm = num_k <= 48 && units >= 2 * sms * 8;
    g = std::min<int64_t>(two_per_sm ? 2 * sms : sms, std::max<int64_t>(n_tiles, cdiv(units, kMinSlabsPerCta)));
    const int64_t slots = 2 * sms;
    int64_t aligned = 0;
    for (int64_t s = 1; s <= num_k / kMinSlabsPerCta; ++s)
      if (num_k % s == 0 && n_tiles * s <= slots) aligned = n_tiles * s;
    if (aligned > 0 && aligned * 20 >= g * (nm <= 16 ? 15 : 12)) g = aligned;
  }
  g = std::min<int64_t>(g, units);
  return static_cast<int>(std::max<int64_t>(g, 1));
}

// a: E4M3 codes [m, k] with scales sfa, or (qx) bf16 [m, k] with row stride
// lda elements, quantized in the kernel (sfa unused).
static fp8mm_status launch_small_m(const void* a, const uint8_t* sfa, const void* b, const uint8_t* sfb, int64_t m,
                                   int64_t n, int64_t k, void* c, int64_t ldc, const fp8mm_opts* opt,
                                   cudaStream_t stream, const DeviceInfo& dev, bool qx = false, int64_t lda = 0) {
  const int nm = small_m_tile(m);
  DecodeArgs p{};
  p.m = static_cast<int>(m);
  p.n = static_cast<int>(n);
  p.k = static_cast<int>(k);
  p.num_k = static_cast<int>(cdiv(k, 128));
  p.n_tiles = static_cast<int>(cdiv(n, 128));
  p.units = static_cast<int64_t>(p.n_tiles) * p.num_k;
  p.c = static_cast<__nv_bfloat16*>(c);
  p.ldc = ldc;
  p.sfw = sfb;
  p.sfx = sfa;
  p.n_kc = p.num_k;
  p.timeout_ns = wait_timeout_ns();
  p.prefetch_w = (opt != nullptr && (opt->flags & FP8MM_FLAG_WEIGHTS_READY)) ? 1 : 0;
  const bool via_ws = opt != nullptr && (opt->flags & FP8MM_FLAG_SPLIT_VIA_WORKSPACE);
  const int64_t requested = opt != nullptr ? opt->small_m_ctas : 0;
  p.ctas = small_m_ctas(p.units, p.n_tiles, p.num_k, nm, requested, dev.sms);
  p.cluster_s = via_ws ? 0 : cluster_split(p.ctas, p.n_tiles, p.num_k);
  if (p.cluster_s == 0) {
    if (opt != nullptr && opt->workspace != nullptr) {
      const size_t need = fp8mm_workspace_bytes(m, n, k, p.ctas);
      if (opt->workspace_bytes < need || !aligned(opt->workspace, 256)) return FP8MM_ERR_WORKSPACE;
      p.partials = static_cast<float*>(opt->workspace);
      p.tickets = reinterpret_cast<unsigned*>(static_cast<uint8_t*>(opt->workspace) +
                                              small_m_partials_bytes(p.ctas, nm));
    } else {
      // No workspace: a tile-aligned split reduced in clusters where one
      // fits (automatic count only), else one CTA per weight tile over all
      // of K (no partial sums).
      const int64_t g = (requested > 0 || via_ws) ? 0 : best_cluster_ctas(p.n_tiles, p.num_k, 2 * dev.sms);
      p.ctas = static_cast<int>(g > 0 ? g : p.n_tiles);
      p.cluster_s = g > 0 ? cluster_split(g, p.n_tiles, p.num_k) : 0;
    }
  }
  p.l2_ahead = small_m_l2_ahead(p.units, p.ctas, dev.sms);
  CUtensorMap tw, tx;
  fp8mm_status st = make_map(&tw, b, k, n, 128);
  if (st != FP8MM_OK) return st;
  if (!qx && (st = make_map(&tx, a, k, m, nm)) != FP8MM_OK) return st;
  if (qx) {  // m <= 8: the activation is read by the kernel itself
    p.x = static_cast<const __nv_bfloat16*>(a);
    p.ldx = lda;
    return launch_small_m_t<16, true>(tw, tw, p, stream, dev.device);
  }
  if (opt != nullptr && (opt->flags & FP8MM_FLAG_SF_A_8X4)) {
    switch (nm) {
      case 16: return launch_small_m_t<16, false, true>(tw, tx, p, stream, dev.device);
      case 32: return launch_small_m_t<32, false, true>(tw, tx, p, stream, dev.device);
      case 48: return launch_small_m_t<48, false, true>(tw, tx, p, stream, dev.device);
      default: return launch_small_m_t<64, false, true>(tw, tx, p, stream, dev.device);
    }
  }
  switch (nm) {
    case 16: return launch_small_m_t<16>(tw, tx, p, stream, dev.device);
    case 32: return launch_small_m_t<32>(tw, tx, p, stream, dev.device);
    case 48: return launch_small_m_t<48>(tw, tx, p, stream, dev.device);
    default: return launch_small_m_t<64>(tw, tx, p, stream, dev.device);
  }
}

}  // namespace fp8mm

using namespace fp8mm;

// ====================================================================== C ABI
extern "C" {

int fp8mm_version(void) { return 10000; }

const char* fp8mm_status_str(fp8mm_status s) {
  switch (s) {
    case FP8MM_OK: return "ok";
    case FP8MM_ERR_NULL: return "null pointer";
    case FP8MM_ERR_SHAPE: return "bad shape";
    case FP8MM_ERR_ALIGN: return "misaligned pointer or leading dimension";
    case FP8MM_ERR_UNSUPPORTED: return "no sm_100 device";
    case FP8MM_ERR_LAUNCH: return "CUDA call failed";
    case FP8MM_ERR_WORKSPACE: return "workspace missing or too small";
    case FP8MM_ERR_DEVICE: return "device-side error (bounded wait expired)";
    default: return "unknown status";
  }
}

int fp8mm_last_cuda_error(void) { return t_last_cuda_error; }

size_t fp8mm_sf_bytes(int64_t rows, int64_t k) {
  if (rows <= 0 || k <= 0) return 0;
  return static_cast<size_t>(cdiv(rows, 128) * 128) * static_cast<size_t>(cdiv(k, 128)) * 4;
}

int64_t fp8mm_sf_offset(int64_t rows, int64_t k, int64_t row, int64_t block) {
  if (rows <= 0 || k <= 0) return -1;
  const int64_t n_kc = cdiv(k, 128);
  if (row < 0 || row >= cdiv(rows, 128) * 128 || block < 0 || block >= n_kc * 4) return -1;
  return ((row / 128) * n_kc + block / 4) * 512 + (row % 32) * 16 + ((row % 128) / 32) * 4 + (block % 4);
}

fp8mm_status fp8mm_sf_to_canonical(const uint8_t* sf, int64_t rows, int64_t k, uint8_t* canonical) {
  if (rows < 0 || k < 0 || k % 32 != 0) return FP8MM_ERR_SHAPE;
  if (rows == 0 || k == 0) return FP8MM_OK;
  if (sf == nullptr || canonical == nullptr) return FP8MM_ERR_NULL;
  const int64_t nkb = k / 32;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < nkb; ++b) canonical[r * nkb + b] = sf[fp8mm_sf_offset(rows, k, r, b)];
  return FP8MM_OK;
}

fp8mm_status fp8mm_sf_from_canonical(const uint8_t* canonical, int64_t rows, int64_t k, uint8_t* sf) {
  if (rows < 0 || k < 0 || k % 32 != 0) return FP8MM_ERR_SHAPE;
  if (rows == 0 || k == 0) return FP8MM_OK;
  if (sf == nullptr || canonical == nullptr) return FP8MM_ERR_NULL;
  std::memset(sf, 0, fp8mm_sf_bytes(rows, k));
  const int64_t nkb = k / 32;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < nkb; ++b) sf[fp8mm_sf_offset(rows, k, r, b)] = canonical[r * nkb + b];
  return FP8MM_OK;
}

int32_t fp8mm_pair_split_plan(int64_t m, int64_t n, int64_t k, int32_t pairs, int32_t* dp_tiles) {
  if (m <= 0 || n <= 0 || k <= 0 || pairs <= 0) {
    if (dp_tiles != nullptr) *dp_tiles = 0;
    return 1;
  }
  const PairPlan plan = pair_plan(m, n, k, pairs);
  if (dp_tiles != nullptr) *dp_tiles = plan.dp_tiles;
  return plan.split;
}

size_t fp8mm_workspace_bytes(int64_t m, int64_t n, int64_t k, int32_t ctas) {
  if (m <= 0 || n <= 0 || k <= 0) return 0;
  int dev = 0, sms = 0;
  if (!(cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0))
    sms = 148;
  cudaGetLastError();  // a host without a GPU leaves an error behind
  if (m > 64) return pair_split_bytes(m, k, sms);
  int g = ctas > 0 ? ctas : sms;
  const int64_t units = cdiv(n, 128) * cdiv(k, 128);
  g = small_m_ctas(units, cdiv(n, 128), cdiv(k, 128), small_m_tile(m), ctas, g);
  const size_t tickets = static_cast<size_t>(cdiv(n, 128)) * sizeof(unsigned);
  return small_m_partials_bytes(g, small_m_tile(m)) + ((tickets + 255) & ~size_t(255));
}

fp8mm_status fp8_quantize_rowwise(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, void* q_e4m3,
                                  int64_t ld_q, float* scale, void* stream) {
  if (rows < 0 || k < 0 || k % 8 != 0) return FP8MM_ERR_SHAPE;
  if (rows == 0) return FP8MM_OK;
  if (scale == nullptr) return FP8MM_ERR_NULL;
  if (!aligned(scale, 4)) return FP8MM_ERR_ALIGN;
  if (k > 0) {  // with k == 0 only the scales are written (x and q are not touched)
    if (ld_x < k || ld_q < k) return FP8MM_ERR_SHAPE;
    if (x_bf16 == nullptr || q_e4m3 == nullptr) return FP8MM_ERR_NULL;
    if (!aligned(x_bf16, 16) || !aligned(q_e4m3, 8) || ld_x % 8 != 0 || ld_q % 8 != 0) return FP8MM_ERR_ALIGN;
  }
  DeviceInfo dev;
  fp8mm_status st = current_device(&dev);
  if (st != FP8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const auto* x = static_cast<const __nv_bfloat16*>(x_bf16);
  auto* q = static_cast<uint8_t*>(q_e4m3);
  const int64_t nvec = k / 8;
  if (nvec > static_cast<int64_t>(kQ1Threads) * 8) {
    const int grid = static_cast<int>(std::min<int64_t>(rows, static_cast<int64_t>(dev.sms) * 8));
    fp8mm_status st2 = launch_pdl(quant_rowwise_2pass_kernel, dim3(grid), dim3(kQ1Threads), 0, s, x, rows, k, ld_x,
                                  q, ld_q, scale);
    return st2 != FP8MM_OK ? st2 : launched();
  }
  const int threads = static_cast<int>(std::min<int64_t>(kQ1Threads, std::max<int64_t>(32, cdiv(nvec, 32) * 32)));
  const int64_t nv = cdiv(std::max<int64_t>(nvec, 1), threads);
  const int per_sm = 2048 / threads;
  const int grid = static_cast<int>(std::min<int64_t>(rows, static_cast<int64_t>(dev.sms) * per_sm));
  auto kern = nv <= 1 ? quant_rowwise_kernel<1>
              : nv <= 2 ? quant_rowwise_kernel<2>
              : nv <= 4 ? quant_rowwise_kernel<4>
                        : quant_rowwise_kernel<8>;
  st = launch_pdl(kern, dim3(grid), dim3(threads), 0, s, x, rows, k, ld_x, q, ld_q, scale);
  return st != FP8MM_OK ? st : launched();
}

fp8mm_status fp8_tensor_scale(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, float* scale,
                              void* stream) {
  if (rows < 0 || k < 0 || k % 8 != 0 || (k > 0 && ld_x < k)) return FP8MM_ERR_SHAPE;
  if (rows * (k / 8) > int64_t{0xFFFFFFFF}) return FP8MM_ERR_SHAPE;
  if (scale == nullptr || (rows > 0 && k > 0 && x_bf16 == nullptr)) return FP8MM_ERR_NULL;
  if (!aligned(scale, 4) || (rows > 0 && k > 0 && (!aligned(x_bf16, 16) || ld_x % 8 != 0))) return FP8MM_ERR_ALIGN;
  DeviceInfo dev;
  fp8mm_status st = current_device(&dev);
  if (st != FP8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_pdl(tensor_scale_zero_kernel, dim3(1), dim3(1), 0, s, reinterpret_cast<unsigned*>(scale));
  if (st != FP8MM_OK) return st;
  if (rows > 0 && k > 0) {
    // contiguous tensors are one flat run of vectors, strided ones go row by
    // row; at most eight blocks per SM
    const int64_t per_block = kTensorThreads * kAmaxUnroll;
    const int64_t want = ld_x == k ? cdiv(rows * (k / 8), per_block)
                                   : cdiv(rows, std::max<int64_t>(1, cdiv(per_block, k / 8)));
    const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(dev.sms) * 8));
    st = launch_pdl(tensor_amax_kernel, dim3(grid), dim3(kTensorThreads), 0, s,
                    static_cast<const __nv_bfloat16*>(x_bf16), rows, k, ld_x, reinterpret_cast<unsigned*>(scale));
    if (st != FP8MM_OK) return st;
  }
  st = launch_pdl(tensor_scale_finalize_kernel, dim3(1), dim3(1), 0, s, scale);
  return st != FP8MM_OK ? st : launched();
}

fp8mm_status fp8_quantize_static(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, const float* scale,
                                 void* q_e4m3, int64_t ld_q, void* stream) {
  if (rows < 0 || k < 0 || k % 8 != 0) return FP8MM_ERR_SHAPE;
  if (rows == 0 || k == 0) return FP8MM_OK;
  if (ld_x < k || ld_q < k || rows * (k / 8) > int64_t{0xFFFFFFFF}) return FP8MM_ERR_SHAPE;
  if (x_bf16 == nullptr || q_e4m3 == nullptr || scale == nullptr) return FP8MM_ERR_NULL;
  if (!aligned(x_bf16, 16) || !aligned(q_e4m3, 8) || !aligned(scale, 4) || ld_x % 8 != 0 || ld_q % 8 != 0)
    return FP8MM_ERR_ALIGN;
  DeviceInfo dev;
  fp8mm_status st = current_device(&dev);
  if (st != FP8MM_OK) return st;
  const int64_t vecs = rows * (k / 8);
  const int grid = static_cast<int>(std::min<int64_t>(cdiv(vecs, kTensorThreads), static_cast<int64_t>(dev.sms) * 8));
  st = launch_pdl(quant_static_kernel, dim3(grid), dim3(kTensorThreads), 0, static_cast<cudaStream_t>(stream),
                  static_cast<const __nv_bfloat16*>(x_bf16), rows, k, ld_x, scale, static_cast<uint8_t*>(q_e4m3), ld_q);
  return st != FP8MM_OK ? st : launched();
}

fp8mm_status mxfp8_quantize(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, void* q_e4m3, int64_t ld_q,
                            uint8_t* sf, void* stream) {
  if (rows < 0 || k < 0 || k % 32 != 0 || ld_x < k || ld_q < k) return FP8MM_ERR_SHAPE;
  if (rows == 0 || k == 0) return FP8MM_OK;
  if (x_bf16 == nullptr || q_e4m3 == nullptr || sf == nullptr) return FP8MM_ERR_NULL;
  if (!aligned(x_bf16, 16) || !aligned(q_e4m3, 8) || !aligned(sf, 16) || ld_x % 8 != 0 || ld_q % 8 != 0)
    return FP8MM_ERR_ALIGN;
  DeviceInfo dev;
  fp8mm_status st = current_device(&dev);
  if (st != FP8MM_OK) return st;
  const int64_t n_kc = cdiv(k, 128);
  // A few rows and a long K: one warp per (scale line, segment) instead of one
  // per (padded row, segment).  Measured on B200 before a decode GEMM (two
  // launches, CUDA-graph replay): 4096 x 14336 at m = 1 and 8 18.4 -> 17.2 us
  // and 18.5 -> 16.9 us, level at m = 32, 1.3 us slower at m = 64; at k = 4096
  // (fewer segments) it was 0.4-0.6 us slower, so it is used only for these.
  if (rows <= 32 && k >= 8192) {
    const int64_t tasks = 32 * cdiv(n_kc * 4, 32);
    st = launch_pdl(quant_mx_lines_kernel, dim3(static_cast<unsigned>(cdiv(tasks, kQ2Threads / 32))),
                    dim3(kQ2Threads), 0, static_cast<cudaStream_t>(stream),
                    static_cast<const __nv_bfloat16*>(x_bf16), static_cast<int>(rows), k, ld_x,
                    static_cast<uint8_t*>(q_e4m3), ld_q, sf, static_cast<int>(n_kc));
    return st != FP8MM_OK ? st : launched();
  }
  const int64_t rows_pad = cdiv(rows, 128) * 128;
  // one warp per 32-block segment of a padded row, 8 warps per CTA
  const int64_t segments = rows_pad * cdiv(cdiv(k, 128) * 4, 32);
  const int grid = static_cast<int>(std::min<int64_t>(cdiv(segments, kQ2Threads / 32), static_cast<int64_t>(dev.sms) * 8));
  st = launch_pdl(quant_mx_kernel<false>, dim3(grid), dim3(kQ2Threads), 0, static_cast<cudaStream_t>(stream),
                  static_cast<const __nv_bfloat16*>(x_bf16), rows, k, ld_x, static_cast<uint8_t*>(q_e4m3), ld_q, sf,
                  static_cast<int>(n_kc), rows_pad);
  return st != FP8MM_OK ? st : launched();
}

size_t fp8mm_sf8x4_bytes(int64_t rows, int64_t k) {
  if (rows <= 0 || k <= 0) return 0;
  return static_cast<size_t>(cdiv(rows, 8) * 8) * static_cast<size_t>(cdiv(k, 128)) * 4;
}

int64_t fp8mm_sf8x4_offset(int64_t rows, int64_t k, int64_t row, int64_t block) {
  if (rows <= 0 || k <= 0) return -1;
  const int64_t rows8 = cdiv(rows, 8) * 8;
  if (row < 0 || row >= rows8 || block < 0 || block >= cdiv(k, 128) * 4) return -1;
  return ((block / 4) * rows8 + row) * 4 + block % 4;
}

fp8mm_status mxfp8_quantize_8x4(const void* x_bf16, int64_t rows, int64_t k, int64_t ld_x, void* q_e4m3,
                                int64_t ld_q, uint8_t* sf, void* stream) {
  if (rows < 0 || k < 0 || k % 32 != 0 || ld_x < k || ld_q < k) return FP8MM_ERR_SHAPE;
  if (rows == 0 || k == 0) return FP8MM_OK;
  if (x_bf16 == nullptr || q_e4m3 == nullptr || sf == nullptr) return FP8MM_ERR_NULL;
  if (!aligned(x_bf16, 16) || !aligned(q_e4m3, 8) || !aligned(sf, 16) || ld_x % 8 != 0 || ld_q % 8 != 0)
    return FP8MM_ERR_ALIGN;
  DeviceInfo dev;
  fp8mm_status st = current_device(&dev);
  if (st != FP8MM_OK) return st;
  const int64_t n_kc = cdiv(k, 128);
  const int64_t rows_pad = cdiv(rows, 8) * 8;
  const int64_t segments = rows_pad * cdiv(n_kc * 4, 32);
  const int grid = static_cast<int>(std::min<int64_t>(cdiv(segments, kQ2Threads / 32), static_cast<int64_t>(dev.sms) * 8));
  st = launch_pdl(quant_mx_kernel<true>, dim3(grid), dim3(kQ2Threads), 0, static_cast<cudaStream_t>(stream),
                  static_cast<const __nv_bfloat16*>(x_bf16), rows, k, ld_x, static_cast<uint8_t*>(q_e4m3), ld_q, sf,
                  static_cast<int>(n_kc), rows_pad);
  return st != FP8MM_OK ? st : launched();
}

static fp8mm_status check_gemm_common(const void* a, const void* b, int64_t m, int64_t n, int64_t k, const void* c,
                                      int64_t ldc, int64_t k_granule, uintptr_t c_align = 2) {
  if (m < 0 || n < 0 || k < 0 || k % k_granule != 0 || ldc < n) return FP8MM_ERR_SHAPE;
  if (m > INT32_MAX / 2 || n > INT32_MAX / 2 || k > INT32_MAX / 2) return FP8MM_ERR_SHAPE;
  if (m == 0 || n == 0) return FP8MM_OK;
  if (c == nullptr || (k > 0 && (a == nullptr || b == nullptr))) return FP8MM_ERR_NULL;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(c, c_align)) return FP8MM_ERR_ALIGN;
  return FP8MM_OK;
}

static fp8mm_status zero_output(void* c, int64_t m, int64_t n, int64_t ldc, cudaStream_t s) {
  cudaError_t e = cudaMemset2DAsync(c, static_cast<size_t>(ldc) * 2, 0, static_cast<size_t>(n) * 2,
                                    static_cast<size_t>(m), s);
  return e == cudaSuccess ? FP8MM_OK : cuda_fail(e);
}

fp8mm_status fp8_gemm(const void* a_e4m3, const void* b_e4m3, int64_t m, int64_t n, int64_t k, const float* scale_a,
                      const float* scale_b, void* c_bf16, int64_t ldc, const fp8mm_opts* opt, void* stream) {
  fp8mm_status st = check_gemm_common(a_e4m3, b_e4m3, m, n, k, c_bf16, ldc, 16);
  if (st != FP8MM_OK || m == 0 || n == 0) return st;
  if (k > 0 && (scale_a == nullptr || scale_b == nullptr)) return FP8MM_ERR_NULL;
  if (!aligned(scale_a, 4) || !aligned(scale_b, 4)) return FP8MM_ERR_ALIGN;
  if (opt != nullptr && (opt->kernel == FP8MM_KERNEL_SMALL_M || opt->kernel < FP8MM_KERNEL_AUTO ||
                         opt->kernel > FP8MM_KERNEL_TILED_1SM_N128))
    return FP8MM_ERR_SHAPE;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != FP8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k == 0) return zero_output(c_bf16, m, n, ldc, s);
  const int kind = opt ? opt->kernel : FP8MM_KERNEL_AUTO;
  const int split = tiled_split(opt, kind, m, n, k, dev.sms);
  if (split < 0) return FP8MM_ERR_WORKSPACE;
  const Tiled tk = tiled_choice(kind, m, n, k, split > 0, dev.sms);
  if (tk == Tiled::kPair)
    return launch_pair(false, a_e4m3, b_e4m3, nullptr, nullptr, m, n, k, scale_a, scale_b, c_bf16, ldc, s, dev,
                       nullptr, nullptr, split > 0 ? opt->workspace : nullptr);
  return launch_tiled(false, a_e4m3, b_e4m3, nullptr, nullptr, m, n, k, scale_a, scale_b, c_bf16, ldc, s, dev,
                      nullptr, nullptr, tk == Tiled::k1SmN128);
}

fp8mm_status fp8_gemm_e4m3_out(const void* a_e4m3, const void* b_e4m3, int64_t m, int64_t n, int64_t k,
                               const float* scale_a, const float* scale_b, const float* scale_out, void* c_e4m3,
                               int64_t ldc, const fp8mm_opts* opt, void* stream) {
  fp8mm_status st = check_gemm_common(a_e4m3, b_e4m3, m, n, k, c_e4m3, ldc, 16, 1);
  if (st != FP8MM_OK || m == 0 || n == 0) return st;
  if (scale_out == nullptr || (k > 0 && (scale_a == nullptr || scale_b == nullptr))) return FP8MM_ERR_NULL;
  if (!aligned(scale_a, 4) || !aligned(scale_b, 4) || !aligned(scale_out, 4)) return FP8MM_ERR_ALIGN;
  if (opt != nullptr && (opt->kernel == FP8MM_KERNEL_SMALL_M || opt->kernel < FP8MM_KERNEL_AUTO ||
                         opt->kernel > FP8MM_KERNEL_TILED_1SM_N128))
    return FP8MM_ERR_SHAPE;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != FP8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k == 0) {  // C = 0 encodes to 0x00
    cudaError_t e = cudaMemset2DAsync(c_e4m3, static_cast<size_t>(ldc), 0, static_cast<size_t>(n),
                                      static_cast<size_t>(m), s);
    return e == cudaSuccess ? FP8MM_OK : cuda_fail(e);
  }
  auto* c8 = static_cast<uint8_t*>(c_e4m3);
  const int kind = opt ? opt->kernel : FP8MM_KERNEL_AUTO;
  const int split = tiled_split(opt, kind, m, n, k, dev.sms);
  if (split < 0) return FP8MM_ERR_WORKSPACE;
  const Tiled tk = tiled_choice(kind, m, n, k, split > 0, dev.sms);
  if (tk == Tiled::kPair)
    return launch_pair(false, a_e4m3, b_e4m3, nullptr, nullptr, m, n, k, scale_a, scale_b, nullptr, ldc, s, dev, c8,
                       scale_out, split > 0 ? opt->workspace : nullptr);
  return launch_tiled(false, a_e4m3, b_e4m3, nullptr, nullptr, m, n, k, scale_a, scale_b, nullptr, ldc, s, dev, c8,
                      scale_out, tk == Tiled::k1SmN128);
}

fp8mm_status mxfp8_gemm(const void* a_e4m3, const uint8_t* sf_a, const void* b_e4m3, const uint8_t* sf_b, int64_t m,
                        int64_t n, int64_t k, void* c_bf16, int64_t ldc, const fp8mm_opts* opt, void* stream) {
  fp8mm_status st = check_gemm_common(a_e4m3, b_e4m3, m, n, k, c_bf16, ldc, 32);
  if (st != FP8MM_OK || m == 0 || n == 0) return st;
  if (k > 0 && (sf_a == nullptr || sf_b == nullptr)) return FP8MM_ERR_NULL;
  if (!aligned(sf_a, 16) || !aligned(sf_b, 16)) return FP8MM_ERR_ALIGN;
  const int kind = opt ? opt->kernel : FP8MM_KERNEL_AUTO;
  if (kind == FP8MM_KERNEL_SMALL_M && m > 64) return FP8MM_ERR_SHAPE;
  if (kind < FP8MM_KERNEL_AUTO || kind > FP8MM_KERNEL_TILED_1SM_N128) return FP8MM_ERR_SHAPE;
  // the 8x4 activation-scale layout is read by the small-M kernel only
  if (opt != nullptr && (opt->flags & FP8MM_FLAG_SF_A_8X4) &&
      !(kind == FP8MM_KERNEL_SMALL_M || (kind == FP8MM_KERNEL_AUTO && m <= 64)))
    return FP8MM_ERR_SHAPE;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != FP8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k == 0) return zero_output(c_bf16, m, n, ldc, s);
  const bool small = (kind == FP8MM_KERNEL_SMALL_M) || (kind == FP8MM_KERNEL_AUTO && m <= 64);
  if (small) return launch_small_m(a_e4m3, sf_a, b_e4m3, sf_b, m, n, k, c_bf16, ldc, opt, s, dev);
  const int split = tiled_split(opt, kind, m, n, k, dev.sms);
  if (split < 0) return FP8MM_ERR_WORKSPACE;
  const Tiled tk = tiled_choice(kind, m, n, k, split > 0, dev.sms);
  if (tk == Tiled::kPair)
    return launch_pair(true, a_e4m3, b_e4m3, sf_a, sf_b, m, n, k, nullptr, nullptr, c_bf16, ldc, s, dev, nullptr,
                       nullptr, split > 0 ? opt->workspace : nullptr);
  return launch_tiled(true, a_e4m3, b_e4m3, sf_a, sf_b, m, n, k, nullptr, nullptr, c_bf16, ldc, s, dev, nullptr,
                      nullptr, tk == Tiled::k1SmN128);
}

// Largest m whose activation is quantized inside the small-M kernel; above it
// the per-CTA re-quantization of every K slab costs more than a separate
// quantizer launch, which then writes into the workspace.
constexpr int64_t kQuantInKernelMaxM = 8;

static size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

size_t fp8mm_quantize_gemm_workspace_bytes(int64_t m, int64_t n, int64_t k, int32_t ctas) {
  if (m <= 0 || n <= 0 || k <= 0 || m > 64) return 0;
  const size_t gemm = fp8mm_workspace_bytes(m, n, k, ctas);
  if (m <= kQuantInKernelMaxM) return gemm;
  return gemm + align256(static_cast<size_t>(m * k)) + align256(fp8mm_sf_bytes(m, k));
}

fp8mm_status mxfp8_quantize_gemm(const void* a_bf16, int64_t lda, const void* b_e4m3, const uint8_t* sf_b,
                                 int64_t m, int64_t n, int64_t k, void* c_bf16, int64_t ldc, const fp8mm_opts* opt,
                                 void* stream) {
  if (m > 64) return FP8MM_ERR_SHAPE;
  fp8mm_status st = check_gemm_common(a_bf16, b_e4m3, m, n, k, c_bf16, ldc, 32);
  if (st != FP8MM_OK || m == 0 || n == 0) return st;
  if (k > 0 && (lda < k || lda % 8 != 0)) return lda < k ? FP8MM_ERR_SHAPE : FP8MM_ERR_ALIGN;
  if (k > 0 && sf_b == nullptr) return FP8MM_ERR_NULL;
  if (!aligned(sf_b, 16)) return FP8MM_ERR_ALIGN;
  const int kind = opt ? opt->kernel : FP8MM_KERNEL_AUTO;
  if (kind != FP8MM_KERNEL_AUTO && kind != FP8MM_KERNEL_SMALL_M) return FP8MM_ERR_SHAPE;
  if (m > kQuantInKernelMaxM) {  // the quantized activation goes to the workspace tail
    if (opt == nullptr || opt->workspace == nullptr) return FP8MM_ERR_WORKSPACE;
    if (opt->workspace_bytes < fp8mm_quantize_gemm_workspace_bytes(m, n, k, opt->small_m_ctas) ||
        !aligned(opt->workspace, 256))
      return FP8MM_ERR_WORKSPACE;
  }
  DeviceInfo dev;
  if ((st = current_device(&dev)) != FP8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k == 0) return zero_output(c_bf16, m, n, ldc, s);
  if (m <= kQuantInKernelMaxM)
    return launch_small_m(a_bf16, nullptr, b_e4m3, sf_b, m, n, k, c_bf16, ldc, opt, s, dev, true, lda);
  uint8_t* tail = static_cast<uint8_t*>(opt->workspace) + fp8mm_workspace_bytes(m, n, k, opt->small_m_ctas);
  uint8_t* xq = tail;
  uint8_t* sfx = tail + align256(static_cast<size_t>(m * k));
  if ((st = mxfp8_quantize(a_bf16, m, k, lda, xq, k, sfx, stream)) != FP8MM_OK) return st;
  return launch_small_m(xq, sfx, b_e4m3, sf_b, m, n, k, c_bf16, ldc, opt, s, dev);
}

fp8mm_status concat_mla_k(const void* k_nope, const void* k_rope, void* k_out, int64_t num_tokens,
                          int64_t num_heads, int64_t nope_dim, int64_t rope_dim, int64_t elem_bytes,
                          int64_t nope_stride_t, int64_t nope_stride_h, int64_t rope_stride_t,
                          int64_t rope_stride_h, int64_t out_stride_t, int64_t out_stride_h, void* stream) {
  if (num_tokens < 0 || num_heads < 0 || nope_dim <= 0 || rope_dim <= 0) return FP8MM_ERR_SHAPE;
  if (elem_bytes != 1 && elem_bytes != 2) return FP8MM_ERR_SHAPE;
  if (num_tokens == 0 || num_heads == 0) return FP8MM_OK;
  const int64_t nope_b = nope_dim * elem_bytes, rope_b = rope_dim * elem_bytes;
  const int64_t row_chunks = (nope_b + rope_b) / 16;
  if (nope_b % 16 != 0 || rope_b % 16 != 0) return FP8MM_ERR_ALIGN;
  if (num_tokens * num_heads > (int64_t{1} << 31) || num_tokens * num_heads * row_chunks > int64_t{0xFFFFFFFF})
    return FP8MM_ERR_SHAPE;
  if (nope_stride_h < nope_dim || out_stride_h < nope_dim + rope_dim || rope_stride_h < 0 ||
      (rope_stride_h > 0 && rope_stride_h < rope_dim) || nope_stride_t < 0 || rope_stride_t < 0 ||
      out_stride_t < nope_dim + rope_dim)
    return FP8MM_ERR_SHAPE;
  if (k_nope == nullptr || k_rope == nullptr || k_out == nullptr) return FP8MM_ERR_NULL;
  const int64_t strides[6] = {nope_stride_t, nope_stride_h, rope_stride_t, rope_stride_h, out_stride_t, out_stride_h};
  for (int64_t st : strides)
    if ((st * elem_bytes) % 16 != 0) return FP8MM_ERR_ALIGN;
  if (!aligned(k_nope, 16) || !aligned(k_rope, 16) || !aligned(k_out, 16)) return FP8MM_ERR_ALIGN;
  DeviceInfo dev;
  fp8mm_status st = current_device(&dev);
  if (st != FP8MM_OK) return st;
  ConcatArgs p{};
  p.nope = static_cast<const uint8_t*>(k_nope);
  p.rope = static_cast<const uint8_t*>(k_rope);
  p.out = static_cast<uint8_t*>(k_out);
  p.heads = static_cast<uint32_t>(num_heads);
  p.nope_chunks = static_cast<uint32_t>(nope_b / 16);
  p.row_chunks = static_cast<uint32_t>(row_chunks);
  p.total_chunks = static_cast<uint32_t>(num_tokens * num_heads * row_chunks);
  p.nope_st = nope_stride_t * elem_bytes;
  p.nope_sh = nope_stride_h * elem_bytes;
  p.rope_st = rope_stride_t * elem_bytes;
  p.rope_sh = rope_stride_h * elem_bytes;
  p.out_st = out_stride_t * elem_bytes;
  p.out_sh = out_stride_h * elem_bytes;
  const int grid = static_cast<int>(
      std::min<int64_t>(cdiv(static_cast<int64_t>(p.total_chunks), kConcatThreads), static_cast<int64_t>(dev.sms) * 8));
  st = launch_pdl(concat_mla_k_kernel, dim3(grid), dim3(kConcatThreads), 0, static_cast<cudaStream_t>(stream), p);
  return st != FP8MM_OK ? st : launched();
}

unsigned int fp8mm_last_device_error(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    t_last_cuda_error = static_cast<int>(e);
    return 0xFFFFFFFFu;
  }
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
  const unsigned int zero = 0;
  cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  return v;
}

fp8mm_status fp8mm_selftest_wait_timeout(uint32_t timeout_us, void* stream) {
  DeviceInfo dev;
  fp8mm_status st = current_device(&dev);
  if (st != FP8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  selftest_wait_kernel<<<1, 32, 0, s>>>(static_cast<uint64_t>(timeout_us) * 1000ull);
  if ((st = launched()) != FP8MM_OK) return st;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  const unsigned int word = fp8mm_last_device_error();
  if (word == 0xFFFFFFFFu) return FP8MM_ERR_LAUNCH;
  return ((word & 0xFFu) == kDevErrTimeout && ((word >> 8) & 0xFFu) == kSiteSelfTest) ? FP8MM_ERR_DEVICE
                                                                                          : FP8MM_OK;
}

}  // extern "C"

// ====================================================================== no-allocation variant
// The small-M kernel with its split-K scratch in a fixed array inside the
// library, for callers that cannot allocate (see fp8mm.h).  Nothing above
// this point is changed by it.
namespace fp8mm {

constexpr size_t kNoAllocTicketBytes = size_t(64) << 10;  // one u32 per weight tile: 16384 tiles
constexpr size_t kNoAllocPartialBytes = size_t(FP8MM_NOALLOC_SCRATCH_BYTES) - kNoAllocTicketBytes;

// Partial sums first, arrival counters in the last 64 KiB.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FP8MM_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device, looked up once
// per device (host code may not use the symbol itself as a device pointer).
static fp8mm_status noalloc_scratch(int dev, unsigned char** out) {
  static unsigned char* addr[64] = {};
  if (dev < 0 || dev >= 64) return FP8MM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return cuda_fail(e == cudaSuccess ? cudaErrorInvalidSymbol : e);
    addr[dev] = static_cast<unsigned char*>(p);
  }
  *out = addr[dev];
  return FP8MM_OK;
}

}  // namespace fp8mm

extern "C" fp8mm_status mxfp8_gemm_small_m_noalloc(const void* a_e4m3, const uint8_t* sf_a, const void* b_e4m3,
                                                   const uint8_t* sf_b, int64_t m, int64_t n, int64_t k,
                                                   void* c_bf16, int64_t ldc, void* stream) {
  fp8mm_status st = check_gemm_common(a_e4m3, b_e4m3, m, n, k, c_bf16, ldc, 32);
  if (st != FP8MM_OK) return st;
  if (m > 64) return FP8MM_ERR_SHAPE;
  if (m == 0 || n == 0) return FP8MM_OK;
  if (k > 0 && (sf_a == nullptr || sf_b == nullptr)) return FP8MM_ERR_NULL;
  if (!aligned(sf_a, 16) || !aligned(sf_b, 16)) return FP8MM_ERR_ALIGN;
  const int64_t n_tiles = cdiv(n, 128);
  if (static_cast<size_t>(n_tiles) * sizeof(unsigned) > kNoAllocTicketBytes) return FP8MM_ERR_WORKSPACE;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != FP8MM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k == 0) return zero_output(c_bf16, m, n, ldc, s);
  unsigned char* scratch = nullptr;
  if ((st = noalloc_scratch(dev.device, &scratch)) != FP8MM_OK) return st;

  const int nm = small_m_tile(m);
  DecodeArgs p{};
  p.m = static_cast<int>(m);
  p.n = static_cast<int>(n);
  p.k = static_cast<int>(k);
  p.num_k = static_cast<int>(cdiv(k, 128));
  p.n_tiles = static_cast<int>(n_tiles);
  p.units = static_cast<int64_t>(p.n_tiles) * p.num_k;
  p.c = static_cast<__nv_bfloat16*>(c_bf16);
  p.ldc = ldc;
  p.sfw = sf_b;
  p.sfx = sf_a;
  p.n_kc = p.num_k;
  p.timeout_ns = wait_timeout_ns();
  // mxfp8_gemm's automatic CTA count, capped at what the partial-sum region
  // holds (2 slots of 128 x nm fp32 each)
  const int64_t per_cta = 2 * static_cast<int64_t>(nm) * 128 * static_cast<int64_t>(sizeof(float));
  int64_t g = small_m_ctas(p.units, p.n_tiles, p.num_k, nm, 0, dev.sms);
  g = std::min<int64_t>(g, static_cast<int64_t>(kNoAllocPartialBytes) / per_cta);
  g = std::max<int64_t>(1, std::min<int64_t>(g, p.units));
  p.ctas = static_cast<int>(g);
  p.cluster_s = cluster_split(g, p.n_tiles, p.num_k);  // tile-aligned: reduced in clusters, scratch unused
  p.partials = reinterpret_cast<float*>(scratch);
  p.tickets = reinterpret_cast<unsigned*>(scratch + kNoAllocPartialBytes);
  p.l2_ahead = small_m_l2_ahead(p.units, p.ctas, dev.sms);
  // the counters must start at zero; a previous call that stopped early may have left some set
  cudaError_t e = cudaMemsetAsync(p.tickets, 0, static_cast<size_t>(n_tiles) * sizeof(unsigned), s);
  if (e != cudaSuccess) return cuda_fail(e);

  CUtensorMap tw, tx;
  if ((st = make_map(&tw, b_e4m3, k, n, 128)) != FP8MM_OK) return st;
  if ((st = make_map(&tx, a_e4m3, k, m, nm)) != FP8MM_OK) return st;
  switch (nm) {
    case 16: return launch_small_m_t<16>(tw, tx, p, s, dev.device);
    case 32: return launch_small_m_t<32>(tw, tx, p, s, dev.device);
    case 48: return launch_small_m_t<48>(tw, tx, p, s, dev.device);
    default: return launch_small_m_t<64>(tw, tx, p, s, dev.device);
  }
}
