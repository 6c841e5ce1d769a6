// kvcache.cuh -- FP8 key assembly for multi-head latent attention.
//
// concat_mla_k (page "[flashinfer] FlashInfer, FP8 지원으로 장문 컨텍스트 추론
// 성능을 극적으로 향상시키다", 코드 분석 items 1 and 3: the nope part of a
// key row and its rope part, 128 and 64 elements, concatenated per head):
//   k[t, h, 0:nope]         = k_nope[t, h, :]
//   k[t, h, nope:nope+rope] = k_rope[t, h, :]
// with k_rope's head stride allowed to be 0 (one rope vector per token,
// broadcast to every head, as multi-head latent attention stores it), for
// 1-byte (E4M3 / E5M2) or 2-byte (bf16 / fp16) elements: a pure copy, so the
// output bytes are the input bytes.  The page's kernel gives each
// (token, head) row one warp with 4- and 2-byte vectors per thread; here the
// output is cut into 16-byte chunks and each thread of the grid copies one
// chunk per step (coalesced 16-byte loads and stores; the rope chunks of a
// token are re-read by its heads from L1/L2).  The kernel is HBM-bound.
#pragma once

#include <cstdint>

#include "ptx.cuh"
#include "quant.cuh"

namespace fp8mm {

struct ConcatArgs {
  const uint8_t* nope;  // byte pointers; strides below are in bytes
  const uint8_t* rope;
  uint8_t* out;
  uint32_t heads;
  uint32_t nope_chunks;   // nope row bytes / 16
  uint32_t row_chunks;    // (nope + rope) row bytes / 16
  uint32_t total_chunks;  // tokens * heads * row_chunks (< 2^32)
  int64_t nope_st, nope_sh, rope_st, rope_sh, out_st, out_sh;
};

constexpr int kConcatThreads = 256;

__global__ void __launch_bounds__(kConcatThreads) concat_mla_k_kernel(const ConcatArgs p) {
  griddep_launch_dependents();
  griddep_wait();  // the inputs may be written by the preceding kernel
  const uint32_t stride = gridDim.x * kConcatThreads;
  for (uint32_t c = blockIdx.x * kConcatThreads + threadIdx.x; c < p.total_chunks; c += stride) {
    const uint32_t row = c / p.row_chunks;  // (token, head)
    const uint32_t j = c - row * p.row_chunks;
    const uint32_t t = row / p.heads;
    const uint32_t h = row - t * p.heads;
    const uint8_t* src = (j < p.nope_chunks)
                             ? p.nope + static_cast<int64_t>(t) * p.nope_st + static_cast<int64_t>(h) * p.nope_sh + j * 16
                             : p.rope + static_cast<int64_t>(t) * p.rope_st + static_cast<int64_t>(h) * p.rope_sh +
                                   (j - p.nope_chunks) * 16;
    const uint4 v = ld_stream_16(src);
    *reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(t) * p.out_st + static_cast<int64_t>(h) * p.out_sh +
                              j * 16) = v;
  }
}

}  // namespace fp8mm
