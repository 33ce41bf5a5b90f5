// LoRA dropout on the adapter input (QLoRA Appendix B.2 trains with LoRA
// dropout; it acts on the input of the adapter only):
//   drop(X) = X * m / (1 - p),  m the caller's keep mask.
// The masked copy Xm = X * m is exact in bf16; the 1/(1 - p) factor is folded
// into the scale of the products that read Xm.
//
// Mask layout: uint32 words over the row-major [M x K] elements, bit b of
// word w keeps element 32 w + b (K a multiple of 32, so a word never spans
// two rows).
#pragma once

#include "common.cuh"

namespace qlora {

// Xm = X * m, eight bf16 elements (one 16-byte load and store) per thread.
__global__ void __launch_bounds__(256) dropout_mask_kernel(const uint16_t *__restrict__ X,
                                                           const uint32_t *__restrict__ mask, int64_t numel,
                                                           uint16_t *__restrict__ Xm) {
  pdl_trigger();
  pdl_wait();
  const int64_t n8 = numel >> 3;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n8; e += stride) {
    const uint4 x = ld_dep_v4(X + 8 * e);
    const uint32_t bits = (ld_dep_u32(mask + (e >> 2)) >> (8 * (int)(e & 3))) & 0xFFu;
    uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint32_t keep = (((bits >> (2 * h)) & 1u) ? 0x0000FFFFu : 0u) | (((bits >> (2 * h + 1)) & 1u) ? 0xFFFF0000u : 0u);
      w[h] &= keep;
    }
    reinterpret_cast<uint4 *>(Xm)[e] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace qlora
