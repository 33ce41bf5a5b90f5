// Shared-input adapter products of a grouped forward at many tokens (QLoRA
// §2 Eq. 3 / §3 Eq. 5, T = s X L1 per linear): linears that read the same
// layer input X get one product T_cat = X [L1_a | L1_b | ...] (fp32,
// [M x R], R = the sum of their ranks), which t_scatter_kernel splits into
// each linear's T = s_i T_cat[:, off_i : off_i + r_i] as a bf16 hi/lo pair
// [M x 2 r_i] (hi = bf16(T), lo = bf16(T - hi)), the layout the linear's Y
// product and its backward read.
#pragma once

#include "common.cuh"

namespace qlora {

constexpr int kScatterMax = 8;

struct TScatterArgs {
  const float *t_cat;            // [M x R] fp32
  int64_t M;
  int R;                         // columns of t_cat
  int count;
  int off[kScatterMax + 1];      // first column of each linear; off[count] = R
  int r[kScatterMax];
  float s[kScatterMax];
  __nv_bfloat16 *T[kScatterMax]; // [M x 2 r_i] each
};

// One thread per T_cat element (grid-stride).  Launched as a programmatic
// dependent of the product that wrote T_cat.
__global__ void __launch_bounds__(256) t_scatter_kernel(const __grid_constant__ TScatterArgs a) {
  pdl_trigger();
  pdl_wait();
  const int64_t count = a.M * a.R;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = e / a.R;
    const int n = (int)(e - m * a.R);
    int i = 0;
#pragma unroll
    for (int k = 1; k < kScatterMax; ++k) i += (k < a.count && n >= a.off[k]) ? 1 : 0;
    const int c = n - a.off[i], r = a.r[i];
    const float v = a.s[i] * ld_dep_f32(a.t_cat + e);
    const __nv_bfloat16 hb = __float2bfloat16_rn(v);
    __nv_bfloat16 *t = a.T[i] + m * 2 * r;
    t[c] = hb;
    t[r + c] = __float2bfloat16_rn(v - __bfloat162float(hb));
  }
}

}  // namespace qlora
