// Shared parts of the few-token forward (QLoRA §3 Eq. 5 at decode-sized M,
// up to 128 tokens): the LoRA branch around the fused doubleDequant product
// of decode_fwd.cuh, and the bookkeeping of a group of linears.
//
//   Y[M x N] = bf16( X W_hat^T + (s X L1) L2 )
//
// Three launches per call (one linear or a group of them), chained with
// programmatic dependent launch:
//   lora_down_small_kernel   adds K-slices of X L1 into an fp32 accumulator;
//   nf4_decode_fwd_kernel    streams the weight and adds X W_hat^T into an fp32
//                            [M x N] accumulator (decode_fwd.cuh; it does not
//                            need T, so it overlaps the first kernel);
//   lora_epilogue_kernel     Y = bf16(acc + s T L2), and T = s X L1 as a bf16
//                            hi/lo pair for the backward.
// The accumulators must be zero at launch (the host clears them with one
// memset in stream order).  The product's partial sums are added with
// red.global.add, so the low bits of Y depend on the order in which CTAs
// finish.
//
// Groups: one chain of the three launches may serve up to kMaxGroup linears
// that see the same tokens (GM > 1; e.g. the projections of a decoder layer
// that read its input, whose launch gaps and per-linear tails it removes).
// Their units (T slices, weight items, output column slices) are
// concatenated into one flat list per kernel; a unit finds its linear from
// the list's start offsets, then its place in that linear with a
// multiply-high by a divisor fixed at launch (DivU31).  A single linear is a
// group of one (GM = 1).
#pragma once

#include "common.cuh"

namespace qlora {

constexpr int kMaxGroup = 8;         // linears per group launch
constexpr int kFewMaxM = 128;        // tokens of the few-token forward

// The linear, among the `count` members of a group, of flat unit `u`:
// beg[i] is the first unit of member i (beg[0] = 0, increasing).
template <int GM>
__device__ __forceinline__ int group_member(const int (&beg)[GM], int count, int u) {
  int l = 0;
#pragma unroll
  for (int i = 1; i < GM; ++i) l += (i < count && u >= beg[i]) ? 1 : 0;
  return l;
}

// Division of n (0 <= n < 2^31) by a divisor d >= 1 fixed at launch, as a
// multiply-high and a shift (Granlund and Montgomery, "Division by invariant
// integers using multiplication", 1994): with l = ceil(log2 d) and
// mul = ceil(2^(31 + l) / d) (< 2^32 for d >= 2), n / d = umulhi(n, mul) >>
// (l - 1); mul = 0 stands for d = 1.
struct DivU31 {
  uint32_t mul, shr;
  __device__ __forceinline__ uint32_t div(uint32_t n) const { return mul ? (__umulhi(n, mul) >> shr) : n; }
};

inline DivU31 make_div_u31(uint32_t d) {
  DivU31 r = {0u, 0u};
  if (d <= 1) return r;
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  r.mul = (uint32_t)(((1ull << (31 + l)) + d - 1) / d);
  r.shr = l - 1;
  return r;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void red_add_f32(float *p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// T accumulation for few tokens: tacc[M x r] += X[:, k-slice] L1[k-slice, :]
// for a 64-wide K slice per CTA (blockIdx.x, flat over the group's linears)
// and a 64-wide column slice (blockIdx.y).  Inputs are staged in shared
// memory with coalesced loads (X in chunks of 32 tokens), then each thread
// forms 4 tokens x 1 column over the slice and adds it with red.global.add.
// Lets its dependent launch start immediately.
constexpr int kTSliceK = 64;
constexpr int kTokChunk = 32;

struct TdMember {
  const __nv_bfloat16 *X;    // [M x K]
  const __nv_bfloat16 *L1;   // [K x r]
  float *tacc;               // [M x r] fp32, zero at launch
  int K, r;
};

template <int GM>
struct TdArgs {
  int M, count;
  int beg[GM];               // first K slice of each linear
  TdMember m[GM];
};

template <int GM>
__global__ void __launch_bounds__(256) lora_down_small_kernel(const __grid_constant__ TdArgs<GM> a) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float xs[kTokChunk][kTSliceK + 1];
  __shared__ float ls[kTSliceK][65];
  const int l = group_member<GM>(a.beg, a.count, blockIdx.x);
  const TdMember &mb = a.m[l];
  const int K = mb.K, r = mb.r, M = a.M;
  const __nv_bfloat16 *__restrict__ X = mb.X;
  const __nv_bfloat16 *__restrict__ L1 = mb.L1;
  float *__restrict__ tacc = mb.tacc;
  const int k0 = (blockIdx.x - a.beg[l]) * kTSliceK;
  const int kn = min(kTSliceK, K - k0);
  const int j0 = blockIdx.y * 64;
  if (j0 >= r) return;       // a column slice beyond this linear's rank
  const int jn = min(64, r - j0);
  for (int i = threadIdx.x; i < kTSliceK * 64; i += blockDim.x) {
    const int k = i >> 6, jj = i & 63;
    ls[k][jj] = (k < kn && jj < jn) ? __bfloat162float(L1[(int64_t)(k0 + k) * r + j0 + jj]) : 0.f;
  }
  const int jj = threadIdx.x & 63;
  for (int mc = 0; mc < M; mc += kTokChunk) {
    const int mn = min(kTokChunk, M - mc);
    __syncthreads();   // ls staged; the previous chunk's xs no longer read
    for (int i = threadIdx.x; i < kTokChunk * kTSliceK; i += blockDim.x) {
      const int m = i / kTSliceK, k = i - m * kTSliceK;
      xs[m][k] = (m < mn && k < kn) ? __bfloat162float(X[(int64_t)(mc + m) * K + k0 + k]) : 0.f;
    }
    __syncthreads();
    for (int m0 = (threadIdx.x >> 6) * 4; m0 < mn; m0 += 16) {
      float t[4] = {0.f, 0.f, 0.f, 0.f};
      for (int k = 0; k < kn; ++k) {
        const float lv = ls[k][jj];
#pragma unroll
        for (int i = 0; i < 4; ++i) t[i] = __fmaf_rn(xs[m0 + i][k], lv, t[i]);
      }
      if (jj < jn) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (m0 + i < mn) red_add_f32(tacc + (mc + m0 + i) * r + j0 + jj, t[i]);
      }
    }
  }
}

// Y[tok][n] = bf16(acc[tok][n] + sum_j (s T)[tok][j] L2[j][n]).  A CTA owns 64
// columns (blockIdx.x, flat over the group's linears) of 32 tokens
// (blockIdx.y): it stages their L2 slice (r x 64) before waiting for the
// product kernel (L2 is an input), then s T of its tokens, then thread
// (column c, token group q) forms tokens q, q+4, ..., q+28.  Blocks of a
// linear's first column slice also write T = s X L1 of their tokens as a bf16
// hi/lo pair.  Launched as a programmatic dependent of the product kernel.
struct EpMember {
  const float *acc;          // [M x N] fp32
  const float *tacc;         // [M x r] fp32 (X L1, unscaled)
  const __nv_bfloat16 *L2;   // [r x N]
  __nv_bfloat16 *Y;          // [M x N]
  __nv_bfloat16 *T_save;     // [M x 2r] or null
  int N, r;
  float s;
};

template <int GM>
struct EpArgs {
  int M, count;
  int beg[GM];               // first column slice of each linear
  EpMember m[GM];
};

template <int GM>
__global__ void __launch_bounds__(256) lora_epilogue_kernel(const __grid_constant__ EpArgs<GM> a) {
  extern __shared__ float esm[];
  const int l = group_member<GM>(a.beg, a.count, blockIdx.x);
  const EpMember &me = a.m[l];
  const int M = a.M, N = me.N, r = me.r;
  const float s = me.s;
  const float *__restrict__ acc = me.acc;
  const float *__restrict__ tacc = me.tacc;
  const __nv_bfloat16 *__restrict__ L2 = me.L2;
  float *ts = esm;                                                        // [32 x r] s*T
  __nv_bfloat16 *l2s = reinterpret_cast<__nv_bfloat16 *>(esm + kTokChunk * r);  // [r x 64]
  const int slice = blockIdx.x - a.beg[l];
  const int nb = slice * 64;
  const int ncols = min(64, N - nb);
  const int mb = blockIdx.y * kTokChunk;
  const int mn = min(kTokChunk, M - mb);
  for (int i = threadIdx.x; i < r * 8; i += blockDim.x) {
    const int jj = i >> 3, c = i & 7;  // 16-byte chunk c of row jj of the slice
    uint4 v = make_uint4(0, 0, 0, 0);
    if (8 * c < ncols) v = __ldg(reinterpret_cast<const uint4 *>(L2 + (int64_t)jj * N + nb) + c);
    reinterpret_cast<uint4 *>(l2s + jj * 64)[c] = v;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = threadIdx.x; i < mn * r; i += blockDim.x) ts[i] = s * ld_dep_f32(tacc + (int64_t)mb * r + i);
  __syncthreads();
  if (slice == 0 && me.T_save) {
    __nv_bfloat16 *T_save = me.T_save;
    for (int i = threadIdx.x; i < mn * r; i += blockDim.x) {
      const float v = ts[i];
      const int m = mb + i / r, jj = i % r;
      const __nv_bfloat16 hb = __float2bfloat16_rn(v);
      T_save[(int64_t)m * 2 * r + jj] = hb;
      T_save[(int64_t)m * 2 * r + r + jj] = __float2bfloat16_rn(v - __bfloat162float(hb));
    }
  }
  const int c = threadIdx.x & 63, q = threadIdx.x >> 6;
  const int n = nb + c;
  if (c >= ncols) return;
  constexpr int kTok = kTokChunk / 4;
  float y[kTok];
#pragma unroll
  for (int i = 0; i < kTok; ++i) {
    const int m = q + 4 * i;
    y[i] = m < mn ? ld_dep_f32(acc + (int64_t)(mb + m) * N + n) : 0.f;
  }
  for (int jj = 0; jj < r; ++jj) {
    const float l2 = __bfloat162float(l2s[jj * 64 + c]);
#pragma unroll
    for (int i = 0; i < kTok; ++i) {
      const int m = q + 4 * i;
      if (m < mn) y[i] = __fmaf_rn(ts[m * r + jj], l2, y[i]);
    }
  }
  __nv_bfloat16 *Y = me.Y;
#pragma unroll
  for (int i = 0; i < kTok; ++i) {
    const int m = q + 4 * i;
    if (m < mn) Y[(int64_t)(mb + m) * N + n] = __float2bfloat16_rn(y[i]);
  }
}

}  // namespace qlora
