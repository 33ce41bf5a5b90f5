// Fused doubleDequant + product for few tokens (QLoRA §3 Eq. 5 / Eq. 6 at
// decode-sized M): the frozen-weight bytes dominate, so every NF4 weight is
// read once from HBM and decoded on the fly into tensor-core fragments -- no
// bf16 copy of the weight is ever written.
//
//   Y[M x N] = bf16( X W_hat^T + (s X L1) L2 ),   M <= 16*MT (MT in {1, 2})
//
// Three launches per linear, chained with programmatic dependent launch:
//   lora_down_small_kernel   adds K-slices of X L1 into an fp32 accumulator;
//   gemv_fwd_kernel          streams the weight and adds X W_hat^T into an fp32
//                            [M x N] accumulator (does not need T, so it
//                            overlaps the first kernel completely);
//   gemv_epilogue_kernel     Y = bf16(acc + s T L2), and T = s X L1 as a bf16
//                            hi/lo pair for the backward.
//
// gemv_fwd_kernel: persistent, 160 threads per CTA, 2 CTAs per SM.
//   * Operands: mma.sync m16n8k16 (bf16 in, fp32 accumulate) with the tokens
//     as the A operand (16 per tile) and the weight as the B operand (8 output
//     features per tile), so one X fragment feeds 8 weight tiles.
//   * Warp 4 (producer): per stage, 64 weight rows x 256 K of packed codes
//     (TMA, 128-byte swizzle), the X tile ([token][64-block][64], TMA 3-D,
//     128-byte swizzle) and the 64 x 4 block constants
//     c2_hat = fma(E4M3(code8), c1, mean) computed by its lanes into shared
//     memory; the stage's mbarrier completes on the TMA bytes plus the
//     constants' arrival.
//   * Warp w in 0..3 (consumers) takes 64-block w of every stage for all 64
//     rows.  Decode: each byte of codes is two consecutive weights; it indexes
//     a 256-entry shared table of bf16x2 (NF4[lo nibble], NF4[hi nibble]),
//     replicated once per lane so every lookup is bank-conflict free, and the
//     entry is directly a B-fragment register.  The block constant is applied
//     in fp32 after the block's four MMAs (per-block partial accumulators):
//     Y = sum_b c2_hat_b (X_b . bf16(NF4[codes_b])).  This equals X W_hat^T up
//     to bf16 rounding placement: the constant multiplies in fp32 instead of
//     being folded into a bf16 weight first.
//   * K inside a block is permuted identically for A and B: lane column j,
//     k-step s, slot u <-> k = 16 j + 4 s + u, so a lane's codes of a row are
//     one 8-byte run per block and its X operand one 32-byte run.
//   * A unit is 64 rows x 512 K (2 stages).  The four warps' partial sums are
//     reduced through shared memory and added into the fp32 [M x N]
//     accumulator with red.global.add (L2 resident).
// The two accumulators must be zero at launch (the host clears them with one
// memset in stream order).  Split-K additions make the low bits of Y depend
// on the order in which CTAs finish.
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace qlora {

constexpr int kGvRows = 64;          // weight rows per stage / unit
constexpr int kGvStageK = 256;       // K per pipeline stage (4 blocks of 64)
constexpr int kGvUnitK = 512;        // K per unit (2 stages)
constexpr int kGvThreads = 160;      // 4 decode/MMA warps + 1 producer warp
constexpr int kGvMaxM = 32;
constexpr int kGvLutBytes = 256 * 32 * 4;   // 256 entries x 32 lane copies x bf16x2

template <int MT>
struct GvCfg {
  static constexpr int kCodeBytes = kGvRows * 128;          // 64 rows x 256 codes
  static constexpr int kXBytes = 16 * MT * kGvStageK * 2;   // 16*MT tokens x 256 bf16
  static constexpr int kScaleBytes = 4 * kGvRows * 4;       // [block][row] fp32
  static constexpr int kStageBytes = kCodeBytes + kXBytes + kScaleBytes;
  static constexpr int kStages = MT == 1 ? 3 : 2;
  static constexpr int kRedBytes = 4 * 32 * 32 * MT * 4;    // per-warp partials, 32 lanes x 32*MT floats
  static constexpr int kSmemBytes = kGvLutBytes + kStages * kStageBytes + kRedBytes + 256 + 1024;
};

struct GvArgs {
  int M, N, K, r;
  int nks;               // units per 64-row block
  int units;
  float s;
  const uint8_t *c2_fp8;
  const float *c1;
  const float *mu;
  const __nv_bfloat16 *L2;   // [r x N]
  float *acc;            // [M x N] fp32, zero at launch
  int *err;
};

// D += A * B, or D = A * B when `zero` (C read as 0).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void red_add_f32(float *p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// bf16x2 decode of one byte of codes through the lane's copy of the table:
// entry b sits at lut + (b * 32 + lane) * 4.
__device__ __forceinline__ uint32_t lut_decode(uint32_t lane_base, uint32_t word, int byte) {
  const uint32_t b = __byte_perm(word, 0u, 0x4440 + byte);   // zero-extended byte
  return lds32(lane_base + b * 128u);
}

// Raw block constants of one stage for one producer lane: rows lane and
// lane + 32 of the 64-row tile, the stage's 4 blocks.
struct GvConsts {
  uint32_t code8[8];
  float c1[8];
  __device__ __forceinline__ void load(const GvArgs &p, int u, int st, int lane, int kblocks) {
    int rb = 0, kb0 = 0;
    const bool live = u < p.units;
    if (live) {
      rb = u / p.nks;
      const int ks = u - rb * p.nks;
      kb0 = (ks * kGvUnitK + st * kGvStageK) >> 6;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = rb * kGvRows + lane + 32 * (i >> 2);
      const int kb = kb0 + (i & 3);
      code8[i] = 0;
      c1[i] = 0.f;
      if (live && row < p.N && kb < kblocks) {
        const int64_t b = (int64_t)row * kblocks + kb;
        code8[i] = __ldg(p.c2_fp8 + b);
        c1[i] = __ldg(p.c1 + (b >> 8));
      }
    }
  }
};

template <int MT>
struct GvProducer {
  using Cfg = GvCfg<MT>;
  const GvArgs *p;
  uint8_t *stage_base;
  uint64_t *full_bar, *empty_bar;
  const CUtensorMap *tmCodes, *tmX;
  int kblocks, lane, stage, u, st;
  uint32_t phase, used, last_parity;
  float mu;

  __device__ __forceinline__ void init(const GvArgs &pp, uint8_t *sb, uint64_t *fb, uint64_t *eb,
                                       const CUtensorMap *tc, const CUtensorMap *tx, int kb) {
    p = &pp;
    stage_base = sb;
    full_bar = fb;
    empty_bar = eb;
    tmCodes = tc;
    tmX = tx;
    kblocks = kb;
    lane = lane_id();
    stage = 0;
    phase = used = last_parity = 0;
    u = blockIdx.x;
    st = 0;
    mu = __ldg(pp.mu);
  }

  // Issue item (u, st) whose constants are in `cur`; start loading the next
  // item's constants into `nxt`.  Returns false on a pipeline timeout.
  __device__ __forceinline__ bool item(const GvConsts &cur, GvConsts &nxt) {
    const GvArgs &P = *p;
    const int rb = u / P.nks, ks = u - rb * P.nks;
    const int kbeg = ks * kGvUnitK;
    const int nst = min(kGvUnitK, P.K - kbeg) > kGvStageK ? 2 : 1;
    int nu = u, nstn = st + 1;
    if (nstn == nst) {
      nu = u + gridDim.x;
      nstn = 0;
    }
    nxt.load(P, nu, nstn, lane, kblocks);
    const int k0 = kbeg + st * kGvStageK;
    bool got = true;
    if (lane == 0) {
      got = mbar_wait(smem_u32(empty_bar + stage), phase ^ 1, P.err, DEV_TIMEOUT_PRODUCER);
      if (got) {
        const uint32_t fb = smem_u32(full_bar + stage);
        mbar_arrive_expect_tx(fb, Cfg::kCodeBytes + Cfg::kXBytes);
        const uint32_t sc = smem_u32(stage_base + stage * Cfg::kStageBytes);
        tma_load_2d(sc, tmCodes, fb, k0 >> 1, rb * kGvRows);
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
            "[%2];" ::"r"(sc + Cfg::kCodeBytes),
            "l"(reinterpret_cast<uint64_t>(tmX)), "r"(fb), "r"(0), "r"(k0 >> 6), "r"(0)
            : "memory");
        used |= 1u << stage;
        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
      }
    }
    if (!__shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0)) return false;
    // block constants -> [block][row] fp32 of the stage (free: the empty wait above)
    float *scales = reinterpret_cast<float *>(stage_base + stage * Cfg::kStageBytes + Cfg::kCodeBytes + Cfg::kXBytes);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      scales[(i & 3) * kGvRows + lane + 32 * (i >> 2)] = __fmaf_rn(e4m3_to_f32((uint8_t)cur.code8[i]), cur.c1[i], mu);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(full_bar + stage));   // constants in place
    if (++stage == Cfg::kStages) {
      stage = 0;
      phase ^= 1;
    }
    u = nu;
    st = nstn;
    return true;
  }

  // Never leave the CTA while a tensor copy is still landing in shared memory.
  __device__ __forceinline__ void drain() {
    if (lane == 0)
      for (int i = 0; i < Cfg::kStages; ++i)
        if (used & (1u << i))
          mbar_wait(smem_u32(full_bar + i), (last_parity >> i) & 1u, p->err, DEV_TIMEOUT_DRAIN);
  }
};

template <int MT>
__global__ void __launch_bounds__(kGvThreads, 2)
    gemv_fwd_kernel(const __grid_constant__ CUtensorMap tmCodes, const __grid_constant__ CUtensorMap tmX,
                    const __grid_constant__ GvArgs p) {
  using Cfg = GvCfg<MT>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *stage_base = smem + kGvLutBytes;                       // 1024-aligned (LUT is 32 KB)
  float *red = reinterpret_cast<float *>(stage_base + S * Cfg::kStageBytes);
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(red) + Cfg::kRedBytes);
  uint64_t *empty_bar = full_bar + S;

  const int warp = warp_id();
  const int lane = lane_id();
  const int kblocks = p.K >> 6;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the epilogue may launch and wait

  // the byte -> (NF4[lo], NF4[hi]) bf16x2 table, one copy per lane
  {
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
    for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
      const int b = i >> 5;
      const __nv_bfloat162 v = __floats2bfloat162_rn(kNF4[b & 15], kNF4[b >> 4]);
      lut[i] = *reinterpret_cast<const uint32_t *>(&v);
    }
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(full_bar + i), 2);   // TMA (with tx) + constants
      mbar_init(smem_u32(empty_bar + i), 4);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmCodes);
      tma_prefetch_desc(&tmX);
    }
    GvProducer<MT> pr;
    pr.init(p, stage_base, full_bar, empty_bar, &tmCodes, &tmX, kblocks);
    // Flat walk over (unit, stage) items, unrolled by two: the block constants
    // of the next item load into the other register set while this one is
    // issued, so their latency never stalls the ring.
    GvConsts ca, cb;
    ca.load(p, pr.u, pr.st, lane, kblocks);
    while (pr.u < p.units) {
      if (!pr.item(ca, cb)) break;
      if (pr.u >= p.units || !pr.item(cb, ca)) break;
    }
    pr.drain();
  } else {
    // ------------------------------------------------------------ consumers
    const int g = lane >> 2, j = lane & 3;
    const uint32_t lane_base = smem_u32(smem) + lane * 4;
    int stage = 0;
    uint32_t phase = 0;
    float acc[8][MT][4];
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      const int rb = u / p.nks, ks = u - rb * p.nks;
      const int kbeg = ks * kGvUnitK;
      const int nst = min(kGvUnitK, p.K - kbeg) > kGvStageK ? 2 : 1;
#pragma unroll
      for (int t = 0; t < 8; ++t)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[t][m][0] = acc[t][m][1] = acc[t][m][2] = acc[t][m][3] = 0.f;
      for (int st = 0; st < nst; ++st) {
        if (!mbar_wait(smem_u32(full_bar + stage), phase, p.err, DEV_TIMEOUT_MMA)) {
          ok = false;
          break;
        }
        const uint32_t sc = smem_u32(stage_base + stage * Cfg::kStageBytes);
        const uint32_t sx = sc + Cfg::kCodeBytes;
        const uint32_t ss = sx + Cfg::kXBytes;
        // A fragments of block `warp` for its 4 k-steps: tokens g (+16m) and g+8 (+16m),
        // X[tok][16j .. 16j+15] = chunks 2j, 2j+1 of line (tok*4 + warp)
        uint32_t afr[MT][4][4];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          uint4 x[2][2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int line = (g + 8 * hh + 16 * m) * 4 + warp;
#pragma unroll
            for (int c = 0; c < 2; ++c) x[hh][c] = lds128(sx + line * 128 + (((2 * j + c) ^ (line & 7)) << 4));
          }
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint4 &lo = x[0][s >> 1], &hi = x[1][s >> 1];
            afr[m][s][0] = (s & 1) ? lo.z : lo.x;   // token g,   k 4s+0..1
            afr[m][s][1] = (s & 1) ? hi.z : hi.x;   // token g+8, k 4s+0..1
            afr[m][s][2] = (s & 1) ? lo.w : lo.y;   // token g,   k 4s+2..3
            afr[m][s][3] = (s & 1) ? hi.w : hi.y;   // token g+8, k 4s+2..3
          }
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          // codes of row 8t+g in block `warp`: bytes [8j, 8j+8) = 16 weights
          const int row = 8 * t + g;
          const uint32_t boff = warp * 32 + j * 8;             // byte offset in the 128-byte line
          const uint2 cw = lds64(sc + row * 128 + ((((boff >> 4)) ^ (row & 7)) << 4) + (boff & 15));
          // block constants of rows 8t+2j, 8t+2j+1 (the D fragment's columns)
          const uint2 sv = lds64(ss + (warp * kGvRows + 8 * t + 2 * j) * 4);
          uint32_t bfr[8];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            bfr[b] = lut_decode(lane_base, cw.x, b);
            bfr[4 + b] = lut_decode(lane_base, cw.y, b);
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            float pd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s = 0; s < 4; ++s) mma_bf16_16816(pd, afr[m][s], bfr[2 * s], bfr[2 * s + 1]);
            const float s0 = __uint_as_float(sv.x), s1 = __uint_as_float(sv.y);
            acc[t][m][0] = __fmaf_rn(s0, pd[0], acc[t][m][0]);
            acc[t][m][1] = __fmaf_rn(s1, pd[1], acc[t][m][1]);
            acc[t][m][2] = __fmaf_rn(s0, pd[2], acc[t][m][2]);
            acc[t][m][3] = __fmaf_rn(s1, pd[3], acc[t][m][3]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(empty_bar + stage));
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      // reduce the four warps' partial sums and add them into the accumulator
      float *myred = red + (warp * 32 + lane) * (32 * MT);
#pragma unroll
      for (int t = 0; t < 8; ++t)
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int v = 0; v < 4; ++v) myred[(t * MT + m) * 4 + v] = acc[t][m][v];
      named_bar_sync(1, 128);
      // thread (lane', warp') sums element e = warp'*8*MT .. of lane' across the 4 warps
      for (int e = warp * 8 * MT; e < (warp + 1) * 8 * MT; ++e) {
        float v = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < 4; ++w2) v += red[(w2 * 32 + lane) * (32 * MT) + e];
        const int t = e / (4 * MT), m = (e / 4) % MT, q = e & 3;
        const int tok = 16 * m + g + ((q & 2) ? 8 : 0);
        const int row = rb * kGvRows + 8 * t + 2 * j + (q & 1);
        if (tok < p.M && row < p.N) red_add_f32(p.acc + (int64_t)tok * p.N + row, v);
      }
      named_bar_sync(1, 128);
    }
  }
  // Complete only after the T launch this grid overlapped has completed, so
  // that the epilogue launched after this grid sees T.
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// T accumulation for few tokens: tacc[M x r] += X[:, k-slice] L1[k-slice, :]
// for a 64-wide K slice per CTA (blockIdx.x) and a 64-wide column slice
// (blockIdx.y).  Inputs are staged in shared memory with coalesced loads, then
// each thread forms 4 tokens x 1 column over the slice and adds it with
// red.global.add.  Lets its dependent launch start immediately.
constexpr int kTSliceK = 64;

__global__ void __launch_bounds__(256) lora_down_small_kernel(const __nv_bfloat16 *__restrict__ X,
                                                              const __nv_bfloat16 *__restrict__ L1, int M, int K,
                                                              int r, float *__restrict__ tacc) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float xs[kGvMaxM][kTSliceK + 1];
  __shared__ float ls[kTSliceK][65];
  const int k0 = blockIdx.x * kTSliceK;
  const int kn = min(kTSliceK, K - k0);
  const int j0 = blockIdx.y * 64;
  const int jn = min(64, r - j0);
  for (int i = threadIdx.x; i < kGvMaxM * kTSliceK; i += blockDim.x) {
    const int m = i / kTSliceK, k = i - m * kTSliceK;
    xs[m][k] = (m < M && k < kn) ? __bfloat162float(X[(int64_t)m * K + k0 + k]) : 0.f;
  }
  for (int i = threadIdx.x; i < kTSliceK * 64; i += blockDim.x) {
    const int k = i >> 6, jj = i & 63;
    ls[k][jj] = (k < kn && jj < jn) ? __bfloat162float(L1[(int64_t)(k0 + k) * r + j0 + jj]) : 0.f;
  }
  __syncthreads();
  const int jj = threadIdx.x & 63;
  for (int m0 = (threadIdx.x >> 6) * 4; m0 < M; m0 += 16) {
    float t[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < kn; ++k) {
      const float l = ls[k][jj];
#pragma unroll
      for (int i = 0; i < 4; ++i) t[i] = __fmaf_rn(xs[m0 + i][k], l, t[i]);
    }
    if (jj < jn) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (m0 + i < M) red_add_f32(tacc + (m0 + i) * r + j0 + jj, t[i]);
    }
  }
}

// Y[tok][n] = bf16(acc[tok][n] + sum_j (s T)[tok][j] L2[j][n]).  A CTA owns 64
// columns: it stages their L2 slice (r x 64) before waiting for the product
// kernel (L2 is an input), then s T, then thread (column c, token group q)
// forms tokens q, q+4, q+8, ...  Block 0 also writes T = s X L1 as a bf16
// hi/lo pair.  Launched as a programmatic dependent of gemv_fwd_kernel.
__global__ void __launch_bounds__(256) gemv_epilogue_kernel(const float *__restrict__ acc,
                                                            const float *__restrict__ tacc,
                                                            const __nv_bfloat16 *__restrict__ L2, int M, int N, int r,
                                                            float s, __nv_bfloat16 *__restrict__ Y,
                                                            __nv_bfloat16 *__restrict__ T_save) {
  extern __shared__ float esm[];
  float *ts = esm;                                                 // [M x r] s*T
  __nv_bfloat16 *l2s = reinterpret_cast<__nv_bfloat16 *>(esm + M * r);  // [r x 64]
  const int nb = blockIdx.x * 64;
  const int ncols = min(64, N - nb);
  for (int i = threadIdx.x; i < r * 8; i += blockDim.x) {
    const int jj = i >> 3, c = i & 7;  // 16-byte chunk c of row jj of the slice
    uint4 v = make_uint4(0, 0, 0, 0);
    if (8 * c < ncols) v = __ldg(reinterpret_cast<const uint4 *>(L2 + (int64_t)jj * N + nb) + c);
    reinterpret_cast<uint4 *>(l2s + jj * 64)[c] = v;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = threadIdx.x; i < M * r; i += blockDim.x) ts[i] = s * __ldcg(tacc + i);
  __syncthreads();
  if (blockIdx.x == 0 && T_save) {
    for (int i = threadIdx.x; i < M * r; i += blockDim.x) {
      const float v = ts[i];
      const int m = i / r, jj = i - m * r;
      const __nv_bfloat16 hb = __float2bfloat16_rn(v);
      T_save[(int64_t)m * 2 * r + jj] = hb;
      T_save[(int64_t)m * 2 * r + r + jj] = __float2bfloat16_rn(v - __bfloat162float(hb));
    }
  }
  const int c = threadIdx.x & 63, q = threadIdx.x >> 6;
  const int n = nb + c;
  if (c >= ncols) return;
  constexpr int kTok = kGvMaxM / 4;
  float y[kTok];
#pragma unroll
  for (int i = 0; i < kTok; ++i) {
    const int m = q + 4 * i;
    y[i] = m < M ? __ldcg(acc + (int64_t)m * N + n) : 0.f;
  }
  for (int jj = 0; jj < r; ++jj) {
    const float l2 = __bfloat162float(l2s[jj * 64 + c]);
#pragma unroll
    for (int i = 0; i < kTok; ++i) {
      const int m = q + 4 * i;
      if (m < M) y[i] = __fmaf_rn(ts[m * r + jj], l2, y[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < kTok; ++i) {
    const int m = q + 4 * i;
    if (m < M) Y[(int64_t)m * N + n] = __float2bfloat16_rn(y[i]);
  }
}

}  // namespace qlora
