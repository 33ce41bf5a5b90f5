// Grouped rank-r products of the QLoRA linear: the backward's (QLoRA §3, the
// paragraph after Eq. 6: gradients flow to the adapter only)
//
//   G_i   = s_i dY_i L2_i^T          [M x r]   contraction over n_out
//   dL2_i = T_i^T dY_i               [r x N]   contraction over the tokens
//   dL1_i = X_i^T G_i                [K x r]   contraction over the tokens
//
// and the forward's adapter down-projection (§2 Eq. 3, §3 Eq. 5)
//
//   T_i   = s_i X_i L1_i             [M x r]   contraction over k_in
//
// Each is a skinny product that streams one big operand (dY or X) once; one
// launch per product spends a large share of its time in launch ramp, first
// loads and the last tiles' epilogue.  This kernel runs a list of such
// problems in ONE persistent launch:
//   - every problem is a set of 128-row output tiles (optionally split along
//     the reduction), and the units of all problems form one list, ordered by
//     decreasing length, which the CTAs walk in boustrophedon rounds
//     (CTA c takes unit kG + c in even rounds and kG + G - 1 - c in odd ones),
//     so the longest units are spread first and the rounds even out;
//   - the TMA ring, the MMA issue and the double-buffered TMEM accumulator run
//     across unit and problem boundaries without a pause;
//   - a problem may have several 2r-wide n-tiles, one per linear, over one
//     shared A operand: dL1 of linears that read the same X walks each
//     128-row strip of X^T for all of them on neighbouring CTAs, so the strip
//     comes from HBM once and from L2 for the rest.
// Split units write fp32 partials [split][rows][width]; rank_finalize_kernel
// sums every split problem of a launch in a fixed order, so the results do
// not depend on timing.
//
// The warp roles are those of tc_gemm_kernel: warp 0 loads A, warp 6 loads B,
// warp 1 allocates TMEM and issues tcgen05.mma, warps 2..5 drain the
// accumulator.  The MMA N (64 or 128), the operands' major-ness and the
// stage width (one or two 64-wide k-blocks per TMA box) are per problem.
#pragma once

#include <algorithm>
#include <climits>
#include <map>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "tc_gemm.cuh"

namespace qlora {

constexpr int kRankMaxProbs = 16;
constexpr int kRankMaxOuts = 16;
constexpr int kRankStages = 3;
constexpr int kRankAStage = 2 * kBM * kBK * 2;        // two k-blocks of 128 A rows: 32 KB
constexpr int kRankStageBytes = 2 * kRankAStage;      // + two k-blocks of up to 128 B rows
constexpr int kRankMnChunk = 2 * kBK * 128;           // a 64-wide MN-major chunk of 128 k-rows: 16 KB
constexpr int kRankTmemCols = 256;                    // two 128-column accumulators
constexpr int kRankBarBytes = 256;
constexpr int kRankSmemBytes = kRankStages * kRankStageBytes + kRankBarBytes + 1024;
static_assert(kRankSmemBytes <= 232448, "shared memory per CTA");

// One output: an n-tile of a problem.  D(i, j) goes to ptr + i*ld_row +
// j*ld_col (fp32, or bf16 with lo = bf16(v - hi) at +lo_off when lo_off > 0),
// scaled by alpha; a split problem writes unscaled partials to `part`.
struct RankOut {
  void *ptr;
  float *part;
  int64_t ld_row, ld_col, lo_off;
  float alpha;
  int out_f32;
};

struct RankProb {
  int rows;          // output rows (rows of A)
  int m_tiles, n_tiles;
  int bn;            // B rows per n-tile = MMA N: 64 or 128
  int ncols;         // valid output columns per n-tile, before the fold
  int fold;          // 0, or: output column j < fold is D(i, j) + D(i, j + fold)
  int nkb;           // 64-wide k-blocks of the reduction
  int splits, kb_per_split;
  int a_mn, b_mn;    // operand stored contiguous along the output rows / columns
  int wide;          // both maps are 3-D boxes of two k-blocks
  int unit0;         // first unit of this problem in the launch's list
  int out0;          // its n-tiles' outputs: out[out0 .. out0 + n_tiles)
};

struct RankArgs {
  int nprob, units, nout;
  RankProb prob[kRankMaxProbs];
  RankOut out[kRankMaxOuts];
  int *err;
};

struct RankMaps {
  CUtensorMap m[2 * kRankMaxProbs];   // A, B of problem p at 2p, 2p + 1
};

struct RankUnit {
  int p, mt, nt, split;
};

__host__ __device__ __forceinline__ RankUnit rank_unit(const RankArgs &a, int u) {
  RankUnit r;
  int p = 0;
  while (p + 1 < a.nprob && u >= a.prob[p + 1].unit0) ++p;
  const RankProb &q = a.prob[p];
  int l = u - q.unit0;
  r.p = p;
  r.nt = l % q.n_tiles;
  l /= q.n_tiles;
  r.mt = l % q.m_tiles;
  r.split = l / q.m_tiles;
  return r;
}

// The unit of CTA b of G in round k: boustrophedon over the grid.
__host__ __device__ __forceinline__ int rank_unit_at(int k, int G, int b) {
  return k * G + ((k & 1) ? (G - 1 - b) : b);
}

__device__ __forceinline__ int rank_unit_of(int k, int G) { return rank_unit_at(k, G, (int)blockIdx.x); }

// Store 32 consecutive columns col0.. of row `row` (values before alpha).
__device__ __forceinline__ void rank_store(const RankOut &o, const RankProb &q, int row, int col0, int width,
                                           int split, const float (&v)[32]) {
  if (q.splits > 1) {
    float *d = o.part + ((int64_t)split * q.rows + row) * width + col0;
    if (col0 + 32 <= width && (width & 3) == 0) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        reinterpret_cast<float4 *>(d)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < width) d[j] = v[j];
    }
    return;
  }
  const float alpha = o.alpha;
  if (o.out_f32) {
    float *d = reinterpret_cast<float *>(o.ptr);
    if (o.ld_col == 1 && col0 + 32 <= width && (o.ld_row & 3) == 0) {
      float4 *dst = reinterpret_cast<float4 *>(d + (int64_t)row * o.ld_row + col0);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(alpha * v[4 * j], alpha * v[4 * j + 1], alpha * v[4 * j + 2], alpha * v[4 * j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < width) d[(int64_t)row * o.ld_row + (int64_t)(col0 + j) * o.ld_col] = alpha * v[j];
    }
    return;
  }
  __nv_bfloat16 *d = reinterpret_cast<__nv_bfloat16 *>(o.ptr);
  const int64_t lo = o.lo_off;
  if (o.ld_col == 1 && col0 + 32 <= width && (o.ld_row & 7) == 0 && (lo & 7) == 0) {
    uint4 *dst = reinterpret_cast<uint4 *>(d + (int64_t)row * o.ld_row + col0);
    uint4 *dst_lo = reinterpret_cast<uint4 *>(d + (int64_t)row * o.ld_row + col0 + lo);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t w[4], wl[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float v0 = alpha * v[8 * j + 2 * h];
        const float v1 = alpha * v[8 * j + 2 * h + 1];
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
        w[h] = *reinterpret_cast<const uint32_t *>(&b2);
        const __nv_bfloat162 l2 = __floats2bfloat162_rn(v0 - __low2float(b2), v1 - __high2float(b2));
        wl[h] = *reinterpret_cast<const uint32_t *>(&l2);
      }
      dst[j] = make_uint4(w[0], w[1], w[2], w[3]);
      if (lo > 0) dst_lo[j] = make_uint4(wl[0], wl[1], wl[2], wl[3]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j < width) {
        const float x = alpha * v[j];
        const __nv_bfloat16 hb = __float2bfloat16_rn(x);
        const int64_t off = (int64_t)row * o.ld_row + (int64_t)(col0 + j) * o.ld_col;
        d[off] = hb;
        if (lo > 0) d[off + lo] = __float2bfloat16_rn(x - __bfloat162float(hb));
      }
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    rank_gemm_kernel(const __grid_constant__ RankMaps maps, const __grid_constant__ RankArgs p) {
  constexpr int S = kRankStages;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment: the 128B-swizzle pattern repeats every 8 rows of 128 B.
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + S * kRankStageBytes);
  uint64_t *empty_bar = full_bar + S;
  uint64_t *tfull_bar = empty_bar + S;    // [2]
  uint64_t *tempty_bar = tfull_bar + 2;   // [2]
  uint64_t *done_bar = tempty_bar + 2;    // [1]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  const int G = (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(full_bar + i), 2);   // the A and the B producer
      mbar_init(smem_u32(empty_bar + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(tfull_bar + i), 1);
      mbar_init(smem_u32(tempty_bar + i), 4);   // one arrive per epilogue warp
    }
    mbar_init(smem_u32(done_bar), 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane < 2 * p.nprob) tma_prefetch_desc(&maps.m[lane]);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kRankTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();
  pdl_wait();

  if (warp == 0 || warp == kProdBWarp) {
    // ------------------------------------------------------------ producers
    if (lane == 0) {
      const bool isA = warp == 0;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0;          // stages that received at least one load
      uint32_t last_parity = 0;   // parity of the last load issued into each stage
      bool ok = true;
      for (int k = 0; k * G < p.units && ok; ++k) {
        const int u = rank_unit_of(k, G);
        if (u >= p.units) continue;
        const RankUnit ru = rank_unit(p, u);
        const RankProb &q = p.prob[ru.p];
        const CUtensorMap *tm = &maps.m[2 * ru.p + (isA ? 0 : 1)];
        const int row0 = isA ? ru.mt * kBM : ru.nt * q.bn;
        const int kb0 = ru.split * q.kb_per_split;
        const int kb1 = min(q.nkb, kb0 + q.kb_per_split);
        const bool wide = q.wide != 0;
        const int mn = isA ? q.a_mn : q.b_mn;
        const int rows = isA ? kBM : q.bn;
        // a box is counted in full, also where it reaches past the range
        // (zero-filled out of bounds, or k-blocks the MMAs skip)
        const uint32_t bytes = (uint32_t)(wide ? 2 : 1) * (uint32_t)rows * 128u;
        for (int kb = kb0; kb < kb1; kb += wide ? 2 : 1) {
          if (!mbar_wait(smem_u32(empty_bar + stage), phase ^ 1, p.err, DEV_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(full_bar + stage);
          mbar_arrive_expect_tx(fb, bytes);
          const uint32_t dst = smem_u32(smem + stage * kRankStageBytes) + (isA ? 0u : (uint32_t)kRankAStage);
          if (wide) {
            // K-major maps {64 k, rows, k-blocks} land as [k-block][row][64];
            // MN-major maps {64 mn, k, 64-wide chunks} as [chunk][k][64].
            if (!mn) tma_load_3d(dst, tm, fb, 0, row0, kb);
            else tma_load_3d(dst, tm, fb, 0, kb * kBK, row0 >> 6);
          } else if (!mn) {
            tma_load_2d(dst, tm, fb, kb * kBK, row0);
          } else {
            for (int j = 0; j < rows / 64; ++j) tma_load_2d(dst + j * kRankMnChunk, tm, fb, row0 + 64 * j, kb * kBK);
          }
          used |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Never leave while a tensor copy may still be landing in shared memory.
      for (int i = 0; i < S; ++i) {
        if (!(used & (1u << i))) continue;
        if (!mbar_wait(smem_u32(full_bar + i), (last_parity >> i) & 1u, p.err, DEV_TIMEOUT_DRAIN)) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int t = 0;
      for (int k = 0; k * G < p.units && ok; ++k) {
        const int u = rank_unit_of(k, G);
        if (u >= p.units) continue;
        const RankUnit ru = rank_unit(p, u);
        const RankProb &q = p.prob[ru.p];
        const int acc = t & 1;
        const uint32_t use = (uint32_t)(t >> 1);
        ++t;
        if (!mbar_wait(smem_u32(tempty_bar + acc), (use & 1u) ^ 1u, p.err, DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 128);
        const uint32_t idesc = idesc_bf16_f32(kBM, q.bn, q.a_mn, q.b_mn);
        const int kb0 = ru.split * q.kb_per_split;
        const int kb1 = min(q.nkb, kb0 + q.kb_per_split);
        const int step = q.wide ? 2 : 1;
        const uint32_t b_kblock = q.b_mn ? 8192u : (uint32_t)q.bn * 128u;
        uint32_t accumulate = 0;
        for (int kb = kb0; kb < kb1; kb += step) {
          if (!mbar_wait(smem_u32(full_bar + stage), phase, p.err, DEV_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kRankStageBytes);
          const uint32_t sb = sa + kRankAStage;
          const int nk = min(step, kb1 - kb);
          for (int kk = 0; kk < nk; ++kk) {
            // K-major: k-block kk is the next [rows][64] tile and the 16-wide
            // k-slice starts 32 B into each swizzled row.  MN-major: k-block kk
            // starts 64 k-rows (8 KB) into each chunk, the k-slice 16 k-rows
            // (2 KB) further.
            const uint32_t ak = q.a_mn ? sa + kk * 8192u : sa + kk * (uint32_t)(kBM * 128);
            const uint32_t bk = sb + kk * b_kblock;
#pragma unroll
            for (int j = 0; j < kBK / 16; ++j) {
              const uint64_t ad = q.a_mn ? smem_desc_sw128(ak + j * 2048, kRankMnChunk, 1024)
                                         : smem_desc_sw128(ak + j * 32, 16, 1024);
              const uint64_t bd = q.b_mn ? smem_desc_sw128(bk + j * 2048, kRankMnChunk, 1024)
                                         : smem_desc_sw128(bk + j * 32, 16, 1024);
              tc_mma_f16(d_tmem, ad, bd, idesc, accumulate);
              accumulate = 1;
            }
          }
          tc_commit(smem_u32(empty_bar + stage));   // frees the stage once these MMAs have read it
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        tc_commit(smem_u32(tfull_bar + acc));   // accumulator ready for the epilogue
      }
      // All MMAs issued by this thread must finish before TMEM is released.
      tc_commit(smem_u32(done_bar));
      mbar_wait(smem_u32(done_bar), 0, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp < kProdBWarp) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    int t = 0;
    for (int k = 0; k * G < p.units; ++k) {
      const int u = rank_unit_of(k, G);
      if (u >= p.units) continue;
      const RankUnit ru = rank_unit(p, u);
      const RankProb &q = p.prob[ru.p];
      const int acc = t & 1;
      const uint32_t use = (uint32_t)(t >> 1);
      ++t;
      // Warp-uniform wait: tcgen05.ld below must be executed by all 32 lanes.
      const bool got = mbar_wait(smem_u32(tfull_bar + acc), use & 1u, p.err, DEV_TIMEOUT_EPILOGUE);
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      tc_fence_after();
      const RankOut &o = p.out[q.out0 + ru.nt];
      const int row = ru.mt * kBM + quarter * 32 + lane;
      const bool row_ok = row < q.rows;
      const uint32_t tb = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * 128);
      if (q.fold) {
        const int W = q.fold;
#pragma unroll 1
        for (int c = 0; c < (W < 32 ? 32 : W); c += 32) {
          uint32_t r[32];
          float v[32];
          tmem_ld_32x32b_x32(tb + (uint32_t)c, r);
          tmem_wait_ld();
          if (W >= 32) {
            uint32_t r2[32];
            tmem_ld_32x32b_x32(tb + (uint32_t)(c + W), r2);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) + __uint_as_float(r2[j]);
          } else if (W == 16) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = j < 16 ? __uint_as_float(r[j]) + __uint_as_float(r[j + 16]) : 0.f;
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = j < 8 ? __uint_as_float(r[j]) + __uint_as_float(r[j + 8]) : 0.f;
          }
          if (row_ok) rank_store(o, q, row, c, W, ru.split, v);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < q.bn; c += 32) {
          uint32_t r[32];
          float v[32];
          tmem_ld_32x32b_x32(tb + (uint32_t)c, r);
          tmem_wait_ld();
          if (!row_ok || c >= q.ncols) continue;
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          rank_store(o, q, row, c, q.ncols, ru.split, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(tempty_bar + acc));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kRankTmemCols);
}

// Fixed-order sum of the split partials of several problems of one launch.
struct RankFinJob {
  const float *part;   // [splits][rows][width] fp32
  void *out;
  int64_t ld_row, ld_col, lo_off;
  int64_t elem0;       // first element of this job in the launch's flat range
  int splits, rows, width, out_f32;
  float alpha;
};

struct RankFinArgs {
  int njobs;
  int64_t total;
  RankFinJob job[kRankMaxOuts];
};

__global__ void __launch_bounds__(256) rank_finalize_kernel(const __grid_constant__ RankFinArgs a) {
  pdl_trigger();
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < a.total; i += (int64_t)gridDim.x * blockDim.x) {
    int j = 0;
    while (j + 1 < a.njobs && i >= a.job[j + 1].elem0) ++j;
    const RankFinJob &f = a.job[j];
    const int64_t e = i - f.elem0;
    const int64_t count = (int64_t)f.rows * f.width;
    float s = 0.f;
    for (int k = 0; k < f.splits; ++k) s += ld_dep_f32(f.part + (int64_t)k * count + e);
    s *= f.alpha;
    const int64_t row = e / f.width, col = e - row * f.width;
    const int64_t off = row * f.ld_row + col * f.ld_col;
    if (f.out_f32) {
      reinterpret_cast<float *>(f.out)[off] = s;
    } else {
      __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(f.out);
      const __nv_bfloat16 hb = __float2bfloat16_rn(s);
      o[off] = hb;
      if (f.lo_off > 0) o[off + f.lo_off] = __float2bfloat16_rn(s - __bfloat162float(hb));
    }
  }
}


// ------------------------------------------------------------------ host side
// Scheduling of a launch, shared by the library's launcher and the host check
// of the walk (tests/host/rank_walk_check.cu).

// One problem as the planner sees it: its tiles (128-row tiles times n-tiles)
// and the 64-wide k-blocks of its reduction.
struct RankShape {
  int64_t m_tiles, tiles, nkb;
};

// Splits of each problem's reduction, chosen by simulating the kernel's walk:
// units in order of decreasing length, CTA c taking unit kG + c in even rounds
// and kG + G - 1 - c in odd ones.  A unit costs its k-blocks plus one (the
// hand-over between units); a split unit three more (its partial's store and
// the finalize's read, each 32 KB at r = 64 against 16 KB of A per k-block).
// The plan with the smallest largest CTA load wins.  Plans are cached by shape.
constexpr int kRankMinKb = 4;

inline void plan_rank(const RankShape *sh, int n, int sms, int *splits) {
  static std::mutex mu;
  static std::map<std::vector<int64_t>, std::vector<int>> cache;
  std::vector<int64_t> key{sms, n};
  for (int i = 0; i < n; ++i) key.insert(key.end(), {sh[i].tiles, sh[i].nkb});
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      std::copy(it->second.begin(), it->second.end(), splits);
      return;
    }
  }
  std::vector<int64_t> cand;
  for (int i = 0; i < n; ++i)
    for (int s = 1; s <= 32; ++s) {
      const int64_t L = (sh[i].nkb + s - 1) / s;
      if (L >= kRankMinKb || s == 1) cand.push_back(L);
    }
  std::sort(cand.begin(), cand.end());
  cand.erase(std::unique(cand.begin(), cand.end()), cand.end());
  std::vector<int> best(n, 1), cur(n);
  int64_t best_span = INT64_MAX, best_units = INT64_MAX;
  std::vector<int64_t> load;
  std::vector<std::pair<int64_t, int64_t>> runs;   // (cost, count), longest first
  for (int64_t L : cand) {
    runs.clear();
    int64_t units = 0;
    for (int i = 0; i < n; ++i) {
      int64_t s = std::max<int64_t>(1, (sh[i].nkb + L - 1) / L);
      const int64_t kbps = (sh[i].nkb + s - 1) / s;
      s = (sh[i].nkb + kbps - 1) / kbps;
      cur[i] = (int)s;
      runs.push_back({kbps + 1 + (s > 1 ? 3 : 0), sh[i].tiles * s});
      units += sh[i].tiles * s;
    }
    std::stable_sort(runs.begin(), runs.end(), [](auto &a, auto &b) { return a.first > b.first; });
    const int64_t G = std::max<int64_t>(1, std::min<int64_t>(units, sms));
    load.assign((size_t)G, 0);
    int64_t u = 0;
    for (auto &rc : runs)
      for (int64_t c = 0; c < rc.second; ++c, ++u) {
        const int64_t k = u / G, pos = u - k * G;
        load[(size_t)((k & 1) ? G - 1 - pos : pos)] += rc.first;
      }
    const int64_t span = *std::max_element(load.begin(), load.end());
    if (span < best_span || (span == best_span && units < best_units)) {
      best_span = span;
      best_units = units;
      best = cur;
    }
  }
  std::copy(best.begin(), best.end(), splits);
  std::lock_guard<std::mutex> lock(mu);
  cache.emplace(std::move(key), std::move(best));
}

// The order of the problems in a launch, as the plan assumed: longest units
// first (stable).  kbps receives each problem's k-blocks per split.
inline void rank_order(const RankShape *sh, const int *splits, int n, int64_t *kbps, int *order) {
  for (int i = 0; i < n; ++i) {
    kbps[i] = (sh[i].nkb + splits[i] - 1) / splits[i];
    order[i] = i;
  }
  std::stable_sort(order, order + n, [&](int a, int b) {
    return kbps[a] + (splits[a] > 1 ? 3 : 0) > kbps[b] + (splits[b] > 1 ? 3 : 0);
  });
}

}  // namespace qlora
