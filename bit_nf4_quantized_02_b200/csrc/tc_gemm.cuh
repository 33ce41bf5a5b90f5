// Persistent tcgen05 GEMM engine for every dense product of the QLoRA linear.
//
//   D[M x N] = alpha * sum_seg A_seg[M x K_seg] * B_seg[N x K_seg]^T
//
// One kernel, warp-specialised, one CTA per SM (or one CTA pair per two SMs):
//   warps 0, 6    TMA producers of A and of B: 128-byte-swizzled tiles into a
//                 ring of shared-memory stages (mbarrier full/empty pairs);
//                 a stage holds one or (WIDE) two 64-wide k-blocks;
//   warp 1        allocates TMEM, one thread issues tcgen05.mma (bf16 in, fp32
//                 accumulate) into one of two TMEM accumulators;
//   warps 2..5    epilogue: tcgen05.ld the accumulator, scale, convert, store;
//                 the second accumulator lets the next tile's MMAs overlap.
// It is launched as a programmatic dependent: the set-up (barriers, TMEM)
// overlaps the previous kernel, and every role starts after pdl_wait().
// Each segment has its own operand major-ness (K-major = contiguous along the
// reduction; MN-major = contiguous along the output rows/columns), selected
// per MMA through the instruction descriptor, so X*W^T, dY*W (W read in its
// stored layout), X^T*G and the LoRA extra K-steps all run on this engine.
// A split of the reduction (split-K; of segment 0, or of every segment when
// they have equal lengths) writes fp32 partials that a finalize kernel sums
// in a fixed order.  The fold form adds accumulator columns j and j + fold,
// so a product against a [hi | lo] pair of bf16 halves (2 fold columns, one N
// tile) streams its other operand once.  In the CTA-pair form (cta_group::2, a cluster of two
// CTAs) the pair computes 256-row tiles: each CTA stages its 128 rows of A
// and half of B's rows, the leader CTA issues 256-row MMAs that read both
// CTAs' shared memory, and each CTA's epilogue drains its own 128 rows of
// the accumulator -- half the B bytes per SM of the single-CTA form.
// A bf16 output can also be stored as a hi/lo pair
// (hi = bf16(v), lo = bf16(v - hi)) so that a later product can consume it
// at nearly fp32 accuracy as two bf16 operands.
#pragma once

#include "common.cuh"

namespace qlora {

constexpr int kBM = 128;   // MMA M (TMEM lanes)
constexpr int kBK = 64;    // one 128-byte swizzle row of bf16
constexpr int kGemmThreads = 224;
constexpr int kProdBWarp = 6;   // the B producer; warp 0 produces A

struct TcSeg {
  int nkb;   // 64-wide k-blocks in this segment
  int a_mn;  // A is MN-major (contiguous along M)
  int b_mn;  // B is MN-major (contiguous along N)
  int wide;  // both tensor maps are 3-D boxes of two k-blocks (WIDE kernels only)
};

struct TcGemmArgs {
  int M, N;
  int m_tiles, n_tiles, splits, kb_per_split;
  int nseg;
  int split_all;            // split-K applies to every segment (equal k-block counts)
  TcSeg seg[2];
  float alpha;
  void *out;
  int64_t ld_row, ld_col;   // element strides of D(i, j) in `out` (unsplit output)
  int64_t lo_off;           // bf16 output only: if > 0 also store lo = bf16(v - hi) at +lo_off
  int out_f32;              // 1: fp32 output, 0: bf16
  int fold;                 // fold form: output column j < fold is D(i, j) + D(i, j + fold)
  // Optional masked addend of a bf16 output (unsplit, not folded): before
  // rounding, D(i, j) += add_scale * Z(i, j) where bit (i*N + j) of add_mask
  // is set (Z bf16 with row stride add_ld; N a multiple of 32).  LoRA dropout
  // uses it to gate the adapter term of dX.
  const uint16_t *add;
  const uint32_t *add_mask;
  float add_scale;
  int64_t add_ld;
  int *err;
};

// v[j] += add_scale * Z(row, col0 + j) for the kept columns of a 32-column chunk.
__device__ __forceinline__ void tc_add_masked(const TcGemmArgs &p, int row, int col0, float (&v)[32]) {
  const uint32_t m = ld_dep_u32(p.add_mask + (((int64_t)row * p.N + col0) >> 5));
  const uint16_t *z = p.add + (int64_t)row * p.add_ld + col0;
  if ((p.add_ld & 7) == 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 w = ld_dep_v4(z + 8 * q);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int j = 8 * q + 2 * h;
        if ((m >> j) & 1u) v[j] += p.add_scale * __uint_as_float(ww[h] << 16);
        if ((m >> (j + 1)) & 1u) v[j + 1] += p.add_scale * __uint_as_float(ww[h] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if ((m >> j) & 1u) v[j] += p.add_scale * __uint_as_float(ld_dep_u16(z + j) << 16);
  }
}

// Fold-form store of 32 consecutive output columns col0.. of row `row` (the
// values before alpha; split partials go to the dense [split][M][fold] buffer).
__device__ __forceinline__ void tc_store_fold(const TcGemmArgs &p, int row, int col0, int split, const float (&v)[32]) {
  const int W = p.fold;
  if (p.splits > 1) {
    float *o = reinterpret_cast<float *>(p.out) + ((int64_t)split * p.M + row) * W + col0;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j < W) o[j] = v[j];
    return;
  }
  const float alpha = p.alpha;
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (col0 + j < W) {
      const float x = alpha * v[j];
      const int64_t off = (int64_t)row * p.ld_row + (int64_t)(col0 + j) * p.ld_col;
      if (p.out_f32) {
        reinterpret_cast<float *>(p.out)[off] = x;
      } else {
        __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(p.out);
        const __nv_bfloat16 hb = __float2bfloat16_rn(x);
        o[off] = hb;
        if (p.lo_off > 0) o[off + p.lo_off] = __float2bfloat16_rn(x - __bfloat162float(hb));
      }
    }
}

// BN: output columns per tile.  PAIR: tile of 2*kBM rows computed by a CTA
// pair, each CTA holding kBM rows of A and BN/2 rows of B.  WIDE: a stage
// holds two k-blocks, each operand loaded by one 3-D box spanning both (a
// segment that cannot use 3-D boxes fills only the first k-block of a stage).
template <int BN, bool PAIR = false, bool WIDE = false>
struct TcCfg {
  static constexpr int kTileM = PAIR ? 2 * kBM : kBM;
  static constexpr int kBRows = PAIR ? BN / 2 : BN;   // B rows staged by one CTA
  static constexpr int kABytes = kBM * kBK * 2;       // one k-block of A
  static constexpr int kBBytes = kBRows * kBK * 2;    // one k-block of B
  static constexpr int kKB = WIDE ? 2 : 1;            // k-blocks per stage
  static constexpr int kAStage = kKB * kABytes;
  static constexpr int kStageBytes = kKB * (kABytes + kBBytes);
  // MN-major operands are stored as 64-element-wide chunks of kKB*64 k-rows.
  static constexpr int kMnChunk = kKB * 64 * 128;
  static constexpr int kStages = WIDE ? (PAIR || BN == 128 ? 3 : (BN == 64 ? 4 : 2))
                                      : (PAIR ? 7 : (BN == 256 ? 4 : (BN == 128 ? 6 : 8)));
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = kStages * kStageBytes + kBarBytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
  static_assert(!PAIR || BN % 128 == 0, "each CTA of a pair stages whole 64-row B atoms");
};

__device__ __forceinline__ void tc_unit_coords(int u, const TcGemmArgs &p, int &mt, int &nt, int &split) {
  const int tiles = p.m_tiles * p.n_tiles;
  split = u / tiles;
  const int t = u - split * tiles;
  // sweep 16 M-tiles across all N-tiles: B panels stay in L2 (8 re-read them
  // from DRAM twice as often; 32 let the A panels crowd L2: both slower)
  constexpr int kGroupM = 16;
  const int per_group = kGroupM * p.n_tiles;
  const int group = t / per_group;
  const int first_m = group * kGroupM;
  const int gm = min(p.m_tiles - first_m, kGroupM);
  const int r = t - group * per_group;
  mt = first_m + r % gm;
  nt = r / gm;
}

__device__ __forceinline__ void tc_seg_range(const TcGemmArgs &p, int s, int split, int &kb0, int &kb1) {
  if (s == 0 || p.split_all) {
    kb0 = split * p.kb_per_split;
    kb1 = min(p.seg[s].nkb, kb0 + p.kb_per_split);
  } else {
    kb0 = 0;
    kb1 = split == 0 ? p.seg[1].nkb : 0;
  }
}

// DROPZ (LoRA dropout in dX, pair form): segment 1 (the adapter term) goes
// into the tile's second accumulator instead of the first, and the epilogue
// stores alpha * D0 + add_scale * m * D1 with the keep mask m (add_mask).
// The two accumulators then serve one tile, so tiles do not overlap.
template <int BN, bool PAIR = false, bool FOLD = false, bool WIDE = false, bool DROPZ = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tA0, const __grid_constant__ CUtensorMap tB0,
                   const __grid_constant__ CUtensorMap tA1, const __grid_constant__ CUtensorMap tB1,
                   const TcGemmArgs p) {
  using Cfg = TcCfg<BN, PAIR, WIDE>;
  constexpr int S = Cfg::kStages;
  // Pair form: the grid is a 1-D array of 2-CTA clusters; CTA rank 0 leads.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int first_unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int unit_stride = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment: the 128B-swizzle pattern repeats every 8 rows of 128 B.
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *bar_area = smem + S * Cfg::kStageBytes;
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(bar_area);
  uint64_t *empty_bar = full_bar + S;
  uint64_t *tfull_bar = empty_bar + S;       // [2]
  uint64_t *tempty_bar = tfull_bar + 2;      // [2]
  uint64_t *done_bar = tempty_bar + 2;       // [1]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(full_bar + i), 2);    // the A and the B producer (of the leader, in a pair)
      mbar_init(smem_u32(empty_bar + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(tfull_bar + i), 1);
      mbar_init(smem_u32(tempty_bar + i), PAIR ? 8 : 4);  // one arrive per epilogue warp (of both CTAs)
    }
    mbar_init(smem_u32(done_bar), 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tA0);
    tma_prefetch_desc(&tB0);
    if (p.nseg > 1) {
      tma_prefetch_desc(&tA1);
      tma_prefetch_desc(&tB1);
    }
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(smem_u32(tmem_slot), Cfg::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  // Pair form: neither CTA may touch its peer's barriers before they exist.
  if (PAIR) {
    __syncwarp();   // the cluster barrier is warp-aligned: reconverge after the role branches
    cluster_sync();
  } else {
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Launched as a programmatic dependent: the set-up above overlapped the
  // previous kernel; its results are visible after the wait.
  pdl_trigger();
  pdl_wait();

  const int units = p.m_tiles * p.n_tiles * p.splits;

  if (warp == 0 || warp == kProdBWarp) {
    // ------------------------------------------------------------ producers
    // One thread streams A and another B: the TMA engine overlaps the copies
    // of different issuing threads, while one thread's copies are served
    // largely one after another.  Each arms the full barrier with its own
    // bytes (in a pair, both CTAs' bytes of its operand).
    if (lane == 0) {
      const bool isA = warp == 0;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0;           // stages that received at least one load
      uint32_t last_parity = 0;    // parity of the last load issued into each stage
      bool ok = true;
      // Loads of either CTA of a pair complete on the leader's full barrier,
      // which expects both CTAs' bytes.
      auto load = [&](uint32_t dst, const CUtensorMap *m, uint32_t bar, int x, int y) {
        if (PAIR) tma_load_2d_pair(dst, m, bar, x, y); else tma_load_2d(dst, m, bar, x, y);
      };
      auto load3 = [&](uint32_t dst, const CUtensorMap *m, uint32_t bar, int y, int z) {
        if (PAIR) tma_load_3d_pair(dst, m, bar, 0, y, z); else tma_load_3d(dst, m, bar, 0, y, z);
      };
      const int a_row0 = (int)rank * kBM;           // this CTA's rows within the tile
      const int b_row0 = (int)rank * Cfg::kBRows;
      for (int u = first_unit; u < units && ok; u += unit_stride) {
        int mt, nt, split;
        tc_unit_coords(u, p, mt, nt, split);
        const int am = mt * Cfg::kTileM + a_row0;
        const int bn0 = nt * BN + b_row0;
        for (int s = 0; s < p.nseg && ok; ++s) {
          const CUtensorMap *ta = s == 0 ? &tA0 : &tA1;
          const CUtensorMap *tb = s == 0 ? &tB0 : &tB1;
          int kb0, kb1;
          tc_seg_range(p, s, split, kb0, kb1);
          const bool wide = WIDE && p.seg[s].wide;
          const int step = wide ? 2 : 1;
          for (int kb = kb0; kb < kb1; kb += step) {
            if (!mbar_wait(smem_u32(empty_bar + stage), phase ^ 1, p.err, DEV_TIMEOUT_PRODUCER)) {
              ok = false;
              break;
            }
            const uint32_t fb_local = smem_u32(full_bar + stage);
            const uint32_t fb = PAIR ? mapa_shared(fb_local, 0) : fb_local;
            // a box is counted in full, also where it reaches past the
            // segment (those k-blocks are zero-filled or simply not used)
            const uint32_t bytes = isA ? (wide ? Cfg::kAStage : Cfg::kABytes)
                                       : (wide ? Cfg::kStageBytes - Cfg::kAStage : Cfg::kBBytes);
            if (leader) mbar_arrive_expect_tx(fb_local, (PAIR ? 2 : 1) * bytes);
            const uint32_t sa = smem_u32(smem + stage * Cfg::kStageBytes);
            const uint32_t sb = sa + Cfg::kAStage;
            if (wide) {
              // K-major maps are {64 k, rows, k-blocks}: smem [k-block][row][64].
              // MN-major maps are {64 mn, k, 64-wide mn chunks}: smem [chunk][k][64].
              if (isA) {
                if (!p.seg[s].a_mn) load3(sa, ta, fb, am, kb);
                else load3(sa, ta, fb, kb * kBK, am >> 6);
              } else {
                if (!p.seg[s].b_mn) load3(sb, tb, fb, bn0, kb);
                else load3(sb, tb, fb, kb * kBK, bn0 >> 6);
              }
            } else if (isA) {
              if (!p.seg[s].a_mn) {
                load(sa, ta, fb, kb * kBK, am);
              } else {
                load(sa, ta, fb, am, kb * kBK);
                load(sa + Cfg::kMnChunk, ta, fb, am + 64, kb * kBK);
              }
            } else {
              if (!p.seg[s].b_mn) {
                load(sb, tb, fb, kb * kBK, bn0);
              } else {
#pragma unroll
                for (int j = 0; j < Cfg::kBRows / 64; ++j) load(sb + j * Cfg::kMnChunk, tb, fb, bn0 + 64 * j, kb * kBK);
              }
            }
            used |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == S) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
      }
      // Drain: never leave the CTA while a tensor copy is still landing in
      // shared memory.  A single CTA watches its full barriers.  In a pair the
      // copies complete on the leader's barriers, so each CTA instead waits
      // until the MMAs have consumed the last fill of every stage (its empty
      // barrier completes the phase of that fill's parity); after one wait
      // runs out the rest are skipped, the copies having long landed.
      for (int i = 0; i < S; ++i) {
        if (!(used & (1u << i))) continue;
        const uint32_t par = (last_parity >> i) & 1u;
        const bool done = PAIR ? mbar_wait(smem_u32(empty_bar + i), par, p.err, DEV_TIMEOUT_DRAIN)
                               : mbar_wait(smem_u32(full_bar + i), par, p.err, DEV_TIMEOUT_DRAIN);
        if (!done) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Pair form: the leader alone issues; the peer's tensor core works on the
    // leader's instructions.
    if (lane == 0 && leader) {
      uint32_t idesc[2];
      for (int s = 0; s < 2; ++s) idesc[s] = idesc_bf16_f32(Cfg::kTileM, BN, p.seg[s].a_mn, p.seg[s].b_mn);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int t = 0;
      for (int u = first_unit; u < units && ok; u += unit_stride, ++t) {
        int mt, nt, split;
        tc_unit_coords(u, p, mt, nt, split);
        constexpr int kAccs = DROPZ ? 1 : 2;
        const int acc = t % kAccs;
        const uint32_t use = (uint32_t)(t / kAccs);
        if (!mbar_wait<PAIR>(smem_u32(tempty_bar + acc), (use & 1u) ^ 1u, p.err, DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        uint32_t accumulate = 0;
        for (int s = 0; s < p.nseg && ok; ++s) {
          int kb0, kb1;
          tc_seg_range(p, s, split, kb0, kb1);
          if (DROPZ && s == 1) {   // the adapter term into the second accumulator
            d_tmem = tmem_base + (uint32_t)BN;
            accumulate = 0;
          }
          const int a_mn = p.seg[s].a_mn, b_mn = p.seg[s].b_mn;
          const int step = (WIDE && p.seg[s].wide) ? 2 : 1;
          for (int kb = kb0; kb < kb1; kb += step) {
            if (!mbar_wait(smem_u32(full_bar + stage), phase, p.err, DEV_TIMEOUT_MMA)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + stage * Cfg::kStageBytes);
            const uint32_t sb = sa + Cfg::kAStage;
            const int nk = min(step, kb1 - kb);
            for (int kk = 0; kk < nk; ++kk) {
              // K-major: k-block kk is the next [rows][64] tile; the 16-wide
              // k-slice starts 32 B into each swizzled row.  MN-major: k-block
              // kk starts 64 k-rows (8 KB) into each chunk, the k-slice 16
              // k-rows (2 KB) further.
              const uint32_t ak = a_mn ? sa + kk * 8192 : sa + kk * Cfg::kABytes;
              const uint32_t bk = b_mn ? sb + kk * 8192 : sb + kk * Cfg::kBBytes;
#pragma unroll
              for (int k = 0; k < kBK / 16; ++k) {
                const uint64_t ad = a_mn ? smem_desc_sw128(ak + k * 2048, Cfg::kMnChunk, 1024)
                                         : smem_desc_sw128(ak + k * 32, 16, 1024);
                const uint64_t bd = b_mn ? smem_desc_sw128(bk + k * 2048, Cfg::kMnChunk, 1024)
                                         : smem_desc_sw128(bk + k * 32, 16, 1024);
                if (PAIR) tc_mma_f16_pair(d_tmem, ad, bd, idesc[s], accumulate);
                else tc_mma_f16(d_tmem, ad, bd, idesc[s], accumulate);
                accumulate = 1;
              }
            }
            // frees the stage (in both CTAs of a pair) once these MMAs have read it
            if (PAIR) tc_commit_pair(smem_u32(empty_bar + stage), 0x3);
            else tc_commit(smem_u32(empty_bar + stage));
            if (++stage == S) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
        // accumulator ready for the epilogue(s)
        if (PAIR) tc_commit_pair(smem_u32(tfull_bar + acc), 0x3);
        else tc_commit(smem_u32(tfull_bar + acc));
      }
      // All MMAs issued by this thread must finish before TMEM is released.
      if (PAIR) tc_commit_pair(smem_u32(done_bar), 0x1);
      else tc_commit(smem_u32(done_bar));
      mbar_wait(smem_u32(done_bar), 0, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp < kProdBWarp) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int t = 0;
    // The accumulator is released with one arrive per warp, on the leader's
    // barrier in the pair form.
    const uint32_t tempty0 = PAIR ? mapa_shared(smem_u32(tempty_bar), 0) : smem_u32(tempty_bar);
    for (int u = first_unit; u < units; u += unit_stride, ++t) {
      int mt, nt, split;
      tc_unit_coords(u, p, mt, nt, split);
      constexpr int kAccs = DROPZ ? 1 : 2;
      const int acc = t % kAccs;
      const uint32_t use = (uint32_t)(t / kAccs);
      // Warp-uniform wait: tcgen05.ld below must be executed by all 32 lanes.
      const bool got = mbar_wait(smem_u32(tfull_bar + acc), use & 1u, p.err, DEV_TIMEOUT_EPILOGUE);
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      tc_fence_after();
      const int row = mt * Cfg::kTileM + (int)rank * kBM + q * 32 + lane;
      const bool row_ok = row < p.M;
      const float alpha = p.alpha;
      if constexpr (FOLD) {
        // one N tile of 2*fold columns: output column j = column j + column j + fold
        const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
        for (int c = 0; c < (p.fold < 32 ? 32 : p.fold); c += 32) {
          uint32_t r[32];
          float v[32];
          tmem_ld_32x32b_x32(tb + (uint32_t)c, r);
          tmem_wait_ld();
          if (p.fold >= 32) {
            uint32_t r2[32];
            tmem_ld_32x32b_x32(tb + (uint32_t)(c + p.fold), r2);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) + __uint_as_float(r2[j]);
          } else if (p.fold == 16) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = j < 16 ? __uint_as_float(r[j]) + __uint_as_float(r[j + 16]) : 0.f;
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = j < 8 ? __uint_as_float(r[j]) + __uint_as_float(r[j + 8]) : 0.f;
          }
          if (row_ok) tc_store_fold(p, row, c, split, v);
        }
      } else
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + c), r);
        [[maybe_unused]] uint32_t r2[32];
        if constexpr (DROPZ) tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(BN + c), r2);
        tmem_wait_ld();
        const int col0 = nt * BN + c;
        if (!row_ok || col0 >= p.N) continue;
        if (p.splits > 1) {
          // split-K partial: dense fp32 [split][M][N], summed by the finalize pass
          float *o = reinterpret_cast<float *>(p.out) + ((int64_t)split * p.M + row) * p.N + col0;
          if (col0 + 32 <= p.N && (p.N & 3) == 0) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              reinterpret_cast<float4 *>(o)[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                                             __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < p.N) o[j] = __uint_as_float(r[j]);
          }
        } else if (p.out_f32) {
          float *o = reinterpret_cast<float *>(p.out);
          if (p.ld_col == 1 && col0 + 32 <= p.N && (p.ld_row & 3) == 0) {
            float4 *dst = reinterpret_cast<float4 *>(o + (int64_t)row * p.ld_row + col0);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(alpha * __uint_as_float(r[4 * j]), alpha * __uint_as_float(r[4 * j + 1]),
                                   alpha * __uint_as_float(r[4 * j + 2]), alpha * __uint_as_float(r[4 * j + 3]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < p.N) o[(int64_t)row * p.ld_row + (int64_t)(col0 + j) * p.ld_col] = alpha * __uint_as_float(r[j]);
          }
        } else {
          __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(p.out);
          const int64_t lo = p.lo_off;
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = alpha * __uint_as_float(r[j]);
          if constexpr (DROPZ) {
            const uint32_t m = ld_dep_u32(p.add_mask + (((int64_t)row * p.N + col0) >> 5));
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if ((m >> j) & 1u) v[j] += p.add_scale * __uint_as_float(r2[j]);
          } else if (p.add) {
            tc_add_masked(p, row, col0, v);
          }
          if (p.ld_col == 1 && col0 + 32 <= p.N && (p.ld_row & 7) == 0 && (lo & 7) == 0) {
            uint4 *dst = reinterpret_cast<uint4 *>(o + (int64_t)row * p.ld_row + col0);
            uint4 *dst_lo = reinterpret_cast<uint4 *>(o + (int64_t)row * p.ld_row + col0 + lo);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t w[4], wl[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const float v0 = v[8 * j + 2 * h];
                const float v1 = v[8 * j + 2 * h + 1];
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
              if (col0 + j < p.N) {
                const __nv_bfloat16 hb = __float2bfloat16_rn(v[j]);
                const int64_t off = (int64_t)row * p.ld_row + (int64_t)(col0 + j) * p.ld_col;
                o[off] = hb;
                if (lo > 0) o[off + lo] = __float2bfloat16_rn(v[j] - __bfloat162float(hb));
              }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR) mbar_arrive_cluster(tempty0 + 8u * (uint32_t)acc);
        else mbar_arrive(tempty0 + 8u * (uint32_t)acc);
      }
    }
  }

  tc_fence_before();
  // Pair form: no CTA leaves (or frees TMEM) while its peer may still signal
  // its barriers or its MMAs may still run.
  if (PAIR) {
    __syncwarp();   // the cluster barrier is warp-aligned: reconverge after the role branches
    cluster_sync();
  } else {
    __syncthreads();
  }
  tc_fence_after();
  if (warp == 1) {
    if (PAIR) tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
    else tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

// Fixed-order sum of split-K partials (dense fp32 [splits][M][N]) into the
// output D(i, j) at dst + i*ld_row + j*ld_col, with the same bf16 hi/lo and
// fp32 options as the GEMM epilogue.
__global__ void __launch_bounds__(256) splitk_finalize_kernel(const float *__restrict__ part, int splits, int M,
                                                              int N, float alpha, void *dst, int64_t ld_row,
                                                              int64_t ld_col, int64_t lo_off, int dst_f32) {
  pdl_trigger();
  pdl_wait();
  const int64_t count = (int64_t)M * N;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int k = 0; k < splits; ++k) s += ld_dep_f32(part + (int64_t)k * count + i);
    s *= alpha;
    const int64_t row = i / N, col = i - row * N;
    const int64_t off = row * ld_row + col * ld_col;
    if (dst_f32) {
      reinterpret_cast<float *>(dst)[off] = s;
    } else {
      __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(dst);
      const __nv_bfloat16 hb = __float2bfloat16_rn(s);
      o[off] = hb;
      if (lo_off > 0) o[off + lo_off] = __float2bfloat16_rn(s - __bfloat162float(hb));
    }
  }
}

}  // namespace qlora
