// Fused doubleDequant + tensor-core product for up to 128 tokens (QLoRA §3
// Eq. 5 with the frozen weight decoded on the fly, Eq. 6): the NF4 weight is
// streamed from HBM once and decoded straight into tensor memory, where
// tcgen05 MMAs read it as their A operand -- no bf16 copy of the weight is
// written to HBM or to shared memory.
//
//   acc[M x N] += X W_hat^T        (fp32, L2-resident; zero at launch)
//
// computed transposed, acc^T = W_hat X^T: the weight rows are the 128-row MMA M
// dimension (TMEM lanes) and the tokens the MMA N dimension (MP = tokens
// padded to 16, 32, 64 or 128).  The LoRA branch and the bf16 output come
// from the kernels around it (lora_down_small_kernel before it, which it
// overlaps as a programmatic dependent, and lora_epilogue_kernel after;
// few_token.cuh).
//
// The decoded weight is exactly doubleDequant's bf16 weight (bit-identical to
// qlora_dequant): W_hat = bf16(fp32(level[c] * c2_hat)) with c2_hat =
// fma(E4M3(code8), c1, mu), the block constant of the weight's 64-block.
// A byte of two codes looks up the fp32 pair (level[lo], level[hi]) in a
// fixed 256-entry table; one packed fp32 multiply (mul.rn.f32x2) applies the
// block's c2_hat and one conversion rounds the pair to bf16 -- the same two
// roundings as the dequant kernel, with no per-block table to build.
//
// One persistent CTA per SM, 14 warps:
//   warps 0..3    epilogue: tcgen05.ld of the accumulator (lane = weight row,
//                 column = token) and red.global.add into acc;
//   warps 4..11   two decoder warpgroups; group g decodes the items (row
//                 tile, 256-K stage) g, g + 2, ... of the CTA's range.  Thread t
//                 of a group owns weight row t of the tile (TMEM lane t): it
//                 reads its row's 128 code bytes from the stage (128-byte
//                 swizzle, conflict-free 16-byte loads), and per byte
//                 extracts it (one byte permute), forms the address of its
//                 replica of the table entry (one multiply-add), loads the
//                 fp32 pair (8 bytes; the table holds 16 replicas, so each
//                 half-warp's lookups hit 32 distinct banks), multiplies it
//                 by c2_hat (one packed fp32 multiply) and rounds it to a bf16
//                 pair (one conversion).  Each 64-block's 32 pairs go to TMEM
//                 with one tcgen05.st (32 columns of the group's A slot);
//   warp 12       producer: lane 0 loads, per stage, 128 weight rows x 256 K
//                 of packed codes (128-byte swizzle) into the codes ring and
//                 the stage's X as four K-major 128-byte-swizzled atoms of MP
//                 tokens (one 3-D box) into the X ring, with TMA.  A decoder
//                 thread copies its row's 128 code bytes into registers as
//                 soon as they land and the slot goes back to the producer at
//                 once, so nearly the whole codes ring (up to 8 x 16 KB) is
//                 in flight: at HBM rate a stage takes thousands of cycles to
//                 land, and slots held while their data is decoded starved
//                 the memory pipeline.  The X ring is released by the MMAs'
//                 one commit per item, which also frees the decoding group's
//                 TMEM slot;  The raw block constants of a row (its four E4M3
//                 codes and c1) are loaded by the decoder thread that owns
//                 the row, into registers, two of its items ahead: gathered
//                 by one producer warp, 128 rows of scattered 4-byte copies
//                 per stage set the pace of the whole kernel;
//   warp 13       allocates TMEM; one thread issues tcgen05.mma (M = 128,
//                 N = MP, K = 16; A from the group's TMEM slot, B from the X
//                 atoms) into one of two TMEM accumulators.
// TMEM columns: [0, 2 MP) the two accumulators, then one 128-column A slot
// per decoder group (K = 256 bf16 of 128 rows).
// Work: the items are split into equal contiguous ranges, one per CTA; the
// CTA adds its partial sums into acc whenever its range moves to the next
// row tile, and at its end.  Groups of linears concatenate their items (see
// the group note in few_token.cuh).
#pragma once

#include "common.cuh"
#include "quant.cuh"
#include "few_token.cuh"

namespace qlora {

constexpr int kDfRows = 128;                  // weight rows per tile (MMA M, TMEM lanes)
constexpr int kDfStageK = 256;                // K per stage: four 64-blocks
constexpr int kDfLutEntries = 256;            // one per code byte (two codes)
constexpr int kDfLutReplicas = 16;            // one per lane of a half-warp (8-byte loads)
constexpr int kDfLutBytes = kDfLutEntries * kDfLutReplicas * 8;

// One linear of a launch: its shape, block constants and accumulator.
struct DfMember {
  int N, K;
  int kstages;           // ceil(K / 256)
  DivU31 ks_div;         // division by kstages
  const uint8_t *c2_fp8;
  const float *c1;
  const float *mu;
  float *acc;            // [M x N] fp32, zero at launch
};

// A group of linears that see the same tokens: their (row tile, stage) items
// are concatenated, linear after linear (see the group note in few_token.cuh).
template <int GM>
struct DfArgs {
  int M;
  int count;             // linears in the group
  int items;             // row tiles x kstages, summed over the group
  int beg[GM];           // first item of each linear
  DfMember m[GM];
  float levels[16];      // the 16-level code table (shared by the group)
  int *err;
};

// Per linear: its packed codes in boxes of 128 rows x 128 bytes, and X as
// [64-block][token][64] in boxes of the four atoms of a stage.
template <int GM>
struct DfMaps {
  CUtensorMap codes[GM];
  CUtensorMap x[GM];
};

// Item `it` of a group -> its linear l, row tile rt and stage ks.
template <int GM>
__device__ __forceinline__ const DfMember &df_item(const DfArgs<GM> &p, int it, int &l, int &rt, int &ks) {
  l = group_member<GM>(p.beg, p.count, it);
  const DfMember &m = p.m[l];
  const int li = it - p.beg[l];
  rt = (int)m.ks_div.div((uint32_t)li);
  ks = li - rt * m.kstages;
  return m;
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// The contiguous range of items [i0, i1) of CTA b among g.
__device__ __forceinline__ void df_range(int items, int b, int g, int &i0, int &i1) {
  i0 = (int)(((int64_t)items * b) / g);
  i1 = (int)(((int64_t)items * (b + 1)) / g);
}

// c2_hat of block kb0 + j of weight row n from its raw constants (j < 4, the
// block inside the weight).
__device__ __forceinline__ float df_c2hat(uint4 raw, int n, int kb0, int j, int kblocks, float mu) {
  const int64_t b0 = (int64_t)n * kblocks + kb0;
  const int sh = (int)(b0 & 3) + j;                  // byte index in the 8-byte pair
  const uint32_t code8 = (sh < 4 ? raw.x >> (8 * sh) : raw.y >> (8 * (sh - 4))) & 0xFFu;
  const float c1 = ((b0 + j) >> 8) == (b0 >> 8) ? __uint_as_float(raw.z) : __uint_as_float(raw.w);
  return __fmaf_rn(e4m3_to_f32((uint8_t)code8), c1, mu);
}

template <int MP>
struct DfCfg {
  static_assert(MP == 16 || MP == 32 || MP == 64 || MP == 128, "MMA N");
  static constexpr int kGroups = 2;                           // decoder warpgroups
  static constexpr int kDecWarp0 = 4;
  static constexpr int kProdWarp = kDecWarp0 + 4 * kGroups;
  static constexpr int kMmaWarp = kProdWarp + 1;
  static constexpr int kThreads = 32 * (kMmaWarp + 1);
  static constexpr int kCodeBytes = kDfRows * 128;            // 128 rows x 256 codes
  static constexpr int kXBytes = 4 * MP * 128;                // 4 atoms of MP rows x 64 bf16
  static constexpr int kBarBytes = 1024;
  static constexpr int kMaxSmem = 232448;                     // per CTA on sm_100
  static constexpr int kRingBytes = kMaxSmem - 1024 - kDfLutBytes - kBarBytes;
  // X ring: 64 KB of stages (at least two); the codes ring takes the rest, up to 8 stages
  static constexpr int kXStages = (65536 / kXBytes) < 2 ? 2 : (65536 / kXBytes > 8 ? 8 : 65536 / kXBytes);
  static constexpr int kCodeStagesFit = (kRingBytes - kXStages * kXBytes) / kCodeBytes;
  static constexpr int kCodeStages = kCodeStagesFit > 8 ? 8 : kCodeStagesFit;
  static constexpr int kSmemBytes = kCodeStages * kCodeBytes + kXStages * kXBytes + kDfLutBytes + kBarBytes + 1024;
  static constexpr int kACols = kDfStageK / 2;                // 32-bit TMEM columns per A slot
  static constexpr int kTmemCols = 512;
  static_assert(kCodeStages >= 2, "pipeline depth");
  static_assert(kCodeBytes % 1024 == 0 && kXBytes % 1024 == 0, "128-byte-swizzle boxes start 1 KB aligned");
  static_assert(2 * MP + kGroups * kACols <= kTmemCols, "TMEM columns");
  static_assert(kXStages >= kGroups, "an item's completion barrier outlives its group's next item");
  static_assert(kSmemBytes <= kMaxSmem, "shared memory per CTA");
};

// The fp32 pair at a shared-memory address (8-byte aligned).
__device__ __forceinline__ uint64_t lds64(uint32_t addr) {
  uint64_t v;
  asm("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(addr));
  return v;
}

// {c, c} as a packed fp32 pair.
__device__ __forceinline__ uint64_t f32x2_splat(float c) {
  uint64_t v;
  asm("mov.b64 %0, {%1, %1};" : "=l"(v) : "f"(c));
  return v;
}

// bf16 pair (low half = element 0) of the fp32 products p * c, each rounded
// to fp32 and then to bf16 (round to nearest even both times).
__device__ __forceinline__ uint32_t mul_round_bf16x2(uint64_t p, uint64_t c) {
  uint64_t y;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(p), "l"(c));
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(y));
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Raw block constants of weight row n for stage ks, in registers, in the
// layout df_c2hat reads: the two aligned 32-bit words of c2_fp8 holding the
// row's (up to) four E4M3 codes of the stage, then c1 of the first and of
// the last of those blocks.  Words that reach past the end of c2_fp8 are
// read byte by byte.  Rows past the weight read nothing.
__device__ __forceinline__ uint4 df_load_raw(const DfMember &m, int n, int ks) {
  uint4 raw = make_uint4(0, 0, 0, 0);
  if (n >= m.N) return raw;
  const int kblocks = m.K >> 6;
  const int kb0 = ks * 4;
  const int nb = min(4, kblocks - kb0);
  const int64_t nblk = (int64_t)m.N * kblocks;
  const int64_t b0 = (int64_t)n * kblocks + kb0;
  const int64_t last = b0 + nb - 1;
  const int64_t w0 = b0 >> 2;
  uint32_t wv[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int64_t w = w0 + k;
    if (k == 1 && (last >> 2) == w0) break;
    if (4 * w + 3 < nblk) {
      wv[k] = __ldg(reinterpret_cast<const uint32_t *>(m.c2_fp8) + w);
    } else {
      for (int64_t b = 4 * w; b < nblk; ++b) wv[k] |= (uint32_t)__ldg(m.c2_fp8 + b) << (8 * (int)(b - 4 * w));
    }
  }
  raw.x = wv[0];
  raw.y = wv[1];
  raw.z = __float_as_uint(__ldg(m.c1 + (b0 >> 8)));
  raw.w = __float_as_uint(__ldg(m.c1 + (last >> 8)));
  return raw;
}

template <int MP, int GM>
__global__ void __launch_bounds__(DfCfg<MP>::kThreads, 1)
    nf4_decode_fwd_kernel(const __grid_constant__ DfMaps<GM> maps, const __grid_constant__ DfArgs<GM> p) {
  using Cfg = DfCfg<MP>;
  constexpr int SC = Cfg::kCodeStages;
  constexpr int SX = Cfg::kXStages;
  constexpr int G = Cfg::kGroups;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *xring = smem + SC * Cfg::kCodeBytes;
  uint8_t *lut = xring + SX * Cfg::kXBytes;
  uint64_t *cfull_bar = reinterpret_cast<uint64_t *>(lut + kDfLutBytes);   // [SC] codes landed
  uint64_t *cempty_bar = cfull_bar + SC;                // [SC] codes copied out by the decoders
  uint64_t *xfull_bar = cempty_bar + SC;                // [SX] X landed
  uint64_t *idone_bar = xfull_bar + SX;                 // [SX] item rel's MMAs done (slot rel % SX)
  uint64_t *afull_bar = idone_bar + SX;                 // [G]
  uint64_t *tfull_bar = afull_bar + G;                  // [2]
  uint64_t *tempty_bar = tfull_bar + 2;                 // [2]
  uint64_t *done_bar = tempty_bar + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the epilogue may launch and wait

  // The table: entry v (a code byte) holds the fp32 pair (level[v & 15],
  // level[v >> 4]) in replica j at byte 128 v + 8 j.
  for (int i = threadIdx.x; i < kDfLutEntries * kDfLutReplicas; i += blockDim.x) {
    const int v = i / kDfLutReplicas;
    reinterpret_cast<float2 *>(lut)[i] = make_float2(p.levels[v & 15], p.levels[v >> 4]);
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < SC; ++i) {
      mbar_init(smem_u32(cfull_bar + i), 1);                 // the TMA bytes
      mbar_init(smem_u32(cempty_bar + i), 4);                // the four warps of the decoding group
    }
    for (int i = 0; i < SX; ++i) {
      mbar_init(smem_u32(xfull_bar + i), 1);                 // the TMA bytes
      mbar_init(smem_u32(idone_bar + i), 1);                 // the MMAs' commit
    }
    for (int i = 0; i < G; ++i) mbar_init(smem_u32(afull_bar + i), 4);   // the four warps of a decoder group
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(tfull_bar + i), 1);
      mbar_init(smem_u32(tempty_bar + i), 4);
    }
    mbar_init(smem_u32(done_bar), 1);
    fence_mbar_init();
  }
  if (warp == Cfg::kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  int i0, i1;
  df_range(p.items, blockIdx.x, gridDim.x, i0, i1);

  if (warp == Cfg::kProdWarp) {
    // ------------------------------------------------------------ producer
    if (lane < p.count) {
      tma_prefetch_desc(&maps.codes[lane]);
      tma_prefetch_desc(&maps.x[lane]);
    }
    if (lane == 0) {
      bool ok = true;
      for (int it = i0; it < i1 && ok; ++it) {
        const int rel = it - i0;
        int l, rt, ks;
        df_item<GM>(p, it, l, rt, ks);
        const int cs = rel % SC, xs = rel % SX;
        if (!mbar_wait(smem_u32(cempty_bar + cs), ((uint32_t)(rel / SC) & 1u) ^ 1u, p.err, DEV_TIMEOUT_PRODUCER)) break;
        fence_proxy_async_smem();   // the decoders' loads of this slot before the copy's writes
        const uint32_t cb = smem_u32(cfull_bar + cs);
        mbar_arrive_expect_tx(cb, Cfg::kCodeBytes);
        tma_load_2d(smem_u32(smem + cs * Cfg::kCodeBytes), &maps.codes[l], cb, ks * (kDfStageK / 2), rt * kDfRows);
        // the X slot's previous item (rel - SX) has had its MMAs
        if (!mbar_wait(smem_u32(idone_bar + xs), ((uint32_t)(rel / SX) & 1u) ^ 1u, p.err, DEV_TIMEOUT_PRODUCER)) {
          ok = false;
          break;
        }
        const uint32_t xb = smem_u32(xfull_bar + xs);
        mbar_arrive_expect_tx(xb, Cfg::kXBytes);
        tma_load_3d(smem_u32(xring + xs * Cfg::kXBytes), &maps.x[l], xb, 0, 0, ks * 4);
      }
      // Drain: the copies of the last uses of every slot have landed.
      const int n = i1 - i0;
      for (int rel = n - SC > 0 ? n - SC : 0; rel < n; ++rel)
        if (!mbar_wait(smem_u32(cfull_bar + rel % SC), (uint32_t)(rel / SC) & 1u, p.err, DEV_TIMEOUT_DRAIN)) break;
      for (int rel = n - SX > 0 ? n - SX : 0; rel < n; ++rel)
        if (!mbar_wait(smem_u32(xfull_bar + rel % SX), (uint32_t)(rel / SX) & 1u, p.err, DEV_TIMEOUT_DRAIN)) break;
    }
  } else if (warp == Cfg::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // Every synchronising operation of this thread between MMAs (an mbarrier
    // wait, a tcgen05 fence, a commit) waits for the MMAs in flight, hundreds
    // of cycles each at these sizes (measured), so an item costs it as few as
    // possible: one wait (the decoder group signals its A slot only once the
    // item's X tile has landed too), one fence and one commit.  Batching the
    // items of both decoder groups under one wait was measured slower: with
    // one TMEM slot per group, decoding then no longer overlaps the MMAs.
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kDfRows, MP, 0, 0);
      int t = 0;               // row-tile segments started
      uint32_t accumulate = 0;
      for (int it = i0; it < i1; ++it) {
        int l, rt, ks;
        const DfMember &m = df_item<GM>(p, it, l, rt, ks);
        const int rel = it - i0;
        const int g = rel % G;
        const uint32_t use = (uint32_t)(rel / G);     // this group's item count before this one
        const int xs = rel % SX;
        const bool first = it == i0 || ks == 0;
        const bool last = it == i1 - 1 || ks == m.kstages - 1;
        const int acc = t & 1;
        if (first) {
          if (!mbar_wait(smem_u32(tempty_bar + acc), ((t >> 1) & 1u) ^ 1u, p.err, DEV_TIMEOUT_MMA)) break;
          accumulate = 0;
        }
        if (!mbar_wait(smem_u32(afull_bar + g), use & 1u, p.err, DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * MP);
        const uint32_t a_tmem = tmem_base + (uint32_t)(2 * MP + g * Cfg::kACols);
        const int nk = 4 * min(4, (m.K >> 6) - ks * 4);   // 16-wide k-steps of the stage's real blocks
        // k-step k reads A columns 8k and, as B, atom k / 4 of the item's X
        // (MP rows x 128 B) at byte 32 (k % 4) inside it: a constant offset of
        // the item's descriptor (its address field counts 16 B), so the loop
        // carries no arithmetic.
        const uint64_t b0 = smem_desc_sw128(smem_u32(xring + xs * Cfg::kXBytes), 16, 1024);
        if (nk == 16) {
          tc_mma_f16_ts(d_tmem, a_tmem, b0, idesc, accumulate);
#pragma unroll
          for (int k = 1; k < 16; ++k)
            tc_mma_f16_ts(d_tmem, a_tmem + 8 * k, b0 + (uint64_t)(((k >> 2) * (MP * 128) + (k & 3) * 32) >> 4), idesc, 1u);
        } else {
          for (int k = 0; k < nk; ++k)
            tc_mma_f16_ts(d_tmem, a_tmem + 8 * k, b0 + (uint64_t)(((k >> 2) * (MP * 128) + (k & 3) * 32) >> 4), idesc,
                          k == 0 ? accumulate : 1u);
        }
        accumulate = 1;
        // the item's completion frees its X slot and its group's A slot
        tc_commit(smem_u32(idone_bar + xs));
        if (last) {
          tc_commit(smem_u32(tfull_bar + acc));      // partial sums of this row tile ready
          ++t;
        }
      }
      tc_commit(smem_u32(done_bar));
      mbar_wait(smem_u32(done_bar), 0, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp >= Cfg::kDecWarp0 && warp < Cfg::kProdWarp) {
    // ------------------------------------------------------------ decoders
    const int g = (warp - Cfg::kDecWarp0) >> 2;
    const int quad = warp & 3;                    // TMEM lane quarter of this warp
    const int t = quad * 32 + lane;               // weight row within the tile
    const uint32_t lut_lane = smem_u32(lut) + 8u * (uint32_t)(lane & (kDfLutReplicas - 1));
    const uint32_t a_row = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(2 * MP + g * Cfg::kACols);
    const uint32_t cswz = (uint32_t)(t & 7) << 4;
    // the raw constants of this group's item it + u G (none past the range)
    auto raw_of = [&](int u) -> uint4 {
      const int it = i0 + g + u * G;
      if (it >= i1) return make_uint4(0, 0, 0, 0);
      int l, rt, ks;
      const DfMember &m = df_item<GM>(p, it, l, rt, ks);
      return df_load_raw(m, rt * kDfRows + t, ks);
    };
    // Decode the group's item u with its constants `raw`, then start loading
    // the constants of item u + 2 into `raw`.  Returns false on a timeout.
    auto item = [&](int u, uint4 &raw) -> bool {
      const int it = i0 + g + u * G;
      const int rel = it - i0;
      const int cs = rel % SC;
      int l, rt, ks;
      const DfMember &m = df_item<GM>(p, it, l, rt, ks);
      const int kblocks = m.K >> 6;
      const int nkb = min(4, kblocks - ks * 4);
      const int n = rt * kDfRows + t;
      const float mu = __ldg(m.mu);
      uint64_t c2[4];     // {c2_hat, c2_hat} of the stage's four blocks
#pragma unroll
      for (int j = 0; j < 4; ++j)
        c2[j] = f32x2_splat((j < nkb && n < m.N) ? df_c2hat(raw, n, ks * 4, j, kblocks, mu) : 0.f);
      raw = raw_of(u + 2);
      // the row's 128 code bytes into registers (16-byte chunks of its
      // swizzled line), and the stage's codes slot back to the producer
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(cfull_bar + cs), (uint32_t)(rel / SC) & 1u, p.err,
                                             DEV_TIMEOUT_MMA)))
        return false;
      const uint32_t sc = smem_u32(smem + cs * Cfg::kCodeBytes) + t * 128;
      uint4 qv[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) qv[c] = lds128(sc + (((uint32_t)c << 4) ^ cswz));
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(cempty_bar + cs));
      // the MMAs of this group's previous item (rel - G) have read its A
      // slot.  The X ring has at least G slots, so that item's completion is
      // the latest one the barrier can have seen: the next one on it needs
      // this item's MMAs, which need this group's decode below.
      if (rel >= G) {
        const int prev = rel - G;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(idone_bar + prev % SX), (uint32_t)(prev / SX) & 1u, p.err,
                                               DEV_TIMEOUT_MMA)))
          return false;
      }
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (j >= nkb) break;
        const uint32_t q[8] = {qv[2 * j].x, qv[2 * j].y, qv[2 * j].z, qv[2 * j].w,
                               qv[2 * j + 1].x, qv[2 * j + 1].y, qv[2 * j + 1].z, qv[2 * j + 1].w};
        uint32_t e[32];
#pragma unroll
        for (int w = 0; w < 8; ++w)
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t v = __byte_perm(q[w], 0u, 0x4440u | (uint32_t)b);   // code byte b, zero-extended
            e[4 * w + b] = mul_round_bf16x2(lds64(lut_lane + v * 128u), c2[j]);
          }
        tmem_st_32x32b_x32(a_row + 32 * j, e);
      }
      tmem_wait_st();
      tc_fence_before();
      // the item's X tile has landed too (the MMA issuer does not wait for it)
      const int xs = rel % SX;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(xfull_bar + xs), (uint32_t)(rel / SX) & 1u, p.err,
                                             DEV_TIMEOUT_MMA)))
        return false;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(afull_bar + g));   // A slot written, X landed
      return true;
    };
    uint4 ra = raw_of(0), rb = raw_of(1);
    for (int u = 0; i0 + g + u * G < i1; u += 2) {
      if (!item(u, ra)) break;
      if (i0 + g + (u + 1) * G >= i1 || !item(u + 1, rb)) break;
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp;              // TMEM lane quarter
    int t = 0;
    for (int it = i0; it < i1; ++it) {
      int l, rt, ks;
      const DfMember &m = df_item<GM>(p, it, l, rt, ks);
      if (!(it == i1 - 1 || ks == m.kstages - 1)) continue;   // not the end of a row-tile segment
      const int acc = t & 1;
      const bool got = mbar_wait(smem_u32(tfull_bar + acc), (t >> 1) & 1u, p.err, DEV_TIMEOUT_EPILOGUE);
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      tc_fence_after();
      const int n = rt * kDfRows + q * 32 + lane;
#pragma unroll 1
      for (int cc = 0; cc < MP; cc += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * MP + cc), r);
        tmem_wait_ld();
        if (n < m.N) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (cc + i < p.M) red_add_f32(m.acc + (int64_t)(cc + i) * m.N + n, __uint_as_float(r[i]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(tempty_bar + acc));
      ++t;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == Cfg::kMmaWarp) tmem_dealloc(tmem_base, Cfg::kTmemCols);
  // Complete only after the T launch this grid overlapped has completed, so
  // that the epilogue launched after this grid sees T.
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace qlora
