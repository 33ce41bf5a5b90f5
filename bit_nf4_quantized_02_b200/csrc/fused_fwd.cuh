// Fused doubleDequant + tensor-core product for up to 128 tokens (QLoRA §3
// Eq. 5 with the frozen weight decoded on the fly, Eq. 6): the NF4 weight is
// streamed from HBM once, decoded to bf16 in shared memory and consumed there
// by tcgen05 MMAs -- no bf16 copy of the weight is ever written to HBM.
//
//   acc[M x N] += X W_hat^T        (fp32, L2-resident; zero at launch)
//
// computed transposed, acc^T = W_hat X^T, so that the weight rows are the
// 128-row MMA M dimension and the tokens the MMA N dimension (MP = tokens
// padded to 16, 32, 64 or 128).  The LoRA branch and the bf16 output come
// from the kernels around it: lora_down_small_kernel before (this kernel is
// its programmatic dependent and runs alongside it) and gemv_epilogue_kernel
// after.
//
// One persistent CTA per SM (4G + 6 warps, G = 4 decoder groups, 2 at 128
// tokens where shared memory is tighter):
//   warp 4G+4    producer: lane 0 loads, per stage, 128 weight rows x 256 K
//                of packed codes (128-byte swizzle) and the X tile of those
//                256 K as four K-major 128-byte-swizzled atoms of MP tokens
//                (one 3-D box) with TMA; all lanes copy the stage's raw
//                block constants (E4M3 codes, c1) into it with cp.async;
//   warps 0..4G-1 decoders, G groups of four: group g decodes the 64-blocks
//                j = g, g + G, ... of every stage; thread t of a group owns
//                weight row t.  A block's 64 weights share one constant, so
//                the thread builds the block's 16-entry table bf16(NF4[c] *
//                c2_hat) (bit-identical to qlora_dequant), looks the codes up
//                with byte permutes into registers, and stores the 128-byte
//                bf16 row into the group's next A slot (canonical K-major
//                layout without swizzle: 8-row x 16-byte core matrices) once
//                the tensor core has read the slot's previous block, then makes it visible to the tensor core
//                (fence.proxy.async) and signals the MMA warp;
//                the block constant c2_hat = fma(E4M3(code8), c1, mu) is
//                formed from the stage's raw constants;
//   warp 4G+5    allocates TMEM; one thread issues tcgen05.mma (M = 128,
//                N = MP, K = 16; bf16 in, fp32 accumulate) from the A slots
//                and the X atoms into one of two TMEM accumulators;
//   warps 4G..4G+3 epilogue: tcgen05.ld of the accumulator (lane = weight row,
//                column = token) and red.global.add into acc.
// Work: the (128-row tile, 256-K stage) items of the weight are split into
// equal contiguous ranges, one per CTA; a CTA adds its partial sums into acc
// whenever its range moves to the next row tile, and at its end.  A group of
// linears that see the same tokens (GM > 1) concatenates their items, linear
// after linear; a row tile never spans two linears, so the accumulator
// hand-off is unchanged.
#pragma once

#include "common.cuh"
#include "quant.cuh"
#include "gemv.cuh"

namespace qlora {

constexpr int kFtRows = 128;            // weight rows per tile (MMA M, TMEM lanes)
constexpr int kFtStageK = 256;          // K per TMA stage: four 64-blocks
constexpr int kFtMaxM = 128;

// Decoder groups: group g (four warps, thread t = weight row t) decodes the
// 64-blocks j = g, g + G, ... of every stage into its own ring of A slots, so
// each slot has a single writer and its barriers never run more than one
// phase ahead of a waiter.
template <int MP>
struct FtCfg {
  static_assert(MP == 16 || MP == 32 || MP == 64 || MP == 128, "MMA N");
  static constexpr int kGroups = MP == 128 ? 2 : 4;
  static constexpr int kDecWarps = 4 * kGroups;
  static constexpr int kEpiWarp0 = kDecWarps;                 // four epilogue warps
  static constexpr int kProdWarp = kDecWarps + 4;
  static constexpr int kMmaWarp = kDecWarps + 5;
  static constexpr int kThreads = 32 * (kDecWarps + 6);
  static constexpr int kCodeBytes = kFtRows * 128;            // 128 rows x 256 codes
  static constexpr int kXBytes = 4 * MP * 128;                // 4 atoms of MP rows x 64 bf16
  static constexpr int kCstBytes = kFtRows * 16;              // raw block constants of 128 rows
  static constexpr int kStageBytes = kCodeBytes + kXBytes + kCstBytes;
  static constexpr int kABytes = kFtRows * 128;               // 128 rows x 64 bf16
  static constexpr int kSlots = 1;                            // A slots per decoder group
  static constexpr int kStages = MP <= 32 ? 4 : (MP == 64 ? 3 : 2);
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kStages * kStageBytes + kGroups * kSlots * kABytes + kBarBytes + 1024;
  static constexpr int kTmemCols = 2 * MP <= 32 ? 32 : (2 * MP <= 64 ? 64 : (2 * MP <= 128 ? 128 : 256));
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

struct FtMember {
  int N, K;
  int kstages;           // ceil(K / 256)
  DivU31 ks_div;         // division by kstages
  const uint8_t *c2_fp8;
  const float *c1;
  const float *mu;
  float *acc;            // [M x N] fp32, zero at launch
};

// A group of linears that see the same tokens: their (row tile, stage) items
// are concatenated, linear after linear (see the group note in gemv.cuh).
template <int GM>
struct FtArgs {
  int M;
  int count;             // linears in the group
  int items;             // row tiles x kstages, summed over the group
  int beg[GM];           // first item of each linear
  FtMember m[GM];
  float levels[16];      // the 16-level code table (shared by the group)
  int *err;
};

// Per linear: its packed codes in boxes of 128 rows x 128 bytes, and X as
// [64-block][token][64] in boxes of the four atoms of a stage.
template <int GM>
struct FtMaps {
  CUtensorMap codes[GM];
  CUtensorMap x[GM];
};

// Item `it` of a group -> its linear l, row tile rt and stage ks.
template <int GM>
__device__ __forceinline__ const FtMember &ft_item(const FtArgs<GM> &p, int it, int &l, int &rt, int &ks) {
  l = group_member<GM>(p.beg, p.count, it);
  const FtMember &m = p.m[l];
  const int li = it - p.beg[l];
  rt = (int)m.ks_div.div((uint32_t)li);
  ks = li - rt * m.kstages;
  return m;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Generic-proxy shared-memory writes -> visible to the async proxy (tensor core).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
__device__ __forceinline__ void ft_range(int items, int b, int g, int &i0, int &i1) {
  i0 = (int)(((int64_t)items * b) / g);
  i1 = (int)(((int64_t)items * (b + 1)) / g);
}

// 4-byte global -> shared copy, completed asynchronously (cp.async).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// Arrive on `bar` once this thread's earlier cp.async copies have landed (the
// arrival counts toward the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Raw block constants of one weight row for one stage (16 bytes in the stage's
// constant area): the two aligned 32-bit words of c2_fp8 holding the row's four
// E4M3 codes (byte (n * kblocks + kb0) & 3 of the first word is block kb0), and
// c1 of the first and the last of those blocks (they differ when the row's
// blocks straddle a 256-group).  Producer lane `lane` fills rows lane + 32 i.
__device__ __forceinline__ void ft_copy_consts(const FtMember &p, uint32_t area, int rt, int ks, int lane) {
  const int kblocks = p.K >> 6;
  const int kb0 = ks * 4;
  const int nb = min(4, kblocks - kb0);
  const int64_t nblk = (int64_t)p.N * kblocks;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = lane + 32 * i;
    const int n = rt * kFtRows + row;
    if (n >= p.N) continue;
    const uint32_t dst = area + row * 16;
    const int64_t b0 = (int64_t)n * kblocks + kb0;
    const int64_t w0 = b0 >> 2;
    const int64_t last = b0 + nb - 1;                 // last block read
    const int nw = (last >> 2) == w0 ? 1 : 2;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (k >= nw) break;
      const int64_t w = w0 + k;
      if (4 * w + 3 < nblk) {
        cp_async4(dst + 4 * k, p.c2_fp8 + 4 * w);
      } else {
        // the array ends inside this word: byte loads, no read past its end
        uint32_t v = 0;
        for (int64_t b = 4 * w; b < nblk; ++b) v |= (uint32_t)__ldg(p.c2_fp8 + b) << (8 * (int)(b - 4 * w));
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(dst + 4 * k), "r"(v) : "memory");
      }
    }
    cp_async4(dst + 8, p.c1 + (b0 >> 8));
    cp_async4(dst + 12, p.c1 + (last >> 8));
  }
}

// c2_hat of block kb0 + j of weight row n from its raw constants (j < 4, the
// block inside the weight).
__device__ __forceinline__ float ft_c2hat(uint4 raw, int n, int kb0, int j, int kblocks, float mu) {
  const int64_t b0 = (int64_t)n * kblocks + kb0;
  const int sh = (int)(b0 & 3) + j;                  // byte index in the 8-byte pair
  const uint32_t code8 = (sh < 4 ? raw.x >> (8 * sh) : raw.y >> (8 * (sh - 4))) & 0xFFu;
  const float c1 = ((b0 + j) >> 8) == (b0 >> 8) ? __uint_as_float(raw.z) : __uint_as_float(raw.w);
  return __fmaf_rn(e4m3_to_f32((uint8_t)code8), c1, mu);
}

template <int MP, int GM>
__global__ void __launch_bounds__(FtCfg<MP>::kThreads, 1)
    nf4_fused_fwd_kernel(const __grid_constant__ FtMaps<GM> maps, const __grid_constant__ FtArgs<GM> p) {
  using Cfg = FtCfg<MP>;
  constexpr int S = Cfg::kStages;
  constexpr int G = Cfg::kGroups;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int R = Cfg::kSlots;
  uint8_t *a_area = smem + S * Cfg::kStageBytes;                 // R A slots per decoder group
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(a_area + G * R * Cfg::kABytes);
  uint64_t *empty_bar = full_bar + S;
  uint64_t *afull_bar = empty_bar + S;                  // [G * R]
  uint64_t *aempty_bar = afull_bar + G * R;             // [G * R]
  uint64_t *tfull_bar = aempty_bar + G * R;             // [2]
  uint64_t *tempty_bar = tfull_bar + 2;                 // [2]
  uint64_t *done_bar = tempty_bar + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);

  const int warp = warp_id();
  const int lane = lane_id();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the epilogue may launch and wait

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(full_bar + i), 1 + 32);             // TMA bytes + the producer lanes' constants
      mbar_init(smem_u32(empty_bar + i), Cfg::kDecWarps + 1);   // decoders done with codes/constants + MMAs with X
    }
    for (int i = 0; i < G * R; ++i) {
      mbar_init(smem_u32(afull_bar + i), 4);                 // the four warps of a decoder group
      mbar_init(smem_u32(aempty_bar + i), 1);
    }
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
  ft_range(p.items, blockIdx.x, gridDim.x, i0, i1);

  if (warp == Cfg::kProdWarp) {
    // ------------------------------------------------------------ producer
    // Lane 0 drives the TMA ring; every lane copies the raw block constants of
    // rows lane + 32 i of the stage into its constant area asynchronously and
    // arrives on the stage's full barrier when they have landed.
    if (lane < p.count) {
      tma_prefetch_desc(&maps.codes[lane]);
      tma_prefetch_desc(&maps.x[lane]);
    }
    int stage = 0;
    uint32_t phase = 0, used = 0, last_parity = 0;
    for (int it = i0; it < i1; ++it) {
      int l, rt, ks;
      const FtMember &m = ft_item<GM>(p, it, l, rt, ks);
      const bool got = mbar_wait(smem_u32(empty_bar + stage), phase ^ 1, p.err, DEV_TIMEOUT_PRODUCER);
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      const uint32_t fb = smem_u32(full_bar + stage);
      const uint32_t sc = smem_u32(smem + stage * Cfg::kStageBytes);
      if (lane == 0) {
        mbar_arrive_expect_tx(fb, Cfg::kCodeBytes + Cfg::kXBytes);
        tma_load_2d(sc, &maps.codes[l], fb, ks * (kFtStageK / 2), rt * kFtRows);
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
            "[%2];" ::"r"(sc + Cfg::kCodeBytes),
            "l"(reinterpret_cast<uint64_t>(&maps.x[l])), "r"(fb), "r"(0), "r"(0), "r"(ks * 4)
            : "memory");
      }
      used |= 1u << stage;
      last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
      ft_copy_consts(m, sc + Cfg::kCodeBytes + Cfg::kXBytes, rt, ks, lane);
      cp_async_arrive_noinc(fb);
      if (++stage == S) {
        stage = 0;
        phase ^= 1;
      }
    }
    // Drain: every lane's copies and lane 0's tensor copies have landed once
    // the last phase of each used stage has completed.
    for (int i = 0; i < S; ++i)
      if (used & (1u << i)) {
        const bool done = mbar_wait(smem_u32(full_bar + i), (last_parity >> i) & 1u, p.err, DEV_TIMEOUT_DRAIN);
        if (!__all_sync(0xFFFFFFFFu, done)) break;
      }
  } else if (warp == Cfg::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kFtRows, MP, 0, 0);
      const uint32_t a0 = smem_u32(a_area);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t reads[G];       // slots read per group: the next read waits for write number reads[g]
#pragma unroll
      for (int g = 0; g < G; ++g) reads[g] = 0;
      int t = 0;               // segments (row tiles) started
      bool ok = true;
      uint32_t accumulate = 0;
      for (int it = i0; it < i1 && ok; ++it) {
        int l, rt, ks;
        const FtMember &m = ft_item<GM>(p, it, l, rt, ks);
        const int kblocks = m.K >> 6;
        const bool first = it == i0 || ks == 0;
        const bool last = it == i1 - 1 || ks == m.kstages - 1;
        const int acc = t & 1;
        if (first) {
          if (!mbar_wait(smem_u32(tempty_bar + acc), ((t >> 1) & 1u) ^ 1u, p.err, DEV_TIMEOUT_MMA)) break;
          tc_fence_after();
          accumulate = 0;
        }
        if (!mbar_wait(smem_u32(full_bar + stage), phase, p.err, DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t sx = smem_u32(smem + stage * Cfg::kStageBytes) + Cfg::kCodeBytes;
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * MP);
        const int nkb = min(4, kblocks - ks * 4);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (j >= nkb) break;
          const int g = j % G;
          const int slot = g * R + (int)(reads[g] % R);
          if (!mbar_wait(smem_u32(afull_bar + slot), (reads[g] / R) & 1u, p.err, DEV_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = a0 + slot * Cfg::kABytes;
          const uint32_t sb = sx + j * (MP * 128);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // A: no swizzle, K-adjacent core matrices 128 B apart, 8-row groups 1 KB apart
            tc_mma_f16(d_tmem, smem_desc_noswz(sa + k * 256, 128, 1024), smem_desc_sw128(sb + k * 32, 16, 1024),
                       idesc, accumulate);
            accumulate = 1;
          }
          tc_commit(smem_u32(aempty_bar + slot));   // slot free once these MMAs have read it
          ++reads[g];
        }
        if (!ok) break;
        tc_commit(smem_u32(empty_bar + stage));      // X tile consumed
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
        if (last) {
          tc_commit(smem_u32(tfull_bar + acc));      // partial sums of this row tile ready
          ++t;
        }
      }
      tc_commit(smem_u32(done_bar));
      mbar_wait(smem_u32(done_bar), 0, p.err, DEV_TIMEOUT_DRAIN);
    }
  } else if (warp < Cfg::kDecWarps) {
    // ------------------------------------------------------------ decoders
    const int g = warp >> 2;                      // 64-blocks j = g, g + G, ... of every stage
    const int t = (warp & 3) * 32 + lane;         // weight row within the tile
    const uint32_t sa0 = smem_u32(a_area) + g * R * Cfg::kABytes + (t >> 3) * 1024 + (t & 7) * 16;  // row t, chunk 0
    const uint32_t cswz = (uint32_t)(t & 7) << 4;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t writes = 0;     // blocks this group has stored into its slot
    for (int it = i0; it < i1; ++it) {
      int l, rt, ks;
      const FtMember &m = ft_item<GM>(p, it, l, rt, ks);
      const int kblocks = m.K >> 6;
      const float mu = __ldg(m.mu);
      const int nkb = min(4, kblocks - ks * 4);
      const bool got = mbar_wait(smem_u32(full_bar + stage), phase, p.err, DEV_TIMEOUT_MMA);
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      const uint32_t sc = smem_u32(smem + stage * Cfg::kStageBytes) + t * 128;
      const uint4 raw = *reinterpret_cast<const uint4 *>(smem + stage * Cfg::kStageBytes + Cfg::kCodeBytes +
                                                         Cfg::kXBytes + t * 16);
      const int n = rt * kFtRows + t;
      bool ok = true;
#pragma unroll
      for (int j = g; j < 4; j += G) {
        if (j >= nkb) break;
        // this row's 32 code bytes of block j: 16-byte chunks 2j, 2j+1 of its swizzled 128-byte line
        const uint4 qa = lds128(sc + (((uint32_t)(2 * j) << 4) ^ cswz));
        const uint4 qb = lds128(sc + (((uint32_t)(2 * j + 1) << 4) ^ cswz));
        const uint32_t q[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
        BlockTable tb;
        tb.build(n < m.N ? ft_c2hat(raw, n, ks * 4, j, kblocks, mu) : 0.f, p.levels);
        // decode the row's 64 weights into registers, then wait for the slot
        uint32_t e[32];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          const uint32_t m7 = q[w] & 0x77777777u, s4 = q[w] << 4;
          tb.lookup4(m7, prmt(s4, q[w], 0xD9C8u), e[4 * w], e[4 * w + 1]);
          tb.lookup4(m7 >> 16, prmt(s4, q[w], 0xFBEAu), e[4 * w + 2], e[4 * w + 3]);
        }
        const int slot = g * R + (int)(writes % R);
        const bool free_slot = mbar_wait(smem_u32(aempty_bar + slot), ((writes / R) & 1u) ^ 1u, p.err,
                                         DEV_TIMEOUT_MMA);
        if (!__all_sync(0xFFFFFFFFu, free_slot)) {
          ok = false;
          break;
        }
        const uint32_t sa = sa0 + (uint32_t)(writes % R) * Cfg::kABytes;
#pragma unroll
        for (int w = 0; w < 8; ++w) sts128(sa + w * 128, e[4 * w], e[4 * w + 1], e[4 * w + 2], e[4 * w + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(afull_bar + slot));
        ++writes;
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty_bar + stage));   // codes and constants of this stage consumed
      if (++stage == S) {
        stage = 0;
        phase ^= 1;
      }
    }
  } else if (warp >= Cfg::kEpiWarp0 && warp < Cfg::kEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;          // TMEM lane quarter
    int t = 0;
    for (int it = i0; it < i1; ++it) {
      int l, rt, ks;
      const FtMember &m = ft_item<GM>(p, it, l, rt, ks);
      if (!(it == i1 - 1 || ks == m.kstages - 1)) continue;   // not the end of a row-tile segment
      const int acc = t & 1;
      const bool got = mbar_wait(smem_u32(tfull_bar + acc), (t >> 1) & 1u, p.err, DEV_TIMEOUT_EPILOGUE);
      if (!__all_sync(0xFFFFFFFFu, got)) break;
      tc_fence_after();
      const int n = rt * kFtRows + q * 32 + lane;
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
