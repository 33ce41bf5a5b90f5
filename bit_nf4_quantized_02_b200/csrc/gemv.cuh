// Fused doubleDequant + product for few tokens (QLoRA §3 Eq. 5 / Eq. 6 at
// decode-sized M): the frozen-weight bytes dominate, so every NF4 weight is
// read once from HBM and decoded in registers straight into tensor-core
// fragments -- no bf16 copy of the weight is ever written.
//
//   Y[M x N] = bf16( X W_hat^T + (s X L1) L2 ),   M <= 8*NT (NT in {1, 2, 4})
//
// Three launches per call (one linear or a group of them, below), chained
// with programmatic dependent launch:
//   lora_down_small_kernel   adds K-slices of X L1 into an fp32 accumulator;
//   gemv_fwd_kernel          streams the weight and adds X W_hat^T into an fp32
//                            [M x N] accumulator (does not need T, so it
//                            overlaps the first kernel completely);
//   gemv_epilogue_kernel     Y = bf16(acc + s T L2), and T = s X L1 as a bf16
//                            hi/lo pair for the backward.
// gemv_fwd_kernel, persistent, 160 threads per CTA (4 CTAs per SM up to 16
// tokens, 3 at 32):
//   * warp 4 is a TMA producer: per stage, 64 weight rows x 256 K of packed
//     codes (128-byte swizzle) and the matching X tile (3-D view of X,
//     [token][64-block][64], 128-byte swizzle) into a ring of mbarrier stages;
//   * warps 0..3 each own 16 weight rows.  Lane (g, j) decodes rows g and g+8
//     of NF4 block j of the stage -- 64 weights per row, all under one
//     constant -- through a 16-entry bf16 table T_b[c] = bf16(NF4[c] * c2_hat)
//     (bit-identical to qlora_dequant) held as byte planes and indexed with
//     byte permutes, and feeds them as the A operand of mma.sync m16n8k16
//     (bf16 in, fp32 accumulate) against X as the B operand.
//   * The K positions inside a stage are permuted consistently for A and B:
//     logical k-step s, slot u of lane-column j <-> physical k = 64 j + 4 s + u,
//     so each lane's codes are one contiguous 32-byte run per row and its X
//     operand is one 16-byte run per two steps; both are bank-conflict free
//     under the 128-byte swizzle.
//   * A unit is 64 rows x 512 K; partial products are added into an fp32
//     [M x N] accumulator with red.global.add (L2 resident); all CTAs do the
//     same amount of work (no per-block finishing step on the critical path).
// The two accumulators must be zero at launch (the host clears them with one
// memset in stream order).  Split-K additions make the low bits of Y depend
// on the order in which CTAs finish.
//
// Groups: one chain of the three launches may serve up to kMaxGroup linears
// that see the same tokens (GM > 1; e.g. the seven projections of a decoder
// layer, whose launch gaps and per-linear tails it removes).  Their units
// (T slices, weight units, output column slices) are concatenated into one
// flat list per kernel; a unit finds its linear from the list's start
// offsets, then its place in that linear with a multiply-high by a divisor
// fixed at launch (DivU31).  A single linear is a group of one (GM = 1).
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace qlora {

constexpr int kGvRows = 64;          // weight rows per unit (4 warps x 16)
constexpr int kGvStageK = 256;       // K per pipeline stage
constexpr int kGvUnitK = 512;        // K per unit (2 stages)
constexpr int kGvThreads = 160;      // 4 decode/MMA warps + 1 producer warp
constexpr int kGvMaxM = 32;

template <int NT>
struct GvCfg {
  static constexpr int kCodeBytes = kGvRows * 128;          // 64 rows x 256 codes
  static constexpr int kXBytes = 8 * NT * kGvStageK * 2;    // padded tokens x 256 bf16
  static constexpr int kStageBytes = kCodeBytes + kXBytes;
  // 4 CTAs per SM (at most 48 KB and 96 registers each) up to 16 tokens; at
  // 32 tokens the register cap would spill, so 3 CTAs of 72 KB.
  static constexpr int kCtasPerSm = NT == 4 ? 3 : 4;
  static constexpr int kStages = NT == 1 ? 4 : 3;
  // + 1024 alignment slack + 256 barrier area
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;
};

constexpr int kMaxGroup = 8;         // linears per group launch

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

struct GvMember {
  int N, K;
  int nks;               // units per 64-row block
  DivU31 nks_div;        // division by nks
  const uint8_t *c2_fp8;
  const float *c1;
  const float *mu;
  float *acc;            // [M x N] fp32, zero at launch
};

template <int GM>
struct GvArgs {
  int M;
  int count;             // linears in the group
  int units;             // units of all of them
  int beg[GM];           // first unit of each linear
  GvMember m[GM];
  float levels[16];      // the 16-level code table (shared by the group)
  int *err;
};

// Per linear: its packed codes [N x K/2] in boxes of 64 rows x 128 bytes, and
// X as [token][64-block][64] in boxes of 8 NT tokens x 4 blocks.
template <int GM>
struct GvMaps {
  CUtensorMap codes[GM];
  CUtensorMap x[GM];
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// prmt in its default mode, where a selector nibble with bit 3 set replicates
// the sign bit of the selected byte.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void red_add_f32(float *p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// Release/acquire fence at GPU scope (lighter than the sequentially
// consistent fence of __threadfence()).
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }


// The 16 decoded values of one 64-block, bf16(NF4[c] * c2_hat), stored as two
// byte planes: lo[i] holds the low bytes of entries 4i..4i+3, hi[i] the high
// bytes.
struct BlockTable {
  uint32_t lo[4], hi[4];
  __device__ __forceinline__ void build(float c2h, const float *levels) {
    uint32_t e[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat162 p = __floats2bfloat162_rn(__fmul_rn(levels[2 * i], c2h), __fmul_rn(levels[2 * i + 1], c2h));
      e[i] = *reinterpret_cast<const uint32_t *>(&p);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lo[i] = __byte_perm(e[2 * i], e[2 * i + 1], 0x6420);
      hi[i] = __byte_perm(e[2 * i], e[2 * i + 1], 0x7531);
    }
  }
  // Four codes (nibbles of the low 16 bits of `sel7`, bit 3 cleared) whose
  // bit-3 flags are the byte mask `m8` -> two bf16x2 words {T[c0],T[c1]},
  // {T[c2],T[c3]}.
  __device__ __forceinline__ void lookup4(uint32_t sel7, uint32_t m8, uint32_t &p01, uint32_t &p23) const {
    const uint32_t la = __byte_perm(lo[0], lo[1], sel7);
    const uint32_t lb = __byte_perm(lo[2], lo[3], sel7);
    const uint32_t ha = __byte_perm(hi[0], hi[1], sel7);
    const uint32_t hb = __byte_perm(hi[2], hi[3], sel7);
    const uint32_t l = (lb & m8) | (la & ~m8);
    const uint32_t h = (hb & m8) | (ha & ~m8);
    p01 = __byte_perm(l, h, 0x5140);
    p23 = __byte_perm(l, h, 0x7362);
  }
};

// Raw constants of a lane's two (row, block) pairs for one (unit, stage) item.
struct ConstPrefetch {
  uint32_t code8[2];
  float c1[2];
  float mu;
  bool ok[2];
  template <int GM>
  __device__ __forceinline__ void load(const GvArgs<GM> &p, int u, int st, int r0, int j) {
    ok[0] = ok[1] = false;
    code8[0] = code8[1] = 0;
    c1[0] = c1[1] = 0.f;
    mu = 0.f;
    if (u >= p.units) return;
    const int l = group_member<GM>(p.beg, p.count, u);
    const GvMember &m = p.m[l];
    const int lu = u - p.beg[l];
    const int rb = (int)m.nks_div.div((uint32_t)lu), ks = lu - rb * m.nks;
    const int kblocks = m.K >> 6;
    const int kb = ((ks * kGvUnitK + st * kGvStageK) >> 6) + j;
    if (kb >= kblocks) return;
    mu = __ldg(m.mu);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int n = rb * kGvRows + r0 + 8 * i;
      if (n < m.N) {
        const int64_t b = (int64_t)n * kblocks + kb;
        code8[i] = __ldg(m.c2_fp8 + b);
        c1[i] = __ldg(m.c1 + (b >> 8));
        ok[i] = true;
      }
    }
  }
  __device__ __forceinline__ float c2hat(int i) const {
    return ok[i] ? __fmaf_rn(e4m3_to_f32((uint8_t)code8[i]), c1[i], mu) : 0.f;
  }
};

// State of one decode/MMA warp of gemv_fwd_kernel.
template <int NT, int GM>
struct GvConsumer {
  using Cfg = GvCfg<NT>;
  const GvArgs<GM> *p;
  uint8_t *smem;
  uint64_t *full_bar, *empty_bar;
  int g, j, r0, lane;
  int stage;
  uint32_t phase;
  int u, st;
  float d[2][NT][4];  // two accumulator chains (even / odd k-steps)

  __device__ __forceinline__ void init(const GvArgs<GM> &pp, uint8_t *sm, uint64_t *fb, uint64_t *eb) {
    p = &pp;
    smem = sm;
    full_bar = fb;
    empty_bar = eb;
    lane = lane_id();
    g = lane >> 2;
    j = lane & 3;
    r0 = warp_id() * 16 + g;
    stage = 0;
    phase = 0;
    u = blockIdx.x;
    st = 0;
  }

  // Process item (u, st) whose constants are in `cur`; start loading the next
  // item's constants into `nxt`.  Returns false on a pipeline timeout.
  __device__ __forceinline__ bool item(const ConstPrefetch &cur, ConstPrefetch &nxt) {
    const GvArgs<GM> &P = *p;
    const int l = group_member<GM>(P.beg, P.count, u);
    const GvMember &m = P.m[l];
    const int lu = u - P.beg[l];
    const int rb = (int)m.nks_div.div((uint32_t)lu), ks = lu - rb * m.nks;
    const int kbeg = ks * kGvUnitK;
    const int nst = min(kGvUnitK, m.K - kbeg) > kGvStageK ? 2 : 1;
    const int n0 = rb * kGvRows + r0, n1 = n0 + 8;
    if (st == 0) {
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int t = 0; t < NT; ++t) d[c][t][0] = d[c][t][1] = d[c][t][2] = d[c][t][3] = 0.f;
    }
    BlockTable tb0, tb1;
    tb0.build(cur.c2hat(0), P.levels);
    tb1.build(cur.c2hat(1), P.levels);
    int nu = u, nstn = st + 1;
    if (nstn == nst) {
      nu = u + gridDim.x;
      nstn = 0;
    }
    nxt.load(P, nu, nstn, r0, j);
    if (!mbar_wait(smem_u32(full_bar + stage), phase, P.err, DEV_TIMEOUT_MMA)) return false;
    const uint32_t sc = smem_u32(smem + stage * Cfg::kStageBytes);
    const uint32_t sx = sc + Cfg::kCodeBytes;
    // codes of rows r0, r0+8: 16-byte chunks 2j, 2j+1 of their 128-byte lines
    uint32_t q0[8], q1[8];
    {
      const uint4 a = lds128(sc + r0 * 128 + (((2 * j) ^ (r0 & 7)) << 4));
      const uint4 b = lds128(sc + r0 * 128 + (((2 * j + 1) ^ (r0 & 7)) << 4));
      const uint4 c = lds128(sc + (r0 + 8) * 128 + (((2 * j) ^ (r0 & 7)) << 4));
      const uint4 e = lds128(sc + (r0 + 8) * 128 + (((2 * j + 1) ^ (r0 & 7)) << 4));
      q0[0] = a.x; q0[1] = a.y; q0[2] = a.z; q0[3] = a.w; q0[4] = b.x; q0[5] = b.y; q0[6] = b.z; q0[7] = b.w;
      q1[0] = c.x; q1[1] = c.y; q1[2] = c.z; q1[3] = c.w; q1[4] = e.x; q1[5] = e.y; q1[6] = e.z; q1[7] = e.w;
    }
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      // X operand for steps 2w, 2w+1: token g + 8t, line (token*4 + j), chunk w
      uint4 xb[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const int line = (g + 8 * t) * 4 + j;
        xb[t] = lds128(sx + line * 128 + ((w ^ (line & 7)) << 4));
      }
      const uint32_t m0 = q0[w] & 0x77777777u, m1 = q1[w] & 0x77777777u;
      const uint32_t s0 = q0[w] << 4, s1 = q1[w] << 4;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t a[4];
        const uint32_t msel = h ? 0xFBEAu : 0xD9C8u;
        tb0.lookup4(h ? (m0 >> 16) : m0, prmt(s0, q0[w], msel), a[0], a[2]);
        tb1.lookup4(h ? (m1 >> 16) : m1, prmt(s1, q1[w], msel), a[1], a[3]);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint32_t b0 = h ? xb[t].z : xb[t].x;
          const uint32_t b1 = h ? xb[t].w : xb[t].y;
          mma_bf16_16816(d[h][t], a, b0, b1);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(empty_bar + stage));
    if (++stage == Cfg::kStages) {
      stage = 0;
      phase ^= 1;
    }
    if (st == nst - 1) {
      // the unit is complete: add its partial products into the accumulator
      float *acc = m.acc;
      const int N = m.N;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const int tok = 8 * t + 2 * j;
        const float v0 = d[0][t][0] + d[1][t][0], v1 = d[0][t][1] + d[1][t][1];
        const float v2 = d[0][t][2] + d[1][t][2], v3 = d[0][t][3] + d[1][t][3];
        if (tok < P.M) {
          if (n0 < N) red_add_f32(acc + (int64_t)tok * N + n0, v0);
          if (n1 < N) red_add_f32(acc + (int64_t)tok * N + n1, v2);
        }
        if (tok + 1 < P.M) {
          if (n0 < N) red_add_f32(acc + (int64_t)(tok + 1) * N + n0, v1);
          if (n1 < N) red_add_f32(acc + (int64_t)(tok + 1) * N + n1, v3);
        }
      }
    }
    u = nu;
    st = nstn;
    return true;
  }
};

template <int NT, int GM>
__global__ void __launch_bounds__(kGvThreads, GvCfg<NT>::kCtasPerSm)
    gemv_fwd_kernel(const __grid_constant__ GvMaps<GM> maps, const __grid_constant__ GvArgs<GM> p) {
  using Cfg = GvCfg<NT>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + S * Cfg::kStageBytes);
  uint64_t *empty_bar = full_bar + S;

  const int warp = warp_id();
  const int lane = lane_id();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the epilogue may launch and wait

  // ---------------------------------------------------------------- main loop
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(full_bar + i), 1);
      mbar_init(smem_u32(empty_bar + i), 4);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // Lane 0 drives the TMA ring; all lanes prefetch the next stage's block
    // constants (one code8 run per weight row) into L2 for the decode warps.
    if (lane < p.count) {
      tma_prefetch_desc(&maps.codes[lane]);
      tma_prefetch_desc(&maps.x[lane]);
    }
    int stage = 0;
    uint32_t phase = 0, used = 0, last_parity = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      const int l = group_member<GM>(p.beg, p.count, u);
      const GvMember &m = p.m[l];
      const int lu = u - p.beg[l];
      const int rb = (int)m.nks_div.div((uint32_t)lu), ks = lu - rb * m.nks;
      const int kbeg = ks * kGvUnitK;
      const int nst = min(kGvUnitK, m.K - kbeg) > kGvStageK ? 2 : 1;
      const int kblocks = m.K >> 6;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int n = rb * kGvRows + lane + 32 * i;
        if (n < m.N) asm volatile("prefetch.global.L2 [%0];" ::"l"(m.c2_fp8 + (int64_t)n * kblocks + (kbeg >> 6)));
      }
      for (int st = 0; st < nst; ++st) {
        bool got = true;
        if (lane == 0) {
          got = mbar_wait(smem_u32(empty_bar + stage), phase ^ 1, p.err, DEV_TIMEOUT_PRODUCER);
          if (got) {
            const uint32_t fb = smem_u32(full_bar + stage);
            mbar_arrive_expect_tx(fb, Cfg::kStageBytes);
            const uint32_t sc = smem_u32(smem + stage * Cfg::kStageBytes);
            const int k0 = kbeg + st * kGvStageK;
            tma_load_2d(sc, &maps.codes[l], fb, k0 >> 1, rb * kGvRows);
            asm volatile(
                "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
                "%5}], [%2];" ::"r"(sc + Cfg::kCodeBytes),
                "l"(reinterpret_cast<uint64_t>(&maps.x[l])), "r"(fb), "r"(0), "r"(k0 >> 6), "r"(0)
                : "memory");
            used |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
        }
        if (!__shfl_sync(0xFFFFFFFFu, got ? 1 : 0, 0)) {
          ok = false;
          break;
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    if (lane == 0)
      for (int i = 0; i < S; ++i)
        if (used & (1u << i)) mbar_wait(smem_u32(full_bar + i), (last_parity >> i) & 1u, p.err, DEV_TIMEOUT_DRAIN);
  } else {
    GvConsumer<NT, GM> c;
    c.init(p, smem, full_bar, empty_bar);
    // Flat walk over this CTA's (unit, stage) items, unrolled by two so the
    // block constants of the next item load into the other buffer (no copies
    // of in-flight loads) while the current item is decoded.
    ConstPrefetch pa, pb;
    pa.load(p, c.u, c.st, c.r0, c.j);
    while (c.u < p.units) {
      if (!c.item(pa, pb)) break;
      if (c.u >= p.units || !c.item(pb, pa)) break;
    }
  }
  // Complete only after the T launch this grid overlapped has completed, so
  // that the epilogue launched after this grid sees T.
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
__global__ void __launch_bounds__(256) gemv_epilogue_kernel(const __grid_constant__ EpArgs<GM> a) {
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
