// NF4 blockwise quantizer, Double Quantization and doubleDequant kernels.
//
// QLoRA paper (aiingo.vercel.app/paper/paper-2305-14314):
//   §2 "Block-wise k-bit Quantization": flatten, cut into blocks of B, one
//      absmax constant per block (Eqs. 1-2);
//   §3 "4-bit NormalFloat Quantization" + Appendix E: the 16 NF4 levels;
//   §3 "Double Quantization": the fp32 constants c2 are mean-centred and
//      quantized to 8-bit floats in blocks of 256, giving c2_fp8 and c1;
//   §3 "QLoRA", Eq. 6: doubleDequant(c1, c2, W) = dequant(dequant(c1, c2), W).
//
// Storage format produced here (the library's on-device NF4 tensor):
//   codes   uint8 [ceil(numel/2)]  element 2i in the low nibble of byte i,
//                                  element 2i+1 in the high nibble;
//   c2_fp8  uint8 [nblk]           OCP E4M3 code of (c2_b - mu) / c1_beta;
//   c1      fp32  [ceil(nblk/256)] absmax(c2 - mu) / 448 per 256-block;
//   mu      fp32  [1]              mean of c2 over the whole tensor;
// with nblk = ceil(numel/64) and c2_b = max |w| over block b.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace qlora {

// The 16-level code tables, in code order (all exact in fp32):
//   kLevels[QLORA_TABLE_NF4]: the NF4 levels of Appendix E;
//   kLevels[QLORA_TABLE_FP4]: FP4 (E2M1), the 4-bit float of §4 (Tables 2-4)
//     that NF4 is compared against: its values {0, 0.5, 1, 1.5, 2, 3, 4, 6}
//     and their negatives divided by 6 (fp32 quotients), both zero codes +0.
// Code 7 is the exact zero of either table.
constexpr int kNumTables = 2;
#define QLORA_LEVEL_TABLES  \
    {-1.0f, \
    -0.6961928009986877f, \
    -0.5250730514526367f, \
    -0.39491748809814453f, \
    -0.28444138169288635f, \
    -0.18477343022823334f, \
    -0.09105003625154495f, \
    0.0f, \
    0.07958029955625534f, \
    0.16093020141124725f, \
    0.24611230194568634f, \
    0.33791524171829224f, \
    0.44070982933044434f, \
    0.5626170039176941f, \
    0.7229568362236023f, \
    1.0f}, \
    {-1.0f, -0x1.555556p-1f, -0.5f, -0x1.555556p-2f, -0.25f, -0x1.555556p-3f, -0x1.555556p-4f, 0.0f, \
     0.0f, 0x1.555556p-4f, 0x1.555556p-3f, 0.25f, 0x1.555556p-2f, 0.5f, 0x1.555556p-1f, 1.0f},
__constant__ float kLevels[kNumTables][16] = {QLORA_LEVEL_TABLES};
// The same tables on the host, to pass a weight's levels to the decode
// kernels as launch arguments (constant offsets in the parameter space).
static const float kLevelsHost[kNumTables][16] = {QLORA_LEVEL_TABLES};
#undef QLORA_LEVEL_TABLES

constexpr int kQuantComputeWarps = 28;                       // warps that quantize groups
constexpr int kQuantThreads = 32 * (kQuantComputeWarps + 1);  // + one producer warp
constexpr int kQuantMaxCtas = 148 * 8;                        // bound on the partial sums (one per CTA)
constexpr int kQuantChunk = 8192;                             // weights per bulk copy: 16 groups of 512
constexpr int kQuantRingBytes = 160 * 1024;

// Decision thresholds for the nearest-level search.  Level j+1 beats level j
// exactly when x exceeds their midpoint m_j = (q_j + q_{j+1}) / 2, which is
// exact in fp64; ties stay at the lower level.  For an fp32 x,
// "x > m_j"  <=>  "x > RD_fp32(m_j)", so comparing against the midpoint
// rounded toward -inf keeps the decision exact in fp32.
struct NF4Thresholds {
  float t[15];
  __device__ __forceinline__ void init(int table) {
#pragma unroll
    for (int j = 0; j < 15; ++j)
      t[j] = __double2float_rd(((double)kLevels[table][j] + (double)kLevels[table][j + 1]) * 0.5);
  }
  // code = #{ j : x > m_j } by a 4-step binary search over the sorted thresholds.
  __device__ __forceinline__ uint32_t encode(float x) const {
    const bool b3 = x > t[7];
    const float s2 = b3 ? t[11] : t[3];
    const bool b2 = x > s2;
    const float s1 = b3 ? (b2 ? t[13] : t[9]) : (b2 ? t[5] : t[1]);
    const bool b1 = x > s1;
    const float s0 = b3 ? (b2 ? (b1 ? t[14] : t[12]) : (b1 ? t[10] : t[8]))
                        : (b2 ? (b1 ? t[6] : t[4]) : (b1 ? t[2] : t[0]));
    const bool b0 = x > s0;
    return ((uint32_t)b3 << 3) | ((uint32_t)b2 << 2) | ((uint32_t)b1 << 1) | (uint32_t)b0;
  }
};

// Exact nearest-level codes without a division for almost every weight.
// [-1, 1] is cut into kCodeBins bins of width 2^-13; in bin units x sits at
// X = (x + 1) * kCodeBins / 2 and threshold t_j at P_j = (t_j + 1) *
// kCodeBins / 2.  The estimate of x = fp32(w / absmax) is E = w * sc +
// kCodeBins / 2 with sc = RN(1/absmax) * kCodeBins/2 (a power-of-two
// scaling, exact), taken with one fused multiply-add (below): w * RN(1/absmax)
// and x each carry one rounding of relative size <= 2^-24 of w / absmax,
// whose magnitude is <= 1, so |E - X| <= 8192 * 2 * 2^-24 = 2^-10.  The
// estimated bin e = floor(E) therefore puts X in (e - 2^-10, e + 1 + 2^-10).
// A bin e whose widened interval [e - d, e + 1 + d] (d = 2^-8, four times
// that bound) holds no threshold gives every x that can land in it the same
// code, #{j : P_j < e}, and that code is the table entry.  A bin whose
// widened interval holds a threshold j (thresholds are at least 341 bins
// apart, so at most one) holds kCodeBoundary | j, and its weights take the
// exact division: the code is then j + (x > t_j).  That is the bin holding
// P_j, and its neighbour only when P_j lies within d of their common edge:
// one bin per threshold in almost every case, 0.09% of the bins.
//
// The table is indexed by e + 1 so that the rounding overshoots e = -1 and
// e = kCodeBins (x within an ulp of -1 or 1) stay inside it; both hold the
// code of the end they lie at.  In shared memory it is followed by zeros up
// to kCodeLutSpan entries, the range of the 15-bit index below, so that no
// value of a weight (a NaN included) can index outside it.
constexpr int kCodeBins = 16384;
constexpr int kCodeLutEntries = kCodeBins + 2;
// Positions in fixed point, 2^16 units per bin: P_j * 2^16 = (t_j + 1) * 2^29
// is an integer below 2^30 for every threshold of magnitude >= 2^-6 or zero
// (all of both tables'), and (e + 1) * 2^16 + d stays below 2^31.
constexpr int kCodeFixBits = 16;
constexpr int kCodeFixMargin = 1 << (kCodeFixBits - 8);   // d = 2^-8 of a bin

// Each CTA builds the table in its shared memory from the same thresholds
// the exact path uses, before it waits for the kernel ahead of it (so the
// build overlaps that kernel's tail).  Entries from kCodeLutBytes on are
// zero.
//
// A warp fills 32 consecutive words (128 entries, lane l word l) per pass.
// The 128 bins of a pass with their margins span less than the gap between
// two thresholds, so at most one threshold matters to a pass: the warp
// counts the thresholds below its first bin's widened interval with one
// ballot, and a lane whose four bins lie wholly below the next threshold
// (margins included) stores that count four times; the few lanes near a
// threshold resolve their four entries one by one.
constexpr int kCodeLutBytes = (kCodeLutEntries + 3) / 4 * 4;
constexpr int kCodeLutSpan = 32768;
constexpr uint32_t kCodeBoundary = 0x80;

__device__ __forceinline__ void build_code_lut(uint8_t *lut, int table, int *pos_s) {
  if (threadIdx.x < 16) {
    int p = 0x7FFFFFFF;   // entry 15: past every bin
    if (threadIdx.x < 15) {
      const float t = __double2float_rd(((double)kLevels[table][threadIdx.x] + (double)kLevels[table][threadIdx.x + 1]) * 0.5);
      p = (int)floor(((double)t + 1.0) * (double)(1 << (13 + kCodeFixBits)));
    }
    pos_s[threadIdx.x] = p;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int my_p = lane < 15 ? pos_s[lane] : 0x7FFFFFFF;
  uint32_t *lw = reinterpret_cast<uint32_t *>(lut);
  for (int w0 = (threadIdx.x & ~31); w0 < kCodeLutSpan / 4; w0 += blockDim.x) {
    const int w = w0 + lane;
    // bin of entry i is i - 1; the pass starts at bin 4 * w0 - 1
    const int pass_lo = (4 * w0 - 1) * (1 << kCodeFixBits) - kCodeFixMargin;
    const int c = __popc(__ballot_sync(0xFFFFFFFFu, my_p < pass_lo));
    uint32_t v = 0;
    if (4 * w < kCodeLutBytes) {
      const int pc = pos_s[c];
      const int lane_hi = (4 * w + 3) * (1 << kCodeFixBits) + kCodeFixMargin;   // last bin 4w + 2, its upper edge
      if (pc > lane_hi) {
        v = (uint32_t)c * 0x01010101u;
      } else {
        const int pn = pos_s[min(c + 1, 15)];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = 4 * w + k - 1;
          const int lo = e * (1 << kCodeFixBits) - kCodeFixMargin, hi = (e + 1) * (1 << kCodeFixBits) + kCodeFixMargin;
          const bool past = pc < lo;            // threshold c lies below this bin's interval
          const int j = c + (past ? 1 : 0);     // the first threshold not below it
          const int pj = past ? pn : pc;
          const uint32_t ent = pj <= hi ? (kCodeBoundary | (uint32_t)j) : (uint32_t)j;
          v |= ent << (8 * k);
        }
      }
    }
    lw[w] = v;
  }
}

// Table index of v given sc = (1/absmax) * kCodeBins/2: the fused multiply-add
// rounded toward zero lands in [2^23, 2^24), where the low bits of the result
// are floor(v * sc + kCodeBins/2 + 1) = b + 1 exactly (2^23 has none set).
// The 15-bit mask keeps any other value (a NaN weight) inside the span.
__device__ __forceinline__ uint32_t code_lut_index(float v, float sc) {
  const float y = __fmaf_rz(v, sc, 8388608.0f + (float)(kCodeBins / 2 + 1));
  return __float_as_uint(y) & (uint32_t)(kCodeLutSpan - 1);
}

// Four table entries (bytes) -> one word, entry i in byte i.
__device__ __forceinline__ uint32_t pack_entries(uint32_t e0, uint32_t e1, uint32_t e2, uint32_t e3) {
  return __byte_perm(__byte_perm(e0, e1, 0x0040), __byte_perm(e2, e3, 0x0040), 0x5410);
}

// Eight entries in two words -> eight 4-bit codes (the low nibble of each
// entry; for a boundary entry that is its threshold index j), element i in
// bits [4i, 4i+4).
__device__ __forceinline__ uint32_t pack_nibbles(uint32_t a, uint32_t b) {
  a &= 0x0F0F0F0Fu;
  b &= 0x0F0F0F0Fu;
  a |= a >> 4;   // byte 0: e0 | e1 << 4, byte 2: e2 | e3 << 4
  b |= b >> 4;
  return __byte_perm(a, b, 0x6420);
}

// The boundary entries of four entry words in one mask: entry k of word w
// (element 4w + k of the sixteen) at bit 8k + 7 - 4 (w & 1) - (w >> 1), i.e.
// the words' flag bits 7, 3, 6 and 2 of each byte.
__device__ __forceinline__ uint32_t boundary_mask(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
  const uint32_t a = (w0 & 0x80808080u) | ((w2 & 0x80808080u) >> 1);
  const uint32_t b = (w1 & 0x80808080u) | ((w3 & 0x80808080u) >> 1);
  return a | (b >> 4);
}

// The element (0..15) of bit p of boundary_mask.
__device__ __forceinline__ int boundary_element(int p) {
  return (p >> 3) | (~p & 4) | ((~p & 1) << 3);
}

// Sixteen consecutive weights loaded from global memory (two or four 16-byte
// loads): the groups after the last whole chunk, which the last CTA
// quantizes without the ring.
template <typename TW>
struct Raw16;
template <>
struct Raw16<float> {
  float4 q[4];
  __device__ __forceinline__ void load(const float *__restrict__ p) {
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = ld_dep_f4(p + 4 * i);
  }
  __device__ __forceinline__ void unpack(float (&v)[16]) const {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[4 * i] = q[i].x; v[4 * i + 1] = q[i].y; v[4 * i + 2] = q[i].z; v[4 * i + 3] = q[i].w;
    }
  }
};
template <>
struct Raw16<__nv_bfloat16> {
  uint4 q[2];
  __device__ __forceinline__ void load(const __nv_bfloat16 *__restrict__ p) {
#pragma unroll
    for (int i = 0; i < 2; ++i) q[i] = ld_dep_v4(p + 8 * i);
  }
  __device__ __forceinline__ void unpack(float (&v)[16]) const {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t w[4] = {q[h].x, q[h].y, q[h].z, q[h].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * h + 2 * i] = __uint_as_float(w[i] << 16);
        v[8 * h + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
  }
};

// Element i (0..15, a run-time index) of the sixteen unpacked weights, by a
// select tree: the fix-up below reads it from registers, since the ring slot
// the weights came from may already be refilled (and the tail groups come
// from global memory).
__device__ __forceinline__ float select16(const float (&v)[16], int i) {
  float a[8], b[4];
#pragma unroll
  for (int k = 0; k < 8; ++k) a[k] = (i & 1) ? v[2 * k + 1] : v[2 * k];
#pragma unroll
  for (int k = 0; k < 4; ++k) b[k] = (i & 2) ? a[2 * k + 1] : a[2 * k];
  const float c0 = (i & 4) ? b[1] : b[0], c1 = (i & 4) ? b[3] : b[2];
  return (i & 8) ? c1 : c0;
}

__device__ __forceinline__ float load1(const float *p) { return ld_dep_f32(p); }
__device__ __forceinline__ float load1(const __nv_bfloat16 *p) { return __uint_as_float(ld_dep_u16(p) << 16); }

// Deterministic CTA-wide fp64 sum (fixed reduction tree).
__device__ __forceinline__ double cta_sum_f64(double v, double *scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xFFFFFFFFu, v, o);
  if (lane_id() == 0) scratch[warp_id()] = v;
  __syncthreads();
  double s = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += scratch[w];
  __syncthreads();
  return s;  // valid in thread 0
}

// K1: per 64-block absmax c2, nearest-level codes, nibble packing, and one
// fp64 partial sum of c2 per CTA (for the Double-Quantization mean).
//
// Work is in groups of eight 64-blocks (512 weights): a warp quantizes a
// group with lane l owning weights [16 l, 16 l + 16), i.e. 4 lanes per block,
// the block absmax reduced over those 4 lanes.
//
// One persistent CTA per SM.  The weights stream through shared memory: one
// producer thread keeps a ring of chunks (16 groups, 8192 weights) in flight
// with bulk copies (cp.async.bulk, completing on the slot's mbarrier) -- about
// 160 KB per SM, enough to keep HBM busy; loading each group into the
// registers of the warp that quantizes it left too few bytes in flight.  The
// 28 compute warps take the CTA's groups in turn (warp w: its groups w, w +
// 28, ...), and a slot goes back to the producer once its 16 groups are done.
// The groups after the last whole chunk are quantized by the last CTA from
// global memory, and so are the (at most eight) blocks after the last whole
// group, one warp per block.
constexpr float kTinyAbsmax = 1e-30f;   // below this 1/absmax may overflow: exact division

// Quantize one group's sixteen weights of this lane (v), whose 64-block has
// the absmax `amax` (already reduced over the block's four lanes): two words
// of packed nibble codes.
__device__ __forceinline__ void quant_lane16(const float (&v)[16], float amax, const uint8_t *lut, const float *thr,
                                             const NF4Thresholds &th, uint32_t &pk0, uint32_t &pk1) {
  pk0 = pk1 = 0x77777777u;   // all-zero block: every element is the exact-zero level
  if (amax >= kTinyAbsmax) {
    const float sc = __frcp_rn(amax) * (float)(kCodeBins / 2);
    uint32_t e[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) e[i] = lut[code_lut_index(v[i], sc)];
    const uint32_t w0 = pack_entries(e[0], e[1], e[2], e[3]), w1 = pack_entries(e[4], e[5], e[6], e[7]);
    const uint32_t w2 = pack_entries(e[8], e[9], e[10], e[11]), w3 = pack_entries(e[12], e[13], e[14], e[15]);
    pk0 = pack_nibbles(w0, w1);
    pk1 = pack_nibbles(w2, w3);
    if ((w0 | w1 | w2 | w3) & 0x80808080u) {
      // Boundary weights (a few per warp): exact division, code = j + (x > t_j).
      uint32_t m = boundary_mask(w0, w1, w2, w3);
      while (m) {
        const int i = boundary_element(__ffs(m) - 1);
        m &= m - 1;
        const int sh = 4 * (i & 7);
        uint32_t &pk = i < 8 ? pk0 : pk1;
        const uint32_t j = (pk >> sh) & 0xFu;
        const uint32_t c = j + (__fdiv_rn(select16(v, i), amax) > thr[j] ? 1u : 0u);
        pk = (pk & ~(0xFu << sh)) | (c << sh);
      }
    }
  } else if (amax != 0.f) {
    pk0 = pk1 = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      pk0 |= th.encode(__fdiv_rn(v[i], amax)) << (4 * i);
      pk1 |= th.encode(__fdiv_rn(v[8 + i], amax)) << (4 * i);
    }
  }
}

// max(a, b, c) in one instruction (three-input max.f32, sm_100); a NaN input
// is ignored as by fmaxf.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Group g of the tensor, this lane's sixteen weights in v: codes and c2 out,
// the lane's share of the c2 sum into acc.
__device__ __forceinline__ void quant_group(const float (&v)[16], int64_t g, const uint8_t *lut, const float *thr,
                                            const NF4Thresholds &th, uint8_t *__restrict__ codes,
                                            float *__restrict__ c2, double &acc) {
  const int lane = lane_id();
  const float m0 = fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2]));
  const float m1 = fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5]));
  const float m2 = fmax3(fabsf(v[6]), fabsf(v[7]), fabsf(v[8]));
  const float m3 = fmax3(fabsf(v[9]), fabsf(v[10]), fabsf(v[11]));
  const float m4 = fmax3(fabsf(v[12]), fabsf(v[13]), fabsf(v[14]));
  // (a block of NaN weights keeps c2 = 0, as the running fmaxf from 0 gave)
  float amax = fmax3(fmax3(m0, m1, m2), fmax3(m3, m4, fabsf(v[15])), 0.f);
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
  uint32_t pk0, pk1;
  quant_lane16(v, amax, lut, thr, th, pk0, pk1);
  reinterpret_cast<uint2 *>(codes)[(g << 5) + lane] = make_uint2(pk0, pk1);
  if ((lane & 3) == 0) {
    c2[(g << 3) + (lane >> 2)] = amax;
    acc += (double)amax;
  }
}

// Sixteen consecutive weights from shared memory (16-byte aligned).
template <typename TW>
__device__ __forceinline__ void lds_unpack16(uint32_t addr, float (&v)[16]);
template <>
__device__ __forceinline__ void lds_unpack16<float>(uint32_t addr, float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 q;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(q.x), "=r"(q.y), "=r"(q.z), "=r"(q.w) : "r"(addr + 16 * i));
    v[4 * i] = __uint_as_float(q.x); v[4 * i + 1] = __uint_as_float(q.y);
    v[4 * i + 2] = __uint_as_float(q.z); v[4 * i + 3] = __uint_as_float(q.w);
  }
}
template <>
__device__ __forceinline__ void lds_unpack16<__nv_bfloat16>(uint32_t addr, float (&v)[16]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t w[4];
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr + 16 * h));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * h + 2 * i] = __uint_as_float(w[i] << 16);
      v[8 * h + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

// Bulk copy global -> shared of `bytes` (multiple of 16; both addresses
// 16-byte aligned), completing on mbarrier `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

template <typename TW>
struct QuantCfg {
  static constexpr int kChunkBytes = kQuantChunk * (int)sizeof(TW);
  static constexpr int kStages = kQuantRingBytes / kChunkBytes;     // 10 (bf16) or 5 (fp32)
  static constexpr int kSmemBytes = kQuantRingBytes + 2 * kStages * 8 + 1024;   // + the static code table
  static_assert(kStages >= 2 && kStages <= 16, "ring depth");
};

template <typename TW>
__global__ void __launch_bounds__(kQuantThreads, 1) nf4_quantize_kernel(const TW *__restrict__ W, int64_t numel,
                                                                    uint8_t *__restrict__ codes,
                                                                    float *__restrict__ c2,
                                                                    double *__restrict__ partial, int table,
                                                                    int *err) {
  using Cfg = QuantCfg<TW>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t qsm_raw[];
  uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(qsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + kQuantRingBytes);
  uint64_t *empty = full + S;
  // The code table is a static shared array: its address is a constant of
  // the kernel, so a lookup is one shared load with the index as its only
  // register operand (through a pointer into dynamic shared memory it was a
  // generic load with 64-bit address arithmetic, measured ALU-bound).
  __shared__ __align__(16) uint8_t lut[kCodeLutSpan];
  __shared__ double red[kQuantThreads / 32];
  __shared__ float thr[16];
  __shared__ int pos_s[16];
  NF4Thresholds th;
  th.init(table);
  if (threadIdx.x < 15)
    thr[threadIdx.x] =
        __double2float_rd(((double)kLevels[table][threadIdx.x] + (double)kLevels[table][threadIdx.x + 1]) * 0.5);
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), kQuantChunk / 512);      // one arrival per group of the chunk
    }
    fence_mbar_init();
  }
  build_code_lut(lut, table, pos_s);
  __syncthreads();
  pdl_trigger();
  pdl_wait();
  const int warp = warp_id();
  const int lane = lane_id();
  const int64_t ngroups = numel >> 9;
  const int64_t nchunks = numel / kQuantChunk;
  // this CTA's chunks: blockIdx.x + i * gridDim.x, i < mine
  const int64_t mine = (int64_t)blockIdx.x < nchunks ? (nchunks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  constexpr int kGroupsPerChunk = kQuantChunk / 512;
  double acc = 0.0;

  if (warp == kQuantComputeWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int64_t i = 0; i < mine; ++i) {
        const int st = (int)(i % S);
        if (!mbar_wait(smem_u32(empty + st), ((uint32_t)(i / S) & 1u) ^ 1u, err, DEV_TIMEOUT_PRODUCER)) break;
        fence_proxy_async_smem();   // the readers' loads of this slot before the copy's writes
        const uint32_t fb = smem_u32(full + st);
        mbar_arrive_expect_tx(fb, Cfg::kChunkBytes);
        bulk_g2s(smem_u32(ring + st * Cfg::kChunkBytes), W + (blockIdx.x + i * gridDim.x) * (int64_t)kQuantChunk,
                 Cfg::kChunkBytes, fb);
      }
      // A CTA never exits with bulk copies into its shared memory in flight.
      for (int64_t i = mine > S ? mine - S : 0; i < mine; ++i)
        if (!mbar_wait(smem_u32(full + (int)(i % S)), (uint32_t)(i / S) & 1u, err, DEV_TIMEOUT_DRAIN)) break;
    }
  } else {
    // ------------------------------------------------------------ compute warps
    // This warp's groups q = warp, warp + 28, ...: chunk i = q / 16 (of this
    // CTA), group gi = q % 16 in it, ring slot i % S with phase (i / S) & 1,
    // all tracked incrementally in 32-bit integers (a 64-bit division per
    // group cost the ALU-bound loop measurably).
    constexpr int kStepChunks = kQuantComputeWarps / kGroupsPerChunk;
    constexpr int kStepGroups = kQuantComputeWarps % kGroupsPerChunk;
    static_assert(kStepChunks + 1 < S, "a step crosses at most one ring wrap");
    const int nq = (int)(mine * kGroupsPerChunk);
    int i = warp / kGroupsPerChunk, gi = warp % kGroupsPerChunk;
    int st = i % S;
    uint32_t ph = (uint32_t)(i / S) & 1u;
    for (int q = warp; q < nq; q += kQuantComputeWarps) {
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(full + st), ph, err, DEV_TIMEOUT_MMA))) break;
      float v[16];
      lds_unpack16<TW>(smem_u32(ring + st * Cfg::kChunkBytes) + (uint32_t)((gi * 512 + lane * 16) * (int)sizeof(TW)), v);
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(empty + st));   // this group's weights are in registers
      const int64_t g = ((int64_t)blockIdx.x + (int64_t)i * gridDim.x) * kGroupsPerChunk + gi;
      quant_group(v, g, lut, thr, th, codes, c2, acc);
      int di = kStepChunks;
      gi += kStepGroups;
      if (gi >= kGroupsPerChunk) {
        gi -= kGroupsPerChunk;
        ++di;
      }
      i += di;
      st += di;
      if (st >= S) {
        st -= S;
        ph ^= 1u;
      }
    }
    // The last CTA: the groups after the last whole chunk, from global memory.
    if (blockIdx.x == gridDim.x - 1) {
      for (int64_t g = nchunks * kGroupsPerChunk + warp; g < ngroups; g += kQuantComputeWarps) {
        Raw16<TW> cur;
        cur.load(W + (g << 9) + (lane << 4));
        float v[16];
        cur.unpack(v);
        quant_group(v, g, lut, thr, th, codes, c2, acc);
      }
      // Tail: blocks [8*ngroups, nblk), at most 8, one warp each.
      const int64_t nblk = (numel + 63) >> 6;
      const int64_t b = (ngroups << 3) + warp;
      if (warp < 8 && b < nblk) {
        const int64_t s = b << 6;
        const int64_t i0 = s + 2 * lane, i1 = i0 + 1;
        const float v0 = i0 < numel ? load1(W + i0) : 0.f;
        const float v1 = i1 < numel ? load1(W + i1) : 0.f;
        float amax = fmaxf(fabsf(v0), fabsf(v1));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        uint32_t k0 = 7, k1 = 7;
        if (amax != 0.f) {
          k0 = th.encode(__fdiv_rn(v0, amax));
          k1 = i1 < numel ? th.encode(__fdiv_rn(v1, amax)) : 0u;
        } else if (i1 >= numel) {
          k1 = 0;
        }
        if (i0 < numel) codes[i0 >> 1] = (uint8_t)(k0 | (k1 << 4));
        if (lane == 0) {
          c2[b] = amax;
          acc += (double)amax;
        }
      }
    }
  }

  const double s = cta_sum_f64(acc, red);
  if (threadIdx.x == 0) partial[blockIdx.x] = s;
}

// E4M3 (OCP, finite-only) encode with round-to-nearest-even and saturation to
// +/-448, by the hardware conversion.
__device__ __forceinline__ uint8_t f32_to_e4m3_satfinite(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x), "f"(x));
  return (uint8_t)(r & 0xFFu);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t code) {
  const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
  return __half2float(__half(h));
}

// K2: Double Quantization of c2.  Every CTA first forms the same mean mu from
// the K1 partials in a fixed order (so mu is deterministic and identical in
// all CTAs), then quantizes 256-blocks of c2 - mu, one warp per block (lane l
// owns entries [8l, 8l+8)):
//   c1 = absmax(c2 - mu) / 448,  code8 = E4M3(fp32((c2 - mu) / c1)).
constexpr int kDqWarps = 8;

__global__ void __launch_bounds__(32 * kDqWarps) dq_constants_kernel(const float *__restrict__ c2, int64_t nblk,
                                                                    const double *__restrict__ partial, int npartial,
                                                                    uint8_t *__restrict__ c2_fp8,
                                                                    float *__restrict__ c1, float *__restrict__ mu_out) {
  __shared__ double red[kDqWarps];
  __shared__ float mu_s;
  pdl_trigger();
  pdl_wait();
  double acc = 0.0;
  for (int i = threadIdx.x; i < npartial; i += blockDim.x) acc += ld_dep_f64(partial + i);
  const double total = cta_sum_f64(acc, red);
  if (threadIdx.x == 0) {
    mu_s = __double2float_rn(__ddiv_rn(total, (double)nblk));
    if (blockIdx.x == 0) *mu_out = mu_s;
  }
  __syncthreads();
  const float mu = mu_s;
  const int lane = lane_id();
  const int64_t nb256 = (nblk + 255) >> 8;
  for (int64_t beta = (int64_t)blockIdx.x * kDqWarps + warp_id(); beta < nb256; beta += (int64_t)gridDim.x * kDqWarps) {
    const int64_t i0 = (beta << 8) + (lane << 3);
    const bool full = i0 + 8 <= nblk;
    float d[8];
    if (full) {
      const float4 a = ld_dep_f4(c2 + i0);
      const float4 b = ld_dep_f4(c2 + i0 + 4);
      const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) d[k] = __fsub_rn(x[k], mu);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) d[k] = i0 + k < nblk ? __fsub_rn(ld_dep_f32(c2 + i0 + k), mu) : 0.f;
    }
    float A = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) A = fmaxf(A, fabsf(d[k]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) A = fmaxf(A, __shfl_xor_sync(0xFFFFFFFFu, A, o));
    const float c1v = __fdiv_rn(A, 448.0f);
    uint32_t q[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) q[k] = c1v == 0.f ? 0u : (uint32_t)f32_to_e4m3_satfinite(__fdiv_rn(d[k], c1v));
    if (full) {
      reinterpret_cast<uint2 *>(c2_fp8 + i0)[0] =
          make_uint2(q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24), q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24));
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (i0 + k < nblk) c2_fp8[i0 + k] = (uint8_t)q[k];
    }
    if (lane == 0) c1[beta] = c1v;
  }
}

// K3: doubleDequant (Eq. 6) to bf16:
//   c2_hat = fma(E4M3(code8_b), c1_beta, mu)   (one rounding)
//   W_hat  = bf16_rne(fp32(NF4[code] * c2_hat))
// Streamed in chunks of kDqChunk weights (128 blocks of 64, inside one
// 256-block group, so one c1 per chunk).  CTA b takes chunks b, b + grid,
// ...; thread 0 brings each chunk's packed codes (4 KB) and E4M3 block codes
// (128 B) into a ring of shared-memory stages with bulk copies
// (cp.async.bulk, completing on the stage's mbarrier), kDqStages chunks ahead,
// so every SM keeps tens of KB of reads in flight.  Thread t decodes the
// 32-bit code words t, t + 256, t + 512, ... of a stage (8 weights each), so
// each warp's 16-byte stores cover 512 contiguous bytes.  The last CTA
// converts the weights after the last whole chunk with plain loads.
constexpr int kDqChunk = 8192;
constexpr int kDqCodeBytes = kDqChunk / 2;
constexpr int kDqC2Bytes = kDqChunk / 64;
constexpr int kDqStageBytes = kDqCodeBytes + kDqC2Bytes;
constexpr int kDqStages = 6;
constexpr int kDqThreads = 256;
constexpr int kDqCtasPerSm = 8;
constexpr int kDqWordsPerThread = kDqCodeBytes / 4 / kDqThreads;
static_assert(kDqCodeBytes == 4 * kDqWordsPerThread * kDqThreads, "whole code words per thread");
static_assert(256 % (kDqChunk / 64) == 0, "a chunk lies inside one 256-block group");
static_assert(kDqStageBytes % 16 == 0 && kDqC2Bytes % 16 == 0, "bulk-copy sizes and offsets");


// Eight weights from one 32-bit word of codes (element i in bits [4i, 4i+4)).
__device__ __forceinline__ uint4 dq_decode8(uint32_t q, float c2h, const float *lut) {
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __fmul_rn(lut[(q >> (8 * i)) & 0xF], c2h);
    const float hi = __fmul_rn(lut[(q >> (8 * i + 4)) & 0xF], c2h);
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    o[i] = *reinterpret_cast<const uint32_t *>(&p);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__global__ void __launch_bounds__(kDqThreads, kDqCtasPerSm) nf4_dequant_kernel(
    const uint8_t *__restrict__ codes, const uint8_t *__restrict__ c2_fp8, const float *__restrict__ c1,
    const float *__restrict__ mu_p, int64_t numel, __nv_bfloat16 *__restrict__ out, int table, int *err) {
  __shared__ __align__(128) uint8_t stage[kDqStages][kDqStageBytes];
  __shared__ __align__(8) uint64_t full[kDqStages];
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = kLevels[table][threadIdx.x];
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDqStages; ++i) mbar_init(smem_u32(&full[i]), 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();
  const float mu = ld_dep_f32(mu_p);
  const int64_t nchunks = numel / kDqChunk;
  const int64_t step = gridDim.x;
  const int64_t mine = (int64_t)blockIdx.x < nchunks ? (nchunks - 1 - blockIdx.x) / step + 1 : 0;
  auto issue = [&](int64_t j) {   // thread 0: chunk number j of this CTA into stage j % kDqStages
    const int64_t chunk = blockIdx.x + j * step;
    const uint32_t bar = smem_u32(&full[j % kDqStages]);
    const uint32_t dst = smem_u32(stage[j % kDqStages]);
    mbar_arrive_expect_tx(bar, kDqStageBytes);
    bulk_g2s(dst, codes + chunk * kDqCodeBytes, kDqCodeBytes, bar);
    bulk_g2s(dst + kDqCodeBytes, c2_fp8 + chunk * kDqC2Bytes, kDqC2Bytes, bar);
  };
  int64_t issued = 0, done = 0;
  if (threadIdx.x == 0)
    for (; issued < mine && issued < kDqStages; ++issued) issue(issued);
  const int t = threadIdx.x;
  // c1 of a chunk (one per chunk), loaded a chunk ahead
  auto c1_of = [&](int64_t j) { return ld_dep_f32(c1 + (((blockIdx.x + j * step) * (kDqChunk / 64)) >> 8)); };
  float c1_next = mine > 0 ? c1_of(0) : 0.f;
  for (; done < mine; ++done) {
    const int st = (int)(done % kDqStages);
    const bool got = mbar_wait(smem_u32(&full[st]), (uint32_t)((done / kDqStages) & 1), err, DEV_TIMEOUT_MMA);
    if (__syncthreads_or(!got)) break;
    const int64_t chunk = blockIdx.x + done * step;
    const float c1v = c1_next;
    if (done + 1 < mine) c1_next = c1_of(done + 1);
    const uint8_t *sc = stage[st];
    uint4 *dst = reinterpret_cast<uint4 *>(out + chunk * kDqChunk);
#pragma unroll
    for (int i = 0; i < kDqWordsPerThread; ++i) {
      const int w = t + kDqThreads * i;                           // code word of the chunk
      const uint32_t q = reinterpret_cast<const uint32_t *>(sc)[w];
      const float c2h = __fmaf_rn(e4m3_to_f32(sc[kDqCodeBytes + (w >> 3)]), c1v, mu);
      dst[w] = dq_decode8(q, c2h, lut);
    }
    __syncthreads();   // stage st consumed by every thread
    if (threadIdx.x == 0 && issued < mine) {
      fence_proxy_async_smem();   // those reads before the refill's writes
      issue(issued++);
    }
  }
  // A CTA never exits with bulk copies into its shared memory in flight.
  if (done < mine && threadIdx.x == 0)
    for (int64_t j = done; j < issued; ++j)
      if (!mbar_wait(smem_u32(&full[j % kDqStages]), (uint32_t)((j / kDqStages) & 1), err, DEV_TIMEOUT_DRAIN)) break;
  // Weights after the last whole chunk: 8 per thread, then a scalar rest.
  if (blockIdx.x == gridDim.x - 1) {
    const int64_t n8 = numel >> 3;
    for (int64_t e = nchunks * (kDqChunk / 8) + t; e < n8; e += kDqThreads) {
      const int64_t b = e >> 3;
      const float c2h = __fmaf_rn(e4m3_to_f32((uint8_t)ld_dep_u8(c2_fp8 + b)), ld_dep_f32(c1 + (b >> 8)), mu);
      reinterpret_cast<uint4 *>(out)[e] = dq_decode8(ld_dep_u32(codes + 4 * e), c2h, lut);
    }
    if (t < (numel & 7)) {
      const int64_t i = (n8 << 3) + t;
      const int64_t b = i >> 6;
      const float c2h = __fmaf_rn(e4m3_to_f32((uint8_t)ld_dep_u8(c2_fp8 + b)), ld_dep_f32(c1 + (b >> 8)), mu);
      const uint32_t code = (ld_dep_u8(codes + (i >> 1)) >> ((i & 1) * 4)) & 0xF;
      out[i] = __float2bfloat16_rn(__fmul_rn(lut[code], c2h));
    }
  }
}

}  // namespace qlora
