// libqlora: host side of the C ABI declared in include/qlora.h.
//
// One translation unit: the kernels live in the included .cuh files.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>

#include "qlora.h"
#include "common.cuh"
#include "quant.cuh"
#include "tc_gemm.cuh"
#include "few_token.cuh"
#include "decode_fwd.cuh"
#include "dropout.cuh"
#include "rank_gemm.cuh"

namespace qlora {

__device__ int g_dev_err;

// Sets the device's wait limit (stream-ordered, one thread).
__global__ void set_wait_limit_kernel(unsigned long long ns) { g_wait_limit_ns = ns; }

// Diagnostics: one thread waits, through the same bounded wait as every
// pipeline, for the first phase of an mbarrier that nothing arrives on.  The
// wait runs out after the device's wait limit, records DEV_TIMEOUT_DIAG and
// returns.  No copy or MMA is issued, so nothing is in flight at exit.
__global__ void diag_expired_wait_kernel(int *err) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(smem_u32(&bar), 1);
  fence_mbar_init();
  mbar_wait(smem_u32(&bar), 0, err, DEV_TIMEOUT_DIAG);
}

namespace {

constexpr int kMaxDevices = 64;

// Per-device state.  `sms` and `err` are written once, under g_mu, before
// `init` is published with release order; readers check `init` with acquire
// order first.  The per-kernel set-up slots (a shared-memory limit set, an
// occupancy figure) are filled lazily by once(): 0 means not done yet.
struct DeviceInfo {
  std::atomic<bool> init{false};
  int sms = 0;
  int *err = nullptr;                    // device address of g_dev_err
  std::atomic<int> gemm_attr[16];        // [wide][fold][BN 64/128/256 or 3 = pair]: 1 once the smem limit is set
  std::atomic<int> pair_clusters[3];     // co-resident 2-CTA clusters of the pair GEMM [form]
  std::atomic<int> decode_smem_set[8];   // few-token product: smem limit set [group form][token padding]
  std::atomic<int> quant_smem_set[2];    // quantizer: smem limit set [bf16, fp32 input]
  std::atomic<int> rank_smem_set{0};     // grouped rank-r products: smem limit set
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

int current_device_info(DeviceInfo **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  DeviceInfo &d = g_dev[dev];
  if (!d.init.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!d.init.load(std::memory_order_relaxed)) {
      if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return QLORA_ERR_CUDA;
      if (cudaGetSymbolAddress(reinterpret_cast<void **>(&d.err), g_dev_err) != cudaSuccess) return QLORA_ERR_CUDA;
      d.init.store(true, std::memory_order_release);
    }
  }
  *out = &d;
  return QLORA_OK;
}

// One-time set-up step of a device: runs f() (a positive result, or <= 0 on
// failure) under the device mutex the first time, stores its result in
// `slot` and returns it; later calls return the stored value.
template <class F>
int once(std::atomic<int> &slot, F &&f) {
  int v = slot.load(std::memory_order_acquire);
  if (v > 0) return v;
  std::lock_guard<std::mutex> lock(g_mu);
  v = slot.load(std::memory_order_relaxed);
  if (v > 0) return v;
  v = f();
  if (v > 0) slot.store(v, std::memory_order_release);
  return v;
}

// ---------------------------------------------------------------- event log
// Opt-in timing of the library's own kernel launches: while enabled, every
// launch is bracketed by a pair of CUDA events recorded on its stream.
struct ProfLog {
  bool on = false;
  int used = 0;
  int cap = 0;
  int dev = -1;
  cudaEvent_t *ev = nullptr;  // 2 * cap events
  int *kind = nullptr;        // cap
};
ProfLog g_prof;
std::mutex g_prof_mu;

struct ProfScope {
  int slot = -1;
  cudaStream_t st;
  ProfScope(int kind, cudaStream_t s) : st(s) {
    if (!g_prof.on) return;
    std::lock_guard<std::mutex> lock(g_prof_mu);
    if (!g_prof.on || g_prof.used >= g_prof.cap) return;
    slot = g_prof.used++;
    g_prof.kind[slot] = kind;
    cudaEventRecord(g_prof.ev[2 * slot], st);
  }
  ~ProfScope() {
    if (slot >= 0) cudaEventRecord(g_prof.ev[2 * slot + 1], st);
  }
};

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

int launch_status() { return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

// Launch `kernel` on `st` as a programmatic dependent of the previous launch.
// Every kernel launched this way waits (griddepcontrol.wait) before it touches
// memory another kernel writes or reads.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  // While the per-launch event log records, the events between launches
  // serialise them anyway; plain launches then time each kernel alone.
  cfg.numAttrs = g_prof.on ? 0 : 1;
  if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) return QLORA_ERR_CUDA;
  return launch_status();
}


// ---------------------------------------------------------------- TMA maps
using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A bf16 operand of the GEMM engine.  K-major: `rows` x `kext` with row stride
// `ld` elements, contiguous along the reduction.  MN-major: `kext` rows of
// `rows` contiguous elements (row stride `ld`), i.e. contiguous along M or N.
struct Operand {
  const void *ptr;
  int64_t rows;   // extent along the output dimension (M for A, N for B)
  int64_t kext;   // extent along the reduction
  int64_t ld;     // elements between consecutive rows of the stored matrix
  int mn_major;
};

int make_tmap(CUtensorMap *m, const Operand &o, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return QLORA_ERR_CUDA;
  cuuint64_t dims[2], strides[1];
  cuuint32_t box[2], estr[2] = {1, 1};
  if (!o.mn_major) {
    dims[0] = (cuuint64_t)o.kext;
    dims[1] = (cuuint64_t)o.rows;
    box[0] = 64;
    box[1] = (cuuint32_t)box_rows;
  } else {
    dims[0] = (cuuint64_t)o.rows;
    dims[1] = (cuuint64_t)o.kext;
    box[0] = 64;
    box[1] = 64;
  }
  strides[0] = (cuuint64_t)o.ld * 2;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(o.ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

// The same operand as 3-D boxes of two k-blocks, for the GEMM's wide stages.
// K-major: dims {64, rows, kext/64} with the k-block stride 128 B, so a box
// {64, box_rows, 2} lands as [k-block][row][64].  MN-major: dims {64, kext,
// rows/64} with the chunk stride 128 B, a box {64, 128, box_rows/64} lands
// as [chunk][k][64].  Only whole 64-wide blocks may be described this way (a
// partial one would read into the next row), hence wide_ok().
bool wide_ok(const Operand &o) { return o.mn_major ? o.rows % 64 == 0 : o.kext % 64 == 0; }

int make_tmap3(CUtensorMap *m, const Operand &o, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return QLORA_ERR_CUDA;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3], estr[3] = {1, 1, 1};
  dims[0] = 64;
  box[0] = 64;
  if (!o.mn_major) {
    dims[1] = (cuuint64_t)o.rows;
    dims[2] = (cuuint64_t)(o.kext / 64);
    box[1] = (cuuint32_t)box_rows;
    box[2] = 2;
  } else {
    dims[1] = (cuuint64_t)o.kext;
    dims[2] = (cuuint64_t)(o.rows / 64);
    box[1] = 128;
    box[2] = (cuuint32_t)(box_rows / 64);
  }
  strides[0] = (cuuint64_t)o.ld * 2;
  strides[1] = 128;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(o.ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

struct GemmSeg {
  Operand A, B;   // A.kext == B.kext
};

// Masked addend of a bf16 GEMM output (see TcGemmArgs::add).
struct GemmAddend {
  const uint16_t *z;
  const uint32_t *mask;
  float scale;
  int64_t ld;
};

int pick_bn(int64_t N) { return N <= 64 ? 64 : (N <= 128 ? 128 : 256); }

// Split-K factor for a single-segment product whose tile grid leaves SMs idle:
// as many splits as fit in one wave, so no CTA runs a second unit (these are
// the HBM-streaming rank-r products; one longer unit per SM streams faster
// than more, shorter units over several waves).
void choose_splits(int64_t tiles, int64_t nkb, int sms, bool allow, int *splits, int *kbps) {
  int s = 1;
  if (allow && tiles > 0 && tiles < sms && nkb > 1) {
    s = (int)std::max<int64_t>(1, std::min<int64_t>(nkb, sms / tiles));
  }
  int k = (int)((nkb + s - 1) / s);
  if (k < 1) k = 1;
  *kbps = k;
  *splits = (int)((nkb + k - 1) / k);
  if (*splits < 1) *splits = 1;
}

// Split-K partials of a product with N columns (w output columns after a fold).
size_t gemm_split_ws_bytes(int64_t M, int64_t N, int64_t K, int sms, bool allow, int64_t w = -1) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  if (w < 0) w = N;
  const int bn = pick_bn(N);
  const int64_t tiles = ((M + kBM - 1) / kBM) * ((N + bn - 1) / bn);
  int splits, kbps;
  choose_splits(tiles, (K + kBK - 1) / kBK, sms, allow, &splits, &kbps);
  return splits > 1 ? align_up((size_t)splits * (size_t)M * (size_t)w * 4) : 0;
}

// The hi/lo fold applies when both halves (2w columns) fit one tile and the
// epilogue's 32-column chunks line up with the halves.
bool can_fold(int64_t w) { return w == 8 || w == 16 || (w % 32 == 0 && 2 * w <= 256); }

template <int BN, bool FOLD, bool WIDE>
int launch_gemm_bn(const CUtensorMap *maps, TcGemmArgs &args, int sms, DeviceInfo *dev, cudaStream_t st, int kind) {
  using Cfg = TcCfg<BN, false, WIDE>;
  auto kernel = tc_gemm_kernel<BN, false, FOLD, WIDE>;
  const int idx = (BN == 64 ? 0 : (BN == 128 ? 1 : 2)) + (FOLD ? 4 : 0) + (WIDE ? 8 : 0);
  if (once(dev->gemm_attr[idx], [&] {
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) ==
                       cudaSuccess
                   ? 1
                   : 0;
      }) <= 0)
    return QLORA_ERR_CUDA;
  const int units = args.m_tiles * args.n_tiles * args.splits;
  const int grid = std::max(1, std::min(units, sms));
  ProfScope prof(kind, st);
  return launch_pdl(kernel, dim3(grid), dim3(kGemmThreads), Cfg::kSmemBytes, st, maps[0], maps[1], maps[2], maps[3],
                    args);
}

// CTA-pair GEMM (256 x 256 tiles): a persistent grid of 2-CTA clusters, as
// many as can be resident at once.
template <bool WIDE, bool DROPZ = false>
int launch_gemm_pair(const CUtensorMap *maps, TcGemmArgs &args, DeviceInfo *dev, cudaStream_t st, int kind) {
  constexpr int BN = 256;
  using Cfg = TcCfg<BN, true, WIDE>;
  auto kernel = tc_gemm_kernel<BN, true, false, WIDE, DROPZ>;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;   // the occupancy query takes the cluster shape alone
  const int form = DROPZ ? 2 : (WIDE ? 1 : 0);
  const int resident = once(dev->pair_clusters[form], [&] {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) != cudaSuccess)
      return 0;
    cfg.gridDim = dim3(2 * (unsigned)dev->sms, 1, 1);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess) return 0;
    return clusters;
  });
  if (resident <= 0) return QLORA_ERR_CUDA;
  const int units = args.m_tiles * args.n_tiles * args.splits;
  const int clusters = std::max(1, std::min(units, resident));
  cfg.gridDim = dim3(2 * (unsigned)clusters, 1, 1);
  cfg.numAttrs = g_prof.on ? 1 : 2;   // a programmatic dependent of the previous kernel, unless the event log records
  ProfScope prof(kind, st);
  if (cudaLaunchKernelEx(&cfg, kernel, maps[0], maps[1], maps[2], maps[3], args) != cudaSuccess) return QLORA_ERR_CUDA;
  return launch_status();
}

// The CTA-pair form serves the wide products (N > 128) that are not split
// along K and have at least two 128-row tiles.
bool use_pair(int bn, int splits, int64_t M) { return bn == 256 && splits == 1 && M > kBM; }

// D[M x N] = alpha * sum_seg A_seg B_seg^T, written to `out` with strides
// (ld_row, ld_col) as bf16 (optionally with a lo part at +lo_off) or fp32.
// If `split_ws` is given and the tile grid leaves SMs idle, the reduction is
// split (segment 0 only, or every segment when `split_all`), the fp32
// partials go to split_ws and a finalize pass sums them in a fixed order.
int tc_gemm(cudaStream_t st, DeviceInfo *dev, int64_t M, int64_t N, int nseg, const GemmSeg *segs, float alpha,
            void *out, int64_t ld_row, int64_t ld_col, int out_f32, float *split_ws, int kind, int64_t lo_off = 0,
            bool split_all = false, int fold = 0, const GemmAddend *add = nullptr) {
  if (M <= 0 || N <= 0) return QLORA_OK;
  // the addend is applied by the direct bf16 epilogue only; add->z == nullptr
  // asks for segment 1 as the masked term (the pair form's second accumulator)
  if (add && (split_ws || out_f32 || fold || N % 32)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const bool dropz = add && !add->z;
  if (dropz && nseg != 2) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t)INT32_MAX / 2 || N > (int64_t)INT32_MAX / 2) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int bn = pick_bn(N);
  CUtensorMap maps[4];
  std::memset(maps, 0, sizeof(maps));
  TcGemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.M = (int)M;
  a.N = (int)N;
  a.m_tiles = (int)((M + kBM - 1) / kBM);
  a.n_tiles = (int)((N + bn - 1) / bn);
  a.nseg = nseg;
  for (int s = 0; s < nseg; ++s) a.seg[s].nkb = (int)((segs[s].A.kext + kBK - 1) / kBK);
  if (split_all && (nseg < 2 || a.seg[1].nkb != a.seg[0].nkb)) split_all = false;
  int splits, kbps;
  choose_splits((int64_t)a.m_tiles * a.n_tiles, a.seg[0].nkb, dev->sms,
                split_ws != nullptr && (nseg == 1 || split_all), &splits, &kbps);
  const bool pair = use_pair(bn, splits, M) && fold == 0;
  if (pair) a.m_tiles = (int)((M + 2 * kBM - 1) / (2 * kBM));
  // Wide stages (two k-blocks per 3-D box) wherever segment 0 allows them;
  // the single-CTA 256-column form keeps one k-block per stage.
  bool seg_wide[2] = {false, false};
  for (int s = 0; s < nseg; ++s)
    seg_wide[s] = a.seg[s].nkb >= 2 && wide_ok(segs[s].A) && wide_ok(segs[s].B);
  const bool wide = seg_wide[0] && (pair || bn <= 128);
  const int brows = pair ? bn / 2 : bn;
  for (int s = 0; s < nseg; ++s) {
    a.seg[s].a_mn = segs[s].A.mn_major;
    a.seg[s].b_mn = segs[s].B.mn_major;
    a.seg[s].wide = wide && seg_wide[s];
    int rc = a.seg[s].wide ? make_tmap3(&maps[2 * s], segs[s].A, kBM) : make_tmap(&maps[2 * s], segs[s].A, kBM);
    if (rc) return rc;
    rc = a.seg[s].wide ? make_tmap3(&maps[2 * s + 1], segs[s].B, brows)
                       : make_tmap(&maps[2 * s + 1], segs[s].B, brows);
    if (rc) return rc;
  }
  if (nseg == 1) maps[2] = maps[0], maps[3] = maps[1];
  a.splits = splits;
  a.kb_per_split = kbps;
  a.split_all = split_all ? 1 : 0;
  a.err = dev->err;
  a.ld_row = ld_row;
  a.ld_col = ld_col;
  a.lo_off = lo_off;
  a.fold = fold;
  if (add) {
    a.add = add->z;
    a.add_mask = add->mask;
    a.add_scale = add->scale;
    a.add_ld = add->ld;
  }
  if (splits > 1) {
    a.alpha = 1.f;
    a.out = split_ws;
    a.out_f32 = 1;
  } else {
    a.alpha = alpha;
    a.out = out;
    a.out_f32 = out_f32;
  }
  int rc;
  if (dropz) {
    if (!pair || !wide) return QLORA_ERR_UNSUPPORTED_SHAPE;
    rc = launch_gemm_pair<true, true>(maps, a, dev, st, kind);
  } else if (pair) {
    rc = wide ? launch_gemm_pair<true>(maps, a, dev, st, kind) : launch_gemm_pair<false>(maps, a, dev, st, kind);
  } else if (fold) {
    switch (bn) {
      case 64: rc = wide ? launch_gemm_bn<64, true, true>(maps, a, dev->sms, dev, st, kind)
                         : launch_gemm_bn<64, true, false>(maps, a, dev->sms, dev, st, kind); break;
      case 128: rc = wide ? launch_gemm_bn<128, true, true>(maps, a, dev->sms, dev, st, kind)
                          : launch_gemm_bn<128, true, false>(maps, a, dev->sms, dev, st, kind); break;
      default: rc = launch_gemm_bn<256, true, false>(maps, a, dev->sms, dev, st, kind); break;
    }
  } else {
    switch (bn) {
      case 64: rc = wide ? launch_gemm_bn<64, false, true>(maps, a, dev->sms, dev, st, kind)
                         : launch_gemm_bn<64, false, false>(maps, a, dev->sms, dev, st, kind); break;
      case 128: rc = wide ? launch_gemm_bn<128, false, true>(maps, a, dev->sms, dev, st, kind)
                          : launch_gemm_bn<128, false, false>(maps, a, dev->sms, dev, st, kind); break;
      default: rc = launch_gemm_bn<256, false, false>(maps, a, dev->sms, dev, st, kind); break;
    }
  }
  if (rc || splits == 1) return rc;
  const int64_t W = fold > 0 ? fold : N;
  const int64_t count = M * W;
  const int grid = (int)std::min<int64_t>((count + 255) / 256, (int64_t)dev->sms * 8);
  ProfScope prof(QLORA_KERNEL_SPLITK_FINALIZE, st);
  return launch_pdl(splitk_finalize_kernel, dim3(grid), dim3(256), 0, st, (const float *)split_ws, splits, (int)M,
                    (int)W, alpha, out, ld_row, ld_col, lo_off, out_f32);
}

// ---------------------------------------------------- grouped rank-r products
// Host side of rank_gemm_kernel: one problem per RankJob.
struct RankJob {
  Operand A, B;
  int bn;                    // 64 or 128: B rows per n-tile (the MMA N)
  int n_tiles;
  int ncols;                 // valid output columns per n-tile, before the fold
  int fold;
  RankOut outs[kMaxGroup];   // one per n-tile (part is filled at launch)
  int width() const { return fold ? fold : ncols; }
};

RankShape rank_shape(const RankJob &j) {
  RankShape s;
  s.m_tiles = (j.A.rows + kBM - 1) / kBM;
  s.tiles = s.m_tiles * j.n_tiles;
  s.nkb = (j.A.kext + kBK - 1) / kBK;
  return s;
}

// fp32 partial bytes of a launch of these problems.
size_t rank_part_bytes(const RankJob *jobs, int n, int sms) {
  if (n <= 0) return 0;
  RankShape sh[kRankMaxProbs];
  int splits[kRankMaxProbs];
  for (int i = 0; i < n; ++i) sh[i] = rank_shape(jobs[i]);
  plan_rank(sh, n, sms, splits);
  size_t b = 0;
  for (int i = 0; i < n; ++i)
    if (splits[i] > 1) b += (size_t)jobs[i].n_tiles * align_up((size_t)splits[i] * jobs[i].A.rows * jobs[i].width() * 4);
  return b;
}

// Runs the problems as one rank_gemm_kernel launch (then, if any is split,
// one rank_finalize_kernel launch).  `part` holds rank_part_bytes() bytes.
int rank_launch(const RankJob *jobs, int n, uint8_t *part, DeviceInfo *dev, cudaStream_t st, int kind) {
  if (n <= 0) return QLORA_OK;
  if (n > kRankMaxProbs) return QLORA_ERR_UNSUPPORTED_SHAPE;
  RankShape sh[kRankMaxProbs];
  int splits[kRankMaxProbs], order[kRankMaxProbs];
  int64_t kbps[kRankMaxProbs];
  for (int i = 0; i < n; ++i) sh[i] = rank_shape(jobs[i]);
  plan_rank(sh, n, dev->sms, splits);
  rank_order(sh, splits, n, kbps, order);
  RankMaps maps;
  RankArgs a;
  RankFinArgs fin;
  std::memset(&maps, 0, sizeof(maps));
  std::memset(&a, 0, sizeof(a));
  std::memset(&fin, 0, sizeof(fin));
  int64_t units = 0, elem = 0;
  size_t part_off = 0;
  for (int oi = 0; oi < n; ++oi) {
    const int i = order[oi];
    const RankJob &j = jobs[i];
    if (a.nout + j.n_tiles > kRankMaxOuts || j.n_tiles < 1) return QLORA_ERR_UNSUPPORTED_SHAPE;
    if (j.A.rows > INT32_MAX / 2 || j.A.kext > INT32_MAX / 2) return QLORA_ERR_UNSUPPORTED_SHAPE;
    RankProb &q = a.prob[a.nprob];
    q.rows = (int)j.A.rows;
    q.m_tiles = (int)sh[i].m_tiles;
    q.n_tiles = j.n_tiles;
    q.bn = j.bn;
    q.ncols = j.ncols;
    q.fold = j.fold;
    q.nkb = (int)sh[i].nkb;
    q.splits = splits[i];
    q.kb_per_split = (int)kbps[i];
    q.a_mn = j.A.mn_major;
    q.b_mn = j.B.mn_major;
    q.wide = q.nkb >= 2 && wide_ok(j.A) && wide_ok(j.B);
    q.unit0 = (int)units;
    q.out0 = a.nout;
    int rc = q.wide ? make_tmap3(&maps.m[2 * a.nprob], j.A, kBM) : make_tmap(&maps.m[2 * a.nprob], j.A, kBM);
    if (rc) return rc;
    rc = q.wide ? make_tmap3(&maps.m[2 * a.nprob + 1], j.B, j.bn) : make_tmap(&maps.m[2 * a.nprob + 1], j.B, j.bn);
    if (rc) return rc;
    for (int t = 0; t < j.n_tiles; ++t) {
      RankOut o = j.outs[t];
      o.part = nullptr;
      if (q.splits > 1) {
        if (fin.njobs == kRankMaxOuts) return QLORA_ERR_UNSUPPORTED_SHAPE;
        o.part = reinterpret_cast<float *>(part + part_off);
        part_off += align_up((size_t)q.splits * q.rows * j.width() * 4);
        RankFinJob &f = fin.job[fin.njobs++];
        f.part = o.part;
        f.out = o.ptr;
        f.ld_row = o.ld_row;
        f.ld_col = o.ld_col;
        f.lo_off = o.lo_off;
        f.elem0 = elem;
        f.splits = q.splits;
        f.rows = q.rows;
        f.width = j.width();
        f.out_f32 = o.out_f32;
        f.alpha = o.alpha;
        elem += (int64_t)q.rows * j.width();
      }
      a.out[a.nout + t] = o;
    }
    a.nout += j.n_tiles;
    units += sh[i].tiles * q.splits;
    ++a.nprob;
  }
  if (units > INT32_MAX / 2) return QLORA_ERR_UNSUPPORTED_SHAPE;
  a.units = (int)units;
  a.err = dev->err;
  if (once(dev->rank_smem_set, [&] {
        return cudaFuncSetAttribute(rank_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kRankSmemBytes) == cudaSuccess
                   ? 1
                   : 0;
      }) <= 0)
    return QLORA_ERR_CUDA;
  const int grid = (int)std::min<int64_t>(units, dev->sms);
  int rc;
  {
    ProfScope prof(kind, st);
    rc = launch_pdl(rank_gemm_kernel, dim3(grid), dim3(kGemmThreads), kRankSmemBytes, st, maps, a);
  }
  if (rc || fin.njobs == 0) return rc;
  fin.total = elem;
  const int fgrid = (int)std::min<int64_t>((elem + 255) / 256, (int64_t)dev->sms * 8);
  ProfScope prof(QLORA_KERNEL_SPLITK_FINALIZE, st);
  return launch_pdl(rank_finalize_kernel, dim3(fgrid), dim3(256), 0, st, fin);
}

// The adapter's down-projection T = alpha Xt L1 (L1 read MN-major) as a bf16
// hi/lo pair [M x 2r], as one problem of the rank kernel (r <= 128).
RankJob t_job(const uint16_t *Xt, int64_t M, int64_t K, const uint16_t *L1, int r, float alpha, uint16_t *T) {
  RankJob j;
  j.A = {Xt, M, K, K, 0};
  j.B = {L1, r, K, r, 1};
  j.bn = r <= 64 ? 64 : 128;
  j.n_tiles = 1;
  j.ncols = r;
  j.fold = 0;
  j.outs[0] = RankOut{T, nullptr, 2 * r, 1, r, alpha, 0};
  return j;
}

int dequant_launch(const qlora_nf4dq_t *W, __nv_bfloat16 *out, cudaStream_t st, int sms) {
  const int64_t numel = W->n_out * W->k_in;
  if (numel == 0) return QLORA_OK;
  DeviceInfo *dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  const int64_t nchunks = numel / kDqChunk;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(nchunks, (int64_t)sms * kDqCtasPerSm));
  ProfScope prof(QLORA_KERNEL_DEQUANT, st);
  return launch_pdl(nf4_dequant_kernel, dim3(grid), dim3(kDqThreads), 0, st, W->codes, W->c2_fp8, W->c1,
                    W->c2_mean, numel, out, (int)W->table, dev->err);
}

int check_weight(const qlora_nf4dq_t *W) {
  if (!W || !W->codes || !W->c2_fp8 || !W->c1 || !W->c2_mean) return QLORA_ERR_INVALID_ARG;
  if (W->table < 0 || W->table >= kNumTables) return QLORA_ERR_INVALID_ARG;
  if (W->n_out < 0 || W->k_in < 0) return QLORA_ERR_INVALID_ARG;
  if (!aligned(W->codes, 16) || !aligned(W->c2_fp8, 16) || !aligned(W->c1, 16) || !aligned(W->c2_mean, 4))
    return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

// Common validation of the linear entry points.
int check_linear(int64_t M, const qlora_nf4dq_t *W, int r) {
  int rc = check_weight(W);
  if (rc) return rc;
  if (M < 0 || r <= 0) return QLORA_ERR_INVALID_ARG;
  if (W->k_in <= 0 || W->n_out <= 0) return QLORA_ERR_INVALID_ARG;
  if (W->k_in % 64 || W->n_out % 8 || r % 8 || r > QLORA_MAX_RANK) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t)1 << 30 || W->k_in > (int64_t)1 << 30 || W->n_out > (int64_t)1 << 30)
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  return QLORA_OK;
}

int encode_tmap(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *ptr, const cuuint64_t *dims,
                const cuuint64_t *strides, const cuuint32_t *box) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return QLORA_ERR_CUDA;
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dt, rank, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QLORA_OK : QLORA_ERR_CUDA;
}

// One linear of a few-token forward group (host view of its arguments).
struct FwdMember {
  const qlora_nf4dq_t *W;
  const uint16_t *X, *L1, *L2;
  int r;
  float s;
  uint16_t *Y, *T_save;
};

// Workspace of the few-token forward: per linear [acc M*N f32 | tacc M*r f32],
// one linear after the other, all zeroed by one memset per call.
struct FewLayout {
  size_t acc[kMaxGroup], tacc[kMaxGroup];
  size_t zero_bytes, total;
};

FewLayout few_layout(int64_t M, const FwdMember *mem, int count) {
  FewLayout L;
  size_t off = 0;
  for (int i = 0; i < count; ++i) {
    L.acc[i] = align_up(off, 16);
    L.tacc[i] = align_up(L.acc[i] + (size_t)M * mem[i].W->n_out * 4, 16);
    off = L.tacc[i] + (size_t)M * mem[i].r * 4;
  }
  L.zero_bytes = off;
  L.total = align_up(off);
  return L;
}

size_t few_ws_bytes(int64_t M, int64_t N, int r) {
  qlora_nf4dq_t w;
  std::memset(&w, 0, sizeof(w));
  w.n_out = N;
  FwdMember m;
  std::memset(&m, 0, sizeof(m));
  m.W = &w;
  m.r = r;
  return few_layout(M, &m, 1).total;
}

// T accumulation of every linear of the group (a plain launch: it follows all
// earlier work in the stream).
template <int GM>
int launch_lora_down(const FwdMember *mem, int count, int64_t M, const FewLayout &L, uint8_t *ws, cudaStream_t st) {
  TdArgs<GM> a;
  std::memset(&a, 0, sizeof(a));
  a.M = (int)M;
  a.count = count;
  int slices = 0, rmax = 0;
  for (int i = 0; i < count; ++i) {
    const int64_t K = mem[i].W->k_in;
    a.beg[i] = slices;
    a.m[i].X = reinterpret_cast<const __nv_bfloat16 *>(mem[i].X);
    a.m[i].L1 = reinterpret_cast<const __nv_bfloat16 *>(mem[i].L1);
    a.m[i].tacc = reinterpret_cast<float *>(ws + L.tacc[i]);
    a.m[i].K = (int)K;
    a.m[i].r = mem[i].r;
    slices += (int)((K + kTSliceK - 1) / kTSliceK);
    rmax = std::max(rmax, mem[i].r);
  }
  lora_down_small_kernel<GM><<<dim3((unsigned)slices, (unsigned)((rmax + 63) / 64)), 256, 0, st>>>(a);
  return launch_status();
}

// Y = bf16(acc + s T L2) and the T hi/lo pair of every linear of the group,
// as a programmatic dependent of the product kernel just launched.
template <int GM>
int launch_lora_epilogue(const FwdMember *mem, int count, int64_t M, const FewLayout &L, uint8_t *ws,
                         cudaStream_t st) {
  EpArgs<GM> a;
  std::memset(&a, 0, sizeof(a));
  a.M = (int)M;
  a.count = count;
  int slices = 0, rmax = 0;
  for (int i = 0; i < count; ++i) {
    const int64_t N = mem[i].W->n_out;
    a.beg[i] = slices;
    a.m[i].acc = reinterpret_cast<const float *>(ws + L.acc[i]);
    a.m[i].tacc = reinterpret_cast<const float *>(ws + L.tacc[i]);
    a.m[i].L2 = reinterpret_cast<const __nv_bfloat16 *>(mem[i].L2);
    a.m[i].Y = reinterpret_cast<__nv_bfloat16 *>(mem[i].Y);
    a.m[i].T_save = reinterpret_cast<__nv_bfloat16 *>(mem[i].T_save);
    a.m[i].N = (int)N;
    a.m[i].r = mem[i].r;
    a.m[i].s = mem[i].s;
    slices += (int)((N + 63) / 64);
    rmax = std::max(rmax, mem[i].r);
  }
  const size_t esmem = (size_t)kTokChunk * rmax * 4 + (size_t)rmax * 64 * 2;
  if (esmem > 48 * 1024 && cudaFuncSetAttribute(lora_epilogue_kernel<GM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)esmem) != cudaSuccess)
    return QLORA_ERR_CUDA;
  const dim3 grid((unsigned)slices, (unsigned)((M + kTokChunk - 1) / kTokChunk));
  return launch_pdl(lora_epilogue_kernel<GM>, grid, dim3(256), esmem, st, a);
}

// Fused doubleDequant + tcgen05 forward with the weight decoded into TMEM,
// for M <= MP tokens of a group of linears sharing one code table: T
// accumulation, the product (a programmatic dependent of it), then the LoRA
// epilogue.  The accumulators are zero (the caller's memset).
template <int MP, int GM>
int launch_decode_fwd(const FwdMember *mem, int count, int64_t M, const FewLayout &L, uint8_t *ws, DeviceInfo *dev,
                      cudaStream_t st) {
  using Cfg = DfCfg<MP>;
  DfMaps<GM> maps;
  DfArgs<GM> a;
  std::memset(&maps, 0, sizeof(maps));
  std::memset(&a, 0, sizeof(a));
  std::memcpy(a.levels, kLevelsHost[mem[0].W->table], sizeof(a.levels));
  a.M = (int)M;
  a.count = count;
  a.err = dev->err;
  int items = 0;
  for (int i = 0; i < count; ++i) {
    const qlora_nf4dq_t *W = mem[i].W;
    const int64_t N = W->n_out, K = W->k_in;
    {
      const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)N};
      const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
      const cuuint32_t box[2] = {128, (cuuint32_t)kDfRows};
      int rc = encode_tmap(&maps.codes[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, W->codes, dims, strides, box);
      if (rc) return rc;
    }
    {
      // X as [64-block][token][64]: one box = the four K-major atoms of a stage
      const cuuint64_t dims[3] = {64, (cuuint64_t)M, (cuuint64_t)(K / 64)};
      const cuuint64_t strides[2] = {(cuuint64_t)K * 2, 128};
      const cuuint32_t box[3] = {64, (cuuint32_t)MP, 4};
      int rc = encode_tmap(&maps.x[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, mem[i].X, dims, strides, box);
      if (rc) return rc;
    }
    DfMember &m = a.m[i];
    m.N = (int)N;
    m.K = (int)K;
    m.kstages = (int)((K + kDfStageK - 1) / kDfStageK);
    m.ks_div = make_div_u31((uint32_t)m.kstages);
    m.c2_fp8 = W->c2_fp8;
    m.c1 = W->c1;
    m.mu = W->c2_mean;
    m.acc = reinterpret_cast<float *>(ws + L.acc[i]);
    a.beg[i] = items;
    items += (int)((N + kDfRows - 1) / kDfRows) * m.kstages;
  }
  a.items = items;
  const int idx = (GM > 1 ? 4 : 0) + (MP == 16 ? 0 : (MP == 32 ? 1 : (MP == 64 ? 2 : 3)));
  if (once(dev->decode_smem_set[idx], [&] {
        return cudaFuncSetAttribute(nf4_decode_fwd_kernel<MP, GM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    Cfg::kSmemBytes) == cudaSuccess
                   ? 1
                   : 0;
      }) <= 0)
    return QLORA_ERR_CUDA;
  const int grid = std::max(1, std::min(a.items, dev->sms));
  ProfScope prof(QLORA_KERNEL_FUSED_FWD, st);
  // 1. T accumulation; 2. the fused product, overlapping it; 3. the LoRA epilogue.
  int rc = launch_lora_down<GM>(mem, count, M, L, ws, st);
  if (rc) return rc;
  rc = launch_pdl(nf4_decode_fwd_kernel<MP, GM>, dim3(grid), dim3(Cfg::kThreads), (size_t)Cfg::kSmemBytes, st, maps,
                  a);
  if (rc) return rc;
  return launch_lora_epilogue<GM>(mem, count, M, L, ws, st);
}

// The few-token forward of `count` linears sharing one code table, on a
// zeroed workspace: the path by token count.
template <int GM>
int few_token_fwd(const FwdMember *mem, int count, int64_t M, const FewLayout &L, uint8_t *ws, DeviceInfo *dev,
                  cudaStream_t st) {
  // the weight decoded into TMEM for tcgen05 MMAs with N = tokens padded to
  // 16, 32, 64 or 128
  if (M <= 16) return launch_decode_fwd<16, GM>(mem, count, M, L, ws, dev, st);
  if (M <= 32) return launch_decode_fwd<32, GM>(mem, count, M, L, ws, dev, st);
  if (M <= 64) return launch_decode_fwd<64, GM>(mem, count, M, L, ws, dev, st);
  return launch_decode_fwd<128, GM>(mem, count, M, L, ws, dev, st);
}

struct FwdLayout {
  size_t w_hat, t, split, total;
};

FwdLayout fwd_layout(int64_t M, int64_t N, int64_t K, int r, int sms) {
  FwdLayout L;
  L.w_hat = 0;
  L.t = align_up((size_t)N * K * 2);
  L.split = L.t + align_up((size_t)M * 2 * r * 2);
  size_t part = gemm_split_ws_bytes(M, r, K, sms, true);
  if (r <= 128) {
    const RankJob tj = t_job(nullptr, M, K, nullptr, r, 1.f, nullptr);
    part = std::max(part, rank_part_bytes(&tj, 1, sms));
  }
  L.total = L.split + part;
  return L;
}

struct BwdLayout {
  size_t w_hat, g, t, split, total;
};

BwdLayout bwd_layout(int64_t M, int64_t N, int64_t K, int r, int sms) {
  BwdLayout L;
  L.w_hat = 0;
  L.g = align_up((size_t)N * K * 2);
  L.t = L.g + align_up((size_t)M * 2 * r * 2);
  L.split = L.t + align_up((size_t)M * 2 * r * 2);
  size_t sw = 0;
  sw = std::max(sw, gemm_split_ws_bytes(M, r, K, sms, true));   // T = s X L1
  sw = std::max(sw, gemm_split_ws_bytes(M, r, N, sms, true));   // G = s dY L2^T
  if (can_fold(r)) {
    sw = std::max(sw, gemm_split_ws_bytes(N, 2 * r, M, sms, true, r));   // dL2^T = dY^T [T_hi | T_lo], folded
    sw = std::max(sw, gemm_split_ws_bytes(K, 2 * r, M, sms, true, r));   // dL1 = X^T [G_hi | G_lo], folded
  } else {
    sw = std::max(sw, gemm_split_ws_bytes(N, r, M, sms, true));   // dL2^T = dY^T T_hi + dY^T T_lo
    sw = std::max(sw, gemm_split_ws_bytes(K, r, M, sms, true));   // dL1 = X^T G_hi + X^T G_lo
  }
  L.total = L.split + sw;
  return L;
}

}  // namespace

// ----------------------------------------------------- no-allocation scratch
// Fixed scratch of qlora_quantize_nf4_dq_noalloc: fp32 block constants for up
// to 2^22 blocks of 64 (16 MiB), then the fp64 per-CTA partial sums (16 KiB).
constexpr int64_t kNoallocMaxBlocks = QLORA_NOALLOC_MAX_NUMEL / 64;
constexpr size_t kNoallocC2Bytes = (size_t)kNoallocMaxBlocks * 4;
static_assert(kNoallocC2Bytes + (size_t)kQuantMaxCtas * 8 <= QLORA_NOALLOC_SCRATCH_BYTES, "scratch too small");
static __device__ __align__(256) unsigned char g_noalloc_scratch[QLORA_NOALLOC_SCRATCH_BYTES];

namespace {
void *g_noalloc_addr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the static scratch on the current device, looked up once
// per device with that device current (host code cannot use the symbol itself).
int noalloc_scratch(unsigned char **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return QLORA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = reinterpret_cast<unsigned char *>(g_noalloc_addr[dev]);
  return QLORA_OK;
}
}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" {

int qlora_version(void) { return 100; }

int qlora_profile_start(int capacity) {
  if (capacity <= 0 || capacity > (1 << 20)) return QLORA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (g_prof.cap < capacity || g_prof.dev != dev) {
    if (g_prof.ev) {
      int cur = 0;
      cudaGetDevice(&cur);
      cudaSetDevice(g_prof.dev);
      for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
      cudaSetDevice(cur);
      delete[] g_prof.ev;
      delete[] g_prof.kind;
      g_prof.ev = nullptr;
      g_prof.kind = nullptr;
      g_prof.cap = 0;
    }
    g_prof.ev = new cudaEvent_t[2 * capacity];
    g_prof.kind = new int[capacity];
    for (int i = 0; i < 2 * capacity; ++i)
      if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) return QLORA_ERR_CUDA;
    g_prof.cap = capacity;
    g_prof.dev = dev;
  }
  g_prof.used = 0;
  g_prof.on = true;
  return QLORA_OK;
}

int qlora_profile_stop(void) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  g_prof.on = false;
  return g_prof.used;
}

int qlora_profile_read(int i, int *kind, float *ms) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (i < 0 || i >= g_prof.used || !kind || !ms) return QLORA_ERR_INVALID_ARG;
  *kind = g_prof.kind[i];
  if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess) return QLORA_ERR_CUDA;
  return cudaEventElapsedTime(ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

const char *qlora_status_str(int status) {
  switch (status) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_MISALIGNED: return "misaligned pointer (16-byte alignment required)";
    case QLORA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (k_in % 64, n_out % 8, r % 8, r <= 256)";
    case QLORA_ERR_CUDA: return "CUDA runtime error";
    case QLORA_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait expired";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_SCRATCH_LIMIT: return "tensor larger than the fixed scratch of the no-allocation entry point";
    default: return "unknown status";
  }
}

int qlora_get_last_device_error(void *stream) {
  DeviceInfo *dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int h = 0;
  if (cudaMemcpyAsync(&h, dev->err, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return QLORA_ERR_CUDA;
  if (h != 0) {
    if (cudaMemsetAsync(dev->err, 0, sizeof(int), st) != cudaSuccess) return QLORA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return QLORA_ERR_CUDA;
    return QLORA_ERR_DEVICE_TIMEOUT;
  }
  return QLORA_OK;
}

int qlora_set_wait_limit_ns(uint64_t ns, void *stream) {
  if (ns > QLORA_MAX_WAIT_LIMIT_NS) return QLORA_ERR_INVALID_ARG;
  DeviceInfo *dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  set_wait_limit_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(ns == 0 ? kDefaultWaitLimitNs : ns);
  return launch_status();
}

int qlora_diag_expired_wait(void *stream) {
  DeviceInfo *dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  diag_expired_wait_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(dev->err);
  return launch_status();
}

size_t qlora_quantize_workspace_size(int64_t numel) {
  if (numel < 0) return 0;
  const int64_t nblk = (numel + 63) / 64;
  return align_up((size_t)nblk * 4) + align_up((size_t)kQuantMaxCtas * 8);
}

// The quantizer's two launches (K1: absmax, codes and fp64 partial sums of
// c2; K2: the Double-Quantization constants), with c2 and the partial sums
// in the given scratch.
static int quantize_launch(const void *W, int w_dtype, int64_t numel, int table, uint8_t *codes, uint8_t *c2_fp8,
                           float *c1, float *c2_mean, float *c2, double *partial, DeviceInfo *dev, cudaStream_t st) {
  const int64_t nblk = (numel + 63) / 64;
  // one persistent CTA per SM, each streaming whole chunks (fewer CTAs for a
  // small tensor; the groups after the last whole chunk go to the last CTA)
  const int64_t nchunks = numel / kQuantChunk;
  const int grid1 = (int)std::max<int64_t>(1, std::min<int64_t>(nchunks, std::min(kQuantMaxCtas, dev->sms)));
  const bool f32 = w_dtype == QLORA_DTYPE_F32;
  const int smem = f32 ? QuantCfg<float>::kSmemBytes : QuantCfg<__nv_bfloat16>::kSmemBytes;
  if (once(dev->quant_smem_set[f32 ? 1 : 0], [&] {
        return (f32 ? cudaFuncSetAttribute(nf4_quantize_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           smem)
                    : cudaFuncSetAttribute(nf4_quantize_kernel<__nv_bfloat16>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) == cudaSuccess
                   ? 1
                   : 0;
      }) <= 0)
    return QLORA_ERR_CUDA;
  int rc;
  {
    ProfScope prof(QLORA_KERNEL_QUANTIZE, st);
    if (f32)
      rc = launch_pdl(nf4_quantize_kernel<float>, dim3(grid1), dim3(kQuantThreads), (size_t)smem, st,
                      reinterpret_cast<const float *>(W), numel, codes, c2, partial, table, dev->err);
    else
      rc = launch_pdl(nf4_quantize_kernel<__nv_bfloat16>, dim3(grid1), dim3(kQuantThreads), (size_t)smem, st,
                      reinterpret_cast<const __nv_bfloat16 *>(W), numel, codes, c2, partial, table, dev->err);
  }
  if (rc) return rc;
  const int64_t nb256 = (nblk + 255) / 256;
  const int grid2 =
      (int)std::max<int64_t>(1, std::min<int64_t>((nb256 + kDqWarps - 1) / kDqWarps, (int64_t)dev->sms * 4));
  ProfScope prof(QLORA_KERNEL_DQ_CONSTANTS, st);
  return launch_pdl(dq_constants_kernel, dim3(grid2), dim3(32 * kDqWarps), 0, st, (const float *)c2, nblk,
                    (const double *)partial, grid1, c2_fp8, c1, c2_mean);
}

int qlora_quantize_nf4_dq(const void *W, int w_dtype, int64_t n_out, int64_t k_in, uint8_t *codes, uint8_t *c2_fp8,
                          float *c1, float *c2_mean, void *ws, size_t ws_bytes, void *stream) {
  return qlora_quantize_4bit_dq(W, w_dtype, n_out, k_in, QLORA_TABLE_NF4, codes, c2_fp8, c1, c2_mean, ws, ws_bytes,
                                stream);
}

int qlora_quantize_4bit_dq(const void *W, int w_dtype, int64_t n_out, int64_t k_in, int table, uint8_t *codes,
                           uint8_t *c2_fp8, float *c1, float *c2_mean, void *ws, size_t ws_bytes, void *stream) {
  if (n_out < 0 || k_in < 0) return QLORA_ERR_INVALID_ARG;
  if (table < 0 || table >= kNumTables) return QLORA_ERR_INVALID_ARG;
  if (w_dtype != QLORA_DTYPE_F32 && w_dtype != QLORA_DTYPE_BF16) return QLORA_ERR_INVALID_ARG;
  if (k_in > 0 && n_out > INT64_MAX / k_in) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int64_t numel = n_out * k_in;
  if (!c2_mean) return QLORA_ERR_INVALID_ARG;
  if (!aligned(c2_mean, 4)) return QLORA_ERR_MISALIGNED;
  DeviceInfo *dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (numel == 0) return cudaMemsetAsync(c2_mean, 0, sizeof(float), st) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
  if (!W || !codes || !c2_fp8 || !c1) return QLORA_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(c2_fp8, 16) || !aligned(c1, 16)) return QLORA_ERR_MISALIGNED;
  if (!ws || ws_bytes < qlora_quantize_workspace_size(numel)) return QLORA_ERR_WORKSPACE;
  if (!aligned(ws, 16)) return QLORA_ERR_MISALIGNED;
  const int64_t nblk = (numel + 63) / 64;
  float *c2 = reinterpret_cast<float *>(ws);
  double *partial = reinterpret_cast<double *>(reinterpret_cast<uint8_t *>(ws) + align_up((size_t)nblk * 4));
  return quantize_launch(W, w_dtype, numel, table, codes, c2_fp8, c1, c2_mean, c2, partial, dev, st);
}

int qlora_quantize_nf4_dq_noalloc(const void *W, int w_dtype, int64_t n_out, int64_t k_in, uint8_t *codes,
                                  uint8_t *c2_fp8, float *c1, float *c2_mean, void *stream) {
  const int table = QLORA_TABLE_NF4;   // the no-allocation quantizer writes NF4 codes
  if (n_out < 0 || k_in < 0) return QLORA_ERR_INVALID_ARG;
  if (w_dtype != QLORA_DTYPE_F32 && w_dtype != QLORA_DTYPE_BF16) return QLORA_ERR_INVALID_ARG;
  if (k_in > 0 && n_out > QLORA_NOALLOC_MAX_NUMEL / k_in) return QLORA_ERR_SCRATCH_LIMIT;
  const int64_t numel = n_out * k_in;
  if (!c2_mean) return QLORA_ERR_INVALID_ARG;
  if (!aligned(c2_mean, 4)) return QLORA_ERR_MISALIGNED;
  DeviceInfo *dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  unsigned char *scratch;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (numel == 0) return cudaMemsetAsync(c2_mean, 0, sizeof(float), st) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
  if (!W || !codes || !c2_fp8 || !c1) return QLORA_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(c2_fp8, 16) || !aligned(c1, 16)) return QLORA_ERR_MISALIGNED;
  float *c2 = reinterpret_cast<float *>(scratch);
  double *partial = reinterpret_cast<double *>(scratch + kNoallocC2Bytes);
  return quantize_launch(W, w_dtype, numel, table, codes, c2_fp8, c1, c2_mean, c2, partial, dev, st);
}

int qlora_dequant(const qlora_nf4dq_t *W, uint16_t *W_out, void *stream) {
  int rc = check_weight(W);
  if (rc) return rc;
  if (W->k_in > 0 && W->n_out > INT64_MAX / W->k_in) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (W->n_out * W->k_in == 0) return QLORA_OK;
  if (!W_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned(W_out, 16)) return QLORA_ERR_MISALIGNED;
  DeviceInfo *dev;
  rc = current_device_info(&dev);
  if (rc) return rc;
  return dequant_launch(W, reinterpret_cast<__nv_bfloat16 *>(W_out), reinterpret_cast<cudaStream_t>(stream),
                        dev->sms);
}

}  // extern "C"

namespace {

// Forward above the few-token sizes: dequant + tcgen05 GEMMs.  The adapter's
// down-projection reads Xt with scale t_scale: T = t_scale Xt L1 (Xt = X and
// t_scale = s without dropout).
// doubleDequant of W into w_hat (Eq. 6), then Y = X W_hat^T + T_hi L2 (the
// LoRA up-projection as extra K-steps of the same accumulation), given T as
// a bf16 hi/lo pair [M x 2r].
int fwd_y(const uint16_t *X, int64_t M, const qlora_nf4dq_t *W, const uint16_t *L2, int r, const uint16_t *T,
          uint16_t *Y, __nv_bfloat16 *w_hat, DeviceInfo *dev, cudaStream_t st) {
  const int64_t N = W->n_out, K = W->k_in;
  int rc = dequant_launch(W, w_hat, st, dev->sms);
  if (rc) return rc;
  GemmSeg sY[2] = {{{X, M, K, K, 0}, {w_hat, N, K, K, 0}}, {{T, M, r, 2 * r, 0}, {L2, N, r, N, 1}}};
  return tc_gemm(st, dev, M, N, 2, sY, 1.f, Y, N, 1, 0, nullptr, QLORA_KERNEL_GEMM_Y);
}

int fwd_large(const uint16_t *X, const uint16_t *Xt, float t_scale, int64_t M, const qlora_nf4dq_t *W,
              const uint16_t *L1, const uint16_t *L2, int r, uint16_t *Y, uint16_t *T_save, uint8_t *w8,
              const FwdLayout &L, DeviceInfo *dev, cudaStream_t st) {
  const int64_t N = W->n_out, K = W->k_in;
  __nv_bfloat16 *w_hat = reinterpret_cast<__nv_bfloat16 *>(w8 + L.w_hat);
  uint16_t *T = T_save ? T_save : reinterpret_cast<uint16_t *>(w8 + L.t);
  float *split_ws = reinterpret_cast<float *>(w8 + L.split);
  // 1. doubleDequant of the frozen weight into the bf16 workspace (Eq. 6).
  int rc = dequant_launch(W, w_hat, st, dev->sms);
  if (rc) return rc;
  // 2. T = s X L1 (the adapter's down-projection; L1 read MN-major), stored
  //    as a bf16 hi/lo pair [M x 2r]: T ~= T[:, :r] + T[:, r:].
  if (r <= 128) {
    const RankJob tj = t_job(Xt, M, K, L1, r, t_scale, T);
    rc = rank_launch(&tj, 1, reinterpret_cast<uint8_t *>(split_ws), dev, st, QLORA_KERNEL_GEMM_T);
  } else {
    GemmSeg sT = {{Xt, M, K, K, 0}, {L1, r, K, r, 1}};
    rc = tc_gemm(st, dev, M, r, 1, &sT, t_scale, T, 2 * r, 1, 0, split_ws, QLORA_KERNEL_GEMM_T, r);
  }
  if (rc) return rc;
  // 3. Y = X W_hat^T + T_hi L2 (the LoRA up-projection as extra K-steps).
  GemmSeg sY[2] = {{{X, M, K, K, 0}, {w_hat, N, K, K, 0}}, {{T, M, r, 2 * r, 0}, {L2, N, r, N, 1}}};
  return tc_gemm(st, dev, M, N, 2, sY, 1.f, Y, N, 1, 0, nullptr, QLORA_KERNEL_GEMM_Y);
}

// Dropout state of a backward: the adapter reads Xt (the masked input) with
// its scales multiplied by keep = 1/(1 - p), and dX's adapter term goes
// through the mask via Z = G_hi L1^T, added in the dX epilogue.
struct BwdDropout {
  const uint16_t *Xt;
  float keep;
  const uint32_t *mask;
  uint16_t *Z;   // [M x K] workspace
};

int bwd_large(const uint16_t *dY, const uint16_t *X, const uint16_t *T_saved, int64_t M, const qlora_nf4dq_t *W,
              const uint16_t *L1, const uint16_t *L2, int r, float s, uint16_t *dX, void *dL1, void *dL2,
              int out_f32, uint8_t *w8, const BwdLayout &L, const BwdDropout *drop, DeviceInfo *dev,
              cudaStream_t st) {
  const int64_t N = W->n_out, K = W->k_in;
  __nv_bfloat16 *w_hat = reinterpret_cast<__nv_bfloat16 *>(w8 + L.w_hat);
  uint16_t *G = reinterpret_cast<uint16_t *>(w8 + L.g);
  float *split_ws = reinterpret_cast<float *>(w8 + L.split);
  const uint16_t *Xt = drop ? drop->Xt : X;        // what the adapter reads
  const float keep = drop ? drop->keep : 1.f;
  const uint16_t *T = T_saved;
  int rc;
  if (!T) {  // recompute T = s X L1 (hi/lo pair)
    uint16_t *Tw = reinterpret_cast<uint16_t *>(w8 + L.t);
    GemmSeg sT = {{Xt, M, K, K, 0}, {L1, r, K, r, 1}};
    rc = tc_gemm(st, dev, M, r, 1, &sT, s * keep, Tw, 2 * r, 1, 0, split_ws, QLORA_KERNEL_GEMM_T, r);
    if (rc) return rc;
    T = Tw;
  }
  // G = s dY L2^T (L2 [r x N] is K-major for this product), as a hi/lo pair.
  GemmSeg sG = {{dY, M, N, N, 0}, {L2, r, N, N, 0}};
  rc = tc_gemm(st, dev, M, r, 1, &sG, s, G, 2 * r, 1, 0, split_ws, QLORA_KERNEL_GEMM_G, r);
  if (rc) return rc;
  if (dX) {
    // dX = dY W_hat + G_hi L1^T: W_hat [N x K] is read in place as an MN-major B.
    rc = dequant_launch(W, w_hat, st, dev->sms);
    if (rc) return rc;
    if (!drop) {
      GemmSeg sX[2] = {{{dY, M, N, N, 0}, {w_hat, K, N, K, 1}}, {{G, M, r, 2 * r, 0}, {L1, K, r, r, 0}}};
      rc = tc_gemm(st, dev, M, K, 2, sX, 1.f, dX, K, 1, 0, nullptr, QLORA_KERNEL_GEMM_DX);
    } else {
      // With dropout the adapter term is gated by the mask.  When dX runs in
      // the wide pair form, G_hi L1^T accumulates in the tile's second TMEM
      // accumulator and the epilogue stores D0 + keep * m * D1.  Otherwise
      // Z = G_hi L1^T first, then dX = dY W_hat + keep * m * Z, added before
      // the rounding.
      const bool in_tile = M > kBM && K > 128 && N >= 128 && N % 64 == 0;
      if (in_tile) {
        GemmSeg sX[2] = {{{dY, M, N, N, 0}, {w_hat, K, N, K, 1}}, {{G, M, r, 2 * r, 0}, {L1, K, r, r, 0}}};
        const GemmAddend add = {nullptr, drop->mask, keep, K};
        rc = tc_gemm(st, dev, M, K, 2, sX, 1.f, dX, K, 1, 0, nullptr, QLORA_KERNEL_GEMM_DX, 0, false, 0, &add);
      } else {
        GemmSeg sZ = {{G, M, r, 2 * r, 0}, {L1, K, r, r, 0}};
        rc = tc_gemm(st, dev, M, K, 1, &sZ, 1.f, drop->Z, K, 1, 0, nullptr, QLORA_KERNEL_GEMM_Z);
        if (rc) return rc;
        GemmSeg sX = {{dY, M, N, N, 0}, {w_hat, K, N, K, 1}};
        const GemmAddend add = {drop->Z, drop->mask, keep, K};
        rc = tc_gemm(st, dev, M, K, 1, &sX, 1.f, dX, K, 1, 0, nullptr, QLORA_KERNEL_GEMM_DX, 0, false, 0, &add);
      }
    }
    if (rc) return rc;
  }
  // dL2 = T^T dY as dL2^T [N x r] = dY^T (T_hi + T_lo), written transposed,
  // and dL1 = Xt^T (G_hi + G_lo) [K x r] (times keep).  When both halves fit
  // one tile the product runs against the whole [hi | lo] pair (2r columns)
  // and the epilogue adds the halves, so dY and X stream once; otherwise as
  // two accumulated segments over the tokens.
  if (can_fold(r)) {
    GemmSeg s2 = {{dY, N, M, N, 1}, {T, 2 * r, M, 2 * r, 1}};
    rc = tc_gemm(st, dev, N, 2 * r, 1, &s2, 1.f, dL2, 1, N, out_f32, split_ws, QLORA_KERNEL_GEMM_DL2, 0, false, r);
    if (rc) return rc;
    GemmSeg s1 = {{Xt, K, M, K, 1}, {G, 2 * r, M, 2 * r, 1}};
    return tc_gemm(st, dev, K, 2 * r, 1, &s1, keep, dL1, r, 1, out_f32, split_ws, QLORA_KERNEL_GEMM_DL1, 0, false, r);
  }
  const uint16_t *T_lo = T + r;
  GemmSeg s2[2] = {{{dY, N, M, N, 1}, {T, r, M, 2 * r, 1}}, {{dY, N, M, N, 1}, {T_lo, r, M, 2 * r, 1}}};
  rc = tc_gemm(st, dev, N, r, 2, s2, 1.f, dL2, 1, N, out_f32, split_ws, QLORA_KERNEL_GEMM_DL2, 0, true);
  if (rc) return rc;
  const uint16_t *G_lo = G + r;
  GemmSeg s1[2] = {{{Xt, K, M, K, 1}, {G, r, M, 2 * r, 1}}, {{Xt, K, M, K, 1}, {G_lo, r, M, 2 * r, 1}}};
  return tc_gemm(st, dev, K, r, 2, s1, keep, dL1, r, 1, out_f32, split_ws, QLORA_KERNEL_GEMM_DL1, 0, true);
}

// ------------------------------------------ grouped backward (many tokens)
struct BwdMember {
  const uint16_t *dY, *X, *T;   // X: what the adapter reads (the masked input under LoRA dropout)
  const qlora_nf4dq_t *W;
  const uint16_t *L1, *L2;
  int r;
  float s;
  uint16_t *dX;
  void *dL1, *dL2;
  float keep = 1.f;             // LoRA dropout's 1 / (1 - p): scales T's recomputation and dL1
};

// The grouped rank kernel serves ranks whose [hi | lo] pair fits one
// 128-column tile with the fold's chunking.
bool rank_group_ok(int r) { return r <= 64 && can_fold(r); }

// Workspace of a grouped backward.  G holds every member's hi/lo pair side by
// side ([M x sum 2r] bf16), the members that share X (same pointer, K and r)
// next to each other, so that their dL1 products read one [M x 2r*n] operand.
struct BwdGroupLayout {
  size_t g = 0, t = 0, w_hat = 0, part = 0, total = 0;
  int64_t g_ld = 0;
  int64_t g_col[kMaxGroup] = {};
  size_t t_off[kMaxGroup] = {};
  int set_of[kMaxGroup] = {};   // X set of each member
  int nsets = 0;
  int set_first[kMaxGroup] = {}, set_size[kMaxGroup] = {};
};

// The rank problems of the three launches: T (members without T_saved), G and
// dL2 (every member), dL1 (one problem per X set when its n-tiles line up with
// the members' pairs, else one per member).  Pointers into the workspace are
// taken relative to `w8` (nullptr when only sizing).
struct BwdGroupJobs {
  RankJob t[kMaxGroup], gl2[2 * kMaxGroup], l1[kMaxGroup];
  int nt = 0, ngl2 = 0, nl1 = 0;
};

void bwd_group_jobs(int64_t M, const BwdMember *mem, int count, const BwdGroupLayout &L, uint8_t *w8, bool f32,
                    bool t_all, BwdGroupJobs &J) {
  auto at = [w8](size_t off) { return reinterpret_cast<uint16_t *>(reinterpret_cast<uintptr_t>(w8) + off); };
  uint16_t *G = at(L.g);
  for (int i = 0; i < count; ++i) {
    const BwdMember &m = mem[i];
    const int64_t N = m.W->n_out, K = m.W->k_in;
    const int r = m.r;
    const uint16_t *T = m.T;
    if (!T || t_all) {   // T = s X L1 as a hi/lo pair
      uint16_t *Tw = at(L.t + L.t_off[i]);
      RankJob &j = J.t[J.nt++];
      j.A = {m.X, M, K, K, 0};
      j.B = {m.L1, r, K, r, 1};
      j.bn = 64;
      j.n_tiles = 1;
      j.ncols = r;
      j.fold = 0;
      j.outs[0] = RankOut{Tw, nullptr, 2 * r, 1, r, m.s * m.keep, 0};
      T = Tw;
    }
    RankJob &jg = J.gl2[J.ngl2++];   // G = s dY L2^T (L2 [r x N] is K-major here)
    jg.A = {m.dY, M, N, N, 0};
    jg.B = {m.L2, r, N, N, 0};
    jg.bn = 64;
    jg.n_tiles = 1;
    jg.ncols = r;
    jg.fold = 0;
    jg.outs[0] = RankOut{G + L.g_col[i], nullptr, L.g_ld, 1, r, m.s, 0};
    RankJob &j2 = J.gl2[J.ngl2++];   // dL2^T = dY^T [T_hi | T_lo], folded, written transposed
    j2.A = {m.dY, N, M, N, 1};
    j2.B = {T, 2 * r, M, 2 * r, 1};
    j2.bn = 2 * r <= 64 ? 64 : 128;
    j2.n_tiles = 1;
    j2.ncols = 2 * r;
    j2.fold = r;
    j2.outs[0] = RankOut{m.dL2, nullptr, 1, N, 0, 1.f, f32 ? 1 : 0};
  }
  for (int sidx = 0; sidx < L.nsets; ++sidx) {
    const int first = L.set_first[sidx], n = L.set_size[sidx];
    const BwdMember &m0 = mem[first];
    const int64_t K = m0.W->k_in;
    const int r = m0.r;
    const bool joint = 2 * r == 64 || 2 * r == 128;   // n-tile t = member t's [hi | lo]
    int members[kMaxGroup], k = 0;
    for (int i = 0; i < count; ++i)
      if (L.set_of[i] == sidx) members[k++] = i;
    if (joint) {
      RankJob &j = J.l1[J.nl1++];   // dL1 = X^T [G_hi | G_lo] of every member of the set
      j.A = {m0.X, K, M, K, 1};
      j.B = {G + L.g_col[first], (int64_t)n * 2 * r, M, L.g_ld, 1};
      j.bn = 2 * r;
      j.n_tiles = n;
      j.ncols = 2 * r;
      j.fold = r;
      for (int t = 0; t < n; ++t) j.outs[t] = RankOut{mem[members[t]].dL1, nullptr, r, 1, 0, mem[members[t]].keep, f32 ? 1 : 0};
    } else {
      for (int t = 0; t < n; ++t) {
        const int i = members[t];
        RankJob &j = J.l1[J.nl1++];
        j.A = {m0.X, K, M, K, 1};
        j.B = {G + L.g_col[i], 2 * r, M, L.g_ld, 1};
        j.bn = 64;
        j.n_tiles = 1;
        j.ncols = 2 * r;
        j.fold = r;
        j.outs[0] = RankOut{mem[i].dL1, nullptr, r, 1, 0, mem[i].keep, f32 ? 1 : 0};
      }
    }
  }
}

BwdGroupLayout bwd_group_layout(int64_t M, const BwdMember *mem, int count, int sms) {
  BwdGroupLayout L;
  // X sets, in order of first appearance
  for (int i = 0; i < count; ++i) {
    int s = -1;
    for (int k = 0; k < L.nsets && s < 0; ++k) {
      const BwdMember &f = mem[L.set_first[k]];
      if (f.X == mem[i].X && f.W->k_in == mem[i].W->k_in && f.r == mem[i].r && f.keep == mem[i].keep) s = k;
    }
    if (s < 0) {
      s = L.nsets++;
      L.set_first[s] = i;
    }
    L.set_of[i] = s;
    ++L.set_size[s];
  }
  int64_t col = 0;
  for (int s = 0; s < L.nsets; ++s)
    for (int i = 0; i < count; ++i)
      if (L.set_of[i] == s) {
        L.g_col[i] = col;
        col += 2 * mem[i].r;
      }
  L.g_ld = col;
  size_t t_bytes = 0, w_bytes = 0;
  for (int i = 0; i < count; ++i) {
    L.t_off[i] = t_bytes;
    t_bytes += align_up((size_t)M * 2 * mem[i].r * 2);
    w_bytes = std::max(w_bytes, (size_t)mem[i].W->n_out * mem[i].W->k_in * 2);
  }
  L.g = 0;
  L.t = align_up((size_t)M * L.g_ld * 2);
  L.w_hat = L.t + t_bytes;
  L.part = L.w_hat + align_up(w_bytes);
  // T space for every member: the size does not depend on which T_saved are given
  BwdGroupJobs J;
  bwd_group_jobs(M, mem, count, L, nullptr, false, true, J);
  size_t pb = 0;
  for (int i = 0; i < J.nt; ++i) pb = std::max(pb, rank_part_bytes(&J.t[i], 1, sms));   // one launch each
  pb = std::max(pb, rank_part_bytes(J.gl2, J.ngl2, sms));
  pb = std::max(pb, rank_part_bytes(J.l1, J.nl1, sms));
  L.total = L.part + pb;
  return L;
}

// The backward of linears whose rank products run grouped (rank_group_ok):
// [T of members without T_saved] -> G and dL2 of all -> dL1 per X set ->
// per member doubleDequant and dX = dY W_hat + G_hi L1^T.
// With LoRA dropout (`drop`, a group of one whose X is the masked input) the
// adapter term of dX goes through the mask as in bwd_large.
int bwd_group_large(int64_t M, const BwdMember *mem, int count, bool f32, uint8_t *w8, const BwdGroupLayout &L,
                    DeviceInfo *dev, cudaStream_t st, const BwdDropout *drop = nullptr) {
  if (drop && count != 1) return QLORA_ERR_UNSUPPORTED_SHAPE;
  BwdGroupJobs J;
  bwd_group_jobs(M, mem, count, L, w8, f32, false, J);
  uint8_t *part = w8 + L.part;
  int rc;
  for (int i = 0; i < J.nt; ++i) {   // a member without T_saved: recompute it alone
    rc = rank_launch(&J.t[i], 1, part, dev, st, QLORA_KERNEL_GEMM_T);
    if (rc) return rc;
  }
  rc = rank_launch(J.gl2, J.ngl2, part, dev, st, QLORA_KERNEL_RANK_G_DL2);
  if (rc) return rc;
  rc = rank_launch(J.l1, J.nl1, part, dev, st, QLORA_KERNEL_RANK_DL1);
  if (rc) return rc;
  __nv_bfloat16 *w_hat = reinterpret_cast<__nv_bfloat16 *>(w8 + L.w_hat);
  const uint16_t *G = reinterpret_cast<const uint16_t *>(w8 + L.g);
  for (int i = 0; i < count; ++i) {
    const BwdMember &m = mem[i];
    if (!m.dX) continue;
    const int64_t N = m.W->n_out, K = m.W->k_in;
    rc = dequant_launch(m.W, w_hat, st, dev->sms);
    if (rc) return rc;
    const Operand g_hi = {G + L.g_col[i], M, m.r, L.g_ld, 0};
    const Operand l1t = {m.L1, K, m.r, m.r, 0};
    if (!drop) {
      GemmSeg sX[2] = {{{m.dY, M, N, N, 0}, {w_hat, K, N, K, 1}}, {g_hi, l1t}};
      rc = tc_gemm(st, dev, M, K, 2, sX, 1.f, m.dX, K, 1, 0, nullptr, QLORA_KERNEL_GEMM_DX);
    } else if (M > kBM && K > 128 && N >= 128 && N % 64 == 0) {
      // the masked adapter term in the pair tile's second accumulator
      GemmSeg sX[2] = {{{m.dY, M, N, N, 0}, {w_hat, K, N, K, 1}}, {g_hi, l1t}};
      const GemmAddend add = {nullptr, drop->mask, drop->keep, K};
      rc = tc_gemm(st, dev, M, K, 2, sX, 1.f, m.dX, K, 1, 0, nullptr, QLORA_KERNEL_GEMM_DX, 0, false, 0, &add);
    } else {
      GemmSeg sZ = {g_hi, l1t};
      rc = tc_gemm(st, dev, M, K, 1, &sZ, 1.f, drop->Z, K, 1, 0, nullptr, QLORA_KERNEL_GEMM_Z);
      if (rc) return rc;
      GemmSeg sX = {{m.dY, M, N, N, 0}, {w_hat, K, N, K, 1}};
      const GemmAddend add = {drop->Z, drop->mask, drop->keep, K};
      rc = tc_gemm(st, dev, M, K, 1, &sX, 1.f, m.dX, K, 1, 0, nullptr, QLORA_KERNEL_GEMM_DX, 0, false, 0, &add);
    }
    if (rc) return rc;
  }
  return QLORA_OK;
}

// Xm = X * m into the workspace.
int dropout_launch(const uint16_t *X, const uint32_t *mask, int64_t numel, uint16_t *Xm, DeviceInfo *dev,
                   cudaStream_t st) {
  if (numel == 0) return QLORA_OK;
  const int64_t n8 = numel >> 3;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((n8 + 255) / 256, (int64_t)dev->sms * 16));
  ProfScope prof(QLORA_KERNEL_DROPOUT_MASK, st);
  return launch_pdl(dropout_mask_kernel, dim3(grid), dim3(256), 0, st, X, mask, numel, Xm);
}

}  // namespace

extern "C" {

size_t qlora_linear_fwd_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r) {
  if (M < 0 || n_out <= 0 || k_in <= 0 || r <= 0) return 0;
  if (M <= kFewMaxM) return few_ws_bytes(M, n_out, r);
  DeviceInfo *dev;
  const int sms = current_device_info(&dev) == QLORA_OK ? dev->sms : 148;
  return fwd_layout(M, n_out, k_in, r, sms).total;
}

size_t qlora_linear_bwd_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r) {
  if (M < 0 || n_out <= 0 || k_in <= 0 || r <= 0) return 0;
  DeviceInfo *dev;
  const int sms = current_device_info(&dev) == QLORA_OK ? dev->sms : 148;
  if (M > 0 && rank_group_ok(r)) {   // the single-linear backward runs as a group of one
    qlora_nf4dq_t w;
    std::memset(&w, 0, sizeof(w));
    w.n_out = n_out;
    w.k_in = k_in;
    const BwdMember m = {nullptr, nullptr, nullptr, &w, nullptr, nullptr, r, 1.f, nullptr, nullptr, nullptr};
    return bwd_group_layout(M, &m, 1, sms).total;
  }
  return bwd_layout(M, n_out, k_in, r, sms).total;
}

int qlora_linear_fwd(const uint16_t *X, int64_t M, const qlora_nf4dq_t *W, const uint16_t *L1, const uint16_t *L2,
                     int r, float s, uint16_t *Y, uint16_t *T_save, void *ws, size_t ws_bytes, void *stream) {
  int rc = check_linear(M, W, r);
  if (rc) return rc;
  if (M == 0) return QLORA_OK;
  if (!X || !L1 || !L2 || !Y) return QLORA_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(L1, 16) || !aligned(L2, 16) || !aligned(Y, 16) || (T_save && !aligned(T_save, 16)))
    return QLORA_ERR_MISALIGNED;
  DeviceInfo *dev;
  rc = current_device_info(&dev);
  if (rc) return rc;
  const int64_t N = W->n_out, K = W->k_in;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (M <= kFewMaxM) {
    // Few tokens: the weight bytes dominate; one fused decode + product pass.
    const FwdMember mem = {W, X, L1, L2, r, s, Y, T_save};
    const FewLayout L = few_layout(M, &mem, 1);
    if (!ws || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
    uint8_t *w8 = reinterpret_cast<uint8_t *>(ws);
    if (cudaMemsetAsync(w8, 0, L.zero_bytes, st) != cudaSuccess) return QLORA_ERR_CUDA;
    return few_token_fwd<1>(&mem, 1, M, L, w8, dev, st);
  }
  const FwdLayout L = fwd_layout(M, N, K, r, dev->sms);
  if (!ws || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
  return fwd_large(X, X, s, M, W, L1, L2, r, Y, T_save, reinterpret_cast<uint8_t *>(ws), L, dev, st);
}

// ------------------------------------------------ grouped forward, many tokens
// Sets of members that read the same X (same pointer and K), in order of
// their first member: set_of[i] is member i's set.
static int x_sets(const FwdMember *mem, int count, int *set_of) {
  int n = 0;
  for (int i = 0; i < count; ++i) {
    set_of[i] = -1;
    for (int j = 0; j < i; ++j)
      if (mem[j].X == mem[i].X && mem[j].W->k_in == mem[i].W->k_in) {
        set_of[i] = set_of[j];
        break;
      }
    if (set_of[i] < 0) set_of[i] = n++;
  }
  return n;
}

// Workspace: the bf16 weight (largest member, reused member after member);
// L1_cat bf16 [K x R] of the largest set that shares X with equal ranks of 64
// or 128; each member's T pair [M x 2r] (used where it passes no T_save); the
// split partials of the largest adapter launch.
struct GroupLargeLayout {
  size_t w_hat, l1_cat, t_own[kMaxGroup], split, total;
};

// The adapter down-projections of the members of one X set (same input
// pointer and K) as problems of one rank launch: with equal ranks of 64 or 128
// one problem over L1_cat = [L1_a | L1_b | ...] whose n-tile k is member k
// (each 128-row strip of X is read for all members on neighbouring CTAs),
// otherwise one problem per member.  Returns false when a rank is above 128.
static bool fwd_set_jobs(int64_t M, const FwdMember *mem, const int *idx, int n, uint16_t *const *T,
                         const uint16_t *l1_cat, RankJob *jobs, int *njobs, bool *joint) {
  const FwdMember &m0 = mem[idx[0]];
  const int64_t K = m0.W->k_in;
  bool same = true;
  for (int k = 0; k < n; ++k) {
    if (mem[idx[k]].r > 128) return false;
    same = same && mem[idx[k]].r == m0.r;
  }
  *joint = same && n > 1 && (m0.r == 64 || m0.r == 128);
  if (*joint) {
    RankJob &j = jobs[0];
    j.A = {m0.X, M, K, K, 0};
    j.B = {l1_cat, (int64_t)n * m0.r, K, (int64_t)n * m0.r, 1};
    j.bn = m0.r;
    j.n_tiles = n;
    j.ncols = m0.r;
    j.fold = 0;
    for (int k = 0; k < n; ++k) j.outs[k] = RankOut{T[k], nullptr, 2 * m0.r, 1, m0.r, mem[idx[k]].s, 0};
    *njobs = 1;
  } else {
    for (int k = 0; k < n; ++k) {
      const FwdMember &m = mem[idx[k]];
      jobs[k] = t_job(m.X, M, K, m.L1, m.r, m.s, T[k]);
    }
    *njobs = n;
  }
  return true;
}

static GroupLargeLayout group_large_layout(int64_t M, const FwdMember *mem, int count, int sms) {
  int set_of[kMaxGroup];
  const int nsets = x_sets(mem, count, set_of);
  size_t w = 0, l1cat = 0, split = 0;
  for (int i = 0; i < count; ++i) w = std::max(w, (size_t)mem[i].W->n_out * mem[i].W->k_in * 2);
  for (int s = 0; s < nsets; ++s) {
    int idx[kMaxGroup], n = 0;
    for (int i = 0; i < count; ++i)
      if (set_of[i] == s) idx[n++] = i;
    int64_t R = 0;
    for (int k = 0; k < n; ++k) R += mem[idx[k]].r;
    uint16_t *T[kMaxGroup] = {};
    RankJob jobs[kMaxGroup];
    int nj = 0;
    bool joint = false;
    if (n > 1 && fwd_set_jobs(M, mem, idx, n, T, nullptr, jobs, &nj, &joint)) {
      split = std::max(split, rank_part_bytes(jobs, nj, sms));
      if (joint) l1cat = std::max(l1cat, (size_t)mem[idx[0]].W->k_in * R * 2);
    } else {
      for (int k = 0; k < n; ++k) {
        const FwdMember &m = mem[idx[k]];
        const FwdLayout FL = fwd_layout(M, m.W->n_out, m.W->k_in, m.r, sms);
        split = std::max(split, FL.total - FL.split);
      }
    }
  }
  GroupLargeLayout L;
  size_t off = 0;
  L.w_hat = off;
  off += align_up(w);
  L.l1_cat = off;
  off += align_up(l1cat);
  for (int i = 0; i < count; ++i) {
    L.t_own[i] = off;
    off += align_up((size_t)M * 2 * mem[i].r * 2);
  }
  L.split = off;
  off += align_up(split);
  L.total = off;
  return L;
}

// The grouped forward at many tokens (M > 128) on a workspace laid out by
// group_large_layout: per X set one rank launch for the members' T, then each
// member's doubleDequant and Y product.
static int group_large_fwd(int64_t M, const FwdMember *mem, int count, uint8_t *w8, const GroupLargeLayout &L,
                           DeviceInfo *dev, cudaStream_t st) {
  int set_of[kMaxGroup];
  const int nsets = x_sets(mem, count, set_of);
  __nv_bfloat16 *w_hat = reinterpret_cast<__nv_bfloat16 *>(w8 + L.w_hat);
  for (int s = 0; s < nsets; ++s) {
    int idx[kMaxGroup], n = 0;
    for (int i = 0; i < count; ++i)
      if (set_of[i] == s) idx[n++] = i;
    uint16_t *T[kMaxGroup];
    for (int k = 0; k < n; ++k) {
      const FwdMember &m = mem[idx[k]];
      T[k] = m.T_save ? m.T_save : reinterpret_cast<uint16_t *>(w8 + L.t_own[idx[k]]);
    }
    int rc;
    uint16_t *l1_cat = reinterpret_cast<uint16_t *>(w8 + L.l1_cat);
    RankJob jobs[kMaxGroup];
    int nj = 0;
    bool joint = false;
    if (n == 1 || !fwd_set_jobs(M, mem, idx, n, T, l1_cat, jobs, &nj, &joint)) {
      for (int k = 0; k < n; ++k) {
        const FwdMember &m = mem[idx[k]];
        FwdLayout FL;
        FL.w_hat = L.w_hat;
        FL.t = L.t_own[idx[k]];
        FL.split = L.split;
        FL.total = L.total;
        rc = fwd_large(m.X, m.X, m.s, M, m.W, m.L1, m.L2, m.r, m.Y, m.T_save, w8, FL, dev, st);
        if (rc) return rc;
      }
      continue;
    }
    if (joint) {   // L1_cat [K x n r]: member k's L1 [K x r] in columns k r .. k r + r
      const int64_t K = mem[idx[0]].W->k_in;
      const int r = mem[idx[0]].r;
      for (int k = 0; k < n; ++k)
        if (cudaMemcpy2DAsync(l1_cat + (int64_t)k * r, (size_t)n * r * 2, mem[idx[k]].L1, (size_t)r * 2,
                              (size_t)r * 2, (size_t)K, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
          return QLORA_ERR_CUDA;
    }
    rc = rank_launch(jobs, nj, w8 + L.split, dev, st, QLORA_KERNEL_GEMM_T);
    if (rc) return rc;
    for (int k = 0; k < n; ++k) {
      const FwdMember &m = mem[idx[k]];
      rc = fwd_y(m.X, M, m.W, m.L2, m.r, T[k], m.Y, w_hat, dev, st);
      if (rc) return rc;
    }
  }
  return QLORA_OK;
}

// ------------------------------------------------------------- grouped forward
static_assert(kMaxGroup == QLORA_MAX_GROUP, "group size of the C ABI");
// Members are validated as by qlora_linear_fwd; the few-token path runs one
// launch chain per code table present (normally one for the whole group).
static int check_fwd_group(const qlora_fwd_member_t *members, int count, int64_t M) {
  if (count < 0 || count > QLORA_MAX_GROUP || (count > 0 && !members)) return QLORA_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    const qlora_fwd_member_t &m = members[i];
    int rc = check_linear(M, m.W, m.r);
    if (rc) return rc;
    if (M == 0) continue;
    if (!m.X || !m.L1 || !m.L2 || !m.Y) return QLORA_ERR_INVALID_ARG;
    if (!aligned(m.X, 16) || !aligned(m.L1, 16) || !aligned(m.L2, 16) || !aligned(m.Y, 16) ||
        (m.T_save && !aligned(m.T_save, 16)))
      return QLORA_ERR_MISALIGNED;
  }
  return QLORA_OK;
}

static void fwd_members(const qlora_fwd_member_t *members, int count, FwdMember *mem) {
  for (int i = 0; i < count; ++i) {
    const qlora_fwd_member_t &m = members[i];
    mem[i] = FwdMember{m.W, m.X, m.L1, m.L2, m.r, m.s, m.Y, m.T_save};
  }
}

size_t qlora_linear_fwd_group_workspace_size(const qlora_fwd_member_t *members, int count, int64_t M) {
  if (M < 0 || count < 0 || count > QLORA_MAX_GROUP || (count > 0 && !members)) return 0;
  for (int i = 0; i < count; ++i)
    if (!members[i].W || members[i].W->n_out <= 0 || members[i].W->k_in <= 0 || members[i].r <= 0) return 0;
  FwdMember mem[kMaxGroup];
  fwd_members(members, count, mem);
  if (M <= kFewMaxM) return few_layout(M, mem, count).total;
  DeviceInfo *dev;
  const int sms = current_device_info(&dev) == QLORA_OK ? dev->sms : 148;
  return group_large_layout(M, mem, count, sms).total;
}

int qlora_linear_fwd_group(const qlora_fwd_member_t *members, int count, int64_t M, void *ws, size_t ws_bytes,
                           void *stream) {
  int rc = check_fwd_group(members, count, M);
  if (rc) return rc;
  if (count == 0 || M == 0) return QLORA_OK;
  DeviceInfo *dev;
  rc = current_device_info(&dev);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  FwdMember mem[kMaxGroup];
  fwd_members(members, count, mem);
  if (M <= kFewMaxM) {
    const FewLayout L = few_layout(M, mem, count);
    if (!ws || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
    uint8_t *w8 = reinterpret_cast<uint8_t *>(ws);
    if (cudaMemsetAsync(w8, 0, L.zero_bytes, st) != cudaSuccess) return QLORA_ERR_CUDA;
    for (int t = 0; t < kNumTables; ++t) {
      FwdMember sub[kMaxGroup];
      FewLayout SL = L;
      int n = 0;
      for (int i = 0; i < count; ++i)
        if (mem[i].W->table == t) {
          sub[n] = mem[i];
          SL.acc[n] = L.acc[i];
          SL.tacc[n] = L.tacc[i];
          ++n;
        }
      if (n == 0) continue;
      rc = n == 1 ? few_token_fwd<1>(sub, 1, M, SL, w8, dev, st) : few_token_fwd<kMaxGroup>(sub, n, M, SL, w8, dev, st);
      if (rc) return rc;
    }
    return QLORA_OK;
  }
  // Many tokens: members that share X share one adapter down-projection; then
  // each runs its own doubleDequant and tensor-core product, in order.
  const GroupLargeLayout L = group_large_layout(M, mem, count, dev->sms);
  if (!ws || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
  return group_large_fwd(M, mem, count, reinterpret_cast<uint8_t *>(ws), L, dev, st);
}

int qlora_linear_bwd(const uint16_t *dY, const uint16_t *X, const uint16_t *T_saved, int64_t M,
                     const qlora_nf4dq_t *W, const uint16_t *L1, const uint16_t *L2, int r, float s, uint16_t *dX,
                     void *dL1, void *dL2, int grad_dtype, void *ws, size_t ws_bytes, void *stream) {
  int rc = check_linear(M, W, r);
  if (rc) return rc;
  if (grad_dtype != QLORA_DTYPE_F32 && grad_dtype != QLORA_DTYPE_BF16) return QLORA_ERR_INVALID_ARG;
  if (!L1 || !L2 || !dL1 || !dL2) return QLORA_ERR_INVALID_ARG;
  if (M > 0 && (!dY || !X)) return QLORA_ERR_INVALID_ARG;
  if (!aligned(L1, 16) || !aligned(L2, 16) || !aligned(dL1, 16) || !aligned(dL2, 16) || (dY && !aligned(dY, 16)) ||
      (X && !aligned(X, 16)) || (dX && !aligned(dX, 16)) || (T_saved && !aligned(T_saved, 16)))
    return QLORA_ERR_MISALIGNED;
  DeviceInfo *dev;
  rc = current_device_info(&dev);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t N = W->n_out, K = W->k_in;
  const size_t gsz = grad_dtype == QLORA_DTYPE_F32 ? 4 : 2;
  if (M == 0) {  // no tokens: the adapter gradients are zero
    if (cudaMemsetAsync(dL1, 0, (size_t)K * r * gsz, st) != cudaSuccess) return QLORA_ERR_CUDA;
    if (cudaMemsetAsync(dL2, 0, (size_t)r * N * gsz, st) != cudaSuccess) return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  if (rank_group_ok(r)) {   // a group of one: G and dL2 in one launch, then dL1
    const BwdMember m = {dY, X, T_saved, W, L1, L2, r, s, dX, dL1, dL2};
    const BwdGroupLayout L = bwd_group_layout(M, &m, 1, dev->sms);
    if (!ws || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
    return bwd_group_large(M, &m, 1, grad_dtype == QLORA_DTYPE_F32, reinterpret_cast<uint8_t *>(ws), L, dev, st);
  }
  const BwdLayout L = bwd_layout(M, N, K, r, dev->sms);
  if (!ws || ws_bytes < L.total) return QLORA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
  return bwd_large(dY, X, T_saved, M, W, L1, L2, r, s, dX, dL1, dL2, grad_dtype == QLORA_DTYPE_F32,
                   reinterpret_cast<uint8_t *>(ws), L, nullptr, dev, st);
}

static int check_bwd_member(const qlora_bwd_member_t &m, int64_t M) {
  int rc = check_linear(M, m.W, m.r);
  if (rc) return rc;
  if (!m.L1 || !m.L2 || !m.dL1 || !m.dL2) return QLORA_ERR_INVALID_ARG;
  if (M > 0 && (!m.dY || !m.X)) return QLORA_ERR_INVALID_ARG;
  if (!aligned(m.L1, 16) || !aligned(m.L2, 16) || !aligned(m.dL1, 16) || !aligned(m.dL2, 16) ||
      (m.dY && !aligned(m.dY, 16)) || (m.X && !aligned(m.X, 16)) || (m.dX && !aligned(m.dX, 16)) ||
      (m.T_saved && !aligned(m.T_saved, 16)))
    return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

static BwdMember bwd_member(const qlora_bwd_member_t &m) {
  return BwdMember{m.dY, m.X, m.T_saved, m.W, m.L1, m.L2, m.r, m.s, m.dX, m.dL1, m.dL2};
}

// Grouped members first (one layout), the others one at a time after them.
static size_t bwd_group_ws(int64_t M, const qlora_bwd_member_t *members, int count, int sms) {
  BwdMember grp[kMaxGroup];
  int ng = 0;
  size_t other = 0;
  for (int i = 0; i < count; ++i) {
    const qlora_bwd_member_t &m = members[i];
    if (rank_group_ok(m.r)) grp[ng++] = bwd_member(m);
    else other = std::max(other, bwd_layout(M, m.W->n_out, m.W->k_in, m.r, sms).total);
  }
  return std::max(other, ng ? bwd_group_layout(M, grp, ng, sms).total : (size_t)0);
}

size_t qlora_linear_bwd_group_workspace_size(const qlora_bwd_member_t *members, int count, int64_t M) {
  if (M < 0 || count < 0 || count > QLORA_MAX_GROUP || (count > 0 && !members)) return 0;
  for (int i = 0; i < count; ++i)
    if (!members[i].W || members[i].W->n_out <= 0 || members[i].W->k_in <= 0 || members[i].r <= 0) return 0;
  if (M == 0) return 0;
  DeviceInfo *dev;
  const int sms = current_device_info(&dev) == QLORA_OK ? dev->sms : 148;
  return bwd_group_ws(M, members, count, sms);
}

int qlora_linear_bwd_group(const qlora_bwd_member_t *members, int count, int64_t M, int grad_dtype, void *ws,
                           size_t ws_bytes, void *stream) {
  if (count < 0 || count > QLORA_MAX_GROUP || (count > 0 && !members) || M < 0) return QLORA_ERR_INVALID_ARG;
  if (grad_dtype != QLORA_DTYPE_F32 && grad_dtype != QLORA_DTYPE_BF16) return QLORA_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    const int rc = check_bwd_member(members[i], M);
    if (rc) return rc;
  }
  if (count == 0) return QLORA_OK;
  DeviceInfo *dev;
  int rc = current_device_info(&dev);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool f32 = grad_dtype == QLORA_DTYPE_F32;
  if (M == 0) {  // no tokens: the adapter gradients are zero
    const size_t gsz = f32 ? 4 : 2;
    for (int i = 0; i < count; ++i) {
      const qlora_bwd_member_t &m = members[i];
      if (cudaMemsetAsync(m.dL1, 0, (size_t)m.W->k_in * m.r * gsz, st) != cudaSuccess) return QLORA_ERR_CUDA;
      if (cudaMemsetAsync(m.dL2, 0, (size_t)m.r * m.W->n_out * gsz, st) != cudaSuccess) return QLORA_ERR_CUDA;
    }
    return QLORA_OK;
  }
  if (!ws || ws_bytes < bwd_group_ws(M, members, count, dev->sms)) return QLORA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
  uint8_t *w8 = reinterpret_cast<uint8_t *>(ws);
  BwdMember grp[kMaxGroup];
  int ng = 0;
  for (int i = 0; i < count; ++i)
    if (rank_group_ok(members[i].r)) grp[ng++] = bwd_member(members[i]);
  if (ng) {
    const BwdGroupLayout L = bwd_group_layout(M, grp, ng, dev->sms);
    rc = bwd_group_large(M, grp, ng, f32, w8, L, dev, st);
    if (rc) return rc;
  }
  for (int i = 0; i < count; ++i) {
    const qlora_bwd_member_t &m = members[i];
    if (rank_group_ok(m.r)) continue;
    const BwdLayout L = bwd_layout(M, m.W->n_out, m.W->k_in, m.r, dev->sms);
    rc = bwd_large(m.dY, m.X, m.T_saved, M, m.W, m.L1, m.L2, m.r, m.s, m.dX, m.dL1, m.dL2, f32, w8, L, nullptr,
                   dev, st);
    if (rc) return rc;
  }
  return QLORA_OK;
}

// ---------------------------------------------------------------- LoRA dropout
// Workspace: the plain large-M layout, then Xm [M x K] bf16 (and, backward,
// Z [M x K] bf16).
size_t qlora_linear_fwd_dropout_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r) {
  if (M < 0 || n_out <= 0 || k_in <= 0 || r <= 0) return 0;
  DeviceInfo *dev;
  const int sms = current_device_info(&dev) == QLORA_OK ? dev->sms : 148;
  return fwd_layout(M, n_out, k_in, r, sms).total + align_up((size_t)M * k_in * 2);
}

// The backward's own layout (that of a group of one where the rank-r products
// run grouped), then Xm [M x K] and Z [M x K] bf16.
static size_t bwd_dropout_base(int64_t M, int64_t n_out, int64_t k_in, int r, int sms) {
  if (M > 0 && rank_group_ok(r)) {
    qlora_nf4dq_t w;
    std::memset(&w, 0, sizeof(w));
    w.n_out = n_out;
    w.k_in = k_in;
    BwdMember m = {nullptr, nullptr, nullptr, &w, nullptr, nullptr, r, 1.f, nullptr, nullptr, nullptr};
    return bwd_group_layout(M, &m, 1, sms).total;
  }
  return bwd_layout(M, n_out, k_in, r, sms).total;
}

size_t qlora_linear_bwd_dropout_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r) {
  if (M < 0 || n_out <= 0 || k_in <= 0 || r <= 0) return 0;
  DeviceInfo *dev;
  const int sms = current_device_info(&dev) == QLORA_OK ? dev->sms : 148;
  return bwd_dropout_base(M, n_out, k_in, r, sms) + 2 * align_up((size_t)M * k_in * 2);
}

int qlora_linear_fwd_dropout(const uint16_t *X, int64_t M, const qlora_nf4dq_t *W, const uint16_t *L1,
                             const uint16_t *L2, int r, float s, const uint32_t *mask, float p, uint16_t *Y,
                             uint16_t *T_save, uint16_t *Xm_save, void *ws, size_t ws_bytes, void *stream) {
  int rc = check_linear(M, W, r);
  if (rc) return rc;
  if (!(p >= 0.f && p < 1.f)) return QLORA_ERR_INVALID_ARG;
  if (M == 0) return QLORA_OK;
  if (!X || !L1 || !L2 || !Y || !mask) return QLORA_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(L1, 16) || !aligned(L2, 16) || !aligned(Y, 16) || !aligned(mask, 16) ||
      (T_save && !aligned(T_save, 16)) || (Xm_save && !aligned(Xm_save, 16)))
    return QLORA_ERR_MISALIGNED;
  DeviceInfo *dev;
  rc = current_device_info(&dev);
  if (rc) return rc;
  const int64_t N = W->n_out, K = W->k_in;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const FwdLayout L = fwd_layout(M, N, K, r, dev->sms);
  if (!ws || ws_bytes < qlora_linear_fwd_dropout_workspace_size(M, N, K, r)) return QLORA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
  uint8_t *w8 = reinterpret_cast<uint8_t *>(ws);
  uint16_t *Xm = Xm_save ? Xm_save : reinterpret_cast<uint16_t *>(w8 + L.total);
  rc = dropout_launch(X, mask, M * K, Xm, dev, st);
  if (rc) return rc;
  return fwd_large(X, Xm, s / (1.f - p), M, W, L1, L2, r, Y, T_save, w8, L, dev, st);
}

int qlora_linear_bwd_dropout(const uint16_t *dY, const uint16_t *X, const uint16_t *T_saved,
                             const uint16_t *Xm_saved, int64_t M, const qlora_nf4dq_t *W, const uint16_t *L1,
                             const uint16_t *L2, int r, float s, const uint32_t *mask, float p, uint16_t *dX,
                             void *dL1, void *dL2, int grad_dtype, void *ws, size_t ws_bytes, void *stream) {
  int rc = check_linear(M, W, r);
  if (rc) return rc;
  if (!(p >= 0.f && p < 1.f)) return QLORA_ERR_INVALID_ARG;
  if (grad_dtype != QLORA_DTYPE_F32 && grad_dtype != QLORA_DTYPE_BF16) return QLORA_ERR_INVALID_ARG;
  if (!L1 || !L2 || !dL1 || !dL2) return QLORA_ERR_INVALID_ARG;
  if (M > 0 && (!dY || !X || !mask)) return QLORA_ERR_INVALID_ARG;
  if (!aligned(L1, 16) || !aligned(L2, 16) || !aligned(dL1, 16) || !aligned(dL2, 16) || (dY && !aligned(dY, 16)) ||
      (X && !aligned(X, 16)) || (dX && !aligned(dX, 16)) || (T_saved && !aligned(T_saved, 16)) ||
      (mask && !aligned(mask, 16)) || (Xm_saved && !aligned(Xm_saved, 16)))
    return QLORA_ERR_MISALIGNED;
  DeviceInfo *dev;
  rc = current_device_info(&dev);
  if (rc) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t N = W->n_out, K = W->k_in;
  const size_t gsz = grad_dtype == QLORA_DTYPE_F32 ? 4 : 2;
  if (M == 0) {
    if (cudaMemsetAsync(dL1, 0, (size_t)K * r * gsz, st) != cudaSuccess) return QLORA_ERR_CUDA;
    if (cudaMemsetAsync(dL2, 0, (size_t)r * N * gsz, st) != cudaSuccess) return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  const size_t base = bwd_dropout_base(M, N, K, r, dev->sms);
  if (!ws || ws_bytes < base + 2 * align_up((size_t)M * K * 2)) return QLORA_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return QLORA_ERR_MISALIGNED;
  uint8_t *w8 = reinterpret_cast<uint8_t *>(ws);
  uint16_t *Z = reinterpret_cast<uint16_t *>(w8 + base + align_up((size_t)M * K * 2));
  const uint16_t *Xm = Xm_saved;
  if (!Xm) {   // recompute the masked input
    uint16_t *Xw = reinterpret_cast<uint16_t *>(w8 + base);
    rc = dropout_launch(X, mask, M * K, Xw, dev, st);
    if (rc) return rc;
    Xm = Xw;
  }
  const BwdDropout drop = {Xm, 1.f / (1.f - p), mask, Z};
  const bool f32 = grad_dtype == QLORA_DTYPE_F32;
  if (rank_group_ok(r)) {   // the rank-r products as in the plain backward, on the masked input
    BwdMember m = {dY, Xm, T_saved, W, L1, L2, r, s, dX, dL1, dL2};
    m.keep = drop.keep;
    const BwdGroupLayout L = bwd_group_layout(M, &m, 1, dev->sms);
    return bwd_group_large(M, &m, 1, f32, w8, L, dev, st, &drop);
  }
  const BwdLayout L = bwd_layout(M, N, K, r, dev->sms);
  return bwd_large(dY, X, T_saved, M, W, L1, L2, r, s, dX, dL1, dL2, f32, w8, L, &drop, dev, st);
}

}  // extern "C"
