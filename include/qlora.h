/*
 * qlora.h -- C ABI of the B200 (sm_100a) QLoRA NF4 library (libqlora.so).
 *
 * The operations are those of "QLoRA: Efficient Finetuning of Quantized LLMs"
 * (Dettmers et al.; page aiingo.vercel.app/paper/paper-2305-14314):
 *   - blockwise absmax quantization of a frozen weight to the 4-bit NormalFloat
 *     type (§2 "Block-wise k-bit Quantization"; §3 "4-bit NormalFloat
 *     Quantization", Eq. 4; exact levels in Appendix E), block size 64;
 *   - Double Quantization of the per-block fp32 constants to 8-bit floats in
 *     blocks of 256 after subtracting their mean (§3 "Double Quantization");
 *   - doubleDequant to bfloat16 (§3 "QLoRA", Eq. 6);
 *   - the QLoRA linear layer Y = X doubleDequant(c1, c2, W) + s X L1 L2
 *     (§2 Eq. 3, §3 Eq. 5) and its backward, which produces dX through the
 *     dequantized frozen weight and gradients for the adapter L1, L2 only
 *     (§3, paragraph after Eq. 6).  There is no dW.
 *
 * Conventions shared by every entry point
 *   - Memory: every pointer argument is a DEVICE pointer owned by the caller,
 *     except where a parameter says otherwise.  The library never allocates
 *     device memory: scratch space is passed in as (ws, ws_bytes) and must be
 *     at least the size the matching *_workspace_size() function returns.
 *   - Streams: `stream` is a cudaStream_t (NULL = legacy default stream).
 *     Every call only enqueues work on that stream and never synchronizes
 *     the stream or the device (the diagnostics below say where they do);
 *     outputs are valid once the stream has reached that point.  The first
 *     call on a device reads its SM count and the address of the
 *     library's device error word, and enqueues nothing else.  (The library
 *     uses the process's shared CUDA runtime.  Under CUDA's default lazy
 *     module loading, the runtime loads each kernel at its first launch in
 *     the process and may wait for the device to do so; with
 *     CUDA_MODULE_LOADING=EAGER it loads them with the context instead.)  The kernels
 *     are launched as programmatic dependents of the kernel before them in
 *     the stream (they may start their set-up while it finishes) and wait
 *     for it before touching any memory, so the ordering is that of plain
 *     stream order.
 *   - bfloat16 data is passed as uint16_t bit patterns.
 *   - Alignment: every device pointer must be 16-byte aligned (W->c2_mean and
 *     c2_mean only need 4 bytes).
 *   - Errors: every call returns an int status (QLORA_OK = 0 or a negative
 *     QLORA_ERR_*); argument errors are detected on the host before anything
 *     is enqueued.  A kernel never traps: if a pipeline wait inside a kernel
 *     exceeds its time bound (qlora_set_wait_limit_ns) the kernel records a
 *     device error and returns, which qlora_get_last_device_error() reports.
 *     The device error word is one per device, not per stream: it holds the
 *     first failure of any stream's kernels since it was last cleared.
 *   - Shapes: W is stored as [n_out x k_in] row-major (a PyTorch Linear.weight;
 *     the paper's W in R^{h x o} transposed).  Blocks of 64 run along the
 *     row-major flattening, so with k_in % 64 == 0 every block lies inside one
 *     output row.
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define QLORA_OK 0
#define QLORA_ERR_INVALID_ARG (-1)       /* null pointer, negative size, bad dtype, bad rank */
#define QLORA_ERR_MISALIGNED (-2)        /* a pointer violates the alignment rule above */
#define QLORA_ERR_UNSUPPORTED_SHAPE (-3) /* k_in % 64, n_out % 8 or r % 8 not 0, r > 256, size limits */
#define QLORA_ERR_CUDA (-4)              /* a CUDA runtime call or launch failed */
#define QLORA_ERR_DEVICE_TIMEOUT (-5)    /* a kernel's bounded wait expired (see below) */
#define QLORA_ERR_WORKSPACE (-6)         /* ws is NULL or smaller than required */
#define QLORA_ERR_SCRATCH_LIMIT (-7)     /* too large for the fixed scratch of a no-allocation entry point */

/* ---- dtypes ---------------------------------------------------------------- */
#define QLORA_DTYPE_F32 0
#define QLORA_DTYPE_BF16 1

/* Largest LoRA rank supported by the linear entry points. */
#define QLORA_MAX_RANK 256

/*
 * A quantized weight: a view of caller-owned device buffers (not owned).
 * n = n_out * k_in elements, nblk = ceil(n / 64) blocks, n1 = ceil(nblk / 256).
 */
typedef struct {
  int64_t n_out, k_in;    /* logical shape of W: [n_out x k_in] row-major            */
  const uint8_t *codes;   /* [ceil(n/2)] NF4 codes, 2 per byte: element 2i in the low
                             nibble of byte i, element 2i+1 in the high nibble         */
  const uint8_t *c2_fp8;  /* [nblk] OCP E4M3 code of (c2_b - mean) / c1               */
  const float *c1;        /* [n1] second-level constants: absmax(c2 - mean) / 448    */
  const float *c2_mean;   /* [1] mean of the first-level constants c2                 */
  int32_t table;          /* the 16-level code table: QLORA_TABLE_NF4 (0, the default
                             of a zero-initialised struct) or QLORA_TABLE_FP4        */
} qlora_nf4dq_t;

/* 16-level code tables (code order; code 7 is the exact zero of both):
 *   QLORA_TABLE_NF4  the NF4 levels of Appendix E;
 *   QLORA_TABLE_FP4  FP4 (E2M1), the 4-bit float of §4 (Tables 2-4) that NF4
 *                    is compared against: {0, 0.5, 1, 1.5, 2, 3, 4, 6} and
 *                    their negatives divided by 6 (float32 quotients), with
 *                    both zero codes holding +0.  Blocking, Double
 *                    Quantization and doubleDequant are the same for both. */
#define QLORA_TABLE_NF4 0
#define QLORA_TABLE_FP4 1

/* ---- quantizer -------------------------------------------------------------- */

/* Scratch bytes qlora_quantize_nf4_dq needs for a tensor of `numel` elements. */
QLORA_API size_t qlora_quantize_workspace_size(int64_t numel);

/*
 * NF4 + Double Quantization of a frozen weight (§2 blockwise quantization,
 * §3 NF4 and Double Quantization, Appendix E levels).
 *   W        [n_out x k_in] fp32 or bf16 (w_dtype), finite values.
 *   For each 64-block b of the row-major flattening: c2_b = max |w|;
 *   code = nearest NF4 level to fp32(w / c2_b) (IEEE division; exact ties go to
 *   the lower level; an all-zero block gets the exact-zero code 7); codes are
 *   packed two per byte (see qlora_nf4dq_t).
 *   Then mean = fp32(sum c2 / nblk) (deterministic fp64 sum) and for each
 *   256-block beta of c2: d = fp32(c2 - mean), c1_beta = fp32(max|d| / 448),
 *   c2_fp8 = E4M3 round-to-nearest-even, saturating, of fp32(d / c1_beta)
 *   (code 0 when c1_beta == 0).
 *   Outputs: codes [ceil(n/2)], c2_fp8 [nblk], c1 [n1], c2_mean [1].
 *   Any n_out, k_in >= 0 (a final partial block uses only its real elements).
 */
/* The same quantizer with the code table chosen by `table` (QLORA_TABLE_*);
 * qlora_quantize_nf4_dq is table QLORA_TABLE_NF4.  Returns
 * QLORA_ERR_INVALID_ARG for an unknown table. */
QLORA_API int qlora_quantize_4bit_dq(const void *W, int w_dtype, int64_t n_out, int64_t k_in, int table,
                                     uint8_t *codes, uint8_t *c2_fp8, float *c1, float *c2_mean, void *ws,
                                     size_t ws_bytes, void *stream);
QLORA_API int qlora_quantize_nf4_dq(const void *W, int w_dtype, int64_t n_out, int64_t k_in, uint8_t *codes,
                          uint8_t *c2_fp8, float *c1, float *c2_mean, void *ws, size_t ws_bytes, void *stream);

/*
 * qlora_quantize_nf4_dq without a workspace argument.  The paper has no
 * counterpart: this is a convenience of the library.
 *
 * Who needs it: callers that cannot allocate device memory at the point where
 * they quantize -- for example code that runs under a framework which owns all
 * device memory through its own pool (allocating behind its back breaks its
 * accounting and limits), or latency-critical code that must not pay for
 * cudaMalloc's implicit device-wide synchronization.  Such callers pass only
 * the inputs and outputs.
 *
 * Scratch: the fp32 block constants and the fp64 partial sums live in one
 * static device array inside the library, QLORA_NOALLOC_SCRATCH_BYTES long.
 * Every GPU on which the library is loaded holds that array until the process
 * exits.  Limit: n_out * k_in <= QLORA_NOALLOC_MAX_NUMEL (2^28 weights, e.g. a
 * 16384 x 16384 matrix); larger tensors return QLORA_ERR_SCRATCH_LIMIT before
 * anything is enqueued.  This entry point never allocates or frees device
 * memory.
 *
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture.  Concurrency: all calls share the one array and it keeps
 * the last call's contents, so calls that may overlap on the GPU (different
 * streams without ordering) race and must be serialized by the caller.  Every
 * scratch entry a call reads is first written by the same call.
 * Outputs, rules and results are identical to qlora_quantize_nf4_dq.
 */
#define QLORA_NOALLOC_MAX_NUMEL ((int64_t)1 << 28)
#define QLORA_NOALLOC_SCRATCH_BYTES (((size_t)1 << 24) + 16384)
QLORA_API int qlora_quantize_nf4_dq_noalloc(const void *W, int w_dtype, int64_t n_out, int64_t k_in, uint8_t *codes,
                                            uint8_t *c2_fp8, float *c1, float *c2_mean, void *stream);

/*
 * doubleDequant (§3 Eq. 6) of the whole weight to bf16:
 *   c2_hat = fma_fp32(E4M3(c2_fp8_b), c1_beta, mean)  (one rounding),
 *   W_out  = bf16_rne(fp32(NF4[code] * c2_hat)).
 *   W_out  [n_out x k_in] bf16, row-major.  No workspace.
 */
QLORA_API int qlora_dequant(const qlora_nf4dq_t *W, uint16_t *W_out, void *stream);

/* ---- QLoRA linear ------------------------------------------------------------ */

/* Scratch bytes for qlora_linear_fwd / qlora_linear_bwd at these sizes. */
QLORA_API size_t qlora_linear_fwd_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r);
QLORA_API size_t qlora_linear_bwd_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r);

/*
 * Forward (§2 Eq. 3 / §3 Eq. 5 with the scale s of Eq. 3):
 *   Y = X doubleDequant(W)^T + T L2,  T = s X L1.
 *   X [M x K] bf16, L1 [K x r] bf16, L2 [r x N] bf16, Y [M x N] bf16 (out).
 *   T_save [M x 2r] bf16 (out, may be NULL): the adapter down-projection
 *   T = s X L1 (fp32 accumulation) kept for the backward as a pair of bf16
 *   halves, T ~= T_save[:, :r] + T_save[:, r:] (hi = bf16(T),
 *   lo = bf16(T - hi); relative error about 2^-17).  The forward's up-projection
 *   uses the hi half; the backward's dL2 = T^T dY uses both, so that the long
 *   reduction over tokens does not amplify a bf16 rounding of T.
 *   K = W->k_in (multiple of 64), N = W->n_out (multiple of 8), r a multiple of
 *   8 in [8, 256].  All products accumulate in fp32 on the tensor cores.
 *   Reproducibility: above 128 tokens every reduction is summed in a fixed
 *   order, so equal inputs give equal bits run to run.  At 1-128 tokens the
 *   partial sums of Y and T over K are added with fp32 atomics (red.add), so
 *   Y and T may differ in their last bits between runs (always within the
 *   stated tolerance); the decoded weight itself is exact.
 */
QLORA_API int qlora_linear_fwd(const uint16_t *X, int64_t M, const qlora_nf4dq_t *W, const uint16_t *L1, const uint16_t *L2,
                     int r, float s, uint16_t *Y, uint16_t *T_save, void *ws, size_t ws_bytes, void *stream);

/*
 * Backward (§3, paragraph after Eq. 6: adapter gradients only, the gradient
 * passing through the weight dequantized to bf16):
 *   G   = s dY L2^T                  [M x r] (internal, bf16 hi/lo pair)
 *   dX  = dY doubleDequant(W) + G L1^T   [M x K] bf16 (out; may be NULL to skip)
 *   dL2 = T^T dY                     [r x N] (out)
 *   dL1 = X^T G                      [K x r] (out)
 *   T_saved [M x 2r] bf16 (hi/lo pair) from the forward, or NULL to recompute.
 *   dL1, dL2 are written (not accumulated) as grad_dtype (QLORA_DTYPE_BF16 or
 *   QLORA_DTYPE_F32).  Shape rules as for the forward.
 */
QLORA_API int qlora_linear_bwd(const uint16_t *dY, const uint16_t *X, const uint16_t *T_saved, int64_t M,
                     const qlora_nf4dq_t *W, const uint16_t *L1, const uint16_t *L2, int r, float s, uint16_t *dX,
                     void *dL1, void *dL2, int grad_dtype, void *ws, size_t ws_bytes, void *stream);

/*
 * Grouped forward: the forward of up to QLORA_MAX_GROUP linears that see the
 * same M tokens, each computing what qlora_linear_fwd computes (§2 Eq. 3 / §3
 * Eq. 5) up to the order of its fp32 additions, e.g. the q, k, v, gate and up
 * projections of a decoder layer, which all read the layer's normalised
 * input.
 *   members[count]: a HOST array; member i names its own X [M x K_i], weight
 *   W_i (host pointer to the view), L1 [K_i x r_i], L2 [r_i x N_i], scale s_i,
 *   output Y [M x N_i] and optional T_save [M x 2 r_i] (layouts, shape and
 *   alignment rules of qlora_linear_fwd).  Members may share X (read only);
 *   no output may overlap another member's input or output.
 *   With M <= 128 the whole group runs as one chain of three kernels (T
 *   accumulation, fused doubleDequant + product, LoRA epilogue) over the
 *   concatenated work of all members, instead of one chain per linear: the
 *   per-linear launch gaps and tails of the few-token path disappear.
 *   Members of different code tables (W->table) run as one chain per table.
 *   With M > 128, the adapter down-projections T_i = s_i X L1_i of members
 *   that read the same X (same pointer and K) run as one launch of the
 *   grouped rank-r kernel (ranks up to 128; a set holding a larger rank runs
 *   each member's own forward); with equal ranks of 64 or 128 their L1 are first
 *   copied side by side, X [L1_a | L1_b | ...], so that each strip of X is
 *   read for all of them together.  Every member's T is written as its hi/lo
 *   pair; then every member runs its own doubleDequant and tensor-core
 *   product, in order.
 *   LoRA dropout is not part of the grouped forward (qlora_linear_fwd_dropout
 *   runs it per linear).  count = 0 or M = 0: nothing is done.  Workspace:
 *   qlora_linear_fwd_group_workspace_size(), which returns 0 for invalid
 *   arguments.
 * Errors: those of qlora_linear_fwd for any member, and QLORA_ERR_INVALID_ARG
 * for count outside [0, QLORA_MAX_GROUP] or a NULL members array.
 */
#define QLORA_MAX_GROUP 8

typedef struct {
  const uint16_t *X;          /* [M x W->k_in] bf16 */
  const qlora_nf4dq_t *W;     /* host pointer to the weight view */
  const uint16_t *L1;         /* [k_in x r] bf16 */
  const uint16_t *L2;         /* [r x n_out] bf16 */
  int32_t r;
  float s;
  uint16_t *Y;                /* [M x n_out] bf16, written */
  uint16_t *T_save;           /* [M x 2r] bf16 hi/lo pair, written; or NULL */
} qlora_fwd_member_t;

QLORA_API size_t qlora_linear_fwd_group_workspace_size(const qlora_fwd_member_t *members, int count, int64_t M);
QLORA_API int qlora_linear_fwd_group(const qlora_fwd_member_t *members, int count, int64_t M, void *ws,
                                     size_t ws_bytes, void *stream);

/*
 * Grouped backward: the backward of up to QLORA_MAX_GROUP linears whose output
 * gradients are available together (a layer's q, k and v after the attention
 * backward; gate and up after the SwiGLU backward), each computing exactly
 * what qlora_linear_bwd computes (same formulas, layouts and shape rules, all
 * members on the same M tokens).  For members with r in {8, 16, 32, 64}:
 *   - G and dL2 of all of them run as one launch of the grouped rank-r
 *     kernel, dL1 as a second one, where members that read the same X (same
 *     pointer, k_in and r) share one pass over X;
 *   - then each member's doubleDequant and dX = dY W_hat + G_hi L1^T.
 * Members with other ranks run the single-linear backward one after another.
 * Split reductions are summed in a fixed order: results are reproducible run
 * to run, but may differ in the last bits from a call on a different group
 * (a different split of the same reduction).
 * Outputs of different members must not overlap each other or any input.
 * Workspace: qlora_linear_bwd_group_workspace_size() bytes (the same members
 * and M; independent of which T_saved are NULL), 256-byte aligned.
 * Errors: as qlora_linear_bwd, for the first failing member; QLORA_ERR_INVALID_ARG
 * for count outside [0, QLORA_MAX_GROUP] or a NULL member array with count > 0.
 */
typedef struct {
  const uint16_t *dY;         /* [M x n_out] bf16 */
  const uint16_t *X;          /* [M x k_in] bf16 */
  const uint16_t *T_saved;    /* [M x 2r] bf16 hi/lo pair from the forward, or NULL to recompute */
  const qlora_nf4dq_t *W;
  const uint16_t *L1;         /* [k_in x r] bf16 */
  const uint16_t *L2;         /* [r x n_out] bf16 */
  int r;
  float s;
  uint16_t *dX;               /* [M x k_in] bf16, written; or NULL to skip */
  void *dL1;                  /* [k_in x r], grad_dtype, written */
  void *dL2;                  /* [r x n_out], grad_dtype, written */
} qlora_bwd_member_t;

QLORA_API size_t qlora_linear_bwd_group_workspace_size(const qlora_bwd_member_t *members, int count, int64_t M);
QLORA_API int qlora_linear_bwd_group(const qlora_bwd_member_t *members, int count, int64_t M, int grad_dtype,
                                     void *ws, size_t ws_bytes, void *stream);

/*
 * LoRA dropout (QLoRA Appendix B.2 trains with LoRA dropout, p = 0.1 up to
 * 13B and 0.05 at 33B and 65B).  It acts on the adapter's input only:
 *   Y  = X W_hat^T + T L2,   T = s drop(X) L1,   drop(X) = X * m / (1 - p);
 *   dX = dY W_hat + (G L1^T) * m / (1 - p),  G = s dY L2^T;
 *   dL2 = T^T dY,  dL1 = drop(X)^T G.
 * The keep mask m is an input: uint32 words over the row-major [M x K]
 * elements of X, bit b of word w keeping element 32 w + b (so [M x K/32]
 * words, 16-byte aligned; the same mask must be passed to the forward and
 * the backward of a step).  0 <= p < 1; p = 0 with an all-ones mask computes
 * the plain linear.  Xm_save [M x K] bf16 (out, may be NULL) receives the
 * masked input X * m; passing it back as Xm_saved spares the backward its
 * recomputation (NULL: recomputed from X and the mask).  Other arguments,
 * layouts and T_save are those of qlora_linear_fwd / qlora_linear_bwd.  Every
 * token count takes the dequant + tensor-core path.  Workspace:
 * *_dropout_workspace_size().
 * Errors: as qlora_linear_fwd / _bwd, plus QLORA_ERR_INVALID_ARG for a NULL
 * mask (M > 0) or p outside [0, 1).
 */
QLORA_API size_t qlora_linear_fwd_dropout_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r);
QLORA_API size_t qlora_linear_bwd_dropout_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r);
QLORA_API int qlora_linear_fwd_dropout(const uint16_t *X, int64_t M, const qlora_nf4dq_t *W, const uint16_t *L1,
                                       const uint16_t *L2, int r, float s, const uint32_t *mask, float p,
                                       uint16_t *Y, uint16_t *T_save, uint16_t *Xm_save, void *ws, size_t ws_bytes,
                                       void *stream);
QLORA_API int qlora_linear_bwd_dropout(const uint16_t *dY, const uint16_t *X, const uint16_t *T_saved,
                                       const uint16_t *Xm_saved, int64_t M, const qlora_nf4dq_t *W,
                                       const uint16_t *L1, const uint16_t *L2, int r, float s, const uint32_t *mask,
                                       float p, uint16_t *dX, void *dL1, void *dL2, int grad_dtype, void *ws,
                                       size_t ws_bytes, void *stream);

/* ---- diagnostics ----------------------------------------------------------------- */

/* Static description of a status code. */
QLORA_API const char *qlora_status_str(int status);

/*
 * Bound on every wait inside the library's kernels (a pipeline stage waiting
 * for its data, a producer waiting for a free stage), for the current device.
 * A wait that runs longer records QLORA_ERR_DEVICE_TIMEOUT in the device
 * error word and the kernel returns without finishing its work (no trap, no
 * copy or MMA left in flight).  The default is QLORA_DEFAULT_WAIT_LIMIT_NS
 * (4 s), far above any legitimate wait.  The new limit is set by a one-thread
 * kernel enqueued on `stream` and applies to kernels that start after it.
 * ns = 0 restores the default; ns > QLORA_MAX_WAIT_LIMIT_NS (60 s) returns
 * QLORA_ERR_INVALID_ARG.
 */
#define QLORA_DEFAULT_WAIT_LIMIT_NS 4000000000ull
#define QLORA_MAX_WAIT_LIMIT_NS 60000000000ull
QLORA_API int qlora_set_wait_limit_ns(uint64_t ns, void *stream);

/*
 * Diagnostics of the failure path: enqueues on `stream` one thread that
 * waits, through the same bounded wait as every pipeline of the library, on
 * a barrier that nothing completes.  The wait runs out after the device's
 * wait limit; the kernel then records a device timeout and returns, so that
 * the next qlora_get_last_device_error() returns QLORA_ERR_DEVICE_TIMEOUT.
 * It touches no caller memory.  Meant for tests of error handling, with a
 * short limit set first.
 */
QLORA_API int qlora_diag_expired_wait(void *stream);

/*
 * Synchronizes `stream`, then returns and clears the device error word of the
 * current device: QLORA_OK, or QLORA_ERR_DEVICE_TIMEOUT if a kernel gave up a
 * bounded wait since the last call (the kernel's outputs are then invalid),
 * or QLORA_ERR_CUDA if the synchronization itself failed.
 */
QLORA_API int qlora_get_last_device_error(void *stream);

/*
 * Kernel timing log (diagnostics).  qlora_profile_start(capacity) enables it
 * for the current device: each subsequent kernel launch of this library is
 * bracketed by two CUDA events recorded on the launch's stream, for the first
 * `capacity` launches (later ones are not logged).  qlora_profile_stop()
 * disables it and returns the number of logged launches.  qlora_profile_read(i)
 * then returns launch i's kernel kind (QLORA_KERNEL_*) and its elapsed
 * milliseconds (waiting for its end event).  The log's events are host-side
 * CUDA objects created by start(); no device memory is allocated.
 */
#define QLORA_KERNEL_QUANTIZE 1
#define QLORA_KERNEL_DQ_CONSTANTS 2
#define QLORA_KERNEL_DEQUANT 3
#define QLORA_KERNEL_GEMM_T 10      /* T = s X L1 */
#define QLORA_KERNEL_GEMM_Y 11      /* Y = X W_hat^T + T L2 */
#define QLORA_KERNEL_GEMM_G 12      /* G = s dY L2^T */
#define QLORA_KERNEL_GEMM_DX 13     /* dX = dY W_hat + G L1^T */
#define QLORA_KERNEL_GEMM_DL2 14    /* dL2 = T^T dY */
#define QLORA_KERNEL_GEMM_DL1 15    /* dL1 = X^T G */
#define QLORA_KERNEL_GEMM_Z 16      /* Z = G L1^T (dropout backward) */
#define QLORA_KERNEL_RANK_G_DL2 17  /* G = s dY L2^T and dL2 = T^T dY of every linear of a backward, one launch */
#define QLORA_KERNEL_RANK_DL1 18    /* dL1 = X^T G of every linear of a backward, one launch */
#define QLORA_KERNEL_SPLITK_FINALIZE 20
#define QLORA_KERNEL_FUSED_FWD 31   /* few-token forward chain (up to 128 tokens): T, fused decode + tcgen05 product, LoRA epilogue */
#define QLORA_KERNEL_DROPOUT_MASK 40 /* Xm = X * m (LoRA dropout) */
QLORA_API int qlora_profile_start(int capacity);
QLORA_API int qlora_profile_stop(void);
QLORA_API int qlora_profile_read(int i, int *kind, float *ms);

/* Library version (major * 10000 + minor * 100 + patch). */
QLORA_API int qlora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H_ */
