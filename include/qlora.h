/*
 * qlora.h -- C ABI of the B200 (sm_100a) QLoRA NF4 linear-layer library.
 *
 * The layer: a frozen weight W0[N, K] (out x in) stored as 4-bit NormalFloat
 * codes with one absmax scale per 64 weights, the scales themselves stored as
 * FP8-E4M3 with one FP32 second-level scale per 256 scales, plus a BF16 LoRA
 * adapter A[r, K], B[N, r] with scaling s = lora_alpha / r.
 *
 * Sources (web pages on QLoRA, cited by title and section/equation):
 *   "QLoRA: Efficient Fine-Tuning" (fermi.ai wiki): Step 1 eq. 1 (block absmax
 *     normalisation, alpha = 1), eq. 2 (NF4 levels q_i = Phi^-1((i-1/2)/16)),
 *     "snapped to the nearest NF4 quantile level"; Step 2 (double
 *     quantization, 8-bit floats, block 256); Step 3 eq. 3 (h = W0 x + B A x,
 *     W0 dequantized to BF16 at runtime; PEFT snippet: scaled by alpha / r);
 *     Step 4 eq. 5 (adapter gradients).
 *   "What is QLoRA?" (aquanode.io), "The three pieces": block of 64, scale
 *     overhead 0.127 bits/param, BF16 conversion on the fly for each matmul.
 *   "QLoRA & 4-bit Fine-Tuning" (prepfeed), Innovation 2: W ~ c1 * W_NF4, c1
 *     quantized from FP32 to FP8 with a second scale c2; follow-up 1:
 *     dequantization on the fly in every forward and backward pass.
 *
 * Conventions shared by every entry point:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller (device or
 *     unified memory).  The library allocates and frees device memory only in
 *     qlora_paged_alloc / qlora_paged_free, which a caller calls explicitly for
 *     optimizer state; its only other device state is the fixed scratch array
 *     of qlora_linear_fwd_noalloc (a static symbol).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).  Work
 *     is enqueued on it and the call returns after validating the arguments;
 *     results are ready when the stream reaches that point.
 *   - Kernels are launched as programmatic dependents (they may start while
 *     the preceding kernel of the stream finishes).  Each waits for that
 *     kernel before it completes and before it touches anything that kernel
 *     writes, so it completes only after everything before it on the stream;
 *     the first kernel of a call also waits before it touches anything at
 *     all.  A caller's kernel that follows a library call on the stream sees
 *     all of the call's results, as usual (a caller's own programmatic
 *     dependent must wait with griddepcontrol.wait before reading them).
 *   - Outputs must not overlap the call's inputs or each other.
 *   - Row-major layouts.  BF16 tensors are arrays of uint16 bit patterns.
 *   - Every check (arguments, alignment, workspace, TMA descriptor encoding)
 *     runs before the first enqueue: a call that returns INVALID_ARG,
 *     UNSUPPORTED, MISALIGNED or WORKSPACE has enqueued nothing.  CUDA means a
 *     runtime call or a kernel launch failed; launches of the same call that
 *     came before the failing one stay enqueued.
 *   - Device-side failures (a bounded wait that ran out, a non-finite weight)
 *     are recorded in the workspace's status word and read by qlora_get_error.
 *   - Not thread-safe with respect to the trace hook; otherwise re-entrant.
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

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, bad codebook */
  QLORA_ERR_UNSUPPORTED = 2,   /* blocksize != 64, dq_block != 256, shape outside v1 limits */
  QLORA_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
  QLORA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than qlora_workspace_bytes() */
  QLORA_ERR_CUDA = 5,          /* a CUDA runtime/driver call or launch failed */
  QLORA_ERR_NONFINITE = 6,     /* quantize saw an Inf/NaN weight (outputs undefined) */
  QLORA_ERR_TIMEOUT = 7        /* a kernel's bounded wait ran out; it stopped early */
} qlora_status;

typedef enum {
  QLORA_OP_QUANTIZE = 0,
  QLORA_OP_FWD = 1,
  QLORA_OP_BWD = 2
} qlora_op;

/*
 * A quantized weight (all buffers on the device, caller-owned).
 *   codes   uint8[rows*cols/2]: flat row-major order, two codes per byte, the
 *           even element in the low nibble; code j selects codebook[j].
 *   scales  uint8[rows*cols/64]: one OCP FP8-E4M3FN byte per block of 64
 *           consecutive weights of a row (needs cols % 64 == 0).
 *   c2      float[ceil(rows*cols/(64*256))]: one FP32 second-level scale per
 *           256 consecutive blocks in flat order (the last group may be short).
 *   codebook  the 16 ascending FP32 levels the codes index (by value).
 * Alignment: codes 16 bytes, scales and c2 4 bytes (else QLORA_ERR_MISALIGNED).
 * Dequantized weight: s_b = RN32(fp8(scales[b]) * c2[b/256]);
 *                     W'  = BF16_RNE(RN32(codebook[code] * s_b)).
 */
typedef struct {
  uint8_t *codes;
  uint8_t *scales;
  float *c2;
  int64_t rows;        /* N: output features */
  int64_t cols;        /* K: input features, a multiple of blocksize */
  int32_t blocksize;   /* 64 */
  int32_t dq_block;    /* 256 */
  float codebook[16];
} qlora_nf4_weight;

/* Human-readable name of a status code (static string; never NULL). */
QLORA_API const char *qlora_status_string(qlora_status st);

/* Library version string, e.g. "1.0.0 sm_100a". */
QLORA_API const char *qlora_version(void);

/*
 * The 16 NF4 levels of eq. 2 ("QLoRA: Efficient Fine-Tuning", Step 1):
 * q_i = Phi^-1((i - 1/2)/16), i = 1..16, divided by q_16 so that they span
 * [-1, 1] like eq. 1's normalised weights, rounded to FP32, ascending.
 * Host-only; writes out[0..15].  The library accepts any strictly ascending,
 * finite 16-entry table; this is the default one.
 */
QLORA_API qlora_status qlora_nf4_codebook_eq2(float out[16]);

/*
 * Bytes of each buffer of a quantized rows x cols weight ("What is QLoRA?",
 * "The three pieces": 4 bits + 8/64 + 32/(64*256) = 4.127 bits per weight).
 * Host-only.  Errors: INVALID_ARG (null output, rows/cols <= 0),
 * UNSUPPORTED (blocksize != 64, dq_block != 256, cols % 64 != 0).
 */
QLORA_API qlora_status qlora_nf4_storage_bytes(int64_t rows, int64_t cols, int32_t blocksize, int32_t dq_block,
                                     size_t *codes_bytes, size_t *scales_bytes, size_t *c2_bytes);

/*
 * Workspace bytes that `op` needs for T tokens, an N x K weight and rank r.
 * Host-only; 0 on invalid arguments.  The workspace is caller-owned device
 * memory, 256-byte aligned, that must be zeroed once (qlora_workspace_init)
 * before its first use; every call leaves its counters zero again.  Calls that
 * share a workspace must be ordered on one stream.
 */
QLORA_API size_t qlora_workspace_bytes(int32_t op, int64_t T, int64_t N, int64_t K, int32_t r);

/* Zero a workspace (one cudaMemsetAsync on `stream`). */
QLORA_API qlora_status qlora_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * Synchronize `stream`, read and clear the workspace status word.
 * Returns QLORA_OK, QLORA_ERR_NONFINITE, QLORA_ERR_TIMEOUT or QLORA_ERR_CUDA.
 */
QLORA_API qlora_status qlora_get_error(void *ws, void *stream);

/*
 * Quantize a BF16 weight w[rows, cols] to NF4 with double quantization.
 *   eq. 1 (alpha = 1): c1_b = max |w| over block b (64 consecutive weights);
 *   w_hat = RN32(w / c1_b) (IEEE fp32 division; 0 for an all-zero block);
 *   code = number of thresholds t_j <= w_hat, t_j = the smallest fp32 that is
 *     >= (codebook[j] + codebook[j+1]) / 2 -- i.e. the nearest level, ties up;
 *   double quantization (Step 2; prepfeed Innovation 2): per 256 blocks
 *     c2 = RN32(max c1 / 448), scale byte = E4M3_RNE_satfinite(RN32(c1 / c2))
 *     (0 when c2 == 0).
 * `out` supplies the three device buffers (sizes from qlora_nf4_storage_bytes);
 * the call fills out->rows/cols/blocksize/dq_block/codebook.
 * ws: at least qlora_workspace_bytes(QLORA_OP_QUANTIZE, ...) bytes (status word).
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED (w, codes not 16-byte aligned),
 * WORKSPACE, CUDA.  A non-finite weight is reported later by qlora_get_error.
 */
QLORA_API qlora_status qlora_quantize_nf4(const void *w_bf16, int64_t rows, int64_t cols, int32_t blocksize,
                                int32_t dq_block, const float codebook[16], qlora_nf4_weight *out,
                                void *ws, size_t ws_bytes, void *stream);

/*
 * qlora_quantize_nf4 with options (flags, OR-ed; 0 is qlora_quantize_nf4):
 *   QLORA_QUANT_SNAP_DQ_SCALE -- snap each block's codes against the scale it
 *     is dequantized with, s_b = RN32(fp8(f_b) * c2), instead of the exact c1:
 *     w_hat = RN32(w / s_b) (0 where s_b = 0), code = nearest level as above.
 *     The pages do not say whether the codes come from c1 or from the
 *     double-quantized scale ("QLoRA & 4-bit Fine-Tuning", Innovation 2 gives
 *     quantization, then double quantization); snapping against s_b lowers
 *     each weight's reconstruction error.  Scale bytes and c2 are unchanged.
 * Errors: as qlora_quantize_nf4; INVALID_ARG for an unknown flag.
 */
#define QLORA_QUANT_SNAP_DQ_SCALE 1u
QLORA_API qlora_status qlora_quantize_nf4_ex(const void *w_bf16, int64_t rows, int64_t cols, int32_t blocksize,
                                             int32_t dq_block, const float codebook[16], uint32_t flags,
                                             qlora_nf4_weight *out, void *ws, size_t ws_bytes, void *stream);

/*
 * Dequantize to BF16: w_out[rows, cols] = W' as defined above ("What is
 * QLoRA?": NF4 converted to BF16 on the fly; prepfeed: W ~ c1 * W_NF4).
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, CUDA.
 */
QLORA_API qlora_status qlora_dequantize(const qlora_nf4_weight *qw, void *w_bf16_out, void *stream);

/*
 * Adapter merge for export ("QLoRA: Efficient Fine-Tuning", Step 3: eq. 3's
 * two terms as one matrix):
 *   w_out[n, k] = BF16_RNE(fma(s, d, W'[n, k])),  d = sum_j B[n, j] A[j, k] in
 *   FP32 (j ascending), W' the BF16 dequantized weight.
 * A[r, K] (16-byte aligned), B[N, r] (2-byte aligned): BF16, row-major;
 * w_out[N, K]: BF16, 16-byte aligned, overwritten.  1 <= r <= 128.  The result
 * can be quantized again with qlora_quantize_nf4.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, CUDA.
 */
QLORA_API qlora_status qlora_merge_adapter(const qlora_nf4_weight *qw, const void *A, const void *B, int32_t r,
                                           float s, void *w_out, void *stream);

/*
 * Forward, eq. 3 with the PEFT scaling (Step 3):
 *   y[T, N] = x[T, K] W'^T + s (x A^T) B^T, BF16 out, FP32 accumulation,
 *   W' dequantized inside the matmul and never written to memory.
 * x[T, K], A[r, K], B[N, r], y[T, N]: BF16, row-major, 16-byte aligned.
 * Requires N % 8 == 0, 1 <= r <= 128; T == 0 is a no-op.
 * ws: at least qlora_workspace_bytes(QLORA_OP_FWD, T, N, K, r) bytes.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA.
 */
QLORA_API qlora_status qlora_linear_fwd(const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A,
                              const void *B, int32_t r, float s, void *y, void *ws, size_t ws_bytes,
                              void *stream);

/*
 * Backward (Step 4 eq. 5, and the gradient through the frozen weight):
 *   dU = s dY B;  dX = dY W' + dU A;  dB = s dY^T (x A^T);  dA = dU^T x.
 * dy[T, N], x[T, K], A[r, K], B[N, r]; outputs dx[T, K], dA[r, K], dB[N, r]
 * (BF16, overwritten, not accumulated).  Same requirements as the forward.
 * ws: at least qlora_workspace_bytes(QLORA_OP_BWD, T, N, K, r) bytes.
 * Streams: all work is ordered on `stream`.  For r <= 64, where it pays, U is
 * computed first and dU and dB then share one read of dY (as in
 * qlora_linear_bwd_saved); the launch computing dA (with dB otherwise) follows
 * the dX GEMM and runs on the SMs its last round of tiles leaves idle.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA.
 */
QLORA_API qlora_status qlora_linear_bwd(const void *dy, const void *x, int64_t T, const qlora_nf4_weight *qw,
                              const void *A, const void *B, int32_t r, float s, void *dx, void *dA,
                              void *dB, void *ws, size_t ws_bytes, void *stream);

/*
 * The LoRA activation saved for the backward ("QLoRA: Efficient Fine-Tuning",
 * Step 4 eq. 5 takes x "cached from the forward pass"; here the cached value
 * is its rank-r image U = s x A^T, which is all that dB needs of x).
 * Layout, caller-owned device memory of qlora_saved_u_bytes(T, r) bytes,
 * 16-byte aligned: two BF16 planes of sU^T [r, ceil8(T)] (row stride
 * ceil8(T)), hi = bf16(v) at offset 0 and lo = bf16(v - hi) at offset
 * qlora_saved_u_bytes(T, r) / 2, so that hi + lo carries about 16 significant
 * bits of v = s (x A^T)[t, j].  Returns 0 on invalid arguments.
 */
QLORA_API size_t qlora_saved_u_bytes(int64_t T, int32_t r);

/*
 * qlora_linear_fwd that also writes U to u_save (layout above).  Same
 * arguments, requirements and errors, plus u_save (INVALID_ARG if null when
 * T > 0, MISALIGNED if not 16-byte aligned).  At T <= 16 the rank-r product
 * then runs on the tensor-core kernel instead of the decode cluster kernel.
 */
QLORA_API qlora_status qlora_linear_fwd_save(const void *x, int64_t T, const qlora_nf4_weight *qw, const void *A,
                                             const void *B, int32_t r, float s, void *y, void *u_save, void *ws,
                                             size_t ws_bytes, void *stream);

/*
 * qlora_linear_bwd that takes U from a preceding qlora_linear_fwd_save of the
 * same x, A, s and T instead of recomputing it from x, so that x is read once
 * (for dA).  dU and dB both contract dY: for r <= 64, one kernel reads each
 * tile of dY once for both (block partial sums in the workspace, summed in a
 * fixed order by the next launch), unless those partial sums would cost more
 * than the second read of dY that they replace; otherwise dU and dB run as two
 * launches side by side.  Results equal qlora_linear_bwd's within the rounding
 * of the FP32 sums and do not depend on timing.  u_saved is read, never
 * written.  Errors: as qlora_linear_bwd; INVALID_ARG if u_saved is null when
 * T > 0, MISALIGNED if it is not 16-byte aligned.
 */
QLORA_API qlora_status qlora_linear_bwd_saved(const void *dy, const void *x, int64_t T, const qlora_nf4_weight *qw,
                                              const void *A, const void *B, int32_t r, float s, const void *u_saved,
                                              void *dx, void *dA, void *dB, void *ws, size_t ws_bytes,
                                              void *stream);

/*
 * The forward of several projections at decode-sized token counts in one pair
 * of launches (a grouped call; the pages have no counterpart: in a decoder the
 * q, k, v projections share their input, and so do gate and up).  Problem i
 * computes y_i = x_i W'_i^T + s_i (x_i A_i^T) B_i^T exactly as qlora_linear_fwd
 * would, with the arguments and requirements of that call; all share T.
 * 1 <= n <= 8; 0 <= T <= 16 (UNSUPPORTED above); at most 16384 weight-row
 * tiles of 32 over all problems (UNSUPPORTED).  ws: at least
 * qlora_decode_batch_workspace_bytes(n, probs, T) bytes, 256-byte aligned,
 * zeroed once before first use like any workspace.  The problems' outputs must
 * not overlap their inputs or each other.
 * Errors: as qlora_linear_fwd for any problem; INVALID_ARG for n or probs.
 */
typedef struct {
  const void *x;                 /* [T, K] BF16 */
  const qlora_nf4_weight *qw;    /* N x K */
  const void *A;                 /* [r, K] BF16 */
  const void *B;                 /* [N, r] BF16 */
  int32_t r;
  float s;
  void *y;                       /* [T, N] BF16, written */
} qlora_fwd_problem;
QLORA_API size_t qlora_decode_batch_workspace_bytes(int32_t n, const qlora_fwd_problem *probs, int64_t T);
QLORA_API qlora_status qlora_linear_fwd_decode_batch(int32_t n, const qlora_fwd_problem *probs, int64_t T, void *ws,
                                                     size_t ws_bytes, void *stream);

/*
 * Forward without a caller-supplied workspace/*
 * Forward without a caller-supplied workspace (no counterpart on the pages: a
 * deployment aid).  For callers that cannot allocate device memory: code that
 * runs under a host framework which owns every device allocation (a serving
 * runtime's plugin interface that hands in only input and output buffers), or
 * that must not allocate at call time.  Computes exactly what qlora_linear_fwd
 * computes; the caller still passes x, the weight, A, B and y.
 *
 * Scratch: a fixed array of QLORA_NOALLOC_SCRATCH_BYTES (4 MiB) in the
 * library's device memory, reserved on every GPU that loads the library until
 * the process exits.  The call allocates and frees nothing.  Sizes whose
 * qlora_workspace_bytes(QLORA_OP_FWD, T, N, K, r) exceeds the array are
 * rejected with QLORA_ERR_WORKSPACE (e.g. T = 4096 fits at r = 16 on a
 * 14336 x 4096 weight, but not at r = 64).
 *
 * The first call on a device looks up the array's device address on that
 * device (make it before any stream capture); the lookup is repeated after
 * the device's context was replaced (cudaDeviceReset).  Every call zeroes the
 * array's split counters on `stream`, then reuses the array; all calls share
 * the one array, so calls that may overlap on the GPU (different streams, or
 * concurrent host threads) race and must be serialized by the caller.
 * All arguments are checked before anything is enqueued (T == 0 enqueues
 * nothing).  A device-side failure (a bounded wait that ran out) is recorded
 * in the array's status word and kept there until qlora_noalloc_get_error
 * reads and clears it.
 * Errors: as qlora_linear_fwd; QLORA_ERR_WORKSPACE for sizes beyond the array.
 */
#define QLORA_NOALLOC_SCRATCH_BYTES (4u << 20)
QLORA_API qlora_status qlora_linear_fwd_noalloc(const void *x, int64_t T, const qlora_nf4_weight *qw,
                                                const void *A, const void *B, int32_t r, float s, void *y,
                                                void *stream);

/*
 * The status query of qlora_linear_fwd_noalloc on the current device:
 * synchronize `stream`, read and clear the fixed array's status word.
 * Returns QLORA_OK, QLORA_ERR_TIMEOUT or QLORA_ERR_CUDA (as qlora_get_error).
 */
QLORA_API qlora_status qlora_noalloc_get_error(void *stream);

/*
 * Failure-detection self-test (a diagnostic; the pages have no counterpart).
 * Launches one kernel whose thread waits, with the bounded mbarrier wait that
 * every pipeline of the library uses, on a barrier that nothing arrives on;
 * after limit_us microseconds the wait gives up, records the timeout in the
 * workspace's status word and the kernel returns.  qlora_get_error(ws, stream)
 * then returns QLORA_ERR_TIMEOUT.  The kernels' own waits keep their 2 s
 * limit.  limit_us in [1, 2000000]; ws: at least 256 bytes, 256-byte aligned,
 * or NULL for the fixed array of qlora_linear_fwd_noalloc on the current device
 * (then read with qlora_noalloc_get_error).
 * Errors: WORKSPACE, INVALID_ARG, CUDA.
 */
QLORA_API qlora_status qlora_wait_selftest(void *ws, size_t ws_bytes, uint32_t limit_us, void *stream);

/*
 * The adapters' optimizer step ("What is QLoRA?", "The three pieces": paged
 * optimizers; "Worked example: Llama 3.1 8B": adapters in fp32 with gradients
 * and Adam moments).  Adam (Kingma & Ba, 2015) with decoupled weight decay
 * (Loshchilov & Hutter, 2019), elementwise over n parameters:
 *   p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
 *   p <- p - lr (m / (1 - b1^step)) / (sqrt(v / (1 - b2^step)) + eps)
 * in FP32 (IEEE division and square root).  param, m, v: float[n], updated in
 * place (device or unified memory, e.g. from qlora_paged_alloc); grad_bf16:
 * BF16[n] (dA or dB of qlora_linear_bwd); param_bf16: BF16[n] output, the
 * rounded new parameters for the next forward, or NULL.  All 16-byte aligned.
 * step >= 1 counts the optimizer steps taken, this one included.
 * Errors: INVALID_ARG (null buffer, step < 1, beta outside [0, 1), eps <= 0,
 * non-finite lr or wd), MISALIGNED, CUDA.
 */
typedef struct {
  float lr;
  float beta1;          /* e.g. 0.9 */
  float beta2;          /* e.g. 0.999 */
  float eps;            /* e.g. 1e-8 */
  float weight_decay;   /* decoupled; 0 for plain Adam */
  int32_t step;
} qlora_adam_hparams;
QLORA_API qlora_status qlora_adam_step(float *param, float *m, float *v, const void *grad_bf16, void *param_bf16,
                                       int64_t n, const qlora_adam_hparams *h, void *stream);

/*
 * Unified ("paged") memory for optimizer state ("QLoRA & 4-bit Fine-Tuning",
 * Innovation 3: the state is paged out to host memory when the GPU runs short
 * and back when it is needed).  qlora_paged_alloc: cudaMallocManaged of
 * `bytes` with the current device as preferred location; *ptr is usable by
 * every kernel of this library and by the host.  qlora_paged_free releases it
 * (NULL is a no-op).  qlora_paged_prefetch moves `bytes` at ptr to the
 * current device (to_host = 0) or to host memory (to_host != 0), ordered on
 * `stream`; without it pages move on first touch.
 * Errors: INVALID_ARG (null, zero bytes), CUDA.
 */
QLORA_API qlora_status qlora_paged_alloc(size_t bytes, void **ptr);
QLORA_API qlora_status qlora_paged_free(void *ptr);
QLORA_API qlora_status qlora_paged_prefetch(void *ptr, size_t bytes, int32_t to_host, void *stream);

/*
 * Launch trace (profiling hook).  While attached, every kernel the library
 * launches records recs[i].start before and recs[i].stop after it on the
 * call's stream (cudaEvent_t handles the caller created; launches then run one
 * after another on that stream), and fills kernel id,
 * units and the algorithmic work of that launch.  *count counts the launches;
 * launches beyond `capacity` are counted but not recorded.  Pass recs = NULL
 * to detach.  Process-wide; not thread-safe.
 */
typedef struct {
  int32_t kernel;      /* qlora_kernel_name(kernel) names it */
  int32_t pad_;
  void *start;         /* cudaEvent_t, caller-created */
  void *stop;          /* cudaEvent_t, caller-created */
  double flops;        /* algorithmic FLOPs of this launch (0 if bandwidth-bound) */
  double bytes;        /* algorithmic DRAM bytes of this launch */
} qlora_trace_rec;

QLORA_API qlora_status qlora_trace_attach(qlora_trace_rec *recs, int32_t capacity, int32_t *count);
QLORA_API const char *qlora_kernel_name(int32_t kernel);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H_ */
