/*
 * qlora_nf4.h — C ABI of the B200 (sm_100a) QLoRA frozen-NF4 linear layer.
 *
 * The method (web pages on QLoRA; main source "QLoRA: Efficient Finetuning of
 * Quantized LLMs", intuitivepapers.ai):
 *   - §NormalFloat: a 16-level NormalFloat-4 code book (7 negative levels, an
 *     exact zero, 8 positive levels, ends at -1 and +1);
 *   - §Quantize in blocks: the flattened weight is cut into blocks of 64
 *     consecutive elements, each with its own absmax constant;
 *   - §Double quantization: the block constants, mean-centred, are stored as
 *     8-bit floats in groups of 256 with one float32 scale per group;
 *   - §The QLoRA layer, end to end: Y = X·W + s·(X·L1)·L2 with W dequantised
 *     to bfloat16 on the fly; backward gives dX through W and the adapter,
 *     and gradients for L1, L2 only.
 * Around the layer: the optimiser step of the adapters (qlora_adamw_step),
 * merging a trained adapter into the quantised base and requantising
 * (qlora_merge_requantize), and the storage-format variants the pages compare
 * NF4 with (qlora_quantize_format and its companions).
 *
 * Conventions of this library:
 *   W  [N, K]  frozen weight, bfloat16, row-major (out x in, as a framework
 *              Linear stores it); quantisation blocks run along the flat
 *              row-major index, so K must be a multiple of 64.
 *   X  [M, K]  activations, bfloat16 row-major.  M >= 1 tokens.
 *   A  [K, r]  first adapter factor (the pages' L1), bfloat16 row-major.
 *   B  [r, N]  second adapter factor (L2), bfloat16 row-major.
 *   s          adapter scale alpha / r.
 *   Y  [M, N] = X·W_hatᵀ + s·(X·A)·B, bfloat16 (float32 accumulation).
 *   W_hat = doubleDequant(W_NF4), bfloat16, never written to HBM by the
 *   forward or backward pass.
 *
 * Stored NF4 weight (all buffers on the device, owned by the caller):
 *   codes  N·K/2 bytes: element 2j of the flat weight in the HIGH nibble of
 *          byte j, element 2j+1 in the LOW nibble; 16-byte aligned.
 *   c2q    N·K/64 bytes: OCP FP8 E4M3FN code e_b of each block's centred
 *          absmax (block b = flat elements [64b, 64b+64)).
 *   c1     ceil(N·K/64/256) float32: group scale S_g (group g = blocks
 *          [256g, 256g+256) of the flat block index; may straddle rows; the
 *          last group may be partial).
 *   mean   1 float32: mu, the mean of all block absmax values.
 *   Reconstruction: c2_hat_b = fmaf(e_b, S_g, mu);
 *                   w_hat = bf16_rn(float32(level[code] · c2_hat_b)).
 *
 * bfloat16 tensors are passed as uint16_t bit patterns.  All sizes are in
 * elements unless stated.  Every device pointer must be 16-byte aligned unless
 * its entry point says otherwise.
 * `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 * asynchronous on `stream`, never synchronises and never allocates.
 *
 * Errors: the return value reports host-side validation and launch errors;
 * nothing is launched when validation fails.  Conditions detected on the
 * device are OR-ed into *dev_err (a device int, nullable) as QLORA_DEVERR_*
 * bits; read it after synchronising the stream.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,       /* null pointer, non-positive size, bad op */
  QLORA_ERR_UNSUPPORTED_SHAPE = 2, /* K % 64 != 0, r not in {8,16,...,256}, N % 8 != 0, overflow */
  QLORA_ERR_MISALIGNED = 3,        /* a device pointer is not 16-byte aligned */
  QLORA_ERR_CUDA = 4,              /* a CUDA runtime / driver call failed */
  QLORA_ERR_WORKSPACE = 5,         /* workspace missing or smaller than qlora_workspace_size() */
  QLORA_ERR_NO_DEVICE = 6,         /* the current device is not sm_100 */
  QLORA_ERR_TOO_LARGE = 7          /* shape exceeds qlora_quantize_noalloc's static scratch (N*K <= 2^26) */
} qlora_status;

/* Bits OR-ed into *dev_err by kernels. */
#define QLORA_DEVERR_NONFINITE 1   /* a weight to quantise (given, or merged) held Inf/NaN */
#define QLORA_DEVERR_TIMEOUT   2   /* a pipeline wait exceeded its bound; outputs are undefined */

typedef struct qlora_nf4_weight {
  int64_t N, K;      /* logical shape of W */
  uint8_t *codes;    /* N*K/2 bytes   */
  uint8_t *c2q;      /* N*K/64 bytes  */
  float *c1;         /* ceil(N*K/16384) floats */
  float *mean;       /* 1 float       */
} qlora_nf4_weight;

enum { QLORA_OP_QUANTIZE = 0, QLORA_OP_FORWARD = 1, QLORA_OP_BACKWARD = 2, QLORA_OP_MERGE = 3 };

/* Human-readable name of a status code (static string). */
const char *qlora_status_string(qlora_status st);

/*
 * Diagnostic with no counterpart on the pages: the CUDA runtime's message
 * (static string) for the last CUDA failure that made a call on this host
 * thread return QLORA_ERR_CUDA, or "no error"; *code (nullable) receives its
 * cudaError_t value (0 when none).
 */
const char *qlora_last_cuda_error(int *code);

/*
 * qlora_build_codebook — host only.  §NormalFloat (intuitivepapers.ai): the
 * offset recipe (tail probability 0.9677083; 8 positive normal quantiles at
 * probabilities evenly spaced from the offset towards 1/2, 7 negative ones
 * likewise, an exact 0; sorted; divided by the largest magnitude).  Quantiles
 * come from Wichura's AS 241 (1988) refined by one Newton step on erfc, in
 * float64, then rounded to float32.
 * levels[16]    : ascending, levels[0] = -1, levels[7] = 0, levels[15] = +1.
 * thresholds[15]: thresholds[i] = smallest float32 strictly above the exact
 *                 midpoint (levels[i]+levels[i+1])/2, so that
 *                 code(x) = #{i : x >= thresholds[i]} is the nearest level with
 *                 ties going to the lower index.
 * Either pointer may be NULL.  Returns QLORA_OK.
 */
qlora_status qlora_build_codebook(float levels[16], float thresholds[15]);

/* Byte sizes of the three stored arrays of an N x K weight (mean is 4 bytes). */
qlora_status qlora_nf4_sizes(int64_t N, int64_t K, size_t *codes_bytes, size_t *c2q_bytes,
                             size_t *c1_bytes);

/*
 * Workspace bytes an operation needs (op = QLORA_OP_*; M and r are ignored for
 * QLORA_OP_QUANTIZE and QLORA_OP_MERGE).  The caller allocates it (16-byte aligned) and passes it
 * to the call; it holds no state between calls.
 */
qlora_status qlora_workspace_size(int op, int64_t M, int64_t N, int64_t K, int r, size_t *bytes);

/*
 * qlora_quantize — §Quantize in blocks, §NormalFloat, §Double quantization.
 * W: device, N*K bfloat16 (the shape comes from out->N, out->K).
 * Per block: c2 = max|w| (float32); x = float32(w / c2); code = nearest level
 * (ties to the lower index; an all-zero block gives the zero level, 7).
 * Second level: mu = mean of all c2 in a fixed order (per group of 256 blocks
 * a float64 pairwise tree — h = 128, 64, ..., 1: a[i] += a[i+h] — then the same
 * tree over the group sums zero-padded to a power of two; float64 divide by
 * the block count, rounded to float32); dev = float32(c2 - mu);
 * S_g = float32(max|dev| over the group / 448); e = E4M3(dev / S_g) with
 * round-to-nearest-even and saturation (S_g = 0 gives e = 0).
 * Writes out->codes, out->c2q, out->c1, out->mean.  A non-finite weight sets
 * QLORA_DEVERR_NONFINITE in *dev_err (outputs then unspecified).
 * Deterministic: identical inputs give identical bits.
 */
qlora_status qlora_quantize(const uint16_t *W, const qlora_nf4_weight *out, void *ws,
                            size_t ws_bytes, int *dev_err, void *stream);

/*
 * qlora_quantize_noalloc — the same quantiser (identical output bits to
 * qlora_quantize) for callers that cannot allocate device memory: a plugin or
 * custom-op interface that passes buffers but no allocator, or a runtime whose
 * memory plan forbids new allocations while it runs.  No counterpart on the
 * pages: it only changes where the scratch lives.  Instead of a caller-provided
 * workspace it uses a static device array built into the library (about 4 MiB,
 * held by every GPU that loads the library until the process exits), so it
 * calls no cudaMalloc, cudaFree or allocating routine.
 * Limit: N*K <= 2^26 (e.g. 8192 x 8192); larger weights return
 * QLORA_ERR_TOO_LARGE and launch nothing.
 * Each call looks up the array's device address on the current device; a call
 * on a stream that is being captured uses the address remembered from an
 * earlier call on that device instead (and fails with QLORA_ERR_CUDA if there
 * was none), so make the first call on each device before any stream capture.
 * The lookup on every other call keeps the address right after cudaDeviceReset
 * or a new primary context, which reload the library's module elsewhere.
 * All calls share the array: calls that overlap on the GPU (different
 * streams or host threads) race and give undefined results; calls ordered on
 * one stream are safe.  The array keeps the last call's contents; nothing in it
 * needs clearing between calls.
 * W, out, dev_err, stream: as for qlora_quantize.
 */
qlora_status qlora_quantize_noalloc(const uint16_t *W, const qlora_nf4_weight *out, int *dev_err, void *stream);

/*
 * qlora_dequantize — doubleDequant of §The QLoRA layer, end to end, written
 * out to HBM (for tests and inspection; the layer itself never does this).
 * W_out: device, N*K bfloat16.
 */
qlora_status qlora_dequantize(const qlora_nf4_weight *w, uint16_t *W_out, void *stream);

/*
 * qlora_merge_requantize — merge a trained adapter into the quantised base and
 * requantise ("QLoRA: quantising the part you are not training", addaly.com,
 * §What it costs: merging into the quantised base means requantising).  The
 * layer computes X·Ŵᵀ + s·(X·A)·B (§The QLoRA layer, end to end,
 * intuitivepapers.ai), so the merged weight is
 *   W_eff[n][k] = bf16_rn( float32( ŵ[n][k] + s · sum_j A[k][j]·B[j][n] ) )
 * with ŵ = doubleDequant(w), the sum accumulated in float32 on the tensor
 * cores (order unspecified), and one float32 rounding of ŵ + s·sum (a fused
 * multiply-add).  W_eff is then quantised exactly as qlora_quantize does.
 * w   : the stored weight (device buffers), N x K.
 * A   : device, K x r bfloat16 row-major; B: device, r x N bfloat16 row-major
 *       (the layer's adapter); r % 8 == 0, r <= 256; N % 8 == 0.
 * s   : the adapter scale alpha / r.
 * out : the new stored weight, same N, K.  It may be w itself (in place);
 *       otherwise none of its buffers may overlap any of w's.
 * W_merged : device N x K bfloat16 (nullable): receives W_eff; must not
 *       overlap w or out.
 * ws  : qlora_workspace_size(QLORA_OP_MERGE, 0, N, K, r) bytes (the
 *       quantiser's workspace).
 * A non-finite merged weight sets QLORA_DEVERR_NONFINITE in *dev_err; a
 * pipeline wait that runs out sets QLORA_DEVERR_TIMEOUT (outputs then
 * unspecified).  Errors: QLORA_ERR_INVALID_ARG (null pointer, shape mismatch,
 * partial overlap of out and w), QLORA_ERR_UNSUPPORTED_SHAPE, QLORA_ERR_MISALIGNED,
 * QLORA_ERR_WORKSPACE, QLORA_ERR_NO_DEVICE, QLORA_ERR_CUDA.
 */
qlora_status qlora_merge_requantize(const qlora_nf4_weight *w, const uint16_t *A, const uint16_t *B, int r,
                                    float s, const qlora_nf4_weight *out, uint16_t *W_merged, void *ws,
                                    size_t ws_bytes, int *dev_err, void *stream);

/*
 * qlora_linear_forward — §LoRA and §The QLoRA layer, end to end (forward).
 *   T_save (nullable, device, M x r bfloat16) receives bf16(s · X·A), the
 *   scaled adapter activation the backward pass reuses.
 *   Y (device, M x N bfloat16) = X·W_hatᵀ + (bf16(s·X·A))·B, float32 accumulate.
 * W_hat is produced tile by tile inside the GEMM (tensor cores, tcgen05) and
 * never stored.  ws: qlora_workspace_size(QLORA_OP_FORWARD, ...) bytes.
 */
qlora_status qlora_linear_forward(const qlora_nf4_weight *w, const uint16_t *X, int64_t M,
                                  const uint16_t *A, const uint16_t *B, int r, float s,
                                  uint16_t *Y, uint16_t *T_save, void *ws, size_t ws_bytes,
                                  int *dev_err, void *stream);

/*
 * qlora_linear_backward — §The QLoRA layer, end to end (backward).
 *   U  = dY·Bᵀ                                   (M x r)
 *   dX = dY·W_hat + bf16(s·U)·Aᵀ                 (M x K bfloat16; nullable = skip)
 *   dA = Xᵀ·bf16(s·U)                            (K x r float32)
 *   dB = T_savedᵀ·dY                             (r x N float32)
 * T_saved is the forward's T_save = bf16(s·X·A); NULL recomputes it from X and A.
 * No gradient for W is formed.  ws: qlora_workspace_size(QLORA_OP_BACKWARD, ...).
 */
qlora_status qlora_linear_backward(const qlora_nf4_weight *w, const uint16_t *X,
                                   const uint16_t *dY, int64_t M, const uint16_t *A,
                                   const uint16_t *B, int r, float s, const uint16_t *T_saved,
                                   uint16_t *dX, float *dA, float *dB, void *ws, size_t ws_bytes,
                                   int *dev_err, void *stream);

/* ---------------------------------------------------------------- diagnostics
 * (no counterpart on the pages: instrumentation for measurement)            */

/*
 * One AdamW step on the trained adapter factors, all tensors in one launch.
 * "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai), §Where
 * finetuning memory goes: Adam keeps a running mean and variance of each
 * trained weight's gradients in 32-bit floats; §The QLoRA layer, end to end:
 * only the adapters (L1 = A, L2 = B) carry gradients and optimiser state.  The
 * update is AdamW (Loshchilov and Hutter, decoupled weight decay) in PyTorch's
 * arrangement, per element at step t >= 1:
 *   p <- p·(1 - lr·wd);  m <- m + (1 - b1)·(g - m);  v <- b2·v + (1 - b2)·g²;
 *   p <- p - lr/(1 - b1^t) · m / (sqrt(v)/sqrt(1 - b2^t) + eps)
 * in float32.  Parameters are kept as float32 master values; when param_bf16
 * is set, the bfloat16 copy the linear layer reads (round to nearest even) is
 * written after the update.  All pointers are device pointers, 16-byte
 * aligned; m and v must be zero before step 1; tensors must not overlap.
 * Errors: QLORA_ERR_INVALID_ARG for null pointers, count outside
 * 1..QLORA_ADAMW_MAX_TENSORS, n < 1, step < 1, lr < 0, wd < 0, beta outside
 * [0, 1) or eps <= 0; QLORA_ERR_MISALIGNED for unaligned pointers.
 */
#define QLORA_ADAMW_MAX_TENSORS 16
typedef struct {
  float *param;         /* float32 master values, updated in place */
  uint16_t *param_bf16; /* nullable: bfloat16 copy written after the update */
  const float *grad;    /* float32 gradient, e.g. dA or dB of qlora_linear_backward */
  float *m;             /* first moment, float32, updated in place */
  float *v;             /* second moment, float32, updated in place */
  int64_t n;            /* elements */
} qlora_adamw_tensor;

qlora_status qlora_adamw_step(const qlora_adamw_tensor *tensors, int count, float lr, float beta1, float beta2,
                              float eps, float weight_decay, int64_t step, void *stream);

/*
 * Diagnostic with no counterpart on the pages: exercises on the device the
 * error path that every pipeline wait of this library takes when its bound
 * runs out.  Launches one CTA that waits, with the library's bounded mbarrier
 * wait and a limit of timeout_us microseconds (1 .. 10^7), on a barrier that
 * nothing arrives on.  The wait gives up, QLORA_DEVERR_TIMEOUT is OR-ed into
 * *dev_err (required), *gave_up (device int, nullable) is set to 1, and the
 * kernel returns normally: no fault, and the context stays usable.
 */
qlora_status qlora_selftest_bounded_wait(unsigned timeout_us, int *dev_err, int *gave_up, void *stream);

/*
 * Storage-format variants, for the quantisation study that sets NF4 against
 * other 4-bit types, block sizes and treatments of the block constants
 * ("QLoRA: Efficient Finetuning of Quantized LLMs", intuitivepapers.ai:
 * §Quantize in blocks, §NormalFloat — the uniform Int4 grid —, §Double
 * quantization, §It matches 16-bit finetuning — "4-bit float variants";
 * "QLoRA Review", tildalice.io, §What Would Trip You Up in Practice — block
 * size trades precision against overhead).  The linear layer itself always
 * uses NF4, blocks of 64 and E4M3 constants (qlora_nf4_weight above).
 *
 * Code books (16 ascending float32 levels in [-1, 1]):
 *   QLORA_CB_NF4       the NF4 levels of qlora_build_codebook;
 *   QLORA_CB_INT4      k/7 for k = -8..7 (the symmetric absmax integer grid;
 *                      -8/7 is never the nearest level of a value in [-1, 1]);
 *   QLORA_CB_FP4_E2M1  +-{0, 0.5, 1, 1.5, 2, 3, 4, 6} / 6;
 *   QLORA_CB_FP4_E3M0  +-{0, 0.25, 0.5, 1, 2, 4, 8, 16} / 16
 *                      (the float layouts' +0 and -0 are both the level +0).
 * Block sizes 32, 64, 128, 256 (consecutive weights along K; K % block == 0).
 * Block constants (absmax c of each block):
 *   QLORA_DQ_NONE  stored as float32;
 *   QLORA_DQ_E4M3  the second quantisation of qlora_quantize (mean, groups of
 *                  256 blocks, E4M3 codes of the centred constants);
 *   QLORA_DQ_INT8  the same with the int8 absmax grid: S_g = float32(amax_g/127),
 *                  e = round-half-even(float32(dev/S_g)), reconstruction
 *                  fmaf(e, S_g, mu).
 * Codes: x = float32(w / c), nearest level, ties to the lower index (of two
 * equal levels the first); an all-zero block codes to the first zero level.
 */
enum { QLORA_CB_NF4 = 0, QLORA_CB_INT4 = 1, QLORA_CB_FP4_E2M1 = 2, QLORA_CB_FP4_E3M0 = 3 };
enum { QLORA_DQ_NONE = 0, QLORA_DQ_E4M3 = 1, QLORA_DQ_INT8 = 2 };

typedef struct qlora_format {
  int codebook;  /* QLORA_CB_* */
  int block;     /* 32, 64, 128 or 256 */
  int dq;        /* QLORA_DQ_* */
} qlora_format;

typedef struct qlora_qweight {
  int64_t N, K;
  qlora_format fmt;
  uint8_t *codes;  /* N*K/2 bytes, two codes per byte (even element in the high nibble) */
  void *consts;    /* per block: float32 c (DQ_NONE) or one byte (E4M3 code / int8) */
  float *c1;       /* per group of 256 blocks (DQ_E4M3, DQ_INT8; else unused, may be NULL) */
  float *mean;     /* 1 float (DQ_E4M3, DQ_INT8; else unused, may be NULL) */
} qlora_qweight;

/* Levels and thresholds of a code book (host); thresholds as in
 * qlora_build_codebook, with the threshold of the upper of two equal levels
 * raised to the next one.  QLORA_ERR_INVALID_ARG for an unknown code book. */
qlora_status qlora_format_codebook(int codebook, float levels[16], float thresholds[15]);

/* Byte sizes of codes, consts and c1 for a format and shape. */
qlora_status qlora_format_sizes(const qlora_format *fmt, int64_t N, int64_t K, size_t *codes_bytes,
                                size_t *consts_bytes, size_t *c1_bytes);

/* Workspace bytes of qlora_quantize_format for a format and shape. */
qlora_status qlora_format_workspace_size(const qlora_format *fmt, int64_t N, int64_t K, size_t *bytes);

/*
 * qlora_quantize_format — W (device, N x K bfloat16) into w's buffers in the
 * format w->fmt.  ws: qlora_format_workspace_size() bytes (16-byte aligned).
 * The mean and group sums follow qlora_quantize's fixed order.  A non-finite
 * weight sets QLORA_DEVERR_NONFINITE.  Deterministic.  All device pointers
 * 16-byte aligned.  Errors: QLORA_ERR_INVALID_ARG (null pointer, unknown code
 * book or constant mode), QLORA_ERR_UNSUPPORTED_SHAPE (block not 32/64/128/256,
 * K % block != 0), QLORA_ERR_MISALIGNED, QLORA_ERR_WORKSPACE.
 */
qlora_status qlora_quantize_format(const uint16_t *W, const qlora_qweight *w, void *ws, size_t ws_bytes,
                                   int *dev_err, void *stream);

/* w_hat = bf16_rn(float32(level[code] * c_hat)) for every weight, into W_out
 * (device, N x K bfloat16); c_hat = c, or the reconstructed constant. */
qlora_status qlora_dequantize_format(const qlora_qweight *w, uint16_t *W_out, void *stream);

/*
 * qlora_quant_error — error of a round trip, for the study's curves.
 * W, W_hat: device, n bfloat16 each (16-byte aligned).  stats: device,
 * 3 doubles (8-byte aligned), overwritten:
 * stats[0] = sum (w - w_hat)^2, stats[1] = sum w^2, stats[2] = max |w - w_hat|
 * (sums in float64; their order is unspecified).
 */
qlora_status qlora_quant_error(const uint16_t *W, const uint16_t *W_hat, int64_t n, double *stats, void *stream);

/* Number of kernels this library has launched in this process so far. */
uint64_t qlora_kernel_launch_count(void);

/*
 * Optional timing hooks.  Each argument is a cudaEvent_t or NULL.  While set,
 * every qlora_linear_forward records fwd_begin / fwd_end on its stream
 * immediately before / after launching the dequant GEMM that produces Y (the
 * small-M kernel when M <= 64), and every
 * qlora_linear_backward records bwd_begin / bwd_end around the fused dequant
 * GEMM that produces dX; every qlora_merge_requantize records fwd_begin /
 * fwd_end around its merge-and-code kernel.  Passing all NULL disables the hooks.  The setting is
 * process-wide and not thread-safe.
 */
qlora_status qlora_set_timing_events(void *fwd_begin, void *fwd_end, void *bwd_begin, void *bwd_end);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_NF4_H */
