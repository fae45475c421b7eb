/*
 * qlora_nf4.h -- C ABI of the B200 (sm_100a) library for the frozen NF4 linear
 * layer with a LoRA adapter, as the QLoRA pages define it.
 *
 * What the layer computes (sources named by page title and section):
 *   - "QLoRA" (Ultralytics glossary), "How QLoRA works": every frozen weight is a
 *     4-bit code into 16 levels placed at normal quantiles, with one absmax scale
 *     per block of 64 weights; the block scales are themselves quantised to 8 bits
 *     in blocks of 256; the forward pass dequantises NF4 to bfloat16 right before
 *     the matmul and adds the LoRA path; the backward pass computes gradients
 *     through the dequantised weights and updates only the two LoRA matrices.
 *   - "Grokking QLoRA" (vnread), "Double Quantization": the 8-bit second level is FP8.
 *   - "What is LoRA?" (IBM) and "Mastering model fine-tuning" (ezsol.ir),
 *     "Low-Rank Adaptation (LoRA)": Delta W = B A with rank r; lora_alpha scales it.
 *
 * Notation: W [N, K] row-major (nn.Linear convention y = X W^T), N = rows =
 * out_features, K = cols = in_features; X [M, K]; A [r, K]; B [N, r]; s = alpha / r
 * (float32).  Block = 64 consecutive elements of row-major W (K % 64 == 0, so a
 * block never crosses a row); group = 256 consecutive blocks (the last group of a
 * tensor may be short; groups may cross rows).  nb = N*K/64, ng = ceil(nb/256).
 *
 * Formats fixed by this library (readings of the pages):
 *   codes        N*K/2 bytes; byte i = code[2i] | code[2i+1] << 4 (row-major order)
 *   scale_codes  nb bytes, OCP FP8 E4M3 (sign bit 0): q = E4M3_rne_sat(S / c2)
 *   c2           ng float32: c2 = max(S over the group) / 448 (0 for an all-zero group)
 *   code         argmin_j |fl32(w / S) - L_j| in float32, lowest j on ties; S == 0 -> 7
 *   dequantised  w' = bf16_rne(fl32(L[code] * fl32(E4M3(q) * c2)))
 *
 * Conventions shared by every entry point:
 *   - Pointers named in a qlora_nf4_tensor, qlora_lora or as X/Y/dY/dX/dA/dB/ws
 *     are DEVICE pointers, allocated and owned by the caller.  Tensor pointers must
 *     be 16-byte aligned; ws must be 256-byte aligned.
 *   - The library never allocates, frees or synchronises (except
 *     qlora_read_status, which synchronises the stream it is given).  All scratch
 *     comes from the caller's workspace ws (qlora_workspace_bytes() tells how much).
 *     The first QLORA_STATUS_BYTES of ws hold a device status word and two
 *     counters of the one-kernel decode forward (an arrival count and a call
 *     generation).  A new workspace must start zeroed (at least its first
 *     QLORA_STATUS_BYTES and, for the forward with M <= 16, the s*T entries
 *     after them: allocate it zeroed).  Every completed call leaves the arrival
 *     count at zero; after a call whose kernel did not complete, or one that
 *     recorded QLORA_ERR_TIMEOUT, call qlora_clear_status before reusing ws.
 *   - Argument checks run on the host before any launch; a failed check returns an
 *     error code and launches nothing.  A failed launch returns QLORA_ERR_CUDA.
 *     Errors found on the device (non-finite weights, a bounded wait that timed
 *     out) are OR-ed into the status word; qlora_read_status() returns them.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Entry points are thread-safe and keep no per-call state.  Nothing is printed
 *     and no C++ exception crosses this boundary.
 *   - Only sm_100 devices are supported (QLORA_ERR_NO_DEVICE otherwise).
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QLORA_NF4_ABI_VERSION 2
#define QLORA_BLOCK 64          /* weights per first-level absmax block */
#define QLORA_GROUP 256         /* first-level scales per second-level group */
#define QLORA_STATUS_BYTES 256  /* bytes at the start of ws reserved for the status word */
#define QLORA_MAX_RANK 256

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

typedef struct CUstream_st *qlora_stream_t; /* same handle type as cudaStream_t */

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARGUMENT = 1,   /* null pointer, bad enum, bad rank or M */
  QLORA_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 64 != 0, or a dimension out of range */
  QLORA_ERR_MISALIGNED = 3,         /* a tensor pointer is not 16-byte aligned (ws: 256) */
  QLORA_ERR_WORKSPACE_TOO_SMALL = 4,
  QLORA_ERR_NONFINITE = 5,          /* device: a block held a NaN or an infinity */
  QLORA_ERR_TIMEOUT = 6,            /* device: a bounded wait gave up */
  QLORA_ERR_CUDA = 7,               /* a CUDA runtime call or launch failed */
  QLORA_ERR_NO_DEVICE = 8           /* the current device is not an sm_100 GPU */
} qlora_status;

typedef enum { QLORA_F32 = 0, QLORA_BF16 = 1 } qlora_dtype;

/* Format of the 8-bit second-level scale codes.  The double-quantisation bullet
 * of the glossary page ("How QLoRA works") says only "8 bits in blocks of 256";
 * "Grokking QLoRA" (vnread), "Double Quantization", names FP8.  E4M3 is the
 * default; the other two are alternative readings with the same structure:
 * per group of 256 scales c2 = fl32(max S / F) and q = enc(fl32(S / c2)), the
 * decoded scale S' = fl32(dec(q) * c2), with
 *   QLORA_SCALE_E4M3  OCP FP8 E4M3, F = 448, round to nearest even, saturating
 *   QLORA_SCALE_E5M2  OCP FP8 E5M2, F = 57344, round to nearest even, saturating
 *   QLORA_SCALE_U8    unsigned byte q = rne(x) clamped to 255, dec(q) = q, F = 255 */
typedef enum { QLORA_SCALE_E4M3 = 0, QLORA_SCALE_E5M2 = 1, QLORA_SCALE_U8 = 2 } qlora_scale_format;

/* Quantised weight W [rows, cols]; three caller-owned device buffers, sized by
 * qlora_nf4_storage_bytes(). */
typedef struct {
  int64_t rows;          /* N */
  int64_t cols;          /* K, a multiple of 64 */
  uint8_t *codes;        /* rows*cols/2 bytes, packed nibbles */
  uint8_t *scale_codes;  /* nb bytes, in scale_format */
  float *c2;             /* ng float32 second-level constants */
  int32_t scale_format;  /* qlora_scale_format (0, E4M3, when the struct is zero-initialised); set
                            before qlora_nf4_quantize and kept with the buffers it wrote */
} qlora_nf4_tensor;

/* LoRA adapter: A [r, K] and B [N, r], both bf16 row-major device buffers.
 * r in [8, 256] and a multiple of 8. */
typedef struct {
  int32_t r;
  float alpha;
  const void *A;
  const void *B;
} qlora_lora;

/* Version of this ABI (QLORA_NF4_ABI_VERSION). */
QLORA_API int qlora_abi_version(void);

/* Copies the 16 float32 NF4 levels the kernels use into out[0..15] (host memory).
 * They are the normal-quantile levels of the glossary page's snippet ("How QLoRA
 * works"), each rounded once to float32. */
QLORA_API void qlora_nf4_codebook(float out[16]);

/* Bytes of the three buffers of a quantised [rows, cols] tensor.  Any of the
 * out-pointers may be NULL.  Returns their sum, or 0 if cols % 64 != 0 or a
 * dimension is not positive. */
QLORA_API size_t qlora_nf4_storage_bytes(int64_t rows, int64_t cols, size_t *codes_bytes,
                               size_t *scale_codes_bytes, size_t *c2_bytes);

/* Workspace bytes for qlora_linear_fwd (for_backward = 0) or qlora_linear_bwd
 * (for_backward = 1) with M tokens, W [N, K] and rank r; 0 for invalid sizes.
 * The entry points also accept less, down to QLORA_STATUS_BYTES + (256-byte
 * rounded) M*r*2 bytes for the forward and QLORA_STATUS_BYTES + 4 * that for the
 * backward (QLORA_ERR_WORKSPACE_TOO_SMALL below it); the size returned here adds
 * fp32 partial planes that let the rank-r GEMMs (X A^T, dY B) split their K
 * range over more CTAs when M > 16.  Results are the same either way to within
 * float32 rounding order. */
QLORA_API size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t r, int for_backward);

/* Workspace bytes for qlora_linear_fwd_multi's faster path: the forward minimum
 * for M tokens plus a float32 [M, N] buffer (256-byte rounded); 0 for invalid
 * sizes or M > 16. */
QLORA_API size_t qlora_workspace_bytes_multi(int64_t M, int64_t N, int64_t K, int32_t r);

/* Quantise W [out->rows, out->cols] (float32 or bf16, row-major, device) to NF4
 * with double-quantised scales (glossary page, "How QLoRA works": NF4 and double
 * quantisation bullets).  Writes out->codes, out->scale_codes, out->c2.
 * ws: device workspace of at least QLORA_STATUS_BYTES (status word).  A block
 * holding a NaN or an infinity sets QLORA_ERR_NONFINITE in the status word; the
 * contents of that block's outputs are then unspecified. */
QLORA_API qlora_status qlora_nf4_quantize(const void *W, qlora_dtype w_dtype, const qlora_nf4_tensor *out,
                                void *ws, qlora_stream_t stream);

/* Dequantise to W_out [rows, cols] row-major (bf16; float32 holds the same
 * bf16-exact values, for tests), the step the glossary page places right
 * before the matmul. */
QLORA_API qlora_status qlora_nf4_dequantize(const qlora_nf4_tensor *w, void *W_out, qlora_dtype out_dtype,
                                  qlora_stream_t stream);

/* Forward of the frozen linear layer with LoRA (glossary page, "How QLoRA
 * works", forward rule):  Y [M, N] = X W'^T + s (X A^T) B^T.
 *   X      bf16 [M, K] device
 *   Y      [M, N] device, bf16 or float32 (y_dtype)
 *   T_save nullable bf16 [2, M, r] device: receives T = X A^T for the backward
 *          pass as the pair T_hi = bf16(T) (first M*r elements) and
 *          T_lo = bf16(T - T_hi) (next M*r), so T_hi + T_lo carries ~16 bits
 *   ws     device workspace of ws_bytes >= qlora_workspace_bytes(M, N, K, r, 0)
 * M >= 1.  M <= 16 takes the decode (GEMV) path; larger M the tensor-core path. */
QLORA_API qlora_status qlora_linear_fwd(const qlora_nf4_tensor *W, const qlora_lora *adapter, const void *X,
                              int64_t M, void *Y, qlora_dtype y_dtype, void *T_save, void *ws,
                              size_t ws_bytes, qlora_stream_t stream);

/* Backward (glossary page, "How QLoRA works": gradients through the dequantised
 * weights, only the LoRA matrices updated).  With U = dY B:
 *   dX [M, K] = dY W' + s U A          (dx_dtype: bf16 or float32)
 *   dA [r, K] = s U^T X                (grad_dtype: bf16 or float32)
 *   dB [N, r] = s dY^T T,  T = X A^T   (grad_dtype)
 * T_saved: nullable bf16 [2, M, r] pair from qlora_linear_fwd; NULL recomputes it.
 * dY bf16 [M, N].  dX, dA, dB are overwritten (not accumulated).  W gets no
 * gradient. */
QLORA_API qlora_status qlora_linear_bwd(const qlora_nf4_tensor *W, const qlora_lora *adapter, const void *X,
                              const void *dY, int64_t M, const void *T_saved, void *dX,
                              qlora_dtype dx_dtype, void *dA, void *dB, qlora_dtype grad_dtype,
                              void *ws, size_t ws_bytes, qlora_stream_t stream);

/* Forward of the frozen linear layer with LoRA for callers that cannot allocate
 * device memory when they call in: same inputs, outputs and results as
 * qlora_linear_fwd, but with no workspace argument.  Examples are a plugin run
 * from another runtime's launch callback, where cudaMalloc is not allowed
 * because it synchronises the device and breaks the host's memory plan, or a
 * serving loop whose device memory budget is fixed up front.
 * This entry point has no counterpart on the QLoRA pages; it is a deployment
 * convenience.  Its scratch (status word and the s*T buffer) is one static
 * device array of QLORA_NOALLOC_SCRATCH_BYTES that the library holds on every
 * GPU that loads it until the process exits.  Sizes whose workspace
 * (qlora_workspace_bytes(M, N, K, r, 0)) exceeds it return
 * QLORA_ERR_UNSUPPORTED_SHAPE and launch nothing.
 * The first call on a device looks up the array's device address (with that
 * device current); make that first call before any stream capture.  Every call
 * on a device shares the one array and the contents left by the last call: calls
 * that overlap on the GPU (different streams, or other threads) race on it, so
 * serialise them.  Device-side status of these calls is not readable: when a
 * kernel of such a call records a device-side error (a bounded wait that gave
 * up), the call has still returned QLORA_OK and Y and T_save are undefined.
 * A failed address lookup returns QLORA_ERR_CUDA and is retried by the next
 * call. */
#define QLORA_NOALLOC_SCRATCH_BYTES (256u + 2u * 1024u * 1024u)
QLORA_API qlora_status qlora_linear_fwd_noalloc(const qlora_nf4_tensor *W, const qlora_lora *adapter,
                                                const void *X, int64_t M, void *Y, qlora_dtype y_dtype,
                                                void *T_save, qlora_stream_t stream);

/* Forward and backward with LoRA dropout ("Mastering model fine-tuning"
 * (ezsol.ir), "Low-Rank Adaptation (LoRA)": its LoRA configuration sets
 * lora_dropout).  The adapter branch reads D(X) = X * keep / (1 - p):
 *   Y  = X W'^T + s (D(X) A^T) B^T,  T = D(X) A^T (saved as by qlora_linear_fwd)
 *   dX = dY W' + s ((dY B) A) * keep / (1 - p),  dA = s (dY B)^T D(X),  dB = s dY^T T
 *   keep  device uint8 [M, K/8], 16-byte aligned: bit (k % 8) of byte k / 8 of
 *         row m is 1 to keep X[m, k] (the drawn mask; the caller draws it)
 *   p     drop probability, 0 <= p < 1
 * Other arguments as qlora_linear_fwd / qlora_linear_bwd.  ws needs room for a
 * masked copy of X as well: qlora_workspace_bytes_dropout() (the entry points
 * accept down to the plain minimum plus that copy). */
QLORA_API size_t qlora_workspace_bytes_dropout(int64_t M, int64_t N, int64_t K, int32_t r, int for_backward);
QLORA_API qlora_status qlora_linear_fwd_dropout(const qlora_nf4_tensor *W, const qlora_lora *adapter, const void *X,
                                                const void *keep, float p, int64_t M, void *Y, qlora_dtype y_dtype,
                                                void *T_save, void *ws, size_t ws_bytes, qlora_stream_t stream);
QLORA_API qlora_status qlora_linear_bwd_dropout(const qlora_nf4_tensor *W, const qlora_lora *adapter, const void *X,
                                                const void *dY, const void *keep, float p, int64_t M,
                                                const void *T_saved, void *dX, qlora_dtype dx_dtype, void *dA,
                                                void *dB, qlora_dtype grad_dtype, void *ws, size_t ws_bytes,
                                                qlora_stream_t stream);

/* Decode forward of one NF4 base serving several adapters at once ("What is
 * LoRA?" (IBM): one shared frozen base, many small LoRA modules swapped per task;
 * "QLoRA" glossary page, "Trade-offs": adapters are small enough to store and
 * swap per task).  Token t uses adapters[adapter_of_token[t]]:
 *   Y[t] = X[t] W'^T + s_t (X[t] A_t^T) B_t^T,   s_t = alpha_t / r.
 *   adapters          host array of n_adapters >= 1 adapters, all of one rank r
 *   adapter_of_token  HOST int32 [M], values in [0, n_adapters)
 *   X bf16 [M, K], Y [M, N] (y_dtype) device; 1 <= M <= 16
 *   ws                device workspace, as qlora_linear_fwd's for M tokens; given
 *                     qlora_workspace_bytes_multi(M, N, K, r) bytes (room for a
 *                     float32 [M, N] base product) and r / 8 a power of two, the
 *                     adapters' term runs as a separate pass over all SMs after
 *                     the base GEMV (faster); results agree to float32 rounding
 *                     order either way
 * Runs the staged decode kernel: N % 16 == 0, K % 256 == 0 and (K <= 4096 or
 * K % 4096 == 0), else QLORA_ERR_UNSUPPORTED_SHAPE.  No T is saved (decode). */
QLORA_API qlora_status qlora_linear_fwd_multi(const qlora_nf4_tensor *W, const qlora_lora *adapters,
                                              int32_t n_adapters, const int32_t *adapter_of_token, const void *X,
                                              int64_t M, void *Y, qlora_dtype y_dtype, void *ws, size_t ws_bytes,
                                              qlora_stream_t stream);

/* Merged export of a trained adapter ("QLoRA" glossary page, "Trade-offs":
 * merging into the base model needs it dequantised to 16 bit; "What is LoRA?"
 * (IBM): the low-rank update merges into the frozen weights for deployment):
 *   W_out [N, K] bf16 = bf16_rne(W' + s B A),  s = alpha / r,
 * with W' the dequantised NF4 weight, s B A from the bf16 adapter on tensor
 * cores (tcgen05) with float32 accumulation, the sum in float32, rounded to
 * bf16 once.  W_out: device, 16-byte aligned, caller-owned, overwritten.  Errors
 * as for qlora_linear_fwd (invalid tensor or adapter, misalignment, no device).
 * Takes no workspace: a device-side error (a bounded wait that gave up) is
 * recorded in the library status word of the device, read by
 * qlora_read_library_status. */
QLORA_API qlora_status qlora_lora_merge(const qlora_nf4_tensor *W, const qlora_lora *adapter, void *W_out,
                                        qlora_stream_t stream);

/* AdamW hyper-parameters: learning rate lr >= 0, 0 <= beta1, beta2 < 1,
 * eps > 0, decoupled weight decay >= 0. */
typedef struct qlora_adamw_hparams {
  float lr;
  float beta1;
  float beta2;
  float eps;
  float weight_decay;
} qlora_adamw_hparams;

/* One AdamW step (decoupled weight decay, bias-corrected; "Grokking QLoRA"
 * (vnread), "Paged Optimizers": Adam keeps a momentum and a variance for every
 * trained parameter) on n float32 parameters, in place:
 *   m = b1 m + (1 - b1) g;  v = b2 v + (1 - b2) g^2;
 *   p = p (1 - lr wd) - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
 * t = step >= 1.  param, grad, exp_avg, exp_avg_sq: device float32 [n], 16-byte
 * aligned (m and v start at zero before step 1).  param_bf16: nullable device
 * bf16 [n], 8-byte aligned; receives bf16(p), the copy the layer reads.  Used
 * on the flat buffer of every layer's A and B after the data-parallel
 * all-reduce of their gradients.  QLORA_ERR_INVALID_ARGUMENT for n < 1, step
 * < 1, a missing pointer or hyper-parameters out of range. */
QLORA_API qlora_status qlora_adamw_step(float *param, void *param_bf16, const float *grad, float *exp_avg,
                                        float *exp_avg_sq, int64_t n, const qlora_adamw_hparams *hp, int64_t step,
                                        qlora_stream_t stream);

/* Zero the status word and the decode forward's arrival count at the start of
 * ws (enqueued on stream).  The call generation is kept: the decode forward's
 * s*T entries in ws are tagged with it, and a generation that went backwards
 * could make a previous call's entries look current. */
QLORA_API qlora_status qlora_clear_status(void *ws, qlora_stream_t stream);

/* Test hook for the device-side error path (no counterpart on the QLoRA pages).
 * Launches one CTA that runs the protocol every pipelined kernel of the library
 * follows when a bounded wait gives up: it waits on a barrier that nothing
 * completes for limit_us microseconds (1 .. 2,000,000), records
 * QLORA_ERR_TIMEOUT in the status word of ws, lets its other warps leave, waits
 * for the copy it has in flight (a read of the first QLORA_STATUS_BYTES of ws)
 * and frees its tensor memory.  The GPU context stays usable afterwards.
 * QLORA_ERR_INVALID_ARGUMENT for a NULL ws or a limit out of range. */
QLORA_API qlora_status qlora_selftest_bounded_wait(void *ws, uint32_t limit_us, qlora_stream_t stream);

/* Synchronise `stream`, read the status word at the start of ws and return the
 * first error it records (QLORA_OK if none).  The word is left unchanged. */
QLORA_API qlora_status qlora_read_status(const void *ws, qlora_stream_t stream);

/* Synchronise `stream`, read the status word that the library holds on the
 * current device for the calls that take no workspace (qlora_lora_merge), clear
 * it and return the first error it recorded (QLORA_OK if none). */
QLORA_API qlora_status qlora_read_library_status(qlora_stream_t stream);

/* Static, human-readable name of a status code. */
QLORA_API const char *qlora_status_string(qlora_status status);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
