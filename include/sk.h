/*
 * sk.h -- C ABI of the sketched linear layer (libsk.so, B200 / sm_100a).
 *
 * The layer ("SpaLLM: Unified Compressive Adaptation of LLMs with Sketching",
 * section 2.2, Eq. 1): each row of an n x d weight is split into `gpr`
 * contiguous groups of gs = d / gpr columns ("groups per row"); every group
 * keeps a lookup table (LUT) of k = 2^bits fp16 values and a frozen one-hot
 * sketching matrix, stored as an index map idx[i][j] in [0, k).  The
 * effective weight is
 *
 *     Theta_hat[i][j] = lut[task][i][j / gs][idx[i][j]].
 *
 * Several LUT sets ("tasks") may share one index map (section 2.3); token t
 * then uses lut[task[t]].
 *
 * Data layouts (all row-major and contiguous, device memory unless stated):
 *   packed : the index map in the packed format below, sk_packed_bytes() bytes.
 *   lut    : IEEE fp16 bits, [ntask][n][gpr][k].
 *   X      : bf16 bits, [T][d]        (layer input, one row per token).
 *   Y, dY  : bf16 bits, [T][n]        (layer output and its gradient).
 *   dX     : bf16 bits, [T][d].
 *   dlut   : fp32, [ntask][n][gpr][k] (gradient of the loss w.r.t. lut).
 *   task   : int32 [T] task id per token, or NULL (every token uses LUT set 0).
 *
 * Packed index format (this library's own; the pages leave index storage
 * open): each row is packed on its own and zero-padded to a multiple of 16
 * bytes (sk_packed_row_bytes).  4-bit: two per byte, index j in nibble (j & 1)
 * of byte j >> 1, low nibble first.  2-bit: four per byte, index j at bits
 * 2*(j & 3) of byte j >> 2.  3-bit: 32 indices per three little-endian uint32
 * words; index j of a 32-index chunk starts at bit 3*(j mod 32) of the 96-bit
 * chunk.
 *
 * Shape rules, checked on the host before anything is launched:
 *   bits in {2, 3, 4}; n >= 1 and n % 8 == 0; d >= 32; gpr >= 1;
 *   d % gpr == 0 and (d / gpr) % 32 == 0 (so every 32-column chunk lies in one
 *   group); T >= 0 (T == 0 launches nothing and returns SK_OK); ntask >= 1.
 *
 * Ownership: the caller allocates and owns every buffer, including any
 * workspace (size from sk_workspace_bytes).  Device pointers must be 16-byte
 * aligned.  Outputs must not overlap inputs.  The library keeps no state
 * besides a device-side check word (sk_device_check) and never allocates
 * device memory.
 *
 * Errors: a non-OK status means nothing was launched, except SK_ERR_CUDA,
 * which reports a failed launch (the CUDA error string is in sk_last_error()).
 * Errors of kernels that already ran asynchronously surface at the caller's
 * next synchronisation, as usual in CUDA.  Data checks that need the device
 * (a task id outside [0, ntask), an index >= 2^bits given to sk_pack) do not
 * stop the kernel: the affected output is written as zero / masked and a bit
 * is set in the device check word, which sk_device_check() reads.
 *
 * Streams: every call is asynchronous on the given stream (NULL = the legacy
 * default stream).
 *
 * Devices and threads: a call runs on the calling thread's current CUDA device
 * (cudaSetDevice).  Any host thread may call, including one that has made no
 * CUDA call yet (an autograd worker thread, for instance): the library binds
 * that device's primary context to the thread before its first driver call.
 */
#ifndef SK_H_
#define SK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SK_ABI_VERSION 1

typedef struct CUstream_st* sk_stream_t; /* same type as cudaStream_t */

typedef enum {
  SK_OK = 0,
  SK_ERR_INVALID_ARG = 1,  /* bad pointer, size, shape or overlap          */
  SK_ERR_UNSUPPORTED = 2,  /* valid but not handled (e.g. no sm_100 device) */
  SK_ERR_CUDA = 3,         /* a CUDA call or launch failed                   */
  SK_ERR_DEVICE_CHECK = 4  /* sk_device_check found a flagged input          */
} sk_status;

/* Device check word bits (sk_device_check). */
#define SK_CHECK_TASK_RANGE 1u   /* a task id outside [0, ntask) was seen      */
#define SK_CHECK_INDEX_RANGE 2u  /* sk_pack saw an index >= 2^bits             */
#define SK_CHECK_TIMEOUT 4u      /* a kernel gave up waiting on its own pipeline
                                    (an internal error; its outputs are invalid) */
#define SK_CHECK_NOT_SPD 8u      /* sk_inverse_factor met a pivot <= 0: the damped
                                    Gram matrix is not positive definite       */
#define SK_CHECK_LUT_ORDER 16u   /* sk_sketch_round was given a LUT that is not
                                    ascending                                   */

/* Operation selectors for sk_workspace_bytes. */
#define SK_OP_FWD 0
#define SK_OP_BWD_INPUT 1
#define SK_OP_BWD_LUT 2

int sk_abi_version(void);
const char* sk_status_string(sk_status s);
/* Detail of the last non-OK status returned on this host thread ("" if none). */
const char* sk_last_error(void);

/* Bytes of one packed row: ceil(d * bits / 8) rounded up to 16.  0 if bits or d is invalid. */
size_t sk_packed_row_bytes(int64_t d, int bits);
/* n * sk_packed_row_bytes(d, bits).  0 if the arguments are invalid. */
size_t sk_packed_bytes(int64_t n, int64_t d, int bits);

/*
 * sk_pack: idx (device uint8 [n][d], values < 2^bits) -> packed (device,
 * packed_bytes >= sk_packed_bytes(n, d, bits)).  Padding bytes are written as
 * zero.  An index >= 2^bits is masked to its low bits and sets
 * SK_CHECK_INDEX_RANGE.  This is step a0 (off the timed path): it encodes the
 * one-hot sketching matrix of Eq. 1 as its column indices.
 */
sk_status sk_pack(const uint8_t* idx, int64_t n, int64_t d, int bits,
                  void* packed, size_t packed_bytes, sk_stream_t stream);

/* sk_unpack: the inverse of sk_pack (device packed -> device uint8 [n][d]). */
sk_status sk_unpack(const void* packed, int64_t n, int64_t d, int bits,
                    uint8_t* idx, sk_stream_t stream);

/*
 * sk_dequant: writes the dense effective weight of LUT set `task` as bf16 bits
 * [n][d] (Eq. 1 with groups per row), each value the round-to-nearest-even
 * bf16 of the fp16 table entry.  The fused kernels use exactly these values.
 * Meant for tests and for a dense-GEMM comparison; not on the hot path.
 */
sk_status sk_dequant(const void* packed, const uint16_t* lut, int bits, int gpr,
                     int64_t n, int64_t d, int task, int ntask,
                     uint16_t* theta, sk_stream_t stream);

/*
 * Workspace bytes that the call selected by `op` (SK_OP_*) needs for these
 * shapes; 0 means no workspace (a NULL workspace is then fine).
 * SK_OP_BWD_LUT: required by the tensor-core LUT gradient (partial bins).
 * SK_OP_FWD with ntask > 1: the task routing of the tensor-core forward
 * (permutation, tile list and X in task order); optional -- without it a
 * batch with several LUT sets runs on the CUDA-core kernel.
 * SK_OP_BWD_INPUT with ntask > 1: the same routing for the tensor-core input
 * gradient (dY in task order); optional in the same way.
 * SK_OP_BWD_LUT with ntask > 1 (and task ids): the task routing of the
 * tensor-core LUT gradient (X and dY in task order, each set's tokens padded
 * to a multiple of 64 positions) plus the partial bins of every LUT set;
 * optional -- without it the batch runs on the CUDA-core kernel.  With one
 * LUT set the tensor-core LUT gradient requires its workspace.
 */
size_t sk_workspace_bytes(int op, int64_t n, int64_t d, int bits, int gpr,
                          int64_t T, int ntask);

/*
 * sk_linear_fwd: Y = X Theta_hat^T, token t with LUT set task[t].
 * SpaLLM section 2.3: one compressed matmul per layer, no adapter branch.
 * Accumulation is fp32; weights enter the tensor cores as bf16 (the RNE
 * rounding of the fp16 table values, as sk_dequant writes them); Y is rounded
 * to bf16 (RNE).
 */
sk_status sk_linear_fwd(const void* packed, const uint16_t* lut, int bits, int gpr,
                        int64_t n, int64_t d, const uint16_t* X, int64_t T,
                        const int32_t* task, int ntask, uint16_t* Y,
                        void* workspace, size_t workspace_bytes, sk_stream_t stream);

/*
 * sk_linear_fwd_group: the forward of several layers that see the same number
 * of tokens, in one call: for every layer l, Y_l = X_l Theta_hat_l^T exactly as
 * sk_linear_fwd computes it (same precision, same LUT-set rule).  Typical use:
 * the projections of a decoder block at decode batch sizes, where each layer
 * alone is too small to keep the GPU busy across a launch boundary.
 *
 * With 4-bit indices, 1 <= T <= 16 and one LUT set per call (or several sets
 * and a single token) the layers run in one launch, spread over the SMs in
 * proportion to their size; otherwise the call runs sk_linear_fwd for each
 * layer in order, without a workspace.  Layers may share an input X (the
 * q/k/v or gate/up projections of a block); no layer's Y may overlap any
 * buffer of any layer.  `task` and `ntask` apply to every layer.  At most
 * SK_MAX_GROUP_LAYERS layers; the array itself is host memory and is not
 * kept after the call returns.
 */
#define SK_MAX_GROUP_LAYERS 8
typedef struct {
  const void* packed;      /* device, packed index map of the layer */
  const uint16_t* lut;     /* device fp16 [ntask][n][gpr][2^bits]     */
  int gpr;
  int64_t n, d;
  const uint16_t* X;       /* device bf16 [T][d]                       */
  uint16_t* Y;             /* device bf16 [T][n]                       */
} sk_layer;
sk_status sk_linear_fwd_group(const sk_layer* layers, int nlayers, int bits, int64_t T,
                              const int32_t* task, int ntask, sk_stream_t stream);

/*
 * sk_linear_bwd_input: dX = dY Theta_hat (chain rule through the frozen
 * sketch; the layer has to pass gradients back to earlier layers).  Same
 * precision rules as sk_linear_fwd.
 */
sk_status sk_linear_bwd_input(const void* packed, const uint16_t* lut, int bits, int gpr,
                              int64_t n, int64_t d, const uint16_t* dY, int64_t T,
                              const int32_t* task, int ntask, uint16_t* dX,
                              void* workspace, size_t workspace_bytes, sk_stream_t stream);

/*
 * sk_linear_bwd_lut: the LUT gradient of the corrected Eq. 6 ("Sketch to
 * Adapt" OpenReview discussion, reply Q1): dL/dw = dL/dy (M X)^T, i.e.
 *
 *     dlut[task][i][g][c] = sum over tokens t with task[t] == task and
 *                           columns j of group g with idx[i][j] == c
 *                           of dY[t][i] * X[t][j].
 *
 * The loss is linear in the LUT, so no LUT values are needed.  The dense
 * n x d gradient is never written to memory.  accumulate = 0 overwrites dlut,
 * 1 adds to it.  fp32 throughout; the result is deterministic (no float
 * atomics).
 */
sk_status sk_linear_bwd_lut(const void* packed, int bits, int gpr, int64_t n, int64_t d,
                            const uint16_t* X, const uint16_t* dY, int64_t T,
                            const int32_t* task, int ntask, float* dlut, int accumulate,
                            void* workspace, size_t workspace_bytes, sk_stream_t stream);

/*
 * sk_linear_bwd_lut_noalloc: the LUT gradient of sk_linear_bwd_lut, for
 * callers that cannot allocate device memory when they need it (a plugin
 * inside another framework's executor that owns all device memory, a loop that
 * has reserved its whole memory budget up front, code that must not call
 * cudaMalloc because it synchronises the device).  The pages have no
 * counterpart: this is a deployment convenience of this library.
 *
 * It allocates nothing: where sk_linear_bwd_lut would take a caller workspace,
 * this call uses one fixed array of SK_NOALLOC_SCRATCH_BYTES (32 MiB) in
 * device memory.  The array is part of the library's backward-kernel module:
 * a process holds those 32 MiB on every device where that module is loaded
 * (the first tensor-core input or LUT gradient, or the first call of this
 * function, on that device; every device the library initialises when CUDA
 * loads modules eagerly), until it exits, whether or not it ever calls this
 * function.  The caller still passes the inputs and dlut.  Arguments, layouts, results and
 * errors are those of sk_linear_bwd_lut; in addition a layer whose scratch
 * need (sk_workspace_bytes(SK_OP_BWD_LUT, ...)) exceeds the array is rejected
 * with SK_ERR_INVALID_ARG before anything is launched.
 *
 * The first call on a device looks up the array's device address with that
 * device current; make that first call before any stream capture.  The
 * address is cached per device and context: after a device reset the next
 * call looks it up again (again outside any stream capture).  Every call
 * shares the one array and it keeps the last call's contents (each call
 * overwrites every entry it reads, so nothing has to start at zero): calls that
 * overlap on the GPU (different streams, concurrently replayed graphs) race and
 * corrupt each other's results, so order them on one stream.
 */
#define SK_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
sk_status sk_linear_bwd_lut_noalloc(const void* packed, int bits, int gpr, int64_t n, int64_t d,
                                    const uint16_t* X, const uint16_t* dY, int64_t T,
                                    const int32_t* task, int ntask, float* dlut, int accumulate,
                                    sk_stream_t stream);

/*
 * sk_bin_counts: the static bin sizes of the one-hot sketch (Eq. 1),
 * counts[i][g][c] = the number of columns j of group g in row i with
 * idx[i][j] == c, as int32 [n][gpr][2^bits] in device memory.  They sum to
 * d / gpr over c.  The averaging variant of the LUT update divides the LUT
 * gradient by them (SpaLLM section 2.1: the gradients of the virtual
 * parameters that share a trainable value are averaged).  Shape rules and
 * errors as sk_linear_bwd_lut.
 */
sk_status sk_bin_counts(const void* packed, int bits, int gpr, int64_t n, int64_t d, int32_t* counts,
                        sk_stream_t stream);

/*
 * sk_lut_adamw / sk_lut_sgd: one optimizer step on the LUT values.  The pages
 * train the LUTs but name no optimizer; these are the plain textbook
 * updates on fp32 master copies, elementwise over ntask * n * gpr * 2^bits
 * entries (device fp32 arrays of that length, layout [ntask][n][gpr][k]):
 *
 *   g = grad / max(counts, 1)  if counts != NULL (averaging; counts [n][gpr][k]
 *                               from sk_bin_counts, shared by every LUT set)
 *   AdamW: p *= 1 - lr * weight_decay;  m = beta1 m + (1 - beta1) g;
 *          v = beta2 v + (1 - beta2) g^2;
 *          p -= lr * (m / (1 - beta1^step)) / (sqrt(v / (1 - beta2^step)) + eps)
 *   SGD:   p -= lr * g
 *
 * master, m and v are updated in place (m and v start at zero); grad is the
 * output of sk_linear_bwd_lut.  When lut is not NULL the fp16 LUTs the layer
 * reads ([ntask][n][gpr][k], IEEE fp16 bits) receive the round-to-nearest-even
 * fp16 of the new master values.  step >= 1; 0 <= beta1, beta2 < 1; eps > 0.
 * Outputs must not overlap inputs other than themselves.
 */
sk_status sk_lut_adamw(float* master, float* m, float* v, const float* grad, const int32_t* counts, int ntask,
                       int64_t n, int gpr, int bits, float lr, float beta1, float beta2, float eps,
                       float weight_decay, int step, uint16_t* lut, sk_stream_t stream);
sk_status sk_lut_sgd(float* master, const float* grad, const int32_t* counts, int ntask, int64_t n, int gpr,
                     int bits, float lr, uint16_t* lut, sk_stream_t stream);

/*
 * Sketching stage ("SpaLLM: Unified Compressive Adaptation of LLMs with
 * Sketching", section 2.2; "Sketch to Adapt" OpenReview discussion, concern
 * 1): from a dense weight Theta (float32 [n][d]) and calibration activations
 * X (bf16 [s][d]; the pages use 128 sequences of 2048 tokens) to the index
 * map and the first fp16 LUTs.  Run once per layer; every buffer is device
 * memory owned by the caller; nothing is allocated.  The usual chain is
 *   sk_gram -> sk_inverse_factor -> sk_lloyd -> sk_sketch_round -> sk_pack.
 *
 * sk_gram: H (float32 [d][d]) = X^T X, or H += X^T X when accumulate != 0
 * (calibration data may come in batches).  Tensor cores, fp32 accumulation.
 * 0 <= s < 2^31, 64 <= d <= 65536, d % 8 == 0.  s == 0 zeroes H (or leaves
 * it when accumulating).
 *
 * sk_inverse_factor: damping, then the inverse factor in float64.  A zero
 * diagonal entry of H counts as 1, then damp * mean(diag H) is added to the
 * diagonal (the pages are silent on damping; this follows the error-
 * compensated rounding they cite).  Only the upper triangle of H is read.
 * Outputs U (float64 [d][d], upper triangular, H^-1 = U^T U) and hinv_diag
 * (float64 [d], the diagonal of H^-1).  workspace: at least
 * sk_inverse_factor_workspace_bytes(d) bytes.  A damped H that is not
 * positive definite sets SK_CHECK_NOT_SPD (the outputs then hold NaNs).
 *
 * sk_lloyd: weighted Lloyd's algorithm per (row, group), weights
 * 1 / hinv_diag[j], k = 2^bits centroids started evenly over the group's
 * [min, max]; a value joins the centroid whose float32 midpoints bracket it
 * (a value on a midpoint goes to the lower one), a centroid becomes the
 * float64 weighted mean of its members rounded to float32 (an empty cluster
 * keeps its centroid); stops when an update moves no value, or after
 * max_iter updates.  Writes lut (fp16 bits [n][gpr][k], ascending) and, if
 * iters is not NULL, the updates run per (row, group) (int32 [n][gpr]).
 * d % gpr == 0 and d / gpr <= 16384 (else SK_ERR_UNSUPPORTED).  theta must
 * be finite.
 *
 * sk_sketch_round: the index map (uint8 [n][d], values < 2^bits).  Columns
 * are mapped in order: column j of every row goes to the nearest entry of
 * its group's LUT (float32 midpoints, ties to the lower entry) of its current
 * value w_j, and the later columns c of the row move by
 * -(w_j - q_j) / U_jj * U_jc (the Optimal Brain Surgeon update over the
 * columns not yet mapped; the reading of the discussion's Eq. 13).  Values
 * are carried in float64.  lut: fp16 bits [n][gpr][k], ascending per group
 * (a descending pair sets SK_CHECK_LUT_ORDER).  workspace: at least
 * sk_sketch_round_workspace_bytes(n, d) bytes.
 */
size_t sk_inverse_factor_workspace_bytes(int64_t d);
size_t sk_sketch_round_workspace_bytes(int64_t n, int64_t d);
sk_status sk_gram(const uint16_t* X, int64_t s, int64_t d, float* H, int accumulate, sk_stream_t stream);
sk_status sk_inverse_factor(const float* H, int64_t d, double damp, double* U, double* hinv_diag, void* workspace,
                            size_t workspace_bytes, sk_stream_t stream);
sk_status sk_lloyd(const float* theta, const double* hinv_diag, int bits, int gpr, int64_t n, int64_t d, int max_iter,
                   uint16_t* lut, int32_t* iters, sk_stream_t stream);
sk_status sk_sketch_round(const float* theta, const double* U, const uint16_t* lut, int bits, int gpr, int64_t n,
                          int64_t d, uint8_t* idx, void* workspace, size_t workspace_bytes, sk_stream_t stream);

/*
 * sk_device_check: synchronises `stream`, stores the device check word
 * (SK_CHECK_* bits, 0 = nothing flagged) in *flags and clears it if `clear`.
 * Returns SK_ERR_DEVICE_CHECK when any bit was set, else SK_OK.
 */
sk_status sk_device_check(uint32_t* flags, int clear, sk_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SK_H_ */
