/*
 * larosa.h -- C ABI of the B200 (sm_100a) rotated-sparse linear library.
 *
 * The library computes, for each token (activation row) entering a linear
 * layer, the LaRoSA hot path:
 *
 *   1. rotate:   x_rot = x . Q              (Q orthogonal, d x d)
 *   2. Top-K:    keep the K entries of x_rot of largest magnitude
 *   3. multiply: y = sparse(x_rot) . W_rot,  W_rot = Q^T . W prepared offline,
 *                reading only the K selected rows of W_rot.
 *
 * Source of each step (page title, section):
 *   - "La RoSA: Enhancing LLM Efficiency via Layerwise Rotated Sparse
 *     Activation" (summary page, 方法详解 / 技术框架): a rotation stage that
 *     multiplies each layer's input activation by an orthogonal matrix, then
 *     a sparsification stage that keeps the K largest-magnitude entries and
 *     zeroes the rest.
 *   - Same paper, abstract: layerwise orthogonal rotations of the input
 *     activations; Top-K selection in the rotated activations gives the same
 *     sparsity on every token; activation sparsity cuts memory transfers.
 *   - The counter-rotation W_rot = Q^T W is not printed on the pages; it is
 *     what keeps the layer's output unchanged at K = d, because Q Q^T = I.
 *
 * Conventions shared by every entry point
 *   - Activations are row vectors; a batch of M tokens is a row-major [M x d]
 *     array.  Weights are row-major [d_in x d_out]: row i holds input
 *     channel i's weights (the transpose of torch.nn.Linear.weight), so the
 *     K selected rows of W_rot are K contiguous runs of memory.
 *   - Every pointer argument is a DEVICE pointer owned by the caller, except
 *     where marked "host".  The library never allocates or frees memory.
 *   - Every compute call is asynchronous on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Kernels are launched with programmatic
 *     dependent launch, so a call may begin its set-up while the previous
 *     kernel on the stream drains; it reads no activation before that kernel
 *     has completed.
 *   - Host-side validation happens before anything is enqueued; on failure
 *     the call returns a nonzero larosa_status and enqueues nothing.
 *   - Device-side conditions (a non-finite activation reaching Top-K, an
 *     out-of-range index, a pipeline wait that exceeded its time limit) set
 *     bits in a caller-provided `int* dev_status` word (see LAROSA_DEV_*);
 *     read it with larosa_check().  dev_status may be NULL, in which case
 *     those conditions are not reported.  Kernels never trap or spin without
 *     bound: every wait inside a kernel gives up after a time limit (two
 *     seconds unless changed with larosa_set_wait_limit_ns), sets
 *     LAROSA_DEV_TIMEOUT and exits.
 *   - Workspace: the sparse linear and the fused call use caller-provided
 *     scratch `ws`
 *     of `ws_bytes` bytes, at least larosa_workspace_bytes(...).  It must be
 *     16-byte aligned and ZERO-FILLED before its first use; every call that
 *     completes leaves its counter words consistent again, so the same
 *     buffer serves the next call on the same stream without clearing, also
 *     when that call has other sizes (the persistent words sit at the same
 *     offsets in the layout of every size).  After a device-side error, zero
 *     it again.  Calls that may run concurrently (on different streams) need
 *     distinct workspaces.
 *   - Data types: `dtype` is LAROSA_BF16 (bf16 activations and weights) or
 *     LAROSA_F32 (fp32 activations and weights).  Rotated activations, kept
 *     values and outputs are always fp32; all accumulation is fp32.
 *   - Alignment: weight, activation and output base pointers 16-byte
 *     aligned, and the row length of every weight a multiple of 16 bytes
 *     (rotations and dense weights: a multiple of 8 elements); otherwise
 *     LAROSA_ERR_ALIGN.
 *   - Sizes: 1 <= M <= LAROSA_MAX_M, 1 <= d <= LAROSA_MAX_D, 0 <= K <= d.
 */
#ifndef LAROSA_H
#define LAROSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without including the CUDA runtime header. */
typedef struct CUstream_st *larosa_stream_t;

#define LAROSA_VERSION 100 /* 1.0.0 */
#define LAROSA_MAX_M 16
#define LAROSA_MAX_D 32768

/* Return codes. */
typedef enum {
  LAROSA_OK = 0,
  LAROSA_ERR_INVALID_ARG = 1,      /* NULL pointer, negative size, bad enum */
  LAROSA_ERR_SHAPE = 2,            /* sizes out of range (M, d, K) */
  LAROSA_ERR_ALIGN = 3,            /* pointer or row length not aligned */
  LAROSA_ERR_UNSUPPORTED_DTYPE = 4,
  LAROSA_ERR_CUDA = 5,             /* a CUDA runtime call failed */
  LAROSA_ERR_WORKSPACE = 6,        /* ws NULL or smaller than required */
  LAROSA_ERR_NONFINITE = 7,        /* device: NaN/Inf reached Top-K */
  LAROSA_ERR_TIMEOUT = 8,          /* device: a pipeline wait gave up */
  LAROSA_ERR_INDEX = 9,            /* device: an index was out of range */
  LAROSA_ERR_LIST = 10             /* device (debug checks): a kept list repeats an
                                      index, or a list the library wrote is not
                                      in ascending order */
} larosa_status;

/* Element types of activations and weights. */
typedef enum { LAROSA_F32 = 0, LAROSA_BF16 = 1 } larosa_dtype;

/* Bits a kernel ORs into *dev_status. */
#define LAROSA_DEV_NONFINITE 0x1
#define LAROSA_DEV_TIMEOUT 0x2
#define LAROSA_DEV_INDEX 0x4
#define LAROSA_DEV_LIST 0x8 /* only with the debug checks on (larosa_set_debug) */

/* Human-readable name of a larosa_status value (static string, never NULL). */
const char *larosa_status_string(int status);

/* LAROSA_VERSION of the built library. */
int larosa_version(void);

/*
 * Text of the last CUDA runtime failure behind an LAROSA_ERR_CUDA returned on
 * the calling thread ("" if none).  Static per-thread storage.
 */
const char *larosa_last_error_string(void);

/*
 * Rotation storage.  The orthogonal rotation Q of a layer input is stored as
 * its transpose Qt = Q^T, row-major [d x d]: row j of Qt is column j of Q, so
 * each rotated entry x_rot[j] = sum_i x[i] Q[i][j] is the dot product of x
 * with one contiguous row, and the offline counter-rotation is the plain
 * product Qt . W.  (In PyTorch terms: Qt = Q.T.contiguous() for
 * x_rot = x @ Q.)
 */

/*
 * Offline counter-rotation of a weight (step 0, not on the per-token path):
 *   W_rot[i][j] = sum_k Qt[i][k] * W[k][j],   i.e. W_rot = Q^T . W.
 * Qt: [d_in x d_in], W: [d_in x d_out], W_rot: [d_in x d_out], all row-major
 * and all of type `dtype`.  fp32 accumulation; bf16 outputs are rounded to
 * nearest even.  Projections that share an input (q|k|v, gate|up) are packed
 * by passing their weights concatenated along d_out.  W_rot must not overlap
 * Qt or W.
 */
int larosa_prepare_weights(const void *Qt, const void *W, void *W_rot,
                           int d_in, int d_out, int dtype,
                           larosa_stream_t stream);

/*
 * Folded rotation (offline): moves the rotation of a layer's input into the
 * layer that produces it, so that the producer outputs x_rot = x . Q and the
 * per-token path runs with the identity rotation (larosa_rotate_topk_linear
 * or larosa_rotate_threshold_linear with Qt = NULL) and without streaming Q.
 * For a producer x = h . Wt_prev^T whose weight is given in torch.nn.Linear
 * layout Wt_prev [d x d_prev] (one row per output channel):
 *   Wt_prev_rot[i][j] = sum_k Qt[i][k] * Wt_prev[k][j],  i.e. Q^T . Wt_prev,
 * which is the nn.Linear weight of the producer of x . Q, since
 * h . (Q^T . Wt_prev)^T = (h . Wt_prev^T) . Q.  The pages leave open where
 * the rotation is applied; folding is exact only where nothing nonlinear
 * lies between the producer's product and the rotated input.  Same kernel
 * and rounding as larosa_prepare_weights (fp32 accumulation, bf16 rounded
 * to nearest even); Qt: [d x d], Wt_prev, Wt_prev_rot: [d x d_prev].
 */
int larosa_fold_rotation(const void *Qt, const void *Wt_prev,
                         void *Wt_prev_rot, int d, int d_prev, int dtype,
                         larosa_stream_t stream);

/*
 * Rotation (step 1): x_rot[m][j] = sum_i x[m][i] * Q[i][j]
 *                                = sum_i x[m][i] * Qt[j][i].
 * x: [M x d] of `dtype`, Qt: [d x d] of `dtype`, x_rot: [M x d] fp32.
 * Streams all of Qt once per call (an HBM-bound GEMV for small M).  Needs
 * d a multiple of 8, and x and Qt 16-byte aligned.  Uses no workspace.
 */
int larosa_rotate(const void *x, const void *Qt, float *x_rot, int M, int d,
                  int dtype, larosa_stream_t stream);

/*
 * Exact per-token Top-K by magnitude (step 2).
 * For each of the M rows of x_rot ([M x d] fp32) keeps the K entries of
 * largest |x_rot|; among equal magnitudes the lower index wins (+0 and -0
 * are equal).  Writes idx [M x K] int32 in ascending index order and
 * val [M x K] fp32 = the kept entries with their signs.  A NaN or Inf in a
 * row sets LAROSA_DEV_NONFINITE; that row's output is then unspecified (but
 * every index written is within [0, d)).  K = 0 writes nothing.
 */
int larosa_topk(const float *x_rot, int M, int d, int K, int32_t *idx,
                float *val, int *dev_status, larosa_stream_t stream);

/*
 * Steps 1 and 2 for one token (La RoSA summary, 方法详解 / 技术框架: rotate the
 * layer input by its orthogonal matrix, then keep the K largest magnitudes;
 * abstract: Top-K gives the same sparsity on every token):
 *   x_rot = x . Q;  (idx, val) = TopK(x_rot, K)  with larosa_topk's rule.
 * x: [d] of `dtype`, Qt = Q^T: [d x d] of `dtype`, x_rot: [d] fp32,
 * idx: [K] int32 ascending, val: [K] fp32.  One kernel: every CTA computes a
 * share of x_rot and the last one to finish selects.  d a multiple of 8;
 * x, Qt and x_rot 16-byte aligned.  ws: at least
 * larosa_workspace_bytes(1, d, 1, K) bytes; it holds a counter that is zero
 * between calls, so calls sharing a workspace must not overlap.  A NaN or
 * Inf in x_rot sets LAROSA_DEV_NONFINITE.
 */
int larosa_rotate_topk(const void *x, const void *Qt, float *x_rot,
                       int32_t *idx, float *val, int d, int K, void *ws,
                       size_t ws_bytes, int *dev_status, int dtype,
                       larosa_stream_t stream);

/*
 * Sparse linear (step 3): y[m][j] = sum_k val[m][k] * W_rot[idx[m][k]][j].
 * idx/val: [M x K] as written by larosa_topk (each row's indices distinct;
 * ascending order is not required for correctness).  W_rot: [d_in x d_out]
 * of `dtype`; only the rows named in idx are read.  y: [M x d_out] fp32.
 * For M > 1 the rows named by any token are streamed once and shared; with
 * bf16 weights every row is, as a dense tensor-core product with each
 * token's coefficient row (zero at the rows it did not keep), since the
 * tokens' kept rows cover most rows (84 % at two tokens and 40 % sparsity,
 * nearly all from four on) -- except where two to four tokens keep so few
 * rows that streaming only their union is faster (an expected union below
 * 30 % of the rows for two tokens, 20 % for three or four).
 * An index outside [0, d_in) sets LAROSA_DEV_INDEX and contributes nothing.
 * ws: at least larosa_workspace_bytes(M, d_in, d_out, K) bytes.
 */
int larosa_sparse_linear(const int32_t *idx, const float *val, int M, int K,
                         const void *W_rot, int d_in, int d_out, float *y,
                         void *ws, size_t ws_bytes, int dtype,
                         int *dev_status, larosa_stream_t stream);

/*
 * Steps 1-3 in one call, one stream, no host synchronisation:
 *   x_rot = x . Q;  (idx, val) = TopK(x_rot, K);  y = sparse(x_rot) . W_rot.
 * x: [M x d_in] of `dtype`; Qt = Q^T: [d_in x d_in]; W_rot: [d_in x d_out] of
 * `dtype` (from larosa_prepare_weights with the same Qt); y: [M x d_out] fp32.
 * Qt = NULL selects the identity rotation (x_rot = x widened to fp32, W_rot
 * the plain weight): the unrotated fixed-K mode, for comparison with the
 * magnitude-pruning methods the La RoSA abstract compares against (TEAL,
 * CATS).  For one token this is one cooperative kernel: every CTA rotates a share
 * of x, a selector CTA finds the K-th entry, and the rest stream the kept
 * rows of W_rot by column tiles (when the grid cannot be made resident it
 * falls back to larosa_rotate_topk's kernel followed by the one-token
 * gather).  That kernel is launched as a programmatic dependent of the
 * previous kernel on the stream: before the previous kernel has finished it
 * only asks for its first rows of Qt to be brought into L2, a hint that does
 * not change what is read later.  For M > 1 the steps run as
 * separate kernels.  The intermediate x_rot, idx and val live in the
 * workspace at the offsets larosa_workspace_layout() gives (the kept list
 * in ascending index order).  d_in a multiple of 8; x, Qt, W_rot and y
 * 16-byte aligned.  ws: at least larosa_workspace_bytes(M, d_in, d_out, K)
 * bytes; for M = 1 it holds counters that are zero between calls, so calls
 * sharing a workspace must not overlap.
 */
int larosa_rotate_topk_linear(const void *x, const void *Qt, const void *W_rot,
                              int M, int d_in, int d_out, int K, float *y,
                              void *ws, size_t ws_bytes, int *dev_status,
                              int dtype, larosa_stream_t stream);

/*
 * Steps 2 and 3 for a vector that is already rotated (La RoSA summary,
 * 方法详解 / 技术框架: keep the K largest magnitudes of each rotated
 * activation vector, then multiply by the counter-rotated weight):
 *   (idx, val) = TopK(x_rot, K) with larosa_topk's rule;
 *   y = sum_k val[k] * W_rot[idx[k]].
 * x_rot: [M x d_in] fp32 (as larosa_rotate writes it, or the output of a
 * producer whose weight was counter-rotated with larosa_fold_rotation);
 * W_rot: [d_in x d_out] of `dtype`; y: [M x d_out] fp32.  larosa_topk's
 * kernel, then the sparse linear on its kept lists (from 2 bf16 tokens on,
 * the Top-K kernel also writes the coefficient rows of the tensor-core
 * product, as in larosa_rotate_topk_linear).  The kept list
 * (ascending) lies in the workspace at the offsets larosa_workspace_layout
 * gives.  x_rot, W_rot and y 16-byte aligned, d_out rows of 16 bytes.
 * ws: at least larosa_workspace_bytes(M, d_in, d_out, K) bytes.  A NaN or
 * Inf in x_rot sets LAROSA_DEV_NONFINITE.
 */
int larosa_topk_linear(const float *x_rot, const void *W_rot, int M, int d_in,
                       int d_out, int K, float *y, void *ws, size_t ws_bytes,
                       int *dev_status, int dtype, larosa_stream_t stream);

/*
 * Threshold selection (R-Sparse report, 研究流程与方法 / R-Sparse框架设计: the
 * input channels with |x_j| >= t are kept, the rest masked; the count kept
 * varies from token to token):
 *   nnz[m] = |S_m|,  S_m = { i : |x_rot[m][i]| >= t }.
 * x_rot: [M x d] fp32.  idx/val: [M x d]; row m's first nnz[m] entries
 * receive S_m in ascending index order and the kept values, the rest of the
 * row is left as it was.  nnz: [M] int32.  Magnitudes are compared exactly
 * (+0 and -0 are equal); t <= 0 keeps every entry, t = +Inf only infinite
 * ones; t = NaN returns LAROSA_ERR_INVALID_ARG.  A NaN or Inf in x_rot sets
 * LAROSA_DEV_NONFINITE.  One CTA per token.
 */
int larosa_threshold(const float *x_rot, int M, int d, float t, int32_t *idx,
                     float *val, int32_t *nnz, int *dev_status,
                     larosa_stream_t stream);

/*
 * Rotation, threshold selection and sparse linear in one call (the
 * threshold function sigma_t of the R-Sparse report in place of the Top-K):
 *   x_rot = x . Q;  S_m = { i : |x_rot[m][i]| >= t };
 *   y[m] = sum_{i in S_m} x_rot[m][i] * W_rot[i].
 * Arguments as for larosa_rotate_topk_linear, with t in place of K (Qt =
 * NULL again selects the identity rotation, the TEAL/CATS-style mode).  For
 * one token one cooperative kernel as for the Top-K (no selection step: the
 * gather CTAs stream their kept rows as soon as every CTA has rotated);
 * otherwise rotation, larosa_threshold's kernel and the sparse linear: for
 * several bf16 tokens the dense tensor-core product with the coefficient
 * rows the threshold kernel writes (every row of W_rot is streamed, since the
 * kept share is known only on the device), else the row-streaming sparse
 * linear over the kept rows (for M > 1 over the union of the tokens' sets).
 * ws: at least larosa_workspace_bytes(M, d_in, d_out, d_in) bytes; x_rot,
 * idx and val ([M x d_in] each, as larosa_threshold writes them) lie at the
 * offsets larosa_workspace_layout(M, d_in, d_out, d_in, ...) gives and nnz
 * at larosa_workspace_nnz_offset(M, d_in, d_out, d_in, ...).
 */
int larosa_rotate_threshold_linear(const void *x, const void *Qt,
                                   const void *W_rot, int M, int d_in,
                                   int d_out, float t, float *y, void *ws,
                                   size_t ws_bytes, int *dev_status, int dtype,
                                   larosa_stream_t stream);

/*
 * Sparse + low-rank linear (R-Sparse report, 研究流程与方法 / R-Sparse框架设计,
 * hybrid computation): the entries a selection drops are sent through
 * rank-r factors of the weight instead of being discarded:
 *   y[m] = sum_k val[m][k] * W[idx[m][k]]  +  ((x[m] - sigma(x[m])) . A_r) . B_r,
 * where sigma(x[m]) is x[m] with every entry outside idx[m] set to zero.
 * x: [M x d_in] fp32, the vector the selection was made on (x_rot for the
 * rotated path; idx/val then come from larosa_topk or larosa_threshold on
 * it, val = x at idx).  W: [d_in x d_out], A_r: [d_in x r], B_r: [r x d_out],
 * all of `dtype` (the factors of an offline SVD W ~ U S V^T: A_r = U_r
 * S_r^1/2, B_r = S_r^1/2 V_r^T); y: [M x d_out] fp32.  d_out and r rows of
 * 16 bytes; x, W, A_r, B_r, y 16-byte aligned.  One token (r <= 2048):
 * one cooperative kernel, in which column-tile CTAs stream the kept rows of
 * W while factor CTAs, each over a range of x, compute partials of
 * u = dropped . A_r (reading only the dropped rows of A_r), then the
 * column-tile CTAs add the partials of their entries of u and stream the
 * rows of B_r with those coefficients into the same sums.  Otherwise: the
 * sparse linear on the kept list, then u = dropped . A_r and y_r = u . B_r
 * -- for bf16 with 64 <= r <= d_in as tensor-core products fed with the
 * dropped part's and u's bf16 head/tail coefficient rows, else by the
 * row-streaming GEMV with fp32 coefficients -- and y += y_r.  The workspace must be zero-filled before its first use (the
 * one-token kernel keeps counters there, zero again after every call).
 * ws: at least larosa_lowrank_workspace_bytes(M, d_in, d_out, K, r) bytes.
 */
int larosa_sparse_lowrank_linear(const float *x, const int32_t *idx,
                                 const float *val, int M, int K, const void *W,
                                 const void *A_r, const void *B_r, int d_in,
                                 int d_out, int r, float *y, void *ws,
                                 size_t ws_bytes, int dtype, int *dev_status,
                                 larosa_stream_t stream);

/* Workspace bytes of larosa_sparse_lowrank_linear (0 for out-of-range sizes). */
size_t larosa_lowrank_workspace_bytes(int M, int d_in, int d_out, int K, int r);

/*
 * Dense baseline: y[m][j] = sum_i x[m][i] * Wt[j][i], i.e. y = x . W for the
 * dense layer, with the weight in torch.nn.Linear layout Wt = W^T
 * [d_out x d_in] (each output a dot product with one contiguous row), by the
 * same streaming machinery as the rotation (no cuBLAS).  x: [M x d_in] of
 * `dtype`, y: [M x d_out] fp32.  d_in a multiple of 8; x and Wt 16-byte
 * aligned.  Uses no workspace.
 */
int larosa_dense_linear(const void *x, const void *Wt, int M, int d_in,
                        int d_out, float *y, int dtype,
                        larosa_stream_t stream);

/*
 * larosa_sparse_linear without a workspace, for callers that cannot allocate
 * device memory where they call the library: an operator slot in another
 * runtime that passes only inputs and outputs, or a latency-critical loop in
 * which cudaMalloc/cudaFree (which may synchronise the device) are not
 * allowed.  The LaRoSA pages have no counterpart: this is a deployment
 * variant of step 3, computing the same y with the same kernels.
 *
 * Arguments as for larosa_sparse_linear, minus ws/ws_bytes.  One token
 * needs no scratch when the cluster gather fits the GPU (its partial sums
 * stay in distributed shared memory; on B200 that holds for every accepted
 * size); otherwise, and for several tokens, the split-K partials and row
 * bookkeeping live in a file-scope device array of
 * LAROSA_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds
 * until the process exits.  larosa_sparse_linear_noalloc_bytes() gives the
 * scratch a size needs.  Sizes whose scratch would exceed the array (in
 * practice only large multi-token batches, e.g. 16 fp32 tokens with
 * d_in = 32768) return LAROSA_ERR_WORKSPACE with the byte counts in
 * larosa_last_error_string().  The call allocates nothing; it clears the
 * words that must start at zero with cudaMemsetAsync on `stream`.  All calls
 * on one device share the array, so calls that may overlap on that GPU race:
 * serialise them.  The first call on each device looks up the array's device
 * address and sizes its kernels (host-side CUDA queries); make that first
 * call before any stream capture.
 */
int larosa_sparse_linear_noalloc(const int32_t *idx, const float *val, int M,
                                 int K, const void *W_rot, int d_in, int d_out,
                                 float *y, int dtype, int *dev_status,
                                 larosa_stream_t stream);

/* Size of the file-scope scratch array behind larosa_sparse_linear_noalloc. */
#define LAROSA_NOALLOC_SCRATCH_BYTES (2u << 20)

/*
 * Bytes of that array larosa_sparse_linear_noalloc would use for these sizes
 * on the current device (0: none, the one-token cluster gather).  A result
 * above LAROSA_NOALLOC_SCRATCH_BYTES means the call would be refused with
 * LAROSA_ERR_WORKSPACE.  Allocates and launches nothing (host-side device
 * queries only).  Returns 0 for out-of-range sizes or an unknown dtype too.
 */
size_t larosa_sparse_linear_noalloc_bytes(int M, int d_in, int d_out, int K,
                                          int dtype);

/*
 * Workspace bytes sufficient for every entry point above called with these
 * sizes (M tokens, d_in inputs, d_out outputs, K kept).  Returns 0 for
 * out-of-range sizes.
 */
size_t larosa_workspace_bytes(int M, int d_in, int d_out, int K);

/*
 * Byte offsets inside the workspace of the fused call's intermediates:
 * x_rot ([M x d_in] fp32), idx ([M x K] int32) and val ([M x K] fp32).
 * Any output pointer may be NULL.  Returns LAROSA_ERR_SHAPE for
 * out-of-range sizes.
 */
int larosa_workspace_layout(int M, int d_in, int d_out, int K,
                            size_t *x_rot_offset, size_t *idx_offset,
                            size_t *val_offset);

/*
 * Byte offset inside the workspace of the threshold call's kept counts
 * (nnz, [M] int32).  Returns LAROSA_ERR_SHAPE for out-of-range sizes.
 */
int larosa_workspace_nnz_offset(int M, int d_in, int d_out, int K,
                                size_t *nnz_offset);

/*
 * Byte offset inside the workspace of the one-token fused call's
 * synchronisation block (M = 1 only; LAROSA_ERR_SHAPE otherwise).  Its
 * 32-bit words: [0] and [1] count the arrivals of even and odd calls, [3]
 * is the number of the last call whose selection was published, [4] and
 * [5] (one 64-bit word) the K-th entry it published with the call's 16-bit
 * tag; then the per-tile completion counters and
 * the magnitude histograms of the two call parities.  A caller never needs
 * to touch it (it is zero between calls); it is exposed for diagnosis and
 * for tests of the bounded waits: a call whose arrival counter does not
 * start at zero can never see its exact count and gives up after the wait
 * limit with LAROSA_DEV_TIMEOUT.
 */
int larosa_workspace_sync_offset(int M, int d_in, int d_out, int K,
                                 size_t *sync_offset);

/* Range accepted by larosa_set_wait_limit_ns (besides 0). */
#define LAROSA_MIN_WAIT_LIMIT_NS 1000ull
#define LAROSA_MAX_WAIT_LIMIT_NS 60000000000ull

/*
 * Sets the time after which every wait inside a kernel gives up (reporting
 * LAROSA_DEV_TIMEOUT), for launches enqueued after this call; work already
 * enqueued or captured in a CUDA graph keeps the limit it was launched
 * with.  limit_ns = 0 restores the default (2 s); otherwise it must lie in
 * [LAROSA_MIN_WAIT_LIMIT_NS, LAROSA_MAX_WAIT_LIMIT_NS], else
 * LAROSA_ERR_INVALID_ARG and nothing changes.  Process-wide; `previous`
 * (host, may be NULL) receives the limit in force before the call.
 */
int larosa_set_wait_limit_ns(uint64_t limit_ns, uint64_t *previous);

/*
 * Debug checks (off unless the environment variable LAROSA_DEBUG is set to
 * a nonzero integer when the library is first used, or this call turns them
 * on).  While on, every call that takes or writes kept lists also launches
 * a check of them on the same stream, after (for lists the library writes:
 * larosa_topk, larosa_rotate_topk, larosa_rotate_topk_linear,
 * larosa_topk_linear) or before (for the caller's lists: larosa_sparse_linear,
 * larosa_sparse_linear_noalloc, larosa_sparse_lowrank_linear) the compute:
 * each row's indices must lie in [0, d_in) (else LAROSA_DEV_INDEX), be
 * distinct and, where the library wrote them, ascending (else
 * LAROSA_DEV_LIST), and the values finite (else LAROSA_DEV_NONFINITE).
 * Results are unchanged; the check costs one small launch per call and
 * reports only where dev_status is not NULL.  on = 0 turns them off, 1 on;
 * anything else is LAROSA_ERR_INVALID_ARG.  Process-wide; `previous` (host,
 * may be NULL) receives the setting in force before the call.
 */
int larosa_set_debug(int on, int *previous);

/* Largest split count larosa_set_split_k accepts. */
#define LAROSA_MAX_SPLIT_K 8

/*
 * Split of the reduction in the tensor-core kernels of 2 to 16 bf16 tokens
 * (the rotation, the dense product and the sparse linear): splits = 0 lets
 * the library choose (a wave model over the SMs, the default, also chosen
 * by the environment variable LAROSA_SPLIT_K when the library is first
 * used), 1 ... LAROSA_MAX_SPLIT_K forces that many CTAs per output tile
 * (fewer where the reduction has fewer 64- or 128-input chunks).  The splits
 * of a tile form a thread-block cluster and add their partials in rank
 * order, so a fixed split gives results that repeat bit for bit; different
 * splits round differently (each within the fp32 summation bound).  Other
 * values are LAROSA_ERR_INVALID_ARG.  Process-wide, for calls made after
 * it; `previous` (host, may be NULL) receives the setting before the call.
 */
int larosa_set_split_k(int splits, int *previous);

/*
 * Waits for `stream`, reads *dev_status (device pointer) and returns
 * LAROSA_OK when it is zero, else the status of its lowest set bit
 * (NONFINITE, TIMEOUT, INDEX, LIST).  If `flags_out` (host) is not NULL it
 * receives the raw bits.  Does not clear the word.
 */
int larosa_check(const int *dev_status, larosa_stream_t stream, int *flags_out);

#ifdef __cplusplus
}
#endif

#endif /* LAROSA_H */
