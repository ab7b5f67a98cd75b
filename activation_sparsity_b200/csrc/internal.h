// Host-side interfaces between the C-ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace larosa {

// Geometry of one launch of the row-streaming GEMV (see rowstream.cu).
struct GemvPlan {
  int col_tile = 0;        // Wc: output columns per CTA
  int tpr = 0;             // consumer threads per weight row (Wc / columns per thread)
  int rows_per_stage = 0;  // weight rows per pipeline stage
  int pitch = 0;           // bytes between two weight rows of a stage
  int n_col_tiles = 0;     // ceil(d_out / Wc)
  int splits = 0;          // CTAs along the row dimension (a multiple of cluster)
  int cluster = 1;         // CTAs per thread-block cluster (along the splits)
  int max_rows_per_cta = 0;
  size_t smem_bytes = 0;
  // scratch needed in the workspace
  size_t partial_floats = 0;  // n_col_tiles * (splits / cluster) * M * Wc (0 if one cluster per tile)
  size_t ticket_words = 0;    // n_col_tiles * cluster (0 if one cluster per tile)
};

enum class Elem { F32 = 0, BF16 = 1 };

// Arguments of one row-streaming GEMV:
//   y[m][c] = sum_r coef(m, r) * W[row(r)][c],  r in [0, n_rows)
// row(r) = rows[r] (gather) or r (dense); coef(m, r) = coef[m*coef_ld + (coef_by_row ? row(r) : r)].
struct GemvArgs {
  const void* W = nullptr;
  Elem w_elem = Elem::BF16;
  int d_out = 0;
  int row_bound = 0;
  const int32_t* rows = nullptr;
  int n_rows = 0;
  const int* n_rows_dev = nullptr;
  const void* coef = nullptr;
  Elem coef_elem = Elem::F32;
  int coef_ld = 0;
  int coef_by_row = 0;
  int M = 1;
  float* y = nullptr;
  int y_ld = 0;
  float* partials = nullptr;
  unsigned* tickets = nullptr;
  int* dev_status = nullptr;
};

// Plans a launch for the current device.  Returns cudaSuccess or the error of
// the device query.
cudaError_t plan_gemv(Elem w_elem, Elem coef_elem, int M, int d_out, int n_rows_max, GemvPlan* plan);

// Enqueues the GEMV with programmatic dependent launch on `stream`.
cudaError_t launch_gemv(const GemvArgs& a, const GemvPlan& plan, cudaStream_t stream);

// Top-K: one 1024-thread CTA per token.  With hl != nullptr (d a multiple of
// 8) it also writes the tokens' dense coefficient rows as bf16 head and tail
// for the tensor-core sparse linear: hl[m][0, d) heads, hl[M + m][0, d) tails.
cudaError_t launch_topk(const float* x_rot, int M, int d, int K, int32_t* idx, float* val,
                        int* dev_status, cudaStream_t stream, __nv_bfloat16* hl = nullptr);

// The same dense head/tail coefficient rows from given kept lists (idx/val
// [M x K], indices distinct within a row): one CTA per token.
// Debug checks (debug.cu): each of the M rows of idx/val ([M x K]) has
// distinct indices in [0, d), ascending where `ascending`, and finite values;
// violations set LAROSA_DEV_INDEX, LAROSA_DEV_LIST or LAROSA_DEV_NONFINITE.
// Launches nothing when dev_status is NULL or there is no entry.
cudaError_t launch_check_lists(const int32_t* idx, const float* val, int M, int K, int d, bool ascending,
                               int* dev_status, cudaStream_t stream);
// Process-wide settings (api.cu): the debug checks, and the forced split
// count of the tensor-core kernels of several tokens (0: chosen per shape).
bool debug_checks();
int split_k_override();

cudaError_t launch_coef_rows(const int32_t* idx, const float* val, int M, int K, int d, __nv_bfloat16* hl,
                             int* dev_status, cudaStream_t stream);

// Threshold selection: one 1024-thread CTA per token keeps |x_rot| >= t
// (t_key: bit pattern of t, 0 for t <= 0), writes the kept (idx, val) in
// ascending order into rows of length d and the count to nnz[m]; with coef
// != nullptr also the coefficient row (x where kept, else 0) and the bitmap
// of kept rows, as launch_scatter does.
cudaError_t launch_threshold(const float* x_rot, int M, int d, uint32_t t_key, int32_t* idx,
                             float* val, int32_t* nnz, float* coef, unsigned* bitmap,
                             int* dev_status, cudaStream_t stream, __nv_bfloat16* hl = nullptr);

// Low-rank compensation: x_drop = x with each token's kept entries zeroed;
// y += add (n elements).
cudaError_t launch_dropped(const float* x, const int32_t* idx, int M, int K, int d, float* x_drop,
                           int* dev_status, cudaStream_t stream);
// The dropped part's bf16 head and tail coefficient rows, hl [2 x M x d]
// (x with idx's K kept entries of each token zeroed; K = 0: x itself), for
// the tensor-core factor products.  d a multiple of 8.
cudaError_t launch_dropped_rows(const float* x, const int32_t* idx, int M, int K, int d, __nv_bfloat16* hl,
                                int* dev_status, cudaStream_t stream);
cudaError_t launch_add(float* y, const float* add, int n, cudaStream_t stream);

// x_rot[i] = x[i] widened to fp32 (the identity rotation), n elements.
cudaError_t launch_widen(const void* x, float* x_rot, int n, Elem elem, cudaStream_t stream);

// M > 1: scatter each token's (idx, val) into a dense zero-filled coefficient
// row and mark the rows used by any token in `bitmap` (d_in bits).
cudaError_t launch_scatter(const int32_t* idx, const float* val, int M, int K, int d_in,
                           float* coef, unsigned* bitmap, int* dev_status, cudaStream_t stream);

// M > 1: compacts the bitmap into the ascending union list `rows` and its
// count, then clears the bitmap.
cudaError_t launch_union(unsigned* bitmap, int d_in, int32_t* rows, int* count,
                         cudaStream_t stream);

// Geometry of the one-token gather (see onetoken.cu): `cluster` CTAs per
// column tile of `col_tile` columns (a thread-block cluster in the list-mode
// gather; plain CTAs in the fused kernel).
struct StreamPlan {
  bool ok = false;
  int cluster = 0;
  int n_tiles = 0;
  int col_tile = 0;
  int tpr = 0;             // threads per weight row
  int list_cap = 0;        // kept entries per CTA
  size_t smem = 0;         // dynamic shared memory of a launch
  size_t smem_alloc = 0;   // the size the occupancy was computed for
  size_t partial_floats = 0;  // workspace floats for per-CTA partials (fused kernel)
  int aux_ctas = 0;        // low-rank kernel: factor CTAs
  int aux_len = 0;         // low-rank kernel: indices of x per factor CTA at most
};

struct GatherArgs {
  const void* W = nullptr;  // [d_in x d_out] row-major
  int d_out = 0;
  int row_bound = 0;        // d_in
  int n = 0;                // list length K
  const void* coef = nullptr;     // val[K]
  const int32_t* rows = nullptr;  // idx[K]
  float* y = nullptr;
  int* dev_status = nullptr;
};

// Plans a one-token gather of K kept rows (indices idx[], coefficients val[])
// of a row-major [* x d_out] weight; plan->ok is false when it does not fit.
cudaError_t plan_gather(Elem w_elem, int d_out, int K, StreamPlan* plan);
cudaError_t launch_gather(Elem w_elem, const GatherArgs& a, const StreamPlan& plan,
                          cudaStream_t stream);

// Row-dot GEMV y[m][j] = sum_i x[m][i] A[j][i] for M <= 16 tokens, A row-major
// [n_out x n_in] (the rotation through Q^T, or a dense layer in
// torch.nn.Linear layout).  n_in a multiple of 8; x and A 16-byte aligned.
cudaError_t launch_rowdot(Elem e, const void* A, const void* x, float* y, int M, int n_in,
                          int n_out, cudaStream_t stream);

// The same row-dot product for 2 to 16 bf16 tokens on tcgen05 (TMEM
// accumulator, TMA-fed shared-memory operands); rot_umma_applies tells
// whether the shapes suit it (n_in a multiple of 64).
bool rot_umma_applies(int M, int n_in, int n_out);
cudaError_t launch_rot_umma(const void* A, const void* x, float* y, int M, int n_in, int n_out,
                            int* dev_status, cudaStream_t stream);

// The sparse linear of 2 to 16 tokens as a dense tensor-core product over
// every row of W (bf16) with the per-token coefficient rows (zero where a
// token did not keep the row), given as bf16 head and tail hl [2 x M x d_in]
// (launch_topk or launch_coef_rows): y = (head + tail) . W on tcgen05.
bool umma_gemv_applies(int M, int d_in, int d_out);
// Whether the dense product pays for M tokens keeping K of d_in rows each:
// umma_gemv_applies, unless few tokens keep so few rows that streaming only
// their union (expected share 1 - (1 - K / d_in)^M for independent
// selections: below 0.3 for 2 tokens, 0.2 for 3-4) is faster.
bool umma_gemv_pays(int M, int d_in, int d_out, int K);
// accumulate: y += the product; hl_out (not null): the product written as
// bf16 head/tail rows [2 x M x d_out] (the next product's coefficients)
// instead of y.
cudaError_t launch_umma_gemv(const void* W, const __nv_bfloat16* hl, float* y, int M, int d_in, int d_out,
                             int* dev_status, cudaStream_t stream, bool accumulate = false,
                             __nv_bfloat16* hl_out = nullptr);

// One token: x_rot = x . Q (through Qt = Q^T), then the last CTA to finish
// writes the kept list (idx, val: the K largest |x_rot|, ties to the lower
// index, ascending) for a list-mode gather launched right after it.
// `ticket` must be zero before the call and is zero again after it.
struct RotSelArgs {
  const void* x = nullptr;
  const void* Qt = nullptr;
  float* x_rot = nullptr;
  int32_t* idx = nullptr;
  float* val = nullptr;
  unsigned* ticket = nullptr;
  int d = 0;
  int K = 0;
  int* dev_status = nullptr;
};

// True when d is a multiple of 8 and the selection fits in shared memory.
bool rotsel_fits(Elem e, int d);
cudaError_t launch_rotsel(Elem e, const RotSelArgs& a, cudaStream_t stream);

// One token, one cooperative launch: rotation, Top-K by a selector CTA, and
// the gather of the kept rows (onetoken.cu, fused_kernel).  `sync` points to
// kFusedSyncBytes of the caller's workspace, zero before the first call and
// kept consistent by every call after it; calls that share it must not
// overlap on the GPU.
constexpr int kFusedSyncWords = 8;
constexpr int kFusedMaxTiles = 512;
constexpr int kFusedHistBins = 4096;  // bits 30..19 of |x_rot|
constexpr size_t kFusedSyncBytes =
    (kFusedSyncWords + 2 * kFusedMaxTiles + 2 * kFusedHistBins) * 4;
struct FusedArgs {
  const void* x = nullptr;
  const void* Qt = nullptr;
  const void* W = nullptr;
  float* x_rot = nullptr;
  int32_t* idx = nullptr;
  float* val = nullptr;
  float* y = nullptr;
  float* partials = nullptr;  // plan.partial_floats floats of workspace
  unsigned* sync = nullptr;
  int d_in = 0;
  int d_out = 0;
  int K = 0;
  int* dev_status = nullptr;
  bool threshold = false;  // keep |x_rot| >= t (t_key) instead of the Top-K
  uint32_t t_key = 0;
  int32_t* nnz = nullptr;  // threshold mode: the kept count
};
// With Qt == nullptr the rotation is the identity (x_rot = x widened).

// plan->ok is false when the shape does not fit (then use the two-kernel path).
cudaError_t plan_fused(Elem w_elem, int d_in, int d_out, int K, StreamPlan* plan);
cudaError_t launch_fused(Elem w_elem, const FusedArgs& a, const StreamPlan& plan,
                         cudaStream_t stream);

// Sparse + low rank for one token in one cooperative launch (onetoken.cu,
// lowrank_kernel): y = sum_k val[k] W[idx[k]] + ((x - sigma(x)) . A_r) . B_r,
// x fp32 [d_in], sigma(x) the kept entries of x.  Workspace: u (r floats),
// partials (plan.partial_floats floats) and sync (2 + n_tiles words, zero
// between calls).  plan->ok is false when the shape does not fit (d_in >
// 16384, r > 2048, or the grid cannot be resident).
struct LowrankArgs {
  const float* x = nullptr;
  const int32_t* idx = nullptr;
  const float* val = nullptr;
  const void* W = nullptr;
  const void* A_r = nullptr;
  const void* B_r = nullptr;
  float* y = nullptr;
  float* u = nullptr;
  float* partials = nullptr;
  unsigned* sync = nullptr;
  int d_in = 0;
  int d_out = 0;
  int K = 0;
  int r = 0;
  int* dev_status = nullptr;
};
// u of the one-launch kernel: the factor CTAs' partials, [aux_ctas x r]
// floats; at most kLowrankMaxFactorCtas x r.
constexpr int kLowrankMaxFactorCtas = 64;
cudaError_t plan_lowrank(Elem w_elem, int d_in, int d_out, int K, int r, StreamPlan* plan);
cudaError_t launch_lowrank(Elem w_elem, const LowrankArgs& a, const StreamPlan& plan, cudaStream_t stream);

// W_rot = Qt . W with Qt = Q^T given row-major.
cudaError_t launch_prepare(const void* Q, const void* W, void* W_rot, int d_in, int d_out,
                           Elem elem, cudaStream_t stream);

}  // namespace larosa
