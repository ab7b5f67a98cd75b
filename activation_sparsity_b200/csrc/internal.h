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

// Top-K: one 1024-thread CTA per token.
cudaError_t launch_topk(const float* x_rot, int M, int d, int K, int32_t* idx, float* val,
                        int* dev_status, cudaStream_t stream);

// M > 1: scatter each token's (idx, val) into a dense zero-filled coefficient
// row and mark the rows used by any token in `bitmap` (d_in bits).
cudaError_t launch_scatter(const int32_t* idx, const float* val, int M, int K, int d_in,
                           float* coef, unsigned* bitmap, int* dev_status, cudaStream_t stream);

// M > 1: compacts the bitmap into the ascending union list `rows` and its
// count, then clears the bitmap.
cudaError_t launch_union(unsigned* bitmap, int d_in, int32_t* rows, int* count,
                         cudaStream_t stream);

// W_rot = Q^T W.
cudaError_t launch_prepare(const void* Q, const void* W, void* W_rot, int d_in, int d_out,
                           Elem elem, cudaStream_t stream);

}  // namespace larosa
