// C ABI of the library: argument validation, workspace layout and the
// sequencing of kernels for each entry point (see include/larosa.h).
//
//   rotation, dense baseline   rowdot (onetoken.cu) for one token; umma_kernel
//                              (rot_umma.cu, tcgen05) for 2-16 bf16 tokens
//   Top-K alone                topk_kernel (topk.cu)
//   sparse linear, M = 1       cluster gather over idx/val (onetoken.cu)
//   sparse linear, M > 1       bf16: coefficient rows (topk.cu) + the tcgen05
//                              product over every row, unless 2-4 tokens keep
//                              few rows; else scatter + union (union.cu) +
//                              rowstream (rowstream.cu)
//   rotation + Top-K, M = 1    rotsel (onetoken.cu): its last CTA selects
//   fused, M = 1               fused_kernel (onetoken.cu): one cooperative launch;
//                              where it does not fit, rotsel -> list gather
//   fused, M > 1               rotation -> topk (writing the coefficient rows
//                              where the tcgen05 product is taken) -> sparse linear
//   threshold, M = 1           fused_kernel in threshold mode; where it does not
//                              fit, rowdot -> threshold -> rowstream over the list
//   threshold, M > 1           rotation -> threshold (bf16: writes the coefficient
//                              rows for the tcgen05 product; else the coefficient
//                              rows and the bitmap) -> union -> rowstream
//   no Qt (identity rotation)  as above with widen in place of the rotation
//   sparse + low rank          one token: lowrank_kernel (onetoken.cu), one
//                              launch; several: the sparse linear, then the two
//                              factor products (bf16: coefficient rows from
//                              lowrank.cu and tcgen05; else the dropped part and
//                              row-streaming GEMVs), y += y_r
//   debug checks               check_lists_kernel (debug.cu) around the calls
//                              that take or write kept lists, when enabled
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "internal.h"

using larosa::Elem;
using larosa::GemvArgs;
using larosa::GemvPlan;

namespace {

constexpr int kMaxDout = 65536;
constexpr size_t kTicketWords = 2048;
// The last ticket word belongs to the one-token rotate + select kernel; the
// multi-token split-K tickets use the words below it.
constexpr size_t kSplitKTicketWords = kTicketWords - 1;
constexpr size_t kRotSelTicket = kTicketWords - 1;
constexpr size_t kBitmapWords = LAROSA_MAX_D / 32;
// Fixed header, at the same offsets in the layout of every size, so that
// calls of different sizes may share one workspace: words that must be zero
// before a call and are zero after it, then the one-token fused kernel's
// synchronisation block, whose call number and alternating counters persist
// from one call to the next (a call of another size that laid its own
// intermediates over them would leave the next one-token call a counter that
// can never reach its count).
constexpr size_t kOffTickets = 0;
constexpr size_t kOffBitmap = kOffTickets + kTicketWords * 4;
constexpr size_t kOffFusedSync = (kOffBitmap + kBitmapWords * 4 + 255) / 256 * 256;
constexpr size_t kHeaderEnd = kOffFusedSync + larosa::kFusedSyncBytes;

thread_local char g_last_error[256] = "";

int cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
  return LAROSA_ERR_CUDA;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(int dtype) { return dtype == LAROSA_BF16 ? 2 : 4; }

Elem elem_of(int dtype) { return dtype == LAROSA_BF16 ? Elem::BF16 : Elem::F32; }

bool valid_dtype(int dtype) { return dtype == LAROSA_BF16 || dtype == LAROSA_F32; }

// Row length (elements) of a row-major weight is a multiple of 16 bytes.
bool row_aligned(int n, int dtype) { return (n * elem_size(dtype)) % 16 == 0; }

struct Layout {
  size_t fused_sync = 0;  // the fused kernel's synchronisation block (M = 1; in the fixed header)
  size_t x_rot = 0, idx = 0, val = 0, nnz = 0;
  size_t partials = 0;
  size_t coef = 0, urows = 0, ucount = 0;
  size_t coef_hl = 0;  // M > 1: the coefficients' bf16 head and tail for the tensor-core GEMV
  size_t total = 0;
  bool list_gemv = false;  // M = 1: the row-streaming GEMV over a list of up to d_in rows fits
};

int sparse_rows_max(int M, int d_in, int K) {
  return M == 1 ? K : (int)std::min<long long>(d_in, (long long)M * K);
}

int make_layout_uncached(int M, int d_in, int d_out, int K, Layout* L);

// Layouts already computed, per device and sizes.
struct LayoutEntry {
  int dev, M, d_in, d_out, K;
  Layout L;
};
std::mutex g_layout_mu;
LayoutEntry g_layouts[256];
int g_layout_n = 0;
int g_layout_next = 0;

// One workspace layout serves every entry point called with these sizes.
int make_layout(int M, int d_in, int d_out, int K, Layout* L) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  {
    std::lock_guard<std::mutex> lock(g_layout_mu);
    for (int i = 0; i < g_layout_n; ++i) {
      const LayoutEntry& en = g_layouts[i];
      if (en.dev == dev && en.M == M && en.d_in == d_in && en.d_out == d_out && en.K == K) {
        *L = en.L;
        return LAROSA_OK;
      }
    }
  }
  const int st = make_layout_uncached(M, d_in, d_out, K, L);
  if (st != LAROSA_OK) return st;
  std::lock_guard<std::mutex> lock(g_layout_mu);
  LayoutEntry& en = g_layouts[g_layout_n < 256 ? g_layout_n++ : (g_layout_next++ & 255)];
  en = LayoutEntry{dev, M, d_in, d_out, K, *L};
  return LAROSA_OK;
}

int make_layout_uncached(int M, int d_in, int d_out, int K, Layout* L) {
  size_t partials = 0;
  L->list_gemv = M == 1;
  for (int dt = 0; dt < 2; ++dt) {
    const Elem w = dt == 0 ? Elem::F32 : Elem::BF16;
    if (M == 1) {
      larosa::StreamPlan sl, sf;
      cudaError_t e = larosa::plan_gather(w, d_out, K, &sl);
      if (e == cudaSuccess) e = larosa::plan_fused(w, d_in, d_out, K, &sf);
      if (e != cudaSuccess) return cuda_fail(e, "plan gather");
      if (sf.ok) partials = std::max(partials, sf.partial_floats);
      // the threshold path's fallback streams a list of up to d_in rows
      GemvPlan pt;
      e = larosa::plan_gemv(w, Elem::F32, 1, d_out, d_in, &pt);
      if (e != cudaSuccess) return cuda_fail(e, "plan sparse linear");
      if (pt.ticket_words <= kSplitKTicketWords)
        partials = std::max(partials, pt.partial_floats);
      else
        L->list_gemv = false;
      if (sl.ok) continue;  // the list-mode gather needs no partials
    }
    GemvPlan ps;
    cudaError_t e = larosa::plan_gemv(w, Elem::F32, M, d_out, sparse_rows_max(M, d_in, K), &ps);
    if (e != cudaSuccess) return cuda_fail(e, "plan sparse linear");
    if (ps.ticket_words > kSplitKTicketWords) return LAROSA_ERR_SHAPE;
    partials = std::max(partials, ps.partial_floats);
  }
  size_t off = align_up(kHeaderEnd, 256);
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  L->fused_sync = kOffFusedSync;
  L->x_rot = take((size_t)M * d_in * 4);
  L->idx = take((size_t)M * K * 4);
  L->val = take((size_t)M * K * 4);
  L->nnz = take((size_t)M * 4);
  L->partials = take(partials * 4);
  if (M > 1) {
    L->coef = take((size_t)M * d_in * 4);
    L->urows = take((size_t)d_in * 4);
    L->ucount = take(4);
    L->coef_hl = take((size_t)2 * M * d_in * 2);  // the tensor-core path's coefficient rows
  }
  L->total = off;
  return LAROSA_OK;
}

int check_sizes(int M, int d_in, int d_out, int K) {
  if (M < 1 || M > LAROSA_MAX_M) return LAROSA_ERR_SHAPE;
  if (d_in < 1 || d_in > LAROSA_MAX_D) return LAROSA_ERR_SHAPE;
  if (d_out < 1 || d_out > kMaxDout) return LAROSA_ERR_SHAPE;
  if (K < 0 || K > d_in) return LAROSA_ERR_SHAPE;
  return LAROSA_OK;
}

unsigned char* at(void* ws, size_t off) { return static_cast<unsigned char*>(ws) + off; }

int workspace_ok(void* ws, size_t ws_bytes, const Layout& L) {
  if (ws == nullptr || !aligned16(ws) || ws_bytes < L.total) return LAROSA_ERR_WORKSPACE;
  return LAROSA_OK;
}

// Row-dot operands: rows of n_in elements, n_in a multiple of 8.
bool rowdot_aligned(const void* A, const void* x, int n_in) {
  return aligned16(A) && aligned16(x) && (n_in % 8) == 0;
}

// The rotation's operands, Qt null meaning the identity rotation.
bool rotation_aligned(const void* Qt, const void* x, int d) {
  return (Qt == nullptr || aligned16(Qt)) && aligned16(x) && (d % 8) == 0;
}

int run_rowdot(const void* x, const void* A, float* y, int M, int n_in, int n_out, int dtype,
               cudaStream_t s, const char* what) {
  cudaError_t e = larosa::launch_rowdot(elem_of(dtype), A, x, y, M, n_in, n_out, s);
  return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, what);
}

// x_rot = x . Q, or x widened when Qt is null (the identity rotation).
int run_rotation(const void* x, const void* Qt, float* x_rot, int M, int d, int dtype,
                 cudaStream_t s) {
  if (Qt != nullptr) return run_rowdot(x, Qt, x_rot, M, d, d, dtype, s, "rotation kernel");
  cudaError_t e = larosa::launch_widen(x, x_rot, M * d, elem_of(dtype), s);
  return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "widen kernel");
}

// Threshold t >= 0 as the key it is compared with (sign-cleared fp32 bits);
// t <= 0 keeps everything.
uint32_t threshold_key(float t) {
  if (!(t > 0.f)) return 0u;
  uint32_t k;
  memcpy(&k, &t, sizeof(k));
  return k;
}

// 2 to 16 bf16 tokens: the union of their kept rows is most rows (84 % at
// two tokens and 40 % sparsity, nearly all from four on), so the sparse
// linear is the dense tcgen05 product with each token's coefficient row
// (zero where the token did not keep the row) -- unless two to four tokens
// keep so few rows that streaming their union is faster (umma_gemv_pays).
bool tensor_core_gemv(int M, int d_in, int d_out, int K, int dtype, const Layout& L) {
  return dtype == LAROSA_BF16 && L.coef_hl != 0 && larosa::umma_gemv_pays(M, d_in, d_out, K);
}

int run_sparse(const int32_t* idx, const float* val, int M, int K, const void* W_rot, int d_in,
               int d_out, float* y, int dtype, void* ws, const Layout& L, int* dev_status,
               cudaStream_t s) {
  if (M == 1) {
    larosa::StreamPlan sp;
    cudaError_t e = larosa::plan_gather(elem_of(dtype), d_out, K, &sp);
    if (e != cudaSuccess) return cuda_fail(e, "plan gather");
    if (sp.ok) {
      larosa::GatherArgs a;
      a.W = W_rot;
      a.d_out = d_out;
      a.row_bound = d_in;
      a.n = K;
      a.coef = val;
      a.rows = idx;
      a.y = y;
      a.dev_status = dev_status;
      e = larosa::launch_gather(elem_of(dtype), a, sp, s);
      return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "gather kernel");
    }
  }
  const int n_max = sparse_rows_max(M, d_in, K);
  GemvPlan pl;
  cudaError_t e = larosa::plan_gemv(elem_of(dtype), Elem::F32, M, d_out, n_max, &pl);
  if (e != cudaSuccess) return cuda_fail(e, "plan sparse linear");
  GemvArgs a;
  a.W = W_rot;
  a.w_elem = elem_of(dtype);
  a.d_out = d_out;
  a.row_bound = d_in;
  a.coef_elem = Elem::F32;
  a.M = M;
  a.y = y;
  a.y_ld = d_out;
  a.partials = reinterpret_cast<float*>(at(ws, L.partials));
  a.tickets = reinterpret_cast<unsigned*>(at(ws, kOffTickets));
  a.dev_status = dev_status;
  if (M == 1) {
    a.rows = idx;
    a.n_rows = K;
    a.coef = val;
    a.coef_ld = K;
  } else {
    if (tensor_core_gemv(M, d_in, d_out, K, dtype, L)) {
      // every row is kept by some token at this many tokens: the dense
      // product with the per-token coefficients (zero where not kept)
      __nv_bfloat16* hl = reinterpret_cast<__nv_bfloat16*>(at(ws, L.coef_hl));
      e = larosa::launch_coef_rows(idx, val, M, K, d_in, hl, dev_status, s);
      if (e != cudaSuccess) return cuda_fail(e, "coefficient rows kernel");
      e = larosa::launch_umma_gemv(W_rot, hl, y, M, d_in, d_out, dev_status, s);
      return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "tensor-core sparse linear kernel");
    }
    float* coef = reinterpret_cast<float*>(at(ws, L.coef));
    unsigned* bitmap = reinterpret_cast<unsigned*>(at(ws, kOffBitmap));
    int32_t* urows = reinterpret_cast<int32_t*>(at(ws, L.urows));
    int* ucount = reinterpret_cast<int*>(at(ws, L.ucount));
    e = larosa::launch_scatter(idx, val, M, K, d_in, coef, bitmap, dev_status, s);
    if (e != cudaSuccess) return cuda_fail(e, "scatter kernel");
    e = larosa::launch_union(bitmap, d_in, urows, ucount, s);
    if (e != cudaSuccess) return cuda_fail(e, "union kernel");
    a.rows = urows;
    a.n_rows = n_max;
    a.n_rows_dev = ucount;
    a.coef = coef;
    a.coef_ld = d_in;
    a.coef_by_row = 1;
  }
  e = larosa::launch_gemv(a, pl, s);
  return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "sparse linear kernel");
}

// Workspace of larosa_sparse_lowrank_linear: the sparse linear's layout, then
// the dropped part of x, u = dropped . A_r, y_r = u . B_r and the split-K
// partials of the two GEMVs through the factors.
struct LowrankLayout {
  Layout base;
  size_t x_drop = 0, u = 0, y_r = 0, partials = 0, total = 0;
  // one token in one launch (lowrank_kernel): its u, partials and counters
  bool one_launch = false;
  size_t lr_u = 0, lr_partials = 0, lr_sync = 0;
};

int make_lowrank_layout(int M, int d_in, int d_out, int K, int r, LowrankLayout* LL) {
  int st = make_layout(M, d_in, d_out, K, &LL->base);
  if (st != LAROSA_OK) return st;
  size_t pf = 0;
  for (int dt = 0; dt < 2; ++dt) {
    const Elem w = dt == 0 ? Elem::F32 : Elem::BF16;
    GemvPlan pa, pb;
    cudaError_t e = larosa::plan_gemv(w, Elem::F32, M, r, d_in, &pa);
    if (e == cudaSuccess) e = larosa::plan_gemv(w, Elem::F32, M, d_out, r, &pb);
    if (e != cudaSuccess) return cuda_fail(e, "plan low-rank GEMV");
    if (pa.ticket_words > kSplitKTicketWords || pb.ticket_words > kSplitKTicketWords)
      return LAROSA_ERR_SHAPE;
    pf = std::max(pf, std::max(pa.partial_floats, pb.partial_floats));
  }
  size_t off = align_up(LL->base.total, 256);
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  LL->x_drop = take((size_t)M * d_in * 4);
  LL->u = take((size_t)M * r * 4);
  LL->y_r = take((size_t)M * d_out * 4);
  LL->partials = take(pf * 4);
  if (M == 1) {
    // the one-launch kernel, for either weight type
    size_t lp = 0;
    bool ok = true;
    for (int dt = 0; dt < 2; ++dt) {
      larosa::StreamPlan pl;
      cudaError_t e = larosa::plan_lowrank(dt == 0 ? Elem::F32 : Elem::BF16, d_in, d_out, K, r, &pl);
      if (e != cudaSuccess) return cuda_fail(e, "plan low-rank kernel");
      ok = ok && pl.ok;
      lp = std::max(lp, pl.partial_floats);
    }
    if (ok) {
      LL->one_launch = true;
      LL->lr_sync = take((2 + larosa::kFusedMaxTiles) * 4);
      LL->lr_u = take((size_t)larosa::kLowrankMaxFactorCtas * r * 4);
      LL->lr_partials = take(lp * 4);
    }
  }
  LL->total = off;
  return LAROSA_OK;
}

// out[M x cols] = coef[M x rows] . Wm[rows x cols] (all rows, fp32 coefficients).
int run_dense_gemv(const void* Wm, int rows, int cols, const float* coef, int M, float* out,
                   int dtype, void* ws, float* partials, int* dev_status, cudaStream_t s) {
  GemvPlan pl;
  cudaError_t e = larosa::plan_gemv(elem_of(dtype), Elem::F32, M, cols, rows, &pl);
  if (e != cudaSuccess) return cuda_fail(e, "plan low-rank GEMV");
  GemvArgs a;
  a.W = Wm;
  a.w_elem = elem_of(dtype);
  a.d_out = cols;
  a.row_bound = rows;
  a.rows = nullptr;
  a.n_rows = rows;
  a.coef = coef;
  a.coef_elem = Elem::F32;
  a.coef_ld = rows;
  a.M = M;
  a.y = out;
  a.y_ld = cols;
  a.partials = partials;
  a.tickets = reinterpret_cast<unsigned*>(at(ws, kOffTickets));
  a.dev_status = dev_status;
  e = larosa::launch_gemv(a, pl, s);
  return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "low-rank GEMV kernel");
}

}  // namespace

namespace larosa {
// Lets other translation units of the library report a message through
// larosa_last_error_string().
void set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

namespace {
// An integer environment variable, `fallback` when unset or not a number.
int env_int(const char* name, int fallback) {
  const char* v = getenv(name);
  if (v == nullptr || *v == 0) return fallback;
  char* end = nullptr;
  const long x = strtol(v, &end, 10);
  return (end != nullptr && *end == 0 && x >= INT_MIN && x <= INT_MAX) ? static_cast<int>(x) : fallback;
}
}  // namespace

// -1 until the first use reads the environment
std::atomic<int> g_debug{-1};
std::atomic<int> g_split_k{-1};

bool debug_checks() {
  if (g_debug.load(std::memory_order_relaxed) < 0) {
    int unset = -1;
    g_debug.compare_exchange_strong(unset, env_int("LAROSA_DEBUG", 0) != 0 ? 1 : 0);
  }
  return g_debug.load(std::memory_order_relaxed) == 1;
}

int split_k_override() {
  if (g_split_k.load(std::memory_order_relaxed) < 0) {
    int v = env_int("LAROSA_SPLIT_K", 0);
    if (v < 0 || v > LAROSA_MAX_SPLIT_K) v = 0;
    int unset = -1;
    g_split_k.compare_exchange_strong(unset, v);
  }
  return g_split_k.load(std::memory_order_relaxed);
}
}  // namespace larosa

namespace {
// With the debug checks on: the kept lists idx/val ([M x K]) checked on the
// stream (see larosa_set_debug).
int debug_check_lists(const int32_t* idx, const float* val, int M, int K, int d, bool ascending,
                      int* dev_status, cudaStream_t s) {
  if (!larosa::debug_checks()) return LAROSA_OK;
  const cudaError_t e = larosa::launch_check_lists(idx, val, M, K, d, ascending, dev_status, s);
  return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "list check kernel");
}
}  // namespace

extern "C" {

const char* larosa_status_string(int status) {
  switch (status) {
    case LAROSA_OK: return "LAROSA_OK";
    case LAROSA_ERR_INVALID_ARG: return "LAROSA_ERR_INVALID_ARG: invalid argument";
    case LAROSA_ERR_SHAPE: return "LAROSA_ERR_SHAPE: size out of range";
    case LAROSA_ERR_ALIGN: return "LAROSA_ERR_ALIGN: pointer or row length not 16-byte aligned";
    case LAROSA_ERR_UNSUPPORTED_DTYPE: return "LAROSA_ERR_UNSUPPORTED_DTYPE: unsupported data type";
    case LAROSA_ERR_CUDA: return "LAROSA_ERR_CUDA: a CUDA runtime call failed";
    case LAROSA_ERR_WORKSPACE: return "LAROSA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case LAROSA_ERR_NONFINITE: return "LAROSA_ERR_NONFINITE: a NaN or Inf reached Top-K";
    case LAROSA_ERR_TIMEOUT: return "LAROSA_ERR_TIMEOUT: a kernel wait exceeded its time limit";
    case LAROSA_ERR_INDEX: return "LAROSA_ERR_INDEX: an index was out of range";
    case LAROSA_ERR_LIST: return "LAROSA_ERR_LIST: a kept list repeats an index or is out of order";
    default: return "unknown larosa status";
  }
}

int larosa_version(void) { return LAROSA_VERSION; }

const char* larosa_last_error_string(void) { return g_last_error; }

size_t larosa_workspace_bytes(int M, int d_in, int d_out, int K) {
  if (check_sizes(M, d_in, d_out, K) != LAROSA_OK) return 0;
  Layout L;
  if (make_layout(M, d_in, d_out, K, &L) != LAROSA_OK) return 0;
  return L.total;
}

int larosa_workspace_layout(int M, int d_in, int d_out, int K, size_t* x_rot_offset,
                            size_t* idx_offset, size_t* val_offset) {
  int st = check_sizes(M, d_in, d_out, K);
  if (st != LAROSA_OK) return st;
  Layout L;
  st = make_layout(M, d_in, d_out, K, &L);
  if (st != LAROSA_OK) return st;
  if (x_rot_offset) *x_rot_offset = L.x_rot;
  if (idx_offset) *idx_offset = L.idx;
  if (val_offset) *val_offset = L.val;
  return LAROSA_OK;
}

int larosa_workspace_nnz_offset(int M, int d_in, int d_out, int K, size_t* nnz_offset) {
  int st = check_sizes(M, d_in, d_out, K);
  if (st != LAROSA_OK) return st;
  Layout L;
  st = make_layout(M, d_in, d_out, K, &L);
  if (st != LAROSA_OK) return st;
  if (nnz_offset) *nnz_offset = L.nnz;
  return LAROSA_OK;
}

int larosa_workspace_sync_offset(int M, int d_in, int d_out, int K, size_t* sync_offset) {
  int st = check_sizes(M, d_in, d_out, K);
  if (st != LAROSA_OK) return st;
  if (M != 1) return LAROSA_ERR_SHAPE;
  Layout L;
  st = make_layout(M, d_in, d_out, K, &L);
  if (st != LAROSA_OK) return st;
  if (sync_offset) *sync_offset = L.fused_sync;
  return LAROSA_OK;
}

int larosa_set_wait_limit_ns(uint64_t limit_ns, uint64_t* previous) {
  if (limit_ns != 0 && (limit_ns < LAROSA_MIN_WAIT_LIMIT_NS || limit_ns > LAROSA_MAX_WAIT_LIMIT_NS))
    return LAROSA_ERR_INVALID_ARG;
  const unsigned long long v = limit_ns == 0 ? larosa::kDefaultWaitLimitNs : limit_ns;
  const unsigned long long old = larosa::g_wait_limit_ns.exchange(v);
  if (previous) *previous = old;
  return LAROSA_OK;
}

int larosa_set_debug(int on, int* previous) {
  if (on != 0 && on != 1) return LAROSA_ERR_INVALID_ARG;
  (void)larosa::debug_checks();  // the environment's setting, if not read yet
  const int old = larosa::g_debug.exchange(on);
  if (previous) *previous = old;
  return LAROSA_OK;
}

int larosa_set_split_k(int splits, int* previous) {
  if (splits < 0 || splits > LAROSA_MAX_SPLIT_K) return LAROSA_ERR_INVALID_ARG;
  (void)larosa::split_k_override();
  const int old = larosa::g_split_k.exchange(splits);
  if (previous) *previous = old;
  return LAROSA_OK;
}

int larosa_prepare_weights(const void* Qt, const void* W, void* W_rot, int d_in, int d_out,
                           int dtype, larosa_stream_t stream) {
  if (!valid_dtype(dtype)) return LAROSA_ERR_UNSUPPORTED_DTYPE;
  if (Qt == nullptr || W == nullptr || W_rot == nullptr) return LAROSA_ERR_INVALID_ARG;
  if (d_in < 1 || d_in > LAROSA_MAX_D || d_out < 1 || d_out > kMaxDout) return LAROSA_ERR_SHAPE;
  if (W_rot == W || W_rot == Qt) return LAROSA_ERR_INVALID_ARG;
  cudaError_t e = larosa::launch_prepare(Qt, W, W_rot, d_in, d_out, elem_of(dtype),
                                         reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "prepare kernel");
}

int larosa_fold_rotation(const void* Qt, const void* Wt_prev, void* Wt_prev_rot, int d, int d_prev,
                         int dtype, larosa_stream_t stream) {
  // Q^T . Wt_prev is the counter-rotation of larosa_prepare_weights applied
  // to the producer's [d x d_prev] weight
  return larosa_prepare_weights(Qt, Wt_prev, Wt_prev_rot, d, d_prev, dtype, stream);
}

int larosa_rotate(const void* x, const void* Qt, float* x_rot, int M, int d, int dtype,
                  larosa_stream_t stream) {
  if (!valid_dtype(dtype)) return LAROSA_ERR_UNSUPPORTED_DTYPE;
  if (x == nullptr || Qt == nullptr || x_rot == nullptr) return LAROSA_ERR_INVALID_ARG;
  const int st = check_sizes(M, d, d, 0);
  if (st != LAROSA_OK) return st;
  if (!rowdot_aligned(Qt, x, d)) return LAROSA_ERR_ALIGN;
  return run_rowdot(x, Qt, x_rot, M, d, d, dtype, reinterpret_cast<cudaStream_t>(stream),
                    "rotation kernel");
}

int larosa_topk(const float* x_rot, int M, int d, int K, int32_t* idx, float* val,
                int* dev_status, larosa_stream_t stream) {
  if (x_rot == nullptr || (K > 0 && (idx == nullptr || val == nullptr)))
    return LAROSA_ERR_INVALID_ARG;
  if (M < 1 || M > LAROSA_MAX_M || d < 1 || d > LAROSA_MAX_D || K < 0 || K > d)
    return LAROSA_ERR_SHAPE;
  cudaError_t e = larosa::launch_topk(x_rot, M, d, K, idx, val, dev_status,
                                      reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "topk kernel");
  return debug_check_lists(idx, val, M, K, d, true, dev_status, reinterpret_cast<cudaStream_t>(stream));
}

int larosa_rotate_topk(const void* x, const void* Qt, float* x_rot, int32_t* idx, float* val, int d,
                       int K, void* ws, size_t ws_bytes, int* dev_status, int dtype,
                       larosa_stream_t stream) {
  if (!valid_dtype(dtype)) return LAROSA_ERR_UNSUPPORTED_DTYPE;
  if (x == nullptr || Qt == nullptr || x_rot == nullptr || (K > 0 && (idx == nullptr || val == nullptr)))
    return LAROSA_ERR_INVALID_ARG;
  int st = check_sizes(1, d, 1, K);
  if (st != LAROSA_OK) return st;
  if (!rowdot_aligned(Qt, x, d) || !aligned16(x_rot)) return LAROSA_ERR_ALIGN;
  if (!larosa::rotsel_fits(elem_of(dtype), d)) return LAROSA_ERR_SHAPE;
  Layout L;
  st = make_layout(1, d, 1, K, &L);
  if (st != LAROSA_OK) return st;
  st = workspace_ok(ws, ws_bytes, L);
  if (st != LAROSA_OK) return st;
  larosa::RotSelArgs r;
  r.x = x;
  r.Qt = Qt;
  r.x_rot = x_rot;
  r.idx = idx;
  r.val = val;
  r.ticket = reinterpret_cast<unsigned*>(at(ws, kOffTickets + kRotSelTicket * 4));
  r.d = d;
  r.K = K;
  r.dev_status = dev_status;
  cudaError_t e = larosa::launch_rotsel(elem_of(dtype), r, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rotate-select kernel");
  return debug_check_lists(idx, val, 1, K, d, true, dev_status, reinterpret_cast<cudaStream_t>(stream));
}

int larosa_sparse_linear(const int32_t* idx, const float* val, int M, int K, const void* W_rot,
                         int d_in, int d_out, float* y, void* ws, size_t ws_bytes, int dtype,
                         int* dev_status, larosa_stream_t stream) {
  if (!valid_dtype(dtype)) return LAROSA_ERR_UNSUPPORTED_DTYPE;
  if (W_rot == nullptr || y == nullptr || (K > 0 && (idx == nullptr || val == nullptr)))
    return LAROSA_ERR_INVALID_ARG;
  int st = check_sizes(M, d_in, d_out, K);
  if (st != LAROSA_OK) return st;
  if (!aligned16(W_rot) || !aligned16(y) || !row_aligned(d_out, dtype)) return LAROSA_ERR_ALIGN;
  Layout L;
  st = make_layout(M, d_in, d_out, K, &L);
  if (st != LAROSA_OK) return st;
  st = workspace_ok(ws, ws_bytes, L);
  if (st != LAROSA_OK) return st;
  st = debug_check_lists(idx, val, M, K, d_in, false, dev_status, reinterpret_cast<cudaStream_t>(stream));
  if (st != LAROSA_OK) return st;
  return run_sparse(idx, val, M, K, W_rot, d_in, d_out, y, dtype, ws, L, dev_status,
                    reinterpret_cast<cudaStream_t>(stream));
}

static int rotate_topk_linear_impl(const void* x, const void* Qt, const void* W_rot, int M, int d_in,
                                   int d_out, int K, float* y, void* ws, size_t ws_bytes,
                                   int* dev_status, int dtype, larosa_stream_t stream) {
  if (!valid_dtype(dtype)) return LAROSA_ERR_UNSUPPORTED_DTYPE;
  if (x == nullptr || W_rot == nullptr || y == nullptr) return LAROSA_ERR_INVALID_ARG;
  int st = check_sizes(M, d_in, d_out, K);
  if (st != LAROSA_OK) return st;
  if (!rotation_aligned(Qt, x, d_in) || !aligned16(W_rot) || !aligned16(y) ||
      !row_aligned(d_out, dtype))
    return LAROSA_ERR_ALIGN;
  Layout L;
  st = make_layout(M, d_in, d_out, K, &L);
  if (st != LAROSA_OK) return st;
  st = workspace_ok(ws, ws_bytes, L);
  if (st != LAROSA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* x_rot = reinterpret_cast<float*>(at(ws, L.x_rot));
  int32_t* idx = reinterpret_cast<int32_t*>(at(ws, L.idx));
  float* val = reinterpret_cast<float*>(at(ws, L.val));
  if (M == 1) {
    // one cooperative kernel: rotation, selection, gather
    larosa::StreamPlan fp;
    cudaError_t e = larosa::plan_fused(elem_of(dtype), d_in, d_out, K, &fp);
    if (e != cudaSuccess) return cuda_fail(e, "plan fused");
    if (fp.ok) {
      larosa::FusedArgs f;
      f.x = x;
      f.Qt = Qt;
      f.W = W_rot;
      f.x_rot = x_rot;
      f.idx = idx;
      f.val = val;
      f.y = y;
      f.partials = reinterpret_cast<float*>(at(ws, L.partials));
      f.sync = reinterpret_cast<unsigned*>(at(ws, L.fused_sync));
      f.d_in = d_in;
      f.d_out = d_out;
      f.K = K;
      f.dev_status = dev_status;
      e = larosa::launch_fused(elem_of(dtype), f, fp, s);
      return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "fused kernel");
    }
  }
  if (M == 1 && Qt != nullptr && larosa::rotsel_fits(elem_of(dtype), d_in)) {
    // rotation whose last CTA writes the kept list, then the list-mode gather
    larosa::StreamPlan sp;
    cudaError_t e = larosa::plan_gather(elem_of(dtype), d_out, K, &sp);
    if (e != cudaSuccess) return cuda_fail(e, "plan gather");
    if (sp.ok) {
      larosa::RotSelArgs r;
      r.x = x;
      r.Qt = Qt;
      r.x_rot = x_rot;
      r.idx = idx;
      r.val = val;
      r.ticket = reinterpret_cast<unsigned*>(at(ws, kOffTickets + kRotSelTicket * 4));
      r.d = d_in;
      r.K = K;
      r.dev_status = dev_status;
      e = larosa::launch_rotsel(elem_of(dtype), r, s);
      if (e != cudaSuccess) return cuda_fail(e, "rotate-select kernel");
      larosa::GatherArgs a;
      a.W = W_rot;
      a.d_out = d_out;
      a.row_bound = d_in;
      a.n = K;
      a.coef = val;
      a.rows = idx;
      a.y = y;
      a.dev_status = dev_status;
      e = larosa::launch_gather(elem_of(dtype), a, sp, s);
      return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "gather kernel");
    }
  }
  st = run_rotation(x, Qt, x_rot, M, d_in, dtype, s);
  if (st != LAROSA_OK) return st;
  if (M > 1 && tensor_core_gemv(M, d_in, d_out, K, dtype, L)) {
    // the Top-K kernel also writes the tokens' coefficient rows for the
    // tensor-core product
    __nv_bfloat16* hl = reinterpret_cast<__nv_bfloat16*>(at(ws, L.coef_hl));
    cudaError_t e = larosa::launch_topk(x_rot, M, d_in, K, idx, val, dev_status, s, hl);
    if (e != cudaSuccess) return cuda_fail(e, "topk kernel");
    e = larosa::launch_umma_gemv(W_rot, hl, y, M, d_in, d_out, dev_status, s);
    return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "tensor-core sparse linear kernel");
  }
  cudaError_t e = larosa::launch_topk(x_rot, M, d_in, K, idx, val, dev_status, s);
  if (e != cudaSuccess) return cuda_fail(e, "topk kernel");
  return run_sparse(idx, val, M, K, W_rot, d_in, d_out, y, dtype, ws, L, dev_status, s);
}

// The kept lists a successful call left in the workspace, checked when the
// debug checks are on.
static int check_workspace_lists(int M, int d_in, int d_out, int K, void* ws, int* dev_status,
                                 larosa_stream_t stream) {
  if (!larosa::debug_checks()) return LAROSA_OK;
  Layout L;
  const int st = make_layout(M, d_in, d_out, K, &L);
  if (st != LAROSA_OK) return st;
  return debug_check_lists(reinterpret_cast<const int32_t*>(at(ws, L.idx)),
                           reinterpret_cast<const float*>(at(ws, L.val)), M, K, d_in, true, dev_status,
                           reinterpret_cast<cudaStream_t>(stream));
}

int larosa_rotate_topk_linear(const void* x, const void* Qt, const void* W_rot, int M, int d_in,
                              int d_out, int K, float* y, void* ws, size_t ws_bytes,
                              int* dev_status, int dtype, larosa_stream_t stream) {
  const int st = rotate_topk_linear_impl(x, Qt, W_rot, M, d_in, d_out, K, y, ws, ws_bytes, dev_status,
                                         dtype, stream);
  return st != LAROSA_OK ? st : check_workspace_lists(M, d_in, d_out, K, ws, dev_status, stream);
}

static int topk_linear_impl(const float* x_rot, const void* W_rot, int M, int d_in, int d_out, int K,
                            float* y, void* ws, size_t ws_bytes, int* dev_status, int dtype,
                            larosa_stream_t stream) {
  if (!valid_dtype(dtype)) return LAROSA_ERR_UNSUPPORTED_DTYPE;
  if (x_rot == nullptr || W_rot == nullptr || y == nullptr) return LAROSA_ERR_INVALID_ARG;
  int st = check_sizes(M, d_in, d_out, K);
  if (st != LAROSA_OK) return st;
  if (!aligned16(x_rot) || !aligned16(W_rot) || !aligned16(y) || !row_aligned(d_out, dtype))
    return LAROSA_ERR_ALIGN;
  Layout L;
  st = make_layout(M, d_in, d_out, K, &L);
  if (st != LAROSA_OK) return st;
  st = workspace_ok(ws, ws_bytes, L);
  if (st != LAROSA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t* idx = reinterpret_cast<int32_t*>(at(ws, L.idx));
  float* val = reinterpret_cast<float*>(at(ws, L.val));
  if (M > 1 && tensor_core_gemv(M, d_in, d_out, K, dtype, L)) {
    __nv_bfloat16* hl = reinterpret_cast<__nv_bfloat16*>(at(ws, L.coef_hl));
    cudaError_t e = larosa::launch_topk(x_rot, M, d_in, K, idx, val, dev_status, s, hl);
    if (e != cudaSuccess) return cuda_fail(e, "topk kernel");
    e = larosa::launch_umma_gemv(W_rot, hl, y, M, d_in, d_out, dev_status, s);
    return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "tensor-core sparse linear kernel");
  }
  cudaError_t e = larosa::launch_topk(x_rot, M, d_in, K, idx, val, dev_status, s);
  if (e != cudaSuccess) return cuda_fail(e, "topk kernel");
  return run_sparse(idx, val, M, K, W_rot, d_in, d_out, y, dtype, ws, L, dev_status, s);
}

int larosa_topk_linear(const float* x_rot, const void* W_rot, int M, int d_in, int d_out, int K, float* y,
                       void* ws, size_t ws_bytes, int* dev_status, int dtype, larosa_stream_t stream) {
  const int st = topk_linear_impl(x_rot, W_rot, M, d_in, d_out, K, y, ws, ws_bytes, dev_status, dtype, stream);
  return st != LAROSA_OK ? st : check_workspace_lists(M, d_in, d_out, K, ws, dev_status, stream);
}

int larosa_threshold(const float* x_rot, int M, int d, float t, int32_t* idx, float* val,
                     int32_t* nnz, int* dev_status, larosa_stream_t stream) {
  if (x_rot == nullptr || idx == nullptr || val == nullptr || nnz == nullptr || t != t)
    return LAROSA_ERR_INVALID_ARG;
  if (M < 1 || M > LAROSA_MAX_M || d < 1 || d > LAROSA_MAX_D) return LAROSA_ERR_SHAPE;
  cudaError_t e = larosa::launch_threshold(x_rot, M, d, threshold_key(t), idx, val, nnz, nullptr,
                                           nullptr, dev_status,
                                           reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "threshold kernel");
}

int larosa_rotate_threshold_linear(const void* x, const void* Qt, const void* W_rot, int M,
                                   int d_in, int d_out, float t, float* y, void* ws,
                                   size_t ws_bytes, int* dev_status, int dtype,
                                   larosa_stream_t stream) {
  if (!valid_dtype(dtype)) return LAROSA_ERR_UNSUPPORTED_DTYPE;
  if (x == nullptr || W_rot == nullptr || y == nullptr || t != t) return LAROSA_ERR_INVALID_ARG;
  int st = check_sizes(M, d_in, d_out, d_in);
  if (st != LAROSA_OK) return st;
  if (!rotation_aligned(Qt, x, d_in) || !aligned16(W_rot) || !aligned16(y) ||
      !row_aligned(d_out, dtype))
    return LAROSA_ERR_ALIGN;
  Layout L;
  st = make_layout(M, d_in, d_out, d_in, &L);
  if (st != LAROSA_OK) return st;
  st = workspace_ok(ws, ws_bytes, L);
  if (st != LAROSA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* x_rot = reinterpret_cast<float*>(at(ws, L.x_rot));
  int32_t* idx = reinterpret_cast<int32_t*>(at(ws, L.idx));
  float* val = reinterpret_cast<float*>(at(ws, L.val));
  int32_t* nnz = reinterpret_cast<int32_t*>(at(ws, L.nnz));
  const uint32_t t_key = threshold_key(t);
  cudaError_t e;
  if (M == 1) {
    // one cooperative kernel: rotation, threshold, gather
    larosa::StreamPlan fp;
    e = larosa::plan_fused(elem_of(dtype), d_in, d_out, d_in, &fp);
    if (e != cudaSuccess) return cuda_fail(e, "plan fused");
    if (fp.ok) {
      larosa::FusedArgs f;
      f.x = x;
      f.Qt = Qt;
      f.W = W_rot;
      f.x_rot = x_rot;
      f.idx = idx;
      f.val = val;
      f.y = y;
      f.partials = reinterpret_cast<float*>(at(ws, L.partials));
      f.sync = reinterpret_cast<unsigned*>(at(ws, L.fused_sync));
      f.d_in = d_in;
      f.d_out = d_out;
      f.K = d_in;
      f.dev_status = dev_status;
      f.threshold = true;
      f.t_key = t_key;
      f.nnz = nnz;
      e = larosa::launch_fused(elem_of(dtype), f, fp, s);
      return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "fused kernel");
    }
    if (!L.list_gemv) return LAROSA_ERR_SHAPE;
  }
  st = run_rotation(x, Qt, x_rot, M, d_in, dtype, s);
  if (st != LAROSA_OK) return st;
  if (M > 1 && dtype == LAROSA_BF16 && L.coef_hl != 0 && larosa::umma_gemv_applies(M, d_in, d_out)) {
    // how many rows the tokens keep is known only on the device: the dense
    // tensor-core product with the coefficient rows the threshold kernel
    // writes, as the Top-K path takes at the sparsities the method uses
    __nv_bfloat16* hl = reinterpret_cast<__nv_bfloat16*>(at(ws, L.coef_hl));
    e = larosa::launch_threshold(x_rot, M, d_in, t_key, idx, val, nnz, nullptr, nullptr, dev_status, s, hl);
    if (e != cudaSuccess) return cuda_fail(e, "threshold kernel");
    e = larosa::launch_umma_gemv(W_rot, hl, y, M, d_in, d_out, dev_status, s);
    return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "tensor-core sparse linear kernel");
  }
  GemvPlan pl;
  e = larosa::plan_gemv(elem_of(dtype), Elem::F32, M, d_out, d_in, &pl);
  if (e != cudaSuccess) return cuda_fail(e, "plan sparse linear");
  GemvArgs a;
  a.W = W_rot;
  a.w_elem = elem_of(dtype);
  a.d_out = d_out;
  a.row_bound = d_in;
  a.coef_elem = Elem::F32;
  a.M = M;
  a.y = y;
  a.y_ld = d_out;
  a.partials = reinterpret_cast<float*>(at(ws, L.partials));
  a.tickets = reinterpret_cast<unsigned*>(at(ws, kOffTickets));
  a.dev_status = dev_status;
  a.n_rows = d_in;
  if (M == 1) {
    // the kept list and its length, read on the device
    e = larosa::launch_threshold(x_rot, 1, d_in, t_key, idx, val, nnz, nullptr, nullptr,
                                 dev_status, s);
    if (e != cudaSuccess) return cuda_fail(e, "threshold kernel");
    a.rows = idx;
    a.n_rows_dev = nnz;
    a.coef = val;
    a.coef_ld = d_in;
  } else {
    // every token's coefficient row and the union of the kept rows
    float* coef = reinterpret_cast<float*>(at(ws, L.coef));
    unsigned* bitmap = reinterpret_cast<unsigned*>(at(ws, kOffBitmap));
    int32_t* urows = reinterpret_cast<int32_t*>(at(ws, L.urows));
    int* ucount = reinterpret_cast<int*>(at(ws, L.ucount));
    e = larosa::launch_threshold(x_rot, M, d_in, t_key, idx, val, nnz, coef, bitmap, dev_status, s);
    if (e != cudaSuccess) return cuda_fail(e, "threshold kernel");
    e = larosa::launch_union(bitmap, d_in, urows, ucount, s);
    if (e != cudaSuccess) return cuda_fail(e, "union kernel");
    a.rows = urows;
    a.n_rows_dev = ucount;
    a.coef = coef;
    a.coef_ld = d_in;
    a.coef_by_row = 1;
  }
  e = larosa::launch_gemv(a, pl, s);
  return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "sparse linear kernel");
}

size_t larosa_lowrank_workspace_bytes(int M, int d_in, int d_out, int K, int r) {
  if (check_sizes(M, d_in, d_out, K) != LAROSA_OK || r < 1 || r > kMaxDout) return 0;
  LowrankLayout LL;
  if (make_lowrank_layout(M, d_in, d_out, K, r, &LL) != LAROSA_OK) return 0;
  return LL.total;
}

int larosa_sparse_lowrank_linear(const float* x, const int32_t* idx, const float* val, int M, int K,
                                 const void* W, const void* A_r, const void* B_r, int d_in,
                                 int d_out, int r, float* y, void* ws, size_t ws_bytes, int dtype,
                                 int* dev_status, larosa_stream_t stream) {
  if (!valid_dtype(dtype)) return LAROSA_ERR_UNSUPPORTED_DTYPE;
  if (x == nullptr || W == nullptr || A_r == nullptr || B_r == nullptr || y == nullptr ||
      (K > 0 && (idx == nullptr || val == nullptr)))
    return LAROSA_ERR_INVALID_ARG;
  int st = check_sizes(M, d_in, d_out, K);
  if (st != LAROSA_OK) return st;
  if (r < 1 || r > kMaxDout) return LAROSA_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(W) || !aligned16(A_r) || !aligned16(B_r) || !aligned16(y) ||
      !row_aligned(d_out, dtype) || !row_aligned(r, dtype))
    return LAROSA_ERR_ALIGN;
  LowrankLayout LL;
  st = make_lowrank_layout(M, d_in, d_out, K, r, &LL);
  if (st != LAROSA_OK) return st;
  if (ws == nullptr || !aligned16(ws) || ws_bytes < LL.total) return LAROSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = debug_check_lists(idx, val, M, K, d_in, false, dev_status, s);
  if (st != LAROSA_OK) return st;
  if (M == 1 && LL.one_launch) {
    // one cooperative launch: kept rows of W, x_drop . A_r, then u . B_r
    larosa::StreamPlan pl;
    cudaError_t e = larosa::plan_lowrank(elem_of(dtype), d_in, d_out, K, r, &pl);
    if (e != cudaSuccess) return cuda_fail(e, "plan low-rank kernel");
    if (pl.ok) {
      larosa::LowrankArgs a;
      a.x = x;
      a.idx = idx;
      a.val = val;
      a.W = W;
      a.A_r = A_r;
      a.B_r = B_r;
      a.y = y;
      a.u = reinterpret_cast<float*>(at(ws, LL.lr_u));
      a.partials = reinterpret_cast<float*>(at(ws, LL.lr_partials));
      a.sync = reinterpret_cast<unsigned*>(at(ws, LL.lr_sync));
      a.d_in = d_in;
      a.d_out = d_out;
      a.K = K;
      a.r = r;
      a.dev_status = dev_status;
      e = larosa::launch_lowrank(elem_of(dtype), a, pl, s);
      return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "low-rank kernel");
    }
  }
  float* x_drop = reinterpret_cast<float*>(at(ws, LL.x_drop));
  float* u = reinterpret_cast<float*>(at(ws, LL.u));
  float* y_r = reinterpret_cast<float*>(at(ws, LL.y_r));
  float* part = reinterpret_cast<float*>(at(ws, LL.partials));
  // y_s: the kept rows of W
  st = run_sparse(idx, val, M, K, W, d_in, d_out, y, dtype, ws, LL.base, dev_status, s);
  if (st != LAROSA_OK) return st;
  if (M > 1 && dtype == LAROSA_BF16 && LL.base.coef_hl != 0 && r <= d_in &&
      larosa::umma_gemv_applies(M, d_in, r) && larosa::umma_gemv_applies(M, r, d_out)) {
    // several bf16 tokens: both factor products on the tensor cores, fed with
    // head/tail coefficient rows of the dropped part (in the coefficient-row
    // buffer, free again once y_s is done); the first writes u directly as
    // head/tail rows (in x_drop's space, which this path does not use:
    // 2 M r bf16 <= M d_in fp32), the second adds y_r into y
    __nv_bfloat16* hl_x = reinterpret_cast<__nv_bfloat16*>(at(ws, LL.base.coef_hl));
    __nv_bfloat16* hl_u = reinterpret_cast<__nv_bfloat16*>(x_drop);
    cudaError_t e = larosa::launch_dropped_rows(x, idx, M, K, d_in, hl_x, dev_status, s);
    if (e != cudaSuccess) return cuda_fail(e, "dropped-part rows kernel");
    e = larosa::launch_umma_gemv(A_r, hl_x, nullptr, M, d_in, r, dev_status, s, false, hl_u);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core factor kernel");
    e = larosa::launch_umma_gemv(B_r, hl_u, y, M, r, d_out, dev_status, s, true);
    return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "tensor-core factor kernel");
  }
  // y_r = ((x - sigma(x)) . A_r) . B_r, then y = y_s + y_r
  cudaError_t e = larosa::launch_dropped(x, idx, M, K, d_in, x_drop, dev_status, s);
  if (e != cudaSuccess) return cuda_fail(e, "dropped-part kernel");
  st = run_dense_gemv(A_r, d_in, r, x_drop, M, u, dtype, ws, part, dev_status, s);
  if (st != LAROSA_OK) return st;
  st = run_dense_gemv(B_r, r, d_out, u, M, y_r, dtype, ws, part, dev_status, s);
  if (st != LAROSA_OK) return st;
  e = larosa::launch_add(y, y_r, M * d_out, s);
  return e == cudaSuccess ? LAROSA_OK : cuda_fail(e, "add kernel");
}

int larosa_dense_linear(const void* x, const void* Wt, int M, int d_in, int d_out, float* y,
                        int dtype, larosa_stream_t stream) {
  if (!valid_dtype(dtype)) return LAROSA_ERR_UNSUPPORTED_DTYPE;
  if (x == nullptr || Wt == nullptr || y == nullptr) return LAROSA_ERR_INVALID_ARG;
  const int st = check_sizes(M, d_in, d_out, d_in);
  if (st != LAROSA_OK) return st;
  if (!rowdot_aligned(Wt, x, d_in)) return LAROSA_ERR_ALIGN;
  return run_rowdot(x, Wt, y, M, d_in, d_out, dtype, reinterpret_cast<cudaStream_t>(stream),
                    "dense kernel");
}

int larosa_check(const int* dev_status, larosa_stream_t stream, int* flags_out) {
  if (dev_status == nullptr) return LAROSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int flags = 0;
  cudaError_t e = cudaMemcpyAsync(&flags, dev_status, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "synchronize");
  if (flags_out) *flags_out = flags;
  if (flags & LAROSA_DEV_NONFINITE) return LAROSA_ERR_NONFINITE;
  if (flags & LAROSA_DEV_TIMEOUT) return LAROSA_ERR_TIMEOUT;
  if (flags & LAROSA_DEV_INDEX) return LAROSA_ERR_INDEX;
  if (flags & LAROSA_DEV_LIST) return LAROSA_ERR_LIST;
  return LAROSA_OK;
}

}  // extern "C"
