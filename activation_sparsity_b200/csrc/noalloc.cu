// Sparse linear for callers that cannot hand the library a workspace.
//
// Some callers cannot allocate device memory on the path where they call the
// library: an operator slot in another runtime that passes only inputs and
// outputs and owns every allocation itself, or a latency-critical loop in
// which cudaMalloc and cudaFree are forbidden because they may synchronise
// the device.  For them larosa_sparse_linear_noalloc computes exactly what
// larosa_sparse_linear computes, with the same kernels and launch geometry.
// One token needs no scratch when the cluster gather fits the GPU (its
// partial sums meet in distributed shared memory; on B200 this holds for
// every size the library accepts), and otherwise falls back to the
// row-streaming GEMV, whose split-K partials use the array below.  Several
// tokens keep their split-K partial sums, reduction tickets and shared-row
// bookkeeping in one file-scope device array of fixed size instead of a
// caller workspace.  larosa_sparse_linear_noalloc_bytes tells a caller,
// without allocating or launching anything, how much of the array a size
// needs, so that it can check a size before relying on it.
//
// That array exists once per GPU that loads this library and stays resident
// until the process exits.  Every call on a device uses the same array, so
// calls whose work may overlap on that GPU (different streams, or different
// host threads) race with each other; serialise them.  The array keeps
// whatever the last call left in it; the words that must start at zero are
// cleared by each call with cudaMemsetAsync on the caller's stream.
#include <stdio.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace larosa {
void set_last_error(const char* msg);
}

namespace {

constexpr size_t kScratchBytes = size_t(2) << 20;  // 2 MiB per device
constexpr int kMaxDevices = 64;
constexpr int kMaxDout = 65536;

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_scratch on the current device, looked up once per
// device with that device current (host code cannot use the symbol itself).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

int fail_cuda(cudaError_t e, const char* where) {
  char buf[200];
  snprintf(buf, sizeof(buf), "larosa_sparse_linear_noalloc: %s: %s", where, cudaGetErrorString(e));
  larosa::set_last_error(buf);
  return LAROSA_ERR_CUDA;
}

// Where each piece of the multi-token (or fallback) scratch lies.
struct ScratchLayout {
  bool tensor_core = false;  // 2-16 bf16 tokens: the dense tcgen05 product where larosa_sparse_linear takes it
  size_t off_bitmap = 0, zero_bytes = 0, off_partials = 0, off_coef = 0, off_rows = 0, off_count = 0;
  size_t off_coef_hl = 0;    // tensor_core: the coefficients' bf16 head and tail
  size_t total = 0;  // 0: no scratch (the one-token cluster gather)
};

bool valid_sizes(int M, int d_in, int d_out, int K) {
  return M >= 1 && M <= LAROSA_MAX_M && d_in >= 1 && d_in <= LAROSA_MAX_D && d_out >= 1 &&
         d_out <= kMaxDout && K >= 0 && K <= d_in;
}

// Plans the call on the current device: *sp (one token) and *pl (otherwise)
// and the scratch layout.
cudaError_t plan_noalloc(larosa::Elem w, int M, int d_in, int d_out, int K, larosa::StreamPlan* sp,
                         larosa::GemvPlan* pl, ScratchLayout* S) {
  *S = ScratchLayout{};
  if (M == 1) {
    cudaError_t e = larosa::plan_gather(w, d_out, K, sp);
    if (e != cudaSuccess) return e;
    if (sp->ok) return cudaSuccess;
  }
  if (M > 1 && w == larosa::Elem::BF16 && larosa::umma_gemv_pays(M, d_in, d_out, K)) {
    // [coefficient heads and tails]: every word is written by each call
    S->tensor_core = true;
    S->off_coef_hl = 0;
    S->total = (size_t)2 * M * d_in * 2;
    return cudaSuccess;
  }
  const int n_max = M == 1 ? K : (int)std::min<long long>(d_in, (long long)M * K);
  cudaError_t e = larosa::plan_gemv(w, larosa::Elem::F32, M, d_out, n_max, pl);
  if (e != cudaSuccess) return e;
  // [tickets][bitmap][partials][coef][rows][count]
  const size_t bitmap_words = M > 1 ? (size_t)(d_in + 31) / 32 : 0;
  S->off_bitmap = up256(pl->ticket_words * 4);
  S->zero_bytes = S->off_bitmap + bitmap_words * 4;  // cleared every call
  S->off_partials = up256(S->zero_bytes);
  S->off_coef = up256(S->off_partials + pl->partial_floats * 4);
  S->off_rows = up256(S->off_coef + (M > 1 ? (size_t)M * d_in * 4 : 0));
  S->off_count = up256(S->off_rows + (M > 1 ? (size_t)d_in * 4 : 0));
  S->total = S->off_count + 4;
  return cudaSuccess;
}

}  // namespace

static_assert(kScratchBytes == LAROSA_NOALLOC_SCRATCH_BYTES, "the header states the scratch size");

extern "C" size_t larosa_sparse_linear_noalloc_bytes(int M, int d_in, int d_out, int K, int dtype) {
  if ((dtype != LAROSA_BF16 && dtype != LAROSA_F32) || !valid_sizes(M, d_in, d_out, K)) return 0;
  larosa::StreamPlan sp;
  larosa::GemvPlan pl;
  ScratchLayout S;
  const larosa::Elem w = dtype == LAROSA_BF16 ? larosa::Elem::BF16 : larosa::Elem::F32;
  if (plan_noalloc(w, M, d_in, d_out, K, &sp, &pl, &S) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return S.total;
}

extern "C" int larosa_sparse_linear_noalloc(const int32_t* idx, const float* val, int M, int K,
                                            const void* W_rot, int d_in, int d_out, float* y,
                                            int dtype, int* dev_status, larosa_stream_t stream) {
  if (dtype != LAROSA_BF16 && dtype != LAROSA_F32) return LAROSA_ERR_UNSUPPORTED_DTYPE;
  if (W_rot == nullptr || y == nullptr || (K > 0 && (idx == nullptr || val == nullptr)))
    return LAROSA_ERR_INVALID_ARG;
  if (M < 1 || M > LAROSA_MAX_M || d_in < 1 || d_in > LAROSA_MAX_D || d_out < 1 ||
      d_out > kMaxDout || K < 0 || K > d_in)
    return LAROSA_ERR_SHAPE;
  const int esz = dtype == LAROSA_BF16 ? 2 : 4;
  if ((reinterpret_cast<uintptr_t>(W_rot) & 15u) != 0 ||
      (reinterpret_cast<uintptr_t>(y) & 15u) != 0 || (d_out * esz) % 16 != 0)
    return LAROSA_ERR_ALIGN;

  const larosa::Elem w = dtype == LAROSA_BF16 ? larosa::Elem::BF16 : larosa::Elem::F32;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  larosa::StreamPlan sp;
  larosa::GemvPlan pl;
  ScratchLayout S;
  cudaError_t e = plan_noalloc(w, M, d_in, d_out, K, &sp, &pl, &S);
  if (e != cudaSuccess) return fail_cuda(e, "plan");
  if (larosa::debug_checks()) {
    // the caller's lists, as larosa_sparse_linear checks them (larosa_set_debug)
    e = larosa::launch_check_lists(idx, val, M, K, d_in, false, dev_status, s);
    if (e != cudaSuccess) return fail_cuda(e, "list check kernel");
  }
  if (M == 1 && sp.ok) {
    // one token: the cluster gather keeps its partial sums in distributed
    // shared memory and needs no scratch at all
    larosa::GatherArgs a;
    a.W = W_rot;
    a.d_out = d_out;
    a.row_bound = d_in;
    a.n = K;
    a.coef = val;
    a.rows = idx;
    a.y = y;
    a.dev_status = dev_status;
    e = larosa::launch_gather(w, a, sp, s);
    return e == cudaSuccess ? LAROSA_OK : fail_cuda(e, "sparse linear kernel");
  }
  const int n_max = M == 1 ? K : (int)std::min<long long>(d_in, (long long)M * K);
  const size_t off_bitmap = S.off_bitmap, zero_bytes = S.zero_bytes, off_partials = S.off_partials;
  const size_t off_coef = S.off_coef, off_rows = S.off_rows, off_count = S.off_count;
  const size_t total = S.total;
  if (total > kScratchBytes) {
    char buf[200];
    snprintf(buf, sizeof(buf),
             "larosa_sparse_linear_noalloc: these sizes need %zu bytes of scratch; the static "
             "scratch holds %zu",
             total, kScratchBytes);
    larosa::set_last_error(buf);
    return LAROSA_ERR_WORKSPACE;
  }

  unsigned char* base = nullptr;
  e = scratch_address(reinterpret_cast<void**>(&base));
  if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress");
  if (S.tensor_core) {
    __nv_bfloat16* hl = reinterpret_cast<__nv_bfloat16*>(base + S.off_coef_hl);
    e = larosa::launch_coef_rows(idx, val, M, K, d_in, hl, dev_status, s);
    if (e != cudaSuccess) return fail_cuda(e, "coefficient rows kernel");
    e = larosa::launch_umma_gemv(W_rot, hl, y, M, d_in, d_out, dev_status, s);
    return e == cudaSuccess ? LAROSA_OK : fail_cuda(e, "tensor-core sparse linear kernel");
  }
  e = cudaMemsetAsync(base, 0, zero_bytes, s);
  if (e != cudaSuccess) return fail_cuda(e, "clear scratch");

  larosa::GemvArgs a;
  a.W = W_rot;
  a.w_elem = w;
  a.d_out = d_out;
  a.row_bound = d_in;
  a.coef_elem = larosa::Elem::F32;
  a.M = M;
  a.y = y;
  a.y_ld = d_out;
  a.partials = reinterpret_cast<float*>(base + off_partials);
  a.tickets = reinterpret_cast<unsigned*>(base);
  a.dev_status = dev_status;
  if (M == 1) {
    a.rows = idx;
    a.n_rows = K;
    a.coef = val;
    a.coef_ld = K;
  } else {
    float* coef = reinterpret_cast<float*>(base + off_coef);
    unsigned* bitmap = reinterpret_cast<unsigned*>(base + off_bitmap);
    int32_t* rows = reinterpret_cast<int32_t*>(base + off_rows);
    int* count = reinterpret_cast<int*>(base + off_count);
    e = larosa::launch_scatter(idx, val, M, K, d_in, coef, bitmap, dev_status, s);
    if (e != cudaSuccess) return fail_cuda(e, "scatter kernel");
    e = larosa::launch_union(bitmap, d_in, rows, count, s);
    if (e != cudaSuccess) return fail_cuda(e, "union kernel");
    a.rows = rows;
    a.n_rows = n_max;
    a.n_rows_dev = count;
    a.coef = coef;
    a.coef_ld = d_in;
    a.coef_by_row = 1;
  }
  e = larosa::launch_gemv(a, pl, s);
  return e == cudaSuccess ? LAROSA_OK : fail_cuda(e, "sparse linear kernel");
}
