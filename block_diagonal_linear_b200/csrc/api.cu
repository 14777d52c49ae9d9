// C ABI of libmonarch.so: argument checks, dispatch to the kernel families,
// the device status word and the bounded-wait test hook.
#include <stdint.h>

#include <initializer_list>

#include "common.cuh"
#include "ptx.cuh"
#include "tc_gemm.cuh"

namespace monarch {

// Device status word: kernels that give up a bounded wait store kStatusTimeout.
__device__ int g_status;

int* status_ptr() {
  int* p = nullptr;
  if (cudaGetSymbolAddress((void**)&p, g_status) != cudaSuccess) return nullptr;
  return p;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static int check_dims(const monarch_dims* d) {
  if (d == nullptr) return MONARCH_ERR_NULL;
  if (d->dtype != MONARCH_F32 && d->dtype != MONARCH_BF16) return MONARCH_ERR_DTYPE;
  if (d->rows < 0 || d->nb1 <= 0 || d->in1 <= 0 || d->out1 <= 0 || d->nb2 <= 0 || d->in2 <= 0 ||
      d->out2 <= 0)
    return MONARCH_ERR_DIMS;
  if ((int64_t)d->nb1 * d->out1 != (int64_t)d->nb2 * d->in2) return MONARCH_ERR_DIMS;
  // every flattened size must stay well inside int64 and int32 grid limits
  const int64_t lim = int64_t(1) << 40;
  if ((int64_t)d->nb1 * d->in1 > lim || (int64_t)d->nb1 * d->out1 > lim ||
      (int64_t)d->nb2 * d->out2 > lim)
    return MONARCH_ERR_DIMS;
  return MONARCH_OK;
}

static int check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (p == nullptr) return MONARCH_ERR_NULL;
    if (!aligned16(p)) return MONARCH_ERR_ALIGN;
  }
  return MONARCH_OK;
}

// Byte range of a tensor argument; empty for a null pointer or no elements.
struct Span {
  uintptr_t p;
  uint64_t n;
};
static Span span(const void* p, int64_t elems, int64_t elem_bytes) {
  return {(uintptr_t)p, (p != nullptr && elems > 0) ? (uint64_t)elems * (uint64_t)elem_bytes : 0};
}
static bool overlap(const Span& a, const Span& b) {
  return a.n != 0 && b.n != 0 && a.p < b.p + b.n && b.p < a.p + a.n;
}
// Every output must be disjoint from every input and from every other output: kernels read
// inputs after earlier kernels of the same call have written outputs.
static int check_alias(std::initializer_list<Span> outs, std::initializer_list<Span> ins) {
  for (const Span* o = outs.begin(); o != outs.end(); ++o) {
    for (const Span& i : ins)
      if (overlap(*o, i)) return MONARCH_ERR_ALIAS;
    for (const Span* o2 = o + 1; o2 != outs.end(); ++o2)
      if (overlap(*o, *o2)) return MONARCH_ERR_ALIAS;
  }
  return MONARCH_OK;
}

__global__ void debug_wait_kernel(uint64_t timeout_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on `bar`: the bounded wait must give up
    if (!ptx::mbar_wait_bounded(&bar, 0, timeout_ns)) atomicExch(status, kStatusTimeout);
  }
  __syncthreads();
}

cudaError_t debug_wait_timeout(uint64_t timeout_ns, int* status, cudaStream_t st) {
  return launch_kernel(debug_wait_kernel, dim3(1), dim3(32), 0, st, false, timeout_ns, status);
}

// 0 = generic FMA kernels, 1 = tcgen05 group kernel, 2 = tcgen05 row-tile kernel,
// 3 = tcgen05 row-tile kernel with the L stage in rounds of output columns,
// 4 = tcgen05 block-diagonal GEMMs and row permutations as separate passes over Y.
int fwd_path(const Shape& s, int dtype) {
  if (dtype != MONARCH_BF16) return 0;
  if (tc_rows_supported(s)) return 2;
  if (tc_wide_supported(s)) return 3;
  if (tc_split_supported(s)) return 4;
  if (tc_fwd_supported(s)) return 1;
  return 0;
}

// 0 = generic FMA kernels, 1 = row-tile / block-GEMM passes with tcgen05 weight gradients,
// 2 = tcgen05 GEMM passes (permutation folded into 64-column gathers), 3 = packed
// block-diagonal tcgen05 GEMM passes with row-transpose passes for the permutations.
int bwd_path(const Shape& s, int dtype) {
  if (dtype != MONARCH_BF16) return 0;
  if (fast_bwd_supported(s)) return 1;
  if (gemm_bwd_supported(s)) return 2;
  if (packed_bwd_supported(s)) return 3;
  return 0;
}

size_t bwd_workspace(const Shape& s, int dtype) {
  switch (bwd_path(s, dtype)) {
    case 1: return fast_bwd_workspace(s);
    case 2: return gemm_bwd_workspace(s);
    case 3: return packed_bwd_workspace(s);
    default: return generic_bwd_workspace(s);
  }
}

// Forward on already-checked arguments (rows > 0).
int fwd_dispatch(const void* X, const void* R, const void* L, void* Y, const Shape& s, int dtype, cudaStream_t st) {
  cudaError_t e;
  const int path = fwd_path(s, dtype);
  if (path != 0) {
    int* status = status_ptr();
    if (status == nullptr) return MONARCH_ERR_CUDA;
    e = path == 2   ? tc_rows_fwd(X, R, L, Y, s, status, st)
        : path == 3 ? tc_wide_fwd(X, R, L, Y, s, status, st)
        : path == 4 ? tc_split_fwd(X, R, L, Y, s, status, st)
                    : tc_fwd(X, R, L, Y, s, status, st);
  } else {
    if (!generic_fwd_supported(s)) return MONARCH_ERR_UNSUPPORTED;
    e = generic_fwd(X, R, L, Y, s, dtype, st);
  }
  return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}

// Backward on already-checked arguments (workspace of bwd_workspace(s, dtype) bytes).
int bwd_dispatch(const void* dY, const void* X, const void* R, const void* L, void* dX, void* dR, void* dL,
                 void* ws, const Shape& s, int dtype, cudaStream_t st, const void* saved) {
  cudaError_t e;
  const int path = bwd_path(s, dtype);
  if (path != 0) {
    int* status = status_ptr();
    if (status == nullptr) return MONARCH_ERR_CUDA;
    e = path == 1   ? fast_bwd(dY, X, R, L, dX, dR, dL, ws, s, status, st, saved)
        : path == 2 ? gemm_bwd(dY, X, R, L, dX, dR, dL, ws, s, status, st, saved)
                    : packed_bwd(dY, X, R, L, dX, dR, dL, ws, s, status, st, saved);
  } else {
    if (!generic_bwd_supported(s)) return MONARCH_ERR_UNSUPPORTED;
    e = generic_bwd(dY, X, R, L, dX, dR, dL, ws, s, dtype, st);
  }
  return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}

}  // namespace monarch

using namespace monarch;

extern "C" {

int monarch_validate(const monarch_dims* d) { return check_dims(d); }

int monarch_fwd_path(const monarch_dims* d) {
  if (check_dims(d) != MONARCH_OK) return -1;
  return fwd_path(to_shape(*d), d->dtype);
}

int monarch_bwd_path(const monarch_dims* d) {
  if (check_dims(d) != MONARCH_OK) return -1;
  return bwd_path(to_shape(*d), d->dtype);
}

int monarch_fwd(const void* X, const void* R, const void* L, const monarch_dims* d, void* Y,
                void* stream) {
  int rc = check_dims(d);
  if (rc != MONARCH_OK) return rc;
  if (d->rows == 0) return MONARCH_OK;
  if ((rc = check_ptrs({X, R, L, Y})) != MONARCH_OK) return rc;
  const Shape s = to_shape(*d);
  const int64_t es = d->dtype == MONARCH_BF16 ? 2 : 4;
  if ((rc = check_alias({span(Y, s.rows * s.n_out(), es)},
                        {span(X, s.rows * s.n_in(), es), span(R, s.n_R(), es), span(L, s.n_L(), es)})) !=
      MONARCH_OK)
    return rc;
  return fwd_dispatch(X, R, L, Y, s, d->dtype, (cudaStream_t)stream);
}

// Forward with caller scratch: the two-pass tcgen05 GEMM forward where it applies (shapes
// whose permutation moves whole 64-column groups), two streaming stage launches for the
// square small-block shapes, otherwise the monarch_fwd kernels.
static int fwd_ws_kind(const Shape& s, int dtype) {
  if (dtype != MONARCH_BF16) return 0;
  if (gemm_bwd_supported(s)) return 5;
  if (tc_stage_fwd_supported(s)) return 6;
  return 0;
}

static size_t fwd_ws_bytes(const Shape& s, int dtype) {
  switch (fwd_ws_kind(s, dtype)) {
    case 5: return gemm_fwd_workspace(s);
    case 6: return (size_t)s.rows * (size_t)s.n_mid() * 2;
    default: return 0;
  }
}

size_t monarch_fwd_workspace_bytes(const monarch_dims* d) {
  if (check_dims(d) != MONARCH_OK) return 0;
  return fwd_ws_bytes(to_shape(*d), d->dtype);
}

int monarch_fwd_ws_path(const monarch_dims* d) {
  if (check_dims(d) != MONARCH_OK) return -1;
  const Shape s = to_shape(*d);
  const int k = fwd_ws_kind(s, d->dtype);
  return k != 0 ? k : fwd_path(s, d->dtype);
}

int monarch_fwd_ws(const void* X, const void* R, const void* L, const monarch_dims* d, void* Y, void* workspace,
                   size_t workspace_bytes, void* stream) {
  int rc = check_dims(d);
  if (rc != MONARCH_OK) return rc;
  if (d->rows == 0) return MONARCH_OK;
  if ((rc = check_ptrs({X, R, L, Y})) != MONARCH_OK) return rc;
  const Shape s = to_shape(*d);
  const size_t need = fwd_ws_bytes(s, d->dtype);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return MONARCH_ERR_WORKSPACE;
  if (need > 0 && ((uintptr_t)workspace & 255u) != 0) return MONARCH_ERR_ALIGN;
  const int64_t es = d->dtype == MONARCH_BF16 ? 2 : 4;
  if ((rc = check_alias({span(Y, s.rows * s.n_out(), es), span(workspace, (int64_t)need, 1)},
                        {span(X, s.rows * s.n_in(), es), span(R, s.n_R(), es), span(L, s.n_L(), es)})) !=
      MONARCH_OK)
    return rc;
  if (need == 0) return fwd_dispatch(X, R, L, Y, s, d->dtype, (cudaStream_t)stream);
  int* status = status_ptr();
  if (status == nullptr) return MONARCH_ERR_CUDA;
  const cudaError_t e = fwd_ws_kind(s, d->dtype) == 5
                            ? gemm_fwd(X, R, L, Y, workspace, s, status, (cudaStream_t)stream)
                            : tc_stage_fwd(X, R, L, Y, workspace, s, status, (cudaStream_t)stream);
  return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}

// What the training forward leaves for the backward: 2 = Z from the fused row-tile forward,
// 3 = Z from the wide-output forward (for the packed backward's streaming stages), 5 = the
// two-pass GEMM forward's workspace (U), 6 = the streaming stages' Z; 0 = nothing (the backward
// recomputes the middle vector).
static int saved_kind(const Shape& s, int dtype) {
  if (dtype != MONARCH_BF16) return 0;
  const int k = fwd_ws_kind(s, dtype);
  if (k == 5 || k == 6) return k;
  if (fwd_path(s, dtype) == 2 && bwd_path(s, dtype) == 1) return 2;
  if (fwd_path(s, dtype) == 3 && bwd_path(s, dtype) == 3 && tc_stage_supported(s)) return 3;
  return 0;
}

static size_t saved_bytes(const Shape& s, int dtype) {
  switch (saved_kind(s, dtype)) {
    case 2:
    case 3:
    case 6: return (size_t)s.rows * (size_t)s.n_mid() * 2;
    case 5: return gemm_fwd_workspace(s);
    default: return 0;
  }
}

size_t monarch_saved_bytes(const monarch_dims* d) {
  if (check_dims(d) != MONARCH_OK) return 0;
  return saved_bytes(to_shape(*d), d->dtype);
}

int monarch_fwd_train(const void* X, const void* R, const void* L, const monarch_dims* d, void* Y, void* saved,
                      size_t saved_bytes_, void* stream) {
  int rc = check_dims(d);
  if (rc != MONARCH_OK) return rc;
  if (d->rows == 0) return MONARCH_OK;
  if ((rc = check_ptrs({X, R, L, Y})) != MONARCH_OK) return rc;
  const Shape s = to_shape(*d);
  const size_t need = saved_bytes(s, d->dtype);
  if (need > 0 && (saved == nullptr || saved_bytes_ < need)) return MONARCH_ERR_WORKSPACE;
  if (need > 0 && ((uintptr_t)saved & 255u) != 0) return MONARCH_ERR_ALIGN;
  const int64_t es = d->dtype == MONARCH_BF16 ? 2 : 4;
  if ((rc = check_alias({span(Y, s.rows * s.n_out(), es), span(saved, (int64_t)need, 1)},
                        {span(X, s.rows * s.n_in(), es), span(R, s.n_R(), es), span(L, s.n_L(), es)})) !=
      MONARCH_OK)
    return rc;
  const cudaStream_t st = (cudaStream_t)stream;
  const int kind = saved_kind(s, d->dtype);
  if (kind == 0) return fwd_dispatch(X, R, L, Y, s, d->dtype, st);
  int* status = status_ptr();
  if (status == nullptr) return MONARCH_ERR_CUDA;
  const cudaError_t e = kind == 2   ? tc_rows_fwd_save(X, R, L, Y, saved, s, status, st)
                        : kind == 3 ? tc_wide_fwd_save(X, R, L, Y, saved, s, status, st)
                        : kind == 5 ? gemm_fwd(X, R, L, Y, saved, s, status, st)
                                    : tc_stage_fwd(X, R, L, Y, saved, s, status, st);
  return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}

int monarch_bwd_saved(const void* dY, const void* X, const void* R, const void* L, const monarch_dims* d,
                      const void* saved, size_t saved_bytes_, void* dX, void* dR, void* dL, void* workspace,
                      size_t workspace_bytes, void* stream) {
  int rc = check_dims(d);
  if (rc != MONARCH_OK) return rc;
  if ((rc = check_ptrs({R, L, dR, dL})) != MONARCH_OK) return rc;
  if (d->rows > 0 && (rc = check_ptrs({dY, X, dX})) != MONARCH_OK) return rc;
  const Shape s = to_shape(*d);
  const size_t need_saved = saved_bytes(s, d->dtype);
  if (need_saved > 0 && (saved == nullptr || saved_bytes_ < need_saved)) return MONARCH_ERR_WORKSPACE;
  if (need_saved > 0 && ((uintptr_t)saved & 255u) != 0) return MONARCH_ERR_ALIGN;
  const size_t need = bwd_workspace(s, d->dtype);
  if (workspace == nullptr || workspace_bytes < need) return MONARCH_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255u) != 0) return MONARCH_ERR_ALIGN;
  const int64_t es = d->dtype == MONARCH_BF16 ? 2 : 4;
  if ((rc = check_alias({span(dX, s.rows * s.n_in(), es), span(dR, s.n_R(), es), span(dL, s.n_L(), es),
                         span(workspace, (int64_t)need, 1)},
                        {span(dY, s.rows * s.n_out(), es), span(X, s.rows * s.n_in(), es),
                         span(R, s.n_R(), es), span(L, s.n_L(), es), span(saved, (int64_t)need_saved, 1)})) !=
      MONARCH_OK)
    return rc;
  return bwd_dispatch(dY, X, R, L, dX, dR, dL, workspace, s, d->dtype, (cudaStream_t)stream,
                      need_saved > 0 ? saved : nullptr);
}

size_t monarch_bwd_workspace_bytes(const monarch_dims* d) {
  if (check_dims(d) != MONARCH_OK) return 0;
  return bwd_workspace(to_shape(*d), d->dtype);
}

int monarch_bwd(const void* dY, const void* X, const void* R, const void* L, const monarch_dims* d,
                void* dX, void* dR, void* dL, void* workspace, size_t workspace_bytes,
                void* stream) {
  int rc = check_dims(d);
  if (rc != MONARCH_OK) return rc;
  if ((rc = check_ptrs({R, L, dR, dL})) != MONARCH_OK) return rc;
  if (d->rows > 0 && (rc = check_ptrs({dY, X, dX})) != MONARCH_OK) return rc;
  const Shape s = to_shape(*d);
  const size_t need = bwd_workspace(s, d->dtype);
  if (workspace == nullptr || workspace_bytes < need) return MONARCH_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255u) != 0) return MONARCH_ERR_ALIGN;
  const int64_t es = d->dtype == MONARCH_BF16 ? 2 : 4;
  if ((rc = check_alias({span(dX, s.rows * s.n_in(), es), span(dR, s.n_R(), es), span(dL, s.n_L(), es),
                         span(workspace, (int64_t)need, 1)},
                        {span(dY, s.rows * s.n_out(), es), span(X, s.rows * s.n_in(), es),
                         span(R, s.n_R(), es), span(L, s.n_L(), es)})) != MONARCH_OK)
    return rc;
  return bwd_dispatch(dY, X, R, L, dX, dR, dL, workspace, s, d->dtype, (cudaStream_t)stream);
}

int monarch_materialise(const void* R, const void* L, const monarch_dims* d, void* M,
                        void* stream) {
  int rc = check_dims(d);
  if (rc != MONARCH_OK) return rc;
  if ((rc = check_ptrs({R, L, M})) != MONARCH_OK) return rc;
  const Shape ms = to_shape(*d);
  const int64_t es = d->dtype == MONARCH_BF16 ? 2 : 4;
  if ((rc = check_alias({span(M, ms.n_out() * ms.n_in(), 4)}, {span(R, ms.n_R(), es), span(L, ms.n_L(), es)})) !=
      MONARCH_OK)
    return rc;
  cudaError_t e = generic_materialise(R, L, (float*)M, to_shape(*d), d->dtype, (cudaStream_t)stream);
  return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}

const char* monarch_status_string(int status) {
  switch (status) {
    case MONARCH_OK: return "ok";
    case MONARCH_ERR_DIMS: return "invalid Monarch dims";
    case MONARCH_ERR_DTYPE: return "unsupported dtype";
    case MONARCH_ERR_ALIGN: return "pointer not 16-byte aligned";
    case MONARCH_ERR_NULL: return "null pointer";
    case MONARCH_ERR_WORKSPACE: return "workspace missing or too small";
    case MONARCH_ERR_CUDA: return "CUDA error";
    case MONARCH_ERR_TIMEOUT: return "bounded device wait timed out";
    case MONARCH_ERR_UNSUPPORTED: return "shape not supported by any kernel";
    case MONARCH_ERR_SCRATCH: return "problem larger than the fixed scratch of monarch_bwd_noalloc";
    case MONARCH_ERR_ALIAS: return "an output or the workspace overlaps another argument";
    default: return "unknown status";
  }
}

int monarch_last_device_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MONARCH_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return MONARCH_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return MONARCH_ERR_CUDA;
  return v == kStatusTimeout ? MONARCH_ERR_TIMEOUT : MONARCH_OK;
}

uint64_t monarch_kernel_launches(void) { return launch_counter().load(std::memory_order_relaxed); }

int monarch_debug_wait_timeout(uint64_t timeout_ns, void* stream) {
  int* status = status_ptr();
  if (status == nullptr) return MONARCH_ERR_CUDA;
  return debug_wait_timeout(timeout_ns, status, (cudaStream_t)stream) == cudaSuccess
             ? MONARCH_OK
             : MONARCH_ERR_CUDA;
}

}  // extern "C"
