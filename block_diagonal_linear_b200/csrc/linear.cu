// MonarchLinear front end: any (in_features, out_features, nblocks), with the factor shapes of
// the MonarchLinear __init__ listing (scatterbrain issue thread), zero padding of the inputs to
// the extended widths, cropping of the outputs, and an optional bias.
//
// Forward:  Xp = [X, 0] (rows x in_ext)  ->  Yp = Monarch(Xp)  ->  Y = Yp[:, :out] + bias.
// Backward: dYp = [dY, 0] -> (dXp, dR, dL) = Monarch backward -> dX = dXp[:, :in];
//           dbias = sum over rows of dY.
// Shapes whose permutation moves whole 64-column groups (e.g. 1024 -> 4096 with 4 blocks) run
// the two-pass tcgen05 GEMM forward with the middle vector in the workspace.
// The padding passes are skipped when the features already equal the extended widths, and
// the output goes through a staging buffer only when it is cropped or gets a bias (the crop
// and the bias add are one pass that rounds once).  The Monarch stages run on the same
// kernel families as monarch_fwd / monarch_bwd.
#include <algorithm>

#include "common.cuh"
#include "ptx.cuh"
#include "tc_gemm.cuh"

namespace monarch {

static bool lin_shape(const monarch_linear_dims& ld, Shape* s) {
  if (ld.in_features <= 0 || ld.out_features <= 0 || ld.nblocks <= 0 || ld.rows < 0) return false;
  const int64_t in_blk = ((int64_t)ld.in_features + ld.nblocks - 1) / ld.nblocks;
  const int64_t out_blk = ((int64_t)ld.out_features + ld.nblocks - 1) / ld.nblocks;
  const int64_t mid = in_blk * ld.nblocks < out_blk * ld.nblocks ? in_blk : out_blk;
  if (in_blk > (1 << 20) || out_blk > (1 << 20)) return false;
  s->rows = ld.rows;
  s->nb1 = s->nb2 = ld.nblocks;
  s->in1 = (int)in_blk;
  s->out1 = s->in2 = (int)mid;
  s->out2 = (int)out_blk;
  s->out_transpose = 0;
  return true;
}

template <typename T>
__global__ void pad_cols_kernel(const T* __restrict__ src, int64_t cols, T* __restrict__ dst, int64_t dcols,
                                int64_t rows) {
  const int64_t n = rows * dcols;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / dcols, c = e % dcols;
    dst[e] = c < cols ? src[r * cols + c] : T(0.f);
  }
}

// dst[r][c] = src[r][c] (+ bias[c]) for c < dcols, src having scols >= dcols columns; rounding once.
template <typename T>
__global__ void crop_bias_kernel(const T* __restrict__ src, int64_t scols, const T* __restrict__ bias,
                                 T* __restrict__ dst, int64_t dcols, int64_t rows) {
  const int64_t n = rows * dcols;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / dcols, c = e % dcols;
    float v = ld_as_f32(src + r * scols + c);
    if (bias != nullptr) v += ld_as_f32(bias + c);
    st_from_f32(dst + e, v);
  }
}

// Column sums of dY over row chunks (fp32 partials), then a fixed-order sum of the chunks.
constexpr int kBiasChunk = 1024;
template <typename T>
__global__ void bias_partial_kernel(const T* __restrict__ dY, int64_t cols, int64_t rows, float* __restrict__ part) {
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int64_t r0 = (int64_t)blockIdx.y * kBiasChunk;
  const int64_t r1 = r0 + kBiasChunk < rows ? r0 + kBiasChunk : rows;
  float acc = 0.f;
  for (int64_t r = r0; r < r1; ++r) acc += ld_as_f32(dY + r * cols + c);
  part[(int64_t)blockIdx.y * cols + c] = acc;
}

template <typename T>
__global__ void bias_reduce_kernel(const float* __restrict__ part, int64_t cols, int nchunks, T* __restrict__ dbias) {
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  float acc = 0.f;
  for (int k = 0; k < nchunks; ++k) acc += part[(int64_t)k * cols + c];
  st_from_f32(dbias + c, acc);
}

static size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

struct LinWs {
  size_t xp, yp, dxp, core, bias, total;
};

static LinWs lin_layout(const monarch_linear_dims& ld, const Shape& s) {
  const size_t es = ld.dtype == MONARCH_BF16 ? 2 : 4;
  const size_t rows = (size_t)s.rows;
  const bool pad_in = ld.in_features != s.n_in(), pad_out = ld.out_features != s.n_out();
  LinWs w;
  w.xp = 0;
  w.yp = w.xp + (pad_in ? al256(rows * (size_t)s.n_in() * es) : 0);
  // forward: cropped / biased output staging; backward: padded dY
  w.dxp = w.yp + ((pad_out || ld.has_bias) ? al256(rows * (size_t)s.n_out() * es) : 0);
  w.core = w.dxp + (pad_in ? al256(rows * (size_t)s.n_in() * es) : 0);
  const bool two_pass = ld.dtype == MONARCH_BF16 && gemm_bwd_supported(s);
  w.bias = w.core + al256(std::max(bwd_workspace(s, ld.dtype), two_pass ? gemm_fwd_workspace(s) : (size_t)0));
  const size_t nchunks = (rows + kBiasChunk - 1) / kBiasChunk;
  w.total = w.bias + al256((nchunks > 0 ? nchunks : 1) * (size_t)ld.out_features * 4);
  return w;
}

template <typename T>
static cudaError_t launch_pad(const void* src, int64_t cols, void* dst, int64_t dcols, int64_t rows, cudaStream_t st) {
  return launch_kernel(pad_cols_kernel<T>, dim3(2 * 148), dim3(256), 0, st, false, (const T*)src, cols, (T*)dst,
                       dcols, rows);
}
template <typename T>
static cudaError_t launch_crop(const void* src, int64_t scols, const void* bias, void* dst, int64_t dcols,
                               int64_t rows, cudaStream_t st) {
  return launch_kernel(crop_bias_kernel<T>, dim3(2 * 148), dim3(256), 0, st, false, (const T*)src, scols,
                       (const T*)bias, (T*)dst, dcols, rows);
}
template <typename T>
static cudaError_t launch_dbias(const void* dY, int64_t cols, int64_t rows, float* part, void* dbias,
                                cudaStream_t st) {
  const int nchunks = (int)((rows + kBiasChunk - 1) / kBiasChunk);
  cudaError_t e;
  if (nchunks > 0 &&
      (e = launch_kernel(bias_partial_kernel<T>, dim3((unsigned)((cols + 255) / 256), (unsigned)nchunks), dim3(256),
                         0, st, false, (const T*)dY, cols, rows, part)) != cudaSuccess)
    return e;
  if (nchunks == 0 && (e = cudaMemsetAsync(part, 0, (size_t)cols * 4, st)) != cudaSuccess) return e;
  return launch_kernel(bias_reduce_kernel<T>, dim3((unsigned)((cols + 255) / 256)), dim3(256), 0, st, false,
                       (const float*)part, cols, nchunks > 0 ? nchunks : 1, (T*)dbias);
}

}  // namespace monarch

using namespace monarch;

extern "C" {

int monarch_linear_shape(const monarch_linear_dims* ld, monarch_dims* d) {
  if (ld == nullptr || d == nullptr) return MONARCH_ERR_NULL;
  if (ld->dtype != MONARCH_F32 && ld->dtype != MONARCH_BF16) return MONARCH_ERR_DTYPE;
  Shape s;
  if (!lin_shape(*ld, &s)) return MONARCH_ERR_DIMS;
  d->rows = s.rows;
  d->nb1 = s.nb1; d->in1 = s.in1; d->out1 = s.out1;
  d->nb2 = s.nb2; d->in2 = s.in2; d->out2 = s.out2;
  d->out_transpose = 0;
  d->dtype = ld->dtype;
  return monarch_validate(d);
}

size_t monarch_linear_workspace_bytes(const monarch_linear_dims* ld) {
  monarch_dims d;
  if (monarch_linear_shape(ld, &d) != MONARCH_OK) return 0;
  return lin_layout(*ld, to_shape(d)).total;
}

int monarch_linear_fwd(const void* X, const void* R, const void* L, const void* bias, const monarch_linear_dims* ld,
                       void* Y, void* workspace, size_t workspace_bytes, void* stream) {
  monarch_dims d;
  int rc = monarch_linear_shape(ld, &d);
  if (rc != MONARCH_OK) return rc;
  if (ld->rows == 0) return MONARCH_OK;
  if (X == nullptr || R == nullptr || L == nullptr || Y == nullptr || (ld->has_bias && bias == nullptr))
    return MONARCH_ERR_NULL;
  if (!aligned16(X) || !aligned16(R) || !aligned16(L) || !aligned16(Y) || (ld->has_bias && !aligned16(bias)))
    return MONARCH_ERR_ALIGN;
  const Shape s = to_shape(d);
  const LinWs w = lin_layout(*ld, s);
  if (workspace == nullptr || workspace_bytes < w.total) return MONARCH_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255u) != 0) return MONARCH_ERR_ALIGN;
  const int64_t es = ld->dtype == MONARCH_BF16 ? 2 : 4;
  const int64_t rows = ld->rows;
  const uintptr_t Yb = (uintptr_t)Y, Ye = Yb + (uint64_t)rows * ld->out_features * es;
  const uintptr_t Wb = (uintptr_t)workspace, We = Wb + w.total;
  auto hits = [&](const void* p, int64_t n) {
    const uintptr_t b = (uintptr_t)p, e = b + (uint64_t)n * es;
    return (b < Ye && Yb < e) || (b < We && Wb < e);
  };
  if (hits(X, rows * ld->in_features) || hits(R, s.n_R()) || hits(L, s.n_L()) ||
      (ld->has_bias && hits(bias, ld->out_features)) || (Yb < We && Wb < Ye))
    return MONARCH_ERR_ALIAS;
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  const bool pad_in = ld->in_features != s.n_in();
  const bool stage_out = ld->out_features != s.n_out() || ld->has_bias;
  const bool bf = ld->dtype == MONARCH_BF16;
  const void* Xp = X;
  if (pad_in) {
    Xp = ws + w.xp;
    cudaError_t e = bf ? launch_pad<__nv_bfloat16>(X, ld->in_features, ws + w.xp, s.n_in(), rows, st)
                       : launch_pad<float>(X, ld->in_features, ws + w.xp, s.n_in(), rows, st);
    if (e != cudaSuccess) return MONARCH_ERR_CUDA;
  }
  void* Yp = stage_out ? (void*)(ws + w.yp) : Y;
  if (ld->dtype == MONARCH_BF16 && gemm_bwd_supported(s)) {
    // two-pass tcgen05 GEMM forward with the middle vector in the workspace
    int* status = status_ptr();
    if (status == nullptr) return MONARCH_ERR_CUDA;
    if (gemm_fwd(Xp, R, L, Yp, ws + w.core, s, status, st) != cudaSuccess) return MONARCH_ERR_CUDA;
  } else if ((rc = fwd_dispatch(Xp, R, L, Yp, s, ld->dtype, st)) != MONARCH_OK) {
    return rc;
  }
  if (stage_out) {
    const void* b = ld->has_bias ? bias : nullptr;
    cudaError_t e = bf ? launch_crop<__nv_bfloat16>(Yp, s.n_out(), b, Y, ld->out_features, rows, st)
                       : launch_crop<float>(Yp, s.n_out(), b, Y, ld->out_features, rows, st);
    if (e != cudaSuccess) return MONARCH_ERR_CUDA;
  }
  return MONARCH_OK;
}

int monarch_linear_bwd(const void* dY, const void* X, const void* R, const void* L, const monarch_linear_dims* ld,
                       void* dX, void* dR, void* dL, void* dbias, void* workspace, size_t workspace_bytes,
                       void* stream) {
  monarch_dims d;
  int rc = monarch_linear_shape(ld, &d);
  if (rc != MONARCH_OK) return rc;
  if (R == nullptr || L == nullptr || dR == nullptr || dL == nullptr || (ld->has_bias && dbias == nullptr))
    return MONARCH_ERR_NULL;
  if (ld->rows > 0 && (dY == nullptr || X == nullptr || dX == nullptr)) return MONARCH_ERR_NULL;
  for (const void* p : std::initializer_list<const void*>{dY, X, R, L, dX, dR, dL, dbias})
    if (p != nullptr && !aligned16(p)) return MONARCH_ERR_ALIGN;
  const Shape s = to_shape(d);
  const LinWs w = lin_layout(*ld, s);
  if (workspace == nullptr || workspace_bytes < w.total) return MONARCH_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255u) != 0) return MONARCH_ERR_ALIGN;
  const int64_t es = ld->dtype == MONARCH_BF16 ? 2 : 4;
  const int64_t rows = ld->rows;
  struct Rg { uintptr_t b, e; };
  auto rg = [&](const void* p, int64_t n) { return Rg{(uintptr_t)p, (uintptr_t)p + (uint64_t)(p ? n : 0) * es}; };
  const Rg outs[5] = {rg(dX, rows * ld->in_features), rg(dR, s.n_R()), rg(dL, s.n_L()),
                      rg(ld->has_bias ? dbias : nullptr, ld->out_features), {(uintptr_t)workspace, (uintptr_t)workspace + w.total}};
  const Rg ins[4] = {rg(dY, rows * ld->out_features), rg(X, rows * ld->in_features), rg(R, s.n_R()), rg(L, s.n_L())};
  auto ov = [](const Rg& a, const Rg& b) { return a.e > a.b && b.e > b.b && a.b < b.e && b.b < a.e; };
  for (int i = 0; i < 5; ++i) {
    for (int k = 0; k < 4; ++k)
      if (ov(outs[i], ins[k])) return MONARCH_ERR_ALIAS;
    for (int k = i + 1; k < 5; ++k)
      if (ov(outs[i], outs[k])) return MONARCH_ERR_ALIAS;
  }
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  const bool bf = ld->dtype == MONARCH_BF16;
  const bool pad_in = ld->in_features != s.n_in(), pad_out = ld->out_features != s.n_out();
  const void* Xp = X;
  const void* dYp = dY;
  void* dXp = dX;
  cudaError_t e;
  if (rows > 0 && pad_in) {
    Xp = ws + w.xp;
    dXp = ws + w.dxp;
    e = bf ? launch_pad<__nv_bfloat16>(X, ld->in_features, ws + w.xp, s.n_in(), rows, st)
           : launch_pad<float>(X, ld->in_features, ws + w.xp, s.n_in(), rows, st);
    if (e != cudaSuccess) return MONARCH_ERR_CUDA;
  }
  if (rows > 0 && pad_out) {
    dYp = ws + w.yp;
    e = bf ? launch_pad<__nv_bfloat16>(dY, ld->out_features, ws + w.yp, s.n_out(), rows, st)
           : launch_pad<float>(dY, ld->out_features, ws + w.yp, s.n_out(), rows, st);
    if (e != cudaSuccess) return MONARCH_ERR_CUDA;
  }
  if ((rc = bwd_dispatch(dYp, Xp, R, L, dXp, dR, dL, ws + w.core, s, ld->dtype, st)) != MONARCH_OK) return rc;
  if (rows > 0 && pad_in) {
    e = bf ? launch_crop<__nv_bfloat16>(dXp, s.n_in(), nullptr, dX, ld->in_features, rows, st)
           : launch_crop<float>(dXp, s.n_in(), nullptr, dX, ld->in_features, rows, st);
    if (e != cudaSuccess) return MONARCH_ERR_CUDA;
  }
  if (ld->has_bias) {
    e = bf ? launch_dbias<__nv_bfloat16>(dY, ld->out_features, rows, (float*)(ws + w.bias), dbias, st)
           : launch_dbias<float>(dY, ld->out_features, rows, (float*)(ws + w.bias), dbias, st);
    if (e != cudaSuccess) return MONARCH_ERR_CUDA;
  }
  return MONARCH_OK;
}

}  // extern "C"
