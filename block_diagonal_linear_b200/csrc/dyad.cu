// DYAD (DYAD abstract: a sum of two matrices, each permutable to a block-sparse counterpart,
// stored as 3-D tensors).  Reading taken, with the reshape-transpose of the Monarch pages:
//   y = BD(W1) x + P_out^T BD(W2) P_in x,
//   (P_in x)[i*nb + k] = x[k*in_blk + i],  (P_out^T v)[k*out_blk + a] = v[a*nb + k],
// W1, W2: (nb, out_blk, in_blk); BD: block-diagonal product on contiguous slices.
//
// bf16 with packable blocks (tensor cores): P_in X and P_out dY are row-transpose passes,
// both block-diagonal stages are packed tcgen05 GEMMs (tc_gemm.cu), the second term's
// output transpose and the sum are one permute-add pass, and the weight gradients are the
// tcgen05 weight-gradient GEMM over the rows (fp32 partials, fixed-order sum).
// Otherwise (fp32, other shapes): generic FMA kernels, one output (or parameter) per thread.
#include "common.cuh"
#include "tc_common.cuh"
#include "tc_gemm.cuh"

namespace monarch {

struct DyadShape {
  int64_t rows;
  int nb, ib, ob;
};

static bool dyad_shape(const monarch_dyad_dims& dd, DyadShape* s) {
  if (dd.rows < 0 || dd.nblocks <= 0 || dd.in_blk <= 0 || dd.out_blk <= 0) return false;
  if ((int64_t)dd.nblocks * dd.in_blk > (1 << 24) || (int64_t)dd.nblocks * dd.out_blk > (1 << 24)) return false;
  s->rows = dd.rows;
  s->nb = dd.nblocks;
  s->ib = dd.in_blk;
  s->ob = dd.out_blk;
  return true;
}

static bool dyad_tc(const DyadShape& s, int dtype) {
  if (dtype != MONARCH_BF16) return false;
  if (s.nb % 8 || s.ib % 8 || s.ob % 8) return false;  // row-transpose passes
  if (pack_factor(s.nb, s.ib, s.ob) == 0 || pack_factor(s.nb, s.ob, s.ib) == 0) return false;
  const int64_t n_in = (int64_t)s.nb * s.ib, n_out = (int64_t)s.nb * s.ob;
  if (n_in > 65536 || n_out > 65536) return false;
  if ((int64_t)s.nb * (s.ib + 2) * 2 > 200 * 1024 || (int64_t)s.ob * (s.nb + 2) * 2 > 200 * 1024 ||
      (int64_t)s.nb * (s.ob + 2) * 2 > 200 * 1024 || (int64_t)s.ib * (s.nb + 2) * 2 > 200 * 1024)
    return false;
  return true;
}

// ---------------------------------------------------------------- generic kernels
template <typename T>
__global__ void dyad_generic_fwd_kernel(const T* __restrict__ X, const T* __restrict__ W1, const T* __restrict__ W2,
                                        T* __restrict__ Y, DyadShape s) {
  const int64_t n_in = (int64_t)s.nb * s.ib, n_out = (int64_t)s.nb * s.ob, total = s.rows * n_out;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / n_out, c = e % n_out;
    const T* x = X + r * n_in;
    const int k = (int)(c / s.ob), o = (int)(c % s.ob);
    float acc = 0.f;
    for (int i = 0; i < s.ib; ++i) acc = fmaf(ld_as_f32(W1 + ((int64_t)k * s.ob + o) * s.ib + i), ld_as_f32(x + (int64_t)k * s.ib + i), acc);
    // second term at output c = k*ob + a: v index a*nb + k = j*ob + o2; P_in x at t = j*ib + q
    const int64_t sv = (int64_t)o * s.nb + k;
    const int j = (int)(sv / s.ob), o2 = (int)(sv % s.ob);
    for (int q = 0; q < s.ib; ++q) {
      const int64_t t = (int64_t)j * s.ib + q;
      const int64_t src = (t % s.nb) * s.ib + t / s.nb;
      acc = fmaf(ld_as_f32(W2 + ((int64_t)j * s.ob + o2) * s.ib + q), ld_as_f32(x + src), acc);
    }
    st_from_f32(Y + e, acc);
  }
}

template <typename T>
__global__ void dyad_generic_dx_kernel(const T* __restrict__ dY, const T* __restrict__ W1, const T* __restrict__ W2,
                                       T* __restrict__ dX, DyadShape s) {
  const int64_t n_in = (int64_t)s.nb * s.ib, n_out = (int64_t)s.nb * s.ob, total = s.rows * n_in;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / n_in, c = e % n_in;
    const T* dy = dY + r * n_out;
    const int k = (int)(c / s.ib), i = (int)(c % s.ib);
    float acc = 0.f;
    for (int o = 0; o < s.ob; ++o) acc = fmaf(ld_as_f32(W1 + ((int64_t)k * s.ob + o) * s.ib + i), ld_as_f32(dy + (int64_t)k * s.ob + o), acc);
    // x[c] feeds P_in x at t = i*nb + k = j*ib + q; dv[j*ob + o2] = dy[((j*ob + o2) % nb)*ob + (j*ob + o2) / nb]
    const int64_t t = (int64_t)i * s.nb + k;
    const int j = (int)(t / s.ib), q = (int)(t % s.ib);
    for (int o2 = 0; o2 < s.ob; ++o2) {
      const int64_t sv = (int64_t)j * s.ob + o2;
      acc = fmaf(ld_as_f32(W2 + ((int64_t)j * s.ob + o2) * s.ib + q), ld_as_f32(dy + (sv % s.nb) * s.ob + sv / s.nb), acc);
    }
    st_from_f32(dX + e, acc);
  }
}

// dW1[k][o][i] = sum_r dY[r][k*ob + o] X[r][k*ib + i];  dW2[j][o2][q] = sum_r dv[r][j*ob + o2] PX[r][j*ib + q]
template <typename T>
__global__ void dyad_generic_dw_kernel(const T* __restrict__ dY, const T* __restrict__ X, T* __restrict__ dW1,
                                       T* __restrict__ dW2, DyadShape s) {
  const int64_t nW = (int64_t)s.nb * s.ob * s.ib;
  const int64_t n_in = (int64_t)s.nb * s.ib, n_out = (int64_t)s.nb * s.ob;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= 2 * nW) return;
  const int64_t f = e % nW;
  const int b = (int)(f / ((int64_t)s.ob * s.ib)), o = (int)((f / s.ib) % s.ob), i = (int)(f % s.ib);
  int64_t ycol, xcol;
  if (e < nW) {
    ycol = (int64_t)b * s.ob + o;
    xcol = (int64_t)b * s.ib + i;
  } else {
    const int64_t sv = (int64_t)b * s.ob + o, t = (int64_t)b * s.ib + i;
    ycol = (sv % s.nb) * s.ob + sv / s.nb;
    xcol = (t % s.nb) * s.ib + t / s.nb;
  }
  float acc = 0.f;
  for (int64_t r = 0; r < s.rows; ++r) acc = fmaf(ld_as_f32(dY + r * n_out + ycol), ld_as_f32(X + r * n_in + xcol), acc);
  st_from_f32((e < nW ? dW1 : dW2) + f, acc);
}

// ---------------------------------------------------------------- workspace
static size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

struct DyadWs {
  size_t w1p, w2p, w1tp, w2tp, px, v, part, total;
  WgradSplit sp;
};

static DyadWs dyad_layout(const DyadShape& s, int dtype) {
  DyadWs w = {};
  if (!dyad_tc(s, dtype)) return w;  // the generic kernels need no workspace
  const int g1 = pack_factor(s.nb, s.ib, s.ob), g2 = pack_factor(s.nb, s.ob, s.ib);
  const size_t rows = (size_t)s.rows, n_in = (size_t)s.nb * s.ib, n_out = (size_t)s.nb * s.ob;
  const size_t wp = (size_t)s.nb * s.ob * g1 * s.ib * 2, wtp = (size_t)s.nb * s.ib * g2 * s.ob * 2;
  int64_t units = 0;
  for (int t = 0; t < 2; ++t) {  // weight-gradient units per split, as wgrad_tc forms them
    int64_t bpg = 1;
    if (s.ob <= 128 && 128 % s.ob == 0 && s.nb % (128 / s.ob) == 0) bpg = 128 / s.ob;
    const int64_t nw = bpg * s.ib, bn = nw >= 256 ? 256 : (nw > 64 ? 128 : 64);
    units += (s.nb / bpg) * ((s.ob + 127) / 128) * ((nw + bn - 1) / bn);
  }
  w.sp = wgrad_split(s.rows, units);
  w.w1p = 0;
  w.w2p = w.w1p + al256(wp);
  w.w1tp = w.w2p + al256(wp);
  w.w2tp = w.w1tp + al256(wtp);
  w.px = w.w2tp + al256(wtp);
  w.v = w.px + al256(rows * n_in * 2);
  w.part = w.v + al256(rows * (n_out > n_in ? n_out : n_in) * 2);
  w.total = w.part + al256((size_t)w.sp.nsplit * 2 * (size_t)s.nb * s.ob * s.ib * 4);
  return w;
}

}  // namespace monarch

using namespace monarch;

extern "C" {

size_t monarch_dyad_workspace_bytes(const monarch_dyad_dims* dd) {
  DyadShape s;
  if (dd == nullptr || (dd->dtype != MONARCH_F32 && dd->dtype != MONARCH_BF16) || !dyad_shape(*dd, &s)) return 0;
  const size_t t = dyad_layout(s, dd->dtype).total;
  return t > 0 ? t : 256;
}

int monarch_dyad_path(const monarch_dyad_dims* dd) {
  DyadShape s;
  if (dd == nullptr || (dd->dtype != MONARCH_F32 && dd->dtype != MONARCH_BF16) || !dyad_shape(*dd, &s)) return -1;
  return dyad_tc(s, dd->dtype) ? 1 : 0;
}

static int dyad_check(const monarch_dyad_dims* dd, DyadShape* s, void* ws, size_t bytes, DyadWs* w) {
  if (dd == nullptr) return MONARCH_ERR_NULL;
  if (dd->dtype != MONARCH_F32 && dd->dtype != MONARCH_BF16) return MONARCH_ERR_DTYPE;
  if (!dyad_shape(*dd, s)) return MONARCH_ERR_DIMS;
  *w = dyad_layout(*s, dd->dtype);
  if (w->total > 0 && (ws == nullptr || bytes < w->total)) return MONARCH_ERR_WORKSPACE;
  if (w->total > 0 && ((uintptr_t)ws & 255u) != 0) return MONARCH_ERR_ALIGN;
  return MONARCH_OK;
}

struct Rg {
  uintptr_t b, e;
};
static Rg rg(const void* p, int64_t n) { return Rg{(uintptr_t)p, (uintptr_t)p + (uint64_t)(p ? n : 0)}; }
static bool ov(const Rg& a, const Rg& b) { return a.e > a.b && b.e > b.b && a.b < b.e && b.b < a.e; }
static bool any_overlap(std::initializer_list<Rg> outs, std::initializer_list<Rg> ins) {
  for (const Rg* o = outs.begin(); o != outs.end(); ++o) {
    for (const Rg& i : ins)
      if (ov(*o, i)) return true;
    for (const Rg* o2 = o + 1; o2 != outs.end(); ++o2)
      if (ov(*o, *o2)) return true;
  }
  return false;
}

int monarch_dyad_fwd(const void* X, const void* W1, const void* W2, const monarch_dyad_dims* dd, void* Y,
                     void* workspace, size_t workspace_bytes, void* stream) {
  DyadShape s;
  DyadWs w;
  int rc = dyad_check(dd, &s, workspace, workspace_bytes, &w);
  if (rc != MONARCH_OK) return rc;
  if (s.rows == 0) return MONARCH_OK;
  for (const void* p : std::initializer_list<const void*>{X, W1, W2, Y}) {
    if (p == nullptr) return MONARCH_ERR_NULL;
    if (!aligned16(p)) return MONARCH_ERR_ALIGN;
  }
  const int64_t es = dd->dtype == MONARCH_BF16 ? 2 : 4;
  const int64_t n_in = (int64_t)s.nb * s.ib, n_out = (int64_t)s.nb * s.ob, nW = (int64_t)s.nb * s.ob * s.ib;
  if (any_overlap({rg(Y, s.rows * n_out * es), rg(workspace, (int64_t)w.total)},
                  {rg(X, s.rows * n_in * es), rg(W1, nW * es), rg(W2, nW * es)}))
    return MONARCH_ERR_ALIAS;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (!dyad_tc(s, dd->dtype)) {
    const dim3 grid(4 * 148), block(256);
    e = dd->dtype == MONARCH_BF16
            ? launch_kernel(dyad_generic_fwd_kernel<__nv_bfloat16>, grid, block, 0, st, false, (const __nv_bfloat16*)X,
                            (const __nv_bfloat16*)W1, (const __nv_bfloat16*)W2, (__nv_bfloat16*)Y, s)
            : launch_kernel(dyad_generic_fwd_kernel<float>, grid, block, 0, st, false, (const float*)X,
                            (const float*)W1, (const float*)W2, (float*)Y, s);
    return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
  }
  int* status = status_ptr();
  if (status == nullptr) return MONARCH_ERR_CUDA;
  char* ws = (char*)workspace;
  const int g1 = pack_factor(s.nb, s.ib, s.ob);
  void *W1p = ws + w.w1p, *W2p = ws + w.w2p, *PX = ws + w.px, *V = ws + w.v;
  if ((e = pack_bd(W1, W1p, s.nb, s.ob, s.ib, g1, false, st)) != cudaSuccess ||
      (e = pack_bd(W2, W2p, s.nb, s.ob, s.ib, g1, false, st)) != cudaSuccess ||
      (e = permute_rows(X, PX, s.rows, s.nb, s.ib, st)) != cudaSuccess ||
      (e = packed_stage(PX, s.rows, W2p, V, s.nb, s.ib, s.ob, g1, status, st)) != cudaSuccess ||
      (e = packed_stage(X, s.rows, W1p, Y, s.nb, s.ib, s.ob, g1, status, st)) != cudaSuccess ||
      (e = permute_rows_add(V, Y, s.rows, s.ob, s.nb, st)) != cudaSuccess)
    return MONARCH_ERR_CUDA;
  return MONARCH_OK;
}

int monarch_dyad_bwd(const void* dY, const void* X, const void* W1, const void* W2, const monarch_dyad_dims* dd,
                     void* dX, void* dW1, void* dW2, void* workspace, size_t workspace_bytes, void* stream) {
  DyadShape s;
  DyadWs w;
  int rc = dyad_check(dd, &s, workspace, workspace_bytes, &w);
  if (rc != MONARCH_OK) return rc;
  for (const void* p : std::initializer_list<const void*>{W1, W2, dW1, dW2}) {
    if (p == nullptr) return MONARCH_ERR_NULL;
    if (!aligned16(p)) return MONARCH_ERR_ALIGN;
  }
  if (s.rows > 0)
    for (const void* p : std::initializer_list<const void*>{dY, X, dX}) {
      if (p == nullptr) return MONARCH_ERR_NULL;
      if (!aligned16(p)) return MONARCH_ERR_ALIGN;
    }
  const int64_t es = dd->dtype == MONARCH_BF16 ? 2 : 4;
  const int64_t n_in = (int64_t)s.nb * s.ib, n_out = (int64_t)s.nb * s.ob, nW = (int64_t)s.nb * s.ob * s.ib;
  if (any_overlap({rg(dX, s.rows * n_in * es), rg(dW1, nW * es), rg(dW2, nW * es), rg(workspace, (int64_t)w.total)},
                  {rg(dY, s.rows * n_out * es), rg(X, s.rows * n_in * es), rg(W1, nW * es), rg(W2, nW * es)}))
    return MONARCH_ERR_ALIAS;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (!dyad_tc(s, dd->dtype)) {
    const dim3 grid(4 * 148), block(256), wgrid((unsigned)((2 * nW + 255) / 256));
    if (dd->dtype == MONARCH_BF16) {
      using T = __nv_bfloat16;
      if (s.rows > 0 && (e = launch_kernel(dyad_generic_dx_kernel<T>, grid, block, 0, st, false, (const T*)dY,
                                           (const T*)W1, (const T*)W2, (T*)dX, s)) != cudaSuccess)
        return MONARCH_ERR_CUDA;
      e = launch_kernel(dyad_generic_dw_kernel<T>, wgrid, block, 0, st, false, (const T*)dY, (const T*)X, (T*)dW1,
                        (T*)dW2, s);
    } else {
      using T = float;
      if (s.rows > 0 && (e = launch_kernel(dyad_generic_dx_kernel<T>, grid, block, 0, st, false, (const T*)dY,
                                           (const T*)W1, (const T*)W2, (T*)dX, s)) != cudaSuccess)
        return MONARCH_ERR_CUDA;
      e = launch_kernel(dyad_generic_dw_kernel<T>, wgrid, block, 0, st, false, (const T*)dY, (const T*)X, (T*)dW1,
                        (T*)dW2, s);
    }
    return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
  }
  int* status = status_ptr();
  if (status == nullptr) return MONARCH_ERR_CUDA;
  char* ws = (char*)workspace;
  const int g2 = pack_factor(s.nb, s.ob, s.ib);
  void *W1tp = ws + w.w1tp, *W2tp = ws + w.w2tp, *PX = ws + w.px, *DV = ws + w.v;
  float* part = (float*)(ws + w.part);
  if (s.rows > 0) {
    // dv = P_out dY (dv[a*nb + k] = dY[k*ob + a]);  dPX = BD(W2^T) dv -> PX's buffer;  dX = BD(W1^T) dY;
    // dX += P_in^T dPX;  then PX = P_in X for dW2
    if ((e = pack_bd(W1, W1tp, s.nb, s.ib, s.ob, g2, true, st)) != cudaSuccess ||
        (e = pack_bd(W2, W2tp, s.nb, s.ib, s.ob, g2, true, st)) != cudaSuccess ||
        (e = permute_rows(dY, DV, s.rows, s.nb, s.ob, st)) != cudaSuccess ||
        (e = packed_stage(DV, s.rows, W2tp, PX, s.nb, s.ob, s.ib, g2, status, st)) != cudaSuccess ||
        (e = packed_stage(dY, s.rows, W1tp, dX, s.nb, s.ob, s.ib, g2, status, st)) != cudaSuccess ||
        (e = permute_rows_add(PX, dX, s.rows, s.ib, s.nb, st)) != cudaSuccess ||
        (e = permute_rows(X, PX, s.rows, s.nb, s.ib, st)) != cudaSuccess)
      return MONARCH_ERR_CUDA;
    const WgradArgs g1 = {dY, n_out, s.ob, X, n_in, s.ib, s.nb, 0, 0, 0, w.sp, 2 * nW, 0};
    const WgradArgs g2 = {DV, n_out, s.ob, PX, n_in, s.ib, s.nb, 0, 0, 0, w.sp, 2 * nW, nW};
    if ((e = wgrad_tc2(g1, g2, s.rows, part, status, st)) != cudaSuccess) return MONARCH_ERR_CUDA;
  } else if ((e = cudaMemsetAsync(part, 0, sizeof(float) * (size_t)w.sp.nsplit * 2 * nW, st)) != cudaSuccess) {
    return MONARCH_ERR_CUDA;
  }
  e = launch_kernel(reduce_partials_kernel, dim3((unsigned)((2 * nW + 255) / 256)), dim3(256), 0, st, true,
                    (const float*)part, (__nv_bfloat16*)dW1, (__nv_bfloat16*)dW2, nW, 2 * nW, w.sp.nsplit);
  return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}

}  // extern "C"
