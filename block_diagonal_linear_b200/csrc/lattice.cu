// Lattice (hypercube) Monarch (scatterbrain thread, the unofficial-implementation comment: a
// row of width n viewed as a d-dimensional lattice, one round of per-line matrices per
// dimension; e.g. 12288 = 16 x 24 x 32 with 768, 512 and 384 matrices).  Rounds run from the
// last (contiguous) axis to the first; round t maps axis t from n_t to m_t; its matrices
// W_t (lines, m_t, n_t) are indexed by the row-major position of the line in the other axes
// (axes already done count with their new lengths).  With two axes this is the two-factor
// product with the output transpose.
//
// bf16 with packable lines (tensor cores): round t is a per-row transpose that moves axis t
// last (P x n_t x B -> P x B x n_t, P and B the products of the axes before and after t),
// a packed tcgen05 block-diagonal stage over the lines, and the transpose back; the last axis
// needs no transposes.  The backward keeps each round's transposed input, runs the rounds in
// reverse with W_t^T, and takes the weight gradients with the tcgen05 weight-gradient GEMM.
// Otherwise (fp32, other shapes): one generic FMA kernel per round, fp32 intermediates.
#include "common.cuh"
#include "tc_common.cuh"
#include "tc_gemm.cuh"

namespace monarch {

constexpr int kMaxAxes = 4;

struct LatShape {
  int64_t rows;
  int d;
  int n[kMaxAxes], m[kMaxAxes];
};

// Lengths of the axes just before round t (axes > t already mapped to m).
static void dims_before(const LatShape& s, int t, int* cur) {
  for (int a = 0; a < s.d; ++a) cur[a] = a > t ? s.m[a] : s.n[a];
}
static int64_t prod(const int* v, int lo, int hi) {
  int64_t p = 1;
  for (int a = lo; a < hi; ++a) p *= v[a];
  return p;
}
static int64_t lines_of(const LatShape& s, int t) {
  int cur[kMaxAxes];
  dims_before(s, t, cur);
  return prod(cur, 0, s.d) / cur[t];
}
static int64_t wsize(const LatShape& s, int t) { return lines_of(s, t) * s.m[t] * s.n[t]; }

static bool lat_shape(const monarch_lattice_dims& ld, LatShape* s) {
  if (ld.rows < 0 || ld.naxes < 1 || ld.naxes > kMaxAxes) return false;
  s->rows = ld.rows;
  s->d = ld.naxes;
  int64_t ni = 1, no = 1;
  for (int a = 0; a < ld.naxes; ++a) {
    if (ld.n_in[a] <= 0 || ld.n_out[a] <= 0) return false;
    s->n[a] = ld.n_in[a];
    s->m[a] = ld.n_out[a];
    ni *= ld.n_in[a];
    no *= ld.n_out[a];
  }
  if (ni > (1 << 24) || no > (1 << 24)) return false;
  // lattice sizes at every round must stay below 2^24 too
  for (int t = s->d - 1; t >= 0; --t) {
    int cur[kMaxAxes];
    dims_before(*s, t, cur);
    if (prod(cur, 0, s->d) > (1 << 24)) return false;
  }
  return true;
}

static bool lat_tc(const LatShape& s, int dtype) {
  if (dtype != MONARCH_BF16 || s.d < 2) return false;
  for (int t = 0; t < s.d; ++t) {
    int cur[kMaxAxes];
    dims_before(s, t, cur);
    const int64_t B = prod(cur, t + 1, s.d), lines = lines_of(s, t);
    if (lines > (1 << 30)) return false;
    if (pack_factor((int)lines, s.n[t], s.m[t]) == 0 || pack_factor((int)lines, s.m[t], s.n[t]) == 0) return false;
    if (s.n[t] % 8 || s.m[t] % 8 || (B > 1 && B % 8)) return false;  // 16-byte TMA x, row-transpose passes
    if (B > 1 && ((int64_t)s.n[t] * (B + 2) * 2 > 200 * 1024 || (int64_t)B * (s.m[t] + 2) * 2 > 200 * 1024 ||
                  (int64_t)s.m[t] * (B + 2) * 2 > 200 * 1024 || (int64_t)B * (s.n[t] + 2) * 2 > 200 * 1024))
      return false;  // one staged row of each transpose must fit in shared memory
    if ((int64_t)pack_factor((int)lines, s.n[t], s.m[t]) * s.n[t] > 4096) return false;
  }
  return true;
}

// ---------------------------------------------------------------- generic round
struct RoundArgs {
  int64_t rows, in_size, out_size;
  int d, t, mt;
  int cur[kMaxAxes];  // lengths before the round
};

template <typename Tin, typename Tw, typename Tout>
__global__ void lattice_round_kernel(const Tin* __restrict__ in, const Tw* __restrict__ W, Tout* __restrict__ out,
                                     RoundArgs a) {
  const int64_t total = a.rows * a.out_size;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / a.out_size;
    int64_t idx = e % a.out_size;
    int c[kMaxAxes];
    for (int s = a.d - 1; s >= 0; --s) {
      const int len = s == a.t ? a.mt : a.cur[s];
      c[s] = (int)(idx % len);
      idx /= len;
    }
    int64_t line = 0, base = 0, stride = 1;
    for (int s = 0; s < a.d; ++s)
      if (s != a.t) line = line * a.cur[s] + c[s];
    for (int s = a.d - 1; s >= 0; --s) {  // input offset with c[t] = 0, and axis t's stride
      if (s == a.t) {
        stride = 1;
        for (int q = s + 1; q < a.d; ++q) stride *= a.cur[q];
      }
    }
    for (int s = 0; s < a.d; ++s) base = base * a.cur[s] + (s == a.t ? 0 : c[s]);
    const Tin* x = in + r * a.in_size + base;
    const Tw* w = W + (line * a.mt + c[a.t]) * a.cur[a.t];
    float acc = 0.f;
    for (int i = 0; i < a.cur[a.t]; ++i) acc = fmaf(ld_as_f32(w + i), ld_as_f32(x + (int64_t)i * stride), acc);
    st_from_f32(out + e, acc);
  }
}

// dW_t[line][b][a] = sum_r G[r][.. b ..] In[r][.. a ..]   (one parameter per thread, rows in order)
template <typename Tw>
__global__ void lattice_dw_kernel(const float* __restrict__ G, const float* __restrict__ In, Tw* __restrict__ dW,
                                  RoundArgs a, int64_t nw) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nw) return;
  const int nt = a.cur[a.t];
  const int ai = (int)(e % nt), bo = (int)((e / nt) % a.mt);
  int64_t line = e / ((int64_t)nt * a.mt);
  int c[kMaxAxes];
  for (int s = a.d - 1; s >= 0; --s) {
    if (s == a.t) continue;
    c[s] = (int)(line % a.cur[s]);
    line /= a.cur[s];
  }
  int64_t gi = 0, xi = 0;
  for (int s = 0; s < a.d; ++s) {
    gi = gi * (s == a.t ? a.mt : a.cur[s]) + (s == a.t ? bo : c[s]);
    xi = xi * a.cur[s] + (s == a.t ? ai : c[s]);
  }
  float acc = 0.f;
  for (int64_t r = 0; r < a.rows; ++r) acc = fmaf(G[r * a.out_size + gi], In[r * a.in_size + xi], acc);
  st_from_f32(dW + e, acc);
}

// dIn[r][.. a ..] = sum_b W_t[line][b][a] G[r][.. b ..]
template <typename Tw, typename Tout>
__global__ void lattice_dx_kernel(const float* __restrict__ G, const Tw* __restrict__ W, Tout* __restrict__ dIn,
                                  RoundArgs a) {
  const int64_t total = a.rows * a.in_size;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / a.in_size;
    int64_t idx = e % a.in_size;
    int c[kMaxAxes];
    for (int s = a.d - 1; s >= 0; --s) {
      c[s] = (int)(idx % a.cur[s]);
      idx /= a.cur[s];
    }
    int64_t line = 0, base = 0, stride = 1;
    for (int s = 0; s < a.d; ++s)
      if (s != a.t) line = line * a.cur[s] + c[s];
    for (int q = a.t + 1; q < a.d; ++q) stride *= a.cur[q];
    for (int s = 0; s < a.d; ++s) base = base * (s == a.t ? a.mt : a.cur[s]) + (s == a.t ? 0 : c[s]);
    const float* g = G + r * a.out_size + base;
    const Tw* w = W + line * a.mt * a.cur[a.t] + c[a.t];
    float acc = 0.f;
    for (int b = 0; b < a.mt; ++b) acc = fmaf(ld_as_f32(w + (int64_t)b * a.cur[a.t]), g[(int64_t)b * stride], acc);
    st_from_f32(dIn + e, acc);
  }
}

template <typename T>
__global__ void widen_kernel(const T* __restrict__ src, float* __restrict__ dst, int64_t n) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
    dst[e] = ld_as_f32(src + e);
}

// Sum of fp32 partials over the splits into one weight tensor (fixed order).
__global__ void lattice_reduce_kernel(const float* __restrict__ part, int64_t p_stride, int64_t off, int nsplit,
                                      __nv_bfloat16* __restrict__ dW, int64_t n) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  float acc = 0.f;
  for (int k = 0; k < nsplit; ++k) acc += part[(int64_t)k * p_stride + off + e];
  dW[e] = __float2bfloat16_rn(acc);
}

static RoundArgs round_args(const LatShape& s, int t) {
  RoundArgs a;
  a.rows = s.rows;
  a.d = s.d;
  a.t = t;
  a.mt = s.m[t];
  dims_before(s, t, a.cur);
  a.in_size = prod(a.cur, 0, s.d);
  a.out_size = a.in_size / a.cur[t] * a.mt;
  return a;
}

// ---------------------------------------------------------------- workspace
static size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

struct LatWs {
  size_t buf[2];          // ping-pong lattices (fp32 generic, bf16 tensor path)
  size_t keep[kMaxAxes];  // per-round inputs kept for the backward (axis t last on the tensor path)
  size_t wpk, part, total;
  int64_t maxlat, wpk_bytes, nparams;
  WgradSplit sp;
};

static LatWs lat_layout(const LatShape& s, int dtype) {
  LatWs w = {};
  const bool tc = lat_tc(s, dtype);
  const size_t es = tc ? 2 : 4;
  int64_t maxlat = prod(s.n, 0, s.d);
  for (int t = s.d - 1; t >= 0; --t) maxlat = std::max<int64_t>(maxlat, round_args(s, t).out_size);
  w.maxlat = maxlat;
  size_t off = 0;
  for (int i = 0; i < 2; ++i) {
    w.buf[i] = off;
    off += al256((size_t)s.rows * maxlat * es);
  }
  for (int t = 0; t < s.d; ++t) {
    w.keep[t] = off;
    off += al256((size_t)s.rows * round_args(s, t).in_size * es);
  }
  // packed weights of the largest round (forward and transposed use the same size bound)
  int64_t wp = 0, np = 0, units = 0;
  for (int t = 0; t < s.d; ++t) {
    const int64_t lines = lines_of(s, t);
    np += wsize(s, t);
    if (tc) {
      const int g1 = pack_factor((int)lines, s.n[t], s.m[t]), g2 = pack_factor((int)lines, s.m[t], s.n[t]);
      wp = std::max<int64_t>(wp, std::max<int64_t>(lines * s.m[t] * g1 * s.n[t], lines * s.n[t] * g2 * s.m[t]));
      int64_t bpg = 1;
      if (s.m[t] <= 128 && 128 % s.m[t] == 0 && lines % (128 / s.m[t]) == 0) bpg = 128 / s.m[t];
      const int64_t nw = bpg * s.n[t], bn = nw >= 256 ? 256 : (nw > 64 ? 128 : 64);
      units = std::max<int64_t>(units, (lines / bpg) * ((s.m[t] + 127) / 128) * ((nw + bn - 1) / bn));
    }
  }
  w.nparams = np;
  w.wpk = off;
  w.wpk_bytes = wp * 2;
  off += al256((size_t)wp * 2);
  w.sp = wgrad_split(s.rows, units > 0 ? units : 1);
  w.part = off;
  if (tc) off += al256((size_t)w.sp.nsplit * np * 4);
  w.total = off;
  return w;
}

template <typename T>
static cudaError_t lat_generic_fwd(const LatShape& s, const void* X, const void* const* W, void* Y, char* ws,
                                   const LatWs& w, cudaStream_t st) {
  const dim3 grid(4 * 148), block(256);
  const float* cur = nullptr;
  int pp = 0;
  for (int t = s.d - 1; t >= 0; --t) {
    const RoundArgs a = round_args(s, t);
    cudaError_t e;
    if (t == 0) {
      e = t == s.d - 1 ? launch_kernel(lattice_round_kernel<T, T, T>, grid, block, 0, st, false, (const T*)X,
                                       (const T*)W[t], (T*)Y, a)
                       : launch_kernel(lattice_round_kernel<float, T, T>, grid, block, 0, st, false, cur,
                                       (const T*)W[t], (T*)Y, a);
    } else {
      float* out = (float*)(ws + w.buf[pp]);
      e = t == s.d - 1 ? launch_kernel(lattice_round_kernel<T, T, float>, grid, block, 0, st, false, (const T*)X,
                                       (const T*)W[t], out, a)
                       : launch_kernel(lattice_round_kernel<float, T, float>, grid, block, 0, st, false, cur,
                                       (const T*)W[t], out, a);
      cur = out;
      pp ^= 1;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename T>
static cudaError_t lat_generic_bwd(const LatShape& s, const void* dY, const void* X, const void* const* W, void* dX,
                                   void* const* dW, char* ws, const LatWs& w, cudaStream_t st) {
  const dim3 grid(4 * 148), block(256);
  cudaError_t e;
  // forward again, keeping every round's input (fp32)
  float* in = (float*)(ws + w.keep[s.d - 1]);
  if ((e = launch_kernel(widen_kernel<T>, grid, block, 0, st, false, (const T*)X, in,
                         s.rows * prod(s.n, 0, s.d))) != cudaSuccess)
    return e;
  for (int t = s.d - 1; t >= 1; --t) {
    float* out = (float*)(ws + w.keep[t - 1]);
    if ((e = launch_kernel(lattice_round_kernel<float, T, float>, grid, block, 0, st, false,
                           (const float*)(ws + w.keep[t]), (const T*)W[t], out, round_args(s, t))) != cudaSuccess)
      return e;
  }
  // G = dY, rounds in reverse (t = 0 .. d-1)
  float* G = (float*)(ws + w.buf[0]);
  if ((e = launch_kernel(widen_kernel<T>, grid, block, 0, st, false, (const T*)dY, G, s.rows * prod(s.m, 0, s.d))) !=
      cudaSuccess)
    return e;
  int pp = 1;
  for (int t = 0; t < s.d; ++t) {
    const RoundArgs a = round_args(s, t);
    const int64_t nw = wsize(s, t);
    if ((e = launch_kernel(lattice_dw_kernel<T>, dim3((unsigned)((nw + 255) / 256)), block, 0, st, false,
                           (const float*)G, (const float*)(ws + w.keep[t]), (T*)dW[t], a, nw)) != cudaSuccess)
      return e;
    if (s.rows == 0) continue;
    if (t == s.d - 1) {
      e = launch_kernel(lattice_dx_kernel<T, T>, grid, block, 0, st, false, (const float*)G, (const T*)W[t], (T*)dX, a);
    } else {
      float* Gn = (float*)(ws + w.buf[pp]);
      e = launch_kernel(lattice_dx_kernel<T, float>, grid, block, 0, st, false, (const float*)G, (const T*)W[t], Gn, a);
      G = Gn;
      pp ^= 1;
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// The workspace lattice buffer that is not p (buf[0] when p is neither).
static void* other_buf(char* ws, const LatWs& w, const void* p) {
  return p == (const void*)(ws + w.buf[0]) ? (void*)(ws + w.buf[1]) : (void*)(ws + w.buf[0]);
}

// Tensor-core forward.  With kept != nullptr (backward): kept[t] receives each round's input
// with axis t last (X itself for the last axis; keep[t] buffers otherwise) and the last
// round's output is not formed.
static cudaError_t lat_tc_fwd(const LatShape& s, const void* X, const void* const* W, void* Y, char* ws,
                              const LatWs& w, int* status, cudaStream_t st, const void** kept) {
  const void* cur = X;  // canonical lattice before the round (a workspace buffer after round d-1)
  for (int t = s.d - 1; t >= 0; --t) {
    const RoundArgs a = round_args(s, t);
    const int64_t P = prod(a.cur, 0, t), B = prod(a.cur, t + 1, s.d), lines = P * B;
    const bool need_out = !(kept != nullptr && t == 0);
    cudaError_t e;
    if (B == 1) {
      if (kept) kept[t] = cur;
      if (!need_out) break;
    } else {
      void* T1 = kept ? (void*)(ws + w.keep[t]) : other_buf(ws, w, cur);
      if ((e = permute_rows(cur, T1, s.rows * P, s.n[t], (int)B, st)) != cudaSuccess) return e;
      if (kept) kept[t] = T1;
      if (!need_out) break;
    }
    const int g = pack_factor((int)lines, s.n[t], s.m[t]);
    void* Wp = ws + w.wpk;
    if ((e = pack_bd(W[t], Wp, (int)lines, s.m[t], s.n[t], g, false, st)) != cudaSuccess) return e;
    if (B == 1) {
      void* dst = t == 0 ? Y : other_buf(ws, w, cur);
      if ((e = packed_stage(cur, s.rows, Wp, dst, (int)lines, s.n[t], s.m[t], g, status, st)) != cudaSuccess) return e;
      cur = dst;
    } else {
      const void* T1 = kept ? kept[t] : other_buf(ws, w, cur);
      // cur's buffer is free once transposed (never X here: the last axis runs first, B == 1)
      void* T2 = kept ? other_buf(ws, w, cur) : (void*)cur;
      if ((e = packed_stage(T1, s.rows, Wp, T2, (int)lines, s.n[t], s.m[t], g, status, st)) != cudaSuccess) return e;
      void* dst = t == 0 ? Y : (kept ? (void*)cur : (void*)T1);
      if ((e = permute_rows(T2, dst, s.rows * P, (int)B, s.m[t], st)) != cudaSuccess) return e;
      cur = dst;
    }
  }
  return cudaSuccess;
}

}  // namespace monarch

using namespace monarch;

extern "C" {

size_t monarch_lattice_workspace_bytes(const monarch_lattice_dims* ld) {
  LatShape s;
  if (ld == nullptr || (ld->dtype != MONARCH_F32 && ld->dtype != MONARCH_BF16) || !lat_shape(*ld, &s)) return 0;
  return lat_layout(s, ld->dtype).total;
}

int monarch_lattice_path(const monarch_lattice_dims* ld) {
  LatShape s;
  if (ld == nullptr || (ld->dtype != MONARCH_F32 && ld->dtype != MONARCH_BF16) || !lat_shape(*ld, &s)) return -1;
  return lat_tc(s, ld->dtype) ? 1 : 0;
}

int64_t monarch_lattice_weight_elems(const monarch_lattice_dims* ld, int32_t axis) {
  LatShape s;
  if (ld == nullptr || !lat_shape(*ld, &s) || axis < 0 || axis >= s.d) return -1;
  return wsize(s, axis);
}

static int lat_check(const monarch_lattice_dims* ld, LatShape* s, void* ws, size_t bytes, LatWs* w) {
  if (ld == nullptr) return MONARCH_ERR_NULL;
  if (ld->dtype != MONARCH_F32 && ld->dtype != MONARCH_BF16) return MONARCH_ERR_DTYPE;
  if (!lat_shape(*ld, s)) return MONARCH_ERR_DIMS;
  *w = lat_layout(*s, ld->dtype);
  if (ws == nullptr || bytes < w->total) return MONARCH_ERR_WORKSPACE;
  if (((uintptr_t)ws & 255u) != 0) return MONARCH_ERR_ALIGN;
  return MONARCH_OK;
}

int monarch_lattice_fwd(const void* X, const void* const* W, const monarch_lattice_dims* ld, void* Y, void* workspace,
                        size_t workspace_bytes, void* stream) {
  LatShape s;
  LatWs w;
  int rc = lat_check(ld, &s, workspace, workspace_bytes, &w);
  if (rc != MONARCH_OK) return rc;
  if (s.rows == 0) return MONARCH_OK;
  if (X == nullptr || Y == nullptr || W == nullptr) return MONARCH_ERR_NULL;
  if (!aligned16(X) || !aligned16(Y)) return MONARCH_ERR_ALIGN;
  for (int t = 0; t < s.d; ++t) {
    if (W[t] == nullptr) return MONARCH_ERR_NULL;
    if (!aligned16(W[t])) return MONARCH_ERR_ALIGN;
  }
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (lat_tc(s, ld->dtype)) {
    int* status = status_ptr();
    if (status == nullptr) return MONARCH_ERR_CUDA;
    e = lat_tc_fwd(s, X, W, Y, (char*)workspace, w, status, st, nullptr);
  } else {
    e = ld->dtype == MONARCH_BF16 ? lat_generic_fwd<__nv_bfloat16>(s, X, W, Y, (char*)workspace, w, st)
                                  : lat_generic_fwd<float>(s, X, W, Y, (char*)workspace, w, st);
  }
  return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
}

int monarch_lattice_bwd(const void* dY, const void* X, const void* const* W, const monarch_lattice_dims* ld, void* dX,
                        void* const* dW, void* workspace, size_t workspace_bytes, void* stream) {
  LatShape s;
  LatWs w;
  int rc = lat_check(ld, &s, workspace, workspace_bytes, &w);
  if (rc != MONARCH_OK) return rc;
  if (W == nullptr || dW == nullptr) return MONARCH_ERR_NULL;
  for (int t = 0; t < s.d; ++t) {
    if (W[t] == nullptr || dW[t] == nullptr) return MONARCH_ERR_NULL;
    if (!aligned16(W[t]) || !aligned16(dW[t])) return MONARCH_ERR_ALIGN;
  }
  if (s.rows > 0 && (dY == nullptr || X == nullptr || dX == nullptr)) return MONARCH_ERR_NULL;
  cudaStream_t st = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  cudaError_t e;
  if (!lat_tc(s, ld->dtype)) {
    e = ld->dtype == MONARCH_BF16 ? lat_generic_bwd<__nv_bfloat16>(s, dY, X, W, dX, dW, ws, w, st)
                                  : lat_generic_bwd<float>(s, dY, X, W, dX, dW, ws, w, st);
    return e == cudaSuccess ? MONARCH_OK : MONARCH_ERR_CUDA;
  }
  int* status = status_ptr();
  if (status == nullptr) return MONARCH_ERR_CUDA;
  float* part = (float*)(ws + w.part);
  const void* kept[kMaxAxes] = {};
  if (s.rows == 0) {
    if ((e = cudaMemsetAsync(part, 0, sizeof(float) * (size_t)w.sp.nsplit * w.nparams, st)) != cudaSuccess)
      return MONARCH_ERR_CUDA;
  } else if ((e = lat_tc_fwd(s, X, W, nullptr, ws, w, status, st, kept)) != cudaSuccess) {
    return MONARCH_ERR_CUDA;
  }
  // rounds in reverse: G (canonical, lengths after the round) -> dW_t and the round's input gradient
  const void* G = dY;
  int64_t poff = 0;
  for (int t = 0; t < s.d && s.rows > 0; ++t) {
    const RoundArgs a = round_args(s, t);
    const int64_t P = prod(a.cur, 0, t), B = prod(a.cur, t + 1, s.d), lines = P * B;
    const void* Gt = G;
    if (B > 1) {
      void* gb = other_buf(ws, w, G);
      if ((e = permute_rows(G, gb, s.rows * P, s.m[t], (int)B, st)) != cudaSuccess) return MONARCH_ERR_CUDA;
      Gt = gb;
    }
    if ((e = wgrad_tc(Gt, lines * s.m[t], s.m[t], kept[t], lines * s.n[t], s.n[t], lines, 0, 0, 0, s.rows,
                      w.sp, part, w.nparams, poff, status, st)) != cudaSuccess)
      return MONARCH_ERR_CUDA;
    const int g2 = pack_factor((int)lines, s.m[t], s.n[t]);
    if ((e = pack_bd(W[t], ws + w.wpk, (int)lines, s.n[t], s.m[t], g2, true, st)) != cudaSuccess)
      return MONARCH_ERR_CUDA;
    void* out = (B == 1 && t == s.d - 1) ? dX : other_buf(ws, w, Gt);
    if ((e = packed_stage(Gt, s.rows, ws + w.wpk, out, (int)lines, s.m[t], s.n[t], g2, status, st)) != cudaSuccess)
      return MONARCH_ERR_CUDA;
    if (B > 1) {
      void* dst = t == s.d - 1 ? dX : other_buf(ws, w, out);
      if ((e = permute_rows(out, dst, s.rows * P, (int)B, s.n[t], st)) != cudaSuccess) return MONARCH_ERR_CUDA;
      G = dst;
    } else {
      G = out;
    }
    poff += wsize(s, t);
  }
  poff = 0;
  for (int t = 0; t < s.d; ++t) {
    const int64_t n = wsize(s, t);
    if ((e = launch_kernel(lattice_reduce_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, true,
                           (const float*)part, w.nparams, poff, w.sp.nsplit, (__nv_bfloat16*)dW[t], n)) != cudaSuccess)
      return MONARCH_ERR_CUDA;
    poff += n;
  }
  return MONARCH_OK;
}

}  // extern "C"
