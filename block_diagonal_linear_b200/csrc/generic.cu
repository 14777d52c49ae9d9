// Generic Monarch kernels: fp32 FMA on the CUDA cores, any shape, fp32 or bf16
// storage.  These serve fp32 workloads (where tensor-core TF32 would not meet
// a 1e-5 normwise tolerance), shapes that have no tcgen05 instantiation, and
// the backward until a fused tensor-core backward covers the shape.
//
// Forward (one CTA = up to kMaxRows rows, whole row in shared memory; few rows spread over
// more CTAs so that small problems still use many SMs):
//   xs <- X rows;  zs[r][p*nb1+k] = sum_i R[k][p][i] xs[r][k*in1+i]
//   (the permutation P is the store index); y[out_index(j,o)] = sum_q L[j][o][q] zs[r][j*in2+q].
// Backward: a row kernel recomputes Z, forms dZ = L^T dV and dX = R^T dU, and
// spills Z and dZ (fp32) to the workspace; a weight-gradient kernel reduces
// dR and dL over row splits; a final kernel sums the splits in fixed order.  The two
// later kernels are launched as programmatic dependents of the one before, so their
// launches overlap it; each waits for its predecessor before reading.
#include "common.cuh"
#include "tc_common.cuh"

namespace monarch {

constexpr int kGenThreads = 256;
constexpr int kMaxRows = 16;
constexpr size_t kGenSmemBudget = 200 * 1024;

static int gen_rows_per_cta(int64_t floats_per_row) {
  int64_t r = (int64_t)(kGenSmemBudget / (sizeof(float) * (size_t)floats_per_row));
  if (r > kMaxRows) r = kMaxRows;
  return (int)r;
}

// Rows per CTA for a launch over `rows` rows: the shared-memory limit, but no more than one
// wave of CTAs needs (every row of a CTA is computed the same way, so this changes no result).
static int gen_rows_for(int64_t rows, int64_t floats_per_row) {
  const int cap = gen_rows_per_cta(floats_per_row);
  const int64_t wave = (rows + num_sms() - 1) / num_sms();
  return (int)(wave < 1 ? 1 : (wave < cap ? wave : cap));
}

bool generic_fwd_supported(const Shape& s) { return gen_rows_per_cta(s.n_in() + s.n_mid()) >= 1; }
bool generic_bwd_supported(const Shape& s) {
  return gen_rows_per_cta(s.n_in() + s.n_out() + 2 * s.n_mid()) >= 1;
}

// acc[r] = fma(w[t*ws], act[r*rs + t*ts], acc[r]) for t = 0, 1, ..., n-1 in that order (r < nr).
// The weights are loaded four at a time before their FMAs, so their load latencies overlap
// instead of following one another.
template <typename T>
__device__ __forceinline__ void fma_rows(float (&acc)[kMaxRows], const T* __restrict__ w, int64_t ws,
                                         const float* act, int64_t rs, int64_t ts, int n, int nr) {
  for (int t0 = 0; t0 < n; t0 += 4) {
    float wv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) wv[u] = t0 + u < n ? ld_as_f32(w + (int64_t)(t0 + u) * ws) : 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (t0 + u < n) {
        const float* a = act + (int64_t)(t0 + u) * ts;
#pragma unroll
        for (int r = 0; r < kMaxRows; ++r)
          if (r < nr) acc[r] = fmaf(wv[u], a[r * rs], acc[r]);
      }
    }
  }
}

// zs[r][p*nb1 + k] = sum_i R[k][p][i] * xs[r][k*in1 + i] for r < nr  (steps a1..a3)
template <typename T>
__device__ void gen_stage_R(const T* __restrict__ R, const float* xs, float* zs, const Shape& s,
                            int nr) {
  const int64_t n_in = s.n_in(), n_mid = s.n_mid();
  for (int64_t idx = threadIdx.x; idx < n_mid; idx += blockDim.x) {
    const int k = (int)(idx / s.out1), p = (int)(idx % s.out1);
    float acc[kMaxRows];
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r) acc[r] = 0.f;
    fma_rows(acc, R + idx * s.in1, 1, xs + (int64_t)k * s.in1, n_in, 1, s.in1, nr);
    const int64_t t = (int64_t)p * s.nb1 + k;
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r)
      if (r < nr) zs[r * n_mid + t] = acc[r];
  }
}

template <typename T>
__global__ void __launch_bounds__(kGenThreads)
    gen_fwd_kernel(const T* __restrict__ X, const T* __restrict__ R, const T* __restrict__ L,
                   T* __restrict__ Y, Shape s, int rpc) {
  extern __shared__ float sm[];
  const int64_t n_in = s.n_in(), n_mid = s.n_mid(), n_out = s.n_out();
  float* xs = sm;
  float* zs = sm + (int64_t)rpc * n_in;
  const int64_t r0 = (int64_t)blockIdx.x * rpc;
  const int nr = (int)min((int64_t)rpc, s.rows - r0);
  for (int64_t e = threadIdx.x; e < nr * n_in; e += blockDim.x) xs[e] = ld_as_f32(X + r0 * n_in + e);
  __syncthreads();
  gen_stage_R(R, xs, zs, s, nr);
  __syncthreads();
  // steps a4, a5
  for (int64_t idx = threadIdx.x; idx < n_out; idx += blockDim.x) {
    const int j = (int)(idx / s.out2), o = (int)(idx % s.out2);
    float acc[kMaxRows];
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r) acc[r] = 0.f;
    fma_rows(acc, L + idx * s.in2, 1, zs + (int64_t)j * s.in2, n_mid, 1, s.in2, nr);
    const int64_t col = s.out_index(j, o);
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r)
      if (r < nr) st_from_f32(Y + (r0 + r) * n_out + col, acc[r]);
  }
}

template <typename T>
__global__ void __launch_bounds__(kGenThreads)
    gen_bwd_rows_kernel(const T* __restrict__ dY, const T* __restrict__ X, const T* __restrict__ R,
                        const T* __restrict__ L, T* __restrict__ dX, float* __restrict__ wsZ,
                        float* __restrict__ wsdZ, Shape s, int rpc) {
  ptx::griddep_launch_dependents();  // the weight-gradient grid waits for this one to complete
  extern __shared__ float sm[];
  const int64_t n_in = s.n_in(), n_mid = s.n_mid(), n_out = s.n_out();
  float* xs = sm;
  float* dvs = xs + (int64_t)rpc * n_in;
  float* zs = dvs + (int64_t)rpc * n_out;
  float* dzs = zs + (int64_t)rpc * n_mid;
  const int64_t r0 = (int64_t)blockIdx.x * rpc;
  const int nr = (int)min((int64_t)rpc, s.rows - r0);
  for (int64_t e = threadIdx.x; e < nr * n_in; e += blockDim.x) xs[e] = ld_as_f32(X + r0 * n_in + e);
  // a6: dV[j][o] = dy[out_index(j,o)], kept in (j, o) order
  for (int64_t e = threadIdx.x; e < nr * n_out; e += blockDim.x) {
    const int64_t r = e / n_out, c = e % n_out;
    const int j = (int)(c / s.out2), o = (int)(c % s.out2);
    dvs[e] = ld_as_f32(dY + (r0 + r) * n_out + s.out_index(j, o));
  }
  __syncthreads();
  gen_stage_R(R, xs, zs, s, nr);  // recompute Z
  // a8: dZ[j][q] = sum_o L[j][o][q] dV[j][o]
  for (int64_t idx = threadIdx.x; idx < n_mid; idx += blockDim.x) {
    const int j = (int)(idx / s.in2), q = (int)(idx % s.in2);
    float acc[kMaxRows];
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r) acc[r] = 0.f;
    fma_rows(acc, L + (int64_t)j * s.out2 * s.in2 + q, s.in2, dvs + (int64_t)j * s.out2, n_out, 1, s.out2, nr);
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r)
      if (r < nr) dzs[r * n_mid + idx] = acc[r];
  }
  __syncthreads();
  // a8 (inverse permutation) + a10: dX[k*in1+i] = sum_p R[k][p][i] dZflat[p*nb1+k]
  for (int64_t idx = threadIdx.x; idx < n_in; idx += blockDim.x) {
    const int k = (int)(idx / s.in1), i = (int)(idx % s.in1);
    float acc[kMaxRows];
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r) acc[r] = 0.f;
    // dZflat index of p is p*nb1 + k
    fma_rows(acc, R + (int64_t)k * s.out1 * s.in1 + i, s.in1, dzs + k, n_mid, s.nb1, s.out1, nr);
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r)
      if (r < nr) st_from_f32(dX + (r0 + r) * n_in + idx, acc[r]);
  }
  // spill Z and dZ for the weight gradients
  for (int64_t e = threadIdx.x; e < nr * n_mid; e += blockDim.x) {
    wsZ[r0 * n_mid + e] = zs[e];
    wsdZ[r0 * n_mid + e] = dzs[e];
  }
}

// Partial weight gradients over one split of the rows (a7, a9).
template <typename T>
__global__ void __launch_bounds__(kGenThreads)
    gen_bwd_wgrad_kernel(const T* __restrict__ dY, const T* __restrict__ X,
                         const float* __restrict__ wsZ, const float* __restrict__ wsdZ,
                         float* __restrict__ partial, Shape s, int nsplit) {
  ptx::griddep_wait();  // Z and dZ from the row kernel
  ptx::griddep_launch_dependents();
  const int64_t nR = s.n_R(), nP = s.n_R() + s.n_L();
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nP) return;
  const int sp = blockIdx.y;
  const int64_t ra = s.rows * sp / nsplit, rb = s.rows * (sp + 1) / nsplit;
  const int64_t n_in = s.n_in(), n_mid = s.n_mid(), n_out = s.n_out();
  float acc = 0.f;
  if (e < nR) {
    const int k = (int)(e / ((int64_t)s.out1 * s.in1));
    const int64_t rem = e % ((int64_t)s.out1 * s.in1);
    const int p = (int)(rem / s.in1), i = (int)(rem % s.in1);
    const int64_t t = (int64_t)p * s.nb1 + k, c = (int64_t)k * s.in1 + i;
    int64_t r = ra;
    for (; r + 4 <= rb; r += 4) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = wsdZ[(r + u) * n_mid + t];
        b[u] = ld_as_f32(X + (r + u) * n_in + c);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) acc = fmaf(a[u], b[u], acc);
    }
    for (; r < rb; ++r) acc = fmaf(wsdZ[r * n_mid + t], ld_as_f32(X + r * n_in + c), acc);
  } else {
    const int64_t e2 = e - nR;
    const int j = (int)(e2 / ((int64_t)s.out2 * s.in2));
    const int64_t rem = e2 % ((int64_t)s.out2 * s.in2);
    const int o = (int)(rem / s.in2), q = (int)(rem % s.in2);
    const int64_t col = s.out_index(j, o), t = (int64_t)j * s.in2 + q;
    int64_t r = ra;
    for (; r + 4 <= rb; r += 4) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = ld_as_f32(dY + (r + u) * n_out + col);
        b[u] = wsZ[(r + u) * n_mid + t];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) acc = fmaf(a[u], b[u], acc);
    }
    for (; r < rb; ++r) acc = fmaf(ld_as_f32(dY + r * n_out + col), wsZ[r * n_mid + t], acc);
  }
  partial[(int64_t)sp * nP + e] = acc;
}

template <typename T>
__global__ void __launch_bounds__(kGenThreads)
    gen_bwd_reduce_kernel(const float* __restrict__ partial, T* __restrict__ dR,
                          T* __restrict__ dL, Shape s, int nsplit) {
  ptx::griddep_wait();  // the partials
  const int64_t nR = s.n_R(), nP = s.n_R() + s.n_L();
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nP) return;
  float acc = 0.f;
  int sp = 0;
  for (; sp + 8 <= nsplit; sp += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = partial[(int64_t)(sp + u) * nP + e];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc += v[u];
  }
  for (; sp < nsplit; ++sp) acc += partial[(int64_t)sp * nP + e];
  if (e < nR)
    st_from_f32(dR + e, acc);
  else
    st_from_f32(dL + (e - nR), acc);
}

template <typename T>
__global__ void __launch_bounds__(kGenThreads)
    gen_materialise_kernel(const T* __restrict__ R, const T* __restrict__ L, float* __restrict__ M,
                           Shape s) {
  const int64_t n_in = s.n_in(), n_out = s.n_out();
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_in * n_out) return;
  const int64_t a = e / n_in, b = e % n_in;
  int j, o;
  if (s.out_transpose) {
    o = (int)(a / s.nb2); j = (int)(a % s.nb2);
  } else {
    j = (int)(a / s.out2); o = (int)(a % s.out2);
  }
  const int k = (int)(b / s.in1), i = (int)(b % s.in1);
  // p with (p*nb1 + k) in [j*in2, (j+1)*in2)
  const int64_t lo_num = (int64_t)j * s.in2 - k, hi_num = (int64_t)(j + 1) * s.in2 - k;
  int64_t p_lo = lo_num <= 0 ? 0 : (lo_num + s.nb1 - 1) / s.nb1;
  int64_t p_hi = hi_num <= 0 ? 0 : (hi_num + s.nb1 - 1) / s.nb1;
  if (p_hi > s.out1) p_hi = s.out1;
  float acc = 0.f;
  for (int64_t p = p_lo; p < p_hi; ++p) {
    const int64_t q = p * s.nb1 + k - (int64_t)j * s.in2;
    acc = fmaf(ld_as_f32(L + ((int64_t)j * s.out2 + o) * s.in2 + q),
               ld_as_f32(R + ((int64_t)k * s.out1 + p) * s.in1 + i), acc);
  }
  M[e] = acc;
}

// ------------------------------------------------------------------ launchers
template <typename T>
static cudaError_t launch_fwd(const void* X, const void* R, const void* L, void* Y, const Shape& s,
                              cudaStream_t st) {
  if (gen_rows_per_cta(s.n_in() + s.n_mid()) < 1) return cudaErrorNotSupported;
  const int rpc = gen_rows_for(s.rows, s.n_in() + s.n_mid());
  const size_t smem = sizeof(float) * (size_t)rpc * (size_t)(s.n_in() + s.n_mid());
  cudaError_t e = ensure_smem_attr((const void*)gen_fwd_kernel<T>, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = (s.rows + rpc - 1) / rpc;
  return launch_kernel(gen_fwd_kernel<T>, dim3((unsigned)grid), dim3(kGenThreads), smem, st, false,
                       (const T*)X, (const T*)R, (const T*)L, (T*)Y, s, rpc);
}

cudaError_t generic_fwd(const void* X, const void* R, const void* L, void* Y, const Shape& s,
                        int dtype, cudaStream_t st) {
  if (s.rows == 0) return cudaSuccess;
  return dtype == MONARCH_BF16 ? launch_fwd<__nv_bfloat16>(X, R, L, Y, s, st)
                               : launch_fwd<float>(X, R, L, Y, s, st);
}

static int gen_nsplit(const Shape& s) {
  const int64_t nP = s.n_R() + s.n_L();
  int64_t n = (int64_t(1) << 21) / (nP > 0 ? nP : 1);
  if (n > 64) n = 64;
  if (n > s.rows / 8) n = s.rows / 8;  // at least eight rows per split
  if (n < 1) n = 1;
  return (int)n;
}

static size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

size_t generic_bwd_workspace(const Shape& s) {
  const size_t zbytes = align256(sizeof(float) * (size_t)s.rows * (size_t)s.n_mid());
  const size_t pbytes =
      align256(sizeof(float) * (size_t)gen_nsplit(s) * (size_t)(s.n_R() + s.n_L()));
  return 2 * zbytes + pbytes;
}

template <typename T>
static cudaError_t launch_bwd(const void* dY, const void* X, const void* R, const void* L, void* dX,
                              void* dR, void* dL, void* ws, const Shape& s, cudaStream_t st) {
  if (gen_rows_per_cta(s.n_in() + s.n_out() + 2 * s.n_mid()) < 1) return cudaErrorNotSupported;
  const int rpc = gen_rows_for(s.rows, s.n_in() + s.n_out() + 2 * s.n_mid());
  const size_t zbytes = align256(sizeof(float) * (size_t)s.rows * (size_t)s.n_mid());
  float* wsZ = (float*)ws;
  float* wsdZ = (float*)((char*)ws + zbytes);
  float* partial = (float*)((char*)ws + 2 * zbytes);
  const int nsplit = gen_nsplit(s);
  const int64_t nP = s.n_R() + s.n_L();
  cudaError_t e;
  if (s.rows > 0) {
    const size_t smem =
        sizeof(float) * (size_t)rpc * (size_t)(s.n_in() + s.n_out() + 2 * s.n_mid());
    e = ensure_smem_attr((const void*)gen_bwd_rows_kernel<T>, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = (s.rows + rpc - 1) / rpc;
    if ((e = launch_kernel(gen_bwd_rows_kernel<T>, dim3((unsigned)grid), dim3(kGenThreads), smem, st, false,
                           (const T*)dY, (const T*)X, (const T*)R, (const T*)L, (T*)dX, wsZ, wsdZ, s,
                           rpc)) != cudaSuccess)
      return e;
  }
  dim3 g((unsigned)((nP + kGenThreads - 1) / kGenThreads), (unsigned)nsplit);
  if ((e = launch_kernel(gen_bwd_wgrad_kernel<T>, g, dim3(kGenThreads), 0, st, true, (const T*)dY,
                         (const T*)X, (const float*)wsZ, (const float*)wsdZ, partial, s, nsplit)) != cudaSuccess)
    return e;
  return launch_kernel(gen_bwd_reduce_kernel<T>, dim3((unsigned)((nP + kGenThreads - 1) / kGenThreads)),
                       dim3(kGenThreads), 0, st, true, (const float*)partial, (T*)dR, (T*)dL, s, nsplit);
}

cudaError_t generic_bwd(const void* dY, const void* X, const void* R, const void* L, void* dX,
                        void* dR, void* dL, void* ws, const Shape& s, int dtype, cudaStream_t st) {
  return dtype == MONARCH_BF16
             ? launch_bwd<__nv_bfloat16>(dY, X, R, L, dX, dR, dL, ws, s, st)
             : launch_bwd<float>(dY, X, R, L, dX, dR, dL, ws, s, st);
}

cudaError_t generic_materialise(const void* R, const void* L, float* M, const Shape& s, int dtype,
                                cudaStream_t st) {
  const int64_t n = s.n_in() * s.n_out();
  const unsigned grid = (unsigned)((n + kGenThreads - 1) / kGenThreads);
  if (dtype == MONARCH_BF16)
    return launch_kernel(gen_materialise_kernel<__nv_bfloat16>, dim3(grid), dim3(kGenThreads), 0, st, false,
                         (const __nv_bfloat16*)R, (const __nv_bfloat16*)L, M, s);
  return launch_kernel(gen_materialise_kernel<float>, dim3(grid), dim3(kGenThreads), 0, st, false,
                       (const float*)R, (const float*)L, M, s);
}

}  // namespace monarch
