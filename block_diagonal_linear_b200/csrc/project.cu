// Dense -> Monarch projection (Monarch abstract: the projection "has an analytical optimal
// solution"; scatterbrain projection question: the slicing rearrange(M, '(p k) (r s) ->
// k r p s')).  For the lattice shapes (in2 == nb1, nb2 == out1, output transpose) every entry
// of a Monarch matrix is one product M[o*nb2 + j][k*in1 + i] = L[j][o][k] * R[k][j][i], so the
// Frobenius-nearest Monarch matrix takes the best rank-1 approximation s u v^T of every slice
// A_jk[o][i] = M[o*nb2 + j][k*in1 + i] and sets L[j][:, k] = sqrt(s) u, R[k][j][:] = sqrt(s) v.
//
// One CTA per slice, fp32: the slice is staged in shared memory and the leading right
// singular vector is found by power iteration on A^T A (v <- A^T A v / |.|) from the slice's
// row of largest norm (first on ties), until the iterate moves by less than 1e-7 (max-norm)
// or after kProjIters steps; then u = A v / |A v|, s = |A v|.  Sign convention: the entry of
// v largest in magnitude (first on ties) is positive.
#include "common.cuh"

namespace monarch {

constexpr int kProjThreads = 256;
constexpr int kProjIters = 2000;
constexpr int kProjMaxFloats = 48 * 1024;  // slice elements staged in shared memory (192 KB)

bool project_supported(const Shape& s) {
  return s.in2 == s.nb1 && s.nb2 == s.out1 && s.out_transpose == 1 &&
         (int64_t)s.out2 * s.in1 + s.in1 + s.out2 + 64 <= kProjMaxFloats;
}

// Sum over the CTA (kProjThreads threads); every thread gets the result.
__device__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = lane < kProjThreads / 32 ? red[lane] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}

__device__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = lane < kProjThreads / 32 ? red[lane] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, o));
  return t;
}

template <typename T>
__global__ void __launch_bounds__(kProjThreads) project_kernel(const float* __restrict__ M, T* __restrict__ R,
                                                                T* __restrict__ L, Shape s) {
  extern __shared__ float sm[];
  const int nrow = s.out2, ncol = s.in1;
  float* A = sm;                     // nrow x ncol
  float* v = A + nrow * ncol;        // ncol
  float* w = v + ncol;               // nrow
  float* red = w + nrow;             // 32 (+ 32 for arg-max)
  int* ired = (int*)(red + 32);
  const int j = blockIdx.x / s.nb1, k = blockIdx.x % s.nb1;
  const int64_t n_in = s.n_in();
  for (int e = threadIdx.x; e < nrow * ncol; e += blockDim.x) {
    const int o = e / ncol, i = e % ncol;
    A[e] = M[((int64_t)o * s.nb2 + j) * n_in + (int64_t)k * ncol + i];
  }
  __syncthreads();
  // start: the row of largest norm (first on ties)
  for (int o = threadIdx.x; o < nrow; o += blockDim.x) {
    float a = 0.f;
    for (int i = 0; i < ncol; ++i) a = fmaf(A[o * ncol + i], A[o * ncol + i], a);
    w[o] = a;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int best = 0;
    for (int o = 1; o < nrow; ++o)
      if (w[o] > w[best]) best = o;
    ired[0] = best;
  }
  __syncthreads();
  const int r0 = ired[0];
  for (int i = threadIdx.x; i < ncol; i += blockDim.x) v[i] = A[r0 * ncol + i];
  __syncthreads();
  float nv = 0.f;
  for (int i = threadIdx.x; i < ncol; i += blockDim.x) nv = fmaf(v[i], v[i], nv);
  nv = sqrtf(block_sum(nv, red));
  if (nv > 0.f) {
    for (int i = threadIdx.x; i < ncol; i += blockDim.x) v[i] /= nv;
    __syncthreads();
    for (int it = 0; it < kProjIters; ++it) {
      for (int o = threadIdx.x; o < nrow; o += blockDim.x) {
        float a = 0.f;
        for (int i = 0; i < ncol; ++i) a = fmaf(A[o * ncol + i], v[i], a);
        w[o] = a;
      }
      __syncthreads();
      float t[4] = {0.f, 0.f, 0.f, 0.f};  // this thread's new v entries (ncol <= 4 * threads)
      float nn = 0.f;
      for (int q = 0, i = threadIdx.x; i < ncol; i += blockDim.x, ++q) {
        float a = 0.f;
        for (int o = 0; o < nrow; ++o) a = fmaf(A[o * ncol + i], w[o], a);
        t[q] = a;
        nn = fmaf(a, a, nn);
      }
      nn = sqrtf(block_sum(nn, red));
      if (nn == 0.f) break;
      float diff = 0.f;
      for (int q = 0, i = threadIdx.x; i < ncol; i += blockDim.x, ++q) {
        const float x = t[q] / nn;
        diff = fmaxf(diff, fabsf(x - v[i]));
        v[i] = x;
      }
      diff = block_max(diff, red);
      if (diff < 1e-7f) break;
    }
  }
  __syncthreads();
  // u s = A v
  for (int o = threadIdx.x; o < nrow; o += blockDim.x) {
    float a = 0.f;
    for (int i = 0; i < ncol; ++i) a = fmaf(A[o * ncol + i], v[i], a);
    w[o] = a;
  }
  __syncthreads();
  float ss = 0.f;
  for (int o = threadIdx.x; o < nrow; o += blockDim.x) ss = fmaf(w[o], w[o], ss);
  const float sig = sqrtf(block_sum(ss, red));
  if (threadIdx.x == 0) {
    int best = 0;
    for (int i = 1; i < ncol; ++i)
      if (fabsf(v[i]) > fabsf(v[best])) best = i;
    ired[1] = best;
  }
  __syncthreads();
  const float sign = (nv > 0.f && v[ired[1]] < 0.f) ? -1.f : 1.f;
  const float rs = sqrtf(sig);
  const float inv = sig > 0.f ? 1.f / sig : 0.f;
  for (int o = threadIdx.x; o < nrow; o += blockDim.x)  // L[j][o][k]
    st_from_f32(L + ((int64_t)j * s.out2 + o) * s.in2 + k, sig > 0.f ? sign * rs * w[o] * inv : 0.f);
  for (int i = threadIdx.x; i < ncol; i += blockDim.x)  // R[k][j][i]
    st_from_f32(R + ((int64_t)k * s.out1 + j) * s.in1 + i, sig > 0.f ? sign * rs * v[i] : 0.f);
}

cudaError_t project(const float* M, void* R, void* L, const Shape& s, int dtype, cudaStream_t st) {
  if (s.in1 > 4 * kProjThreads) return cudaErrorNotSupported;
  const size_t smem = sizeof(float) * ((size_t)s.out2 * s.in1 + s.in1 + s.out2 + 64);
  const unsigned grid = (unsigned)((int64_t)s.nb1 * s.nb2);
  if (dtype == MONARCH_BF16) {
    cudaError_t e = ensure_smem_attr((const void*)project_kernel<__nv_bfloat16>, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(project_kernel<__nv_bfloat16>, dim3(grid), dim3(kProjThreads), smem, st, false, M,
                         (__nv_bfloat16*)R, (__nv_bfloat16*)L, s);
  }
  cudaError_t e = ensure_smem_attr((const void*)project_kernel<float>, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(project_kernel<float>, dim3(grid), dim3(kProjThreads), smem, st, false, M, (float*)R,
                       (float*)L, s);
}

}  // namespace monarch

using namespace monarch;

extern "C" int monarch_project(const void* M, const monarch_dims* d, void* R, void* L, void* stream) {
  int rc = monarch_validate(d);
  if (rc != MONARCH_OK) return rc;
  if (M == nullptr || R == nullptr || L == nullptr) return MONARCH_ERR_NULL;
  if (!aligned16(M) || !aligned16(R) || !aligned16(L)) return MONARCH_ERR_ALIGN;
  const Shape s = to_shape(*d);
  if (!project_supported(s) || s.in1 > 4 * kProjThreads) return MONARCH_ERR_UNSUPPORTED;
  const int64_t es = d->dtype == MONARCH_BF16 ? 2 : 4;
  const uintptr_t mb = (uintptr_t)M, me = mb + (uint64_t)s.n_out() * s.n_in() * 4;
  const uintptr_t rb = (uintptr_t)R, re = rb + (uint64_t)s.n_R() * es;
  const uintptr_t lb = (uintptr_t)L, le = lb + (uint64_t)s.n_L() * es;
  if ((rb < me && mb < re) || (lb < me && mb < le) || (rb < le && lb < re)) return MONARCH_ERR_ALIAS;
  return project(static_cast<const float*>(M), R, L, s, d->dtype, (cudaStream_t)stream) == cudaSuccess
             ? MONARCH_OK
             : MONARCH_ERR_CUDA;
}
