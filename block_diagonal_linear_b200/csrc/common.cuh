// Shared definitions of the Monarch CUDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <initializer_list>
#include <mutex>
#include <unordered_map>

#include "../../include/monarch.h"

namespace monarch {

// Shape passed by value to kernels.  Notation as in monarch.h.
struct Shape {
  int64_t rows;
  int nb1, in1, out1;
  int nb2, in2, out2;
  int out_transpose;
  __host__ __device__ int64_t n_in() const { return (int64_t)nb1 * in1; }
  __host__ __device__ int64_t n_mid() const { return (int64_t)nb1 * out1; }
  __host__ __device__ int64_t n_out() const { return (int64_t)nb2 * out2; }
  __host__ __device__ int64_t n_R() const { return (int64_t)nb1 * out1 * in1; }
  __host__ __device__ int64_t n_L() const { return (int64_t)nb2 * out2 * in2; }
  // Column of v[j][o] in a row of Y (the output permutation).
  __host__ __device__ int64_t out_index(int j, int o) const {
    return out_transpose ? (int64_t)o * nb2 + j : (int64_t)j * out2 + o;
  }
};

inline Shape to_shape(const monarch_dims& d) {
  Shape s;
  s.rows = d.rows;
  s.nb1 = d.nb1; s.in1 = d.in1; s.out1 = d.out1;
  s.nb2 = d.nb2; s.in2 = d.in2; s.out2 = d.out2;
  s.out_transpose = d.out_transpose ? 1 : 0;
  return s;
}

// Element load / store in fp32 for both storage types.
__device__ __forceinline__ float ld_as_f32(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_as_f32(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}
__device__ __forceinline__ void st_from_f32(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_from_f32(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// Kernels launched by this library in this process (host-side count of successful launches).
inline std::atomic<unsigned long long>& launch_counter() {
  static std::atomic<unsigned long long> n{0};
  return n;
}

// Launch `kernel` on `st`; with pdl = true it may begin launching while the previous kernel of
// the stream is still running (programmatic stream serialization).  Every kernel launched this
// way calls ptx::griddep_wait() before it touches global memory that earlier kernels write.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t st, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, ((KArgs)args)...);
  if (e == cudaSuccess) launch_counter().fetch_add(1, std::memory_order_relaxed);
  return e;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (device, kernel, size): the call
// costs microseconds of host time, and the multi-kernel paths launch several kernels per call.
inline cudaError_t ensure_smem_attr(const void* kernel, size_t smem) {
  static std::mutex mu;
  static std::unordered_map<const void*, int> done[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = done[dev].find(kernel);
    if (it != done[dev].end() && it->second >= (int)smem) return cudaSuccess;
  }
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> lock(mu);
    int& v = done[dev][kernel];
    if ((int)smem > v) v = (int)smem;
  }
  return e;
}

// Device status word values (written by kernels, read by the host).
constexpr int kStatusTimeout = 1;

// ---- launchers implemented in the .cu files (all return cudaError_t) ----
cudaError_t generic_fwd(const void* X, const void* R, const void* L, void* Y, const Shape& s,
                        int dtype, cudaStream_t st);
size_t generic_bwd_workspace(const Shape& s);
cudaError_t generic_bwd(const void* dY, const void* X, const void* R, const void* L, void* dX,
                        void* dR, void* dL, void* ws, const Shape& s, int dtype, cudaStream_t st);
cudaError_t generic_materialise(const void* R, const void* L, float* M, const Shape& s, int dtype,
                                cudaStream_t st);
bool generic_fwd_supported(const Shape& s);
bool generic_bwd_supported(const Shape& s);

// tcgen05 fused forward for bf16 (returns cudaErrorNotSupported if the shape has no kernel).
bool tc_fwd_supported(const Shape& s);
cudaError_t tc_fwd(const void* X, const void* R, const void* L, void* Y, const Shape& s,
                   int* status, cudaStream_t st);

// tcgen05 fused forward with 64-row tiles and the whole middle vector on chip (small blocks).
bool tc_rows_supported(const Shape& s);
cudaError_t tc_rows_fwd_save(const void* X, const void* R, const void* L, void* Y, void* Z, const Shape& s,
                             int* status, cudaStream_t st);
cudaError_t tc_rows_fwd(const void* X, const void* R, const void* L, void* Y, const Shape& s,
                        int* status, cudaStream_t st);

// tcgen05 fused forward for transposed outputs wider than the middle vector (768 -> 3072).
bool tc_wide_supported(const Shape& s);
cudaError_t tc_wide_fwd(const void* X, const void* R, const void* L, void* Y, const Shape& s,
                        int* status, cudaStream_t st);
// The same forward also writing the middle vector Z (rows x n_mid, the L stage's input order).
cudaError_t tc_wide_fwd_save(const void* X, const void* R, const void* L, void* Y, void* Z, const Shape& s,
                             int* status, cudaStream_t st);

// Large square blocks (64 x 64, nb1 = nb2): block-diagonal tcgen05 GEMMs and row permutations
// as four passes over Y (no scratch).
// Streaming block-diagonal stages with the row permutation folded into the stores (tc_stage.cu):
//   R:  Z  = P blockdiag(R) X          L:  Y  = P_out blockdiag(L) Z
//   Lt: dU = P^-1 blockdiag(L^T) dV     Rt: dX = blockdiag(R^T) dU
// w_early: W may be read before the kernel's grid-dependency wait -- it is the caller's factor, or
// it was written at least two launches earlier on the stream (that kernel has finished by then).
enum class StageKind { R, L, Lt, Rt };
bool tc_stage_supported(const Shape& s);
bool tc_stage_fwd_supported(const Shape& s);
cudaError_t tc_stage(const void* A, const void* W, void* out, StageKind k, const Shape& s, int* status,
                     cudaStream_t st, bool pdl, bool w_early);
cudaError_t tc_stage_fwd(const void* X, const void* R, const void* L, void* Y, void* Z, const Shape& s,
                         int* status, cudaStream_t st);

bool tc_split_supported(const Shape& s);
cudaError_t tc_split_fwd(const void* X, const void* R, const void* L, void* Y, const Shape& s,
                         int* status, cudaStream_t st);
// Y[r][k*64 + n] = sum_i W[k][n][i] X[r][k*64 + i] (bf16, 64 x 64 blocks; Y may equal X).
cudaError_t bdgemm64(const void* X, const void* W, void* Y, int nb, int64_t rows, int* status,
                     cudaStream_t st, bool pdl);
// dst[r][b*A + a] = src[r][a*B + b] (bf16; dst may equal src; A, B multiples of 8).
cudaError_t permute_rows(const void* src, void* dst, int64_t rows, int A, int B, cudaStream_t st, bool pdl = true);
// dst[r][b*A + a] += src[r][a*B + b] (bf16, fp32 add rounded once; dst distinct from src).
cudaError_t permute_rows_add(const void* src, void* dst, int64_t rows, int A, int B, cudaStream_t st);

// Tensor-core backward of the square small-block shapes (bf16).
bool fast_bwd_supported(const Shape& s);
size_t fast_bwd_workspace(const Shape& s);
// saved: the middle vector Z of this call's rows as the training forward left it (nullptr: recompute)
cudaError_t fast_bwd(const void* dY, const void* X, const void* R, const void* L, void* dX, void* dR,
                     void* dL, void* ws, const Shape& s, int* status, cudaStream_t st,
                     const void* saved = nullptr);

cudaError_t debug_wait_timeout(uint64_t timeout_ns, int* status, cudaStream_t st);

// Kernel-family selection and dispatch on already-checked arguments (api.cu).
int fwd_path(const Shape& s, int dtype);
int bwd_path(const Shape& s, int dtype);
size_t bwd_workspace(const Shape& s, int dtype);
int fwd_dispatch(const void* X, const void* R, const void* L, void* Y, const Shape& s, int dtype, cudaStream_t st);
int bwd_dispatch(const void* dY, const void* X, const void* R, const void* L, void* dX, void* dR, void* dL,
                 void* ws, const Shape& s, int dtype, cudaStream_t st, const void* saved = nullptr);
int* status_ptr();
bool aligned16(const void* p);

}  // namespace monarch
