// Backward of the square small-block shapes (n = 16^2, 32^2; bf16) on the tensor cores.
//
//   1. Rt[k][i][p] = R[k][p][i], Lt[j][q][o] = L[j][o][q]      (tiny transpose kernel)
//   2. dV[r][j*out2 + o] = dY[r][o*nb2 + j]                     (inverse output permutation,
//                                                               block-contiguous dV)
//   3. Z = P R x                                                (row-tile kernel, R stage only)
//   4. dU = P^-1 (L^T dV), dX = R^T dU                          (row-tile kernel on the dual
//                                                               map, dU stored on the side)
// For 64 x 64 blocks (n = 4096) steps 3 and 4 are block-diagonal passes: Z and dU come from
// streaming stages with the permutation folded in (tc_stage.cu), dX from the plain GEMM pass.
//   5. dL[j] = sum_rows dV_j^T Z_j, dR[k] = sum_rows dU_k^T X_k (split-row weight gradient on
//                                                               the tcgen05 GEMM, rows as K:
//                                                               fp32 partials + fixed-order sum)
// The weight-gradient GEMM takes 128 columns of each operand per unit (4 blocks of 32, or 2
// of 64) and keeps the diagonal blocks of the 128 x 128 product.
#include "common.cuh"
#include "tc_common.cuh"
#include "tc_gemm.cuh"

namespace monarch {

cudaError_t tc_rows_middle(const void* X, const void* R, void* Z, const Shape& s, int* status,
                           cudaStream_t st);
cudaError_t tc_rows_dual(const void* dV, const void* Lt, const void* Rt, void* dX, void* dU,
                         const Shape& s, int* status, cudaStream_t st);

// ------------------------------------------------------------------ small kernels
// dV[r][j*out2 + o] = dY[r][o*nb2 + j]: per row an (out2 x nb2) -> (nb2 x out2) element
// transpose.  Each warp takes two rows at a time: all of both rows' 16-byte loads are issued
// before any is used (rows of up to 1024 elements: four chunks a lane each), the rows are
// staged in shared memory with an odd word pitch (nb2 + 2 elements, so the column reads of the
// transpose hit 32 different banks), and written back with 16-byte coalesced stores.
constexpr int kGatherWarps = 8;
constexpr int kGatherChunks = 4;  // 16-byte chunks a lane loads per row (n_out <= 1024)
__global__ void __launch_bounds__(kGatherWarps * 32)
    gather_dv_kernel(const __nv_bfloat16* __restrict__ dY, __nv_bfloat16* __restrict__ dV, Shape s) {
  extern __shared__ __align__(16) uint32_t shw[];
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int n = (int)s.n_out(), nb2 = s.nb2, out2 = s.out2;
  const int pitch = nb2 + 2;          // elements per staged grid row (o)
  const int wpitch = pitch / 2;       // 32-bit words per staged grid row
  const int nch = n / 8;              // 16-byte chunks per row (<= 32 * kGatherChunks)
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  uint32_t* buf = shw + warp * (2 * out2 * wpitch);
  const int64_t stride = (int64_t)gridDim.x * kGatherWarps;
  for (int64_t r0 = (int64_t)blockIdx.x * kGatherWarps + warp; r0 < s.rows; r0 += 2 * stride) {
    const int64_t rr[2] = {r0, r0 + stride};
    uint4 v[2][kGatherChunks];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int i = 0; i < kGatherChunks; ++i) {
        const int c = lane + 32 * i;
        if (rr[h] < s.rows && c < nch) v[h][i] = *(const uint4*)(dY + rr[h] * n + c * 8);
      }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int i = 0; i < kGatherChunks; ++i) {
        const int c = lane + 32 * i;  // chunk c: o = (8c) / nb2, j0 = (8c) % nb2
        if (rr[h] < s.rows && c < nch) {
          uint32_t* d = buf + h * (out2 * wpitch) + ((c * 8) / nb2) * wpitch + ((c * 8) % nb2) / 2;
          d[0] = v[h][i].x; d[1] = v[h][i].y; d[2] = v[h][i].z; d[3] = v[h][i].w;
        }
      }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (rr[h] >= s.rows) continue;
      const uint16_t* hb = (const uint16_t*)(buf + h * (out2 * wpitch));
      __nv_bfloat16* dst = dV + rr[h] * n;
      for (int c = lane; c < nch; c += 32) {  // output chunk: j = (8c) / out2, o0 = (8c) % out2
        const int j = (c * 8) / out2, o0 = (c * 8) % out2;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          w[e] = (uint32_t)hb[(o0 + 2 * e) * pitch + j] | ((uint32_t)hb[(o0 + 2 * e + 1) * pitch + j] << 16);
        *(uint4*)(dst + c * 8) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    __syncwarp();
  }
}

// ------------------------------------------------------------------ weight gradient
__global__ void reduce_partials_kernel(const float* __restrict__ partial, __nv_bfloat16* __restrict__ dR,
                                       __nv_bfloat16* __restrict__ dL, int64_t nR, int64_t nP,
                                       int nsplit) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nP) return;
  float acc = 0.f;
  for (int sp = 0; sp < nsplit; ++sp) acc += partial[(int64_t)sp * nP + e];
  if (e < nR)
    dR[e] = __float2bfloat16_rn(acc);
  else
    dL[e - nR] = __float2bfloat16_rn(acc);
}

// ------------------------------------------------------------------ host
static bool is_fast_square(const Shape& s) {
  const bool sq = s.nb1 == s.in1 && s.in1 == s.out1 && s.out1 == s.nb2 && s.nb2 == s.in2 &&
                  s.in2 == s.out2;
  return sq && (s.nb1 == 16 || s.nb1 == 32) && s.out_transpose == 1;
}

// 64 x 64 blocks with nb1 = nb2 (e.g. n = 4096): the middle vector does not fit on chip, so the
// row stages run as block-diagonal GEMM and row-permutation passes (tc_split.cu).
static bool is_split_square(const Shape& s) { return tc_split_supported(s); }

bool fast_bwd_supported(const Shape& s) { return is_fast_square(s) || is_split_square(s); }

// Weight-gradient units per row split: 128-column groups of dR and of dL.
static WgradSplit wg_split(const Shape& s) {
  return wgrad_split_wave(s.rows, s.n_mid() / 128 + s.n_out() / 128);
}

static size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

struct FastWs {
  size_t rt, lt, dv, z, du, part, total;
};

static FastWs fast_layout(const Shape& s) {
  FastWs w;
  const size_t nR = (size_t)s.n_R(), nL = (size_t)s.n_L();
  w.rt = 0;
  w.lt = w.rt + al256(nR * 2);
  w.dv = w.lt + al256(nL * 2);
  w.z = w.dv + al256((size_t)s.rows * (size_t)s.n_out() * 2);
  w.du = w.z + al256((size_t)s.rows * (size_t)s.n_mid() * 2);
  w.part = w.du + al256((size_t)s.rows * (size_t)s.n_mid() * 2);
  w.total = w.part + al256((size_t)wg_split(s).nsplit * (nR + nL) * 4);
  return w;
}

size_t fast_bwd_workspace(const Shape& s) { return fast_layout(s).total; }

cudaError_t fast_bwd(const void* dY, const void* X, const void* R, const void* L, void* dX, void* dR,
                     void* dL, void* ws, const Shape& s, int* status, cudaStream_t st, const void* saved) {
  const FastWs w = fast_layout(s);
  char* base = (char*)ws;
  __nv_bfloat16* Rt = (__nv_bfloat16*)(base + w.rt);
  __nv_bfloat16* Lt = (__nv_bfloat16*)(base + w.lt);
  __nv_bfloat16* dV = (__nv_bfloat16*)(base + w.dv);
  __nv_bfloat16* Z = (__nv_bfloat16*)(base + w.z);
  __nv_bfloat16* dU = (__nv_bfloat16*)(base + w.du);
  float* part = (float*)(base + w.part);
  const int64_t nR = s.n_R(), nP = s.n_R() + s.n_L();
  cudaError_t e;
  // All launches use programmatic dependent launch: each kernel waits for the previous grid of
  // the stream (griddep_wait) before touching its data, so the next launch and its prologue
  // overlap the tail of the current one.  The factor transposes (Rt, Lt) are needed only from the
  // dual stage on: they are launched right after the Z pass and run concurrently with it.
  const WgradSplit sp = wg_split(s);
  const bool split = is_split_square(s);
  if (split && !s.out_transpose) dV = (__nv_bfloat16*)dY;  // dV[j][o] = dy[j*out2 + o]: no copy
  if (saved != nullptr) Z = (__nv_bfloat16*)saved;  // the training forward's Z: no recompute
  if (s.rows > 0 && split) {
    // dV = P_out^-1 dY;  Z = P (blockdiag(R) X);  dZ = blockdiag(L^T) dV;  dU = P^-1 dZ;
    // dX = blockdiag(R^T) dU.  Z and dZ/dU are permuted in place.
    bool prev = false;  // a kernel of this call precedes (the transposes may then overlap it)
    if (s.out_transpose) {
      if ((e = permute_rows(dY, dV, s.rows, s.out2, s.nb2, st)) != cudaSuccess) return e;
      prev = true;
    }
    if (tc_stage_supported(s)) {
      // the permutations folded into the stages that produce Z and dU (tc_stage.cu)
      if (saved == nullptr) {
        if ((e = tc_stage(X, R, Z, StageKind::R, s, status, st, true, true)) != cudaSuccess) return e;
        prev = true;
      }
      if ((e = factor_transposes(R, Rt, L, Lt, s, 0, st, prev)) != cudaSuccess) return e;
      // Lt comes from the launch just before: read it after the wait
      if ((e = tc_stage(dV, Lt, dU, StageKind::Lt, s, status, st, true, false)) != cudaSuccess) return e;
    } else {
      if (saved == nullptr) {
        if ((e = bdgemm64(X, R, Z, s.nb1, s.rows, status, st, true)) != cudaSuccess) return e;
        if ((e = permute_rows(Z, Z, s.rows, s.nb1, s.out1, st)) != cudaSuccess) return e;
        prev = true;
      }
      if ((e = factor_transposes(R, Rt, L, Lt, s, 0, st, prev)) != cudaSuccess) return e;
      if ((e = bdgemm64(dV, Lt, dU, s.nb2, s.rows, status, st, true)) != cudaSuccess) return e;
      if ((e = permute_rows(dU, dU, s.rows, s.out1, s.nb1, st)) != cudaSuccess) return e;
    }
    if ((e = bdgemm64(dU, Rt, dX, s.nb1, s.rows, status, st, true)) != cudaSuccess) return e;
  } else if (s.rows > 0) {
    const size_t gsm = (size_t)kGatherWarps * 2 * (size_t)s.out2 * (size_t)(s.nb2 + 2) * 2;
    if (s.n_out() > 32 * kGatherChunks * 8) return cudaErrorInvalidValue;
    if ((e = launch_kernel(gather_dv_kernel, dim3(4 * 148), dim3(kGatherWarps * 32), gsm, st, true,
                           (const __nv_bfloat16*)dY, dV, s)) != cudaSuccess)
      return e;
    if (saved == nullptr && (e = tc_rows_middle(X, R, Z, s, status, st)) != cudaSuccess) return e;
    if ((e = factor_transposes(R, Rt, L, Lt, s, 0, st, true)) != cudaSuccess) return e;
    if ((e = tc_rows_dual(dV, Lt, Rt, dX, dU, s, status, st)) != cudaSuccess) return e;
  }
  if (s.rows > 0) {
    // dR[k] = sum_rows dU_k^T X_k;  dL[j] = sum_rows dV_j^T Z_j  (all operands block-contiguous)
    const WgradArgs gR = {dU, s.n_mid(), s.out1, X, s.n_in(), s.in1, s.nb1, 0, 0, 0, sp, nP, 0};
    const WgradArgs gL = {dV, s.n_out(), s.out2, Z, s.n_mid(), s.in2, s.nb2, 0, 0, 0, sp, nP, nR};
    if ((e = wgrad_tc2(gR, gL, s.rows, part, status, st)) != cudaSuccess) return e;
  } else if ((e = cudaMemsetAsync(part, 0, sizeof(float) * (size_t)sp.nsplit * (size_t)nP, st)) != cudaSuccess) {
    return e;
  }
  return launch_kernel(reduce_partials_kernel, dim3((unsigned)((nP + 255) / 256)), dim3(256), 0, st, true,
                       (const float*)part, (__nv_bfloat16*)dR, (__nv_bfloat16*)dL, nR, nP, sp.nsplit);
}

}  // namespace monarch
