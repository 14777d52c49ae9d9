// Backward of the square small-block shapes (n = 16^2, 32^2; bf16) on the tensor cores.
//
//   1. Rt[k][i][p] = R[k][p][i], Lt[j][q][o] = L[j][o][q]      (tiny transpose kernel)
//   2. dV[r][j*out2 + o] = dY[r][o*nb2 + j]                     (inverse output permutation,
//                                                               block-contiguous dV)
//   3. Z = P R x                                                (row-tile kernel, R stage only)
//   4. dU = P^-1 (L^T dV), dX = R^T dU                          (row-tile kernel on the dual
//                                                               map, dU stored on the side)
//   5. dL[j] = sum_rows dV_j^T Z_j, dR[k] = sum_rows dU_k^T X_k (split-row weight gradient,
//                                                               fp32 partials + fixed-order sum)
// The weight-gradient products have one 32x32 (or 16x16) output per block and K = rows,
// too small for a 64/128-row tcgen05 tile without wasting half of it, so they use
// warp-level mma.sync (m16n8k16, bf16 -> fp32) with ldmatrix.trans operand loads.
#include "common.cuh"
#include "tc_common.cuh"

namespace monarch {

cudaError_t tc_rows_middle(const void* X, const void* R, void* Z, const Shape& s, int* status,
                           cudaStream_t st);
cudaError_t tc_rows_dual(const void* dV, const void* Lt, const void* Rt, void* dX, void* dU,
                         const Shape& s, int* status, cudaStream_t st);

// ------------------------------------------------------------------ small kernels
__global__ void transpose_factors_kernel(const __nv_bfloat16* __restrict__ R,
                                         const __nv_bfloat16* __restrict__ L,
                                         __nv_bfloat16* __restrict__ Rt,
                                         __nv_bfloat16* __restrict__ Lt, Shape s) {
  ptx::griddep_wait();  // Rt, Lt may still be read by the previous backward's kernels
  ptx::griddep_launch_dependents();
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t nR = s.n_R(), nL = s.n_L();
  if (e < nR) {  // Rt[k][i][p] = R[k][p][i]
    const int64_t k = e / ((int64_t)s.in1 * s.out1), rem = e % ((int64_t)s.in1 * s.out1);
    const int i = (int)(rem / s.out1), p = (int)(rem % s.out1);
    Rt[e] = R[(k * s.out1 + p) * s.in1 + i];
  } else if (e < nR + nL) {  // Lt[j][q][o] = L[j][o][q]
    const int64_t f = e - nR;
    const int64_t j = f / ((int64_t)s.in2 * s.out2), rem = f % ((int64_t)s.in2 * s.out2);
    const int q = (int)(rem / s.out2), o = (int)(rem % s.out2);
    Lt[f] = L[(j * s.out2 + o) * s.in2 + q];
  }
}

// dV[r][j*out2 + o] = dY[r][o*nb2 + j]: per row an (out2 x nb2) -> (nb2 x out2)
// transpose.  One warp per row: the row is read with 16-byte coalesced loads, staged in
// shared memory with an odd word pitch (nb2 + 2 elements, so the column reads of the
// transpose hit 32 different banks), and written back with 16-byte coalesced stores.
constexpr int kGatherWarps = 8;
__global__ void __launch_bounds__(kGatherWarps * 32)
    gather_dv_kernel(const __nv_bfloat16* __restrict__ dY, __nv_bfloat16* __restrict__ dV, Shape s) {
  extern __shared__ __align__(16) uint32_t shw[];
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int n = (int)s.n_out(), nb2 = s.nb2, out2 = s.out2;
  const int pitch = nb2 + 2;          // elements per staged grid row (o)
  const int wpitch = pitch / 2;       // 32-bit words per staged grid row
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  uint32_t* buf = shw + warp * (out2 * wpitch);
  const uint16_t* hb = (const uint16_t*)buf;
  for (int64_t r = (int64_t)blockIdx.x * kGatherWarps + warp; r < s.rows;
       r += (int64_t)gridDim.x * kGatherWarps) {
    const __nv_bfloat16* src = dY + r * n;
    for (int c = lane; c < n / 8; c += 32) {  // chunk c: o = (8c) / nb2, j0 = (8c) % nb2
      const uint4 v = *(const uint4*)(src + c * 8);
      const int o = (c * 8) / nb2, j0 = (c * 8) % nb2;
      uint32_t* d = buf + o * wpitch + j0 / 2;
      d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
    }
    __syncwarp();
    __nv_bfloat16* dst = dV + r * n;
    for (int c = lane; c < n / 8; c += 32) {  // output chunk: j = (8c) / out2, o0 = (8c) % out2
      const int j = (c * 8) / out2, o0 = (c * 8) % out2;
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[e] = (uint32_t)hb[(o0 + 2 * e) * pitch + j] | ((uint32_t)hb[(o0 + 2 * e + 1) * pitch + j] << 16);
      *(uint4*)(dst + c * 8) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    __syncwarp();
  }
}

// ------------------------------------------------------------------ weight gradient
// C_b[m][n] = sum_r A[r][b*BS + m] * B[r][b*BS + n] for 8 consecutive blocks b per CTA
// (one per warp) over one split of the rows; written as fp32 partials.
constexpr int kWgChunk = 64;  // rows per shared-memory chunk

__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int BS, int CH = kWgChunk>  // CH: rows per shared-memory chunk
__global__ void __launch_bounds__(256, 1)
    wgrad_kernel(const __nv_bfloat16* __restrict__ Al, const __nv_bfloat16* __restrict__ Bl,
                 const __nv_bfloat16* __restrict__ Ar, const __nv_bfloat16* __restrict__ Br,
                 int ngroups_l, int64_t rows, int nsplit, float* __restrict__ partial,
                 int64_t nR, int64_t nP, int ncols) {
  constexpr int PITCH = 8 * BS * 2 + 16;  // bytes per staged row (+16: conflict-free ldmatrix)
  constexpr int TILE = CH * PITCH;
  constexpr int MT = BS / 16, NT = BS / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = blockIdx.y;
  const bool is_l = g < ngroups_l;  // job: dL (A = dV, B = Z) or dR (A = dU, B = X)
  const int b0 = (is_l ? g : g - ngroups_l) * 8;
  const __nv_bfloat16* A = is_l ? Al : Ar;
  const __nv_bfloat16* B = is_l ? Bl : Br;
  const int64_t ra = rows * blockIdx.x / nsplit, rb = rows * (blockIdx.x + 1) / nsplit;
  const int nchunks = (int)((rb - ra + CH - 1) / CH);
  const uint32_t sbase = ptx::smem_u32(smem);
  constexpr int CPR = 8 * BS * 2 / 16;  // 16-byte chunks per staged row per tensor

  auto load = [&](int c, int buf) {
    const int64_t r0 = ra + (int64_t)c * CH;
    for (int q = threadIdx.x; q < 2 * CH * CPR; q += blockDim.x) {
      const int t = q / (CH * CPR), rem = q % (CH * CPR);
      const int rr = rem / CPR, cc = rem % CPR;
      const int64_t r = r0 + rr;
      const bool valid = r < rb;
      const __nv_bfloat16* src = (t == 0 ? A : B) + (valid ? r : ra) * ncols + (int64_t)b0 * BS + cc * 8;
      cp_async_16_zfill(sbase + (uint32_t)((buf * 2 + t) * TILE + rr * PITCH + cc * 16), src, valid);
    }
    ptx::cp_async_commit();
  };

  float acc[MT][NT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  if (nchunks > 0) load(0, 0);
  for (int c = 0; c < nchunks; ++c) {
    const int buf = c & 1;
    if (c + 1 < nchunks) {
      load(c + 1, buf ^ 1);
      ptx::cp_async_wait<1>();
    } else {
      ptx::cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t ta = sbase + (uint32_t)((buf * 2 + 0) * TILE);
    const uint32_t tb = sbase + (uint32_t)((buf * 2 + 1) * TILE);
    const int qm = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int ks = 0; ks < CH / 16; ++ks) {
      uint32_t a[MT][4], b[NT][2];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        // matrices: (rows +0, cols +0), (rows +0, cols +8), (rows +8, cols +0), (rows +8, cols +8)
        const int row = ks * 16 + (qm >> 1) * 8 + ri;
        const int col = warp * BS + mt * 16 + (qm & 1) * 8;
        ldmatrix_x4_trans(ta + row * PITCH + col * 2, a[mt]);
      }
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        // matrices: (rows +0, n +0), (rows +8, n +0), (rows +0, n +8), (rows +8, n +8)
        const int row = ks * 16 + (qm & 1) * 8 + ri;
        const int col = warp * BS + np * 16 + (qm >> 1) * 8;
        uint32_t r4[4];
        ldmatrix_x4_trans(tb + row * PITCH + col * 2, r4);
        b[2 * np][0] = r4[0];
        b[2 * np][1] = r4[1];
        b[2 * np + 1][0] = r4[2];
        b[2 * np + 1][1] = r4[3];
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(acc[mt][nt], a[mt], b[nt][0], b[nt][1]);
    }
    __syncthreads();
  }
  // C_b[m][n] -> partial[split][param]; param of (b, m, n) = [nR +] b*BS*BS + m*BS + n
  const int blk = b0 + warp;
  float* out = partial + (int64_t)blockIdx.x * nP + (is_l ? nR : 0) + (int64_t)blk * BS * BS;
  const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int m0 = mt * 16 + gq, n0 = nt * 8 + 2 * tq;
      out[m0 * BS + n0] = acc[mt][nt][0];
      out[m0 * BS + n0 + 1] = acc[mt][nt][1];
      out[(m0 + 8) * BS + n0] = acc[mt][nt][2];
      out[(m0 + 8) * BS + n0 + 1] = acc[mt][nt][3];
    }
}

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

static int wg_nsplit(const Shape& s) {
  const int ngroups = (s.nb1 + s.nb2) / 8;
  int64_t n = (2 * 148 + ngroups - 1) / ngroups;
  const int64_t maxs = (s.rows + kWgChunk - 1) / kWgChunk;
  if (n > maxs) n = maxs;
  if (n < 1) n = 1;
  return (int)n;
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
  w.total = w.part + al256((size_t)wg_nsplit(s) * (nR + nL) * 4);
  return w;
}

size_t fast_bwd_workspace(const Shape& s) { return fast_layout(s).total; }

cudaError_t fast_bwd(const void* dY, const void* X, const void* R, const void* L, void* dX, void* dR,
                     void* dL, void* ws, const Shape& s, int* status, cudaStream_t st) {
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
  // All six launches use programmatic dependent launch: each kernel waits for the previous
  // grid of the stream (griddep_wait) before touching its data, so the next launch and its
  // prologue overlap the tail of the current one.
  if ((e = launch_kernel(transpose_factors_kernel, dim3((unsigned)((nP + 255) / 256)), dim3(256), 0, st,
                         true, (const __nv_bfloat16*)R, (const __nv_bfloat16*)L, Rt, Lt, s)) != cudaSuccess)
    return e;
  const int nsplit = wg_nsplit(s);
  const bool split = is_split_square(s);
  if (split && !s.out_transpose) dV = (__nv_bfloat16*)dY;  // dV[j][o] = dy[j*out2 + o]: no copy
  if (s.rows > 0 && split) {
    // dV = P_out^-1 dY;  Z = P (blockdiag(R) X);  dZ = blockdiag(L^T) dV;  dU = P^-1 dZ;
    // dX = blockdiag(R^T) dU.  Z and dZ/dU are permuted in place.
    if (s.out_transpose && (e = permute_rows(dY, dV, s.rows, s.out2, s.nb2, st)) != cudaSuccess) return e;
    if ((e = bdgemm64(X, R, Z, s.nb1, s.rows, status, st, true)) != cudaSuccess) return e;
    if ((e = permute_rows(Z, Z, s.rows, s.nb1, s.out1, st)) != cudaSuccess) return e;
    if ((e = bdgemm64(dV, Lt, dU, s.nb2, s.rows, status, st, true)) != cudaSuccess) return e;
    if ((e = permute_rows(dU, dU, s.rows, s.out1, s.nb1, st)) != cudaSuccess) return e;
    if ((e = bdgemm64(dU, Rt, dX, s.nb1, s.rows, status, st, true)) != cudaSuccess) return e;
  } else if (s.rows > 0) {
    const size_t gsm = (size_t)kGatherWarps * (size_t)s.out2 * (size_t)(s.nb2 + 2) * 2;
    if ((e = launch_kernel(gather_dv_kernel, dim3(2 * 148), dim3(kGatherWarps * 32), gsm, st, true,
                           (const __nv_bfloat16*)dY, dV, s)) != cudaSuccess)
      return e;
    if ((e = tc_rows_middle(X, R, Z, s, status, st)) != cudaSuccess) return e;
    if ((e = tc_rows_dual(dV, Lt, Rt, dX, dU, s, status, st)) != cudaSuccess) return e;
  }
  const int ngl = s.nb2 / 8, ngr = s.nb1 / 8;
  dim3 grid((unsigned)nsplit, (unsigned)(ngl + ngr));
  const int ncols = (int)s.n_mid();  // dV, Z, dU, X all have n_mid = n_in = n_out columns here
  if (split) {
    constexpr int smem = 2 * 2 * 32 * (8 * 64 * 2 + 16);
    if ((e = cudaFuncSetAttribute(wgrad_kernel<64, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem)) != cudaSuccess)
      return e;
    e = launch_kernel(wgrad_kernel<64, 32>, grid, dim3(256), smem, st, true, (const __nv_bfloat16*)dV,
                      (const __nv_bfloat16*)Z, (const __nv_bfloat16*)dU, (const __nv_bfloat16*)X, ngl,
                      s.rows, nsplit, part, nR, nP, ncols);
  } else if (s.nb1 == 32) {
    constexpr int smem = 2 * 2 * kWgChunk * (8 * 32 * 2 + 16);
    if ((e = cudaFuncSetAttribute(wgrad_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem)) != cudaSuccess)
      return e;
    e = launch_kernel(wgrad_kernel<32>, grid, dim3(256), smem, st, true, (const __nv_bfloat16*)dV,
                      (const __nv_bfloat16*)Z, (const __nv_bfloat16*)dU, (const __nv_bfloat16*)X, ngl,
                      s.rows, nsplit, part, nR, nP, ncols);
  } else {
    constexpr int smem = 2 * 2 * kWgChunk * (8 * 16 * 2 + 16);
    if ((e = cudaFuncSetAttribute(wgrad_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem)) != cudaSuccess)
      return e;
    e = launch_kernel(wgrad_kernel<16>, grid, dim3(256), smem, st, true, (const __nv_bfloat16*)dV,
                      (const __nv_bfloat16*)Z, (const __nv_bfloat16*)dU, (const __nv_bfloat16*)X, ngl,
                      s.rows, nsplit, part, nR, nP, ncols);
  }
  if (e != cudaSuccess) return e;
  return launch_kernel(reduce_partials_kernel, dim3((unsigned)((nP + 255) / 256)), dim3(256), 0, st, true,
                       (const float*)part, (__nv_bfloat16*)dR, (__nv_bfloat16*)dL, nR, nP, nsplit);
}

}  // namespace monarch
