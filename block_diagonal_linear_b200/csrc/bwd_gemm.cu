// Backward on the generic tcgen05 GEMM (tc_gemm.cu), for shapes whose permutation P moves
// whole 64-column groups: no output transpose, in2 a multiple of nb1, and in2 / nb1 (the
// run of middle positions p that one L block takes from each R block) a multiple of 64 --
// e.g. the nblocks = 4 layer 1024 -> 4096 (R: 4 blocks 256 x 256, L: 4 blocks 1024 x 256).
//
// Index facts used (notation of monarch.h; G = in2 / nb1):
//   Z[j][q] = u[k][p]  with  q = p'*nb1 + k,  p = j*G + p'   (p' < G, k < nb1).
// Reordering the K index of the L stage as kappa = k*G + p' turns Z_j into nb1 column ranges
// u[k][j*G .. j*G + G) of the block-contiguous middle vector U, i.e. whole 64-column groups.
// The same reordering applied to the rows of L^T makes the dual stage write dU directly.
//
//   1. Rt[k][i][p] = R[k][p][i];  Ltp[j][kappa][o] = L[j][o][q(kappa)]      (prep kernel)
//   2. U  = blockdiag(R) X                   (GEMM, block-contiguous u[k][p])
//   3. dU = blockdiag(Ltp) dY                 (GEMM; output groups scattered to u[k][p] order)
//   4. dX = blockdiag(Rt) dU                  (GEMM)
//   5. dR[k] = sum_rows dU_k^T X_k,  dL[j] = sum_rows dY_j^T Z_j   (weight-gradient GEMMs, rows
//      as K, split into chunks; Z_j read from U through the same 64-column groups, its
//      columns mapped back from kappa to q when the partials are written)
//   6. dR, dL = fixed-order sum of the partials (reduce_partials_kernel)
#include "common.cuh"
#include "tc_common.cuh"
#include "tc_gemm.cuh"

namespace monarch {

__global__ void reduce_partials_kernel(const float* __restrict__ partial, __nv_bfloat16* __restrict__ dR,
                                       __nv_bfloat16* __restrict__ dL, int64_t nR, int64_t nP, int nsplit);

static int pick_bn(int n) { return n % 256 == 0 ? 256 : (n % 128 == 0 ? 128 : 64); }

bool gemm_bwd_supported(const Shape& s) {
  if (s.out_transpose) return false;
  if (s.in1 % 64 || s.out1 % 128 || s.out2 % 128 || s.in2 % s.nb1) return false;
  const int G = s.in2 / s.nb1;
  if (G % 64) return false;
  if (s.nb1 * s.out1 != s.nb2 * s.in2) return false;
  if (s.in2 > 65536) return false;  // the forward's column permutation stages one row of L per warp
  return s.n_in() <= (1 << 20) && s.n_out() <= (1 << 20);
}

// ---------------------------------------------------------------- prep
// Block transposes of the factors, with an optional column map:
//   dst[b][c][r] = src[b][r][cmap(c)],  r < A, c < B,  cmap(c) = (c % G)*nbk + c / G  (G > 0), else c.
// One CTA per (block b, 32 source rows): the rows are read with coalesced loads into shared
// memory (row pitch B + 2 elements, so the column reads of the write phase spread over the
// banks), then every destination row segment of 32 values (64 bytes) is written by four
// threads with 16-byte stores.  Needs A % 8 == 0 and B % 8 == 0.
struct FactorT {
  const __nv_bfloat16* src;
  __nv_bfloat16* dst;
  int nblk, A, B, G, nbk;
  int ctas;  // nblk * ceil(A / 32)
};

__device__ __forceinline__ void factor_tile(const FactorT& f, int cta, uint16_t* sm) {
  const int tiles = (f.A + 31) / 32;
  const int b = cta / tiles, r0 = (cta % tiles) * 32;
  const int nr = min(32, f.A - r0);
  const int pitch = f.B + 2;
  const uint16_t* src = (const uint16_t*)f.src + ((int64_t)b * f.A + r0) * f.B;
  const int cpr = f.B / 8;
  for (int c = threadIdx.x; c < nr * cpr; c += blockDim.x) {
    const int rr = c / cpr, cc = c % cpr;
    const uint4 v = *(const uint4*)(src + (int64_t)rr * f.B + cc * 8);
    uint32_t* d = (uint32_t*)(sm + rr * pitch + cc * 8);  // 4-byte aligned: pitch is even
    d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
  }
  __syncthreads();
  uint16_t* dst = (uint16_t*)f.dst + (int64_t)b * f.B * f.A + r0;
  for (int w = threadIdx.x; w < f.B * 4; w += blockDim.x) {
    const int c = w >> 2, t = w & 3;
    if (8 * t >= nr) continue;
    const int q = f.G > 0 ? (c % f.G) * f.nbk + c / f.G : c;
    uint32_t v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      v[e] = (uint32_t)sm[(8 * t + 2 * e) * pitch + q] | ((uint32_t)sm[(8 * t + 2 * e + 1) * pitch + q] << 16);
    *(uint4*)(dst + (int64_t)c * f.A + 8 * t) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

// after_reader: launched (with programmatic dependent launch) right behind a kernel that neither
// reads nor writes Rt / Lt and that passed its own grid-dependency wait before letting this grid
// start; then every earlier reader of Rt / Lt has finished, so the transposes run concurrently
// with that kernel and wait for it only at the end (so that the kernels after this one, which
// wait for this grid, also see that kernel's results).  Otherwise: the usual wait first.
__global__ void __launch_bounds__(256) factor_transpose_kernel(FactorT f0, FactorT f1, int after_reader) {
  extern __shared__ __align__(16) uint16_t fsm[];
  if (!after_reader) ptx::griddep_wait();  // the outputs may still be read by the previous kernels
  ptx::griddep_launch_dependents();
  const int cta = (int)blockIdx.x;
  if (cta < f0.ctas)
    factor_tile(f0, cta, fsm);
  else
    factor_tile(f1, cta - f0.ctas, fsm);
  if (after_reader) ptx::griddep_wait();
}

static FactorT factor_job(const void* src, void* dst, int nblk, int A, int B, int G, int nbk) {
  FactorT f;
  f.src = (const __nv_bfloat16*)src;
  f.dst = (__nv_bfloat16*)dst;
  f.nblk = nblk; f.A = A; f.B = B; f.G = G; f.nbk = nbk;
  f.ctas = nblk * ((A + 31) / 32);
  return f;
}

bool factor_transpose_ok(int A, int B) { return A % 8 == 0 && B % 8 == 0 && B <= 2048; }

__global__ void factor_transpose_flat_kernel(const __nv_bfloat16* __restrict__ R, const __nv_bfloat16* __restrict__ L,
                                             __nv_bfloat16* __restrict__ Rt, __nv_bfloat16* __restrict__ Lt, Shape s,
                                             int G);

// Rt[k][i][p] = R[k][p][i] and Lt[j][c][o] = L[j][o][cmap(c)] in one launch (G as above).
cudaError_t factor_transposes(const void* R, void* Rt, const void* L, void* Lt, const Shape& s, int G,
                              cudaStream_t st, bool after_reader) {
  if (!factor_transpose_ok(s.out1, s.in1) || !factor_transpose_ok(s.out2, s.in2)) {
    const int64_t n = s.n_R() + s.n_L();
    return launch_kernel(factor_transpose_flat_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, true,
                         (const __nv_bfloat16*)R, (const __nv_bfloat16*)L, (__nv_bfloat16*)Rt, (__nv_bfloat16*)Lt, s,
                         G);
  }
  const FactorT f0 = factor_job(R, Rt, s.nb1, s.out1, s.in1, 0, 0);
  const FactorT f1 = factor_job(L, Lt, s.nb2, s.out2, s.in2, G, s.nb1);
  const int bmax = s.in1 > s.in2 ? s.in1 : s.in2;
  const size_t smem = (size_t)32 * (size_t)(bmax + 2) * 2;
  cudaError_t e = ensure_smem_attr((const void*)factor_transpose_kernel, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(factor_transpose_kernel, dim3((unsigned)(f0.ctas + f1.ctas)), dim3(256), smem, st, true, f0,
                       f1, after_reader ? 1 : 0);
}

// Elementwise form of the same transposes, for factor widths beyond the staged tile.
__global__ void factor_transpose_flat_kernel(const __nv_bfloat16* __restrict__ R, const __nv_bfloat16* __restrict__ L,
                                             __nv_bfloat16* __restrict__ Rt, __nv_bfloat16* __restrict__ Lt, Shape s,
                                             int G) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t nR = s.n_R(), nL = s.n_L();
  if (e < nR) {
    const int64_t k = e / ((int64_t)s.in1 * s.out1), rem = e % ((int64_t)s.in1 * s.out1);
    const int i = (int)(rem / s.out1), p = (int)(rem % s.out1);
    Rt[e] = R[(k * s.out1 + p) * s.in1 + i];
  } else if (e < nR + nL) {
    const int64_t f = e - nR;
    const int64_t j = f / ((int64_t)s.in2 * s.out2), rem = f % ((int64_t)s.in2 * s.out2);
    const int c = (int)(rem / s.out2), o = (int)(rem % s.out2);
    const int q = G > 0 ? (c % G) * s.nb1 + c / G : c;
    Lt[f] = L[(j * s.out2 + o) * s.in2 + q];
  }
}

// Lp[row][kappa] = L[row][q(kappa)] for every row of L (one row per warp, staged in shared memory).
constexpr int kPermColWarps = 8;
__global__ void __launch_bounds__(kPermColWarps * 32)
    permute_cols_kernel(const __nv_bfloat16* __restrict__ L, __nv_bfloat16* __restrict__ Lp, int64_t nrows,
                        int ncols, int G, int nbk) {
  extern __shared__ __align__(16) uint16_t pcs[];
  // launched right behind the R-stage GEMM, which does not touch Lp and passed its own
  // grid-dependency wait before this grid could start: run concurrently with it, and wait for
  // it at the end only (the L-stage GEMM after this grid needs both)
  ptx::griddep_launch_dependents();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, nw = blockDim.x / 32;
  uint16_t* buf = pcs + warp * ncols;
  for (int64_t r = (int64_t)blockIdx.x * nw + warp; r < nrows; r += (int64_t)gridDim.x * nw) {
    const uint16_t* src = (const uint16_t*)L + r * ncols;
    for (int c = lane; c < ncols / 8; c += 32) *(uint4*)(buf + c * 8) = *(const uint4*)(src + c * 8);
    __syncwarp();
    uint16_t* dst = (uint16_t*)Lp + r * ncols;
    for (int c = lane; c < ncols / 8; c += 32) {
      uint32_t v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k0 = c * 8 + 2 * e, k1 = k0 + 1;
        v[e] = (uint32_t)buf[(k0 % G) * nbk + k0 / G] | ((uint32_t)buf[(k1 % G) * nbk + k1 / G] << 16);
      }
      *(uint4*)(dst + c * 8) = make_uint4(v[0], v[1], v[2], v[3]);
    }
    __syncwarp();
  }
  ptx::griddep_wait();
}

// ---------------------------------------------------------------- weight gradient
// Split of the rows for the weight-gradient GEMMs: chunks of a multiple of 64 rows, enough of
// them that the two products (dR and dL, one launch) give about two units per SM, but at least
// 256 rows each (every chunk costs one fp32 copy of the parameters in partials), and none of
// them empty (an empty chunk would leave its partials unwritten).
WgradSplit wgrad_split(int64_t rows, int64_t units_per_split) {
  int64_t n = (2 * 148 + units_per_split - 1) / (units_per_split > 0 ? units_per_split : 1);
  const int64_t maxs = rows / 256;
  if (n > maxs) n = maxs;
  if (n < 1) n = 1;
  WgradSplit w;
  const int64_t per = (rows + n - 1) / n;
  w.rows_per_split = ((per + 63) / 64) * 64;
  if (w.rows_per_split < 64) w.rows_per_split = 64;
  w.nsplit = (int)((rows + w.rows_per_split - 1) / w.rows_per_split);
  if (w.nsplit < 1) w.nsplit = 1;
  return w;
}

// dW[b][m][n] = sum_rows A1[r][b*blk_a + m] * gathered(A2)[r][b*blk_b + n] as fp32 partials.
// A1 is block-contiguous with blocks of blk_a columns; A2's block b occupies the logical
// columns [b*blk_b, (b+1)*blk_b).  With b_grp = 0, A2 is block-contiguous too; otherwise its
// 64-column groups are gathered: group g of block b starts at b*b_base + (g / b_grp)*b_gs +
// (g % b_grp)*64.  Partials are in logical column order.
static int wgrad_job(const WgradArgs& w, GemmJob* jp) {
  GemmJob j = {};
  // M side: a group of 128 columns of A1 holding bpg whole blocks, or one block per group in
  // 128-row tiles (rows of a tile beyond the block belong to the next block and are dropped)
  int64_t bpg = 1;  // blocks per group
  if (w.blk_a <= 128 && 128 % w.blk_a == 0 && w.nblocks % (128 / w.blk_a) == 0) bpg = 128 / w.blk_a;
  j.mtiles = (int)((w.blk_a + 127) / 128);
  const int64_t nw = bpg * w.blk_b;  // B columns a group needs
  const int BN = nw >= 256 ? 256 : (nw > 64 ? 128 : 64);
  if ((bpg * w.blk_a) % 8 || (bpg * w.b_base) % 8 || nw % 8) return 0;  // 16-byte TMA x
  if (w.blk_a % 4 || w.blk_b % 4 || w.p_stride % 4 || w.p_off % 4) return 0;  // float4 partials
  j.nb = (int)(w.nblocks / bpg);
  j.ntiles = (int)((nw + BN - 1) / BN);
  j.nsplit = w.sp.nsplit;
  j.split_rows = w.sp.rows_per_split;
  j.a_b = (int)(bpg * w.blk_a);
  j.b_lb = (int)nw;
  if (w.b_grp == 0) {  // contiguous
    j.b_b = (int)nw;
    j.b_grp = 1 << 30;
    j.b_gs = 0;
  } else {
    j.b_b = (int)(bpg * w.b_base);
    j.b_grp = w.b_grp;
    j.b_gs = w.b_gs;
  }
  j.blk_a = w.blk_a;
  j.blk_b = w.blk_b;
  j.p_stride = w.p_stride;
  j.p_off = w.p_off;
  *jp = j;
  return BN;
}

cudaError_t wgrad_tc(const void* A1, int64_t a_cols, int64_t blk_a, const void* A2, int64_t b_cols, int64_t blk_b,
                     int64_t nblocks, int b_base, int b_grp, int b_gs, int64_t rows, WgradSplit sp, float* partial,
                     int64_t p_stride, int64_t p_off, int* status, cudaStream_t st) {
  const WgradArgs w = {A1, a_cols, blk_a, A2, b_cols, blk_b, nblocks, b_base, b_grp, b_gs, sp, p_stride, p_off};
  GemmJob j;
  const int BN = wgrad_job(w, &j);
  if (BN == 0) return cudaErrorInvalidValue;
  return gemm_wgrad(A1, a_cols, A2, b_cols, rows, BN, j, partial, status, st, true);
}

cudaError_t wgrad_tc2(const WgradArgs& w1, const WgradArgs& w2, int64_t rows, float* partial, int* status,
                      cudaStream_t st) {
  GemmJob j1, j2;
  const int bn1 = wgrad_job(w1, &j1), bn2 = wgrad_job(w2, &j2);
  if (bn1 == 0 || bn2 == 0) return cudaErrorInvalidValue;
  if (bn1 != bn2) {
    cudaError_t e = gemm_wgrad(w1.A1, w1.a_cols, w1.A2, w1.b_cols, rows, bn1, j1, partial, status, st, true);
    if (e != cudaSuccess) return e;
    return gemm_wgrad(w2.A1, w2.a_cols, w2.A2, w2.b_cols, rows, bn2, j2, partial, status, st, true);
  }
  const WgradOperands o1 = {w1.A1, w1.a_cols, w1.A2, w1.b_cols}, o2 = {w2.A1, w2.a_cols, w2.A2, w2.b_cols};
  return gemm_wgrad2(o1, j1, o2, j2, rows, bn1, partial, status, st, true);
}

// Row split for one weight-gradient launch on its own: as many chunks (multiples of 64 rows,
// at least 256 rows each) as keep the launch to one wave of units on the SMs.
WgradSplit wgrad_split_wave(int64_t rows, int64_t units_per_split) {
  int64_t n = 148 / (units_per_split > 0 ? units_per_split : 1);
  const int64_t maxs = rows / 256;
  if (n > maxs) n = maxs;
  if (n < 1) n = 1;
  WgradSplit w;
  const int64_t per = (rows + n - 1) / n;
  w.rows_per_split = ((per + 63) / 64) * 64;
  if (w.rows_per_split < 64) w.rows_per_split = 64;
  w.nsplit = (int)((rows + w.rows_per_split - 1) / w.rows_per_split);
  if (w.nsplit < 1) w.nsplit = 1;
  return w;
}

// dR = fixed-order sum of its nsR partials (nR values each, from partial[0]); dL = fixed-order
// sum of its nsL partials (nL values each, after dR's).  The dL partials are in gathered order:
// in-block column kappa holds dL[j][o][q] with q = (kappa % G)*nb1 + kappa / G.  Threads walk
// the partials in their own order (coalesced reads) and scatter the bf16 results.
__global__ void reduce_partials_gathered_kernel(const float* __restrict__ partial, __nv_bfloat16* __restrict__ dR,
                                                __nv_bfloat16* __restrict__ dL, int64_t nR, int64_t nL, int nsR,
                                                int nsL, int in2, int nb1, int G) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nR + nL) return;
  float acc = 0.f;
  if (e < nR) {
    for (int sp = 0; sp < nsR; ++sp) acc += partial[(int64_t)sp * nR + e];
    dR[e] = __float2bfloat16_rn(acc);
  } else {
    const int64_t f = e - nR;  // position in the gathered partial layout
    const float* pl = partial + (int64_t)nsR * nR + f;
    for (int sp = 0; sp < nsL; ++sp) acc += pl[(int64_t)sp * nL];
    const int kappa = (int)(f % in2);
    dL[f - kappa + (int64_t)(kappa % G) * nb1 + kappa / G] = __float2bfloat16_rn(acc);
  }
}

// ---------------------------------------------------------------- host
static size_t al256(size_t b) { return (b + 255) & ~size_t(255); }

struct GemmBwdWs {
  size_t rt, ltp, u, du, part, total;
  WgradSplit spR, spL;  // each weight-gradient job has its own row split
};

// Units of one row chunk of the weight-gradient GEMM: blocks x block/128 m tiles x K/BN n tiles.
static int64_t wgrad_units_one(int nb, int out, int in) {
  const int bn = in >= 256 ? 256 : (in > 64 ? 128 : 64);
  return (int64_t)nb * (out / 128) * ((in + bn - 1) / bn);
}

static GemmBwdWs gemm_bwd_layout(const Shape& s) {
  GemmBwdWs w;
  const size_t nR = (size_t)s.n_R(), nL = (size_t)s.n_L();
  w.spR = wgrad_split_wave(s.rows, wgrad_units_one(s.nb1, s.out1, s.in1));
  w.spL = wgrad_split_wave(s.rows, wgrad_units_one(s.nb2, s.out2, s.in2));
  w.rt = 0;
  w.ltp = w.rt + al256(nR * 2);
  w.u = w.ltp + al256(nL * 2);
  w.du = w.u + al256((size_t)s.rows * (size_t)s.n_mid() * 2);
  w.part = w.du + al256((size_t)s.rows * (size_t)s.n_mid() * 2);
  w.total = w.part + al256(((size_t)w.spR.nsplit * nR + (size_t)w.spL.nsplit * nL) * 4);
  return w;
}

size_t gemm_bwd_workspace(const Shape& s) { return gemm_bwd_layout(s).total; }

cudaError_t gemm_bwd(const void* dY, const void* X, const void* R, const void* L, void* dX, void* dR, void* dL,
                     void* ws, const Shape& s, int* status, cudaStream_t st, const void* saved) {
  const GemmBwdWs w = gemm_bwd_layout(s);
  char* base = (char*)ws;
  __nv_bfloat16* Rt = (__nv_bfloat16*)(base + w.rt);
  __nv_bfloat16* Ltp = (__nv_bfloat16*)(base + w.ltp);
  __nv_bfloat16* U = (__nv_bfloat16*)(base + w.u);
  __nv_bfloat16* dU = (__nv_bfloat16*)(base + w.du);
  float* part = (float*)(base + w.part);
  const int64_t nR = s.n_R(), nL = s.n_L(), nP = nR + nL;
  const int G = s.in2 / s.nb1;
  cudaError_t e;
  if (s.rows > 0) {
    GemmJob j = {};
    int bn;
    if (saved != nullptr) {
      // U from the training forward's workspace: no recompute, and the prep is the first launch
      U = (__nv_bfloat16*)((const char*)saved + gemm_fwd_u_offset(s));
      if ((e = factor_transposes(R, Rt, L, Ltp, s, G, st, false)) != cudaSuccess) return e;
    } else {
      // 2. U = blockdiag(R) X
      bn = pick_bn(s.out1);
      j.nb = s.nb1; j.ntiles = s.out1 / bn; j.kboxes = s.in1 / 64;
      j.a_b = s.in1; j.a_grp = s.in1 / 64; j.a_gs = 0;
      j.b_b = s.out1;
      j.y_b = s.out1; j.y_grp = s.out1 / 64; j.y_gs = 0;
      if ((e = gemm_bd(X, s.rows, s.n_in(), R, (int64_t)s.nb1 * s.out1, s.in1, U, s.n_mid(), bn, j, status, st,
                       true)) != cudaSuccess)
        return e;
      // 1. the factor prep overlaps the U pass (which reads neither Rt nor Ltp)
      if ((e = factor_transposes(R, Rt, L, Ltp, s, G, st, true)) != cudaSuccess) return e;
    }
    // 3. dU = blockdiag(Ltp) dY, output group g of block j -> u[k][j*G + 64*(g % (G/64))], k = g / (G/64)
    j = GemmJob{};
    bn = pick_bn(s.in2);
    j.nb = s.nb2; j.ntiles = s.in2 / bn; j.kboxes = s.out2 / 64;
    j.a_b = s.out2; j.a_grp = s.out2 / 64; j.a_gs = 0;
    j.b_b = s.in2;
    j.y_b = G; j.y_grp = G / 64; j.y_gs = s.out1;
    if ((e = gemm_bd(dY, s.rows, s.n_out(), Ltp, (int64_t)s.nb2 * s.in2, s.out2, dU, s.n_mid(), bn, j, status,
                     st, true)) != cudaSuccess)
      return e;
    // 4. dX = blockdiag(Rt) dU
    j = GemmJob{};
    bn = pick_bn(s.in1);
    j.nb = s.nb1; j.ntiles = s.in1 / bn; j.kboxes = s.out1 / 64;
    j.a_b = s.out1; j.a_grp = s.out1 / 64; j.a_gs = 0;
    j.b_b = s.in1;
    j.y_b = s.in1; j.y_grp = s.in1 / 64; j.y_gs = 0;
    if ((e = gemm_bd(dU, s.rows, s.n_mid(), Rt, (int64_t)s.nb1 * s.in1, s.out1, dX, s.n_in(), bn, j, status, st,
                     true)) != cudaSuccess)
      return e;
    // 5. weight gradients
    const WgradArgs gR = {dU, s.n_mid(), s.out1, X, s.n_in(), s.in1, s.nb1, 0, 0, 0, w.spR, nR, 0};
    const WgradArgs gL = {dY, s.n_out(), s.out2, U, s.n_mid(), s.in2, s.nb2, G, G / 64, s.out1, w.spL, nL,
                          (int64_t)w.spR.nsplit * nR};
    if ((e = wgrad_tc2(gR, gL, s.rows, part, status, st)) != cudaSuccess) return e;
  } else {
    const size_t np = (size_t)w.spR.nsplit * (size_t)nR + (size_t)w.spL.nsplit * (size_t)nL;
    if ((e = cudaMemsetAsync(part, 0, sizeof(float) * np, st)) != cudaSuccess) return e;
  }
  return launch_kernel(reduce_partials_gathered_kernel, dim3((unsigned)((nP + 255) / 256)), dim3(256), 0, st, true,
                       (const float*)part, (__nv_bfloat16*)dR, (__nv_bfloat16*)dL, nR, nL, w.spR.nsplit,
                       w.spL.nsplit, s.in2, s.nb1, G);
}

// ================================================================ two-pass forward
// Y = X M^T for the same shapes as gemm_bwd, with caller scratch:
//   1. Lp[j][o][kappa] = L[j][o][q(kappa)]   (kappa = k*G + p', q = p'*nb1 + k)
//   2. U  = blockdiag(R) X                    (GEMM, block-contiguous u[k][p])
//   3. Y  = blockdiag(Lp) gathered(U)          (GEMM; block j's K stage kb reads the 64 columns
//                                             of U at k*out1 + j*G + 64*(kb % (G/64)))
size_t gemm_fwd_u_offset(const Shape& s) { return al256((size_t)s.n_L() * 2); }

size_t gemm_fwd_workspace(const Shape& s) {
  return al256((size_t)s.n_L() * 2) + al256((size_t)s.rows * (size_t)s.n_mid() * 2);
}

cudaError_t gemm_fwd(const void* X, const void* R, const void* L, void* Y, void* ws, const Shape& s, int* status,
                     cudaStream_t st) {
  if (s.rows == 0) return cudaSuccess;
  __nv_bfloat16* Lp = (__nv_bfloat16*)ws;
  __nv_bfloat16* U = (__nv_bfloat16*)((char*)ws + al256((size_t)s.n_L() * 2));
  const int G = s.in2 / s.nb1;
  cudaError_t e;
  GemmJob j = {};
  int bn = pick_bn(s.out1);
  j.nb = s.nb1; j.ntiles = s.out1 / bn; j.kboxes = s.in1 / 64;
  j.a_b = s.in1; j.a_grp = s.in1 / 64; j.a_gs = 0;
  j.b_b = s.out1;
  j.y_b = s.out1; j.y_grp = s.out1 / 64; j.y_gs = 0;
  if ((e = gemm_bd(X, s.rows, s.n_in(), R, (int64_t)s.nb1 * s.out1, s.in1, U, s.n_mid(), bn, j, status, st, true)) !=
      cudaSuccess)
    return e;
  // the column permutation of L overlaps the R-stage pass; one staged row per warp, up to 8
  // warps, as many as 200 KB of shared memory holds
  const int64_t lrows = (int64_t)s.nb2 * s.out2;
  int nw = (int)((200 * 1024) / ((size_t)s.in2 * 2));
  if (nw > kPermColWarps) nw = kPermColWarps;
  if (nw < 1) return cudaErrorNotSupported;
  const size_t psm = (size_t)nw * (size_t)s.in2 * 2;
  if ((e = ensure_smem_attr((const void*)permute_cols_kernel, (int)psm)) != cudaSuccess) return e;
  if ((e = launch_kernel(permute_cols_kernel, dim3((unsigned)((lrows + nw - 1) / nw)), dim3(nw * 32), psm, st,
                         true, (const __nv_bfloat16*)L, Lp, lrows, s.in2, G, s.nb1)) != cudaSuccess)
    return e;
  j = GemmJob{};
  bn = pick_bn(s.out2);
  j.nb = s.nb2; j.ntiles = s.out2 / bn; j.kboxes = s.in2 / 64;
  j.a_b = G; j.a_grp = G / 64; j.a_gs = s.out1;
  j.b_b = s.out2;
  j.y_b = s.out2; j.y_grp = s.out2 / 64; j.y_gs = 0;
  return gemm_bd(U, s.rows, s.n_mid(), Lp, (int64_t)s.nb2 * s.out2, s.in2, Y, s.n_out(), bn, j, status, st, true);
}

// ================================================================ packed block-diagonal path
// Any bf16 shape whose small blocks pack into 64-multiples: g consecutive blocks of a
// block-diagonal stage are one GEMM against a (g*N) x (g*K) block-diagonal weight tile with
// zeros off the diagonal (g times the flops, which the tensor cores have to spare on these
// memory-bound shapes).  The permutations are per-row transposes:
//   dV = P_out^-1 dY,  dZ = packed(L^T) dV,  dU = P^-1 dZ,  dX = packed(R^T) dU,
//   U = packed(R) X,  Z = P U,  then the weight-gradient GEMMs and the partial sum.
int pack_factor(int nblocks, int kw, int nw) {
  for (int g = 1; g <= 8; ++g)
    if (nblocks % g == 0 && (g * kw) % 64 == 0 && (g * nw) % 64 == 0) return g;
  return 0;
}

struct PackInfo {
  int gz, gx;  // blocks per packed group: L^T stage (K = out2, N = in2), R / R^T stages
};
static PackInfo pack_info(const Shape& s) {
  PackInfo p;
  p.gz = pack_factor(s.nb2, s.out2, s.in2);
  const int a = pack_factor(s.nb1, s.in1, s.out1), b = pack_factor(s.nb1, s.out1, s.in1);
  p.gx = a > b ? a : b;
  if (p.gx && (s.nb1 % p.gx || (p.gx * s.in1) % 64 || (p.gx * s.out1) % 64)) p.gx = 0;
  return p;
}

bool packed_bwd_supported(const Shape& s) {
  const PackInfo p = pack_info(s);
  if (p.gz == 0 || p.gx == 0) return false;
  // the row-transpose passes move 16-byte chunks (8 elements of one grid row)
  if (s.nb1 % 8 || s.out1 % 8 || (s.out_transpose && (s.nb2 % 8 || s.out2 % 8))) return false;
  // packed operand widths (K stages of 64, N tiles of 64..256) and the row-transpose passes
  if ((int64_t)p.gz * s.out2 > 4096 || (int64_t)p.gx * s.in1 > 4096 || (int64_t)p.gx * s.out1 > 4096) return false;
  if (s.n_in() > 65536 || s.n_mid() > 65536 || s.n_out() > 65536) return false;
  if ((int64_t)s.out2 * (s.nb2 + 2) * 2 > 200 * 1024 || (int64_t)s.nb1 * (s.out1 + 2) * 2 > 200 * 1024 ||
      (int64_t)s.out1 * (s.nb1 + 2) * 2 > 200 * 1024)
    return false;
  return true;
}

// Wz[g][jj*in2 + q][jj'*out2 + o] = L[g*gz + jj][o][q] if jj == jj'  (dZ = Wz-stage of dV)
// Wx[g][kk*in1 + i][kk'*out1 + p] = R[g*gx + kk][p][i]                (dX = Wx-stage of dU)
// Wu[g][kk*out1 + p][kk'*in1 + i] = R[g*gx + kk][p][i]                (U  = Wu-stage of X)
__global__ void pack_weights_kernel(const __nv_bfloat16* __restrict__ R, const __nv_bfloat16* __restrict__ L,
                                    __nv_bfloat16* __restrict__ Wz, __nv_bfloat16* __restrict__ Wx,
                                    __nv_bfloat16* __restrict__ Wu, Shape s, int gz, int gx) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int64_t nz = (int64_t)s.nb2 * s.in2 * gz * s.out2;
  const int64_t nx = (int64_t)s.nb1 * s.in1 * gx * s.out1;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
  if (e < nz) {
    const int64_t kw = (int64_t)gz * s.out2, n = e / kw, k = e % kw;  // n = g*gz*in2 + jj*in2 + q
    const int64_t g = n / ((int64_t)gz * s.in2), nn = n % ((int64_t)gz * s.in2);
    const int jj = (int)(nn / s.in2), q = (int)(nn % s.in2), jk = (int)(k / s.out2), o = (int)(k % s.out2);
    Wz[e] = jj == jk ? L[((g * gz + jj) * s.out2 + o) * s.in2 + q] : zero;
  } else if (e < nz + nx) {
    const int64_t f = e - nz, kw = (int64_t)gx * s.out1, n = f / kw, k = f % kw;
    const int64_t g = n / ((int64_t)gx * s.in1), nn = n % ((int64_t)gx * s.in1);
    const int kk = (int)(nn / s.in1), i = (int)(nn % s.in1), kq = (int)(k / s.out1), p = (int)(k % s.out1);
    Wx[f] = kk == kq ? R[((g * gx + kk) * s.out1 + p) * s.in1 + i] : zero;
  } else if (e < nz + 2 * nx) {
    const int64_t f = e - nz - nx, kw = (int64_t)gx * s.in1, n = f / kw, k = f % kw;
    const int64_t g = n / ((int64_t)gx * s.out1), nn = n % ((int64_t)gx * s.out1);
    const int kk = (int)(nn / s.out1), p = (int)(nn % s.out1), kq = (int)(k / s.in1), i = (int)(k % s.in1);
    Wu[f] = kk == kq ? R[((g * gx + kk) * s.out1 + p) * s.in1 + i] : zero;
  }
}

// The factors the streaming-stage form of the packed backward needs, in one launch:
// Wx as in pack_weights_kernel (the packed dX stage) and Lt[j][c][o] = L[j][o][c] (the L^T stage).
__global__ void pack_staged_kernel(const __nv_bfloat16* __restrict__ R, const __nv_bfloat16* __restrict__ L,
                                   __nv_bfloat16* __restrict__ Wx, __nv_bfloat16* __restrict__ Lt, Shape s, int gx) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int64_t nx = (int64_t)s.nb1 * s.in1 * gx * s.out1, nL = s.n_L();
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e < nx) {
    const int64_t kw = (int64_t)gx * s.out1, n = e / kw, k = e % kw;
    const int64_t g = n / ((int64_t)gx * s.in1), nn = n % ((int64_t)gx * s.in1);
    const int kk = (int)(nn / s.in1), i = (int)(nn % s.in1), kq = (int)(k / s.out1), p = (int)(k % s.out1);
    Wx[e] = kk == kq ? R[((g * gx + kk) * s.out1 + p) * s.in1 + i] : __float2bfloat16_rn(0.f);
  } else if (e < nx + nL) {
    const int64_t f = e - nx, per = (int64_t)s.in2 * s.out2, j = f / per, rem = f % per;
    const int c = (int)(rem / s.out2), o = (int)(rem % s.out2);
    Lt[f] = L[(j * s.out2 + o) * s.in2 + c];
  }
}

// Wp[grp][jj*nw + n][jj'*kw + k] = W[grp*g + jj][n][k] if jj == jj' (else 0), from W (nb, nw, kw);
// with trans, W is read as (nb, kw, nw) and transposed: Wp[...][jj*nw + n][jj*kw + k] = W[b][k][n].
__global__ void pack_bd_kernel(const __nv_bfloat16* __restrict__ W, __nv_bfloat16* __restrict__ Wp, int nb,
                               int nw, int kw, int g, int trans) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const int64_t n_all = (int64_t)nb * nw * g * kw;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_all) return;
  const int64_t K = (int64_t)g * kw, row = e / K, col = e % K;
  const int64_t grp = row / ((int64_t)g * nw), rr = row % ((int64_t)g * nw);
  const int jj = (int)(rr / nw), n = (int)(rr % nw), jk = (int)(col / kw), k = (int)(col % kw);
  const int64_t b = grp * g + jj;
  Wp[e] = jj != jk ? __float2bfloat16_rn(0.f)
                   : (trans ? W[(b * kw + k) * nw + n] : W[(b * nw + n) * kw + k]);
}

cudaError_t pack_bd(const void* W, void* Wp, int nb, int nw, int kw, int g, bool trans, cudaStream_t st) {
  const int64_t n_all = (int64_t)nb * nw * g * kw;
  return launch_kernel(pack_bd_kernel, dim3((unsigned)((n_all + 255) / 256)), dim3(256), 0, st, true,
                       (const __nv_bfloat16*)W, (__nv_bfloat16*)Wp, nb, nw, kw, g, trans ? 1 : 0);
}

struct PackedWs {
  size_t wz, wx, wu, dv, dz, du, u, z, part, total;
  WgradSplit sp;
};

static int64_t wgrad_units(int64_t nblocks, int64_t blk_a, int64_t blk_b) {
  int64_t bpg = 1;
  if (blk_a <= 128 && 128 % blk_a == 0 && nblocks % (128 / blk_a) == 0) bpg = 128 / blk_a;
  const int64_t nw = bpg * blk_b;
  const int64_t bn = nw >= 256 ? 256 : (nw > 64 ? 128 : 64);
  return (nblocks / bpg) * ((blk_a + 127) / 128) * ((nw + bn - 1) / bn);
}

static PackedWs packed_layout(const Shape& s) {
  const PackInfo pk = pack_info(s);
  PackedWs w;
  const size_t rows = (size_t)s.rows;
  w.sp = wgrad_split_wave(s.rows, wgrad_units(s.nb1, s.out1, s.in1) + wgrad_units(s.nb2, s.out2, s.in2));
  w.wz = 0;
  w.wx = w.wz + al256((size_t)s.nb2 * s.in2 * pk.gz * s.out2 * 2);
  w.wu = w.wx + al256((size_t)s.nb1 * s.in1 * pk.gx * s.out1 * 2);
  w.dv = w.wu + al256((size_t)s.nb1 * s.in1 * pk.gx * s.out1 * 2);
  w.dz = w.dv + (s.out_transpose ? al256(rows * (size_t)s.n_out() * 2) : 0);
  w.du = w.dz + al256(rows * (size_t)s.n_mid() * 2);
  w.u = w.du + al256(rows * (size_t)s.n_mid() * 2);
  w.z = w.u + al256(rows * (size_t)s.n_mid() * 2);
  w.part = w.z + al256(rows * (size_t)s.n_mid() * 2);
  w.total = w.part + al256((size_t)w.sp.nsplit * (size_t)(s.n_R() + s.n_L()) * 4);
  return w;
}

size_t packed_bwd_workspace(const Shape& s) { return packed_layout(s).total; }

// Y (rows x nb*nw) = packed block-diagonal stage of A (rows x nb*kw) with W (nb*nw x g*kw per group).
cudaError_t packed_stage(const void* A, int64_t rows, const void* W, void* Y, int nb, int kw, int nw, int g,
                                int* status, cudaStream_t st) {
  GemmJob j = {};
  const int K = g * kw, N = g * nw;
  const int bn = pick_bn(N);
  j.nb = nb / g; j.ntiles = N / bn; j.kboxes = K / 64;
  j.a_b = K; j.a_grp = 1 << 30; j.a_gs = 0;
  j.b_b = N;
  j.y_b = N; j.y_grp = 1 << 30; j.y_gs = 0;
  return gemm_bd(A, rows, (int64_t)nb * kw, W, (int64_t)nb * nw, K, Y, (int64_t)nb * nw, bn, j, status, st, true);
}

cudaError_t packed_bwd(const void* dY, const void* X, const void* R, const void* L, void* dX, void* dR, void* dL,
                       void* ws, const Shape& s, int* status, cudaStream_t st, const void* saved) {
  const PackInfo pk = pack_info(s);
  const PackedWs w = packed_layout(s);
  char* base = (char*)ws;
  __nv_bfloat16 *Wz = (__nv_bfloat16*)(base + w.wz), *Wx = (__nv_bfloat16*)(base + w.wx),
                *Wu = (__nv_bfloat16*)(base + w.wu);
  __nv_bfloat16* dV = s.out_transpose ? (__nv_bfloat16*)(base + w.dv) : (__nv_bfloat16*)dY;
  __nv_bfloat16 *dZ = (__nv_bfloat16*)(base + w.dz), *dU = (__nv_bfloat16*)(base + w.du),
                *U = (__nv_bfloat16*)(base + w.u), *Z = (__nv_bfloat16*)(base + w.z);
  float* part = (float*)(base + w.part);
  const int64_t nR = s.n_R(), nL = s.n_L(), nP = nR + nL;
  const int64_t nz = (int64_t)s.nb2 * s.in2 * pk.gz * s.out2, nx = (int64_t)s.nb1 * s.in1 * pk.gx * s.out1;
  cudaError_t e;
  const bool staged = tc_stage_supported(s);
  if (staged) {
    // the streaming stages take the plain L^T (into the otherwise unused packed L^T region); only
    // the dX stage is packed
    if (s.rows > 0 &&
        (e = launch_kernel(pack_staged_kernel, dim3((unsigned)((nx + nL + 255) / 256)), dim3(256), 0, st, true,
                           (const __nv_bfloat16*)R, (const __nv_bfloat16*)L, Wx, Wz, s, pk.gx)) != cudaSuccess)
      return e;
  } else if ((e = launch_kernel(pack_weights_kernel, dim3((unsigned)((nz + 2 * nx + 255) / 256)), dim3(256), 0, st,
                                true, (const __nv_bfloat16*)R, (const __nv_bfloat16*)L, Wz, Wx, Wu, s, pk.gz,
                                pk.gx)) != cudaSuccess) {
    return e;
  }
  if (saved != nullptr && staged) Z = (__nv_bfloat16*)saved;  // kept by the training forward
  const bool need_z = saved == nullptr || !staged;
  if (s.rows > 0) {
    if (s.out_transpose && (e = permute_rows(dY, dV, s.rows, s.out2, s.nb2, st)) != cudaSuccess) return e;
    if (staged) {
      // dU = P^-1 blockdiag(L^T) dV in one streaming stage (no dZ pass, no row transpose); L^T
      // was written two launches back when the dY permutation sits in between
      if ((e = tc_stage(dV, Wz, dU, StageKind::Lt, s, status, st, true, s.out_transpose == 1)) != cudaSuccess)
        return e;
    } else {
      if ((e = packed_stage(dV, s.rows, Wz, dZ, s.nb2, s.out2, s.in2, pk.gz, status, st)) != cudaSuccess) return e;
      if ((e = permute_rows(dZ, dU, s.rows, s.out1, s.nb1, st)) != cudaSuccess) return e;
    }
    if ((e = packed_stage(dU, s.rows, Wx, dX, s.nb1, s.out1, s.in1, pk.gx, status, st)) != cudaSuccess) return e;
    if (staged) {
      // Z = P R x (R is the caller's: its weights may load before the wait)
      if (need_z && (e = tc_stage(X, R, Z, StageKind::R, s, status, st, true, true)) != cudaSuccess) return e;
    } else {
      if ((e = packed_stage(X, s.rows, Wu, U, s.nb1, s.in1, s.out1, pk.gx, status, st)) != cudaSuccess) return e;
      if ((e = permute_rows(U, Z, s.rows, s.nb1, s.out1, st)) != cudaSuccess) return e;
    }
    const WgradArgs gR = {dU, s.n_mid(), s.out1, X, s.n_in(), s.in1, s.nb1, 0, 0, 0, w.sp, nP, 0};
    const WgradArgs gL = {dV, s.n_out(), s.out2, Z, s.n_mid(), s.in2, s.nb2, 0, 0, 0, w.sp, nP, nR};
    if ((e = wgrad_tc2(gR, gL, s.rows, part, status, st)) != cudaSuccess) return e;
  } else if ((e = cudaMemsetAsync(part, 0, sizeof(float) * (size_t)w.sp.nsplit * (size_t)nP, st)) != cudaSuccess) {
    return e;
  }
  return launch_kernel(reduce_partials_kernel, dim3((unsigned)((nP + 255) / 256)), dim3(256), 0, st, true,
                       (const float*)part, (__nv_bfloat16*)dR, (__nv_bfloat16*)dL, nR, nP, w.sp.nsplit);
}

}  // namespace monarch
