// Job description and launchers of the generic tcgen05 GEMM (tc_gemm.cu).
#pragma once

#include "common.cuh"

namespace monarch {

// One GEMM launch.  Column addressing uses one "gathered column" rule throughout: the
// 64-column group g of batch b starts at  b*base + (g / grp)*gs + (g % grp)*64,  which is a
// plain contiguous range when grp covers every group, and otherwise gathers 64-column
// groups that lie gs apart (a permutation whose groups are 64 columns wide).
// Kind 0 (block-diagonal stage, K-major, bf16 out): unit = (m tile of 128 rows, batch b,
// n tile of BN).  A group = K stage kb (a_b, a_grp, a_gs); W rows b*b_b + nt*BN, K columns
// kb*64; output group = nt*(BN/64) + chunk (y_b, y_grp, y_gs).
// Kind 1 (weight gradient, MN-major, fp32 partials): unit = (split, group b, m tile, n tile);
// A columns b*a_b + mt*128 (contiguous), B group = nt*(BN/64) + h (b_b, b_grp, b_gs); rows
// [split*split_rows, +split_rows).  D[m][n] is kept when column m of act1 and the B column
// n lie in the same block: m_g = b*a_b + mt*128 + m, n_g = b*b_lb + nt*BN + n (the logical
// position, before gathering); block = m_g / blk_a must equal n_g / blk_b; the value goes to
// partial[split*p_stride + p_off + block*blk_a*blk_b + (m_g % blk_a)*blk_b + n_g % blk_b]
// (logical column order: a column permutation of gathered operands is applied by the
// partial sum).  blk_a, blk_b, p_off, p_stride are multiples of 4 (float4 stores).
struct GemmJob {
  int kind;
  int nb, mtiles, ntiles, nsplit;
  int kboxes;                 // kind 0: 64-wide K stages per unit
  int a_b, a_grp, a_gs;       // A columns (kind 0 gathered by K stage; kind 1 contiguous)
  int b_b, b_grp, b_gs;       // kind 0: W rows per batch (b_b); kind 1: gathered B columns
  int b_lb;                   // kind 1: logical B column offset per batch (block ownership)
  int y_b, y_grp, y_gs;       // kind 0: gathered output columns
  int64_t rows, split_rows;   // kind 1
  int64_t a_cols, b_cols;     // kind 1: widths of act1, act2
  int64_t blk_a, blk_b;       // kind 1: block widths (M side, N side, before gathering)
  int64_t p_stride, p_off;    // kind 1: partial layout
  int64_t units;
  int ab3d;                   // kind 1: A and B maps are 3-D (64 columns, rows, 64-column chunks)
                              // and a stage fetches each operand with one multi-chunk box
};

__host__ __device__ __forceinline__ int gcol(int b, int base, int g, int grp, int gs) {
  return b * base + (g / grp) * gs + (g % grp) * 64;
}

// Kind 0: A (rows x a_cols), W (w_rows x K), Y (rows x y_cols); BN in {64, 128, 256}.
// job: nb, ntiles, kboxes, a_b, a_grp, a_gs, b_b, y_b, y_grp, y_gs.
cudaError_t gemm_bd(const void* A, int64_t rows, int64_t a_cols, const void* W, int64_t w_rows, int K,
                    void* Y, int64_t y_cols, int BN, GemmJob job, int* status, cudaStream_t st, bool pdl);
// Kind 1: act1 (rows x a_cols), act2 (rows x b_cols); BN in {64, 128, 256}.
// job: nb, mtiles, ntiles, nsplit, split_rows (multiple of 64), a_b, b_b, b_grp, b_gs, b_lb, blk_a, blk_b,
// p_stride, p_off.
cudaError_t gemm_wgrad(const void* A1, int64_t a_cols, const void* A2, int64_t b_cols, int64_t rows, int BN,
                       GemmJob job, float* partial, int* status, cudaStream_t st, bool pdl);
// Two kind-1 jobs with the same BN in one launch (the second job's units follow the first's).
struct WgradOperands {
  const void* A1;
  int64_t a_cols;
  const void* A2;
  int64_t b_cols;
};
cudaError_t gemm_wgrad2(const WgradOperands& o1, GemmJob job1, const WgradOperands& o2, GemmJob job2,
                        int64_t rows, int BN, float* partial, int* status, cudaStream_t st, bool pdl);
// CTA-pair form of a two-job kind-1 launch (tc_pair.cu): BN = 256, M side of each group a
// multiple of 256, one N tile (launch_wgrad_pair, declared where tensor maps are known).
bool wgrad_pair_ok(const GemmJob& j, int BN);

// Row split of the weight-gradient GEMMs (see bwd_gemm.cu).
struct WgradSplit {
  int nsplit;
  int64_t rows_per_split;
};
WgradSplit wgrad_split(int64_t rows, int64_t units_per_split);
WgradSplit wgrad_split_wave(int64_t rows, int64_t units_per_split);
cudaError_t wgrad_tc(const void* A1, int64_t a_cols, int64_t blk_a, const void* A2, int64_t b_cols, int64_t blk_b,
                     int64_t nblocks, int b_base, int b_grp, int b_gs, int64_t rows, WgradSplit sp, float* partial,
                     int64_t p_stride, int64_t p_off, int* status, cudaStream_t st);
// One weight-gradient product of wgrad_tc, for the two-product launch.
struct WgradArgs {
  const void* A1;
  int64_t a_cols, blk_a;
  const void* A2;
  int64_t b_cols, blk_b, nblocks;
  int b_base, b_grp, b_gs;
  WgradSplit sp;
  int64_t p_stride, p_off;  // partial[split*p_stride + p_off + ...]
};
// dR and dL partials (or any two products) in one launch when their N tiles agree, else two.
cudaError_t wgrad_tc2(const WgradArgs& w1, const WgradArgs& w2, int64_t rows, float* partial, int* status,
                      cudaStream_t st);

// Rt[k][i][p] = R[k][p][i] and Lt[j][c][o] = L[j][o][cmap(c)] (bf16), one launch;
// cmap(c) = (c % G)*nb1 + c / G when G > 0, else c.
// after_reader: the launch directly follows (on stream st) one of this library's kernels that does
// not touch Rt / Lt; the transposes then overlap it (see factor_transpose_kernel).
cudaError_t factor_transposes(const void* R, void* Rt, const void* L, void* Lt, const Shape& s, int G,
                              cudaStream_t st, bool after_reader);

// Smallest g <= 8 dividing nblocks with g*kw and g*nw multiples of 64 (0 if none).
int pack_factor(int nblocks, int kw, int nw);
// Packed block-diagonal weights (see bwd_gemm.cu) and the stage that uses them.
cudaError_t pack_bd(const void* W, void* Wp, int nb, int nw, int kw, int g, bool trans, cudaStream_t st);
cudaError_t packed_stage(const void* A, int64_t rows, const void* W, void* Y, int nb, int kw, int nw, int g,
                         int* status, cudaStream_t st);
__global__ void reduce_partials_kernel(const float* __restrict__ partial, __nv_bfloat16* __restrict__ dR,
                                       __nv_bfloat16* __restrict__ dL, int64_t nR, int64_t nP, int nsplit);

bool packed_bwd_supported(const Shape& s);
size_t packed_bwd_workspace(const Shape& s);
// saved: the middle vector Z from the training forward (used when the streaming stages serve the
// shape), or nullptr to recompute it.
cudaError_t packed_bwd(const void* dY, const void* X, const void* R, const void* L, void* dX, void* dR, void* dL,
                       void* ws, const Shape& s, int* status, cudaStream_t st, const void* saved = nullptr);

size_t gemm_fwd_workspace(const Shape& s);
cudaError_t gemm_fwd(const void* X, const void* R, const void* L, void* Y, void* ws, const Shape& s, int* status,
                     cudaStream_t st);

bool gemm_bwd_supported(const Shape& s);
size_t gemm_bwd_workspace(const Shape& s);
// saved: the workspace of the two-pass forward of the same rows (its U is reused; nullptr: recompute U)
cudaError_t gemm_bwd(const void* dY, const void* X, const void* R, const void* L, void* dX, void* dR, void* dL,
                     void* ws, const Shape& s, int* status, cudaStream_t st, const void* saved = nullptr);
// Offset of U in the two-pass forward's workspace.
size_t gemm_fwd_u_offset(const Shape& s);

}  // namespace monarch
