/*
 * monarch.h -- C ABI of libmonarch.so, the B200 (sm_100a) Monarch linear map.
 *
 * The operation (Monarch: Expressive Structured Matrices for Efficient and
 * Accurate Training, abstract; scatterbrain issue thread, "Definition C.3"):
 * a Monarch matrix is a product of two block-diagonal matrices with a fixed
 * reshape-transpose permutation between them,
 *
 *     Y = X * M^T,     M = P_out * L * P * R,
 *
 * applied to every row x of X (rows are independent):
 *   u[k][p]      = sum_i R[k][p][i] * x[k*in1 + i]        (R: nb1 blocks of out1 x in1)
 *   flat[p*nb1+k]= u[k][p]                                 (P: view (nb1,out1), transpose)
 *   Z[j][q]      = flat[j*in2 + q]                         (regroup into nb2 blocks of in2)
 *   v[j][o]      = sum_q L[j][o][q] * Z[j][q]              (L: nb2 blocks of out2 x in2)
 *   y[o*nb2 + j] = v[j][o]   if out_transpose             (P_out: transpose and flatten)
 *   y[j*out2 + o]= v[j][o]   otherwise                     (plain flatten)
 * The permutation direction follows the worked N=4 example of the scatterbrain
 * thread (x_new = [x0, x2, x1, x3]) and its lattice view: R contracts the rows
 * of the (nb1 x in1) grid, L the columns.  Factor tensors use the nn.Linear
 * weight convention of MonarchLinear's blkdiag1 / blkdiag2: (nblocks, out_blk,
 * in_blk), row-major.
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *     row-major, 16-byte aligned.  X is (rows, nb1*in1), Y and dY are
 *     (rows, nb2*out2), R and dR are (nb1, out1, in1), L and dL are
 *     (nb2, out2, in2).  All of X, R, L, Y, dY, dX, dR, dL have the element
 *     type d->dtype (fp32 or bf16).  Accumulation is always fp32; bf16 results
 *     are rounded to nearest-even.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous on it; the library never synchronises the device except in
 *     monarch_last_device_status().
 *   - The library allocates no device memory.  monarch_bwd takes a caller-owned
 *     workspace of at least monarch_bwd_workspace_bytes(d) bytes.
 *   - Outputs (and the workspace) must not overlap any input or one another;
 *     overlapping byte ranges are rejected with MONARCH_ERR_ALIAS before any
 *     device work.
 *   - Return value: MONARCH_OK (0) or a negative MONARCH_ERR_* code.  Nothing
 *     aborts, throws or prints.  A failed call leaves its outputs unspecified.
 *   - Kernel-side bounded waits that give up record MONARCH_ERR_TIMEOUT in a
 *     device status word; read it with monarch_last_device_status().
 */
#ifndef MONARCH_H_
#define MONARCH_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MONARCH_API __attribute__((visibility("default")))
#else
#define MONARCH_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MONARCH_F32 = 0,
  MONARCH_BF16 = 1
} monarch_dtype;

enum {
  MONARCH_OK = 0,
  MONARCH_ERR_DIMS = -1,        /* non-positive sizes, rows < 0, or nb1*out1 != nb2*in2 */
  MONARCH_ERR_DTYPE = -2,       /* dtype not in monarch_dtype */
  MONARCH_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned */
  MONARCH_ERR_NULL = -4,        /* a required pointer is NULL (rows > 0) */
  MONARCH_ERR_WORKSPACE = -5,   /* workspace NULL or smaller than required */
  MONARCH_ERR_CUDA = -6,        /* a CUDA runtime call or kernel launch failed */
  MONARCH_ERR_TIMEOUT = -7,     /* a bounded device wait gave up (device status) */
  MONARCH_ERR_UNSUPPORTED = -8, /* shape too large for any kernel of this library */
  MONARCH_ERR_SCRATCH = -9,     /* monarch_bwd_noalloc: problem needs more than its fixed scratch */
  MONARCH_ERR_ALIAS = -10       /* an output (or the workspace) overlaps an input or another output */
};

/* Shape of one Monarch map.  Scatterbrain thread, MonarchLinear __init__ and
 * Definition C.3: R has nb1 blocks of (out1 x in1), L has nb2 blocks of
 * (out2 x in2), and the middle width must agree: nb1*out1 == nb2*in2. */
typedef struct {
  int64_t rows;          /* rows of X (batch x tokens); 0 is a valid no-op      */
  int32_t nb1, in1, out1;
  int32_t nb2, in2, out2;
  int32_t out_transpose; /* 1: y[o*nb2 + j] = v[j][o];  0: y[j*out2 + o]         */
  int32_t dtype;         /* monarch_dtype of every tensor argument               */
} monarch_dims;

/* Host-only check of a shape: MONARCH_OK or MONARCH_ERR_DIMS / _DTYPE.  Needs
 * no GPU. */
MONARCH_API int monarch_validate(const monarch_dims* d);

/* Forward, steps R -> P -> L -> P_out for every row:  Y = X * M^T.
 * In:  X (rows, nb1*in1), R (nb1,out1,in1), L (nb2,out2,in2).
 * Out: Y (rows, nb2*out2), overwritten.
 * bf16 path: bf16 inputs, fp32 accumulation on the tensor cores, the middle
 * vector rounded to bf16 on chip, Y rounded to bf16.  fp32 path: fp32 FMA.
 * Y must not overlap X, R or L.  For square 64 x 64 blocks with nb1 = nb2
 * (monarch_fwd_path 4) Y also holds the middle vector between the passes, so
 * its contents are unspecified until the call's work on the stream is done. */
MONARCH_API int monarch_fwd(const void* X, const void* R, const void* L, const monarch_dims* d, void* Y,
                void* stream);

/* Forward with caller-provided scratch.  Same operation, arguments and results as
 * monarch_fwd; for shapes whose permutation moves whole 64-column groups (no output
 * transpose, in2 / nb1 a multiple of 64, e.g. nblocks = 4, 1024 -> 4096; monarch_fwd_ws_path
 * 5) it runs two tcgen05 GEMM passes: U = blockdiag(R) X into the workspace, then the L stage
 * reading U through 64-column gathers with L's K index reordered to match (L is reordered
 * into the workspace too).  For 64 blocks of 64 x 64 per factor (n = 4096,
 * monarch_fwd_ws_path 6) it runs two streaming stages, each with its permutation folded
 * into the output stores and its factor's weights resident in shared memory a round of 16
 * blocks at a time: Z = P blockdiag(R) X into the workspace (rows * n_mid bf16), then
 * Y = P_out blockdiag(L) Z.  For other shapes it runs the monarch_fwd kernels and needs no
 * workspace (monarch_fwd_workspace_bytes returns 0; workspace may then be NULL).
 * workspace: >= monarch_fwd_workspace_bytes(d) bytes, 256-byte aligned, caller-owned; it must
 * not overlap the inputs or Y. */
MONARCH_API size_t monarch_fwd_workspace_bytes(const monarch_dims* d);
MONARCH_API int monarch_fwd_ws_path(const monarch_dims* d);
MONARCH_API int monarch_fwd_ws(const void* X, const void* R, const void* L, const monarch_dims* d, void* Y,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Training pair: a forward that keeps what its backward needs, and that backward.
 *
 * monarch_fwd_train computes Y = X * M^T exactly as monarch_fwd_ws does (same kernels, same
 * results) and leaves the middle vector of these rows in `saved`, in the layout the backward's
 * own recompute would produce: for the fused small-block forward (monarch_fwd_path 2), the
 * wide-output forward (monarch_fwd_path 3) when the backward runs the streaming stages (e.g.
 * 768 -> 3072), and the streaming-stage forward (monarch_fwd_ws_path 6) the permuted middle
 * vector Z (rows x n_mid bf16, Z[r][j*in2 + q]); for the two-pass GEMM forward (monarch_fwd_ws_path 5) that
 * forward's whole workspace (the reordered L, then U = blockdiag(R) X).  This is what an
 * autograd framework saves for the backward of a product of factors; it trades a write and a
 * read of rows x n_mid bf16 for the backward's recompute pass (a read of X, a write of the
 * middle vector, and its flops).
 *
 * monarch_bwd_saved computes the same dX, dR, dL as monarch_bwd (bit for bit: the saved middle
 * vector equals the recomputed one) from dY, X, R, L and that `saved` buffer, skipping the
 * recompute.  For shapes and dtypes with nothing to save monarch_saved_bytes returns 0, `saved`
 * may be NULL, monarch_fwd_train runs monarch_fwd and monarch_bwd_saved runs monarch_bwd.
 *
 * saved: >= monarch_saved_bytes(d) bytes, 256-byte aligned, caller-owned; written by
 * monarch_fwd_train, read by monarch_bwd_saved with the same dims and the same X, R, L, and
 * not modified in between.  It must not overlap the other arguments.  workspace (backward):
 * >= monarch_bwd_workspace_bytes(d) bytes, as for monarch_bwd.  Errors as for monarch_fwd_ws
 * and monarch_bwd (MONARCH_ERR_WORKSPACE for a missing or short `saved`). */
MONARCH_API size_t monarch_saved_bytes(const monarch_dims* d);
MONARCH_API int monarch_fwd_train(const void* X, const void* R, const void* L, const monarch_dims* d, void* Y,
                                  void* saved, size_t saved_bytes, void* stream);
MONARCH_API int monarch_bwd_saved(const void* dY, const void* X, const void* R, const void* L,
                                  const monarch_dims* d, const void* saved, size_t saved_bytes, void* dX,
                                  void* dR, void* dL, void* workspace, size_t workspace_bytes, void* stream);

/* Backward of Y = X * M^T for a loss with gradient dY (chain rule; the middle
 * vector is recomputed from X rather than stored):
 *   dV[j][o] = dY[idx(j,o)],  dL[j][o][q] = sum_rows dV[j][o] * Z[j][q],
 *   dZ[j][q] = sum_o L[j][o][q] dV[j][o],  dU[k][p] = dZflat[p*nb1 + k],
 *   dR[k][p][i] = sum_rows dU[k][p] * x[k*in1+i],  dX[k*in1+i] = sum_p R[k][p][i] dU[k][p].
 * In:  dY (rows, n_out), X, R, L.   Out: dX (rows, n_in), dR, dL -- all
 * overwritten (not accumulated).  Weight gradients are reduced over rows in a
 * fixed order, so repeated calls give bitwise-identical results.
 * workspace: device scratch of >= monarch_bwd_workspace_bytes(d) bytes, 256-byte
 * aligned, owned by the caller, not read before it is written. */
MONARCH_API int monarch_bwd(const void* dY, const void* X, const void* R, const void* L, const monarch_dims* d,
                void* dX, void* dR, void* dL, void* workspace, size_t workspace_bytes,
                void* stream);

/* Same as monarch_bwd, for callers that cannot allocate device memory.
 * The pages describe no such entry point; it exists for integration.  Some callers
 * have no way to provide the workspace monarch_bwd wants: code that only receives
 * tensors from a host framework, processes whose device memory pool is fixed in
 * advance, or code that must not call the CUDA allocator at that point.  This
 * entry point runs the same kernels but takes its scratch from a 32 MiB array that
 * is part of the library's device code; it calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *   - Limit: problems whose monarch_bwd_workspace_bytes(d) exceeds 32 MiB are
 *     rejected with MONARCH_ERR_SCRATCH before any device work (for the n = 1024
 *     bf16 shape that is about 2000 rows; larger batches must use monarch_bwd).
 *   - Every GPU that loads the library holds the 32 MiB array until the process
 *     exits.
 *   - Every call looks up the array's device address in the calling thread's
 *     current context (cudaGetSymbolAddress, a host-side query), so the address
 *     stays valid after cudaDeviceReset and in non-primary contexts.  The first
 *     call on a device may also load the library's device code; make that first
 *     call before any stream capture.
 *   - All calls share the one array and it keeps the previous call's contents
 *     (nothing in it needs to start at zero).  Calls whose execution overlaps on
 *     the GPU (different streams, or several host threads on one device) race on
 *     it and give wrong results; serialise them.
 * Arguments, layouts and results are those of monarch_bwd. */
MONARCH_API int monarch_bwd_noalloc(const void* dY, const void* X, const void* R, const void* L,
                                    const monarch_dims* d, void* dX, void* dR, void* dL,
                                    void* stream);

/* Workspace bytes monarch_bwd needs for this shape (0 if d is invalid). */
MONARCH_API size_t monarch_bwd_workspace_bytes(const monarch_dims* d);

/* Dense equivalent for checking (scatterbrain thread: applying the multiply to
 * the identity "is essentially the full matrix"): writes M (n_out, n_in) as
 * FLOAT32 regardless of d->dtype, with Y = X * M^T.  d->rows is ignored.
 * Entry: M[idx(j,o)][k*in1+i] = sum over p with (p*nb1+k) div in2 == j of
 *        L[j][o][(p*nb1+k) mod in2] * R[k][p][i]. */
MONARCH_API int monarch_materialise(const void* R, const void* L, const monarch_dims* d, void* M,
                        void* stream);

/* Human-readable name of a status code (static string). */
MONARCH_API const char* monarch_status_string(int status);

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device: MONARCH_OK, MONARCH_ERR_TIMEOUT (a bounded wait inside a
 * kernel gave up and that kernel skipped its remaining work), or
 * MONARCH_ERR_CUDA if the synchronisation itself failed. */
MONARCH_API int monarch_last_device_status(void* stream);

/* Test hook for the bounded-wait machinery: launches one block that waits on
 * an mbarrier nothing will ever arrive on, giving up after timeout_ns
 * nanoseconds and recording MONARCH_ERR_TIMEOUT in the device status word.
 * Returns the launch status; read the outcome with
 * monarch_last_device_status(). */
MONARCH_API int monarch_debug_wait_timeout(uint64_t timeout_ns, void* stream);

/* Dense -> Monarch projection (Monarch abstract: projecting onto the Monarch set "has an
 * analytical optimal solution"; scatterbrain projection question: the dense matrix sliced
 * with rearrange(M, '(p k) (r s) -> k r p s')).  For the lattice shapes (in2 == nb1,
 * nb2 == out1, out_transpose = 1) every (j, k) slice A_jk[o][i] = M[o*nb2 + j][k*in1 + i] of
 * a Monarch matrix is the rank-1 matrix L[j][:, k] R[k][j][:]^T, and the Frobenius-nearest
 * Monarch matrix takes the best rank-1 approximation s u v^T of every slice:
 * L[j][o][k] = sqrt(s) u[o], R[k][j][i] = sqrt(s) v[i], with the entry of v largest in
 * magnitude made positive.
 * In:  M (n_out, n_in) FLOAT32 row-major (the layout monarch_materialise writes).
 * Out: R, L in d->dtype, overwritten.  fp32 power iteration per slice on the GPU (results
 * agree with an SVD to fp32 accuracy when the slice's two leading singular values are well
 * separated).  MONARCH_ERR_UNSUPPORTED for other shapes or slices wider than 1024 columns.
 * d->rows is ignored. */
MONARCH_API int monarch_project(const void* M, const monarch_dims* d, void* R, void* L, void* stream);

/* ---------------------------------------------------------------- MonarchLinear front end
 * Scatterbrain issue thread, the MonarchLinear __init__ listing: for MonarchLinear(
 * in_features, out_features, nblocks) the block sizes are in_blksz = ceil(in / nblocks) and
 * out_blksz = ceil(out / nblocks), the features are extended to in_blksz * nblocks and
 * out_blksz * nblocks, and the factors are R = blkdiag1 (nblocks, mid, in_blksz) and
 * L = blkdiag2 (nblocks, out_blksz, mid) with mid = in_blksz when the extended input is
 * narrower than the extended output and mid = out_blksz otherwise.  The listing shows no
 * forward; this library reads it as: x zero-padded to the extended width, the Monarch map
 * of that shape with no output transpose (R on contiguous slices, the transpose, L, flatten),
 * the result cut to out_features, plus an optional bias (out_features entries). */
typedef struct {
  int64_t rows;           /* rows of X                                           */
  int32_t in_features, out_features, nblocks;
  int32_t has_bias;       /* 1: bias / dbias arguments are used                  */
  int32_t dtype;          /* monarch_dtype of every tensor argument              */
} monarch_linear_dims;

/* The equivalent monarch_dims of a MonarchLinear (host-only; MONARCH_ERR_DIMS / _DTYPE on a
 * bad size or dtype). */
MONARCH_API int monarch_linear_shape(const monarch_linear_dims* ld, monarch_dims* d);

/* Device workspace bytes monarch_linear_fwd and monarch_linear_bwd need (0 if ld is bad). */
MONARCH_API size_t monarch_linear_workspace_bytes(const monarch_linear_dims* ld);

/* Y (rows, out_features) = crop(Monarch(pad(X))) + bias, X (rows, in_features).  R, L have the
 * shapes monarch_linear_shape gives; bias may be NULL when has_bias is 0.  workspace: device
 * memory of >= monarch_linear_workspace_bytes(ld) bytes, 256-byte aligned, owned by the
 * caller.  Y and the workspace must not overlap the inputs or each other (MONARCH_ERR_ALIAS).
 * Other conventions as monarch_fwd. */
MONARCH_API int monarch_linear_fwd(const void* X, const void* R, const void* L, const void* bias,
                                   const monarch_linear_dims* ld, void* Y, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Backward of monarch_linear_fwd for the upstream gradient dY (rows, out_features): dX (rows,
 * in_features), dR, dL (factor shapes), dbias (out_features, the column sums of dY; only when
 * has_bias), all overwritten.  Same workspace and overlap rules as monarch_linear_fwd. */
MONARCH_API int monarch_linear_bwd(const void* dY, const void* X, const void* R, const void* L,
                                   const monarch_linear_dims* ld, void* dX, void* dR, void* dL,
                                   void* dbias, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- DYAD
 * DYAD abstract (mlsanity summary): a weight that is the sum of two matrices, each permutable
 * to a block-sparse counterpart and stored as a 3-D tensor.  The abstract fixes no
 * permutation; this library takes the reshape-transpose of the Monarch pages on both sides of
 * the second term:
 *   y = BD(W1) x + P_out^T BD(W2) P_in x,
 *   (P_in x)[i*nb + k] = x[k*in_blk + i],   (P_out^T v)[k*out_blk + a] = v[a*nb + k],
 * with W1, W2 of shape (nblocks, out_blk, in_blk), X (rows, nblocks*in_blk), Y (rows,
 * nblocks*out_blk), and BD(W) the block-diagonal product on contiguous slices. */
typedef struct {
  int64_t rows;
  int32_t nblocks, in_blk, out_blk;
  int32_t dtype;          /* monarch_dtype of every tensor argument */
} monarch_dyad_dims;

/* Workspace bytes monarch_dyad_fwd / _bwd need (0 if dd is bad).  Host-only. */
MONARCH_API size_t monarch_dyad_workspace_bytes(const monarch_dyad_dims* dd);
/* 1 = tcgen05 path (bf16, packable blocks, multiples of 8), 0 = generic FMA kernels, -1 = bad
 * dims.  Host-only. */
MONARCH_API int monarch_dyad_path(const monarch_dyad_dims* dd);
/* Y = DYAD(X).  Caller-owned device memory; the workspace (>= monarch_dyad_workspace_bytes,
 * 256-byte aligned) may be NULL when that size is the 256-byte minimum of the generic path.
 * Outputs and workspace must not overlap the inputs or one another (MONARCH_ERR_ALIAS). */
MONARCH_API int monarch_dyad_fwd(const void* X, const void* W1, const void* W2, const monarch_dyad_dims* dd,
                                 void* Y, void* workspace, size_t workspace_bytes, void* stream);
/* (dX, dW1, dW2) of Y = DYAD(X) for the upstream gradient dY (chain rule), all overwritten;
 * weight gradients are summed over rows in a fixed order.  Same rules as monarch_dyad_fwd. */
MONARCH_API int monarch_dyad_bwd(const void* dY, const void* X, const void* W1, const void* W2,
                                 const monarch_dyad_dims* dd, void* dX, void* dW1, void* dW2,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------- lattice (hypercube) Monarch
 * Scatterbrain thread, the unofficial-implementation comment: a row viewed as a lattice with
 * naxes dimensions (row-major, last axis contiguous), one round of per-line matrices per
 * dimension (for width 12288 = 16 x 24 x 32: 768 matrices of 16 x 16, 512 of 24 x 24, 384 of
 * 32 x 32).  Readings taken: rounds run from the last axis to the first; round t maps axis t
 * from n_in[t] to n_out[t]; its weights W[t] have shape (lines_t, n_out[t], n_in[t]), line
 * index = row-major position in the other axes at that point (axes already done count with
 * their new lengths; monarch_lattice_weight_elems gives the element count); the output is the
 * final lattice in row-major order.  Two axes give the two-factor product with the output
 * transpose (W[1] = R, W[0] = L). */
typedef struct {
  int64_t rows;
  int32_t naxes;          /* 1 .. 4 */
  int32_t n_in[4], n_out[4];
  int32_t dtype;          /* monarch_dtype of every tensor argument */
} monarch_lattice_dims;

MONARCH_API size_t monarch_lattice_workspace_bytes(const monarch_lattice_dims* ld);
/* 1 = tcgen05 path (bf16, packable lines, lengths multiples of 8), 0 = generic FMA kernels. */
MONARCH_API int monarch_lattice_path(const monarch_lattice_dims* ld);
/* Elements of W[axis] (lines * n_out[axis] * n_in[axis]), -1 on bad arguments.  Host-only. */
MONARCH_API int64_t monarch_lattice_weight_elems(const monarch_lattice_dims* ld, int32_t axis);
/* Y (rows, prod n_out) = rounds of W over X (rows, prod n_in).  W: host array of naxes device
 * pointers (W[t] for axis t).  workspace: >= monarch_lattice_workspace_bytes(ld), 256-byte
 * aligned.  Same conventions as monarch_fwd. */
MONARCH_API int monarch_lattice_fwd(const void* X, const void* const* W, const monarch_lattice_dims* ld, void* Y,
                                    void* workspace, size_t workspace_bytes, void* stream);
/* (dX, dW[t]) for the upstream gradient dY; dW: host array of naxes device pointers; all
 * outputs overwritten, weight gradients summed over rows in a fixed order. */
MONARCH_API int monarch_lattice_bwd(const void* dY, const void* X, const void* const* W,
                                    const monarch_lattice_dims* ld, void* dX, void* const* dW, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* Number of kernels this library has launched in this process (every device and
 * stream), counted on the host at each successful launch.  Host-only; a caller
 * reads it before and after a region to count that region's launches. */
MONARCH_API uint64_t monarch_kernel_launches(void);

/* Which kernel family monarch_fwd / monarch_bwd would run for this shape:
 * 0 = generic FMA kernels, 1 = tcgen05 fused kernel over (128-row tile, block
 * group) units, 2 = tcgen05 fused kernel over 64-row tiles with the whole middle
 * vector on chip, 3 = the same with the second block-diagonal stage computed in
 * rounds of 8 output columns (transposed outputs wider than the middle vector,
 * e.g. 768 -> 3072), 4 = for square 64 x 64 blocks with nb1 = nb2 (e.g. n = 4096):
 * two tcgen05 block-diagonal GEMM passes and two row-permutation passes over Y (Y
 * doubles as the middle vector's storage; no scratch).  For the backward: 0 = generic FMA
 * kernels, 1 = tensor-core row-tile kernels (or block-GEMM passes for 64 x 64 blocks) for dX
 * and the middle vector, 2 = tcgen05 GEMM passes for shapes whose permutation moves whole
 * 64-column groups (e.g. nblocks = 4, 1024 -> 4096), 3 = packed block-diagonal tcgen05 GEMM
 * passes (g small blocks as one zero-filled block-diagonal tile) with row-transpose passes for
 * the permutations (e.g. 768 -> 3072); every tensor-core family computes the weight
 * gradients as tcgen05 GEMMs over the rows.  Host-only. */
MONARCH_API int monarch_fwd_path(const monarch_dims* d);
MONARCH_API int monarch_bwd_path(const monarch_dims* d);

#ifdef __cplusplus
}
#endif

#endif /* MONARCH_H_ */
