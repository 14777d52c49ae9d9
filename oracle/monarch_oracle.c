/*
 * Monarch oracle: a plain, slow, obviously correct fp64 CPU implementation of
 * the Monarch product Y = X * M^T with M = P_out * L * P * R, and of its
 * training backward (dX, dR, dL).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may include, link or
 * call this file: only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg use it. It shares no code, header or constant with the CUDA
 * kernels.
 *
 * Sources followed (web pages on Monarch matrices):
 *  - "Monarch: Expressive Structured Matrices for Efficient and Accurate
 *    Training", abstract: M is a product of two block-diagonal matrices with
 *    permutations.
 *  - scatterbrain issue thread, "Definition C.3": M = L R up to a permutation of
 *    rows and columns; R block diagonal with b blocks, L with n/b blocks.
 *  - scatterbrain issue thread, MonarchLinear __init__: factors stored as
 *    (nblocks, out_blk, in_blk) tensors (nn.Linear weight convention).
 *  - scatterbrain issue thread, unofficial implementation: the permutation for
 *    N=4 is x_new = [x0, x2, x1, x3]; viewed as a square lattice, one batched
 *    product runs over the rows and the other over the columns.
 *  - The workload descriptions: "x reshaped to (nb1, in1)", the R result
 *    "transposed", L applied, then "transposed and flattened" (or only
 *    "flattened" when there is no output transpose).
 *
 * Notation (per row x of X):
 *   a1  X3[k][i]   = x[k*in1 + i]                         k < nb1, i < in1
 *   a2  u[k][p]    = sum_i R[k][p][i] * X3[k][i]          p < out1
 *   a3  flat[p*nb1 + k] = u[k][p]   (transpose (nb1,out1) -> (out1,nb1))
 *       Z[j][q]    = flat[j*in2 + q]                      j < nb2, q < in2
 *   a4  v[j][o]    = sum_q L[j][o][q] * Z[j][q]           o < out2
 *   a5  y[o*nb2 + j] = v[j][o]   if out_transpose, else y[j*out2 + o] = v[j][o]
 * Backward (chain rule, Z recomputed from X):
 *   a6  dV[j][o]   = dy[idx(j,o)]
 *   a7  dL[j][o][q] += dV[j][o] * Z[j][q]
 *   a8  dZ[j][q]   = sum_o L[j][o][q] * dV[j][o];  dU[k][p] = dZflat[p*nb1 + k]
 *   a9  dR[k][p][i] += dU[k][p] * X3[k][i]
 *   a10 dX3[k][i]  = sum_p R[k][p][i] * dU[k][p]
 * Materialise: M[idx(j,o)][k*in1 + i] =
 *   sum over p with (p*nb1 + k) div in2 == j of L[j][o][(p*nb1 + k) mod in2] * R[k][p][i]
 * (the closed form of the product, written independently of the row loops).
 *
 * Rows are split across pthreads; weight gradients use one fp64 partial per
 * thread, summed in thread order, so results do not depend on scheduling.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t rows;
    int nb1, in1, out1;
    int nb2, in2, out2;
    int out_transpose;
} mo_dims;

static int64_t mo_n_in(const mo_dims* d) { return (int64_t)d->nb1 * d->in1; }
static int64_t mo_n_mid(const mo_dims* d) { return (int64_t)d->nb1 * d->out1; }
static int64_t mo_n_out(const mo_dims* d) { return (int64_t)d->nb2 * d->out2; }

/* Position of v[j][o] in the output row (step a5). */
static int64_t mo_out_index(const mo_dims* d, int j, int o) {
    return d->out_transpose ? (int64_t)o * d->nb2 + j : (int64_t)j * d->out2 + o;
}

int mo_check_dims(const mo_dims* d) {
    if (d->rows < 0 || d->nb1 <= 0 || d->in1 <= 0 || d->out1 <= 0 || d->nb2 <= 0 ||
        d->in2 <= 0 || d->out2 <= 0)
        return -1;
    if ((int64_t)d->nb1 * d->out1 != (int64_t)d->nb2 * d->in2) return -1;
    return 0;
}

/* ---- one row, forward: steps a1..a5 ---- */
static void mo_row_forward(const mo_dims* d, const double* x, const double* R, const double* L,
                           double* flat, double* y) {
    /* a1 + a2 + a3: compute u[k][p] and place it at flat[p*nb1 + k] */
    for (int k = 0; k < d->nb1; ++k) {
        const double* xk = x + (int64_t)k * d->in1;
        for (int p = 0; p < d->out1; ++p) {
            const double* Rkp = R + ((int64_t)k * d->out1 + p) * d->in1;
            double s = 0.0;
            for (int i = 0; i < d->in1; ++i) s += Rkp[i] * xk[i];
            flat[(int64_t)p * d->nb1 + k] = s;
        }
    }
    /* a4 + a5: Z[j][q] = flat[j*in2 + q]; v[j][o] = sum_q L[j][o][q] Z[j][q] */
    for (int j = 0; j < d->nb2; ++j) {
        const double* Zj = flat + (int64_t)j * d->in2;
        for (int o = 0; o < d->out2; ++o) {
            const double* Ljo = L + ((int64_t)j * d->out2 + o) * d->in2;
            double s = 0.0;
            for (int q = 0; q < d->in2; ++q) s += Ljo[q] * Zj[q];
            y[mo_out_index(d, j, o)] = s;
        }
    }
}

/* ---- one row, backward: steps a6..a10, accumulating into dR / dL ---- */
static void mo_row_backward(const mo_dims* d, const double* dy, const double* x, const double* R,
                            const double* L, double* flat, double* dflat, double* dx, double* dR,
                            double* dL) {
    /* recompute Z (a1..a3) */
    for (int k = 0; k < d->nb1; ++k) {
        const double* xk = x + (int64_t)k * d->in1;
        for (int p = 0; p < d->out1; ++p) {
            const double* Rkp = R + ((int64_t)k * d->out1 + p) * d->in1;
            double s = 0.0;
            for (int i = 0; i < d->in1; ++i) s += Rkp[i] * xk[i];
            flat[(int64_t)p * d->nb1 + k] = s;
        }
    }
    /* a6, a7, a8: dV from dy; dL += dV Z^T; dZ = L^T dV */
    for (int j = 0; j < d->nb2; ++j) {
        const double* Zj = flat + (int64_t)j * d->in2;
        double* dZj = dflat + (int64_t)j * d->in2;
        for (int q = 0; q < d->in2; ++q) dZj[q] = 0.0;
        for (int o = 0; o < d->out2; ++o) {
            const double dv = dy[mo_out_index(d, j, o)];
            const double* Ljo = L + ((int64_t)j * d->out2 + o) * d->in2;
            double* dLjo = dL + ((int64_t)j * d->out2 + o) * d->in2;
            for (int q = 0; q < d->in2; ++q) {
                dLjo[q] += dv * Zj[q];
                dZj[q] += Ljo[q] * dv;
            }
        }
    }
    /* a8 (inverse permutation), a9, a10: dU[k][p] = dflat[p*nb1 + k] */
    for (int k = 0; k < d->nb1; ++k) {
        const double* xk = x + (int64_t)k * d->in1;
        double* dxk = dx + (int64_t)k * d->in1;
        for (int i = 0; i < d->in1; ++i) dxk[i] = 0.0;
        for (int p = 0; p < d->out1; ++p) {
            const double du = dflat[(int64_t)p * d->nb1 + k];
            const double* Rkp = R + ((int64_t)k * d->out1 + p) * d->in1;
            double* dRkp = dR + ((int64_t)k * d->out1 + p) * d->in1;
            for (int i = 0; i < d->in1; ++i) {
                dRkp[i] += du * xk[i];
                dxk[i] += Rkp[i] * du;
            }
        }
    }
}

/* ---- threading ---- */
typedef struct {
    const mo_dims* d;
    const double *X, *R, *L, *dY;
    double *Y, *dX, *dR, *dL;
    int64_t r0, r1;
    int backward;
} mo_job;

static void* mo_worker(void* arg) {
    mo_job* job = (mo_job*)arg;
    const mo_dims* d = job->d;
    const int64_t n_in = mo_n_in(d), n_mid = mo_n_mid(d), n_out = mo_n_out(d);
    double* flat = (double*)malloc(sizeof(double) * (size_t)n_mid);
    double* dflat = (double*)malloc(sizeof(double) * (size_t)n_mid);
    for (int64_t r = job->r0; r < job->r1; ++r) {
        if (!job->backward)
            mo_row_forward(d, job->X + r * n_in, job->R, job->L, flat, job->Y + r * n_out);
        else
            mo_row_backward(d, job->dY + r * n_out, job->X + r * n_in, job->R, job->L, flat, dflat,
                            job->dX + r * n_in, job->dR, job->dL);
    }
    free(flat);
    free(dflat);
    return NULL;
}

static int mo_run(const mo_dims* d, const double* X, const double* R, const double* L,
                  const double* dY, double* Y, double* dX, double* dR, double* dL, int backward,
                  int nthreads) {
    if (mo_check_dims(d)) return -1;
    if (nthreads < 1) nthreads = 1;
    if (d->rows < nthreads) nthreads = d->rows > 0 ? (int)d->rows : 1;
    const int64_t nR = (int64_t)d->nb1 * d->out1 * d->in1;
    const int64_t nL = (int64_t)d->nb2 * d->out2 * d->in2;
    mo_job* jobs = (mo_job*)calloc((size_t)nthreads, sizeof(mo_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    double* pR = NULL;
    double* pL = NULL;
    if (backward) {
        pR = (double*)calloc((size_t)(nR * nthreads), sizeof(double));
        pL = (double*)calloc((size_t)(nL * nthreads), sizeof(double));
    }
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].d = d;
        jobs[t].X = X; jobs[t].R = R; jobs[t].L = L; jobs[t].dY = dY;
        jobs[t].Y = Y; jobs[t].dX = dX;
        jobs[t].dR = backward ? pR + (int64_t)t * nR : NULL;
        jobs[t].dL = backward ? pL + (int64_t)t * nL : NULL;
        jobs[t].r0 = d->rows * t / nthreads;
        jobs[t].r1 = d->rows * (t + 1) / nthreads;
        jobs[t].backward = backward;
    }
    for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, mo_worker, &jobs[t]);
    mo_worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
    if (backward) {
        /* fixed-order sum of the per-thread partials */
        for (int64_t e = 0; e < nR; ++e) {
            double s = 0.0;
            for (int t = 0; t < nthreads; ++t) s += pR[(int64_t)t * nR + e];
            dR[e] = s;
        }
        for (int64_t e = 0; e < nL; ++e) {
            double s = 0.0;
            for (int t = 0; t < nthreads; ++t) s += pL[(int64_t)t * nL + e];
            dL[e] = s;
        }
        free(pR);
        free(pL);
    }
    free(jobs);
    free(th);
    return 0;
}

/* Y (rows, n_out) = forward of X (rows, n_in). */
int mo_forward(const mo_dims* d, const double* X, const double* R, const double* L, double* Y,
               int nthreads) {
    return mo_run(d, X, R, L, NULL, Y, NULL, NULL, NULL, 0, nthreads);
}

/* dX (rows, n_in), dR (nb1,out1,in1), dL (nb2,out2,in2) from dY (rows, n_out). */
int mo_backward(const mo_dims* d, const double* dY, const double* X, const double* R,
                const double* L, double* dX, double* dR, double* dL, int nthreads) {
    return mo_run(d, X, R, L, dY, NULL, dX, dR, dL, 1, nthreads);
}

/* Dense M (n_out, n_in) with Y = X M^T, from the closed form of the product. */
int mo_materialise(const mo_dims* d, const double* R, const double* L, double* M) {
    if (mo_check_dims(d)) return -1;
    const int64_t n_in = mo_n_in(d), n_out = mo_n_out(d);
    memset(M, 0, sizeof(double) * (size_t)(n_in * n_out));
    for (int k = 0; k < d->nb1; ++k)
        for (int p = 0; p < d->out1; ++p) {
            const int64_t t = (int64_t)p * d->nb1 + k; /* where u[k][p] lands */
            const int j = (int)(t / d->in2), q = (int)(t % d->in2);
            for (int o = 0; o < d->out2; ++o) {
                const double l = L[((int64_t)j * d->out2 + o) * d->in2 + q];
                double* Mrow = M + mo_out_index(d, j, o) * n_in + (int64_t)k * d->in1;
                const double* Rkp = R + ((int64_t)k * d->out1 + p) * d->in1;
                for (int i = 0; i < d->in1; ++i) Mrow[i] += l * Rkp[i];
            }
        }
    return 0;
}
