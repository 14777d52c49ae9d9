"""fp64 CPU oracle for the Monarch product and its backward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``, never by the product package.
It shares no code with the CUDA path; the two meet only through the seeded
input generator (``block_diagonal_linear_b200.synthetic``), which holds no
arithmetic of the method.

The arithmetic lives in ``monarch_oracle.c`` (plain loops in ``double``);
this module compiles it with gcc on first use and calls it through ctypes.
Every function takes and returns float64 numpy arrays.

Sources (web pages on Monarch matrices): the Monarch abstract (product of two
block-diagonal matrices), the scatterbrain "Definition C.3" issue (M = L R up to
permutations; R has b blocks, L has n/b), the MonarchLinear factor shapes
(nblocks, out_blk, in_blk), the unofficial-implementation comment (permutation
[x0, x2, x1, x3] for N=4, lattice view) and the workload descriptions
(reshape, transpose, flatten). Every function is pinned by tests in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "monarch_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int64),
        ("nb1", ctypes.c_int),
        ("in1", ctypes.c_int),
        ("out1", ctypes.c_int),
        ("nb2", ctypes.c_int),
        ("in2", ctypes.c_int),
        ("out2", ctypes.c_int),
        ("out_transpose", ctypes.c_int),
    ]


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-shared", "-fPIC", "-pthread", _SRC, "-o", tmp]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.mo_forward.argtypes = [ctypes.POINTER(_Dims), dp, dp, dp, dp, ctypes.c_int]
        lib.mo_backward.argtypes = [ctypes.POINTER(_Dims), dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.mo_materialise.argtypes = [ctypes.POINTER(_Dims), dp, dp, dp]
        for f in (lib.mo_forward, lib.mo_backward, lib.mo_materialise):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _dims(d: dict, rows: int) -> _Dims:
    return _Dims(
        int(rows), d["nb1"], d["in1"], d["out1"], d["nb2"], d["in2"], d["out2"],
        int(d.get("out_transpose", 1)),
    )


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def sizes(d: dict) -> tuple[int, int, int]:
    """(n_in, n_mid, n_out) of a Monarch shape."""
    return d["nb1"] * d["in1"], d["nb1"] * d["out1"], d["nb2"] * d["out2"]


def forward(d: dict, X, R, L, nthreads: int | None = None) -> np.ndarray:
    """Y = X M^T, row by row (steps a1..a5), in fp64."""
    X, R, L = _f64(X), _f64(R), _f64(L)
    n_in, _, n_out = sizes(d)
    X2 = X.reshape(-1, n_in)
    Y = np.zeros((X2.shape[0], n_out), dtype=np.float64)
    rc = _load().mo_forward(
        ctypes.byref(_dims(d, X2.shape[0])), _p(X2), _p(R), _p(L), _p(Y),
        nthreads or default_threads(),
    )
    if rc != 0:
        raise ValueError("oracle: bad Monarch dims %r" % (d,))
    return Y


def backward(d: dict, dY, X, R, L, nthreads: int | None = None):
    """(dX, dR, dL) by the chain rule (steps a6..a10), Z recomputed, in fp64."""
    dY, X, R, L = _f64(dY), _f64(X), _f64(R), _f64(L)
    n_in, _, n_out = sizes(d)
    X2 = X.reshape(-1, n_in)
    dY2 = dY.reshape(-1, n_out)
    dX = np.zeros_like(X2)
    dR = np.zeros((d["nb1"], d["out1"], d["in1"]), dtype=np.float64)
    dL = np.zeros((d["nb2"], d["out2"], d["in2"]), dtype=np.float64)
    rc = _load().mo_backward(
        ctypes.byref(_dims(d, X2.shape[0])), _p(dY2), _p(X2), _p(R), _p(L), _p(dX), _p(dR),
        _p(dL), nthreads or default_threads(),
    )
    if rc != 0:
        raise ValueError("oracle: bad Monarch dims %r" % (d,))
    return dX, dR, dL


def materialise(d: dict, R, L) -> np.ndarray:
    """Dense M (n_out, n_in), Y = X M^T, from the closed form of the product."""
    R, L = _f64(R), _f64(L)
    n_in, _, n_out = sizes(d)
    M = np.zeros((n_out, n_in), dtype=np.float64)
    rc = _load().mo_materialise(ctypes.byref(_dims(d, 0)), _p(R), _p(L), _p(M))
    if rc != 0:
        raise ValueError("oracle: bad Monarch dims %r" % (d,))
    return M


def param_count(d: dict) -> int:
    return d["nb1"] * d["out1"] * d["in1"] + d["nb2"] * d["out2"] * d["in2"]


def normwise_rel_err(got, ref) -> float:
    """||got - ref||_F / ||ref||_F in fp64 (0 when both are zero)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.linalg.norm(ref.ravel()))
    num = float(np.linalg.norm((got - ref).ravel()))
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den


# ---------------------------------------------------------------- MonarchLinear front end
# Scatterbrain issue thread, the MonarchLinear __init__ listing: block sizes are the ceilings
# in_blksz = ceil(in / nblocks) and out_blksz = ceil(out / nblocks); the features are extended
# to in_blksz * nblocks and out_blksz * nblocks; when the extended input is narrower than the
# extended output, blkdiag1 is (nblocks, in_blksz, in_blksz) and blkdiag2 (nblocks, out_blksz,
# in_blksz), otherwise blkdiag1 is (nblocks, out_blksz, in_blksz) and blkdiag2 (nblocks,
# out_blksz, out_blksz).  The listing shows no forward; the reading taken here: x is
# zero-padded to the extended width, multiplied as in the nblocks workload (blkdiag1 on
# contiguous slices, transpose, blkdiag2, flatten), the result is cut to out_features, and an
# optional bias is added.

def linear_shape(in_features: int, out_features: int, nblocks: int) -> dict:
    """Monarch shape of MonarchLinear(in_features, out_features, nblocks)."""
    in_blk = -(-in_features // nblocks)
    out_blk = -(-out_features // nblocks)
    mid = in_blk if in_blk * nblocks < out_blk * nblocks else out_blk
    return dict(nb1=nblocks, in1=in_blk, out1=mid, nb2=nblocks, in2=mid, out2=out_blk, out_transpose=0)


def linear_forward(in_features: int, out_features: int, nblocks: int, X, R, L, bias=None,
                   nthreads: int | None = None) -> np.ndarray:
    """y = (M x_padded)[:out_features] + bias for every row x, in fp64."""
    d = linear_shape(in_features, out_features, nblocks)
    X = _f64(X).reshape(-1, in_features)
    n_in, _, _ = sizes(d)
    Xp = np.zeros((X.shape[0], n_in))
    Xp[:, :in_features] = X
    Y = forward(d, Xp, R, L, nthreads)[:, :out_features]
    if bias is not None:
        Y = Y + _f64(bias)[None, :]
    return np.ascontiguousarray(Y)


def linear_backward(in_features: int, out_features: int, nblocks: int, dY, X, R, L,
                    nthreads: int | None = None):
    """(dX, dR, dL, dbias) of linear_forward: the padded output columns get no gradient, the
    padded input columns' gradient is dropped, dbias sums dY over the rows."""
    d = linear_shape(in_features, out_features, nblocks)
    X = _f64(X).reshape(-1, in_features)
    dY = _f64(dY).reshape(-1, out_features)
    n_in, _, n_out = sizes(d)
    Xp = np.zeros((X.shape[0], n_in))
    Xp[:, :in_features] = X
    dYp = np.zeros((dY.shape[0], n_out))
    dYp[:, :out_features] = dY
    dXp, dR, dL = backward(d, dYp, Xp, R, L, nthreads)
    return np.ascontiguousarray(dXp[:, :in_features]), dR, dL, dY.sum(axis=0)


# ---------------------------------------------------------------- dense -> Monarch projection
# Monarch abstract: projecting a dense matrix onto the Monarch set "has an analytical optimal
# solution"; the scatterbrain projection question slices the dense matrix with
# rearrange(M, '(p k) (r s) -> k r p s').  For the lattice shapes (in2 == nb1, nb2 == out1,
# output transpose) every entry of M is one product, M[o*nb2 + j][k*in1 + i] = L[j][o][k] *
# R[k][j][i], so the (j, k) slice A_jk[o][i] = M[o*nb2 + j][k*in1 + i] is the rank-1 matrix
# L[j][:, k] R[k][j][:]^T and the slices cover M without overlap.  The Frobenius-nearest
# Monarch matrix is therefore the best rank-1 approximation of every slice (Eckart-Young):
# A_jk ~ s u v^T, L[j][:, k] = sqrt(s) u, R[k][j][:] = sqrt(s) v.  Sign convention (the
# factors are unique up to a common sign flip): the entry of v largest in magnitude (first
# one on ties) is made positive.

def projection_supported(d: dict) -> bool:
    return d["in2"] == d["nb1"] and d["nb2"] == d["out1"] and int(d.get("out_transpose", 1)) == 1


def project(d: dict, M) -> tuple[np.ndarray, np.ndarray]:
    """(R, L) of the Monarch matrix nearest to the dense M (n_out x n_in) in Frobenius norm."""
    if not projection_supported(d):
        raise ValueError("projection needs a lattice shape (in2 == nb1, nb2 == out1, out_transpose)")
    M = _f64(M)
    nb1, in1, nb2, out2 = d["nb1"], d["in1"], d["nb2"], d["out2"]
    R = np.zeros((nb1, d["out1"], in1))
    L = np.zeros((nb2, out2, d["in2"]))
    for j in range(nb2):
        for k in range(nb1):
            A = M[j::nb2, k * in1:(k + 1) * in1]          # rows o*nb2 + j, columns k*in1 + i
            U, S, Vt = np.linalg.svd(A, full_matrices=False)
            u, s, v = U[:, 0], S[0], Vt[0]
            t = int(np.argmax(np.abs(v)))
            if v[t] < 0:
                u, v = -u, -v
            L[j, :, k] = np.sqrt(s) * u
            R[k, j, :] = np.sqrt(s) * v
    return R, L


# ---------------------------------------------------------------- DYAD
# DYAD abstract (mlsanity summary): the weight is a sum of two matrices, each permutable to a
# block-sparse counterpart and stored as a 3-D tensor.  The abstract fixes no permutation;
# the reading taken here uses the reshape-transpose of the Monarch pages on both sides of the
# second term:
#   y = BD(W1) x + P_out^T BD(W2) P_in x,
#   (P_in x)[i*nb + k] = x[k*in_blk + i]          (view (nb, in_blk), transpose, flatten)
#   (P_out^T v)[k*out_blk + a] = v[a*nb + k]      (the inverse transpose on the output side)
# with W1, W2 of shape (nb, out_blk, in_blk) and BD the block-diagonal product on contiguous
# slices: (BD(W) x)[b*out_blk + o] = sum_i W[b][o][i] x[b*in_blk + i].

def _bd(W, x):
    nb, ob, ib = W.shape
    out = np.empty((x.shape[0], nb * ob))
    for b in range(nb):
        out[:, b * ob:(b + 1) * ob] = x[:, b * ib:(b + 1) * ib] @ W[b].T
    return out


def dyad_forward(W1, W2, X) -> np.ndarray:
    """y = BD(W1) x + P_out^T BD(W2) P_in x for every row x, in fp64 (steps in that order)."""
    W1, W2, X = _f64(W1), _f64(W2), _f64(X)
    nb, ob, ib = W1.shape
    X = X.reshape(-1, nb * ib)
    y1 = _bd(W1, X)
    Px = np.empty_like(X)
    for k in range(nb):
        for i in range(ib):
            Px[:, i * nb + k] = X[:, k * ib + i]
    v = _bd(W2, Px)
    y2 = np.empty_like(v)
    for k in range(nb):
        for a in range(ob):
            y2[:, k * ob + a] = v[:, a * nb + k]
    return y1 + y2


def dyad_backward(W1, W2, X, dY):
    """(dX, dW1, dW2) of dyad_forward by the chain rule, in fp64."""
    W1, W2, X, dY = _f64(W1), _f64(W2), _f64(X), _f64(dY)
    nb, ob, ib = W1.shape
    X = X.reshape(-1, nb * ib)
    dY = dY.reshape(-1, nb * ob)
    Px = np.empty_like(X)
    for k in range(nb):
        for i in range(ib):
            Px[:, i * nb + k] = X[:, k * ib + i]
    dv = np.empty_like(dY)                      # gradient of v: inverse of the output transpose
    for k in range(nb):
        for a in range(ob):
            dv[:, a * nb + k] = dY[:, k * ob + a]
    dW1 = np.stack([dY[:, b * ob:(b + 1) * ob].T @ X[:, b * ib:(b + 1) * ib] for b in range(nb)])
    dW2 = np.stack([dv[:, b * ob:(b + 1) * ob].T @ Px[:, b * ib:(b + 1) * ib] for b in range(nb)])
    dX = _bd(np.transpose(W1, (0, 2, 1)), dY)
    dPx = _bd(np.transpose(W2, (0, 2, 1)), dv)
    for k in range(nb):
        for i in range(ib):
            dX[:, k * ib + i] += dPx[:, i * nb + k]
    return dX, dW1, dW2


# ---------------------------------------------------------------- lattice (hypercube) Monarch
# Scatterbrain thread, the unofficial-implementation comment: view the n inputs as a lattice
# (for n = N the 2-D m x m square; for width 12288 the 3-D lattice [16, 24, 32]); one round per
# dimension applies a separate matrix to every line of the lattice along that dimension
# (768 matrices of 16 x 16 for the first dimension, 512 of 24 x 24 for the second, 384 for the
# third).  Readings taken: a row x is the lattice in row-major order (last axis contiguous);
# the rounds run from the last axis to the first, so that with two axes the map is the
# two-factor product with the output transpose (R on the contiguous rows of the square, L on
# its columns); a round may change the length of its axis (n_t -> m_t, the "uneven rectangle"
# of the same comment); the matrices of round t are indexed by the row-major position of the
# line in the other axes at that point (axes already done count with their new lengths); the
# output is the final lattice in row-major order.

def lattice_shapes(n_in: list, n_out: list) -> list:
    """Weight shapes (lines, m_t, n_t) of every round t (index t = axis)."""
    d = len(n_in)
    shapes = [None] * d
    cur = list(n_in)
    for t in range(d - 1, -1, -1):
        lines = int(np.prod([cur[s] for s in range(d) if s != t]))
        shapes[t] = (lines, n_out[t], n_in[t])
        cur[t] = n_out[t]
    return shapes


def lattice_forward(n_in: list, n_out: list, Ws: list, X) -> np.ndarray:
    """Rounds t = d-1 .. 0 over the lattice of every row, in fp64 (plain loops over lines)."""
    d = len(n_in)
    X = _f64(X)
    rows = X.shape[0]
    cur = list(n_in)
    A = X.reshape([rows] + cur)
    for t in range(d - 1, -1, -1):
        W = _f64(Ws[t])
        others = [s for s in range(d) if s != t]
        # move axis t last, lines in row-major order of the other axes
        At = np.moveaxis(A, 1 + t, -1).reshape(rows, -1, cur[t])
        Bt = np.empty((rows, At.shape[1], n_out[t]))
        for line in range(At.shape[1]):
            Bt[:, line, :] = At[:, line, :] @ W[line].T
        shape_o = [rows] + [cur[s] for s in others] + [n_out[t]]
        A = np.moveaxis(Bt.reshape(shape_o), -1, 1 + t)
        cur[t] = n_out[t]
    return np.ascontiguousarray(A.reshape(rows, -1))


def lattice_backward(n_in: list, n_out: list, Ws: list, X, dY):
    """(dX, [dW_t]) of lattice_forward by the chain rule (inputs of every round recomputed)."""
    d = len(n_in)
    X, dY = _f64(X), _f64(dY)
    rows = X.shape[0]
    cur = list(n_in)
    A = X.reshape([rows] + cur)
    saved = {}
    for t in range(d - 1, -1, -1):                     # forward, keeping each round's input
        W = _f64(Ws[t])
        others = [s for s in range(d) if s != t]
        At = np.moveaxis(A, 1 + t, -1).reshape(rows, -1, cur[t])
        saved[t] = (At, list(cur))
        Bt = np.einsum("rli,loi->rlo", At, W)
        A = np.moveaxis(Bt.reshape([rows] + [cur[s] for s in others] + [n_out[t]]), -1, 1 + t)
        cur[t] = n_out[t]
    G = dY.reshape([rows] + cur)
    dWs = [None] * d
    for t in range(d):                                  # backward, rounds in reverse order
        W = _f64(Ws[t])
        At, cin = saved[t]
        others = [s for s in range(d) if s != t]
        Gt = np.moveaxis(G, 1 + t, -1).reshape(rows, -1, n_out[t])
        dWs[t] = np.einsum("rlo,rli->loi", Gt, At)
        dAt = np.einsum("rlo,loi->rli", Gt, W)
        G = np.moveaxis(dAt.reshape([rows] + [cin[s] for s in others] + [cin[t]]), -1, 1 + t)
    return np.ascontiguousarray(G.reshape(rows, -1)), dWs
