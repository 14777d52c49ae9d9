"""Pins for the fp64 oracle against facts the pages and the mathematics fix.

None of these re-types the oracle's own loops: each check comes from a
different statement of the method (the worked permutation example, the lattice
view, the workload wording as reshape/transpose steps, textbook special cases,
closed-form and brute-force construction of M, automatic differentiation and
finite differences for the backward).
"""
import json
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from block_diagonal_linear_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

SMALL_SHAPES = [
    # square m x m lattices
    dict(nb1=2, in1=2, out1=2, nb2=2, in2=2, out2=2, out_transpose=1),
    dict(nb1=3, in1=3, out1=3, nb2=3, in2=3, out2=3, out_transpose=1),
    dict(nb1=4, in1=4, out1=4, nb2=4, in2=4, out2=4, out_transpose=1),
    # rectangular, the regroup j = t div in2 straddles R blocks
    dict(nb1=2, in1=3, out1=3, nb2=3, in2=2, out2=4, out_transpose=1),
    dict(nb1=3, in1=2, out1=4, nb2=2, in2=6, out2=5, out_transpose=1),
    dict(nb1=3, in1=2, out1=4, nb2=2, in2=6, out2=5, out_transpose=0),
    # nblocks-style two-factor shapes (L keeps the block count, no output transpose)
    dict(nb1=2, in1=4, out1=4, nb2=2, in2=4, out2=8, out_transpose=0),
    dict(nb1=4, in1=3, out1=2, nb2=2, in2=4, out2=3, out_transpose=0),
]


def rand(shape, rng):
    return rng.standard_normal(shape)


def rand_factors(d, rng):
    return rand((d["nb1"], d["out1"], d["in1"]), rng), rand((d["nb2"], d["out2"], d["in2"]), rng)


def eye_blocks(nb, n):
    return np.stack([np.eye(n) for _ in range(nb)])


# ---------------------------------------------------------------- permutation
def test_permutation_worked_example_n4():
    """scatterbrain thread, unofficial-implementation comment: for N=4 (M=2) the
    permutation layer maps x to [x0, x2, x1, x3]."""
    g = json.load(open(os.path.join(GOLDEN, "permutation_n4.json")))
    d = dict(nb1=2, in1=2, out1=2, nb2=2, in2=2, out2=2, out_transpose=0)
    x = np.array([g["x"]], dtype=np.float64)
    # R = I and L = I, no output transpose: y is exactly the permuted input P x.
    y = oracle.forward(d, x, eye_blocks(2, 2), eye_blocks(2, 2))
    assert y[0].tolist() == g["permuted"]
    # With the output transpose the permutation is undone: M = P^T I P I = I.
    d1 = dict(d, out_transpose=1)
    y1 = oracle.forward(d1, x, eye_blocks(2, 2), eye_blocks(2, 2))
    assert y1[0].tolist() == g["x"]


def test_permutation_block_groups_n4():
    """Same comment: one batched product acts on the contiguous groups
    [x0,x1],[x2,x3] (R, the lattice rows) and the other on the strided groups
    [x0,x2],[x1,x3] (L, the lattice columns)."""
    g = json.load(open(os.path.join(GOLDEN, "permutation_n4.json")))
    d = dict(nb1=2, in1=2, out1=2, nb2=2, in2=2, out2=2, out_transpose=1)
    rng = np.random.default_rng(3)
    R, L = rand_factors(d, rng)
    # L = I: M = R acts only inside the contiguous groups.
    M_R = oracle.materialise(d, R, eye_blocks(2, 2))
    # R = I: M = P^T L P acts only inside the strided groups.
    M_L = oracle.materialise(d, eye_blocks(2, 2), L)
    for M, groups, blocks in ((M_R, g["contiguous_blocks"], R), (M_L, g["strided_blocks"], L)):
        mask = np.zeros((4, 4), dtype=bool)
        for b, grp in enumerate(groups):
            for a_i, a in enumerate(grp):
                for c_i, c in enumerate(grp):
                    mask[a, c] = True
                    assert M[a, c] == blocks[b][a_i, c_i]
        assert np.all(M[~mask] == 0.0)


# ---------------------------------------------------------------- forward
@pytest.mark.parametrize("m", [2, 3, 4, 5, 8])
def test_lattice_view_square(m):
    """Lattice view (same comment): reshape x to an m x m grid; R contracts along
    each row, L along each column; the grid is read back in place."""
    d = dict(nb1=m, in1=m, out1=m, nb2=m, in2=m, out2=m, out_transpose=1)
    rng = np.random.default_rng(m)
    R, L = rand_factors(d, rng)
    X = rand((7, m * m), rng)
    G = X.reshape(7, m, m)                       # G[b, row a, col c] = x[a*m + c]
    G1 = np.einsum("apc,bac->bap", R, G)         # row a of the grid, contracted by R[a]
    G2 = np.einsum("poa,bap->bop", L, G1)        # column p of the grid, contracted by L[p]
    Y_lattice = G2.reshape(7, m * m)
    np.testing.assert_allclose(oracle.forward(d, X, R, L), Y_lattice, rtol=1e-12, atol=1e-12)


def test_workload_text_768_to_3072():
    """Workload wording for the 768->3072 shape: x reshaped to (16,48); R gives
    (16,48), transposed to (48,16); L (48 blocks of 64x16) gives (48,64), which is
    transposed and flattened to 3072."""
    w = synthetic.WORKLOADS["r768x3072_bf16"]
    d = synthetic.shape_of(w)
    rng = np.random.default_rng(11)
    R, L = rand_factors(d, rng)
    X = rand((5, 768), rng)
    ys = []
    for x in X:
        u = np.stack([R[k] @ x.reshape(16, 48)[k] for k in range(16)])  # (16,48)
        z = u.T                                                         # (48,16)
        v = np.stack([L[j] @ z[j] for j in range(48)])                  # (48,64)
        ys.append(v.T.reshape(-1))                                      # 3072
    np.testing.assert_allclose(oracle.forward(d, X, R, L), np.array(ys), rtol=1e-12, atol=1e-12)


def test_workload_text_nblocks4():
    """Workload wording for the nblocks=4 layer: X is (B,4,256); blkdiag1 (4,256,256)
    gives (B,4,256), transposed to (B,256,4) and reshaped to (B,4,256); blkdiag2
    (4,1024,256) gives (B,4,1024), flattened to 4096."""
    w = synthetic.WORKLOADS["nblk4_1024x4096_bf16"]
    d = synthetic.shape_of(w)
    rng = np.random.default_rng(12)
    R, L = rand_factors(d, rng)
    X = rand((3, 1024), rng)
    X3 = X.reshape(3, 4, 256)
    U = np.einsum("kpi,bki->bkp", R, X3)                  # (B,4,256)
    Z = np.transpose(U, (0, 2, 1)).reshape(3, 4, 256)     # (B,256,4) -> (B,4,256)
    V = np.einsum("joq,bjq->bjo", L, Z)                   # (B,4,1024)
    np.testing.assert_allclose(oracle.forward(d, X, R, L), V.reshape(3, 4096),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("m", [2, 4, 16])
def test_L_identity_is_block_diagonal(m):
    """L = I leaves a single block-diagonal R (the blockdiag_linear special case)."""
    d = dict(nb1=m, in1=m, out1=m, nb2=m, in2=m, out2=m, out_transpose=1)
    rng = np.random.default_rng(20 + m)
    R, _ = rand_factors(d, rng)
    X = rand((6, m * m), rng)
    B = scipy.linalg.block_diag(*R)
    np.testing.assert_allclose(oracle.forward(d, X, R, eye_blocks(m, m)), X @ B.T,
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n_in,n_mid,n_out", [(5, 7, 3), (16, 16, 16), (8, 3, 11)])
def test_one_block_is_dense_product(n_in, n_mid, n_out):
    """With one block per factor the permutations are trivial and M = L R."""
    for ot in (0, 1):
        d = dict(nb1=1, in1=n_in, out1=n_mid, nb2=1, in2=n_mid, out2=n_out, out_transpose=ot)
        rng = np.random.default_rng(n_in * 100 + n_out)
        R, L = rand_factors(d, rng)
        X = rand((4, n_in), rng)
        M = L[0] @ R[0]
        np.testing.assert_allclose(oracle.forward(d, X, R, L), X @ M.T, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(oracle.materialise(d, R, L), M, rtol=1e-12, atol=1e-12)
        # and with L = I, M = R
        if n_mid == n_out:
            np.testing.assert_array_equal(oracle.materialise(d, R, eye_blocks(1, n_mid)), R[0])


@pytest.mark.parametrize("d", SMALL_SHAPES)
def test_brute_force_unit_vectors_equal_closed_form(d):
    """Build M column by column from forward(e_i) and compare it, exactly, with the
    closed form (integer entries: every fp64 sum is exact)."""
    rng = np.random.default_rng(5)
    n_in, _, n_out = oracle.sizes(d)
    R = rng.integers(-4, 5, size=(d["nb1"], d["out1"], d["in1"])).astype(np.float64)
    L = rng.integers(-4, 5, size=(d["nb2"], d["out2"], d["in2"])).astype(np.float64)
    MT = oracle.forward(d, np.eye(n_in), R, L)  # row i = forward(e_i) = column i of M
    np.testing.assert_array_equal(MT.T, oracle.materialise(d, R, L))
    # and a random integer X through the dense product, exactly
    X = rng.integers(-4, 5, size=(9, n_in)).astype(np.float64)
    np.testing.assert_array_equal(oracle.forward(d, X, R, L), X @ MT)


def test_closed_form_square_entries():
    """Square Monarch: every entry of M is a single product,
    M[o*m + j, k*m + i] = L[j][o][k] * R[k][j][i]."""
    m = 5
    d = dict(nb1=m, in1=m, out1=m, nb2=m, in2=m, out2=m, out_transpose=1)
    rng = np.random.default_rng(9)
    R, L = rand_factors(d, rng)
    M = oracle.materialise(d, R, L)
    for o in range(m):
        for j in range(m):
            for k in range(m):
                for i in range(m):
                    assert M[o * m + j, k * m + i] == L[j, o, k] * R[k, j, i]


@pytest.mark.parametrize("name", ["n256_fp32", "n1024_bf16", "n4096_bf16"])
def test_param_count_square(name):
    """Square n = m^2: two factors of m blocks of m x m each, 2 n sqrt(n) parameters."""
    d = synthetic.WORKLOADS[name]
    n = d["nb1"] * d["in1"]
    assert oracle.param_count(d) == 2 * n * int(round(np.sqrt(n)))


# ---------------------------------------------------------------- backward
def _torch_forward(d, X, R, L):
    """The workload wording as torch reshape/transpose ops (for autograd only)."""
    B = X.shape[0]
    U = torch.einsum("kpi,bki->bkp", R, X.reshape(B, d["nb1"], d["in1"]))
    Z = U.transpose(1, 2).reshape(B, d["nb2"], d["in2"])
    V = torch.einsum("joq,bjq->bjo", L, Z)
    return (V.transpose(1, 2) if d["out_transpose"] else V).reshape(B, -1)


@pytest.mark.parametrize("d", SMALL_SHAPES + [synthetic.shape_of(synthetic.WORKLOADS["n256_fp32"])])
def test_backward_matches_autograd(d):
    """dX, dR, dL equal fp64 automatic differentiation of sum(Y * dY)."""
    rng = np.random.default_rng(17)
    n_in, _, n_out = oracle.sizes(d)
    R, L = rand_factors(d, rng)
    X = rand((13, n_in), rng)
    dY = rand((13, n_out), rng)
    tX, tR, tL = (torch.tensor(a, requires_grad=True) for a in (X, R, L))
    (_torch_forward(d, tX, tR, tL) * torch.tensor(dY)).sum().backward()
    dX, dR, dL = oracle.backward(d, dY, X, R, L)
    for got, ref in ((dX, tX.grad), (dR, tR.grad), (dL, tL.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("d", SMALL_SHAPES)
def test_backward_dense_chain_rule_and_adjoint(d):
    """dX = dY M (dense), and <dY, X M^T> = <dX, X> (adjoint identity)."""
    rng = np.random.default_rng(23)
    n_in, _, n_out = oracle.sizes(d)
    R, L = rand_factors(d, rng)
    X = rand((8, n_in), rng)
    dY = rand((8, n_out), rng)
    M = oracle.materialise(d, R, L)
    dX, _, _ = oracle.backward(d, dY, X, R, L)
    np.testing.assert_allclose(dX, dY @ M, rtol=1e-11, atol=1e-11)
    Y = oracle.forward(d, X, R, L)
    assert abs(np.sum(dY * Y) - np.sum(dX * X)) <= 1e-10 * (1 + abs(np.sum(dY * Y)))


@pytest.mark.parametrize("d", SMALL_SHAPES[:6])
def test_backward_finite_differences(d):
    """Central differences of f = sum(Y * dY) in every entry of R and L."""
    rng = np.random.default_rng(29)
    n_in, _, n_out = oracle.sizes(d)
    R, L = rand_factors(d, rng)
    X = rand((4, n_in), rng)
    dY = rand((4, n_out), rng)
    _, dR, dL = oracle.backward(d, dY, X, R, L)
    h = 1e-4

    def f(R_, L_):
        return float(np.sum(oracle.forward(d, X, R_, L_) * dY))

    fd_R = np.zeros_like(R)
    for idx in np.ndindex(R.shape):
        Rp, Rm = R.copy(), R.copy()
        Rp[idx] += h
        Rm[idx] -= h
        fd_R[idx] = (f(Rp, L) - f(Rm, L)) / (2 * h)
    fd_L = np.zeros_like(L)
    for idx in np.ndindex(L.shape):
        Lp, Lm = L.copy(), L.copy()
        Lp[idx] += h
        Lm[idx] -= h
        fd_L[idx] = (f(R, Lp) - f(R, Lm)) / (2 * h)
    assert oracle.normwise_rel_err(dR, fd_R) < 1e-8
    assert oracle.normwise_rel_err(dL, fd_L) < 1e-8


def test_backward_exact_integers_and_linearity():
    """Integer inputs: the backward is exact; dR does not depend on the scale of R
    (f is linear in R), and dL does not depend on the scale of L."""
    d = dict(nb1=3, in1=2, out1=4, nb2=2, in2=6, out2=5, out_transpose=1)
    w = dict(d, rows=11)
    a = synthetic.make_integer_inputs(w, seed=2)
    dX, dR, dL = oracle.backward(d, a["dY"], a["X"], a["R"], a["L"])
    tX, tR, tL = (torch.tensor(a[k], requires_grad=True) for k in ("X", "R", "L"))
    (_torch_forward(d, tX, tR, tL) * torch.tensor(a["dY"])).sum().backward()
    np.testing.assert_array_equal(dX, tX.grad.numpy())
    np.testing.assert_array_equal(dR, tR.grad.numpy())
    np.testing.assert_array_equal(dL, tL.grad.numpy())
    _, dR3, _ = oracle.backward(d, a["dY"], a["X"], 3 * a["R"], a["L"])
    np.testing.assert_array_equal(dR3, dR)
    _, _, dL3 = oracle.backward(d, a["dY"], a["X"], a["R"], 3 * a["L"])
    np.testing.assert_array_equal(dL3, dL)


def test_thread_count_does_not_change_results():
    d = dict(nb1=4, in1=8, out1=8, nb2=4, in2=8, out2=8, out_transpose=1)
    rng = np.random.default_rng(31)
    R, L = rand_factors(d, rng)
    X = rand((37, 32), rng)
    dY = rand((37, 32), rng)
    a = oracle.backward(d, dY, X, R, L, nthreads=1)
    b = oracle.backward(d, dY, X, R, L, nthreads=5)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_allclose(a[1], b[1], rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(oracle.forward(d, X, R, L, nthreads=1),
                                  oracle.forward(d, X, R, L, nthreads=4))


def test_bad_dims_rejected():
    with pytest.raises(ValueError):
        oracle.forward(dict(nb1=2, in1=2, out1=3, nb2=2, in2=2, out2=2, out_transpose=1),
                       np.zeros((1, 4)), np.zeros((2, 3, 2)), np.zeros((2, 2, 2)))


# ---------------------------------------------------------------- inputs
def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = (rng.standard_normal(10000) * np.exp(rng.uniform(-20, 20, 10000))).astype(np.float32)
    bits = synthetic.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, ref)


def test_synthetic_recipe_is_seeded():
    w = synthetic.WORKLOADS["n256_fp32"]
    a = synthetic.make_inputs(w, seed=4)
    b = synthetic.make_inputs(w, seed=4)
    for k in ("X", "R", "L", "dY"):
        np.testing.assert_array_equal(a[k].f64, b[k].f64)
    assert a["R"].shape == (16, 16, 16)
    assert np.max(np.abs(a["R"].f64)) <= 0.25
