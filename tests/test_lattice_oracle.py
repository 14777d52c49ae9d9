"""Pins for the lattice (hypercube) Monarch oracle.

Pins: the round counts and sizes of the comment's [16, 24, 32] example (768, 512, 384 lines);
with two axes the map equals the two-factor Monarch oracle (square and the 768 -> 3072
rectangle); the dense matrix has one product per entry (closed form over the path of one
lattice point through the rounds), checked entry by entry on small lattices; a round of
identity matrices reduces three axes to independent two-axis problems; the backward matches
torch autograd.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle


def _weights(n_in, n_out, rng):
    return [rng.standard_normal(s) for s in oracle.lattice_shapes(n_in, n_out)]


def test_rounds_of_the_width_12288_example():
    shapes = oracle.lattice_shapes([16, 24, 32], [16, 24, 32])
    assert shapes[0] == (768, 16, 16)
    assert shapes[1] == (512, 24, 24)
    assert shapes[2] == (384, 32, 32)


@pytest.mark.parametrize("d", [
    dict(nb1=4, in1=4, out1=4, nb2=4, in2=4, out2=4, out_transpose=1),
    dict(nb1=16, in1=48, out1=48, nb2=48, in2=16, out2=64, out_transpose=1),
    dict(nb1=3, in1=5, out1=2, nb2=2, in2=3, out2=6, out_transpose=1),
])
def test_two_axes_is_the_two_factor_product(d):
    rng = np.random.default_rng(1)
    R = rng.standard_normal((d["nb1"], d["out1"], d["in1"]))
    L = rng.standard_normal((d["nb2"], d["out2"], d["in2"]))
    X = rng.standard_normal((6, d["nb1"] * d["in1"]))
    # axis 0 (length nb1) -> out2, axis 1 (length in1) -> out1: R is round 1, L is round 0
    Y = oracle.lattice_forward([d["nb1"], d["in1"]], [d["out2"], d["out1"]], [L, R], X)
    np.testing.assert_allclose(Y, oracle.forward(d, X, R, L), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n_in,n_out", [([2, 3, 2], [2, 3, 2]), ([2, 2, 3], [3, 1, 2]), ([3, 2], [2, 4])])
def test_dense_entries_are_single_products(n_in, n_out):
    """M[b][a] = prod over rounds t = d-1..0 of W_t[line][b_t][a_t], where the line index uses
    b for axes already done and a for the others (integer weights: exact)."""
    d = len(n_in)
    rng = np.random.default_rng(2)
    Ws = [rng.integers(-3, 4, size=s).astype(np.float64) for s in oracle.lattice_shapes(n_in, n_out)]
    N_in, N_out = int(np.prod(n_in)), int(np.prod(n_out))
    M = oracle.lattice_forward(n_in, n_out, Ws, np.eye(N_in)).T          # (N_out, N_in)
    for b in itertools.product(*[range(m) for m in n_out]):
        for a in itertools.product(*[range(n) for n in n_in]):
            val = 1.0
            for t in range(d - 1, -1, -1):
                pos = [b[s] if s > t else a[s] for s in range(d)]
                dims = [n_out[s] if s > t else n_in[s] for s in range(d)]
                line = 0
                for s in range(d):
                    if s != t:
                        line = line * dims[s] + pos[s]
                val *= Ws[t][line, b[t], a[t]]
            assert M[np.ravel_multi_index(b, n_out), np.ravel_multi_index(a, n_in)] == val


def test_identity_round_splits_into_two_axis_problems():
    rng = np.random.default_rng(3)
    n = [3, 4, 2]
    Ws = _weights(n, n, rng)
    Ws[0] = np.stack([np.eye(3)] * Ws[0].shape[0])      # the last round (axis 0) does nothing
    X = rng.standard_normal((5, 24))
    Y = oracle.lattice_forward(n, n, Ws, X).reshape(5, 3, 4, 2)
    Xl = X.reshape(5, 3, 4, 2)
    for a0 in range(3):   # per slice a0: rounds over axes 2 then 1 with that slice's matrices
        W2 = Ws[2].reshape(3, 4, 2, 2)[a0]               # lines (a0, a1) -> (4, 2, 2)
        W1 = Ws[1].reshape(3, 2, 4, 4)[a0]               # lines (a0, b2) -> (2, 4, 4)
        ref = oracle.lattice_forward([4, 2], [4, 2], [W1, W2], Xl[:, a0].reshape(5, 8))
        np.testing.assert_allclose(Y[:, a0].reshape(5, 8), ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n_in,n_out", [([2, 3, 2], [2, 3, 2]), ([2, 2, 3], [3, 1, 2]), ([3, 2], [2, 4]),
                                        ([2, 2, 2, 2], [2, 3, 2, 1])])
def test_backward_matches_autograd(n_in, n_out):
    rng = np.random.default_rng(4)
    Ws = _weights(n_in, n_out, rng)
    rows = 5
    X = rng.standard_normal((rows, int(np.prod(n_in))))
    dY = rng.standard_normal((rows, int(np.prod(n_out))))
    tW = [torch.tensor(w, requires_grad=True) for w in Ws]
    tX = torch.tensor(X, requires_grad=True)
    d = len(n_in)
    A = tX.reshape([rows] + list(n_in))
    cur = list(n_in)
    for t in range(d - 1, -1, -1):
        others = [s for s in range(d) if s != t]
        At = torch.movedim(A, 1 + t, -1).reshape(rows, -1, cur[t])
        Bt = torch.einsum("rli,loi->rlo", At, tW[t])
        A = torch.movedim(Bt.reshape([rows] + [cur[s] for s in others] + [n_out[t]]), -1, 1 + t)
        cur[t] = n_out[t]
    (A.reshape(rows, -1) * torch.tensor(dY)).sum().backward()
    dX, dWs = oracle.lattice_backward(n_in, n_out, Ws, X, dY)
    np.testing.assert_allclose(dX, tX.grad.numpy(), rtol=1e-10, atol=1e-10)
    for g, t in zip(dWs, tW):
        np.testing.assert_allclose(g, t.grad.numpy(), rtol=1e-10, atol=1e-10)
