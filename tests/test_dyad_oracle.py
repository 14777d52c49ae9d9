"""Pins for the DYAD oracle (DYAD abstract: a sum of two matrices, each permutable to a
block-sparse counterpart, stored as 3-D tensors; cost rows x cols / #blocks).

Pins that do not re-type the oracle's loops: the first term alone is scipy's block_diag;
for square blocks (nb = in_blk = out_blk) the second term alone is the Monarch product with
R = I (the Monarch oracle, the reshape-transpose of the pages on both sides); the whole map
equals a dense matrix built from explicit permutation matrices; the parameter count is
2 * rows * cols / nb; the backward matches torch autograd.
"""
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle

SHAPES = [(4, 4, 4), (4, 6, 3), (2, 3, 5), (8, 8, 8), (3, 1, 2)]  # (nb, out_blk, in_blk)


def _w(shape, rng):
    return rng.standard_normal(shape)


def _perm_in(nb, ib):
    """P_in as a matrix: (P x)[i*nb + k] = x[k*ib + i]."""
    P = np.zeros((nb * ib, nb * ib))
    for k in range(nb):
        for i in range(ib):
            P[i * nb + k, k * ib + i] = 1.0
    return P


@pytest.mark.parametrize("nb,ob,ib", SHAPES)
def test_first_term_is_block_diagonal(nb, ob, ib):
    rng = np.random.default_rng(1)
    W1 = _w((nb, ob, ib), rng)
    X = rng.standard_normal((7, nb * ib))
    ref = X @ scipy.linalg.block_diag(*W1).T
    np.testing.assert_allclose(oracle.dyad_forward(W1, np.zeros_like(W1), X), ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("m", [2, 4, 8])
def test_second_term_is_monarch_with_identity_R_for_square_blocks(m):
    rng = np.random.default_rng(2)
    W2 = _w((m, m, m), rng)
    X = rng.standard_normal((5, m * m))
    d = dict(nb1=m, in1=m, out1=m, nb2=m, in2=m, out2=m, out_transpose=1)
    ref = oracle.forward(d, X, np.stack([np.eye(m)] * m), W2)
    np.testing.assert_allclose(oracle.dyad_forward(np.zeros_like(W2), W2, X), ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("nb,ob,ib", SHAPES)
def test_dense_matrix_from_permutation_matrices(nb, ob, ib):
    rng = np.random.default_rng(3)
    W1, W2 = _w((nb, ob, ib), rng), _w((nb, ob, ib), rng)
    Pin, Pout = _perm_in(nb, ib), _perm_in(nb, ob)   # P_out has the same form on the output side
    W = scipy.linalg.block_diag(*W1) + Pout.T @ scipy.linalg.block_diag(*W2) @ Pin
    X = rng.standard_normal((6, nb * ib))
    np.testing.assert_allclose(oracle.dyad_forward(W1, W2, X), X @ W.T, rtol=1e-12, atol=1e-11)
    assert 2 * W1.size == 2 * (nb * ob) * (nb * ib) // nb   # parameters: rows x cols / #blocks, twice


@pytest.mark.parametrize("nb,ob,ib", SHAPES)
def test_backward_matches_autograd(nb, ob, ib):
    rng = np.random.default_rng(4)
    W1, W2 = _w((nb, ob, ib), rng), _w((nb, ob, ib), rng)
    X = rng.standard_normal((9, nb * ib))
    dY = rng.standard_normal((9, nb * ob))
    Pin, Pout = (torch.tensor(_perm_in(nb, ib)), torch.tensor(_perm_in(nb, ob)))
    tW1, tW2, tX = (torch.tensor(a, requires_grad=True) for a in (W1, W2, X))
    W = torch.block_diag(*tW1) + Pout.T @ torch.block_diag(*tW2) @ Pin
    ((tX @ W.T) * torch.tensor(dY)).sum().backward()
    dX, dW1, dW2 = oracle.dyad_backward(W1, W2, X, dY)
    for got, ref in ((dX, tX.grad), (dW1, tW1.grad), (dW2, tW2.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=1e-10, atol=1e-10)
