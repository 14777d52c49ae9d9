"""Pins for the dense -> Monarch projection of the oracle.

The slicing is the one the projection question prints, rearrange(M, '(p k) (r s) -> k r p s'),
written here with torch (einops is not used by the oracle).  Pins: a Monarch matrix projects
onto itself (exact recovery); the projection is Frobenius-optimal against random Monarch
competitors and against perturbations of its own factors; the error equals the energy left
outside the leading singular value of every slice; the listing's slicing of the dense matrix
has rank-1 slices for a Monarch matrix.
"""
import numpy as np
import pytest
import torch

import oracle

SHAPES = [
    dict(nb1=4, in1=4, out1=4, nb2=4, in2=4, out2=4, out_transpose=1),
    dict(nb1=3, in1=5, out1=2, nb2=2, in2=3, out2=6, out_transpose=1),   # rectangular lattice
    dict(nb1=8, in1=8, out1=8, nb2=8, in2=8, out2=8, out_transpose=1),
]


def _rand_factors(d, rng):
    return (rng.standard_normal((d["nb1"], d["out1"], d["in1"])),
            rng.standard_normal((d["nb2"], d["out2"], d["in2"])))


def _slices(M, d):
    """'(p k) (r s) -> k r p s' with k = nb2 (row minor), r = nb1 (column major)."""
    t = torch.tensor(M)
    n_out, n_in = t.shape
    k, r = d["nb2"], d["nb1"]
    return t.reshape(n_out // k, k, r, n_in // r).permute(1, 2, 0, 3).numpy()


@pytest.mark.parametrize("d", SHAPES)
def test_slices_of_a_monarch_matrix_are_rank_one(d):
    rng = np.random.default_rng(1)
    R, L = _rand_factors(d, rng)
    T = _slices(oracle.materialise(d, R, L), d)
    for j in range(d["nb2"]):
        for k in range(d["nb1"]):
            s = np.linalg.svd(T[j, k], compute_uv=False)
            assert s[1:].max(initial=0.0) <= 1e-10 * s[0]


@pytest.mark.parametrize("d", SHAPES)
def test_monarch_matrix_projects_onto_itself(d):
    rng = np.random.default_rng(2)
    R, L = _rand_factors(d, rng)
    M = oracle.materialise(d, R, L)
    Rp, Lp = oracle.project(d, M)
    np.testing.assert_allclose(oracle.materialise(d, Rp, Lp), M, rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("d", SHAPES)
def test_projection_error_is_the_energy_outside_each_leading_singular_value(d):
    rng = np.random.default_rng(3)
    n_in, _, n_out = oracle.sizes(d)
    M = rng.standard_normal((n_out, n_in))
    Rp, Lp = oracle.project(d, M)
    err2 = np.sum((oracle.materialise(d, Rp, Lp) - M) ** 2)
    T = _slices(M, d)
    tail = sum(float(np.sum(np.linalg.svd(T[j, k], compute_uv=False)[1:] ** 2))
               for j in range(d["nb2"]) for k in range(d["nb1"]))
    assert err2 == pytest.approx(tail, rel=1e-9)


@pytest.mark.parametrize("d", SHAPES)
def test_projection_beats_other_monarch_matrices(d):
    rng = np.random.default_rng(4)
    n_in, _, n_out = oracle.sizes(d)
    M = rng.standard_normal((n_out, n_in))
    Rp, Lp = oracle.project(d, M)
    best = np.linalg.norm(oracle.materialise(d, Rp, Lp) - M)
    for _ in range(20):
        R, L = _rand_factors(d, rng)
        assert np.linalg.norm(oracle.materialise(d, R, L) - M) > best
        e = 1e-3
        Rq, Lq = Rp + e * rng.standard_normal(Rp.shape), Lp + e * rng.standard_normal(Lp.shape)
        assert np.linalg.norm(oracle.materialise(d, Rq, Lq) - M) >= best - 1e-12


def test_sign_convention_and_rejected_shapes():
    d = SHAPES[0]
    rng = np.random.default_rng(5)
    M = rng.standard_normal((16, 16))
    Rp, _ = oracle.project(d, M)
    for k in range(4):
        for j in range(4):
            v = Rp[k, j]
            assert v[int(np.argmax(np.abs(v)))] > 0
    with pytest.raises(ValueError):
        oracle.project(dict(nb1=4, in1=256, out1=256, nb2=4, in2=256, out2=1024, out_transpose=0),
                       np.zeros((4096, 1024)))
