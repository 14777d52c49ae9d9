"""Pins for the MonarchLinear front end of the oracle, and the library's host-side shape rule.

The factor shapes come from the MonarchLinear __init__ listing of the scatterbrain issue
thread (ceil block sizes, extended features, the in < out rule); the expected shapes below
are worked out by hand from that listing.  The forward and backward are pinned against the
dense matrix of the closed form (oracle.materialise) cropped to the real features, and
against torch autograd of the padded product written with torch operations.
"""
import numpy as np
import pytest
import torch

import block_diagonal_linear_b200 as bdl
import oracle
from test_oracle_pins import _torch_forward

# (in, out, nblocks) -> (R shape, L shape), by hand from the listing
LISTING = [
    ((1024, 4096, 4), ((4, 256, 256), (4, 1024, 256))),   # in_ext 1024 < out_ext 4096
    ((4096, 1024, 4), ((4, 256, 1024), (4, 256, 256))),   # in_ext >= out_ext
    ((1000, 512, 16), ((16, 32, 63), (16, 32, 32))),      # in_blksz = ceil(62.5) = 63
    ((10000, 1024, 4), ((4, 256, 2500), (4, 256, 256))),  # the MLP table's 10000 x 1024 layer
    ((1024, 512, 16), ((16, 32, 64), (16, 32, 32))),
    ((10, 30, 4), ((4, 3, 3), (4, 8, 3))),                # in_ext 12 < out_ext 32
    ((7, 7, 3), ((3, 3, 3), (3, 3, 3))),                  # equal extended widths: the else branch
]


def _factors(shape, rng):
    R = rng.standard_normal((shape["nb1"], shape["out1"], shape["in1"]))
    L = rng.standard_normal((shape["nb2"], shape["out2"], shape["in2"]))
    return R, L


@pytest.mark.parametrize("args,shapes", LISTING)
def test_factor_shapes_follow_the_listing(args, shapes):
    d = oracle.linear_shape(*args)
    assert (d["nb1"], d["out1"], d["in1"]) == shapes[0]
    assert (d["nb2"], d["out2"], d["in2"]) == shapes[1]
    assert d["out_transpose"] == 0
    assert bdl.linear_shape(*args) == d  # the library's host-side rule agrees


@pytest.mark.parametrize("args", [a for a, _ in LISTING if a[0] * a[1] <= 2 ** 22])
@pytest.mark.parametrize("with_bias", [False, True])
def test_forward_is_cropped_dense_product_plus_bias(args, with_bias):
    in_f, out_f, nb = args
    d = oracle.linear_shape(*args)
    rng = np.random.default_rng(5)
    R, L = _factors(d, rng)
    X = rng.standard_normal((9, in_f))
    b = rng.standard_normal(out_f) if with_bias else None
    M = oracle.materialise(d, R, L)[:out_f, :in_f]   # padded inputs contribute nothing
    ref = X @ M.T + (b if with_bias else 0.0)
    np.testing.assert_allclose(oracle.linear_forward(in_f, out_f, nb, X, R, L, b), ref, rtol=1e-12, atol=1e-11)


def test_exact_sizes_without_bias_is_the_plain_product():
    d = oracle.linear_shape(1024, 4096, 4)
    rng = np.random.default_rng(6)
    R, L = _factors(d, rng)
    X = rng.standard_normal((5, 1024))
    assert np.array_equal(oracle.linear_forward(1024, 4096, 4, X, R, L), oracle.forward(d, X, R, L))


@pytest.mark.parametrize("args", [(10, 30, 4), (7, 7, 3), (1000, 512, 16), (30, 10, 4)])
def test_backward_matches_autograd_of_padded_product(args):
    in_f, out_f, nb = args
    d = oracle.linear_shape(*args)
    n_in, _, n_out = oracle.sizes(d)
    rng = np.random.default_rng(7)
    R, L = _factors(d, rng)
    X = rng.standard_normal((11, in_f))
    b = rng.standard_normal(out_f)
    dY = rng.standard_normal((11, out_f))
    tX, tR, tL, tb = (torch.tensor(a, requires_grad=True) for a in (X, R, L, b))
    Xp = torch.nn.functional.pad(tX, (0, n_in - in_f))
    Y = _torch_forward(d, Xp, tR, tL)[:, :out_f] + tb
    (Y * torch.tensor(dY)).sum().backward()
    dX, dR, dL, db = oracle.linear_backward(in_f, out_f, nb, dY, X, R, L)
    for got, ref in ((dX, tX.grad), (dR, tR.grad), (dL, tL.grad), (db, tb.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=1e-10, atol=1e-10)


def test_bad_linear_dims_rejected_by_the_library():
    import ctypes
    d = bdl.MonarchDims()
    for args in ((0, 8, 2), (8, 0, 2), (8, 8, 0), (-1, 8, 2)):
        ld = bdl.linear_dims(*args, rows=4)
        assert bdl.lib().monarch_linear_shape(ctypes.byref(ld), ctypes.byref(d)) == bdl.CODES["MONARCH_ERR_DIMS"]
    ld = bdl.linear_dims(8, 8, 2, rows=4, dtype=7)
    assert bdl.lib().monarch_linear_shape(ctypes.byref(ld), ctypes.byref(d)) == bdl.CODES["MONARCH_ERR_DTYPE"]
    assert bdl.linear_workspace_bytes(0, 8, 2, 4) == 0
