"""GPU parity of the lattice (hypercube) Monarch (monarch_lattice_fwd / _bwd) against the oracle.

Exact element-by-element comparison on sparse-sign inputs (X, dY in {-1, 0, 1}; two +-1 draws
per weight row, so every round at most doubles magnitudes and everything stays a small
integer, exact in bf16 and fp32).  Cases: the comment's 12288 = 16 x 24 x 32 lattice, two-axis
lattices (which must also equal the two-factor library forward), four axes, and uneven rounds.
"""
import numpy as np
import pytest
import torch

import block_diagonal_linear_b200 as bdl
import oracle
from block_diagonal_linear_b200 import synthetic

pytestmark = pytest.mark.gpu

CASES = [  # (n_in, n_out, dtype, rows, expected path)
    ([16, 24, 32], [16, 24, 32], "bf16", 100, 1),
    ([32, 32], [32, 32], "bf16", 300, 1),
    ([16, 16, 16], [16, 16, 16], "bf16", 129, 1),
    ([8, 8, 8, 8], [8, 8, 8, 8], "bf16", 64, 1),
    ([16, 32], [64, 16], "bf16", 200, 1),
    ([2, 2, 3], [3, 1, 2], "f32", 33, 0),
    ([4, 6, 5], [5, 6, 4], "bf16", 33, 0),
]


def _inputs(n_in, n_out, rows, seed):
    rng = np.random.default_rng(seed)
    Ws = [synthetic.sparse_sign_blocks(rng, *s, 2) for s in oracle.lattice_shapes(n_in, n_out)]
    X = rng.choice([-1.0, 0.0, 0.0, 1.0], size=(rows, int(np.prod(n_in))))
    dY = rng.choice([-1.0, 0.0, 0.0, 1.0], size=(rows, int(np.prod(n_out))))
    return Ws, X, dY


def _dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(torch.bfloat16 if dtype == "bf16" else torch.float32).cuda()


def _eq(got, ref, what):
    g = got.double().cpu().numpy()
    t = torch.from_numpy(np.ascontiguousarray(ref))
    assert torch.equal(t.to(torch.bfloat16).double(), t), "%s leaves the exact range" % what
    bad = np.argwhere(g != ref)
    assert bad.size == 0, "%s: %d entries differ, first at %s: %r vs %r" % (
        what, len(bad), tuple(bad[0]), g[tuple(bad[0])], ref[tuple(bad[0])])


@pytest.mark.parametrize("n_in,n_out,dtype,rows,path", CASES)
def test_lattice_forward_exact(n_in, n_out, dtype, rows, path):
    assert bdl.lattice_path(n_in, n_out, dtype) == path
    assert bdl.lattice_weight_shapes(n_in, n_out) == oracle.lattice_shapes(n_in, n_out)
    Ws, X, _ = _inputs(n_in, n_out, rows, 61)
    Y = bdl.lattice_fwd(_dev(X, dtype), [_dev(w, dtype) for w in Ws], n_in, n_out)
    assert bdl.last_device_status() == 0
    _eq(Y, oracle.lattice_forward(n_in, n_out, Ws, X), "Y")


@pytest.mark.parametrize("n_in,n_out,dtype,rows,path", CASES)
def test_lattice_backward_exact(n_in, n_out, dtype, rows, path):
    Ws, X, dY = _inputs(n_in, n_out, rows, 62)
    dX, dWs = bdl.lattice_bwd(_dev(dY, dtype), _dev(X, dtype), [_dev(w, dtype) for w in Ws], n_in, n_out)
    assert bdl.last_device_status() == 0
    rX, rWs = oracle.lattice_backward(n_in, n_out, Ws, X, dY)
    _eq(dX, rX, "dX")
    for t, (g, r) in enumerate(zip(dWs, rWs)):
        _eq(g, r, "dW[%d]" % t)


def test_two_axes_equal_the_two_factor_forward():
    n = [32, 32]
    Ws, X, _ = _inputs(n, n, 256, 63)
    shape = dict(nb1=32, in1=32, out1=32, nb2=32, in2=32, out2=32, out_transpose=1)
    Yl = bdl.lattice_fwd(_dev(X, "bf16"), [_dev(w, "bf16") for w in Ws], n, n)
    Ym = bdl.fwd(_dev(X, "bf16"), _dev(Ws[1], "bf16"), _dev(Ws[0], "bf16"), shape)
    assert torch.equal(Yl, Ym)
