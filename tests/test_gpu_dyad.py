"""GPU parity of DYAD (monarch_dyad_fwd / _bwd) against the fp64 oracle.

Exact element-by-element comparison on sparse-sign inputs (X, dY in {-1, 0, 1}; two +-1
draws per weight row), where every intermediate and result is a small integer and therefore
exact in bf16 and fp32; plus a normwise check on random values at a larger size.
"""
import numpy as np
import pytest
import torch

import block_diagonal_linear_b200 as bdl
import oracle
from block_diagonal_linear_b200 import synthetic

pytestmark = pytest.mark.gpu

CASES = [  # (nb, in_blk, out_blk, dtype, rows, expected path)
    (8, 128, 512, "bf16", 300, 1),
    (32, 32, 32, "bf16", 257, 1),
    (8, 64, 64, "bf16", 129, 1),
    (4, 256, 1024, "bf16", 77, 0),
    (3, 5, 7, "bf16", 50, 0),
    (3, 5, 7, "f32", 50, 0),
]


def _inputs(nb, ib, ob, rows, seed):
    rng = np.random.default_rng(seed)
    W1 = synthetic.sparse_sign_blocks(rng, nb, ob, ib, 2)
    W2 = synthetic.sparse_sign_blocks(rng, nb, ob, ib, 2)
    X = rng.choice([-1.0, 0.0, 0.0, 1.0], size=(rows, nb * ib))
    dY = rng.choice([-1.0, 0.0, 0.0, 1.0], size=(rows, nb * ob))
    return X, W1, W2, dY


def _dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(torch.bfloat16 if dtype == "bf16" else torch.float32).cuda()


def _eq(got, ref, what):
    g = got.double().cpu().numpy()
    t = torch.from_numpy(ref)
    assert torch.equal(t.to(torch.bfloat16).double(), t), "%s leaves the exact range" % what
    bad = np.argwhere(g != ref)
    assert bad.size == 0, "%s: %d entries differ, first at %s: %r vs %r" % (
        what, len(bad), tuple(bad[0]), g[tuple(bad[0])], ref[tuple(bad[0])])


@pytest.mark.parametrize("nb,ib,ob,dtype,rows,path", CASES)
def test_dyad_forward_exact(nb, ib, ob, dtype, rows, path):
    assert bdl.dyad_path(nb, ib, ob, dtype) == path
    X, W1, W2, _ = _inputs(nb, ib, ob, rows, 51)
    Y = bdl.dyad_fwd(_dev(X, dtype), _dev(W1, dtype), _dev(W2, dtype))
    assert bdl.last_device_status() == 0
    _eq(Y, oracle.dyad_forward(W1, W2, X), "Y")


@pytest.mark.parametrize("nb,ib,ob,dtype,rows,path", CASES)
def test_dyad_backward_exact(nb, ib, ob, dtype, rows, path):
    X, W1, W2, dY = _inputs(nb, ib, ob, rows, 52)
    got = bdl.dyad_bwd(_dev(dY, dtype), _dev(X, dtype), _dev(W1, dtype), _dev(W2, dtype))
    assert bdl.last_device_status() == 0
    for g, r, what in zip(got, oracle.dyad_backward(W1, W2, X, dY), ("dX", "dW1", "dW2")):
        _eq(g, r, what)


def test_dyad_random_values_within_tolerance():
    nb, ib, ob, rows = 8, 128, 512, 4096
    rng = np.random.default_rng(53)
    W1 = synthetic.Tensor(rng.uniform(-1, 1, (nb, ob, ib)) / np.sqrt(ib), "bf16").f64
    W2 = synthetic.Tensor(rng.uniform(-1, 1, (nb, ob, ib)) / np.sqrt(ib), "bf16").f64
    X = synthetic.Tensor(rng.standard_normal((rows, nb * ib)), "bf16").f64
    dY = synthetic.Tensor(rng.standard_normal((rows, nb * ob)), "bf16").f64
    Y = bdl.dyad_fwd(_dev(X, "bf16"), _dev(W1, "bf16"), _dev(W2, "bf16"))
    assert oracle.normwise_rel_err(Y.double().cpu().numpy(), oracle.dyad_forward(W1, W2, X)) <= 2e-2
    got = bdl.dyad_bwd(_dev(dY, "bf16"), _dev(X, "bf16"), _dev(W1, "bf16"), _dev(W2, "bf16"))
    for g, r in zip(got, oracle.dyad_backward(W1, W2, X, dY)):
        assert oracle.normwise_rel_err(g.double().cpu().numpy(), r) <= 2e-2
