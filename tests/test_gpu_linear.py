"""GPU parity of the MonarchLinear front end (monarch_linear_fwd / _bwd) against the oracle.

Exact element-by-element comparison on sparse-sign inputs (as in test_gpu_exact.py: every
intermediate and result is a small integer, exact in bf16 and fp32), with a bias in
{-1, 0, 1}.  The cases cover the listing's two shape branches, padded inputs and outputs,
and the kernel families the padded Monarch shape lands on.
"""
import numpy as np
import pytest
import torch

import block_diagonal_linear_b200 as bdl
import oracle
from block_diagonal_linear_b200 import synthetic

pytestmark = pytest.mark.gpu

CASES = [  # (in, out, nblocks, dtype, rows, bias)
    (1024, 4096, 4, "bf16", 300, True),     # the nblocks = 4 workload shape: tensor-core families
    (4096, 1024, 4, "bf16", 257, False),    # in_ext >= out_ext branch; GEMM backward
    (1000, 512, 16, "bf16", 300, True),     # padded input (1000 -> 1008)
    (1000, 500, 16, "bf16", 129, True),     # padded input and output
    (10, 30, 4, "f32", 77, True),
    (30, 10, 4, "f32", 5, False),
]


def _dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(torch.bfloat16 if dtype == "bf16" else torch.float32).cuda()


def _exact_bf16(a):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return bool(torch.equal(t.to(torch.bfloat16).double(), t))


def _inputs(in_f, out_f, nb, rows, seed):
    d = oracle.linear_shape(in_f, out_f, nb)
    w = dict(d, rows=rows)
    inp = synthetic.make_sparse_sign_inputs(w, seed=seed)
    n_in, _, n_out = oracle.sizes(d)
    rng = np.random.default_rng(seed + 1)
    return (inp["X"][:, :in_f].copy(), inp["R"], inp["L"], inp["dY"][:, :out_f].copy(),
            rng.choice([-1.0, 0.0, 1.0], size=out_f))


def _assert_equal(got, ref, what):
    g = got.double().cpu().numpy()
    bad = np.argwhere(g != ref)
    assert bad.size == 0, "%s: %d entries differ, first at %s: %r vs %r" % (
        what, len(bad), tuple(bad[0]), g[tuple(bad[0])], ref[tuple(bad[0])])


@pytest.mark.parametrize("in_f,out_f,nb,dtype,rows,bias", CASES)
def test_linear_forward_exact(in_f, out_f, nb, dtype, rows, bias):
    X, R, L, _, b = _inputs(in_f, out_f, nb, rows, seed=31)
    ref = oracle.linear_forward(in_f, out_f, nb, X, R, L, b if bias else None)
    assert _exact_bf16(ref)
    Y = bdl.linear_fwd(_dev(X, dtype), _dev(R, dtype), _dev(L, dtype), in_f, out_f, nb,
                       bias=_dev(b, dtype) if bias else None)
    assert bdl.last_device_status() == 0
    _assert_equal(Y, ref, "Y")


@pytest.mark.parametrize("in_f,out_f,nb,dtype,rows,bias", CASES)
def test_linear_backward_exact(in_f, out_f, nb, dtype, rows, bias):
    X, R, L, dY, _ = _inputs(in_f, out_f, nb, rows, seed=32)
    refs = oracle.linear_backward(in_f, out_f, nb, dY, X, R, L)
    for r in refs:
        assert _exact_bf16(r)
    got = bdl.linear_bwd(_dev(dY, dtype), _dev(X, dtype), _dev(R, dtype), _dev(L, dtype), in_f, out_f, nb,
                         bias=bias)
    assert bdl.last_device_status() == 0
    for g, r, what in zip(got, refs, ("dX", "dR", "dL", "dbias")):
        if g is None:
            assert not bias and what == "dbias"
            continue
        _assert_equal(g, r, what)


def test_linear_random_values_within_tolerance():
    """Random N(0,1) / U(+-1/sqrt(fan_in)) inputs at a padded bf16 size, normwise 2e-2."""
    in_f, out_f, nb, rows = 1000, 4000, 4, 512
    d = oracle.linear_shape(in_f, out_f, nb)
    inp = synthetic.make_inputs(dict(d, rows=rows, dtype="bf16"), seed=33)
    X = inp["X"].f64[:, :in_f]
    b = synthetic.Tensor(np.random.default_rng(34).uniform(-1, 1, out_f), "bf16").f64
    ref = oracle.linear_forward(in_f, out_f, nb, X, inp["R"].f64, inp["L"].f64, b)
    Y = bdl.linear_fwd(_dev(X, "bf16"), _dev(inp["R"].f64, "bf16"), _dev(inp["L"].f64, "bf16"), in_f, out_f, nb,
                       bias=_dev(b, "bf16"))
    assert oracle.normwise_rel_err(Y.double().cpu().numpy(), ref) <= 2e-2
