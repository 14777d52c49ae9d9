"""Exact element-by-element GPU parity, one case per kernel family, forward and backward.

Inputs come from ``synthetic.make_sparse_sign_inputs``: X and dY in {-1, 0, 1}, factor
blocks with two +-1 draws per row.  Every intermediate (u, Z, v; dV, dZ, dU) is then a
small integer, and so is every result; integers of magnitude <= 256 are exact in bf16 and
every partial sum is exact in fp32, so rounding the middle vector to bf16 on chip and
accumulating in any order changes nothing.  The CUDA path must therefore equal the fp64
oracle exactly, entry by entry (``==``), which a wrong column segment, a dropped K step
or a transposed operand cannot hide behind a normwise tolerance.  Each test first checks
from the drawn factors that the intermediates stay within that exact range, and from
the oracle that the results are representable in the storage dtype.
"""
import numpy as np
import pytest
import torch

import block_diagonal_linear_b200 as bdl
import oracle
from block_diagonal_linear_b200 import synthetic

pytestmark = pytest.mark.gpu
W = synthetic.WORKLOADS

SQ16 = dict(nb1=16, in1=16, out1=16, nb2=16, in2=16, out2=16, out_transpose=1)
ODD = dict(nb1=3, in1=5, out1=4, nb2=2, in2=6, out2=7, out_transpose=0)

# (case id, shape, dtype, rows, expected forward family, expected backward family)
CASES = [
    ("n256_fp32_generic", synthetic.shape_of(W["n256_fp32"]), "f32", 77, 0, 0),
    ("sq16_rows", SQ16, "bf16", 300, 2, 1),
    ("n1024_rows", synthetic.shape_of(W["n1024_bf16"]), "bf16", 300, 2, 1),
    ("r768x3072_wide", synthetic.shape_of(W["r768x3072_bf16"]), "bf16", 300, 3, 3),
    ("n4096_split", synthetic.shape_of(W["n4096_bf16"]), "bf16", 300, 4, 1),
    ("nblk4_group", synthetic.shape_of(W["nblk4_1024x4096_bf16"]), "bf16", 300, 1, 2),
    # enough rows for the CTA-pair kernels (weight gradient and the streamed-weight dU stage)
    ("nblk4_pairs", synthetic.shape_of(W["nblk4_1024x4096_bf16"]), "bf16", 5003, 1, 2),
    # G = in2 / nb1 = 128: two 64-column groups per R block in the gathers
    ("nblk2_gemm", dict(nb1=2, in1=128, out1=256, nb2=2, in2=256, out2=384, out_transpose=0), "bf16", 300, 0, 2),
    ("odd_generic_bf16", ODD, "bf16", 203, 0, 0),
]


def _bf16_exact(a: np.ndarray) -> bool:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return bool(torch.equal(t.to(torch.bfloat16).double(), t))


def _to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    return t.to(torch.bfloat16 if dtype == "bf16" else torch.float32).cuda()


def _host(t: torch.Tensor) -> np.ndarray:
    return t.double().cpu().numpy()


def _check_exact_range(inp):
    R, L = inp["R"], inp["L"]
    u = np.abs(R).sum(axis=2).max()                      # |u| <= row abs-sum of R (|x| <= 1)
    v = u * np.abs(L).sum(axis=2).max()
    dz = np.abs(L).sum(axis=1).max()                     # |dZ| <= column abs-sum of L (|dy| <= 1)
    dx = dz * np.abs(R).sum(axis=1).max()
    assert max(u, v, dz, dx) <= 256, "inputs leave the exact bf16 integer range"


def _ids(c):
    return c[0]


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_forward_exact(case):
    _, shape, dtype, rows, fpath, _ = case
    assert bdl.fwd_path(shape, dtype) == fpath
    inp = synthetic.make_sparse_sign_inputs(dict(shape, rows=rows), seed=21)
    _check_exact_range(inp)
    ref = oracle.forward(shape, inp["X"], inp["R"], inp["L"])
    assert _bf16_exact(ref)
    Y = bdl.fwd(_to_dev(inp["X"], dtype), _to_dev(inp["R"], dtype), _to_dev(inp["L"], dtype), shape)
    assert bdl.last_device_status() == 0
    got = _host(Y)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, "%d entries differ, first at %s: %r vs %r" % (
        len(bad), tuple(bad[0]), got[tuple(bad[0])], ref[tuple(bad[0])])


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_backward_exact(case):
    _, shape, dtype, rows, _, bpath = case
    assert bdl.bwd_path(shape, dtype) == bpath
    inp = synthetic.make_sparse_sign_inputs(dict(shape, rows=rows), seed=22)
    if rows > 1000:
        # the weight gradients sum over rows: keep every 25th row live (all tiles and row splits
        # still run) so that those sums stay in the exact bf16 integer range
        dead = np.arange(rows) % 25 != 0
        inp["X"][dead] = 0.0
        inp["dY"][dead] = 0.0
    _check_exact_range(inp)
    refs = oracle.backward(shape, inp["dY"], inp["X"], inp["R"], inp["L"])
    for r in refs:
        assert _bf16_exact(r), "weight-gradient sums left the exact bf16 range"
    got = bdl.bwd(*(_to_dev(inp[k], dtype) for k in ("dY", "X", "R", "L")), shape)
    assert bdl.last_device_status() == 0
    for g, r, what in zip(got, refs, ("dX", "dR", "dL")):
        g = _host(g)
        bad = np.argwhere(g != r)
        assert bad.size == 0, "%s: %d entries differ, first at %s: %r vs %r" % (
            what, len(bad), tuple(bad[0]), g[tuple(bad[0])], r[tuple(bad[0])])


WS_PATHS = {"nblk4_group": 5, "nblk4_pairs": 5, "nblk2_gemm": 5, "n4096_split": 6}


@pytest.mark.parametrize("case", [c for c in CASES if c[0] in WS_PATHS], ids=_ids)
def test_forward_with_workspace_exact(case):
    """monarch_fwd_ws: the two-pass tcgen05 GEMM forward (U in the workspace, 64-column
    gathers; path 5) or the two streaming stages with folded permutations (Z in the workspace;
    path 6)."""
    name, shape, dtype, rows, _, _ = case
    assert bdl.fwd_ws_path(shape, dtype) == WS_PATHS[name]
    inp = synthetic.make_sparse_sign_inputs(dict(shape, rows=rows), seed=23)
    _check_exact_range(inp)
    ref = oracle.forward(shape, inp["X"], inp["R"], inp["L"])
    Y = bdl.fwd_ws(_to_dev(inp["X"], dtype), _to_dev(inp["R"], dtype), _to_dev(inp["L"], dtype), shape)
    assert bdl.last_device_status() == 0
    got = _host(Y)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, "%d entries differ, first at %s" % (len(bad), tuple(bad[0]))


TRAIN_CASES = [c for c in CASES if c[0] in ("sq16_rows", "n1024_rows", "n4096_split", "nblk4_group", "nblk2_gemm",
                                          "r768x3072_wide")]


@pytest.mark.parametrize("case", TRAIN_CASES, ids=_ids)
def test_training_pair_exact(case):
    """monarch_fwd_train + monarch_bwd_saved: Y, dX, dR, dL equal the oracle entry by entry, with
    the middle vector taken from the forward."""
    name, shape, dtype, rows, _, _ = case
    inp = synthetic.make_sparse_sign_inputs(dict(shape, rows=rows), seed=24)
    _check_exact_range(inp)
    X, R, L, dY = (_to_dev(inp[k], dtype) for k in ("X", "R", "L", "dY"))
    Y, saved = bdl.fwd_train(X, R, L, shape)
    assert saved is not None
    got = bdl.bwd_saved(dY, X, R, L, shape, saved)
    assert bdl.last_device_status() == 0
    refs = (oracle.forward(shape, inp["X"], inp["R"], inp["L"]),) + \
        tuple(oracle.backward(shape, inp["dY"], inp["X"], inp["R"], inp["L"]))
    for g, r, what in zip((Y,) + tuple(got), refs, ("Y", "dX", "dR", "dL")):
        g = _host(g)
        bad = np.argwhere(g != r)
        assert bad.size == 0, "%s: %d entries differ, first at %s" % (what, len(bad), tuple(bad[0]))
