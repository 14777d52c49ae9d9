"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerance: normwise relative error ||G - O||_F / ||O||_F per output tensor,
<= 1e-5 for fp32 inputs and <= 2e-2 for bf16 inputs, on the same seeded inputs.
"""
import numpy as np
import pytest
import torch

import block_diagonal_linear_b200 as bdl
import oracle
from block_diagonal_linear_b200 import synthetic
from gpu_helpers import TOL, dev_inputs, to_dev, to_f64

pytestmark = pytest.mark.gpu
W = synthetic.WORKLOADS

# (workload, rows for the element-by-element oracle check): several 128-row tiles plus a ragged tail
SMALL_ROWS = [
    ("n256_fp32", 64), ("n256_fp32", 1), ("n1024_bf16", 1000), ("n1024_bf16", 77),
    ("r768x3072_bf16", 700), ("n4096_bf16", 300), ("nblk4_1024x4096_bf16", 1000),
    ("nblk4_1024x4096_bf16", 129),
]

RANDOM_SHAPES = [
    dict(nb1=3, in1=5, out1=4, nb2=2, in2=6, out2=7, out_transpose=1),
    dict(nb1=3, in1=5, out1=4, nb2=2, in2=6, out2=7, out_transpose=0),
    dict(nb1=8, in1=8, out1=8, nb2=8, in2=8, out2=8, out_transpose=1),
    dict(nb1=2, in1=64, out1=96, nb2=6, in2=32, out2=40, out_transpose=1),
    dict(nb1=5, in1=1, out1=3, nb2=15, in2=1, out2=2, out_transpose=0),
    dict(nb1=16, in1=16, out1=16, nb2=16, in2=16, out2=16, out_transpose=0),
]


def check(got, ref, dtype, what):
    err = oracle.normwise_rel_err(got, ref)
    assert err <= TOL[dtype], "%s: normwise rel err %.3e > %.1e" % (what, err, TOL[dtype])
    return err


def run_fwd(w, inp):
    d = dev_inputs(inp)
    Y = bdl.fwd(d["X"], d["R"], d["L"], synthetic.shape_of(w))
    assert bdl.last_device_status() == 0
    return to_f64(Y)


def run_bwd(w, inp):
    d = dev_inputs(inp)
    dX, dR, dL = bdl.bwd(d["dY"], d["X"], d["R"], d["L"], synthetic.shape_of(w))
    assert bdl.last_device_status() == 0
    return to_f64(dX), to_f64(dR), to_f64(dL)


@pytest.mark.parametrize("name,rows", SMALL_ROWS)
def test_fwd_matches_oracle(name, rows):
    w = W[name]
    inp = synthetic.make_inputs(w, seed=1, rows=rows)
    Y = run_fwd(w, inp)
    ref = oracle.forward(synthetic.shape_of(w), inp["X"].f64, inp["R"].f64, inp["L"].f64)
    check(Y, ref, w["dtype"], name + " Y")


@pytest.mark.parametrize("name,rows", SMALL_ROWS)
def test_bwd_matches_oracle(name, rows):
    w = W[name]
    inp = synthetic.make_inputs(w, seed=2, rows=rows)
    dX, dR, dL = run_bwd(w, inp)
    rX, rR, rL = oracle.backward(synthetic.shape_of(w), inp["dY"].f64, inp["X"].f64,
                                 inp["R"].f64, inp["L"].f64)
    check(dX, rX, w["dtype"], name + " dX")
    check(dR, rR, w["dtype"], name + " dR")
    check(dL, rL, w["dtype"], name + " dL")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", RANDOM_SHAPES)
def test_random_shapes_fwd_bwd(shape, dtype):
    w = dict(shape, rows=203, dtype=dtype)
    inp = synthetic.make_inputs(w, seed=3)
    Y = run_fwd(w, inp)
    ref = oracle.forward(shape, inp["X"].f64, inp["R"].f64, inp["L"].f64)
    check(Y, ref, dtype, "Y")
    dX, dR, dL = run_bwd(w, inp)
    rX, rR, rL = oracle.backward(shape, inp["dY"].f64, inp["X"].f64, inp["R"].f64, inp["L"].f64)
    check(dX, rX, dtype, "dX")
    check(dR, rR, dtype, "dR")
    check(dL, rL, dtype, "dL")


@pytest.mark.parametrize("name", ["n256_fp32", "n1024_bf16", "r768x3072_bf16", "n4096_bf16",
                                  "nblk4_1024x4096_bf16"])
def test_full_size_sampled_rows_and_directional_identities(name):
    """Full workload size, the launch the benchmark times.  Sampled rows of Y and dX
    against the oracle row by row.  dR and dL through identities that hold at any
    size: Y is linear in R and in L, so for any direction D,
    <dR, D> = <dY, fwd(X, D, L)> and <dL, D> = <dY, fwd(X, R, D)>."""
    w = W[name]
    shape = synthetic.shape_of(w)
    inp = synthetic.make_inputs(w, seed=0)
    d = dev_inputs(inp)
    Y = bdl.fwd(d["X"], d["R"], d["L"], shape)
    dX, dR, dL = bdl.bwd(d["dY"], d["X"], d["R"], d["L"], shape)
    assert bdl.last_device_status() == 0
    rows = w["rows"]
    rng = np.random.default_rng(7)
    sample = np.unique(np.concatenate([rng.choice(rows, size=min(rows, 96), replace=False),
                                       [0, rows - 1]]))
    idx = torch.as_tensor(sample, device="cuda")
    rY = oracle.forward(shape, inp["X"].f64[sample], inp["R"].f64, inp["L"].f64)
    rX, _, _ = oracle.backward(shape, inp["dY"].f64[sample], inp["X"].f64[sample],
                               inp["R"].f64, inp["L"].f64)
    check(to_f64(Y[idx]), rY, w["dtype"], "sampled Y")
    check(to_f64(dX[idx]), rX, w["dtype"], "sampled dX")
    dY64 = inp["dY"].f64
    lhs, rhs = [], []
    for k in range(4):
        dirs = synthetic.make_inputs(w, seed=100 + k, rows=1)
        DR, DL = to_dev(dirs["R"]), to_dev(dirs["L"])
        lhs.append(float(np.sum(to_f64(dR) * dirs["R"].f64)))
        rhs.append(float(np.sum(dY64 * to_f64(bdl.fwd(d["X"], DR, d["L"], shape)))))
        lhs.append(float(np.sum(to_f64(dL) * dirs["L"].f64)))
        rhs.append(float(np.sum(dY64 * to_f64(bdl.fwd(d["X"], d["R"], DL, shape)))))
    check(np.array(lhs), np.array(rhs), w["dtype"], "directional dR/dL")


@pytest.mark.parametrize("name", ["n1024_bf16", "r768x3072_bf16", "n4096_bf16", "nblk4_1024x4096_bf16",
                                  "nblk4_1024x4096_bf16_b1000"])
def test_full_size_bwd_weight_grads_vs_oracle(name):
    """Full workload size: every entry of dX, dR and dL against the fp64 oracle."""
    w = W[name]
    shape = synthetic.shape_of(w)
    inp = synthetic.make_inputs(w, seed=4)
    dX, dR, dL = run_bwd(w, inp)
    rX, rR, rL = oracle.backward(shape, inp["dY"].f64, inp["X"].f64, inp["R"].f64, inp["L"].f64)
    check(dX, rX, "bf16", "dX")
    check(dR, rR, "bf16", "dR")
    check(dL, rL, "bf16", "dL")


@pytest.mark.parametrize("name", sorted(W))
def test_materialise_matches_oracle(name):
    w = W[name]
    inp = synthetic.make_inputs(w, seed=5, rows=1)
    d = dev_inputs(inp)
    M = to_f64(bdl.materialise(d["R"], d["L"], synthetic.shape_of(w)))
    ref = oracle.materialise(synthetic.shape_of(w), inp["R"].f64, inp["L"].f64)
    check(M, ref, "f32", "M")


def test_forward_of_identity_is_dense_matrix():
    """fwd(I) = I M^T: the dense matrix, as in the identity example of the pages."""
    shape = dict(nb1=4, in1=4, out1=4, nb2=4, in2=4, out2=4, out_transpose=1)
    w = dict(shape, rows=16, dtype="f32")
    inp = synthetic.make_inputs(w, seed=6)
    d = dev_inputs(inp)
    eye = torch.eye(16, dtype=torch.float32, device="cuda")
    MT = to_f64(bdl.fwd(eye, d["R"], d["L"], shape))
    M = to_f64(bdl.materialise(d["R"], d["L"], shape))
    np.testing.assert_allclose(MT.T, M, rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("name,rows", [("n1024_bf16", r) for r in (0, 1, 127, 128, 129, 255, 256, 257)]
                         + [("r768x3072_bf16", r) for r in (0, 1, 63, 64, 65, 191, 9473, 20000)]
                         + [("n4096_bf16", r) for r in (0, 1, 127, 129, 1000)])
def test_tc_forward_tile_edges(name, rows):
    w = W[name]
    shape = synthetic.shape_of(w)
    inp = synthetic.make_inputs(w, seed=8, rows=max(rows, 1))
    d = dev_inputs(inp)
    X = d["X"][:rows].contiguous()
    Y = torch.full((rows, w["nb2"] * w["out2"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    bdl.fwd(X, d["R"], d["L"], shape, Y=Y)
    assert bdl.last_device_status() == 0
    if rows:
        ref = oracle.forward(shape, inp["X"].f64[:rows], inp["R"].f64, inp["L"].f64)
        check(to_f64(Y), ref, "bf16", "Y")


@pytest.mark.parametrize("name,rows", [("n1024_bf16", r) for r in (1, 129, 257)]
                         + [("r768x3072_bf16", r) for r in (1, 63, 65, 191, 9473)]
                         + [("n4096_bf16", r) for r in (1, 129, 1000)])
def test_training_pair_tile_edges(name, rows):
    """Ragged row counts: the training forward's kept middle vector (partial last tiles of the Z
    stores) gives the backward the same results as recomputing it, bit for bit."""
    w = W[name]
    shape = synthetic.shape_of(w)
    inp = synthetic.make_inputs(w, seed=31, rows=rows)
    d = dev_inputs(inp)
    Y1 = bdl.fwd_ws(d["X"], d["R"], d["L"], shape)
    Y2, saved = bdl.fwd_train(d["X"], d["R"], d["L"], shape)
    assert saved is not None
    g1 = bdl.bwd(d["dY"], d["X"], d["R"], d["L"], shape)
    g2 = bdl.bwd_saved(d["dY"], d["X"], d["R"], d["L"], shape, saved)
    assert bdl.last_device_status() == 0
    assert torch.equal(Y1, Y2)
    for a, b, what in zip(g1, g2, ("dX", "dR", "dL")):
        assert torch.equal(a, b), what


def test_bwd_deterministic():
    w = W["n1024_bf16"]
    inp = synthetic.make_inputs(w, seed=9, rows=2000)
    d = dev_inputs(inp)
    shape = synthetic.shape_of(w)
    a = bdl.bwd(d["dY"], d["X"], d["R"], d["L"], shape)
    b = bdl.bwd(d["dY"], d["X"], d["R"], d["L"], shape)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_fwd_repeatable_and_no_stale_output():
    w = W["r768x3072_bf16"]
    inp = synthetic.make_inputs(w, seed=10, rows=640)
    d = dev_inputs(inp)
    shape = synthetic.shape_of(w)
    Y1 = bdl.fwd(d["X"], d["R"], d["L"], shape)
    Y2 = torch.full_like(Y1, float("nan"))
    bdl.fwd(d["X"], d["R"], d["L"], shape, Y=Y2)
    assert torch.equal(Y1, Y2)


def test_bounded_wait_reports_timeout_and_context_survives():
    assert bdl.last_device_status() == 0
    assert bdl.debug_wait_timeout(20_000_000) == 0          # 20 ms limit
    assert bdl.last_device_status() == bdl.CODES["MONARCH_ERR_TIMEOUT"]
    assert bdl.last_device_status() == 0                     # cleared on read
    w = W["n256_fp32"]
    inp = synthetic.make_inputs(w, seed=11)
    Y = run_fwd(w, inp)
    check(Y, oracle.forward(synthetic.shape_of(w), inp["X"].f64, inp["R"].f64, inp["L"].f64),
          "f32", "Y after timeout")


def test_workspace_too_small_is_an_error():
    w = W["n256_fp32"]
    inp = synthetic.make_inputs(w, seed=12)
    d = dev_inputs(inp)
    shape = synthetic.shape_of(w)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(bdl.MonarchError) as e:
        bdl.bwd(d["dY"], d["X"], d["R"], d["L"], shape, workspace=ws)
    assert e.value.code == bdl.CODES["MONARCH_ERR_WORKSPACE"]


@pytest.mark.parametrize("name", ["nblk4_1024x4096_bf16", "nblk4_1024x4096_bf16_b1000", "n4096_bf16"])
def test_forward_with_workspace_full_size(name):
    """monarch_fwd_ws at the full workload size (the launch the benchmark times): every entry
    against the oracle, normwise."""
    w = W[name]
    shape = synthetic.shape_of(w)
    inp = synthetic.make_inputs(w, seed=13)
    d = dev_inputs(inp)
    Y = bdl.fwd_ws(d["X"], d["R"], d["L"], shape)
    assert bdl.last_device_status() == 0
    ref = oracle.forward(shape, inp["X"].f64, inp["R"].f64, inp["L"].f64)
    check(to_f64(Y), ref, "bf16", name + " Y (workspace forward)")


@pytest.mark.parametrize("name,rows", [("n4096_bf16", r) for r in (1, 63, 64, 65, 129, 1000, 2405)])
def test_stage_forward_tile_edges(name, rows):
    """The streaming-stage forward (monarch_fwd_ws, path 6) at 64-row unit edges and with more
    units than CTAs: Y pre-filled with NaN, so an entry the drain does not write fails."""
    w = W[name]
    shape = synthetic.shape_of(w)
    assert bdl.fwd_ws_path(shape, "bf16") == 6
    inp = synthetic.make_inputs(w, seed=9, rows=rows)
    d = dev_inputs(inp)
    Y = torch.full((rows, w["nb2"] * w["out2"]), float("nan"), dtype=torch.bfloat16, device="cuda")
    bdl.fwd_ws(d["X"], d["R"], d["L"], shape, Y=Y)
    assert bdl.last_device_status() == 0
    ref = oracle.forward(shape, inp["X"].f64, inp["R"].f64, inp["L"].f64)
    check(to_f64(Y), ref, "bf16", "Y")


@pytest.mark.parametrize("name", ["n1024_bf16", "r768x3072_bf16", "n4096_bf16", "nblk4_1024x4096_bf16"])
def test_training_pair_matches_forward_and_backward_bitwise(name):
    """Full workload size: the training forward's Y equals monarch_fwd_ws's and the saved backward's
    dX, dR, dL equal monarch_bwd's bit for bit (the saved middle vector is the recomputed one)."""
    w = W[name]
    shape = synthetic.shape_of(w)
    inp = synthetic.make_inputs(w, seed=14)
    d = dev_inputs(inp)
    assert bdl.saved_bytes(shape, w["rows"], "bf16") > 0
    Y1 = bdl.fwd_ws(d["X"], d["R"], d["L"], shape)
    Y2, saved = bdl.fwd_train(d["X"], d["R"], d["L"], shape)
    g1 = bdl.bwd(d["dY"], d["X"], d["R"], d["L"], shape)
    g2 = bdl.bwd_saved(d["dY"], d["X"], d["R"], d["L"], shape, saved)
    assert bdl.last_device_status() == 0
    assert torch.equal(Y1, Y2)
    for a, b, what in zip(g1, g2, ("dX", "dR", "dL")):
        assert torch.equal(a, b), what
