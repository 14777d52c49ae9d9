"""GPU parity of the dense -> Monarch projection (monarch_project) against the oracle.

The oracle takes an SVD per slice (fp64); the GPU runs fp32 power iteration per slice, so the
comparison is normwise: 1e-5 on the fp32 factors and on the projected matrix, 2e-2 when the
factors are stored in bf16.  Inputs are Monarch matrices plus small dense noise (the near-
Monarch matrices a projection is used on), so every slice's two leading singular values are
well separated; a pure Monarch matrix must come back unchanged.
"""
import numpy as np
import pytest
import torch

import block_diagonal_linear_b200 as bdl
import oracle

pytestmark = pytest.mark.gpu

SHAPES = [
    dict(nb1=32, in1=32, out1=32, nb2=32, in2=32, out2=32, out_transpose=1),   # n = 1024
    dict(nb1=16, in1=48, out1=48, nb2=48, in2=16, out2=64, out_transpose=1),   # 768 -> 3072
    dict(nb1=64, in1=64, out1=64, nb2=64, in2=64, out2=64, out_transpose=1),   # n = 4096
    dict(nb1=3, in1=5, out1=2, nb2=2, in2=3, out2=6, out_transpose=1),
]


def _near_monarch(d, seed, noise):
    rng = np.random.default_rng(seed)
    R = rng.uniform(-1, 1, (d["nb1"], d["out1"], d["in1"]))
    L = rng.uniform(-1, 1, (d["nb2"], d["out2"], d["in2"]))
    M = oracle.materialise(d, R, L)
    return M + noise * rng.standard_normal(M.shape) * np.abs(M).mean()


@pytest.mark.parametrize("d", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_projection_matches_oracle(d, dtype):
    M = _near_monarch(d, seed=41, noise=1e-2)
    Rr, Lr = oracle.project(d, M)
    Mg = torch.tensor(M, dtype=torch.float32, device="cuda")
    R, L = bdl.project(Mg, d, dtype)
    assert bdl.last_device_status() == 0
    tol = 1e-5 if dtype == "f32" else 2e-2
    Rg, Lg = R.double().cpu().numpy(), L.double().cpu().numpy()
    assert oracle.normwise_rel_err(Rg, Rr) <= tol
    assert oracle.normwise_rel_err(Lg, Lr) <= tol
    assert oracle.normwise_rel_err(oracle.materialise(d, Rg, Lg), oracle.materialise(d, Rr, Lr)) <= tol


def test_monarch_matrix_comes_back_unchanged():
    d = SHAPES[1]
    M = _near_monarch(d, seed=42, noise=0.0)
    Mg = torch.tensor(M, dtype=torch.float32, device="cuda")
    R, L = bdl.project(Mg, d, "f32")
    Mp = oracle.materialise(d, R.double().cpu().numpy(), L.double().cpu().numpy())
    assert oracle.normwise_rel_err(Mp, M) <= 1e-5


def test_projection_rejects_non_lattice_shapes():
    d = dict(nb1=4, in1=256, out1=256, nb2=4, in2=256, out2=1024, out_transpose=0)
    Mg = torch.zeros((4096, 1024), dtype=torch.float32, device="cuda")
    with pytest.raises(bdl.MonarchError) as e:
        bdl.project(Mg, d, "f32")
    assert e.value.code == bdl.CODES["MONARCH_ERR_UNSUPPORTED"]
