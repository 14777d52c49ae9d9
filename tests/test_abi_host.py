"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/monarch.h declares, and rejects bad arguments before it
touches the device."""
import ctypes
import os
import re

import pytest

import block_diagonal_linear_b200 as bdl
from block_diagonal_linear_b200 import synthetic

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "monarch.h")).read()
    return sorted(set(re.findall(r"MONARCH_API\s+[\w\s\*]+?\b(monarch_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 8
    lib = bdl.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(bdl.EXPORTED) == names


def test_status_strings():
    for code in bdl.STATUS:
        assert bdl.status_string(code)
    assert bdl.status_string(-7) == "bounded device wait timed out"


@pytest.mark.parametrize("name", sorted(synthetic.WORKLOADS))
def test_workloads_validate(name):
    w = synthetic.WORKLOADS[name]
    assert bdl.validate(synthetic.shape_of(w), w["rows"], w["dtype"]) == 0


def test_bad_dims_rejected():
    good = dict(nb1=4, in1=8, out1=8, nb2=4, in2=8, out2=8, out_transpose=1)
    assert bdl.validate(good, 3, "f32") == 0
    assert bdl.validate(dict(good, out1=6), 3, "f32") == bdl.CODES["MONARCH_ERR_DIMS"]
    assert bdl.validate(dict(good, nb2=0), 3, "f32") == bdl.CODES["MONARCH_ERR_DIMS"]
    assert bdl.validate(good, -1, "f32") == bdl.CODES["MONARCH_ERR_DIMS"]
    assert bdl.validate(good, 3, 7) == bdl.CODES["MONARCH_ERR_DTYPE"]
    # rows == 0 is a valid no-op shape
    assert bdl.validate(good, 0, "bf16") == 0


def test_fwd_argument_errors_before_device_work():
    lib = bdl.lib()
    shape = dict(nb1=4, in1=8, out1=8, nb2=4, in2=8, out2=8, out_transpose=1)
    d = bdl.make_dims(shape, 5, "f32")
    p = ctypes.c_void_p(4096)
    assert lib.monarch_fwd(None, p, p, ctypes.byref(d), p, None) == bdl.CODES["MONARCH_ERR_NULL"]
    assert lib.monarch_fwd(ctypes.c_void_p(4100), p, p, ctypes.byref(d), p, None) == \
        bdl.CODES["MONARCH_ERR_ALIGN"]
    bad = bdl.make_dims(dict(shape, in2=5), 5, "f32")
    assert lib.monarch_fwd(p, p, p, ctypes.byref(bad), p, None) == bdl.CODES["MONARCH_ERR_DIMS"]
    # rows == 0: nothing to do, even with null tensors
    z = bdl.make_dims(shape, 0, "f32")
    assert lib.monarch_fwd(None, p, p, ctypes.byref(z), None, None) == 0
    assert lib.monarch_fwd(p, p, p, None, p, None) == bdl.CODES["MONARCH_ERR_NULL"]


def test_bwd_workspace_checks_before_device_work():
    lib = bdl.lib()
    shape = synthetic.shape_of(synthetic.WORKLOADS["n1024_bf16"])
    d = bdl.make_dims(shape, 1000, "bf16")
    need = bdl.bwd_workspace_bytes(shape, 1000, "bf16")
    assert need > 0
    p = ctypes.c_void_p(4096)
    rc = lib.monarch_bwd(p, p, p, p, ctypes.byref(d), p, p, p, p, ctypes.c_size_t(need - 1), None)
    assert rc == bdl.CODES["MONARCH_ERR_WORKSPACE"]
    rc = lib.monarch_bwd(p, p, p, p, ctypes.byref(d), p, p, p, None, ctypes.c_size_t(need), None)
    assert rc == bdl.CODES["MONARCH_ERR_WORKSPACE"]
    rc = lib.monarch_bwd(p, p, p, p, ctypes.byref(d), p, p, p, ctypes.c_void_p(4096 + 16),
                         ctypes.c_size_t(need), None)
    assert rc == bdl.CODES["MONARCH_ERR_ALIGN"]
    assert bdl.bwd_workspace_bytes(dict(shape, out1=5), 10, "bf16") == 0


def test_training_pair_sizes_and_checks_before_device_work():
    """monarch_saved_bytes per forward family, and the training pair's argument checks (fake
    device pointers: every call must fail before any device work)."""
    W = synthetic.WORKLOADS
    n1024, n4096 = synthetic.shape_of(W["n1024_bf16"]), synthetic.shape_of(W["n4096_bf16"])
    nblk4, r768 = synthetic.shape_of(W["nblk4_1024x4096_bf16"]), synthetic.shape_of(W["r768x3072_bf16"])
    assert bdl.saved_bytes(n1024, 100, "bf16") == 100 * 1024 * 2  # Z of the fused forward
    assert bdl.saved_bytes(n4096, 100, "bf16") == 100 * 4096 * 2  # Z of the streaming stages
    assert bdl.saved_bytes(nblk4, 100, "bf16") == bdl.fwd_workspace_bytes(nblk4, 100, "bf16")  # L reordered, U
    assert bdl.saved_bytes(r768, 100, "bf16") == 100 * 768 * 2   # Z of the wide-output forward
    assert bdl.saved_bytes(n1024, 100, "f32") == 0
    lib = bdl.lib()
    d = bdl.make_dims(n1024, 1000, "bf16")
    need = bdl.saved_bytes(n1024, 1000, "bf16")
    p, sz = ctypes.c_void_p(1 << 40), ctypes.c_size_t
    assert lib.monarch_fwd_train(p, p, p, ctypes.byref(d), p, None, sz(need), None) == \
        bdl.CODES["MONARCH_ERR_WORKSPACE"]
    assert lib.monarch_fwd_train(p, p, p, ctypes.byref(d), p, p, sz(need - 1), None) == \
        bdl.CODES["MONARCH_ERR_WORKSPACE"]
    assert lib.monarch_fwd_train(p, p, p, ctypes.byref(d), p, ctypes.c_void_p((1 << 40) + 16), sz(need), None) == \
        bdl.CODES["MONARCH_ERR_ALIGN"]
    # saved overlapping X
    assert lib.monarch_fwd_train(p, ctypes.c_void_p(1 << 41), ctypes.c_void_p(1 << 42), ctypes.byref(d),
                                 ctypes.c_void_p(1 << 43), p, sz(need), None) == bdl.CODES["MONARCH_ERR_ALIAS"]
    wneed = bdl.bwd_workspace_bytes(n1024, 1000, "bf16")
    q = [ctypes.c_void_p(k << 36) for k in range(1, 10)]
    assert lib.monarch_bwd_saved(q[0], q[1], q[2], q[3], ctypes.byref(d), None, sz(need), q[4], q[5], q[6], q[7],
                                 sz(wneed), None) == bdl.CODES["MONARCH_ERR_WORKSPACE"]
    assert lib.monarch_bwd_saved(q[0], q[1], q[2], q[3], ctypes.byref(d), q[8], sz(need), q[4], q[5], q[6], q[7],
                                 sz(wneed - 1), None) == bdl.CODES["MONARCH_ERR_WORKSPACE"]
    # an output (dX) overlapping the saved buffer
    assert lib.monarch_bwd_saved(q[0], q[1], q[2], q[3], ctypes.byref(d), q[8], sz(need), q[8], q[5], q[6], q[7],
                                 sz(wneed), None) == bdl.CODES["MONARCH_ERR_ALIAS"]


def test_kernel_family_selection():
    W = synthetic.WORKLOADS
    assert bdl.fwd_path(synthetic.shape_of(W["n1024_bf16"]), "bf16") == 2
    assert bdl.fwd_path(synthetic.shape_of(W["r768x3072_bf16"]), "bf16") == 3
    assert bdl.fwd_path(synthetic.shape_of(W["nblk4_1024x4096_bf16"]), "bf16") == 1
    assert bdl.fwd_path(synthetic.shape_of(W["n4096_bf16"]), "bf16") == 4
    assert bdl.fwd_path(synthetic.shape_of(W["n4096_bf16"]), "f32") == 0
    assert bdl.fwd_path(synthetic.shape_of(W["n256_fp32"]), "f32") == 0
    assert bdl.fwd_path(synthetic.shape_of(W["n256_fp32"]), "bf16") == 2
    assert bdl.fwd_path(dict(nb1=3, in1=5, out1=4, nb2=2, in2=6, out2=7, out_transpose=1), "bf16") == 0
    assert bdl.bwd_path(synthetic.shape_of(W["n1024_bf16"]), "bf16") == 1
    assert bdl.bwd_path(synthetic.shape_of(W["n256_fp32"]), "bf16") == 1
    assert bdl.bwd_path(synthetic.shape_of(W["n256_fp32"]), "f32") == 0
    assert bdl.bwd_path(synthetic.shape_of(W["n4096_bf16"]), "bf16") == 1
    assert bdl.bwd_path(synthetic.shape_of(W["r768x3072_bf16"]), "bf16") == 3
    # workspace forward: two-pass GEMM (5), streaming stages (6), else the monarch_fwd family
    assert bdl.fwd_ws_path(synthetic.shape_of(W["nblk4_1024x4096_bf16"]), "bf16") == 5
    assert bdl.fwd_ws_path(synthetic.shape_of(W["n4096_bf16"]), "bf16") == 6
    assert bdl.fwd_ws_path(synthetic.shape_of(W["n4096_bf16"]), "f32") == 0
    assert bdl.fwd_ws_path(synthetic.shape_of(W["n1024_bf16"]), "bf16") == 2
    assert bdl.fwd_ws_path(synthetic.shape_of(W["r768x3072_bf16"]), "bf16") == 3
    n = synthetic.shape_of(W["n4096_bf16"])
    assert bdl.fwd_workspace_bytes(n, 100, "bf16") == 100 * 4096 * 2
    assert bdl.bwd_path(synthetic.shape_of(W["nblk4_1024x4096_bf16"]), "bf16") == 2
    assert bdl.bwd_path(synthetic.shape_of(W["nblk4_1024x4096_bf16"]), "f32") == 0


def test_overlapping_outputs_rejected_before_device_work():
    """Outputs (and the backward workspace) must not overlap inputs or each other: the 64x64
    path keeps the middle vector in Y, and the backward's kernels read inputs after earlier
    kernels of the same call wrote outputs.  Fake, aligned addresses: every case returns
    before any CUDA call."""
    lib = bdl.lib()
    shape = dict(nb1=4, in1=8, out1=8, nb2=4, in2=8, out2=8, out_transpose=1)
    rows = 5
    d = bdl.make_dims(shape, rows, "f32")
    A = lambda a: ctypes.c_void_p(a)
    x, r, l = 1 << 20, 2 << 20, 3 << 20       # X: 5*32*4 = 640 B, R and L: 1024 B each
    alias = bdl.CODES["MONARCH_ERR_ALIAS"]
    assert lib.monarch_fwd(A(x), A(r), A(l), ctypes.byref(d), A(x + 624), None) == alias  # Y overlaps X
    assert lib.monarch_fwd(A(x), A(r), A(l), ctypes.byref(d), A(r - 16), None) == alias   # Y runs into R
    assert lib.monarch_fwd(A(x), A(r), A(l), ctypes.byref(d), A(l), None) == alias        # Y is L
    need = bdl.bwd_workspace_bytes(shape, rows, "f32")
    dy, dx, dr, dl, ws = 4 << 20, 5 << 20, 6 << 20, 7 << 20, 8 << 20
    ok = dict(dy=dy, x=x, r=r, l=l, dx=dx, dr=dr, dl=dl, ws=ws)

    def bwd(**kw):
        a = dict(ok, **kw)
        return lib.monarch_bwd(A(a["dy"]), A(a["x"]), A(a["r"]), A(a["l"]), ctypes.byref(d), A(a["dx"]),
                               A(a["dr"]), A(a["dl"]), A(a["ws"]), ctypes.c_size_t(need), None)

    assert bwd(dx=dy) == alias                 # dX is dY
    assert bwd(dr=dl) == alias                 # dR is dL
    assert bwd(dl=r + 512) == alias            # dL overlaps R
    assert bwd(ws=x - 256) == alias            # workspace runs into X
    assert bwd(ws=dx) == alias                 # workspace is dX
    assert bdl.status_string(alias) != "unknown status"


def test_binding_checks_tensor_shapes_and_dtypes_first():
    """The binding compares every tensor with the dims before anything reaches the library,
    so mismatched factors fail loudly instead of being read with the wrong layout."""
    import torch
    shape = dict(nb1=4, in1=8, out1=8, nb2=4, in2=8, out2=16, out_transpose=1)
    X = torch.zeros(5, 32, dtype=torch.bfloat16)
    R = torch.zeros(4, 8, 8, dtype=torch.bfloat16)
    L = torch.zeros(4, 16, 8, dtype=torch.bfloat16)
    dY = torch.zeros(5, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="L has shape"):
        bdl.fwd(X, R, L.transpose(1, 2), shape)
    with pytest.raises(ValueError, match="X has shape"):
        bdl.fwd(X[:, :16], R, L, shape)
    with pytest.raises(ValueError, match="one dtype"):
        bdl.fwd(X, R.float(), L, shape)
    with pytest.raises(ValueError, match="dY has shape"):
        bdl.bwd(dY[:, :32], X, R, L, shape)
    with pytest.raises(ValueError, match="Y has shape"):
        bdl.fwd(X, R, L, shape, Y=torch.zeros(5, 32, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="R has shape"):
        bdl.materialise(R[:2], L, shape)
    # correct shapes get past the check and stop at the CUDA-tensor requirement
    with pytest.raises(ValueError, match="CUDA"):
        bdl.fwd(X, R, L, shape)


def test_shape_beyond_every_kernel_is_unsupported_before_device_work():
    """A middle vector wider than the generic kernels' shared-memory row (fp32, 60000 wide)
    is rejected with MONARCH_ERR_UNSUPPORTED on the host (fake, disjoint, aligned pointers)."""
    lib = bdl.lib()
    shape = dict(nb1=1, in1=16, out1=60000, nb2=1, in2=60000, out2=16, out_transpose=1)
    d = bdl.make_dims(shape, 2, "f32")
    assert bdl.validate(shape, 2, "f32") == 0
    A = lambda i: ctypes.c_void_p(i << 24)  # 16 MiB apart: no argument overlaps another
    unsupported = bdl.CODES["MONARCH_ERR_UNSUPPORTED"]
    assert lib.monarch_fwd(A(1), A(2), A(3), ctypes.byref(d), A(4), None) == unsupported
    need = bdl.bwd_workspace_bytes(shape, 2, "f32")
    assert 0 < need < (16 << 24)
    rc = lib.monarch_bwd(A(5), A(1), A(2), A(3), ctypes.byref(d), A(6), A(7), A(8), A(16),
                         ctypes.c_size_t(need), None)
    assert rc == unsupported


def test_oversized_dims_rejected():
    assert bdl.validate(dict(nb1=1 << 21, in1=1 << 20, out1=1, nb2=1, in2=1 << 21, out2=1), 1, "bf16") == \
        bdl.CODES["MONARCH_ERR_DIMS"]
