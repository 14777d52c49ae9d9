"""B200 (sm_100a) Monarch linear map: Python binding of libmonarch.so.

This module only marshals arguments: every step of the forward and backward
runs in the CUDA kernels behind the C ABI declared in ``include/monarch.h``.
PyTorch provides device memory and the current CUDA stream.  There is no CPU
fallback: if the library or a GPU is missing, calls raise.

    Y = X M^T,   M = P_out L P R   (Monarch: products of two block-diagonal
    matrices with a reshape-transpose permutation; scatterbrain issue thread,
    Definition C.3 and the N=4 permutation example)

Shapes use the MonarchLinear convention: R is (nb1, out1, in1), L is
(nb2, out2, in2), X is (rows, nb1*in1), Y is (rows, nb2*out2).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmonarch.so")

MONARCH_F32 = 0
MONARCH_BF16 = 1

STATUS = {
    0: "MONARCH_OK",
    -1: "MONARCH_ERR_DIMS",
    -2: "MONARCH_ERR_DTYPE",
    -3: "MONARCH_ERR_ALIGN",
    -4: "MONARCH_ERR_NULL",
    -5: "MONARCH_ERR_WORKSPACE",
    -6: "MONARCH_ERR_CUDA",
    -7: "MONARCH_ERR_TIMEOUT",
    -8: "MONARCH_ERR_UNSUPPORTED",
    -9: "MONARCH_ERR_SCRATCH",
    -10: "MONARCH_ERR_ALIAS",
}
CODES = {v: k for k, v in STATUS.items()}

EXPORTED = (
    "monarch_validate", "monarch_fwd", "monarch_bwd", "monarch_bwd_workspace_bytes",
    "monarch_materialise", "monarch_status_string", "monarch_last_device_status",
    "monarch_debug_wait_timeout", "monarch_fwd_path", "monarch_bwd_path", "monarch_bwd_noalloc",
    "monarch_kernel_launches", "monarch_fwd_workspace_bytes", "monarch_fwd_ws_path", "monarch_fwd_ws",
    "monarch_saved_bytes", "monarch_fwd_train", "monarch_bwd_saved",
    "monarch_linear_shape", "monarch_linear_workspace_bytes",
    "monarch_linear_fwd", "monarch_linear_bwd", "monarch_project", "monarch_dyad_workspace_bytes",
    "monarch_dyad_path", "monarch_dyad_fwd", "monarch_dyad_bwd", "monarch_lattice_workspace_bytes",
    "monarch_lattice_path", "monarch_lattice_weight_elems", "monarch_lattice_fwd", "monarch_lattice_bwd",
)


class MonarchDims(ctypes.Structure):
    """Mirror of ``monarch_dims`` in include/monarch.h."""
    _fields_ = [
        ("rows", ctypes.c_int64),
        ("nb1", ctypes.c_int32),
        ("in1", ctypes.c_int32),
        ("out1", ctypes.c_int32),
        ("nb2", ctypes.c_int32),
        ("in2", ctypes.c_int32),
        ("out2", ctypes.c_int32),
        ("out_transpose", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
    ]


class MonarchLinearDims(ctypes.Structure):
    """Mirror of ``monarch_linear_dims`` in include/monarch.h."""
    _fields_ = [
        ("rows", ctypes.c_int64),
        ("in_features", ctypes.c_int32),
        ("out_features", ctypes.c_int32),
        ("nblocks", ctypes.c_int32),
        ("has_bias", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
    ]


class MonarchDyadDims(ctypes.Structure):
    """Mirror of ``monarch_dyad_dims`` in include/monarch.h."""
    _fields_ = [
        ("rows", ctypes.c_int64),
        ("nblocks", ctypes.c_int32),
        ("in_blk", ctypes.c_int32),
        ("out_blk", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
    ]


class MonarchLatticeDims(ctypes.Structure):
    """Mirror of ``monarch_lattice_dims`` in include/monarch.h."""
    _fields_ = [
        ("rows", ctypes.c_int64),
        ("naxes", ctypes.c_int32),
        ("n_in", ctypes.c_int32 * 4),
        ("n_out", ctypes.c_int32 * 4),
        ("dtype", ctypes.c_int32),
    ]


class MonarchError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (fn, STATUS.get(code, "?"), code))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmonarch.so (built in-tree by ``block_diagonal_linear_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libmonarch.so is not built; run `python -m block_diagonal_linear_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, dp = ctypes.c_void_p, ctypes.POINTER(MonarchDims)
        L.monarch_validate.argtypes = [dp]
        L.monarch_fwd.argtypes = [vp, vp, vp, dp, vp, vp]
        L.monarch_bwd.argtypes = [vp, vp, vp, vp, dp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.monarch_bwd_workspace_bytes.argtypes = [dp]
        L.monarch_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.monarch_materialise.argtypes = [vp, vp, dp, vp, vp]
        L.monarch_status_string.argtypes = [ctypes.c_int]
        L.monarch_status_string.restype = ctypes.c_char_p
        L.monarch_last_device_status.argtypes = [vp]
        L.monarch_debug_wait_timeout.argtypes = [ctypes.c_uint64, vp]
        L.monarch_bwd_noalloc.argtypes = [vp, vp, vp, vp, dp, vp, vp, vp, vp]
        L.monarch_fwd_path.argtypes = [dp]
        L.monarch_bwd_path.argtypes = [dp]
        L.monarch_fwd_workspace_bytes.argtypes = [dp]
        L.monarch_fwd_workspace_bytes.restype = ctypes.c_size_t
        L.monarch_fwd_ws_path.argtypes = [dp]
        L.monarch_fwd_ws_path.restype = ctypes.c_int
        L.monarch_fwd_ws.argtypes = [vp, vp, vp, dp, vp, vp, ctypes.c_size_t, vp]
        L.monarch_fwd_ws.restype = ctypes.c_int
        L.monarch_saved_bytes.argtypes = [dp]
        L.monarch_saved_bytes.restype = ctypes.c_size_t
        L.monarch_fwd_train.argtypes = [vp, vp, vp, dp, vp, vp, ctypes.c_size_t, vp]
        L.monarch_fwd_train.restype = ctypes.c_int
        L.monarch_bwd_saved.argtypes = [vp, vp, vp, vp, dp, vp, ctypes.c_size_t, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.monarch_bwd_saved.restype = ctypes.c_int
        L.monarch_kernel_launches.argtypes = []
        L.monarch_kernel_launches.restype = ctypes.c_uint64
        lp = ctypes.POINTER(MonarchLinearDims)
        L.monarch_linear_shape.argtypes = [lp, dp]
        L.monarch_linear_shape.restype = ctypes.c_int
        L.monarch_linear_workspace_bytes.argtypes = [lp]
        L.monarch_linear_workspace_bytes.restype = ctypes.c_size_t
        L.monarch_linear_fwd.argtypes = [vp, vp, vp, vp, lp, vp, vp, ctypes.c_size_t, vp]
        L.monarch_linear_fwd.restype = ctypes.c_int
        L.monarch_linear_bwd.argtypes = [vp, vp, vp, vp, lp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.monarch_linear_bwd.restype = ctypes.c_int
        L.monarch_project.argtypes = [vp, dp, vp, vp, vp]
        L.monarch_project.restype = ctypes.c_int
        yp = ctypes.POINTER(MonarchDyadDims)
        L.monarch_dyad_workspace_bytes.argtypes = [yp]
        L.monarch_dyad_workspace_bytes.restype = ctypes.c_size_t
        L.monarch_dyad_path.argtypes = [yp]
        L.monarch_dyad_path.restype = ctypes.c_int
        L.monarch_dyad_fwd.argtypes = [vp, vp, vp, yp, vp, vp, ctypes.c_size_t, vp]
        L.monarch_dyad_fwd.restype = ctypes.c_int
        L.monarch_dyad_bwd.argtypes = [vp, vp, vp, vp, yp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.monarch_dyad_bwd.restype = ctypes.c_int
        tp = ctypes.POINTER(MonarchLatticeDims)
        pp = ctypes.POINTER(ctypes.c_void_p)
        L.monarch_lattice_workspace_bytes.argtypes = [tp]
        L.monarch_lattice_workspace_bytes.restype = ctypes.c_size_t
        L.monarch_lattice_path.argtypes = [tp]
        L.monarch_lattice_path.restype = ctypes.c_int
        L.monarch_lattice_weight_elems.argtypes = [tp, ctypes.c_int32]
        L.monarch_lattice_weight_elems.restype = ctypes.c_int64
        L.monarch_lattice_fwd.argtypes = [vp, pp, tp, vp, vp, ctypes.c_size_t, vp]
        L.monarch_lattice_fwd.restype = ctypes.c_int
        L.monarch_lattice_bwd.argtypes = [vp, vp, pp, tp, vp, pp, vp, ctypes.c_size_t, vp]
        L.monarch_lattice_bwd.restype = ctypes.c_int
        for name in ("monarch_validate", "monarch_fwd", "monarch_bwd", "monarch_materialise",
                     "monarch_last_device_status", "monarch_debug_wait_timeout",
                     "monarch_fwd_path", "monarch_bwd_path", "monarch_bwd_noalloc"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def make_dims(shape: dict, rows: int, dtype) -> MonarchDims:
    """Build a ``monarch_dims`` from a shape dict (nb1, in1, out1, nb2, in2, out2,
    out_transpose), a row count and a dtype ('bf16' / 'f32' / torch dtype / code)."""
    return MonarchDims(
        int(rows), int(shape["nb1"]), int(shape["in1"]), int(shape["out1"]), int(shape["nb2"]),
        int(shape["in2"]), int(shape["out2"]), int(shape.get("out_transpose", 1)),
        dtype_code(dtype),
    )


def dtype_code(dtype) -> int:
    if isinstance(dtype, int):
        return dtype
    if isinstance(dtype, str):
        return {"bf16": MONARCH_BF16, "f32": MONARCH_F32, "fp32": MONARCH_F32}[dtype]
    import torch
    return {torch.bfloat16: MONARCH_BF16, torch.float32: MONARCH_F32}[dtype]


def _torch_dtype(code: int):
    import torch
    return torch.bfloat16 if code == MONARCH_BF16 else torch.float32


def _check(fn: str, rc: int):
    if rc != 0:
        raise MonarchError(fn, rc)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_tensors(shape: dict, rows: int, dtype, **ts):
    """Shapes and dtypes of the tensor arguments against the Monarch dims (raises ValueError)."""
    n_in = shape["nb1"] * shape["in1"]
    n_out = shape["nb2"] * shape["out2"]
    want = {
        "X": (rows, n_in), "dX": (rows, n_in), "Y": (rows, n_out), "dY": (rows, n_out),
        "R": (shape["nb1"], shape["out1"], shape["in1"]), "dR": (shape["nb1"], shape["out1"], shape["in1"]),
        "L": (shape["nb2"], shape["out2"], shape["in2"]), "dL": (shape["nb2"], shape["out2"], shape["in2"]),
    }
    for name, t in ts.items():
        if t is None:
            continue
        if tuple(t.shape) != want[name]:
            raise ValueError("%s has shape %s, the dims need %s" % (name, tuple(t.shape), want[name]))
        if t.dtype != dtype:
            raise ValueError("%s is %s, X is %s: every tensor must have one dtype" % (name, t.dtype, dtype))


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("Monarch kernels take contiguous CUDA tensors")


def validate(shape: dict, rows: int = 0, dtype="bf16") -> int:
    """Host-only shape check; returns the status code (0 = valid)."""
    return lib().monarch_validate(ctypes.byref(make_dims(shape, rows, dtype)))


def fwd_path(shape: dict, dtype="bf16") -> int:
    """Forward kernel family (host-only query): 0 generic FMA, 1 tcgen05 (row tile x block
    group), 2 tcgen05 row tile, 3 tcgen05 row tile with the L stage in output-column rounds,
    4 tcgen05 block-diagonal GEMM and row-permutation passes (64 x 64 blocks)."""
    return lib().monarch_fwd_path(ctypes.byref(make_dims(shape, 1, dtype)))


def bwd_path(shape: dict, dtype="bf16") -> int:
    """Backward kernel family (host-only query): 0 generic FMA, 1 tensor-core kernels."""
    return lib().monarch_bwd_path(ctypes.byref(make_dims(shape, 1, dtype)))


def bwd_workspace_bytes(shape: dict, rows: int, dtype="bf16") -> int:
    return int(lib().monarch_bwd_workspace_bytes(ctypes.byref(make_dims(shape, rows, dtype))))


def fwd(X, R, L, shape: dict, Y=None, stream=None):
    """Y = X M^T on the GPU.  X: (rows, nb1*in1); returns Y (rows, nb2*out2)."""
    import torch
    code = dtype_code(X.dtype)
    n_out = shape["nb2"] * shape["out2"]
    rows = X.shape[0]
    _check_tensors(shape, rows, X.dtype, X=X, R=R, L=L, Y=Y)
    if Y is None:
        Y = torch.empty((rows, n_out), dtype=X.dtype, device=X.device)
    _require_cuda(X, R, L, Y)
    d = make_dims(shape, rows, code)
    _check("monarch_fwd", lib().monarch_fwd(_ptr(X), _ptr(R), _ptr(L), ctypes.byref(d), _ptr(Y),
                                            _stream(stream)))
    return Y


def fwd_workspace_bytes(shape: dict, rows: int, dtype="bf16") -> int:
    return int(lib().monarch_fwd_workspace_bytes(ctypes.byref(make_dims(shape, rows, dtype))))


def fwd_ws_path(shape: dict, dtype="bf16") -> int:
    """Kernel family of monarch_fwd_ws: 5 = two-pass tcgen05 GEMM forward, else fwd_path's."""
    return lib().monarch_fwd_ws_path(ctypes.byref(make_dims(shape, 1, dtype)))


def fwd_ws(X, R, L, shape: dict, Y=None, workspace=None, stream=None):
    """Y = X M^T on the GPU with caller scratch (monarch_fwd_ws); same results as fwd()."""
    import torch
    code = dtype_code(X.dtype)
    rows = X.shape[0]
    _check_tensors(shape, rows, X.dtype, X=X, R=R, L=L, Y=Y)
    if Y is None:
        Y = torch.empty((rows, shape["nb2"] * shape["out2"]), dtype=X.dtype, device=X.device)
    d = make_dims(shape, rows, code)
    need = int(lib().monarch_fwd_workspace_bytes(ctypes.byref(d)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    _require_cuda(X, R, L, Y, workspace)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("monarch_fwd_ws", lib().monarch_fwd_ws(_ptr(X), _ptr(R), _ptr(L), ctypes.byref(d), _ptr(Y),
                                                  _ptr(workspace), ctypes.c_size_t(nbytes), _stream(stream)))
    return Y


def saved_bytes(shape: dict, rows: int, dtype="bf16") -> int:
    """Bytes of the buffer monarch_fwd_train fills for monarch_bwd_saved (0: nothing is saved)."""
    return int(lib().monarch_saved_bytes(ctypes.byref(make_dims(shape, rows, dtype))))


def fwd_train(X, R, L, shape: dict, Y=None, saved=None, stream=None):
    """Training forward (monarch_fwd_train): returns (Y, saved); pass `saved` to bwd_saved."""
    import torch
    code = dtype_code(X.dtype)
    rows = X.shape[0]
    _check_tensors(shape, rows, X.dtype, X=X, R=R, L=L, Y=Y)
    if Y is None:
        Y = torch.empty((rows, shape["nb2"] * shape["out2"]), dtype=X.dtype, device=X.device)
    d = make_dims(shape, rows, code)
    need = int(lib().monarch_saved_bytes(ctypes.byref(d)))
    if saved is None and need > 0:
        saved = torch.empty(need, dtype=torch.uint8, device=X.device)
    _require_cuda(X, R, L, Y, saved)
    nbytes = 0 if saved is None else saved.numel() * saved.element_size()
    _check("monarch_fwd_train", lib().monarch_fwd_train(_ptr(X), _ptr(R), _ptr(L), ctypes.byref(d), _ptr(Y),
                                                        _ptr(saved), ctypes.c_size_t(nbytes), _stream(stream)))
    return Y, saved


def bwd_saved(dY, X, R, L, shape: dict, saved, dX=None, dR=None, dL=None, workspace=None, stream=None):
    """(dX, dR, dL) like bwd(), reusing the middle vector fwd_train saved (monarch_bwd_saved)."""
    import torch
    code = dtype_code(X.dtype)
    rows = X.shape[0]
    _check_tensors(shape, rows, X.dtype, dY=dY, X=X, R=R, L=L, dX=dX, dR=dR, dL=dL)
    if dX is None:
        dX = torch.empty_like(X)
    if dR is None:
        dR = torch.empty_like(R)
    if dL is None:
        dL = torch.empty_like(L)
    d = make_dims(shape, rows, code)
    need = int(lib().monarch_bwd_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _require_cuda(dY, X, R, L, dX, dR, dL, workspace, saved)
    sbytes = 0 if saved is None else saved.numel() * saved.element_size()
    _check("monarch_bwd_saved",
           lib().monarch_bwd_saved(_ptr(dY), _ptr(X), _ptr(R), _ptr(L), ctypes.byref(d), _ptr(saved),
                                   ctypes.c_size_t(sbytes), _ptr(dX), _ptr(dR), _ptr(dL), _ptr(workspace),
                                   ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))
    return dX, dR, dL


def bwd(dY, X, R, L, shape: dict, dX=None, dR=None, dL=None, workspace=None, stream=None):
    """(dX, dR, dL) of Y = X M^T for upstream gradient dY, on the GPU."""
    import torch
    code = dtype_code(X.dtype)
    rows = X.shape[0]
    _check_tensors(shape, rows, X.dtype, dY=dY, X=X, R=R, L=L, dX=dX, dR=dR, dL=dL)
    if dX is None:
        dX = torch.empty_like(X)
    if dR is None:
        dR = torch.empty_like(R)
    if dL is None:
        dL = torch.empty_like(L)
    d = make_dims(shape, rows, code)
    need = int(lib().monarch_bwd_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _require_cuda(dY, X, R, L, dX, dR, dL, workspace)
    _check("monarch_bwd", lib().monarch_bwd(
        _ptr(dY), _ptr(X), _ptr(R), _ptr(L), ctypes.byref(d), _ptr(dX), _ptr(dR), _ptr(dL),
        _ptr(workspace), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
        _stream(stream)))
    return dX, dR, dL


def bwd_noalloc(dY, X, R, L, shape: dict, dX=None, dR=None, dL=None, stream=None):
    """Backward without a workspace argument, for callers that cannot allocate device
    memory: the library's own fixed 32 MiB device scratch is used instead (problems
    needing more raise MonarchError with MONARCH_ERR_SCRATCH).  Calls that overlap on
    the GPU share that scratch and must not run concurrently."""
    import torch
    code = dtype_code(X.dtype)
    _check_tensors(shape, X.shape[0], X.dtype, dY=dY, X=X, R=R, L=L, dX=dX, dR=dR, dL=dL)
    if dX is None:
        dX = torch.empty_like(X)
    if dR is None:
        dR = torch.empty_like(R)
    if dL is None:
        dL = torch.empty_like(L)
    _require_cuda(dY, X, R, L, dX, dR, dL)
    d = make_dims(shape, X.shape[0], code)
    _check("monarch_bwd_noalloc", lib().monarch_bwd_noalloc(
        _ptr(dY), _ptr(X), _ptr(R), _ptr(L), ctypes.byref(d), _ptr(dX), _ptr(dR), _ptr(dL),
        _stream(stream)))
    return dX, dR, dL


def materialise(R, L, shape: dict, M=None, stream=None):
    """Dense M (n_out, n_in) as float32 with Y = X M^T."""
    import torch
    code = dtype_code(R.dtype)
    _check_tensors(shape, 0, R.dtype, R=R, L=L)
    n_in = shape["nb1"] * shape["in1"]
    n_out = shape["nb2"] * shape["out2"]
    if M is None:
        M = torch.empty((n_out, n_in), dtype=torch.float32, device=R.device)
    _require_cuda(R, L, M)
    d = make_dims(shape, 0, code)
    _check("monarch_materialise", lib().monarch_materialise(_ptr(R), _ptr(L), ctypes.byref(d),
                                                            _ptr(M), _stream(stream)))
    return M


def project(M, shape: dict, dtype="f32", R=None, L=None, stream=None):
    """(R, L) of the Monarch matrix nearest to the dense float32 M (n_out, n_in), on the GPU."""
    import torch
    code = dtype_code(dtype)
    n_in = shape["nb1"] * shape["in1"]
    n_out = shape["nb2"] * shape["out2"]
    if tuple(M.shape) != (n_out, n_in) or M.dtype != torch.float32:
        raise ValueError("M must be float32 of shape %s" % ((n_out, n_in),))
    dt = _torch_dtype(code)
    if R is None:
        R = torch.empty((shape["nb1"], shape["out1"], shape["in1"]), dtype=dt, device=M.device)
    if L is None:
        L = torch.empty((shape["nb2"], shape["out2"], shape["in2"]), dtype=dt, device=M.device)
    _check_tensors(shape, 0, dt, R=R, L=L)
    _require_cuda(M, R, L)
    d = make_dims(shape, 0, code)
    _check("monarch_project", lib().monarch_project(_ptr(M), ctypes.byref(d), _ptr(R), _ptr(L),
                                                    _stream(stream)))
    return R, L


def last_device_status(stream=None) -> int:
    """Synchronise the stream and return/clear the device status word."""
    return lib().monarch_last_device_status(_stream(stream))


def debug_wait_timeout(timeout_ns: int, stream=None) -> int:
    return lib().monarch_debug_wait_timeout(ctypes.c_uint64(int(timeout_ns)), _stream(stream))


# ---------------------------------------------------------------- MonarchLinear front end
def linear_dims(in_features: int, out_features: int, nblocks: int, rows: int, dtype="bf16",
                bias: bool = False) -> MonarchLinearDims:
    return MonarchLinearDims(int(rows), int(in_features), int(out_features), int(nblocks), int(bool(bias)),
                             dtype_code(dtype))


def linear_shape(in_features: int, out_features: int, nblocks: int, dtype="bf16") -> dict:
    """Monarch shape (nb1, in1, out1, nb2, in2, out2, out_transpose) of
    MonarchLinear(in_features, out_features, nblocks), computed by the library."""
    d = MonarchDims()
    ld = linear_dims(in_features, out_features, nblocks, 0, dtype)
    _check("monarch_linear_shape", lib().monarch_linear_shape(ctypes.byref(ld), ctypes.byref(d)))
    return dict(nb1=d.nb1, in1=d.in1, out1=d.out1, nb2=d.nb2, in2=d.in2, out2=d.out2,
                out_transpose=d.out_transpose)


def linear_workspace_bytes(in_features: int, out_features: int, nblocks: int, rows: int, dtype="bf16",
                           bias: bool = False) -> int:
    ld = linear_dims(in_features, out_features, nblocks, rows, dtype, bias)
    return int(lib().monarch_linear_workspace_bytes(ctypes.byref(ld)))


def _linear_check(X, R, L, shape, in_features, out_features, **ts):
    rows = X.shape[0] if X is not None else ts["dY"].shape[0]
    want = {"X": (rows, in_features), "dX": (rows, in_features), "Y": (rows, out_features),
            "dY": (rows, out_features), "bias": (out_features,), "dbias": (out_features,),
            "R": (shape["nb1"], shape["out1"], shape["in1"]), "dR": (shape["nb1"], shape["out1"], shape["in1"]),
            "L": (shape["nb2"], shape["out2"], shape["in2"]), "dL": (shape["nb2"], shape["out2"], shape["in2"])}
    for name, t in dict(ts, X=X, R=R, L=L).items():
        if t is None:
            continue
        if tuple(t.shape) != want[name]:
            raise ValueError("%s has shape %s, MonarchLinear needs %s" % (name, tuple(t.shape), want[name]))
        if t.dtype != X.dtype:
            raise ValueError("%s is %s, X is %s: every tensor must have one dtype" % (name, t.dtype, X.dtype))


def linear_fwd(X, R, L, in_features: int, out_features: int, nblocks: int, bias=None, Y=None, workspace=None,
               stream=None):
    """MonarchLinear forward on the GPU: Y = crop(Monarch(pad(X))) + bias."""
    import torch
    rows = X.shape[0]
    shape = linear_shape(in_features, out_features, nblocks, X.dtype)
    _linear_check(X, R, L, shape, in_features, out_features, bias=bias, Y=Y)
    if Y is None:
        Y = torch.empty((rows, out_features), dtype=X.dtype, device=X.device)
    ld = linear_dims(in_features, out_features, nblocks, rows, X.dtype, bias is not None)
    need = int(lib().monarch_linear_workspace_bytes(ctypes.byref(ld)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _require_cuda(X, R, L, bias, Y, workspace)
    _check("monarch_linear_fwd", lib().monarch_linear_fwd(
        _ptr(X), _ptr(R), _ptr(L), _ptr(bias), ctypes.byref(ld), _ptr(Y), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))
    return Y


def linear_bwd(dY, X, R, L, in_features: int, out_features: int, nblocks: int, bias: bool = False, dX=None,
               dR=None, dL=None, dbias=None, workspace=None, stream=None):
    """MonarchLinear backward on the GPU: (dX, dR, dL, dbias); dbias is None without a bias."""
    import torch
    rows = X.shape[0]
    shape = linear_shape(in_features, out_features, nblocks, X.dtype)
    _linear_check(X, R, L, shape, in_features, out_features, dY=dY, dX=dX, dR=dR, dL=dL, dbias=dbias)
    dX = torch.empty_like(X) if dX is None else dX
    dR = torch.empty_like(R) if dR is None else dR
    dL = torch.empty_like(L) if dL is None else dL
    if bias and dbias is None:
        dbias = torch.empty((out_features,), dtype=X.dtype, device=X.device)
    ld = linear_dims(in_features, out_features, nblocks, rows, X.dtype, bias)
    need = int(lib().monarch_linear_workspace_bytes(ctypes.byref(ld)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _require_cuda(dY, X, R, L, dX, dR, dL, dbias, workspace)
    _check("monarch_linear_bwd", lib().monarch_linear_bwd(
        _ptr(dY), _ptr(X), _ptr(R), _ptr(L), ctypes.byref(ld), _ptr(dX), _ptr(dR), _ptr(dL),
        _ptr(dbias if bias else None), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))
    return dX, dR, dL, (dbias if bias else None)


# ---------------------------------------------------------------- DYAD
def dyad_dims(nblocks: int, in_blk: int, out_blk: int, rows: int, dtype="bf16") -> MonarchDyadDims:
    return MonarchDyadDims(int(rows), int(nblocks), int(in_blk), int(out_blk), dtype_code(dtype))


def dyad_path(nblocks: int, in_blk: int, out_blk: int, dtype="bf16") -> int:
    """1 = tcgen05 path, 0 = generic FMA kernels (host-only query)."""
    return lib().monarch_dyad_path(ctypes.byref(dyad_dims(nblocks, in_blk, out_blk, 1, dtype)))


def _dyad_check(W1, W2, rows, **ts):
    nb, ob, ib = W1.shape
    want = {"X": (rows, nb * ib), "dX": (rows, nb * ib), "Y": (rows, nb * ob), "dY": (rows, nb * ob),
            "W1": (nb, ob, ib), "W2": (nb, ob, ib), "dW1": (nb, ob, ib), "dW2": (nb, ob, ib)}
    for name, t in dict(ts, W1=W1, W2=W2).items():
        if t is None:
            continue
        if tuple(t.shape) != want[name]:
            raise ValueError("%s has shape %s, DYAD needs %s" % (name, tuple(t.shape), want[name]))
        if t.dtype != W1.dtype:
            raise ValueError("%s is %s, W1 is %s: every tensor must have one dtype" % (name, t.dtype, W1.dtype))


def dyad_fwd(X, W1, W2, Y=None, workspace=None, stream=None):
    """DYAD forward on the GPU: Y = BD(W1) x + P_out^T BD(W2) P_in x for every row x."""
    import torch
    nb, ob, ib = W1.shape
    rows = X.shape[0]
    _dyad_check(W1, W2, rows, X=X, Y=Y)
    if Y is None:
        Y = torch.empty((rows, nb * ob), dtype=X.dtype, device=X.device)
    dd = dyad_dims(nb, ib, ob, rows, X.dtype)
    need = int(lib().monarch_dyad_workspace_bytes(ctypes.byref(dd)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _require_cuda(X, W1, W2, Y, workspace)
    _check("monarch_dyad_fwd", lib().monarch_dyad_fwd(
        _ptr(X), _ptr(W1), _ptr(W2), ctypes.byref(dd), _ptr(Y), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))
    return Y


def dyad_bwd(dY, X, W1, W2, dX=None, dW1=None, dW2=None, workspace=None, stream=None):
    """DYAD backward on the GPU: (dX, dW1, dW2)."""
    import torch
    nb, ob, ib = W1.shape
    rows = X.shape[0]
    _dyad_check(W1, W2, rows, dY=dY, X=X, dX=dX, dW1=dW1, dW2=dW2)
    dX = torch.empty_like(X) if dX is None else dX
    dW1 = torch.empty_like(W1) if dW1 is None else dW1
    dW2 = torch.empty_like(W2) if dW2 is None else dW2
    dd = dyad_dims(nb, ib, ob, rows, X.dtype)
    need = int(lib().monarch_dyad_workspace_bytes(ctypes.byref(dd)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _require_cuda(dY, X, W1, W2, dX, dW1, dW2, workspace)
    _check("monarch_dyad_bwd", lib().monarch_dyad_bwd(
        _ptr(dY), _ptr(X), _ptr(W1), _ptr(W2), ctypes.byref(dd), _ptr(dX), _ptr(dW1), _ptr(dW2), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))
    return dX, dW1, dW2


# ---------------------------------------------------------------- lattice (hypercube) Monarch
def lattice_dims(n_in, n_out, rows: int, dtype="bf16") -> MonarchLatticeDims:
    if not 1 <= len(n_in) == len(n_out) <= 4:
        raise ValueError("1 to 4 axes, n_in and n_out of one length")
    d = MonarchLatticeDims()
    d.rows, d.naxes, d.dtype = int(rows), len(n_in), dtype_code(dtype)
    for a, (ni, no) in enumerate(zip(n_in, n_out)):
        d.n_in[a], d.n_out[a] = int(ni), int(no)
    return d


def lattice_weight_shapes(n_in, n_out) -> list:
    """(lines, n_out[t], n_in[t]) of every axis t, from the library's host-side rule."""
    d = lattice_dims(n_in, n_out, 0, "f32")
    out = []
    for t in range(len(n_in)):
        n = int(lib().monarch_lattice_weight_elems(ctypes.byref(d), t))
        out.append((n // (n_out[t] * n_in[t]), n_out[t], n_in[t]))
    return out


def lattice_path(n_in, n_out, dtype="bf16") -> int:
    return lib().monarch_lattice_path(ctypes.byref(lattice_dims(n_in, n_out, 1, dtype)))


def _ptr_array(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() for t in ts])


def lattice_fwd(X, Ws, n_in, n_out, Y=None, workspace=None, stream=None):
    """Lattice Monarch forward on the GPU; Ws[t] is the weight tensor of axis t."""
    import torch
    rows = X.shape[0]
    if Y is None:
        Y = torch.empty((rows, int(np.prod(n_out))), dtype=X.dtype, device=X.device)
    d = lattice_dims(n_in, n_out, rows, X.dtype)
    need = int(lib().monarch_lattice_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _require_cuda(X, Y, workspace, *Ws)
    _check("monarch_lattice_fwd", lib().monarch_lattice_fwd(
        _ptr(X), _ptr_array(Ws), ctypes.byref(d), _ptr(Y), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))
    return Y


def lattice_bwd(dY, X, Ws, n_in, n_out, workspace=None, stream=None):
    """Lattice Monarch backward on the GPU: (dX, [dW_t])."""
    import torch
    rows = X.shape[0]
    dX = torch.empty_like(X)
    dWs = [torch.empty_like(w) for w in Ws]
    d = lattice_dims(n_in, n_out, rows, X.dtype)
    need = int(lib().monarch_lattice_workspace_bytes(ctypes.byref(d)))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _require_cuda(dY, X, dX, workspace, *Ws, *dWs)
    _check("monarch_lattice_bwd", lib().monarch_lattice_bwd(
        _ptr(dY), _ptr(X), _ptr_array(Ws), ctypes.byref(d), _ptr(dX), _ptr_array(dWs), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)))
    return dX, dWs


def kernel_launches() -> int:
    """Kernels the library has launched in this process (host-side count)."""
    return int(lib().monarch_kernel_launches())


def status_string(code: int) -> str:
    return lib().monarch_status_string(int(code)).decode()
