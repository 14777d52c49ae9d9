"""Seeded synthetic inputs and the named Monarch workload shapes.

This module serves both the CUDA path (tests, benchmark) and the fp64 oracle,
so it holds none of the method's arithmetic: only shapes, random draws and the
rounding of those draws to the storage dtype.

Recipe (one ``numpy.random.default_rng(seed)`` per call, draws in this order):
  X  ~ N(0, 1)                    shape (rows, n_in)
  R  ~ U(-1/sqrt(in1), 1/sqrt(in1))  shape (nb1, out1, in1)
  L  ~ U(-1/sqrt(in2), 1/sqrt(in2))  shape (nb2, out2, in2)
  dY ~ N(0, 1)                    shape (rows, n_out)
Each draw is made in float64, cast to float32, and for bf16 workloads rounded
to bfloat16 with round-to-nearest-even.  The float64 widening of the stored
values is what the oracle sees, so both sides start from identical numbers.
"""
from __future__ import annotations

import numpy as np

# Workload shapes. Factor tensors are (nblocks, out_blk, in_blk); X is
# (rows, nb1*in1); Y is (rows, nb2*out2); out_transpose=1 writes v[j][o] at
# y[o*nb2 + j] (the final transpose-and-flatten), 0 at y[j*out2 + o].
WORKLOADS = {
    # square n = 256 = 16^2, fp32, 64 rows
    "n256_fp32": dict(nb1=16, in1=16, out1=16, nb2=16, in2=16, out2=16, out_transpose=1,
                      rows=64, dtype="f32"),
    # square n = 1024 = 32^2, bf16, 16384 rows
    "n1024_bf16": dict(nb1=32, in1=32, out1=32, nb2=32, in2=32, out2=32, out_transpose=1,
                       rows=16384, dtype="bf16"),
    # 768 -> 3072 (GPT-2-small FFN up-projection), bf16, 8192 rows
    "r768x3072_bf16": dict(nb1=16, in1=48, out1=48, nb2=48, in2=16, out2=64, out_transpose=1,
                           rows=8192, dtype="bf16"),
    # square n = 4096 = 64^2 training step, bf16, 16384 rows
    "n4096_bf16": dict(nb1=64, in1=64, out1=64, nb2=64, in2=64, out2=64, out_transpose=1,
                       rows=16384, dtype="bf16"),
    # two-factor nblocks = 4 layer, 1024 -> 4096, bf16, 10000 (and 1000) rows
    "nblk4_1024x4096_bf16": dict(nb1=4, in1=256, out1=256, nb2=4, in2=256, out2=1024,
                                 out_transpose=0, rows=10000, dtype="bf16"),
    "nblk4_1024x4096_bf16_b1000": dict(nb1=4, in1=256, out1=256, nb2=4, in2=256, out2=1024,
                                       out_transpose=0, rows=1000, dtype="bf16"),
}

SHAPE_KEYS = ("nb1", "in1", "out1", "nb2", "in2", "out2", "out_transpose")


def shape_of(w: dict) -> dict:
    """The Monarch shape part of a workload (no rows / dtype)."""
    return {k: int(w[k]) for k in SHAPE_KEYS}


def sizes(w: dict) -> tuple[int, int, int]:
    return w["nb1"] * w["in1"], w["nb1"] * w["out1"], w["nb2"] * w["out2"]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest-even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    return ((b + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


class Tensor:
    """One synthetic tensor: its float64 values and its storage representation."""

    def __init__(self, values64: np.ndarray, dtype: str):
        f32 = values64.astype(np.float32)
        self.dtype = dtype
        if dtype == "bf16":
            self.bits = f32_to_bf16_bits(f32)
            self.f64 = bf16_bits_to_f64(self.bits)
        elif dtype == "f32":
            self.bits = f32
            self.f64 = f32.astype(np.float64)
        else:
            raise ValueError("dtype must be 'bf16' or 'f32', got %r" % (dtype,))

    @property
    def shape(self):
        return self.f64.shape


def make_inputs(w: dict, seed: int = 0, rows: int | None = None, dtype: str | None = None):
    """Seeded X, R, L, dY for a workload; returns a dict of :class:`Tensor`."""
    rows = int(w["rows"] if rows is None else rows)
    dtype = dtype or w["dtype"]
    n_in, _, n_out = sizes(w)
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((rows, n_in))
    bR = 1.0 / np.sqrt(w["in1"])
    R = rng.uniform(-bR, bR, size=(w["nb1"], w["out1"], w["in1"]))
    bL = 1.0 / np.sqrt(w["in2"])
    L = rng.uniform(-bL, bL, size=(w["nb2"], w["out2"], w["in2"]))
    dY = rng.standard_normal((rows, n_out))
    return {"X": Tensor(X, dtype), "R": Tensor(R, dtype), "L": Tensor(L, dtype),
            "dY": Tensor(dY, dtype)}


def make_integer_inputs(w: dict, seed: int = 0, rows: int | None = None, vmax: int = 4):
    """Small-integer inputs (|v| <= vmax, exact in bf16 and fp32) for exact-equality checks."""
    rows = int(w["rows"] if rows is None else rows)
    n_in, _, n_out = sizes(w)
    rng = np.random.default_rng(seed)
    X = rng.integers(-vmax, vmax + 1, size=(rows, n_in)).astype(np.float64)
    R = rng.integers(-vmax, vmax + 1, size=(w["nb1"], w["out1"], w["in1"])).astype(np.float64)
    L = rng.integers(-vmax, vmax + 1, size=(w["nb2"], w["out2"], w["in2"])).astype(np.float64)
    dY = rng.integers(-vmax, vmax + 1, size=(rows, n_out)).astype(np.float64)
    return {"X": X, "R": R, "L": L, "dY": dY}


def sparse_sign_blocks(rng, nb: int, out_b: int, in_b: int, nnz: int) -> np.ndarray:
    """(nb, out_b, in_b) blocks whose rows each hold `nnz` draws of +-1 at random columns
    (draws may land on the same column, giving 0 or +-2 there)."""
    W = np.zeros((nb, out_b, in_b), dtype=np.float64)
    for b in range(nb):
        for o in range(out_b):
            cols = rng.integers(0, in_b, size=nnz)
            signs = rng.choice([-1.0, 1.0], size=nnz)
            np.add.at(W[b, o], cols, signs)
    return W


def make_sparse_sign_inputs(w: dict, seed: int = 0, rows: int | None = None, nnz: int = 2):
    """Inputs for exact-equality checks: X and dY in {-1, 0, 1} (zero with probability 1/2),
    factor blocks from :func:`sparse_sign_blocks`.  Every row of a block has absolute sum
    <= nnz, so every intermediate of the method stays a small integer; float64 arrays."""
    rows = int(w["rows"] if rows is None else rows)
    n_in, _, n_out = sizes(w)
    rng = np.random.default_rng(seed)
    X = rng.choice([-1.0, 0.0, 0.0, 1.0], size=(rows, n_in))
    R = sparse_sign_blocks(rng, w["nb1"], w["out1"], w["in1"], nnz)
    L = sparse_sign_blocks(rng, w["nb2"], w["out2"], w["in2"], nnz)
    dY = rng.choice([-1.0, 0.0, 0.0, 1.0], size=(rows, n_out))
    return {"X": X, "R": R, "L": L, "dY": dY}
