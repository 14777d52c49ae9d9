"""Shared helpers of the GPU tests: move synthetic tensors to the device and back."""
import numpy as np
import torch

from block_diagonal_linear_b200 import synthetic

TOL = {"f32": 1e-5, "bf16": 2e-2}   # normwise ||G - O||_F / ||O||_F per output tensor


def to_dev(t: synthetic.Tensor) -> torch.Tensor:
    if t.dtype == "bf16":
        return torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(t.bits)).cuda()


def to_f64(x: torch.Tensor) -> np.ndarray:
    return x.detach().float().cpu().numpy().astype(np.float64)


def dev_inputs(inp: dict) -> dict:
    return {k: to_dev(v) for k, v in inp.items()}
