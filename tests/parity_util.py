"""Shared helpers for the GPU parity tests: move workload tensors to the device,
hand the same inputs to the oracle, compare results."""
import numpy as np
import torch

import oracle
from workloads import bf16_bits

# max_{m,n} |Y - Y_ref| / ||Y_ref[m, :]||_2 for the floating-point products
REL_ROW_TOL = 2e-3


def oracle_input(W: torch.Tensor):
    """(array, dtype tag) of a CPU tensor in the form the oracle takes."""
    if W.dtype == torch.float32:
        return W.contiguous().numpy(), None
    if W.dtype == torch.bfloat16:
        return bf16_bits(W), oracle.BF16
    if W.dtype == torch.float16:
        return W.contiguous().view(torch.int16).numpy().view(np.uint16), oracle.F16
    raise TypeError(W.dtype)


def u16(t: torch.Tensor) -> np.ndarray:
    """uint16 bit pattern of a 16-bit float tensor (any device)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def rel_row_error(Y: np.ndarray, Yref: np.ndarray) -> float:
    Y = np.asarray(Y, np.float64)
    norms = np.linalg.norm(Yref, axis=1)
    norms = np.where(norms == 0, 1.0, norms)
    return float((np.abs(Y - Yref).max(axis=1) / norms).max())
