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


def rel_row_error(Y: np.ndarray, Yref: np.ndarray, rounding_aware: bool = False) -> float:
    """max_{m,n} |Y - Y_ref| / ||Y_ref[m, :]||_2.

    With rounding_aware, each element's error is first reduced by half a bf16
    ulp of Y_ref (the rounding of the bf16 output itself, up to 2^-8 of the
    value): with very few outputs per row one element carries most of the row
    norm and the output rounding alone can exceed the row-normalised bound.
    The workloads' full-size checks use the plain bound."""
    Y = np.asarray(Y, np.float64)
    err = np.abs(Y - Yref)
    if rounding_aware:
        mag = np.abs(Yref)
        e = np.floor(np.log2(np.where(mag > 0, mag, 1.0)))
        half_ulp = np.where(mag > 0, np.exp2(e - 8), 0.0)
        err = np.maximum(err - half_ulp, 0.0)
    norms = np.linalg.norm(Yref, axis=1)
    norms = np.where(norms == 0, 1.0, norms)
    return float((err.max(axis=1) / norms).max())
