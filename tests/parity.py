"""Parity rule between the CUDA path and the oracle.

Tolerance (per output element, S = sum |x*w| over its receptive field, from
the oracle):
  f16 / bf16 : |y - y_ref| <= 2e-3 * S + 1e-6
  f32        : |y - y_ref| <= 1e-5 * S + 1e-7
An element that misses the bound may still pass if it is within the same
bound of the oracle value correctly rounded to the output type (RN(y_ref)):
rounding the exact result to bfloat16 alone can cost 2^-9 |y|, which exceeds
2e-3 * S where |y| is close to S (border outputs with few in-range taps).
The count of elements that needed this second clause is reported.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {"f16": (2e-3, 1e-6), "bf16": (2e-3, 1e-6), "f32": (1e-5, 1e-7)}


def as_f64(y: torch.Tensor) -> np.ndarray:
    return y.detach().cpu().to(torch.float64).numpy()


def compare(y_gpu, y_ref, s_ref, dtype):
    """Returns (n_fail, n_second_clause, worst err/tol) over all elements."""
    y = as_f64(y_gpu) if isinstance(y_gpu, torch.Tensor) else np.asarray(y_gpu, np.float64)
    y = y.reshape(-1)
    y_ref = np.asarray(y_ref, np.float64).reshape(-1)
    s_ref = np.asarray(s_ref, np.float64).reshape(-1)
    if not (y.size == y_ref.size == s_ref.size):
        raise ValueError(f"element counts differ: result {y.size}, oracle {y_ref.size}, magnitudes {s_ref.size}")
    rel, ab = TOL[dtype]
    tol = rel * s_ref + ab
    err = np.abs(y - y_ref)
    bad = ~(err <= tol)            # NaN counts as bad
    n2 = 0
    if bad.any():
        idx = np.nonzero(bad)[0]
        rn = oracle.round_to(y_ref[idx], dtype)
        ok2 = np.abs(y[idx] - rn) <= tol[idx]
        n2 = int(ok2.sum())
        bad[idx[ok2]] = False
    worst = float(np.max(err / tol)) if err.size else 0.0
    return int(bad.sum()), n2, worst


def assert_parity(y_gpu, y_ref, s_ref, dtype, what=""):
    n_fail, n2, worst = compare(y_gpu, y_ref, s_ref, dtype)
    assert n_fail == 0, f"{what}: {n_fail} elements outside tolerance (worst err/tol {worst:.3g})"
    return n2, worst
