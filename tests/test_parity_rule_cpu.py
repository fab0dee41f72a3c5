"""The parity rule itself (tests/parity.py), on hand-made values: the checker
that every GPU parity test relies on must reject what it should."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from tests import parity


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
def test_bound_edges(dtype):
    rel, ab = parity.TOL[dtype]
    y_ref = np.array([0.25, -1.5, 0.0, 3.0])
    s_ref = np.array([1.0, 2.0, 0.5, 4.0])
    tol = rel * s_ref + ab
    assert parity.compare(y_ref.copy(), y_ref, s_ref, dtype)[:2] == (0, 0)
    # exactly on the bound passes; a hair beyond it fails (the values are chosen
    # so that the second clause cannot rescue it: y_ref is exactly representable)
    on = y_ref + tol * np.array([1, -1, 1, -1]) * (1 - 1e-9)
    assert parity.compare(on, y_ref, s_ref, dtype)[0] == 0
    off = y_ref.copy()
    off[1] -= 1.01 * tol[1]
    n_fail, n2, worst = parity.compare(off, y_ref, s_ref, dtype)
    assert (n_fail, n2) == (1, 0) and worst > 1.0
    with pytest.raises(AssertionError, match="1 elements outside tolerance"):
        parity.assert_parity(off, y_ref, s_ref, dtype, "planted")


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_non_finite_results_fail(bad):
    y_ref = np.array([1.0, 2.0])
    s_ref = np.array([1.0, 2.0])
    y = np.array([1.0, bad])
    assert parity.compare(y, y_ref, s_ref, "bf16")[0] == 1


def test_second_clause_accepts_only_the_correctly_rounded_value():
    # |y| close to S: rounding the exact value to bfloat16 costs more than the bound
    s_ref = np.array([1.0])
    tol = 2e-3 * 1.0 + 1e-6
    y_ref = np.array([1.0 + 2.0 ** -7 + 2.0 ** -11])   # rounds 4.9e-4 away: the first clause suffices
    rn = float(torch.tensor(y_ref).to(torch.bfloat16).double())
    assert parity.compare(np.array([rn]), y_ref, s_ref, "bf16")[:2] == (0, 0)
    y_ref2 = np.array([1.0 + 2.0 ** -8 + 2.0 ** -12])  # nearest bfloat16 is 1 + 2^-7, 3.7e-3 away
    rn2 = float(torch.tensor(y_ref2).to(torch.bfloat16).double())
    assert abs(rn2 - y_ref2[0]) > tol
    assert parity.compare(np.array([rn2]), y_ref2, s_ref, "bf16")[:2] == (0, 1)
    # the other neighbour (1 + 2^-8 rounded down: 1.0) is not the correctly rounded value
    assert parity.compare(np.array([1.0]), y_ref2, s_ref, "bf16")[0] == 1


def test_tensor_inputs_and_counts():
    y_ref = np.arange(12, dtype=np.float64).reshape(3, 4) / 8
    s_ref = np.ones((3, 4))
    y = torch.tensor(y_ref, dtype=torch.float16)
    assert parity.compare(y, y_ref, s_ref, "f16")[0] == 0
    with pytest.raises(ValueError, match="element counts differ"):
        parity.compare(torch.zeros(1, dtype=torch.float16), y_ref, s_ref, "f16")
    assert parity.compare(np.zeros(0), np.zeros(0), np.zeros(0), "f32") == (0, 0, 0.0)
