"""CPU check of the coefficients of the software exp2 the softmax uses for part of its
exponentials (Cody & Waite range reduction to f in [-1/2, 1/2] plus a cubic minimax
fit of 2^f): the cubic, evaluated by Horner in fp32 as the kernel does, stays within
the stated relative error bound of 7.5e-5 on the reduced interval, and the bound is
equioscillating (no systematic bias)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def coefficients():
    src = open(f"{ROOT}/block_sparse_online_b200/csrc/ptx_sm100.cuh").read()
    m = re.search(r"c0 = ([0-9.e-]+)f, c1 = ([0-9.e-]+)f;\s+constexpr float c2 = ([0-9.e-]+)f, c3 = ([0-9.e-]+)f;", src)
    return [np.float32(float(v)) for v in m.groups()]


def test_cubic_relative_error_bound():
    c0, c1, c2, c3 = coefficients()
    f = np.linspace(-0.5, 0.5, 2_000_001, dtype=np.float32)
    p = ((c3 * f + c2) * f + c1) * f + c0
    rel = (p.astype(np.float64) - np.exp2(f.astype(np.float64))) / np.exp2(f.astype(np.float64))
    assert np.abs(rel).max() <= 7.6e-5
    assert rel.max() > 5e-5 and rel.min() < -5e-5  # error alternates sign: minimax, not biased
