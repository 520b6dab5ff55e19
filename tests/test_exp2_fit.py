"""CPU: the coefficients of the FMA-pipe exponential in csrc/common.cuh are the
ones the committed fit produces, and its float32 Horner form stays within the
bound stated beside it (relative error <= 2.2e-7 on [-1/2, 1/2], about two
float32 ulps, the accuracy class of the MUFU's ex2.approx)."""
import os
import re

import numpy as np

from schnet_gnn_molecular_b200 import exp2_fit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _device_coefficients():
    src = open(os.path.join(ROOT, "schnet_gnn_molecular_b200", "csrc", "common.cuh")).read()
    body = src[src.index("float2 ex2_fma2(float2 x)"):src.index("float2 sp2x2_fma(float2 p)")]
    lits = [float(x) for x in re.findall(r"dup2\(([0-9.]+)f\)", body)]
    # Horner order in the source: c5, c4, c3, c2, c1, c0
    return np.array(lits[::-1], dtype=np.float32)


def test_device_coefficients_are_the_fit():
    c = exp2_fit.fit()
    assert np.array_equal(_device_coefficients(), c)


def test_fit_error_bound():
    c = exp2_fit.fit()
    assert exp2_fit.max_rel_error(c) <= 2.2e-7
    # the reduction's exactness: 2^f at the interval ends and at 0
    for f, want in [(0.0, 1.0), (-0.5, 2 ** -0.5), (0.5, 2 ** 0.5)]:
        got = float(exp2_fit.horner_f32(c, np.array([f]))[0])
        assert abs(got / want - 1) <= 2.2e-7
