"""The cubic 2^x the attention kernels evaluate on the FMA pipe: its constants
in csrc/common.cuh are the ones eviction_masked_attention_b200/fit_exp2_poly.py
derives, and its fp32 evaluation stays within 7.5e-5 relative error of 2^x over
the arguments the kernels use (scores minus the running maximum, which the lazy
rescale lets reach +8), 1.5e-4 at the clamp (results ~1e-38). The same figures
stand in the kernel header and the fit script."""
import os
import re

import numpy as np

from eviction_masked_attention_b200 import fit_exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _kernel_coeffs():
    """(c0, c1, c2, c3) as written in exp2_fma_x2, where each appears once per lane."""
    src = open(os.path.join(ROOT, "eviction_masked_attention_b200", "csrc", "common.cuh")).read()
    body = src[src.index("void exp2_fma_x2("):]
    body = body[: body.index("f2_split(t")]
    vals = [float(v) for v in re.findall(r"([0-9]\.[0-9]+e[+-][0-9]+)f", body)]
    assert len(vals) == 8 and vals[1::2] == vals[0::2]   # the same constant in both lanes
    c3, c2, c1, c0 = vals[0::2]
    return np.array([c0, c1, c2, c3])


def _eval_fp32(c, x):
    return fit_exp2_poly.eval_fp32(c, x)


def test_constants_match_fit():
    c, err = fit_exp2_poly.fit()
    np.testing.assert_allclose(_kernel_coeffs(), c, rtol=1e-8)
    assert err < 1e-4


BOUND = 7.5e-5        # x > -126
BOUND_CLAMP = 1.5e-4  # x <= -126


def _rel_err(c, x):
    x = np.asarray(x, dtype=np.float32)
    got = _eval_fp32(c, x).astype(np.float64)
    return np.abs(got / np.exp2(np.maximum(x, -126.0).astype(np.float64)) - 1.0)


def test_relative_error_on_reduced_interval():
    # the cubic's own interval, evaluated in float32 exactly as the kernels do
    c = _kernel_coeffs()
    assert _rel_err(c, np.linspace(-0.5, 0.5, 2_000_001)).max() < BOUND


def test_relative_error_over_kernel_range():
    c = _kernel_coeffs()
    x = np.concatenate([np.linspace(-125.999, 8.0, 1_000_001), -np.arange(0, 126), [0.5, -0.5, 7.999]])
    assert _rel_err(c, x).max() < BOUND
    # below the clamp the result stays 2^-126 (within 1.5e-4), never NaN or negative
    low = np.array([-126.0, -126.5, -127.0, -127.3, -200.0, -1e30], np.float32)
    assert _rel_err(c, low).max() < BOUND_CLAMP
    assert (_eval_fp32(c, low) > 0).all()
    # exact powers of two stay within the same bound
    assert abs(_eval_fp32(c, np.array([0.0]))[0] - 1.0) < BOUND

