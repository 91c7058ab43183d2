"""The FMA-pipe exp2 coefficients in ptx_sm100.cuh are the ones fit_exp2_poly.py produces,
and the fit meets its stated bound (host-side; the device evaluation is tested on the GPU
in test_gpu_exp2_poly.py)."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_io_aware_81_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_header_coefficients_match_the_fit():
    src = open(os.path.join(CSRC, "ptx_sm100.cuh")).read()
    line = re.search(r"constexpr float (c1 = [^;]*);", src).group(1)
    coeffs = [float(v.rstrip("f")) for v in re.findall(r"c\d = ([0-9.e+-]+f)", line)]
    c, err = _fit_module().fit(len(coeffs))
    assert np.array_equal(np.float32(coeffs), np.float32(c)), (coeffs, c)
    assert err < 3e-6


def test_fit_reaches_taylor_limit_without_it():
    # an independent check of the fit: the Lawson minimax polynomial must beat the
    # degree-4 Taylor polynomial of 2^f by a wide margin on [-1/2, 1/2]
    f = np.linspace(-0.5, 0.5, 10001)
    ln2 = np.log(2.0)
    taylor = sum((ln2 * f) ** k / np.prod(np.arange(1, k + 1)) for k in range(0, 5))
    taylor_err = np.max(np.abs(taylor / np.exp2(f) - 1))
    _, err = _fit_module().fit(4)
    assert err < taylor_err / 5
