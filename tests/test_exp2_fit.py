"""The FMA-pipe exp2 polynomial: the committed header is what the fitting
script produces, and the fit meets its stated error bound (CPU)."""
import importlib.util
import os
import re

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "scaled_dot_product_13_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2", os.path.join(CSRC, "fit_exp2.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_header_matches_fit_script():
    mod = _fit_module()
    assert open(os.path.join(CSRC, "exp2_poly.h")).read() == mod.render()


def test_fit_is_minimax_and_below_half_precision_rounding():
    mod = _fit_module()
    c, E = mod.remez_relative()
    # equioscillation: the error curve reaches +-E at degree + 2 points
    f = np.linspace(-0.5, 0.5, 100001)
    err = np.polyval(c[::-1], f) / np.exp2(f) - 1.0
    assert abs(np.max(np.abs(err)) - E) < 1e-9
    e32 = mod.fp32_error(c.astype(np.float32))
    # below the rounding of P to fp16 (2^-11) and bf16 (2^-8) by a wide margin
    assert e32 < 2.0 ** -13
    # full range reconstruction 2^n * p(f) against numpy's exp2
    x = np.linspace(-100.0, 8.0, 20001)
    n = np.round(x)
    y = np.ldexp(np.polyval(c[::-1], x - n), n.astype(int))
    assert np.max(np.abs(y / np.exp2(x) - 1.0)) <= E * (1 + 1e-9)


@pytest.mark.gpu
def test_device_exp2_against_exp2f(cuda_lib):
    """The kernels' FMA-pipe exp2 against CUDA's exp2f on the softmax's input
    range (x <= 8 with the lazily moved max), within the fitted bound."""
    text = open(os.path.join(CSRC, "exp2_poly.h")).read()
    bound = float(re.search(r"kExp2PolyMaxRelErr = ([0-9.e+-]+)f", text).group(1))
    for lo, hi in ((-0.5, 0.5), (-30.0, 8.0), (-125.0, -100.0)):
        poly, ref = cuda_lib.exp2_selftest(lo, hi, 1 << 20)
        rel = ((poly.double() - ref.double()).abs() / ref.double()).max().item()
        # exp2f itself is within 2 ulp of 2^x
        assert rel <= bound + 2.5e-7, (lo, hi, rel)
    # far below the range P can hold the result is tiny (not wrapped around)
    poly, _ = cuda_lib.exp2_selftest(-1000.0, -127.0, 4096)
    assert bool((poly >= 0).all()) and poly.max().item() < 2.0 ** -120
