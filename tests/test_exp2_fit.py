"""The cubic of the optional FMA-pipe exponential (csrc/ptx.cuh, exp2_poly_x2) is the output of
csrc/exp2_poly_fit.py: refitting here must reproduce the constants in the header, and the
float32 evaluation the kernel performs must stay within the stated error bound. CPU only."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "transformer_attention_04_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly_fit",
                                                  os.path.join(CSRC, "exp2_poly_fit.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _header_constants():
    text = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = text[text.index("uint64_t exp2_poly_x2"):]
    body = body[:body.index("\n}\n")]
    vals = [float(v) for v in re.findall(r"f2_pack\(([-0-9.e+]+)f,", body)]
    # the four Horner coefficients, highest degree first (c3, c2, c1, c0)
    coeffs = [v for v in vals if abs(v) < 2.0 and v not in (-1.0,)]
    return np.array(coeffs[::-1], dtype=np.float32)


def test_header_constants_are_the_fit():
    m = _fit_module()
    c32 = np.array(m.remez(), dtype=np.float32)
    h = _header_constants()
    assert h.shape == (4,)
    np.testing.assert_allclose(h, c32, rtol=2e-6, atol=0)


def test_float32_evaluation_error_bound():
    m = _fit_module()
    err = m.f32_eval_error(_header_constants())
    assert err < 1.5e-4, err  # far below bf16's half-ulp (2^-9 = 2e-3) that P is rounded to
