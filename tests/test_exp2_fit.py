"""The constants of the kernels' FMA-pipe exp2 against the committed fit that produces them
(host only: reads the CUDA source as text, runs the fit in numpy)."""
import os

import numpy as np


def test_exp2_polynomial_constants_come_from_the_committed_fit():
    """The coefficients compiled into the kernels' FMA-pipe exp2 are what the committed Remez
    fit (csrc/fit_exp2_poly.py) produces, rounded to fp32 -- not constants from elsewhere."""
    import importlib.util
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    csrc = os.path.join(root, "attention_kl_divergence_02_b200", "csrc")
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(csrc, "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c = [np.float32(v) for v in fit.remez_exp2(4)]
    src = open(os.path.join(csrc, "sm100.cuh")).read()
    body = src[src.index("float2 ex2_poly2(float2 u)"):]
    body = body[:body.index("return make_float2")]
    lits = [np.float32(float(v)) for v in re.findall(r"([0-9]\.[0-9]+e[-+][0-9]+)f", body)]
    # Horner from the highest coefficient: c4, c3 (one make_float2 pair each), then c2, c1, c0
    uniq = []
    for v in lits:
        if not uniq or uniq[-1] != v:
            uniq.append(v)
    assert uniq == [c[4], c[3], c[2], c[1], c[0]], (uniq, c)
    f = np.linspace(-0.5, 0.5, 200001)
    assert np.abs(fit.fp32_horner(c, f).astype(np.float64) / 2.0 ** f - 1.0).max() < 3e-6
