"""The coefficients of exp2_poly2 (sm100.cuh) are the ones the committed Remez
script (csrc/fit_exp2_poly.py) produces, and they meet the stated bound."""
import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "protein_pair_representation_layernorm_b200", "csrc")


def _load_fit():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly",
                                                  os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coefficients():
    src = open(os.path.join(CSRC, "sm100.cuh")).read()
    body = src[src.index("float2 exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    # Horner order in the source: c3, c2, then c1, then c0
    vals = [float(v) for v in re.findall(r"make_float2\(([0-9.]+)f, \1f\)", body)]
    c3, c2, c1, c0 = vals[:4]
    return np.array([c0, c1, c2, c3])


def test_header_coefficients_match_the_remez_fit():
    c, bound = _load_fit().remez_exp2()
    hdr = _header_coefficients()
    assert np.allclose(hdr, c, rtol=0, atol=5e-9), (hdr, c)
    assert bound < 7.6e-5


def test_header_coefficients_relative_error_bound():
    c = _header_coefficients().astype(np.float32).astype(np.float64)
    f = np.linspace(-0.5, 0.5, 100001)
    rel = np.abs(np.polyval(c[::-1], f) - np.exp2(f)) / np.exp2(f)
    assert rel.max() < 7.6e-5
    # equioscillation: 5 runs of alternating sign, each reaching the bound
    err = (np.polyval(c[::-1], f) - np.exp2(f)) / np.exp2(f)
    sign = np.sign(err)
    peaks = [0]
    for i in range(1, len(f)):
        if sign[i] != sign[peaks[-1]]:
            peaks.append(i)
        elif abs(err[i]) > abs(err[peaks[-1]]):
            peaks[-1] = i
    assert len(peaks) == 5, len(peaks)
    assert all(abs(abs(err[i]) - rel.max()) < 1e-7 for i in peaks), err[peaks]
