"""The two polynomials the kernels evaluate on the FMA pipe (csrc/fit_polys.py):
the log1p factor of every kernel's softplus, and the exp2 of the FMA-pipe
exponential option.  Checked on the host: the header's constants are what the
fitting script produces, the fits meet their error bounds, and the kernels'
evaluation sequences, emulated in fp32 with fused multiply-adds, match the
functions they replace."""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_state_space_25_b200", "csrc")


def _fit():
    import importlib.util
    spec = importlib.util.spec_from_file_location("fit_polys", os.path.join(CSRC, "fit_polys.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_constants(prefix):
    text = open(os.path.join(CSRC, "ssm_common.cuh")).read()
    found = dict(re.findall(rf"constexpr float {prefix}(\d+) = ([-+0-9.e]+)f;", text))
    return np.array([np.float32(found[str(i)]) for i in range(len(found))], dtype=np.float32)


def _fma32(a, b, c):
    """fp32 fused multiply-add: the exact product and sum rounded once."""
    return (np.float64(a) * np.float64(b) + np.float64(c)).astype(np.float32)


def test_header_constants_are_the_fitted_ones():
    fit = _fit()
    np.testing.assert_array_equal(_header_constants("kExp2Q"), fit.fit_exp2())
    np.testing.assert_array_equal(_header_constants("kLog1pS"), fit.fit_log1p())


def test_fit_error_bounds():
    _, _, errs = _fit().report()
    assert errs["exp2: rel error of 2^r"] < 3e-7
    assert errs["exp2: rel error of 2^r - 1"] < 1e-6
    assert errs["log1p: rel error on [0, 1]"] < 5e-7


def test_softplus_sequence_in_fp32():
    """softplus(x) = max(x, 0) + e s(e), e = 2^(-|x| log2 e), s by Horner with
    fused multiply-adds; e exact here (the kernels take it from the SFU)."""
    s = _header_constants("kLog1pS")
    x = np.linspace(-30.0, 30.0, 120001).astype(np.float32)
    e = np.exp2(-np.abs(x).astype(np.float64) * np.log2(np.e)).astype(np.float32)
    acc = _fma32(s[7], e, s[6])
    for k in range(5, -1, -1):
        acc = _fma32(acc, e, s[k])
    got = _fma32(e, acc, np.maximum(x, np.float32(0)))
    ref = np.logaddexp(0.0, x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 1e-6


def test_exp2_sequence_in_fp32():
    """2^x = 2^j (1 + r q(r)) with j = rint(x) taken from the fp32 sum with
    1.5 2^23, r = x - j, q by Horner with fused multiply-adds, and 2^j added
    to the exponent field."""
    q = _header_constants("kExp2Q")
    x = np.concatenate([np.linspace(-126.0, 126.0, 200001), np.linspace(-2.0, 2.0, 40001)])
    x = x.astype(np.float32)
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    r = _fma32(j, np.float32(-1.0), x)
    acc = _fma32(q[4], r, q[3])
    for k in (2, 1, 0):
        acc = _fma32(acc, r, q[k])
    p = _fma32(acc, r, np.float32(1.0))
    shift = (t.view(np.int32) << 23).astype(np.int32)
    got = (p.view(np.int32) + shift).view(np.float32)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / ref - 1.0)) < 5e-7
