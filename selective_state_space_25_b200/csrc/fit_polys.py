"""Fits the two polynomials the kernels evaluate on the FMA pipe.

1. exp2.  2^x = 2^j * p(r) with j = rint(x), r = x - j in [-1/2, 1/2] and
       p(r) = 1 + r * q(r),   q(r) ~ (2^r - 1) / r,   q of degree 4.
   Writing p this way makes p(0) = 1 exactly and keeps the RELATIVE accuracy
   of p(r) - 1 = 2^r - 1 near r = 0, which is what a decay factor close to
   one needs (the state's memory is 1 / (1 - 2^x)).

2. log1p on [0, 1], for softplus(x) = max(x, 0) + log1p(e^-|x|):
       log1p(e) = e * s(e),   s(e) ~ log1p(e) / e,   s of degree 7,
   again relative, so softplus keeps its relative accuracy for very negative
   x, where it is e^x itself.

Both are fitted for minimax relative error with Lawson's algorithm
(iteratively reweighted least squares on a dense Chebyshev-spaced grid) in
float64, then rounded to fp32.

Run:  python selective_state_space_25_b200/csrc/fit_polys.py
"""
import numpy as np


def lawson(x, f, deg, iters=300):
    V = np.vander(x, deg + 1, increasing=True)
    w = np.ones_like(x) / x.size
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * (sw / f)[:, None], sw, rcond=None)  # relative residual
        err = np.abs(V @ c / f - 1.0)
        w = w * err
        w /= w.sum()
    return c


def exp2_q(r):
    out = np.full_like(r, np.log(2.0))
    nz = np.abs(r) > 1e-12
    out[nz] = np.expm1(r[nz] * np.log(2.0)) / r[nz]
    return out


def log1p_s(e):
    out = np.ones_like(e)
    nz = e > 1e-12
    out[nz] = np.log1p(e[nz]) / e[nz]
    return out


def fit_exp2(deg=4):
    r = np.cos(np.linspace(0, np.pi, 20001)) * 0.5
    return lawson(r, exp2_q(r), deg).astype(np.float32)


def fit_log1p(deg=7):
    e = (1.0 - np.cos(np.linspace(0, np.pi, 20001))) * 0.5
    return lawson(e, log1p_s(e), deg).astype(np.float32)


def report():
    q = fit_exp2()
    s = fit_log1p()
    r = np.linspace(-0.5, 0.5, 200001)
    qv = np.polyval(q.astype(np.float64)[::-1], r)
    e = np.linspace(0.0, 1.0, 200001)
    sv = np.polyval(s.astype(np.float64)[::-1], e)
    errs = {
        "exp2: rel error of 2^r - 1": float(np.max(np.abs(qv / exp2_q(r) - 1.0))),
        "exp2: rel error of 2^r": float(np.max(np.abs((1.0 + r * qv) / np.exp2(r) - 1.0))),
        "log1p: rel error on [0, 1]": float(np.max(np.abs(sv / log1p_s(e) - 1.0))),
    }
    return q, s, errs


if __name__ == "__main__":
    q, s, errs = report()
    for i, v in enumerate(q):
        print(f"constexpr float kExp2Q{i} = {float(v):.9e}f;")
    for i, v in enumerate(s):
        print(f"constexpr float kLog1pS{i} = {float(v):.9e}f;")
    for k, v in errs.items():
        print(f"// {k}: {v:.3e}")
