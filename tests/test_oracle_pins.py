"""Pins of the fp64 oracle to facts the pages and the mathematics fix.

None of these re-run the oracle's own loop in another spelling: each checks
it against a closed form, a special case with a known answer, an invariant,
a brute-force unrolled sum, an independently built permutation, or another
oracle function that is written separately.  Cited passages:

* "手把手拆解Mamba-minimal中的selective_scan实现" (mhpn.cn): §3.1 ZOH for A
  (deltaA = exp(delta A)), §3.2 Euler for B (deltaB_u = delta B u), §4 the
  sequential loop (update, then read out with C), §5 y + u D, §6 the mixed
  ZOH-A / Euler-B strategy.
* "代码连连看——mamba": Mamba.step() -- softplus(dt + bias), the in-place
  state update and y * act(z).
* "关于代码SS2D中的d_state设置" (VMamba issue 206): CrossScan / CrossMerge
  only arrange the sequence.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(1234)


def _softplus_ref(x):
    # textbook definition with torch's threshold (x > 20 -> x)
    return x if x > 20.0 else math.log1p(math.exp(x))


def _silu_ref(z):
    return z / (1.0 + math.exp(-z))


def _rand_problem(b, L, d_in, N, rng, h0=True, z=True):
    u = rng.standard_normal((b, L, d_in))
    dt = 0.5 * rng.standard_normal((b, L, d_in))
    A = -rng.uniform(0.5, 8.0, size=(d_in, N))          # distinct per (d, n)
    B = rng.standard_normal((b, L, N))
    C = rng.standard_normal((b, L, N))
    D = rng.standard_normal(d_in)
    zz = rng.standard_normal((b, L, d_in)) if z else None
    bias = rng.uniform(-4.0, -1.0, size=d_in)
    hh = rng.standard_normal((b, d_in, N)) if h0 else None
    return u, dt, A, B, C, D, zz, bias, hh


# --------------------------------------------------------------------------
# Hand-worked example (exact rationals): decays of exactly 1/2 and 1/4.
# --------------------------------------------------------------------------
def test_hand_worked_scan():
    # A = [-ln 2, -ln 4], delta = 1 (no softplus): exp(delta A) = [1/2, 1/4].
    # B_t = [1, 2], C_t = [1, -1], u = [1, 0, 2], D = 1/2, h0 = 0.
    # t0: h = [1, 2]            y0 = 1 - 2 + 1/2          = -1/2
    # t1: h = [1/2, 1/2]        y1 = 0 + 0                =  0
    # t2: h = [1/4+2, 1/8+4]    y2 = 9/4 - 33/8 + 1       = -7/8
    u = np.array([1.0, 0.0, 2.0]).reshape(1, 3, 1)
    dt = np.ones((1, 3, 1))
    A = np.array([[-math.log(2.0), -math.log(4.0)]])
    B = np.tile([1.0, 2.0], (1, 3, 1))
    C = np.tile([1.0, -1.0], (1, 3, 1))
    y, h = oracle.selective_scan(u, dt, A, B, C, D=np.array([0.5]), delta_softplus=False,
                                 return_last_state=True)
    exp_y = [Fraction(-1, 2), Fraction(0), Fraction(-7, 8)]
    exp_h = [Fraction(9, 4), Fraction(33, 8)]
    np.testing.assert_allclose(y.ravel(), [float(v) for v in exp_y], rtol=0, atol=1e-14)
    np.testing.assert_allclose(h.ravel(), [float(v) for v in exp_h], rtol=0, atol=1e-14)


def test_hand_worked_step():
    # state = [1, 1], x = 2, dt = 1 (no softplus), A = [-ln 2, -ln 4],
    # B = [1, 1], C = [1, 2], D = 1:
    # new state = [1/2 + 2, 1/4 + 2] = [5/2, 9/4];  y = 5/2 + 9/2 + 2 = 9.
    y, st = oracle.state_update(np.ones((1, 1, 2)), np.array([[2.0]]), np.array([[1.0]]),
                                np.array([[-math.log(2.0), -math.log(4.0)]]),
                                np.array([[1.0, 1.0]]), np.array([[1.0, 2.0]]),
                                D=np.array([1.0]), dt_softplus=False)
    np.testing.assert_allclose(st.ravel(), [2.5, 2.25], rtol=0, atol=1e-14)
    np.testing.assert_allclose(y.ravel(), [9.0], rtol=0, atol=1e-13)


# --------------------------------------------------------------------------
# Closed form: constant delta, B, C, u over t, h0 = 0 -> geometric sum.
# --------------------------------------------------------------------------
def test_closed_form_geometric_sum():
    b, L, d_in, N = 2, 50, 3, 5
    rng = np.random.default_rng(7)
    dt_c = rng.uniform(-1.0, 1.0, size=(b, d_in))
    u_c = rng.standard_normal((b, d_in))
    z_c = rng.standard_normal((b, d_in))
    B_c = rng.standard_normal((b, N))
    C_c = rng.standard_normal((b, N))
    A = -rng.uniform(0.2, 3.0, size=(d_in, N))
    D = rng.standard_normal(d_in)
    bias = rng.uniform(-2.0, 0.0, size=d_in)
    u = np.repeat(u_c[:, None, :], L, 1)
    dt = np.repeat(dt_c[:, None, :], L, 1)
    z = np.repeat(z_c[:, None, :], L, 1)
    B = np.repeat(B_c[:, None, :], L, 1)
    C = np.repeat(C_c[:, None, :], L, 1)
    y = oracle.selective_scan(u, dt, A, B, C, D=D, z=z, dt_bias=bias, delta_softplus=True)
    for ib in range(b):
        for d in range(d_in):
            delta = _softplus_ref(dt_c[ib, d] + bias[d])
            for t in range(L):
                acc = 0.0
                for n in range(N):
                    a = math.exp(delta * A[d, n])
                    acc += C_c[ib, n] * delta * B_c[ib, n] * u_c[ib, d] * (1 - a ** (t + 1)) / (1 - a)
                ref = (acc + D[d] * u_c[ib, d]) * _silu_ref(z_c[ib, d])
                assert abs(y[ib, t, d] - ref) <= 1e-12 * max(1.0, abs(ref))


# --------------------------------------------------------------------------
# Sequential == brute-force unrolled sum on tiny inputs.
# h_t = sum_{s<=t} (prod_{r=s+1..t} a_r) delta_s B_s u_s + (prod_{r<=t} a_r) h0
# --------------------------------------------------------------------------
@pytest.mark.parametrize("softplus", [True, False])
def test_sequential_equals_bruteforce(softplus):
    b, L, d_in, N = 2, 9, 3, 4
    u, dt, A, B, C, D, z, bias, h0 = _rand_problem(b, L, d_in, N, RNG)
    if not softplus:
        dt = np.abs(dt)
    y, hl = oracle.selective_scan(u, dt, A, B, C, D=D, z=z, dt_bias=bias,
                                  delta_softplus=softplus, h0=h0, return_last_state=True)
    for ib in range(b):
        for d in range(d_in):
            delta = [dt[ib, t, d] + bias[d] for t in range(L)]
            if softplus:
                delta = [_softplus_ref(v) for v in delta]
            a = [[math.exp(delta[t] * A[d, n]) for n in range(N)] for t in range(L)]
            for t in range(L):
                h = []
                for n in range(N):
                    s_sum = 0.0
                    for s in range(t + 1):
                        prod = 1.0
                        for r in range(s + 1, t + 1):
                            prod *= a[r][n]
                        s_sum += prod * delta[s] * B[ib, s, n] * u[ib, s, d]
                    prod0 = 1.0
                    for r in range(t + 1):
                        prod0 *= a[r][n]
                    h.append(s_sum + prod0 * h0[ib, d, n])
                ref = sum(C[ib, t, n] * h[n] for n in range(N)) + D[d] * u[ib, t, d]
                ref *= _silu_ref(z[ib, t, d])
                assert abs(y[ib, t, d] - ref) <= 1e-12 * max(1.0, abs(ref))
                if t == L - 1:
                    np.testing.assert_allclose(hl[ib, d], h, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# Zero input: u = 0, h0 = 0 give h = 0 and y = 0 whatever dt, z, bias are.
# --------------------------------------------------------------------------
def test_zero_input_zero_output():
    b, L, d_in, N = 2, 17, 5, 16
    u, dt, A, B, C, D, z, bias, _ = _rand_problem(b, L, d_in, N, RNG, h0=False)
    y, hl = oracle.selective_scan(np.zeros_like(u), dt, A, B, C, D=D, z=z, dt_bias=bias,
                                  return_last_state=True)
    assert np.all(y == 0.0) and np.all(hl == 0.0)


# --------------------------------------------------------------------------
# A -> -infinity: exp(delta A) underflows to exactly 0, so with Euler-B
# ([Minimal-scan] §3.2, §6) y_t = (C_t . B_t) delta_t u_t + D u_t.  ZOH-B
# would give (exp(delta A) - 1) / A * B u -> 0 instead.
# --------------------------------------------------------------------------
def test_A_to_minus_infinity_pins_euler_B():
    b, L, d_in, N = 2, 11, 4, 6
    u, dt, _, B, C, D, z, bias, h0 = _rand_problem(b, L, d_in, N, RNG)
    A = -np.exp(40.0) * np.ones((d_in, N))
    y = oracle.selective_scan(u, dt, A, B, C, D=D, z=z, dt_bias=bias, h0=h0)
    for ib in range(b):
        for t in range(L):
            cb = float(np.dot(C[ib, t], B[ib, t]))
            for d in range(d_in):
                delta = _softplus_ref(dt[ib, t, d] + bias[d])
                ref = (cb * delta * u[ib, t, d] + D[d] * u[ib, t, d]) * _silu_ref(z[ib, t, d])
                assert abs(y[ib, t, d] - ref) <= 1e-12 * max(1.0, abs(ref))


# --------------------------------------------------------------------------
# Known values of softplus and SiLU, read through the scan: with A -> -inf,
# N = 1, B = C = 1, u = 1, D = 0 the output is delta; with delta = 1 (no
# softplus) the output is silu(z).
# --------------------------------------------------------------------------
def test_softplus_known_values():
    xs = np.array([0.0, 1.0, -30.0, 25.0, 19.5, -3.0])
    L = xs.size
    y = oracle.selective_scan(np.ones((1, L, 1)), xs.reshape(1, L, 1), np.array([[-np.exp(40.0)]]),
                              np.ones((1, L, 1)), np.ones((1, L, 1)), delta_softplus=True).ravel()
    assert abs(y[0] - math.log(2.0)) < 1e-15                      # softplus(0) = ln 2
    assert abs(y[1] - math.log(1.0 + math.e)) < 1e-15             # ln(1 + e)
    assert abs(y[2] / math.exp(-30.0) - 1.0) < 1e-12              # ~ e^x for x << 0
    assert y[3] == 25.0                                           # threshold: x > 20 -> x
    assert abs(y[4] - 19.5) < 1e-8                                # log1p(e^19.5) ~ 19.5 + 3.4e-9
    assert abs(y[5] - 0.04858735157374206) < 1e-15                # ln(1 + e^-3)


def test_silu_known_values():
    zs = np.array([0.0, 1.0, -1.0, 10.0])
    L = zs.size
    y = oracle.selective_scan(np.ones((1, L, 1)), np.ones((1, L, 1)), np.array([[-np.exp(40.0)]]),
                              np.ones((1, L, 1)), np.ones((1, L, 1)), z=zs.reshape(1, L, 1),
                              delta_softplus=False).ravel()
    # silu(z) = z * sigmoid(z)
    np.testing.assert_allclose(y, [0.0, 0.7310585786300049, -0.2689414213699951,
                                   9.999546021312976], rtol=1e-15, atol=0)


# --------------------------------------------------------------------------
# Scan <-> step consistency ([Minimal-scan] §4 vs [Mamba-step]).
# --------------------------------------------------------------------------
def test_L1_scan_equals_step():
    b, d_in, N = 3, 7, 16
    u, dt, A, B, C, D, z, bias, h0 = _rand_problem(b, 1, d_in, N, RNG)
    y_s, h_s = oracle.selective_scan(u, dt, A, B, C, D=D, z=z, dt_bias=bias, h0=h0,
                                     return_last_state=True)
    y_t, h_t = oracle.state_update(h0, u[:, 0], dt[:, 0], A, B[:, 0], C[:, 0], D=D, z=z[:, 0],
                                   dt_bias=bias)
    np.testing.assert_allclose(y_s[:, 0], y_t, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(h_s, h_t, rtol=1e-14, atol=1e-14)


def test_k_steps_equal_scan_of_length_k():
    b, L, d_in, N = 2, 13, 5, 8
    u, dt, A, B, C, D, z, bias, h0 = _rand_problem(b, L, d_in, N, RNG)
    y_s, h_s = oracle.selective_scan(u, dt, A, B, C, D=D, z=z, dt_bias=bias, h0=h0,
                                     return_last_state=True)
    st = h0
    for t in range(L):
        y_t, st = oracle.state_update(st, u[:, t], dt[:, t], A, B[:, t], C[:, t], D=D,
                                      z=z[:, t], dt_bias=bias)
        np.testing.assert_allclose(y_s[:, t], y_t, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(h_s, st, rtol=1e-12, atol=1e-12)


def test_split_scan_resumes_exactly():
    """Scanning [0, L1) then [L1, L) from the carried state equals one scan."""
    b, L, d_in, N = 2, 20, 3, 4
    u, dt, A, B, C, D, z, bias, h0 = _rand_problem(b, L, d_in, N, RNG)
    y, h = oracle.selective_scan(u, dt, A, B, C, D=D, z=z, dt_bias=bias, h0=h0,
                                 return_last_state=True)
    L1 = 7
    y1, h1 = oracle.selective_scan(u[:, :L1], dt[:, :L1], A, B[:, :L1], C[:, :L1], D=D,
                                   z=z[:, :L1], dt_bias=bias, h0=h0, return_last_state=True)
    y2, h2 = oracle.selective_scan(u[:, L1:], dt[:, L1:], A, B[:, L1:], C[:, L1:], D=D,
                                   z=z[:, L1:], dt_bias=bias, h0=h1, return_last_state=True)
    np.testing.assert_array_equal(np.concatenate([y1, y2], 1), y)
    np.testing.assert_array_equal(h2, h)


def test_linearity_in_u_and_h0():
    """Without the gate, y is linear in (u, h0) for fixed delta, A, B, C, D."""
    b, L, d_in, N = 2, 15, 3, 5
    u1, dt, A, B, C, D, _, bias, h1 = _rand_problem(b, L, d_in, N, RNG, z=False)
    u2 = RNG.standard_normal(u1.shape)
    h2 = RNG.standard_normal(h1.shape)
    # delta must not depend on u: feed the same dt to all three runs
    f = lambda u, h: oracle.selective_scan(u, dt, A, B, C, D=D, dt_bias=bias, h0=h)
    lhs = f(2.0 * u1 - 3.0 * u2, 2.0 * h1 - 3.0 * h2)
    rhs = 2.0 * f(u1, h1) - 3.0 * f(u2, h2)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-11, atol=1e-11)


# --------------------------------------------------------------------------
# Decode: constant inputs -> h_k = h* + a^k (h0 - h*),  h* = delta B x / (1 - a)
# --------------------------------------------------------------------------
def test_decode_fixed_point_closed_form():
    b, d_in, N, steps = 2, 4, 16, 1000
    rng = np.random.default_rng(11)
    st0 = rng.standard_normal((b, d_in, N))
    x = rng.standard_normal((b, d_in))
    dt = rng.standard_normal((b, d_in))
    z = rng.standard_normal((b, d_in))
    B = rng.standard_normal((b, N))
    C = rng.standard_normal((b, N))
    A = -np.tile(np.arange(1, N + 1, dtype=np.float64), (d_in, 1))
    bias = rng.uniform(-6.9, -2.3, size=d_in)
    D = np.ones(d_in)
    st = st0
    for _ in range(steps):
        y, st = oracle.state_update(st, x, dt, A, B, C, D=D, z=z, dt_bias=bias)
    for ib in range(b):
        for d in range(d_in):
            delta = _softplus_ref(dt[ib, d] + bias[d])
            yref = 0.0
            for n in range(N):
                a = math.exp(delta * A[d, n])
                hstar = delta * B[ib, n] * x[ib, d] / (1.0 - a)
                hk = hstar + a ** steps * (st0[ib, d, n] - hstar)
                assert abs(st[ib, d, n] - hk) <= 1e-9 * max(1.0, abs(hk))
                yref += C[ib, n] * hk
            yref = (yref + D[d] * x[ib, d]) * _silu_ref(z[ib, d])
            assert abs(y[ib, d] - yref) <= 1e-9 * max(1.0, abs(yref))


# --------------------------------------------------------------------------
# SS2D: CrossScan / CrossMerge are pure rearrangements ([VMamba-206]).
# --------------------------------------------------------------------------
def _numpy_cross_scan(u, H, W):
    b, L, d = u.shape
    rm = u
    cm = u.reshape(b, H, W, d).transpose(0, 2, 1, 3).reshape(b, L, d)
    return np.stack([rm, cm, rm[:, ::-1], cm[:, ::-1]], axis=1)


def test_ss2d_orders_hand_derived():
    # H = 2, W = 3, pixels p = h*3 + w.  Orders written out by hand.
    H, W = 2, 3
    u = np.arange(6, dtype=np.float64).reshape(1, 6, 1)
    xs = oracle.cross_scan(u, H, W)[0, :, :, 0]
    assert xs[0].tolist() == [0, 1, 2, 3, 4, 5]       # row-major
    assert xs[1].tolist() == [0, 3, 1, 4, 2, 5]       # column-major
    assert xs[2].tolist() == [5, 4, 3, 2, 1, 0]       # row-major reversed
    assert xs[3].tolist() == [5, 2, 4, 1, 3, 0]       # column-major reversed


@pytest.mark.parametrize("H,W", [(5, 7), (1, 9), (8, 1), (4, 4)])
def test_ss2d_cross_scan_matches_numpy(H, W):
    u = RNG.standard_normal((2, H * W, 3))
    np.testing.assert_array_equal(oracle.cross_scan(u, H, W), _numpy_cross_scan(u, H, W))


@pytest.mark.parametrize("H,W", [(5, 7), (1, 9), (3, 3)])
def test_ss2d_merge_of_scan_is_4u(H, W):
    u = RNG.standard_normal((2, H * W, 5))
    np.testing.assert_array_equal(oracle.cross_merge(oracle.cross_scan(u, H, W), H, W), 4.0 * u)


def test_ss2d_single_row_directions_coincide():
    H, W = 1, 13
    u = RNG.standard_normal((1, W, 2))
    xs = oracle.cross_scan(u, H, W)
    np.testing.assert_array_equal(xs[:, 0], xs[:, 1])
    np.testing.assert_array_equal(xs[:, 2], xs[:, 0][:, ::-1])


@pytest.mark.parametrize("N", [1, 4])
def test_ss2d_scan_is_four_1d_scans(N):
    """ss2d = sum over directions of the un-permuted 1-D scans of the
    numpy-permuted sequences."""
    b, H, W, d_in = 2, 3, 5, 4
    L = H * W
    u = RNG.standard_normal((b, L, d_in))
    delta = RNG.standard_normal((b, 4, L, d_in))
    A = -RNG.uniform(0.5, 2.0, size=(4 * d_in, N))
    B = RNG.standard_normal((b, 4, L, N))
    C = RNG.standard_normal((b, 4, L, N))
    D = RNG.standard_normal(4 * d_in)
    bias = RNG.uniform(-3, 0, size=4 * d_in)
    y = oracle.ss2d_scan(u, delta, A, B, C, H, W, D=D, dt_bias=bias)
    xs = _numpy_cross_scan(u, H, W)
    ref = np.zeros_like(u)
    for k in range(4):
        sl = slice(k * d_in, (k + 1) * d_in)
        yk = oracle.selective_scan(xs[:, k], delta[:, k], A[sl], B[:, k], C[:, k], D=D[sl],
                                   dt_bias=bias[sl])
        # undo the permutation of direction k with numpy
        if k == 0:
            ref += yk
        elif k == 1:
            ref += yk.reshape(b, W, H, d_in).transpose(0, 2, 1, 3).reshape(b, L, d_in)
        elif k == 2:
            ref += yk[:, ::-1]
        else:
            ref += yk[:, ::-1].reshape(b, W, H, d_in).transpose(0, 2, 1, 3).reshape(b, L, d_in)
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# Planted mistakes: each of these variants of the recurrence must be caught
# by at least one pin above.  The mutants are built here on the CPU from the
# oracle's building blocks (never on the GPU).
# --------------------------------------------------------------------------
def test_pins_reject_zoh_B_variant():
    # Full ZOH-B: B_bar u = (exp(dA) - 1)/A * B u.  Under A -> -inf it -> 0,
    # which the Euler-B pin above would reject.
    A = -np.exp(40.0)
    delta, Bv, u = 0.3, 1.7, 0.9
    zoh = (math.exp(delta * A) - 1.0) / A * Bv * u
    euler = delta * Bv * u
    assert abs(zoh) < 1e-15 and abs(euler - 0.459) < 1e-12


# --------------------------------------------------------------------------
# SS2D snake order (the "蛇形Scan / 蛇形Merge" variant of [VMamba-206]):
# odd rows right to left in k0, odd columns bottom to top in k1.
# --------------------------------------------------------------------------
def _numpy_snake_scan(u, H, W):
    b, L, d = u.shape
    rm = u.reshape(b, H, W, d).copy()
    rm[:, 1::2] = rm[:, 1::2, ::-1]
    cm = u.reshape(b, H, W, d).transpose(0, 2, 1, 3).copy()    # (b, W, H, d): columns
    cm[:, 1::2] = cm[:, 1::2, ::-1]
    rm, cm = rm.reshape(b, L, d), cm.reshape(b, L, d)
    return np.stack([rm, cm, rm[:, ::-1], cm[:, ::-1]], axis=1)


def test_ss2d_snake_orders_hand_derived():
    # H = 2, W = 3, pixels p = h*3 + w.  Orders written out by hand.
    u = np.arange(6, dtype=np.float64).reshape(1, 6, 1)
    xs = oracle.cross_scan(u, 2, 3, order="snake")[0, :, :, 0]
    assert xs[0].tolist() == [0, 1, 2, 5, 4, 3]       # rows, odd row right to left
    assert xs[1].tolist() == [0, 3, 4, 1, 2, 5]       # columns, odd column bottom to top
    assert xs[2].tolist() == [3, 4, 5, 2, 1, 0]       # reverse of the first
    assert xs[3].tolist() == [5, 2, 1, 4, 3, 0]       # reverse of the second


@pytest.mark.parametrize("H,W", [(5, 7), (1, 9), (8, 1), (4, 4), (3, 6)])
def test_ss2d_snake_matches_numpy(H, W):
    u = RNG.standard_normal((2, H * W, 3))
    np.testing.assert_array_equal(oracle.cross_scan(u, H, W, order="snake"),
                                  _numpy_snake_scan(u, H, W))
    np.testing.assert_array_equal(
        oracle.cross_merge(oracle.cross_scan(u, H, W, order="snake"), H, W, order="snake"), 4.0 * u)


def test_ss2d_snake_scan_is_four_1d_scans():
    b, H, W, d_in, N = 2, 3, 5, 4, 1
    L = H * W
    u = RNG.standard_normal((b, L, d_in))
    delta = RNG.standard_normal((b, 4, L, d_in))
    A = -RNG.uniform(0.5, 2.0, size=(4 * d_in, N))
    B = RNG.standard_normal((b, 4, L, N))
    C = RNG.standard_normal((b, 4, L, N))
    D = RNG.standard_normal(4 * d_in)
    y = oracle.ss2d_scan(u, delta, A, B, C, H, W, D=D, order="snake")
    xs = _numpy_snake_scan(u, H, W)
    perm = _numpy_snake_scan(np.arange(L, dtype=np.float64).reshape(1, L, 1), H, W)[0, :, :, 0]
    ref = np.zeros_like(u)
    for k in range(4):
        sl = slice(k * d_in, (k + 1) * d_in)
        yk = oracle.selective_scan(xs[:, k], delta[:, k], A[sl], B[:, k], C[:, k], D=D[sl])
        ref[:, perm[k].astype(int)] += yk       # step l of direction k lands on pixel perm[k][l]
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# Causal-conv1d decode step ("代码连连看——mamba", Mamba.step(), Conv step):
# roll the window left, append x, dot with the weight, add the bias, SiLU.
# --------------------------------------------------------------------------
def test_conv_step_one_hot_taps():
    b, d_in, K = 2, 3, 4
    cs = RNG.standard_normal((b, d_in, K))
    x = RNG.standard_normal((b, d_in))
    last = np.zeros((d_in, K)); last[:, -1] = 1.0        # newest tap only
    out, new = oracle.conv_step(cs, x, last)
    np.testing.assert_allclose(out, x / (1.0 + np.exp(-x)), rtol=1e-15)
    np.testing.assert_array_equal(new[..., :-1], cs[..., 1:])   # rolled left by one
    np.testing.assert_array_equal(new[..., -1], x)              # x appended
    first = np.zeros((d_in, K)); first[:, 0] = 1.0       # oldest tap: the old second entry
    out0, _ = oracle.conv_step(cs, x, first, bias=np.full(d_in, 0.25))
    v = cs[..., 1] + 0.25
    np.testing.assert_allclose(out0, v / (1.0 + np.exp(-v)), rtol=1e-15)


@pytest.mark.parametrize("K", [2, 3, 4])
def test_conv_steps_equal_causal_convolution(K):
    """T decode steps from a zero window == a causal convolution of the
    sequence with zero left padding, written with numpy.correlate."""
    b, d_in, T = 2, 3, 11
    xs = RNG.standard_normal((b, T, d_in))
    w = RNG.standard_normal((d_in, K))
    bias = RNG.standard_normal(d_in)
    cs = np.zeros((b, d_in, K))
    outs = []
    for t in range(T):
        o, cs = oracle.conv_step(cs, xs[:, t], w, bias)
        outs.append(o)
    got = np.stack(outs, 1)
    for ib in range(b):
        for d in range(d_in):
            padded = np.concatenate([np.zeros(K - 1), xs[ib, :, d]])
            pre = np.correlate(padded, w[d], mode="valid") + bias[d]   # sum_j w[j] x[t-K+1+j]
            np.testing.assert_allclose(got[ib, :, d], pre / (1.0 + np.exp(-pre)), rtol=1e-12,
                                       atol=1e-14)


# --------------------------------------------------------------------------
# Backward scan: gradients of sum(dout * y) + sum(dh_last * h_last).
# Pinned to central finite differences of the (separately pinned) forward
# oracle, and to exact linearity identities that need no differencing.
# --------------------------------------------------------------------------
def _bwd_problem(rng, b=2, L=6, d_in=3, N=4, z=True, h0=True):
    u, dt, A, B, C, D, zz, bias, hh = _rand_problem(b, L, d_in, N, rng, h0=h0, z=z)
    bias = rng.uniform(-1.5, 0.5, size=d_in)       # softplus well inside its smooth branch
    dout = rng.standard_normal((b, L, d_in))
    dhl = rng.standard_normal((b, d_in, N))
    return dict(u=u, delta=dt, A=A, B=B, C=C, D=D, z=zz, dt_bias=bias, h0=hh), dout, dhl


def _loss(args, dout, dhl, softplus=True):
    y, hl = oracle.selective_scan(args["u"], args["delta"], args["A"], args["B"], args["C"],
                                  D=args["D"], z=args["z"], dt_bias=args["dt_bias"],
                                  delta_softplus=softplus, h0=args["h0"], return_last_state=True)
    return float(np.sum(dout * y) + np.sum(dhl * hl))


_GRAD_OF = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
            "z": "dz", "dt_bias": "ddt_bias", "h0": "dh0"}


@pytest.mark.parametrize("softplus", [True, False])
def test_bwd_matches_central_differences(softplus):
    rng = np.random.default_rng(77 + softplus)
    args, dout, dhl = _bwd_problem(rng)
    if not softplus:
        args["delta"] = np.abs(args["delta"]) * 0.3 + 0.05
        args["dt_bias"] = rng.uniform(0.0, 0.1, size=args["dt_bias"].shape)
    g = oracle.selective_scan_bwd(args["u"], args["delta"], args["A"], args["B"], args["C"], dout,
                                  D=args["D"], z=args["z"], dt_bias=args["dt_bias"],
                                  delta_softplus=softplus, h0=args["h0"], dh_last=dhl)
    eps = 1e-6
    for name, gname in _GRAD_OF.items():
        x = args[name]
        fd = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + eps
            fp = _loss(args, dout, dhl, softplus)
            x[idx] = keep - eps
            fm = _loss(args, dout, dhl, softplus)
            x[idx] = keep
            fd[idx] = (fp - fm) / (2 * eps)
        scale = max(1.0, float(np.max(np.abs(fd))))
        np.testing.assert_allclose(g[gname], fd, rtol=0, atol=2e-7 * scale, err_msg=name)


def test_bwd_linearity_identities():
    """Exact identities (no differencing).  Without the gate, y and h_last
    are jointly linear in (u, h0), in C, and -- with h0 = 0 -- the scan part
    is linear in B, so the loss equals the gradient's inner product with the
    argument (Euler's theorem for degree-1 homogeneous functions)."""
    rng = np.random.default_rng(5)
    args, dout, dhl = _bwd_problem(rng, b=3, L=11, d_in=4, N=5, z=False)
    call = lambda a, dh: oracle.selective_scan_bwd(
        a["u"], a["delta"], a["A"], a["B"], a["C"], dout, D=a["D"], dt_bias=a["dt_bias"],
        h0=a["h0"], dh_last=dh)
    y, hl = oracle.selective_scan(args["u"], args["delta"], args["A"], args["B"], args["C"],
                                  D=args["D"], dt_bias=args["dt_bias"], h0=args["h0"],
                                  return_last_state=True)
    g = call(args, dhl)
    F = np.sum(dout * y) + np.sum(dhl * hl)
    assert np.sum(g["du"] * args["u"]) + np.sum(g["dh0"] * args["h0"]) == pytest.approx(F, rel=1e-12)
    Dterm = np.sum(dout * args["u"] * args["D"][None, None, :])
    assert np.sum(g["dC"] * args["C"]) == pytest.approx(np.sum(dout * y) - Dterm, rel=1e-12)
    assert np.sum(g["dD"] * args["D"]) == pytest.approx(Dterm, rel=1e-12)
    args["h0"] = None
    y0, hl0 = oracle.selective_scan(args["u"], args["delta"], args["A"], args["B"], args["C"],
                                    D=args["D"], dt_bias=args["dt_bias"], return_last_state=True)
    g0 = call(args, dhl)
    assert np.sum(g0["dB"] * args["B"]) == pytest.approx(
        np.sum(dout * y0) - Dterm + np.sum(dhl * hl0), rel=1e-12)
    assert np.all(g0["dh0"] == g["dh0"])     # dh0 does not depend on h0


def test_bwd_L1_closed_form():
    """One step from h0 with a scalar decay: every gradient by hand."""
    u, dt, A, B, C, D, h0 = 0.7, -0.3, -2.0, 1.5, -0.8, 0.4, 0.9
    dout, dhl = 1.3, -0.6
    delta = _softplus_ref(dt)
    a = math.exp(delta * A)
    h = a * h0 + delta * B * u
    lam = dout * C + dhl                           # d loss / d h
    g = oracle.selective_scan_bwd(np.full((1, 1, 1), u), np.full((1, 1, 1), dt),
                                  np.full((1, 1), A), np.full((1, 1, 1), B),
                                  np.full((1, 1, 1), C), np.full((1, 1, 1), dout),
                                  D=np.full(1, D), h0=np.full((1, 1, 1), h0),
                                  dh_last=np.full((1, 1, 1), dhl))
    sig = 1.0 / (1.0 + math.exp(-dt))
    exp = dict(du=dout * D + lam * delta * B, dC=dout * h, dD=dout * u, dB=lam * delta * u,
               dA=lam * delta * a * h0, dh0=lam * a,
               ddelta=lam * (A * a * h0 + B * u) * sig)
    for k, v in exp.items():
        assert float(g[k].ravel()[0]) == pytest.approx(v, rel=1e-13, abs=1e-15), k


def test_bwd_absent_D_is_D_zero():
    """Without D (and without dt_bias) the gradients are those at D = 0 (and
    bias = 0): dD and ddt_bias are still defined and equal the explicit-zero
    case exactly."""
    rng = np.random.default_rng(8)
    args, dout, dhl = _bwd_problem(rng, b=2, L=9, d_in=3, N=4)
    base = dict(u=args["u"], delta=args["delta"], A=args["A"], B=args["B"], C=args["C"], dout=dout,
                z=args["z"], h0=args["h0"], dh_last=dhl)
    g_none = oracle.selective_scan_bwd(**base)
    g_zero = oracle.selective_scan_bwd(**base, D=np.zeros(3), dt_bias=np.zeros(3))
    for k in g_zero:
        np.testing.assert_array_equal(g_none[k], g_zero[k], err_msg=k)
    assert np.any(g_none["dD"] != 0)
