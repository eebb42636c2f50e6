"""fp64 CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``selective_state_space_25_b200``) never touches it.

The arithmetic lives in ``ssm_oracle.c`` (plain C, double precision, the
definition of the method written out); this module only compiles it with gcc
and marshals numpy float64 arrays through ctypes.  Every function cites its
passage in the C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ssm_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    with _lock:
        stale = (not os.path.exists(_LIB)) or (
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC))
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                   "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # A test may point the loader at a deliberately broken copy of the
        # oracle (tests/test_oracle_mutants.py) to show the pins catch it.
        path = os.environ.get("SSM_ORACLE_LIB_OVERRIDE")
        if not path:
            build()
            path = _LIB
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.oracle_selective_scan.argtypes = [P] * 8 + [ctypes.c_int, P, P, P] + [I64] * 4
        lib.oracle_selective_scan.restype = None
        lib.oracle_state_update.argtypes = [P] * 9 + [ctypes.c_int, P] + [I64] * 3
        lib.oracle_state_update.restype = None
        lib.oracle_cross_scan.argtypes = [P, P] + [I64] * 4 + [ctypes.c_int]
        lib.oracle_cross_scan.restype = None
        lib.oracle_cross_merge.argtypes = [P, P] + [I64] * 4 + [ctypes.c_int]
        lib.oracle_cross_merge.restype = None
        lib.oracle_ss2d_scan.argtypes = [P] * 7 + [ctypes.c_int, P] + [I64] * 5 + [ctypes.c_int]
        lib.oracle_ss2d_scan.restype = ctypes.c_int
        lib.oracle_conv_step.argtypes = [P] * 5 + [I64] * 3
        lib.oracle_conv_step.restype = None
        lib.oracle_selective_scan_bwd.argtypes = ([P] * 8 + [ctypes.c_int] + [P] * 12
                                                  + [I64] * 4)
        lib.oracle_selective_scan_bwd.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = None
        _lib = lib
    return _lib


def _f64(a, shape=None):
    """Widen to a C-contiguous float64 numpy array (exact for fp32 / bf16)."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu")
        if str(a.dtype) == "torch.bfloat16":
            a = a.float()
        a = a.double().numpy()
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        raise ValueError(f"oracle: expected shape {tuple(shape)}, got {a.shape}")
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def selective_scan(u, delta, A, B, C, D=None, z=None, dt_bias=None,
                   delta_softplus=True, h0=None, return_last_state=False):
    """fp64 selective scan.  u, delta, z: (b, L, d_in); A: (d_in, N);
    B, C: (b, L, N); D, dt_bias: (d_in); h0: (b, d_in, N).
    Returns y (b, L, d_in) [and h_last (b, d_in, N)] as float64 arrays."""
    u = _f64(u)
    b, L, d_in = u.shape
    A = _f64(A)
    N = A.shape[1]
    delta = _f64(delta, (b, L, d_in))
    A = _f64(A, (d_in, N))
    B = _f64(B, (b, L, N))
    C = _f64(C, (b, L, N))
    D = _f64(D, (d_in,))
    z = _f64(z, (b, L, d_in))
    dt_bias = _f64(dt_bias, (d_in,))
    h0 = _f64(h0, (b, d_in, N))
    y = np.empty((b, L, d_in), np.float64)
    h_last = np.empty((b, d_in, N), np.float64) if return_last_state else None
    _load().oracle_selective_scan(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                  _ptr(D), _ptr(z), _ptr(dt_bias), int(bool(delta_softplus)),
                                  _ptr(h0), _ptr(h_last), _ptr(y), b, L, d_in, N)
    return (y, h_last) if return_last_state else y


def selective_scan_bwd(u, delta, A, B, C, dout, D=None, z=None, dt_bias=None,
                       delta_softplus=True, h0=None, dh_last=None):
    """fp64 gradients of sum(dout * y) + sum(dh_last * h_last) for the scan
    of ``selective_scan``.  Returns a dict with du, ddelta (b, L, d_in); dA
    (d_in, N); dB, dC (b, L, N); dD, ddt_bias (d_in); dz (b, L, d_in, only
    with z); dh0 (b, d_in, N)."""
    u = _f64(u)
    b, L, d_in = u.shape
    A = _f64(A)
    N = A.shape[1]
    delta = _f64(delta, (b, L, d_in))
    B = _f64(B, (b, L, N))
    C = _f64(C, (b, L, N))
    D = _f64(D, (d_in,))
    z = _f64(z, (b, L, d_in))
    dt_bias = _f64(dt_bias, (d_in,))
    h0 = _f64(h0, (b, d_in, N))
    dout = _f64(dout, (b, L, d_in))
    dh_last = _f64(dh_last, (b, d_in, N))
    g = dict(du=np.empty((b, L, d_in)), ddelta=np.empty((b, L, d_in)), dA=np.empty((d_in, N)),
             dB=np.empty((b, L, N)), dC=np.empty((b, L, N)), dD=np.empty(d_in),
             dz=np.empty((b, L, d_in)) if z is not None else None,
             ddt_bias=np.empty(d_in), dh0=np.empty((b, d_in, N)))
    rc = _load().oracle_selective_scan_bwd(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
        int(bool(delta_softplus)), _ptr(h0), _ptr(dout), _ptr(dh_last),
        _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]),
        _ptr(g["dD"]), _ptr(g["dz"]), _ptr(g["ddt_bias"]), _ptr(g["dh0"]), b, L, d_in, N)
    if rc != 0:
        raise MemoryError("oracle.selective_scan_bwd: out of memory")
    if z is None:
        del g["dz"]
    return g


def state_update(state, x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True):
    """fp64 one-token update.  state: (b, d_in, N) -- a NEW array is returned,
    the argument is not modified.  x, dt, z: (b, d_in); B, C: (b, N).
    Returns (y (b, d_in), new_state (b, d_in, N))."""
    st = _f64(state).copy()
    b, d_in, N = st.shape
    x = _f64(x, (b, d_in))
    dt = _f64(dt, (b, d_in))
    A = _f64(A, (d_in, N))
    B = _f64(B, (b, N))
    C = _f64(C, (b, N))
    D = _f64(D, (d_in,))
    z = _f64(z, (b, d_in))
    dt_bias = _f64(dt_bias, (d_in,))
    y = np.empty((b, d_in), np.float64)
    _load().oracle_state_update(_ptr(st), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                _ptr(D), _ptr(z), _ptr(dt_bias), int(bool(dt_softplus)),
                                _ptr(y), b, d_in, N)
    return y, st


def conv_step(conv_state, x, weight, bias=None):
    """fp64 causal-conv1d decode step.  conv_state (b, d_in, d_conv) -- a NEW
    array is returned, the argument is not modified; x (b, d_in); weight
    (d_in, d_conv); bias (d_in).  Returns (x_out (b, d_in), new_conv_state)."""
    cs = _f64(conv_state).copy()
    b, d_in, d_conv = cs.shape
    x = _f64(x, (b, d_in))
    weight = _f64(weight, (d_in, d_conv))
    bias = _f64(bias, (d_in,))
    out = np.empty((b, d_in), np.float64)
    _load().oracle_conv_step(_ptr(cs), _ptr(x), _ptr(weight), _ptr(bias), _ptr(out), b, d_in, d_conv)
    return out, cs


ORDERS = {"cross": 0, "snake": 1}


def cross_scan(u, H, W, order="cross"):
    """u (b, H W, d_in) -> xs (b, 4, H W, d_in); order "cross" or "snake"."""
    u = _f64(u)
    b, L, d_in = u.shape
    if L != H * W:
        raise ValueError("oracle.cross_scan: L != H*W")
    xs = np.empty((b, 4, L, d_in), np.float64)
    _load().oracle_cross_scan(_ptr(u), _ptr(xs), b, H, W, d_in, ORDERS[order])
    return xs


def cross_merge(ys, H, W, order="cross"):
    """ys (b, 4, H W, d_in) -> y (b, H W, d_in)."""
    ys = _f64(ys)
    b, K, L, d_in = ys.shape
    if K != 4 or L != H * W:
        raise ValueError("oracle.cross_merge: bad shape")
    y = np.empty((b, L, d_in), np.float64)
    _load().oracle_cross_merge(_ptr(ys), _ptr(y), b, H, W, d_in, ORDERS[order])
    return y


def ss2d_scan(u, delta, A, B, C, H, W, D=None, dt_bias=None, delta_softplus=True,
              order="cross"):
    """fp64 SS2D forward.  u: (b, H W, d_in); delta: (b, 4, H W, d_in);
    A: (4 d_in, N); B, C: (b, 4, H W, N); D, dt_bias: (4 d_in)."""
    u = _f64(u)
    b, L, d_in = u.shape
    A = _f64(A)
    N = A.shape[1]
    delta = _f64(delta, (b, 4, L, d_in))
    A = _f64(A, (4 * d_in, N))
    B = _f64(B, (b, 4, L, N))
    C = _f64(C, (b, 4, L, N))
    D = _f64(D, (4 * d_in,))
    dt_bias = _f64(dt_bias, (4 * d_in,))
    y = np.empty((b, L, d_in), np.float64)
    rc = _load().oracle_ss2d_scan(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C),
                                  _ptr(D), _ptr(dt_bias), int(bool(delta_softplus)),
                                  _ptr(y), b, H, W, d_in, N, ORDERS[order])
    if rc != 0:
        raise MemoryError("oracle.ss2d_scan: allocation failed")
    return y
