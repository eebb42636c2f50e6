"""Thin Python binding of libssmscan.so (include/ssmscan.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, their data pointers and the current CUDA stream are passed to the
C ABI, and a non-OK status becomes an ``SsmError``.  Outputs (and the
workspace the library asks for) are allocated here with torch when the caller
does not pass them; every step of the computation runs in the library's
kernels.  Importing this module fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# SSM_DEBUG_BOUNDS=1 selects the debug-bounds build (every kernel checks its
# global indices and records misses for check_device_errors)
DEBUG_BOUNDS = os.environ.get("SSM_DEBUG_BOUNDS", "") == "1"
LIB_PATH = os.path.join(_PKG, "libssmscan_debug.so" if DEBUG_BOUNDS else "libssmscan.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "ssmscan.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m selective_state_space_25_b200.build` "
        "(the CUDA path has no fallback)")

_lib = ctypes.CDLL(LIB_PATH)

SSM_OK, SSM_ERR_INVALID_ARG, SSM_ERR_UNSUPPORTED, SSM_ERR_WORKSPACE, SSM_ERR_CUDA, \
    SSM_ERR_DEVICE_TIMEOUT, SSM_ERR_DEVICE_BOUNDS = range(7)
SSM_F32, SSM_BF16 = 0, 1
_STATUS = {0: "SSM_OK", 1: "SSM_ERR_INVALID_ARG", 2: "SSM_ERR_UNSUPPORTED", 3: "SSM_ERR_WORKSPACE",
           4: "SSM_ERR_CUDA", 5: "SSM_ERR_DEVICE_TIMEOUT", 6: "SSM_ERR_DEVICE_BOUNDS"}

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_SZ = ctypes.c_size_t

_lib.ssm_last_error.restype = ctypes.c_char_p
_lib.ssm_version.restype = ctypes.c_char_p
_lib.ssm_scan_fwd_workspace_bytes.argtypes = [_I64] * 4
_lib.ssm_scan_fwd_workspace_bytes.restype = _SZ
_lib.ssm_scan_fwd.argtypes = [_P] * 8 + [_INT, _P, _P, _P] + [_I64] * 4 + [_INT, _P, _SZ, _P]
_lib.ssm_scan_fwd.restype = _INT
_lib.ssm_scan_bwd_workspace_bytes.argtypes = [_I64] * 4
_lib.ssm_scan_bwd_workspace_bytes.restype = _SZ
_lib.ssm_scan_bwd_fast_workspace_bytes.argtypes = [_I64] * 4
_lib.ssm_scan_bwd_fast_workspace_bytes.restype = _SZ
_lib.ssm_scan_bwd_saved_workspace_bytes.argtypes = [_I64] * 4
_lib.ssm_scan_bwd_saved_workspace_bytes.restype = _SZ
_lib.ssm_scan_bwd.argtypes = [_P] * 8 + [_INT] + [_P] * 12 + [_I64] * 4 + [_INT, _P, _SZ, _P]
_lib.ssm_scan_bwd.restype = _INT
_lib.ssm_scan_fwd_save.argtypes = [_P] * 8 + [_INT, _P, _P, _P, _P, _SZ] + [_I64] * 4 + [_INT, _P]
_lib.ssm_scan_fwd_save.restype = _INT
_lib.ssm_scan_fwd_save_ex.argtypes = _lib.ssm_scan_fwd_save.argtypes[:-1] + [_P, _SZ, _P]
_lib.ssm_scan_fwd_save_ex.restype = _INT
_lib.ssm_scan_bwd_saved.argtypes = ([_P] * 8 + [_INT] + [_P] * 11 + [_I64] * 4
                                    + [_INT, _P, _SZ, _P])
_lib.ssm_scan_bwd_saved.restype = _INT
_lib.ssm_scan_bwd_saved_ex.argtypes = (_lib.ssm_scan_bwd_saved.argtypes[:-1]
                                       + [_P, _SZ, _P])
_lib.ssm_scan_bwd_saved_ex.restype = _INT
_lib.ss2d_scan_fwd_workspace_bytes.argtypes = [_I64] * 5
_lib.ss2d_scan_fwd_workspace_bytes.restype = _SZ
_lib.ss2d_scan_fwd_fast_workspace_bytes.argtypes = [_I64] * 5
_lib.ss2d_scan_fwd_fast_workspace_bytes.restype = _SZ
_lib.ss2d_scan_fwd.argtypes = [_P] * 7 + [_INT, _P] + [_I64] * 5 + [_INT, _P, _SZ, _P]
_lib.ss2d_scan_fwd.restype = _INT
_lib.ssm_state_update.argtypes = [_P] * 9 + [_INT, _P] + [_I64] * 3 + [_INT, _P]
_lib.ssm_state_update.restype = _INT
_lib.ssm_conv_state_update.argtypes = [_P, _P, _P, _I64] + [_P] * 9 + [_INT, _P] + [_I64] * 3 + [_INT, _P]
_lib.ssm_conv_state_update.restype = _INT
_lib.ss2d_cross_scan.argtypes = [_P, _P] + [_I64] * 4 + [_INT, _P]
_lib.ss2d_cross_scan.restype = _INT
_lib.ss2d_cross_merge.argtypes = [_P, _P] + [_I64] * 4 + [_INT, _P]
_lib.ss2d_cross_merge.restype = _INT
_lib.ss2d_scan_fwd_ex.argtypes = [_P] * 7 + [_INT, _P] + [_I64] * 5 + [_INT, _INT, _P, _SZ, _P]
_lib.ss2d_scan_fwd_ex.restype = _INT
_lib.ss2d_cross_scan_ex.argtypes = [_P, _P] + [_I64] * 4 + [_INT, _INT, _P]
_lib.ss2d_cross_scan_ex.restype = _INT
_lib.ss2d_cross_merge_ex.argtypes = [_P, _P] + [_I64] * 4 + [_INT, _INT, _P]
_lib.ss2d_cross_merge_ex.restype = _INT
SS2D_ORDERS = {"cross": 0, "snake": 1}
_lib.ssm_check_device_errors.argtypes = [_P]
_lib.ssm_check_device_errors.restype = _INT
_lib.ssm_debug_bounds_enabled.argtypes = []
_lib.ssm_debug_bounds_enabled.restype = _INT
_lib.ssm_debug_bounds_self_test.argtypes = [_P]
_lib.ssm_debug_bounds_self_test.restype = _INT


class SsmError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libssmscan.so (for tests that call the C ABI directly)."""
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/ssmscan.h declares."""
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssm_\w+|ss2d_\w+)\s*\(", text)))


def version() -> str:
    return _lib.ssm_version().decode()


def last_error() -> str:
    return _lib.ssm_last_error().decode()


def _check(status: int, where: str) -> None:
    if status != SSM_OK:
        raise SsmError(status, where, last_error())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SSM_BF16
    if t.dtype == torch.float32:
        return SSM_F32
    raise TypeError(f"unsupported activation dtype {t.dtype} (bf16 or fp32)")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, name, shape, dtype, device):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def ssm_scan_fwd_workspace_bytes(b: int, L: int, d_in: int, d_state: int) -> int:
    return int(_lib.ssm_scan_fwd_workspace_bytes(b, L, d_in, d_state))


def ssm_scan_fwd(u, delta, A, B, C, D=None, z=None, dt_bias=None, delta_softplus=True,
                 h0=None, h_last=None, y=None, workspace=None, stream=None, chunk_states=None):
    """Selective scan forward (see include/ssmscan.h).  u, delta, z: (b, L, d_in);
    A: (d_in, N) fp32; B, C: (b, L, N); D, dt_bias: (d_in,) fp32; h0, h_last:
    (b, d_in, N) fp32.  Returns y (b, L, d_in).  With ``chunk_states`` (a
    device buffer of ssm_scan_bwd_workspace_bytes(...) bytes) the forward
    also saves the chunk-start states for ssm_scan_bwd(..., states=...).
    Unless ``workspace`` is given, the split scan's workspace
    (ssm_scan_fwd_workspace_bytes) is allocated when it is not 0."""
    if u.dim() != 3:
        raise ValueError("u must be (b, L, d_in)")
    b, L, d_in = u.shape
    N = A.shape[-1]
    dev, act = u.device, u.dtype
    f32 = torch.float32
    _need(u, "u", (b, L, d_in), act, dev)
    _need(delta, "delta", (b, L, d_in), act, dev)
    _need(A, "A", (d_in, N), f32, dev)
    _need(B, "B", (b, L, N), act, dev)
    _need(C, "C", (b, L, N), act, dev)
    _need(D, "D", (d_in,), f32, dev)
    _need(z, "z", (b, L, d_in), act, dev)
    _need(dt_bias, "dt_bias", (d_in,), f32, dev)
    _need(h0, "h0", (b, d_in, N), f32, dev)
    _need(h_last, "h_last", (b, d_in, N), f32, dev)
    if y is None:
        y = torch.empty_like(u)
    _need(y, "y", (b, L, d_in), act, dev)
    ws_bytes = ssm_scan_fwd_workspace_bytes(b, L, d_in, N)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if chunk_states is not None:
        st = _lib.ssm_scan_fwd_save_ex(
            _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
            int(bool(delta_softplus)), _ptr(h0), _ptr(h_last), _ptr(y), _ptr(chunk_states),
            chunk_states.numel() * chunk_states.element_size(), b, L, d_in, N, _dtype_code(u),
            _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
            _stream(stream))
        _check(st, "ssm_scan_fwd_save")
        return y
    st = _lib.ssm_scan_fwd(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                           _ptr(dt_bias), int(bool(delta_softplus)), _ptr(h0), _ptr(h_last),
                           _ptr(y), b, L, d_in, N, _dtype_code(u), _ptr(workspace),
                           0 if workspace is None else workspace.numel() * workspace.element_size(),
                           _stream(stream))
    _check(st, "ssm_scan_fwd")
    return y


def ssm_scan_bwd_workspace_bytes(b: int, L: int, d_in: int, d_state: int) -> int:
    return int(_lib.ssm_scan_bwd_workspace_bytes(b, L, d_in, d_state))


def ssm_scan_bwd_fast_workspace_bytes(b: int, L: int, d_in: int, d_state: int) -> int:
    return int(_lib.ssm_scan_bwd_fast_workspace_bytes(b, L, d_in, d_state))


def ssm_scan_bwd_saved_workspace_bytes(b: int, L: int, d_in: int, d_state: int) -> int:
    return int(_lib.ssm_scan_bwd_saved_workspace_bytes(b, L, d_in, d_state))


def ssm_scan_bwd(u, delta, A, B, C, dout, D=None, z=None, dt_bias=None, delta_softplus=True,
                 h0=None, dh_last=None, want_dh0=False, workspace=None, stream=None, out=None,
                 states=None):
    """Gradients of sum(dout * y) [+ sum(dh_last * h_last)] for ssm_scan_fwd
    with the same inputs.  Returns a dict: du, ddelta, dz (activation dtype,
    (b, L, d_in); dz only with z); dA (d_in, N), dB, dC (b, L, N), dD,
    ddt_bias (d_in) in fp32; dh0 (b, d_in, N) fp32 when want_dh0.  ``out``
    (a dict returned by an earlier call with the same shapes) is refilled
    in place instead of allocating.  ``states``: the chunk_states buffer a
    forward with the same inputs filled (ssm_scan_fwd(..., chunk_states=));
    the backward then starts from it (ssm_scan_bwd_saved_ex, with ``workspace``
    or an allocated one for its split when channels are few) and h0 is unused."""
    b, L, d_in = u.shape
    N = A.shape[1]
    dev, act, f32 = u.device, u.dtype, torch.float32
    _need(u, "u", (b, L, d_in), act, dev)
    _need(delta, "delta", (b, L, d_in), act, dev)
    _need(A, "A", (d_in, N), f32, dev)
    _need(B, "B", (b, L, N), act, dev)
    _need(C, "C", (b, L, N), act, dev)
    _need(dout, "dout", (b, L, d_in), act, dev)
    _need(D, "D", (d_in,), f32, dev)
    _need(z, "z", (b, L, d_in), act, dev)
    _need(dt_bias, "dt_bias", (d_in,), f32, dev)
    _need(h0, "h0", (b, d_in, N), f32, dev)
    _need(dh_last, "dh_last", (b, d_in, N), f32, dev)
    if out is not None:
        g = {k: out.get(k) for k in ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddt_bias", "dh0")}
        for k, shp, dt in (("du", (b, L, d_in), act), ("ddelta", (b, L, d_in), act),
                           ("dz", (b, L, d_in), act), ("dA", (d_in, N), f32),
                           ("dB", (b, L, N), f32), ("dC", (b, L, N), f32), ("dD", (d_in,), f32),
                           ("ddt_bias", (d_in,), f32), ("dh0", (b, d_in, N), f32)):
            _need(g[k], k, shp, dt, dev)
    else:
        g = dict(du=torch.empty_like(u), ddelta=torch.empty_like(u),
                 dz=torch.empty_like(u) if z is not None else None,
                 dA=torch.empty((d_in, N), dtype=f32, device=dev),
                 dB=torch.empty((b, L, N), dtype=f32, device=dev),
                 dC=torch.empty((b, L, N), dtype=f32, device=dev),
                 dD=torch.empty(d_in, dtype=f32, device=dev),
                 ddt_bias=torch.empty(d_in, dtype=f32, device=dev),
                 dh0=torch.empty((b, d_in, N), dtype=f32, device=dev) if want_dh0 else None)
    if states is not None:
        aux = ssm_scan_bwd_saved_workspace_bytes(b, L, d_in, N)
        if workspace is None and aux > 0:
            workspace = torch.empty(aux, dtype=torch.uint8, device=dev)
        st = _lib.ssm_scan_bwd_saved_ex(
            _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(dt_bias),
            int(bool(delta_softplus)), _ptr(dout), _ptr(dh_last), _ptr(g["du"]),
            _ptr(g["ddelta"]), _ptr(g["dA"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]),
            _ptr(g["dz"]), _ptr(g["ddt_bias"]), _ptr(g["dh0"]), b, L, d_in, N, _dtype_code(u),
            _ptr(states), states.numel() * states.element_size(), _ptr(workspace),
            0 if workspace is None else workspace.numel() * workspace.element_size(),
            _stream(stream))
        _check(st, "ssm_scan_bwd_saved")
        return {k: v for k, v in g.items() if v is not None}
    need = ssm_scan_bwd_fast_workspace_bytes(b, L, d_in, N)  # the fastest path's
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.ssm_scan_bwd(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                           _ptr(dt_bias), int(bool(delta_softplus)), _ptr(h0), _ptr(dout),
                           _ptr(dh_last), _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]),
                           _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]), _ptr(g["dz"]),
                           _ptr(g["ddt_bias"]), _ptr(g["dh0"]), b, L, d_in, N, _dtype_code(u),
                           _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "ssm_scan_bwd")
    return {k: v for k, v in g.items() if v is not None}


def ss2d_scan_fwd_workspace_bytes(b: int, H: int, W: int, d_in: int, d_state: int) -> int:
    return int(_lib.ss2d_scan_fwd_workspace_bytes(b, H, W, d_in, d_state))


def ss2d_scan_fwd_fast_workspace_bytes(b: int, H: int, W: int, d_in: int, d_state: int) -> int:
    return int(_lib.ss2d_scan_fwd_fast_workspace_bytes(b, H, W, d_in, d_state))


def ss2d_scan_fwd(u, delta, A, B, C, H, W, D=None, dt_bias=None, delta_softplus=True, y=None,
                  workspace=None, stream=None, order="cross"):
    """SS2D forward.  u: (b, H W, d_in); delta: (b, 4, H W, d_in); A: (4 d_in, N)
    fp32; B, C: (b, 4, H W, N); D, dt_bias: (4 d_in,) fp32; order "cross" or
    "snake".  Returns y (b, H W, d_in).  Without a ``workspace`` the binding
    allocates the one that lets the call take its fastest path."""
    b, L, d_in = u.shape
    N = A.shape[-1]
    if L != H * W:
        raise ValueError("u.shape[1] must be H*W")
    dev, act, f32 = u.device, u.dtype, torch.float32
    _need(delta, "delta", (b, 4, L, d_in), act, dev)
    _need(A, "A", (4 * d_in, N), f32, dev)
    _need(B, "B", (b, 4, L, N), act, dev)
    _need(C, "C", (b, 4, L, N), act, dev)
    _need(D, "D", (4 * d_in,), f32, dev)
    _need(dt_bias, "dt_bias", (4 * d_in,), f32, dev)
    _need(u, "u", (b, L, d_in), act, dev)
    if y is None:
        y = torch.empty_like(u)
    _need(y, "y", (b, L, d_in), act, dev)
    ws_bytes = ss2d_scan_fwd_fast_workspace_bytes(b, H, W, d_in, N)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = _lib.ss2d_scan_fwd_ex(_ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                               _ptr(dt_bias), int(bool(delta_softplus)), _ptr(y), b, H, W, d_in, N,
                               SS2D_ORDERS[order], _dtype_code(u), _ptr(workspace),
                            0 if workspace is None else workspace.numel() * workspace.element_size(),
                            _stream(stream))
    _check(st, "ss2d_scan_fwd")
    return y


def ssm_state_update(ssm_state, x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True,
                     y=None, stream=None):
    """One decode step; ssm_state (b, d_in, N) fp32 is updated in place.
    x, dt, z: (b, d_in); B, C: (b, N).  Returns y (b, d_in)."""
    b, d_in, N = ssm_state.shape
    dev, act, f32 = x.device, x.dtype, torch.float32
    _need(ssm_state, "ssm_state", (b, d_in, N), f32, dev)
    _need(x, "x", (b, d_in), act, dev)
    _need(dt, "dt", (b, d_in), act, dev)
    _need(A, "A", (d_in, N), f32, dev)
    _need(B, "B", (b, N), act, dev)
    _need(C, "C", (b, N), act, dev)
    _need(D, "D", (d_in,), f32, dev)
    _need(z, "z", (b, d_in), act, dev)
    _need(dt_bias, "dt_bias", (d_in,), f32, dev)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", (b, d_in), act, dev)
    st = _lib.ssm_state_update(_ptr(ssm_state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                               _ptr(D), _ptr(z), _ptr(dt_bias), int(bool(dt_softplus)), _ptr(y),
                               b, d_in, N, _dtype_code(x), _stream(stream))
    _check(st, "ssm_state_update")
    return y


def ssm_conv_state_update(conv_state, conv_weight, ssm_state, x, dt, A, B, C, conv_bias=None,
                          D=None, z=None, dt_bias=None, dt_softplus=True, y=None, stream=None):
    """One decode step with the causal-conv1d step in front; conv_state
    (b, d_in, d_conv) in the activation dtype and ssm_state (b, d_in, N) fp32
    are updated in place.  conv_weight (d_in, d_conv) fp32.  Returns y (b, d_in)."""
    b, d_in, N = ssm_state.shape
    d_conv = conv_state.shape[-1]
    dev, act, f32 = x.device, x.dtype, torch.float32
    _need(conv_state, "conv_state", (b, d_in, d_conv), act, dev)
    _need(conv_weight, "conv_weight", (d_in, d_conv), f32, dev)
    _need(conv_bias, "conv_bias", (d_in,), f32, dev)
    _need(ssm_state, "ssm_state", (b, d_in, N), f32, dev)
    _need(x, "x", (b, d_in), act, dev)
    _need(dt, "dt", (b, d_in), act, dev)
    _need(A, "A", (d_in, N), f32, dev)
    _need(B, "B", (b, N), act, dev)
    _need(C, "C", (b, N), act, dev)
    _need(D, "D", (d_in,), f32, dev)
    _need(z, "z", (b, d_in), act, dev)
    _need(dt_bias, "dt_bias", (d_in,), f32, dev)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", (b, d_in), act, dev)
    st = _lib.ssm_conv_state_update(_ptr(conv_state), _ptr(conv_weight), _ptr(conv_bias), d_conv,
                                    _ptr(ssm_state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
                                    _ptr(D), _ptr(z), _ptr(dt_bias), int(bool(dt_softplus)),
                                    _ptr(y), b, d_in, N, _dtype_code(x), _stream(stream))
    _check(st, "ssm_conv_state_update")
    return y


def ss2d_cross_scan(u, H, W, xs=None, stream=None, order="cross"):
    """xs[b, k, l, d] = u[b, p_k(l), d]; u (b, H W, d_in) -> xs (b, 4, H W, d_in)."""
    b, L, d_in = u.shape
    if xs is None:
        xs = torch.empty((b, 4, L, d_in), dtype=u.dtype, device=u.device)
    _need(u, "u", (b, L, d_in), u.dtype, u.device)
    _need(xs, "xs", (b, 4, L, d_in), u.dtype, u.device)
    _check(_lib.ss2d_cross_scan_ex(_ptr(u), _ptr(xs), b, H, W, d_in, SS2D_ORDERS[order],
                                   _dtype_code(u), _stream(stream)), "ss2d_cross_scan")
    return xs


def ss2d_cross_merge(ys, H, W, y=None, stream=None, order="cross"):
    """y[b, p, d] = sum_k ys[b, k, l_k(p), d]; ys (b, 4, H W, d_in) -> y (b, H W, d_in)."""
    b, K, L, d_in = ys.shape
    if y is None:
        y = torch.empty((b, L, d_in), dtype=ys.dtype, device=ys.device)
    _need(ys, "ys", (b, 4, L, d_in), ys.dtype, ys.device)
    _need(y, "y", (b, L, d_in), ys.dtype, ys.device)
    _check(_lib.ss2d_cross_merge_ex(_ptr(ys), _ptr(y), b, H, W, d_in, SS2D_ORDERS[order],
                                    _dtype_code(ys), _stream(stream)), "ss2d_cross_merge")
    return y


def check_device_errors(stream=None) -> None:
    """Synchronise and raise if a kernel reported a device-side error."""
    _check(_lib.ssm_check_device_errors(_stream(stream)), "ssm_check_device_errors")


def debug_bounds_enabled() -> bool:
    """True when the loaded library is the debug-bounds build."""
    return bool(_lib.ssm_debug_bounds_enabled())


def debug_bounds_self_test(stream=None) -> int:
    """Enqueue the debug-bounds build's self-test (one index one past its
    range: recorded, access skipped); returns the status of the call."""
    return int(_lib.ssm_debug_bounds_self_test(_stream(stream)))
