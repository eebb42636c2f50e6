"""ss2d_scan_fwd_noalloc: the SS2D entry point for callers that cannot
allocate device memory (a host framework that owns every device buffer, or a
real-time loop that must not call cudaMalloc).  Its large-image accumulator
lives in a 16 MiB array the library reserves on each GPU, so the test calls it
through the C ABI on an image whose accumulator does not fit in shared
memory, twice in a row on different inputs, and compares each result with
ss2d_scan_fwd given a workspace.  This file sorts last so that a run that
stops at the first failure has already run every other test."""
import ctypes

import pytest
import torch

from _helpers import TOL, rel_err, to_cuda
from selective_state_space_25_b200.synthetic import ss2d_inputs

pytestmark = pytest.mark.gpu

P, I64, INT = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
SCRATCH_BYTES = 16 << 20


def _noalloc(S):
    fn = S.lib().ss2d_scan_fwd_noalloc
    fn.argtypes = [P] * 7 + [INT, P] + [I64] * 5 + [INT, P]
    fn.restype = INT
    return fn


def _call(fn, S, g, y, b, H, W, d_in):
    return fn(g["u"].data_ptr(), g["delta"].data_ptr(), g["A"].data_ptr(), g["B"].data_ptr(),
              g["C"].data_ptr(), g["D"].data_ptr(), g["dt_bias"].data_ptr(), 1, y.data_ptr(),
              b, H, W, d_in, 1, S.SSM_BF16, torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls(ssm):
    b, H, W, d_in = 2, 80, 81, 16          # 6480 pixels: the accumulator needs scratch
    need = ssm.ss2d_scan_fwd_workspace_bytes(b, H, W, d_in, 1)
    assert 0 < need <= SCRATCH_BYTES
    fn = _noalloc(ssm)
    for seed in (21, 22):                  # two calls in a row, different inputs
        g = to_cuda(ss2d_inputs(b, H, W, d_in, 1, "bf16", seed=seed, with_dt_bias=True))
        ref = ssm.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"],
                                dt_bias=g["dt_bias"])
        y = torch.full_like(g["u"], float("nan"))
        st = _call(fn, ssm, g, y, b, H, W, d_in)
        assert st == ssm.SSM_OK, ssm.last_error()
        torch.cuda.synchronize()
        assert rel_err(y, ref) <= TOL[torch.bfloat16]


def test_noalloc_small_image_and_size_limit(ssm):
    fn = _noalloc(ssm)
    # an image whose accumulator fits in shared memory uses no scratch
    b, H, W, d_in = 2, 9, 11, 8
    g = to_cuda(ss2d_inputs(b, H, W, d_in, 1, "bf16", seed=23, with_dt_bias=True))
    ref = ssm.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"],
                            dt_bias=g["dt_bias"])
    y = torch.empty_like(g["u"])
    assert _call(fn, ssm, g, y, b, H, W, d_in) == ssm.SSM_OK
    torch.cuda.synchronize()
    assert rel_err(y, ref) <= TOL[torch.bfloat16]
    # beyond the static maximum: rejected before anything is launched
    big = dict(g)
    st = fn(g["u"].data_ptr(), g["delta"].data_ptr(), g["A"].data_ptr(), g["B"].data_ptr(),
            g["C"].data_ptr(), None, None, 1, y.data_ptr(), 64, 100, 100, 192, 1, ssm.SSM_BF16, None)
    assert st == ssm.SSM_ERR_WORKSPACE
    assert "static" in ssm.last_error()
    del big
