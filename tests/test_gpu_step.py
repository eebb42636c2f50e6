"""GPU parity of ssm_state_update (one decode step of Mamba.step(), state in
place) against the fp64 oracle, at steps 1, 10 and 1000 of the decode
workload, plus the closed-form fixed point over the whole state."""
import math

import numpy as np
import pytest
import torch

import oracle
from _helpers import TOL, rel_err, to_cuda, to64
from selective_state_space_25_b200.synthetic import WORKLOADS, scan_inputs, step_inputs

pytestmark = pytest.mark.gpu


def gpu_step(S, g, state, y=None):
    return S.ssm_state_update(state, g["x"], g["dt"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                              dt_bias=g["dt_bias"], y=y)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,d_in,N", [(1, 1, 16), (3, 37, 16), (2, 64, 1), (2, 50, 2), (4, 33, 4),
                                      (2, 40, 8), (2, 24, 32), (1, 16, 64)])
def test_step_shapes(ssm, dtype, b, d_in, N):
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = step_inputs(b, d_in, N, dt, seed=b * 1000 + d_in + N)
    g = to_cuda(inp)
    st = g["state"].clone()
    y_ref, st_ref = oracle.state_update(inp["state"], inp["x"], inp["dt"], inp["A"], inp["B"],
                                        inp["C"], D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"])
    y = gpu_step(ssm, g, st)
    assert rel_err(y, y_ref) <= TOL[dtype]
    assert rel_err(st, st_ref) <= 1e-5


def test_step_misaligned_state_and_no_gate(ssm):
    inp = step_inputs(2, 20, 16, "fp32", seed=3, with_z=False)
    g = to_cuda(inp)
    buf = torch.empty(inp["state"].numel() + 4, device="cuda")
    st = buf[1:1 + inp["state"].numel()].view(inp["state"].shape)   # 4-byte, not 16-byte aligned
    st.copy_(g["state"])
    y = gpu_step(ssm, g, st)
    y_ref, st_ref = oracle.state_update(inp["state"], inp["x"], inp["dt"], inp["A"], inp["B"],
                                        inp["C"], D=inp["D"], dt_bias=inp["dt_bias"])
    assert rel_err(y, y_ref) <= 1e-4 and rel_err(st, st_ref) <= 1e-5


def test_decode_workload_steps_1_10_1000(ssm):
    w = WORKLOADS["mamba-decode-step"]
    d = w.dims
    b, d_in, N, steps = d["b"], d["d_in"], d["N"], d["steps"]
    inp = step_inputs(b, d_in, N, w.dtype, w.seed)
    g = to_cuda(inp)
    st = g["state"].clone()
    y = torch.empty(b, d_in, dtype=torch.bfloat16, device="cuda")
    bsel = [0, 1, 128, b - 1]
    sl = lambda t: t[bsel].contiguous()
    o_st = sl(inp["state"])
    o_in = dict(x=sl(inp["x"]), dt=sl(inp["dt"]), B=sl(inp["B"]), C=sl(inp["C"]), z=sl(inp["z"]))
    done = 0
    for check in (1, 10, steps):
        for _ in range(check - done):
            gpu_step(ssm, g, st, y)
            o_y, o_st = oracle.state_update(o_st, o_in["x"], o_in["dt"], inp["A"], o_in["B"],
                                            o_in["C"], D=inp["D"], z=o_in["z"],
                                            dt_bias=inp["dt_bias"])
        done = check
        torch.cuda.synchronize()
        assert rel_err(y[bsel], o_y) <= 2e-2, check
        # fp32 state: the per-step rounding of exp(delta A) compounds over the
        # decode; 1e-3 bounds 1000 steps of it (the decay memory here is
        # longer than 1000 steps for the smallest delta).
        assert rel_err(st[bsel], o_st) <= 1e-3, check

    # closed form over the WHOLE state: h_k = h* + a^k (h0 - h*), h* = delta B x / (1 - a)
    x = to64(inp["x"])[:, :, None]
    dt = to64(inp["dt"]) + to64(inp["dt_bias"])[None, :]
    delta = np.where(dt > 20, dt, np.log1p(np.exp(dt)))[:, :, None]
    a = np.exp(delta * to64(inp["A"])[None])
    hstar = delta * to64(inp["B"])[:, None, :] * x / (1.0 - a)
    hk = hstar + a ** steps * (to64(inp["state"]) - hstar)
    assert rel_err(st, hk) <= 1e-3


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_prefill_then_decode_handoff(ssm, dtype):
    """A prefill scan over L tokens exports h_last; one decode step from that
    state on token L+1 equals the oracle's scan over all L+1 tokens (the
    cached-state path of Mamba.forward in "代码连连看——mamba")."""
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    b, L, d_in, N = 2, 97, 64, 16
    inp = scan_inputs(b, L + 1, d_in, N, dt, seed=31)
    g = to_cuda(inp)
    pre = lambda t: t[:, :L].contiguous()
    state = torch.empty(b, d_in, N, device="cuda")
    y_pre = ssm.ssm_scan_fwd(pre(g["u"]), pre(g["delta"]), g["A"], pre(g["B"]), pre(g["C"]),
                             D=g["D"], z=pre(g["z"]), dt_bias=g["dt_bias"], h_last=state)
    last = lambda t: t[:, L].contiguous()
    y_tok = ssm.ssm_state_update(state, last(g["u"]), last(g["delta"]), g["A"], last(g["B"]),
                                 last(g["C"]), D=g["D"], z=last(g["z"]), dt_bias=g["dt_bias"])
    y_ref, h_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                         D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                         return_last_state=True)
    tol = TOL[dtype]
    assert rel_err(y_pre, y_ref[:, :L]) <= tol
    assert rel_err(y_tok, y_ref[:, L]) <= tol
    assert rel_err(state, h_ref) <= max(tol, 1e-4)
