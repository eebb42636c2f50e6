"""GPU parity of ssm_state_update (one decode step of Mamba.step(), state in
place) against the fp64 oracle, at steps 1, 10 and 1000 of the decode
workload, plus the closed-form fixed point over the whole state."""
import math

import numpy as np
import pytest
import torch

import oracle
from _helpers import TOL, rel_err, to_cuda, to64
from selective_state_space_25_b200.synthetic import WORKLOADS, conv_inputs, scan_inputs, step_inputs

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


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_step_state_16_but_not_32_byte_aligned(ssm, dtype):
    """N = 16 with a state 16- but not 32-byte aligned: the one-thread-per-channel
    kernel needs 32-byte vectors, so the four-lanes-per-channel kernel runs."""
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = step_inputs(3, 45, 16, dt, seed=21)
    g = to_cuda(inp)
    n = inp["state"].numel()
    raw = torch.empty(n + 16, device="cuda")
    base = (raw.data_ptr() // 4) % 8                      # floats past a 32-byte boundary
    off = (4 - base) % 8                                  # land 16 bytes past one
    st = raw[off:off + n].view(inp["state"].shape)
    assert st.data_ptr() % 32 == 16
    st.copy_(g["state"])
    y = gpu_step(ssm, g, st)
    y_ref, st_ref = oracle.state_update(inp["state"], inp["x"], inp["dt"], inp["A"], inp["B"],
                                        inp["C"], D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"])
    assert rel_err(y, y_ref) <= TOL[dtype] and rel_err(st, st_ref) <= 1e-5


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


# ------------------------------------------------ fused causal-conv1d decode step
def gpu_conv_step(S, g, c, conv_state, state, y=None):
    return S.ssm_conv_state_update(conv_state, c["conv_weight"], state, g["x"], g["dt"], g["A"],
                                   g["B"], g["C"], conv_bias=c["conv_bias"], D=g["D"], z=g["z"],
                                   dt_bias=g["dt_bias"], y=y)


def oracle_conv_then_step(inp, c, conv_state, state):
    """Mamba.step() order: the conv step on x, then the SSM step on its output."""
    xc, cs = oracle.conv_step(conv_state, inp["x"], c["conv_weight"], c["conv_bias"])
    y, st = oracle.state_update(state, xc, inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                z=inp["z"], dt_bias=inp["dt_bias"])
    return y, st, cs


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,d_in,N,d_conv", [(1, 1, 16, 4), (3, 37, 16, 4), (2, 64, 1, 2),
                                             (4, 33, 4, 3), (2, 40, 8, 1), (2, 24, 32, 4),
                                             (1, 16, 64, 8), (2, 50, 2, 5)])
def test_conv_step_shapes(ssm, dtype, b, d_in, N, d_conv):
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = step_inputs(b, d_in, N, dt, seed=7 * b + d_in + N)
    c = conv_inputs(b, d_in, d_conv, dt, seed=d_conv + d_in)
    g, gc = to_cuda(inp), to_cuda(c)
    st, cs = g["state"].clone(), gc["conv_state"].clone()
    y = gpu_conv_step(ssm, g, gc, cs, st)
    y_ref, st_ref, cs_ref = oracle_conv_then_step(inp, c, c["conv_state"], inp["state"])
    assert rel_err(y, y_ref) <= TOL[dtype]
    assert rel_err(st, st_ref) <= 1e-5
    np.testing.assert_array_equal(to64(cs), cs_ref)      # the window only moves stored values


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_conv_step_window_not_vector_aligned(ssm, dtype):
    """d_conv = 4 with the window one element off a vector boundary: the
    one-thread-per-channel kernel reads and writes it tap by tap."""
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = step_inputs(2, 33, 16, dt, seed=31)
    c = conv_inputs(2, 33, 4, dt, seed=32)
    g, gc = to_cuda(inp), to_cuda(c)
    st = g["state"].clone()
    n = c["conv_state"].numel()
    raw = torch.empty(n + 1, dtype=gc["conv_state"].dtype, device="cuda")
    cs = raw[1:1 + n].view(c["conv_state"].shape)
    assert cs.data_ptr() % (4 * cs.element_size()) != 0
    cs.copy_(gc["conv_state"])
    y = gpu_conv_step(ssm, g, gc, cs, st)
    y_ref, st_ref, cs_ref = oracle_conv_then_step(inp, c, c["conv_state"], inp["state"])
    assert rel_err(y, y_ref) <= TOL[dtype] and rel_err(st, st_ref) <= 1e-5
    np.testing.assert_array_equal(to64(cs), cs_ref)


def test_conv_step_no_bias_no_gate_misaligned(ssm):
    """Optional conv bias, z and D absent; a 4-byte-aligned state takes the
    scalar kernel."""
    inp = step_inputs(2, 20, 16, "fp32", seed=9, with_z=False)
    inp["D"] = None
    c = conv_inputs(2, 20, 4, "fp32", seed=10, with_bias=False)
    g, gc = to_cuda(inp), to_cuda(c)
    buf = torch.empty(inp["state"].numel() + 4, device="cuda")
    st = buf[1:1 + inp["state"].numel()].view(inp["state"].shape)
    st.copy_(g["state"])
    cs = gc["conv_state"].clone()
    y = gpu_conv_step(ssm, g, gc, cs, st)
    y_ref, st_ref, cs_ref = oracle_conv_then_step(inp, c, c["conv_state"], inp["state"])
    assert rel_err(y, y_ref) <= 1e-4 and rel_err(st, st_ref) <= 1e-5
    np.testing.assert_array_equal(to64(cs), cs_ref)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_conv_step_decode_sequence(ssm, dtype):
    """Twelve decode steps with fresh tokens each step: the window carries
    tokens across steps exactly as the oracle's does."""
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    b, d_in, N, d_conv = 3, 48, 16, 4
    c = conv_inputs(b, d_in, d_conv, dt, seed=21)
    gc = to_cuda(c)
    cs, o_cs = gc["conv_state"].clone(), c["conv_state"]
    first = step_inputs(b, d_in, N, dt, seed=22)
    st, o_st = to_cuda(first)["state"].clone(), first["state"]
    for k in range(12):
        inp = step_inputs(b, d_in, N, dt, seed=100 + k)
        g = to_cuda(inp)
        y = gpu_conv_step(ssm, g, gc, cs, st)
        o_y, o_st, o_cs = oracle_conv_then_step(inp, c, o_cs, o_st)
        assert rel_err(y, o_y) <= TOL[dtype], k
        np.testing.assert_array_equal(to64(cs), o_cs)
    assert rel_err(st, o_st) <= 1e-5


def test_conv_step_rejects_bad_d_conv(ssm):
    inp = to_cuda(step_inputs(1, 8, 16, "fp32", seed=1))
    for d_conv in (0, 9):
        cs = torch.zeros(1, 8, max(d_conv, 1), device="cuda")
        w = torch.zeros(8, max(d_conv, 1), device="cuda")
        st = ssm.lib().ssm_conv_state_update(
            ssm._ptr(cs), ssm._ptr(w), None, d_conv, ssm._ptr(inp["state"]), ssm._ptr(inp["x"]),
            ssm._ptr(inp["dt"]), ssm._ptr(inp["A"]), ssm._ptr(inp["B"]), ssm._ptr(inp["C"]), None,
            None, None, 1, ssm._ptr(torch.empty(1, 8, device="cuda")), 1, 8, 16, 0, None)
        assert st != 0 and "d_conv" in ssm.last_error()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,d_in,N", [(3, 1000, 16), (8, 8192, 16), (5, 40, 4), (2, 616, 64)])
def test_step_large_and_ragged(ssm, dtype, b, d_in, N):
    """Channel counts that are not multiples of a CTA's channels, more
    channels than one wave of CTAs covers, N = 4 and N = 64; three steps in a
    row from the updated state."""
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = step_inputs(b, d_in, N, dt, seed=b + d_in + N)
    g = to_cuda(inp)
    st = g["state"].clone()
    o_st = inp["state"]
    for _ in range(3):
        y = gpu_step(ssm, g, st)
        y_ref, o_st = oracle.state_update(o_st, inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"],
                                          D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"])
        assert rel_err(y, y_ref) <= TOL[dtype]
    assert rel_err(st, o_st) <= 1e-5
    ssm.check_device_errors()
