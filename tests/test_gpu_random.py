"""Seeded random configurations of every kernel family against the fp64 oracle.

Sizes, d_state, dtype, the optional terms (gate, skip, bias, start state,
softplus) and the SS2D order are drawn together, so combinations the
hand-picked shapes of the other files do not list still meet the same
tolerances.  Every case is a fixed seed: a failure names its draw."""
import random

import numpy as np
import pytest
import torch

import oracle
from _helpers import TOL, rel_err, to64, to_cuda
from selective_state_space_25_b200.synthetic import (conv_inputs, scan_inputs, ss2d_inputs,
                                                      step_inputs)

pytestmark = pytest.mark.gpu

STATES = (1, 2, 4, 8, 16, 32, 64)


def _seeds(n, base):
    r = random.Random(base)
    return [r.getrandbits(31) for _ in range(n)]


def _dtype(r):
    return r.choice([("bf16", torch.bfloat16), ("fp32", torch.float32)])


@pytest.mark.parametrize("seed", _seeds(200, 11))
def test_random_scan_forward(ssm, seed):
    r = random.Random(seed)
    b, L, d_in, N = r.randint(1, 3), r.randint(1, 300), r.randint(1, 96), r.choice(STATES)
    dt, dtype = _dtype(r)
    softplus = r.random() < 0.8
    inp = scan_inputs(b, L, d_in, N, dt, seed=seed, with_z=r.random() < 0.7,
                      with_D=r.random() < 0.7, with_dt_bias=r.random() < 0.7,
                      with_h0=r.random() < 0.5)
    if not softplus:  # delta must stay positive for the state to decay
        inp["delta"] = inp["delta"].abs()
        inp["dt_bias"] = None
    g = to_cuda(inp)
    hl = torch.empty(b, d_in, N, device="cuda")
    y = ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                         dt_bias=g["dt_bias"], delta_softplus=softplus, h0=g["h0"], h_last=hl)
    y_ref, h_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                         D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                         h0=inp["h0"], delta_softplus=softplus,
                                         return_last_state=True)
    what = (b, L, d_in, N, dt, softplus)
    assert rel_err(y, y_ref) <= TOL[dtype], what
    assert rel_err(hl, h_ref) <= 1e-4, what


@pytest.mark.parametrize("seed", _seeds(120, 12))
def test_random_scan_backward(ssm, seed):
    r = random.Random(seed)
    b, L, d_in, N = r.randint(1, 2), r.randint(1, 120), r.randint(1, 48), r.choice(STATES)
    dt, dtype = _dtype(r)
    inp = scan_inputs(b, L, d_in, N, dt, seed=seed, with_z=r.random() < 0.7,
                      with_D=r.random() < 0.7, with_dt_bias=r.random() < 0.7,
                      with_h0=r.random() < 0.5)
    gd = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(b, L, d_in, generator=gd).to(dtype)
    dhl = torch.randn(b, d_in, N, generator=gd) if r.random() < 0.5 else None
    g = to_cuda(inp)
    kw = dict(D=g["D"], z=g["z"], dt_bias=g["dt_bias"], h0=g["h0"],
              dh_last=None if dhl is None else dhl.cuda(), want_dh0=True)
    if r.random() < 0.5:  # the training split: the forward saves the states
        states = torch.empty(ssm.ssm_scan_bwd_workspace_bytes(b, L, d_in, N) // 4, device="cuda")
        ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                         dt_bias=g["dt_bias"], h0=g["h0"], chunk_states=states)
        kw["states"] = states
    got = ssm.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout.cuda(), **kw)
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dout,
                                    D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                    h0=inp["h0"], dh_last=dhl)
    what = (b, L, d_in, N, dt, "states" in kw)
    for k in ref:
        if k not in got or got[k] is None:
            continue
        tol = TOL[dtype] if k in ("du", "ddelta", "dz") else (1e-4 if dtype == torch.float32 else 2e-4)
        assert rel_err(got[k], ref[k]) <= tol, (k,) + what


@pytest.mark.parametrize("seed", _seeds(60, 15))
def test_random_split_paths(ssm, seed):
    """Long sequences over few channels: the split forward scan and the split
    backward (self-contained, or from saved states), which the binding's
    default workspaces select, on random sizes, alignments and options."""
    r = random.Random(seed)
    b, L, N = r.randint(1, 2), r.randint(128, 2500), r.choice((8, 16, 32))
    d_in = r.choice([r.randint(1, 64), 8 * r.randint(1, 8)])   # the fast kernels want 8 | d_in
    dt, dtype = _dtype(r)
    mode = r.choice(["forward", "backward", "saved"])
    inp = scan_inputs(b, L, d_in, N, dt, seed=seed, with_z=r.random() < 0.7,
                      with_D=r.random() < 0.7, with_dt_bias=r.random() < 0.7,
                      with_h0=r.random() < 0.5)
    g = to_cuda(inp)
    what = (b, L, d_in, N, dt, mode)
    if mode == "forward":
        hl = torch.empty(b, d_in, N, device="cuda")
        y = ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                             dt_bias=g["dt_bias"], h0=g["h0"], h_last=hl)
        y_ref, h_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"],
                                             inp["C"], D=inp["D"], z=inp["z"],
                                             dt_bias=inp["dt_bias"], h0=inp["h0"],
                                             return_last_state=True)
        assert rel_err(y, y_ref) <= TOL[dtype], what
        assert rel_err(hl, h_ref) <= 1e-4, what
        return
    gd = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(b, L, d_in, generator=gd).to(dtype)
    dhl = torch.randn(b, d_in, N, generator=gd) if r.random() < 0.5 else None
    kw = dict(D=g["D"], z=g["z"], dt_bias=g["dt_bias"], h0=g["h0"],
              dh_last=None if dhl is None else dhl.cuda(), want_dh0=True)
    if mode == "saved":
        states = torch.empty(ssm.ssm_scan_bwd_workspace_bytes(b, L, d_in, N) // 4, device="cuda")
        ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                         dt_bias=g["dt_bias"], h0=g["h0"], chunk_states=states)
        kw["states"] = states
    got = ssm.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout.cuda(), **kw)
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dout,
                                    D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                    h0=inp["h0"], dh_last=dhl)
    for k in ref:
        if k not in got or got[k] is None:
            continue
        tol = TOL[dtype] if k in ("du", "ddelta", "dz") else (1e-4 if dtype == torch.float32 else 2e-4)
        assert rel_err(got[k], ref[k]) <= tol, (k,) + what


@pytest.mark.parametrize("seed", _seeds(160, 13))
def test_random_ss2d(ssm, seed):
    r = random.Random(seed)
    b, H, W, d_in = r.randint(1, 2), r.randint(1, 40), r.randint(1, 40), r.randint(1, 40)
    dt, dtype = _dtype(r)
    order = r.choice(["cross", "snake"])
    softplus = r.random() < 0.8
    inp = ss2d_inputs(b, H, W, d_in, 1, dt, seed=seed, with_D=r.random() < 0.7,
                      with_dt_bias=r.random() < 0.5)
    if not softplus:  # delta must stay positive for the state to decay
        inp["delta"] = inp["delta"].abs()
        inp["dt_bias"] = None
    g = to_cuda(inp)
    y = ssm.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"],
                          dt_bias=g["dt_bias"], delta_softplus=softplus, order=order)
    ref = oracle.ss2d_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W,
                           D=inp["D"], dt_bias=inp["dt_bias"], delta_softplus=softplus,
                           order=order)
    assert rel_err(y, ref) <= TOL[dtype], (b, H, W, d_in, dt, order, softplus)


@pytest.mark.parametrize("seed", _seeds(160, 14))
def test_random_decode_steps(ssm, seed):
    r = random.Random(seed)
    b, d_in, N = r.randint(1, 4), r.randint(1, 300), r.choice(STATES)
    dt, dtype = _dtype(r)
    conv = r.random() < 0.5
    inp = step_inputs(b, d_in, N, dt, seed=seed, with_z=r.random() < 0.7)
    g = to_cuda(inp)
    st = g["state"].clone()
    if conv:
        d_conv = r.randint(1, 8)
        c = conv_inputs(b, d_in, d_conv, dt, seed=seed + 2, with_bias=r.random() < 0.7)
        gc = to_cuda(c)
        cs = gc["conv_state"].clone()
        y = ssm.ssm_conv_state_update(cs, gc["conv_weight"], st, g["x"], g["dt"], g["A"], g["B"],
                                      g["C"], conv_bias=gc["conv_bias"], D=g["D"], z=g["z"],
                                      dt_bias=g["dt_bias"])
        xc, cs_ref = oracle.conv_step(c["conv_state"], inp["x"], c["conv_weight"], c["conv_bias"])
        y_ref, st_ref = oracle.state_update(inp["state"], xc, inp["dt"], inp["A"], inp["B"],
                                            inp["C"], D=inp["D"], z=inp["z"],
                                            dt_bias=inp["dt_bias"])
        np.testing.assert_array_equal(to64(cs), cs_ref)
    else:
        y = ssm.ssm_state_update(st, g["x"], g["dt"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                                 dt_bias=g["dt_bias"])
        y_ref, st_ref = oracle.state_update(inp["state"], inp["x"], inp["dt"], inp["A"], inp["B"],
                                            inp["C"], D=inp["D"], z=inp["z"],
                                            dt_bias=inp["dt_bias"])
    what = (b, d_in, N, dt, conv)
    assert rel_err(y, y_ref) <= TOL[dtype], what
    assert rel_err(st, st_ref) <= 1e-5, what
