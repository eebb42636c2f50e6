"""Runs one call of every kernel family through the debug-bounds library
(SSM_DEBUG_BOUNDS=1 must be set before this module imports the binding):
every global index the kernels compute must fall inside its buffer, the
results must still match the oracle, and the self-test's one out-of-range
index must be reported.  Exits 0 and prints "debug-bounds ok" on success."""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
from _helpers import rel_err, to_cuda  # noqa: E402
from selective_state_space_25_b200 import ssmscan as S  # noqa: E402
from selective_state_space_25_b200.synthetic import (conv_inputs, scan_inputs,  # noqa: E402
                                                      ss2d_inputs, step_inputs)


def check(label, got, ref, tol):
    e = rel_err(got, ref)
    assert e <= tol, f"{label}: error {e}"
    S.check_device_errors()  # raises on a recorded out-of-range index


def main():
    assert S.DEBUG_BOUNDS and S.debug_bounds_enabled(), "not the debug-bounds library"
    oracle.build()
    # forward: one pass (ragged L and d_in, d_state 8 / 16 / 32 / 64), the
    # split scan, the saved-state forward + backward, the generic kernel
    for (b, L, d, N, dt) in [(2, 77, 40, 16, "bf16"), (1, 3000, 64, 16, "bf16"),
                             (2, 50, 32, 32, "fp32"), (1, 40, 32, 64, "bf16"),
                             (2, 45, 17, 2, "fp32"), (2, 65, 24, 8, "bf16")]:
        inp = scan_inputs(b, L, d, N, dt, seed=L + d, with_h0=True)
        g = to_cuda(inp)
        hl = torch.empty(b, d, N, device="cuda")
        y = S.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                           dt_bias=g["dt_bias"], h0=g["h0"], h_last=hl)
        y_ref, h_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                             D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                             h0=inp["h0"], return_last_state=True)
        tol = 2e-2 if dt == "bf16" else 1e-4
        check(f"scan {b, L, d, N, dt}", y, y_ref, tol)
        check(f"h_last {b, L, d, N, dt}", hl, h_ref, tol)
    inp = scan_inputs(2, 70, 32, 16, "bf16", seed=3)
    g = to_cuda(inp)
    states = torch.empty(S.ssm_scan_bwd_workspace_bytes(2, 70, 32, 16) // 4, device="cuda")
    S.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                   dt_bias=g["dt_bias"], chunk_states=states)
    dout = torch.randn(2, 70, 32, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dout,
                                    D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"])
    for saved in (False, True):
        gr = S.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout.cuda(), D=g["D"],
                            z=g["z"], dt_bias=g["dt_bias"], states=states if saved else None)
        for k in ("du", "ddelta", "dB", "dC", "dA"):
            check(f"backward {k} saved={saved}", gr[k], ref[k], 2e-2 if k in ("du", "ddelta") else 2e-4)
    # split backward (few channels): self-contained and from saved states;
    # the binding allocates the split's workspace
    inp = scan_inputs(1, 1000, 32, 8, "bf16", seed=21, with_h0=True)
    g = to_cuda(inp)
    assert S.ssm_scan_bwd_saved_workspace_bytes(1, 1000, 32, 8) > 0
    states = torch.empty(S.ssm_scan_bwd_workspace_bytes(1, 1000, 32, 8) // 4, device="cuda")
    S.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                   dt_bias=g["dt_bias"], h0=g["h0"], chunk_states=states)
    dout = torch.randn(1, 1000, 32, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    ref = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dout,
                                    D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"], h0=inp["h0"])
    for saved in (False, True):
        gr = S.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout.cuda(), D=g["D"],
                            z=g["z"], dt_bias=g["dt_bias"], h0=None if saved else g["h0"],
                            states=states if saved else None, want_dh0=True)
        for k in ("du", "ddelta", "dB", "dC", "dA", "dh0"):
            check(f"split backward {k} saved={saved}", gr[k], ref[k],
                  2e-2 if k in ("du", "ddelta") else 2e-4)
    # SS2D: shared-memory and workspace accumulators, both orders
    # (d_in 13: a partial last channel group, its last pair inactive)
    for (H, W, order, d_in) in [(7, 9, "cross", 16), (5, 6, "snake", 16), (80, 81, "cross", 16),
                                (7, 9, "snake", 13), (80, 81, "cross", 13), (80, 81, "snake", 13)]:
        inp = ss2d_inputs(1, H, W, d_in, 1, "bf16", seed=H + W + d_in)
        g = to_cuda(inp)
        y = S.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"], order=order)
        y_ref = oracle.ss2d_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W,
                                 D=inp["D"], order=order)
        check(f"ss2d {H}x{W} {order} d_in {d_in}", y, y_ref, 2e-2)
    xs = S.ss2d_cross_scan(torch.randn(1, 35, 8).cuda(), 5, 7)
    S.ss2d_cross_merge(xs, 5, 7)
    S.check_device_errors()
    # decode steps
    inp = step_inputs(3, 40, 16, "bf16", seed=4)
    g = to_cuda(inp)
    st = g["state"].clone()
    y = S.ssm_state_update(st, g["x"], g["dt"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                           dt_bias=g["dt_bias"])
    y_ref, st_ref = oracle.state_update(inp["state"], inp["x"], inp["dt"], inp["A"], inp["B"],
                                        inp["C"], D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"])
    check("step", y, y_ref, 2e-2)
    check("step state", st, st_ref, 2e-2)
    c = conv_inputs(3, 40, 4, "bf16", seed=5)
    cg = to_cuda(c)
    st = g["state"].clone()
    y = S.ssm_conv_state_update(cg["conv_state"], cg["conv_weight"], st, g["x"], g["dt"], g["A"],
                                g["B"], g["C"], conv_bias=cg["conv_bias"], D=g["D"], z=g["z"],
                                dt_bias=g["dt_bias"])
    xc, _ = oracle.conv_step(c["conv_state"], inp["x"], c["conv_weight"], c["conv_bias"])
    y_ref, _ = oracle.state_update(inp["state"], xc, inp["dt"], inp["A"], inp["B"], inp["C"],
                                   D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"])
    check("conv step", y, y_ref, 2e-2)
    # the mechanism itself: one index past its range is recorded and reported
    assert S.debug_bounds_self_test() == S.SSM_OK
    try:
        S.check_device_errors()
    except S.SsmError as e:
        assert "SSM_ERR_DEVICE_BOUNDS" in str(e) and "0x80000000" in str(e), str(e)
    else:
        raise AssertionError("the self-test's out-of-range index was not reported")
    S.check_device_errors()  # the word was cleared by the report
    print("debug-bounds ok")


if __name__ == "__main__":
    main()
