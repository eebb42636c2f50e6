"""The oracle still reproduces its stored snapshot (tests/golden/, written by
tests/golden/make_golden.py from the oracle alone)."""
import json
import os

import numpy as np

import oracle
from selective_state_space_25_b200.synthetic import WORKLOADS, scan_inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_fp32_scan.json")


def test_tiny_fp32_scan_snapshot():
    g = json.load(open(GOLDEN))
    w = WORKLOADS[g["workload"]]
    d = w.dims
    assert d == g["dims"] and w.seed == g["seed"]
    inp = scan_inputs(d["b"], d["L"], d["d_in"], d["N"], w.dtype, w.seed)
    y, h = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                 D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                 delta_softplus=True, return_last_state=True)
    got = [y[tuple(i)] for i in g["sample_index"]]
    np.testing.assert_allclose(got, g["sample_y"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y.sum(), g["y_sum"], rtol=1e-12, atol=1e-9)
    np.testing.assert_allclose(h.sum(axis=(1, 2)), g["h_last_sum_per_batch"], rtol=1e-12, atol=1e-9)


def test_tiny_fp32_scan_bwd_snapshot():
    import torch
    g = json.load(open(GOLDEN.replace(".json", "_bwd.json")))
    w = WORKLOADS[g["workload"]]
    d = w.dims
    assert d == g["dims"] and w.seed == g["seed"]
    inp = scan_inputs(d["b"], d["L"], d["d_in"], d["N"], w.dtype, w.seed)
    dout = torch.randn(d["b"], d["L"], d["d_in"], generator=torch.Generator().manual_seed(g["dout_seed"]))
    got = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dout,
                                    D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"])
    assert sorted(got) == sorted(g["sums"])
    for k, v in got.items():
        np.testing.assert_allclose(v.sum(), g["sums"][k], rtol=1e-10, atol=1e-9, err_msg=k)
        np.testing.assert_allclose(v.ravel()[:: max(1, v.size // 16)][:16], g["samples"][k],
                                   rtol=1e-12, atol=1e-12, err_msg=k)
