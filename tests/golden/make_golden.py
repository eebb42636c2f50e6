"""Writes tests/golden/tiny_fp32_scan.json (and tiny_fp32_scan_bwd.json) from
the fp64 oracle ONLY.

The tiny fp32 workload (b=2, L=64, d_in=32, N=16, seed 0: the Mamba block of
"代码连连看——mamba"'s usage example, d_model=16, expand=2, d_state=16) is run
through ``oracle.selective_scan``; 64 sampled outputs, the last state's
per-batch sums and the whole-output sum are stored; for the backward
(``oracle.selective_scan_bwd`` with dout ~ N(0, 1) from torch seed 1) the
sum and a sample of every gradient.  The test
``tests/test_golden.py`` checks the oracle still reproduces them, so an
accidental change to the oracle's arithmetic is visible in review.

Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from selective_state_space_25_b200.synthetic import WORKLOADS, scan_inputs  # noqa: E402


def main():
    w = WORKLOADS["tiny-fp32-scan"]
    d = w.dims
    inp = scan_inputs(d["b"], d["L"], d["d_in"], d["N"], w.dtype, w.seed)
    y, h = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                 D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                 delta_softplus=True, return_last_state=True)
    rng = np.random.default_rng(0)
    idx = np.stack([rng.integers(0, s, 64) for s in y.shape], 1)
    out = {
        "workload": w.name,
        "dims": d,
        "seed": w.seed,
        "source": "oracle.selective_scan (fp64), tests/golden/make_golden.py",
        "sample_index": idx.tolist(),
        "sample_y": [float(y[tuple(i)]) for i in idx],
        "y_sum": float(y.sum()),
        "h_last_sum_per_batch": [float(v) for v in h.sum(axis=(1, 2))],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_fp32_scan.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)

    import torch
    dout = torch.randn(y.shape, generator=torch.Generator().manual_seed(1))
    g = oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dout,
                                  D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"])
    bwd = {"workload": w.name, "dims": d, "seed": w.seed, "dout_seed": 1,
           "source": "oracle.selective_scan_bwd (fp64), tests/golden/make_golden.py",
           "sums": {k: float(v.sum()) for k, v in g.items()},
           "samples": {k: [float(x) for x in v.ravel()[:: max(1, v.size // 16)][:16]]
                       for k, v in g.items()}}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_fp32_scan_bwd.json")
    with open(path, "w") as f:
        json.dump(bwd, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
