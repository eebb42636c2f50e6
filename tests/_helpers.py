"""Shared helpers of the parity tests: the error metric and tolerances.

Error metric (the pages define none): max_i |g_i - r_i| / max(|r_i|, rms(r)),
which is the relative error where outputs are large and an error relative to
the output's RMS where they pass near zero.  Tolerances: 1e-4 for fp32
inputs, 2e-2 for bf16 inputs (the oracle runs on the bf16-rounded values)."""
import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def to64(t):
    if isinstance(t, torch.Tensor):
        t = t.detach().to("cpu")
        if t.dtype == torch.bfloat16:
            t = t.float()
        return t.double().numpy()
    return np.asarray(t, dtype=np.float64)


def rel_err(got, ref) -> float:
    g, r = to64(got), to64(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    if r.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(r * r)))
    scale = np.maximum(np.abs(r), rms)
    scale[scale == 0] = 1.0
    if not np.all(np.isfinite(g)):
        return float("inf")
    return float(np.max(np.abs(g - r) / scale))


def to_cuda(d: dict) -> dict:
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
