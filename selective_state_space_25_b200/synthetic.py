"""Seeded synthetic inputs shared by the CUDA path, its tests and the oracle.

This module only DRAWS inputs: it holds none of the scan's arithmetic.  Every
tensor is drawn on the CPU with a fixed ``torch.Generator`` seed in a fixed
order, then rounded once to the activation dtype (round-to-nearest-even for
bf16), so both sides of a parity test see the same stored values.

Distributions follow the Mamba block's parameterisation as the pages state it:

* ``A = -exp(A_log)`` with the S4D-real init ``A_log = log(arange(1..N))``
  repeated over the channels ("Mamba. От начала до конца", comment thread:
  A_log is (d_in, N) and A = -exp(A_log) elementwise; "手把手拆解Mamba-minimal
  中的selective_scan实现" §7, the initialisation example).  A is formed once
  here in fp32 and handed to both sides.
* ``dt_bias`` is the inverse softplus of a per-channel step size drawn
  log-uniformly in [1e-3, 1e-1], so softplus(dt_bias) lands in that range
  ("代码连连看——mamba", Mamba.step(): the bias of dt_proj is added just
  before the softplus).
* activations u, z, B, C ~ N(0, 1); the pre-softplus dt ~ N(0, 0.5^2) for
  the prefill scans, N(0, 1) for the decode step.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = ["Workload", "WORKLOADS", "scan_inputs", "ss2d_inputs", "step_inputs", "conv_inputs",
           "s4d_real_A", "dt_bias_init"]


@dataclass(frozen=True)
class Workload:
    """A named synthetic workload (sizes, dtype, seed)."""
    name: str
    kind: str                 # "scan" | "scan_bwd" | "scan_bwd_saved" | "ss2d" | "step"
    dims: dict = field(default_factory=dict)
    dtype: str = "bf16"
    seed: int = 0
    note: str = ""

    def elements(self) -> int:
        """b * L * d_in * N (times the 4 directions for SS2D), per step."""
        d = self.dims
        if self.kind in ("scan", "scan_bwd", "scan_bwd_saved"):
            return d["b"] * d["L"] * d["d_in"] * d["N"]
        if self.kind == "ss2d":
            return d["b"] * 4 * d["H"] * d["W"] * d["d_in"] * d["N"]
        return d["b"] * d["d_in"] * d["N"]


WORKLOADS = {
    "tiny-fp32-scan": Workload(
        "tiny-fp32-scan", "scan", dict(b=2, L=64, d_in=32, N=16), "fp32", 0,
        "Mamba(d_model=16, expand=2, d_state=16) on a (2, 64, 16) input"),
    "mamba130m-scan": Workload(
        "mamba130m-scan", "scan", dict(b=8, L=2048, d_in=1536, N=16), "bf16", 1,
        "Mamba-130M-shaped prefill scan"),
    "mamba130m-scan-bwd": Workload(
        "mamba130m-scan-bwd", "scan_bwd", dict(b=8, L=2048, d_in=1536, N=16), "bf16", 1,
        "backward of the Mamba-130M-shaped prefill scan (all input gradients)"),
    "mamba130m-scan-bwd-saved": Workload(
        "mamba130m-scan-bwd-saved", "scan_bwd_saved", dict(b=8, L=2048, d_in=1536, N=16), "bf16",
        1, "the same backward from the chunk states its forward saved (training split)"),
    "mamba1.4b-long-scan": Workload(
        "mamba1.4b-long-scan", "scan", dict(b=2, L=16384, d_in=4096, N=16), "bf16", 2,
        "Mamba-1.4B-shaped long-sequence prefill scan"),
    "vmamba-ss2d": Workload(
        "vmamba-ss2d", "ss2d", dict(b=32, H=56, W=56, d_in=192, N=1), "bf16", 3,
        "VMamba SS2D block, d_state 1, four scan directions"),
    "mamba-decode-step": Workload(
        "mamba-decode-step", "step", dict(b=256, d_in=5120, N=16, steps=1000), "bf16", 4,
        "Mamba.step() state update, fp32 state resident in HBM"),
    "mamba-decode-conv-step": Workload(
        "mamba-decode-conv-step", "step", dict(b=256, d_in=5120, N=16, d_conv=4, steps=1000),
        "bf16", 6, "Mamba.step(): causal-conv1d step fused with the state update"),
}


def _torch_dtype(dtype: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[dtype]


def s4d_real_A(d_in: int, N: int) -> torch.Tensor:
    """A = -exp(A_log), A_log = log(arange(1..N)) repeated over d_in (fp32)."""
    A_log = torch.log(torch.arange(1, N + 1, dtype=torch.float32)).repeat(d_in, 1)
    return -torch.exp(A_log)


def dt_bias_init(d_in: int, gen: torch.Generator) -> torch.Tensor:
    """Inverse softplus of a log-uniform [1e-3, 1e-1] step size (fp32)."""
    lo, hi = math.log(1e-3), math.log(1e-1)
    dt0 = torch.exp(torch.rand(d_in, generator=gen, dtype=torch.float64) * (hi - lo) + lo)
    # x such that log1p(exp(x)) == dt0
    return (dt0 + torch.log(-torch.expm1(-dt0))).float()


def scan_inputs(b: int, L: int, d_in: int, N: int, dtype: str = "bf16", seed: int = 0,
                dt_std: float = 0.5, with_z: bool = True, with_D: bool = True,
                with_dt_bias: bool = True, with_h0: bool = False) -> dict:
    """Inputs of the selective scan, on the CPU.

    Draw order: u, dt, z, B, C, dt_bias, then h0.  Shapes: u, delta, z
    (b, L, d_in); B, C (b, L, N); A (d_in, N); D, dt_bias (d_in); h0
    (b, d_in, N) fp32."""
    g = torch.Generator().manual_seed(seed)
    td = _torch_dtype(dtype)
    u = torch.randn(b, L, d_in, generator=g).to(td)
    delta = (dt_std * torch.randn(b, L, d_in, generator=g)).to(td)
    z = torch.randn(b, L, d_in, generator=g).to(td)
    B = torch.randn(b, L, N, generator=g).to(td)
    C = torch.randn(b, L, N, generator=g).to(td)
    dt_bias = dt_bias_init(d_in, g)
    h0 = torch.randn(b, d_in, N, generator=g) if with_h0 else None
    return dict(u=u, delta=delta, A=s4d_real_A(d_in, N), B=B, C=C,
                D=torch.ones(d_in) if with_D else None,
                z=z if with_z else None,
                dt_bias=dt_bias if with_dt_bias else None,
                h0=h0)


def ss2d_inputs(b: int, H: int, W: int, d_in: int, N: int = 1, dtype: str = "bf16",
                seed: int = 3, with_D: bool = True, with_dt_bias: bool = False) -> dict:
    """Inputs of the SS2D four-direction scan, on the CPU.

    Draw order: u, delta, B, C (then dt_bias when asked for).  u is
    (b, H W, d_in); delta (b, 4, H W, d_in) and B, C (b, 4, H W, N) are in
    each direction's scan order; A_log = 0 so A = -1 (4 d_in, N); D = 1."""
    g = torch.Generator().manual_seed(seed)
    td = _torch_dtype(dtype)
    L = H * W
    u = torch.randn(b, L, d_in, generator=g).to(td)
    delta = torch.randn(b, 4, L, d_in, generator=g).to(td)
    B = torch.randn(b, 4, L, N, generator=g).to(td)
    C = torch.randn(b, 4, L, N, generator=g).to(td)
    A = -torch.exp(torch.zeros(4 * d_in, N))
    dt_bias = dt_bias_init(4 * d_in, g) if with_dt_bias else None
    return dict(u=u, delta=delta, A=A, B=B, C=C,
                D=torch.ones(4 * d_in) if with_D else None, dt_bias=dt_bias)


def step_inputs(b: int, d_in: int, N: int, dtype: str = "bf16", seed: int = 4,
                with_z: bool = True) -> dict:
    """Inputs of the one-token state update, on the CPU.

    Draw order: state, x, z, dt, B, C, dt_bias.  state (b, d_in, N) fp32;
    x, z, dt (b, d_in); B, C (b, N); A = -arange(1..N) per channel; D = 1."""
    g = torch.Generator().manual_seed(seed)
    td = _torch_dtype(dtype)
    state = torch.randn(b, d_in, N, generator=g)
    x = torch.randn(b, d_in, generator=g).to(td)
    z = torch.randn(b, d_in, generator=g).to(td)
    dt = torch.randn(b, d_in, generator=g).to(td)
    B = torch.randn(b, N, generator=g).to(td)
    C = torch.randn(b, N, generator=g).to(td)
    dt_bias = dt_bias_init(d_in, g)
    A = -torch.arange(1, N + 1, dtype=torch.float32).repeat(d_in, 1)
    return dict(state=state, x=x, dt=dt, A=A, B=B, C=C, D=torch.ones(d_in),
                z=z if with_z else None, dt_bias=dt_bias)


def conv_inputs(b: int, d_in: int, d_conv: int = 4, dtype: str = "bf16", seed: int = 5,
                with_bias: bool = True) -> dict:
    """Inputs of the causal-conv1d decode step, on the CPU.

    Draw order: conv_state, conv_weight, conv_bias.  conv_state (b, d_in,
    d_conv) holds past inputs (activation dtype); the depthwise weight
    (d_in, d_conv) and bias (d_in) are fp32, uniform in +-1/sqrt(d_conv) like
    a freshly initialised depthwise Conv1d."""
    g = torch.Generator().manual_seed(seed)
    td = _torch_dtype(dtype)
    conv_state = torch.randn(b, d_in, d_conv, generator=g).to(td)
    bound = 1.0 / math.sqrt(d_conv)
    conv_weight = (torch.rand(d_in, d_conv, generator=g) * 2 - 1) * bound
    conv_bias = (torch.rand(d_in, generator=g) * 2 - 1) * bound
    return dict(conv_state=conv_state, conv_weight=conv_weight,
                conv_bias=conv_bias if with_bias else None)


def workload_inputs(name: str, **overrides) -> dict:
    """Full-size inputs of a named workload (CPU tensors)."""
    w = WORKLOADS[name]
    d = dict(w.dims)
    d.update(overrides)
    if w.kind == "scan":
        return scan_inputs(d["b"], d["L"], d["d_in"], d["N"], w.dtype, w.seed)
    if w.kind in ("scan_bwd", "scan_bwd_saved"):
        inp = scan_inputs(d["b"], d["L"], d["d_in"], d["N"], w.dtype, w.seed)
        g = torch.Generator().manual_seed(w.seed + 1000)
        inp["dout"] = torch.randn(d["b"], d["L"], d["d_in"], generator=g).to(_torch_dtype(w.dtype))
        return inp
    if w.kind == "ss2d":
        return ss2d_inputs(d["b"], d["H"], d["W"], d["d_in"], d["N"], w.dtype, w.seed)
    inp = step_inputs(d["b"], d["d_in"], d["N"], w.dtype, w.seed)
    if "d_conv" in d:
        inp.update(conv_inputs(d["b"], d["d_in"], d["d_conv"], w.dtype, w.seed + 1000))
    return inp
