"""GPU parity of ss2d_scan_fwd and the CrossScan / CrossMerge permutations
against the fp64 oracle (through the C ABI).  The permutations are checked
bit-exactly; the fused four-direction scan within the bf16 / fp32
tolerances."""
import numpy as np
import pytest
import torch

import oracle
from _helpers import TOL, rel_err, to_cuda, to64
from selective_state_space_25_b200.synthetic import WORKLOADS, ss2d_inputs

pytestmark = pytest.mark.gpu


def gpu_ss2d(S, inp, H, W, softplus=True):
    g = to_cuda(inp)
    return S.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"],
                           dt_bias=g["dt_bias"], delta_softplus=softplus)


def oracle_ss2d(inp, H, W, softplus=True):
    return oracle.ss2d_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W,
                            D=inp["D"], dt_bias=inp["dt_bias"], delta_softplus=softplus)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("H,W", [(5, 7), (1, 9), (8, 1), (16, 16), (1, 1), (33, 17)])
def test_cross_scan_bit_exact(ssm, dtype, H, W):
    u = torch.randn(2, H * W, 12).to(dtype)
    xs = ssm.ss2d_cross_scan(u.cuda(), H, W)
    np.testing.assert_array_equal(to64(xs), oracle.cross_scan(u, H, W))


@pytest.mark.parametrize("H,W", [(5, 7), (9, 4), (1, 6)])
def test_cross_merge_of_cross_scan_is_4u(ssm, H, W):
    u = torch.randn(3, H * W, 16).to(torch.bfloat16).cuda()
    y = ssm.ss2d_cross_merge(ssm.ss2d_cross_scan(u, H, W), H, W)
    assert torch.equal(y, 4 * u)


@pytest.mark.parametrize("k", [0, 1, 2, 3])
def test_cross_merge_inverse_permutation_one_hot(ssm, k):
    """With only direction k non-zero, the merge is the exact inverse gather."""
    H, W = 6, 11
    ys = torch.zeros(2, 4, H * W, 8)
    ys[:, k] = torch.randn(2, H * W, 8)
    y = ssm.ss2d_cross_merge(ys.cuda(), H, W)
    np.testing.assert_array_equal(to64(y), oracle.cross_merge(ys, H, W))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,H,W,d_in", [
    (2, 5, 7, 8), (2, 1, 1, 8), (1, 1, 40, 16), (1, 37, 1, 8), (2, 16, 16, 12),
    (2, 23, 29, 24), (1, 56, 56, 16), (1, 3, 300, 8),
])
def test_ss2d_shapes(ssm, dtype, b, H, W, d_in):
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = ss2d_inputs(b, H, W, d_in, 1, dt, seed=H * 100 + W, with_dt_bias=True)
    y = gpu_ss2d(ssm, inp, H, W)
    assert rel_err(y, oracle_ss2d(inp, H, W)) <= TOL[dtype]


def test_ss2d_no_softplus_no_D(ssm):
    inp = ss2d_inputs(2, 9, 13, 16, 1, "fp32", seed=4, with_D=False)
    inp["delta"] = inp["delta"].abs() * 0.2
    y = gpu_ss2d(ssm, inp, 9, 13, softplus=False)
    assert rel_err(y, oracle_ss2d(inp, 9, 13, softplus=False)) <= 1e-4


@pytest.mark.parametrize("order", ["cross", "snake"])
@pytest.mark.parametrize("dtype,b,H,W,d_in", [
    (torch.float32, 2, 7, 9, 16),     # one partial chunk, shared accumulator
    (torch.bfloat16, 1, 13, 11, 13),  # odd d_in: plain staging, ragged channel tile
    (torch.bfloat16, 1, 80, 81, 16),  # workspace accumulator, 21 chunks, the last partial
])
def test_ss2d_steps_past_the_end_cannot_leak(ssm, order, dtype, b, H, W, d_in):
    """The kernel runs whole chunks, and the steps past the end of a direction
    (zero-filled rows) are not forced to identity.  With the softplus off and
    dt_bias = -4 their decay is exp(4) > 1, so their composed maps overflow to
    inf and nan in fp32; the real steps, which all come before them, must not
    see that."""
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = ss2d_inputs(b, H, W, d_in, 1, dt, seed=H * 31 + W, with_dt_bias=True)
    inp["dt_bias"] = torch.full_like(inp["dt_bias"], -4.0)
    # real steps: delta + dt_bias = |delta| + 0.1 > 0, a decaying state
    inp["delta"] = (inp["delta"].float().abs() + 4.1).to(inp["delta"].dtype)
    g = to_cuda(inp)
    y = ssm.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"],
                          dt_bias=g["dt_bias"], delta_softplus=False, order=order)
    assert torch.isfinite(y.float()).all()
    ref = oracle.ss2d_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W,
                           D=inp["D"], dt_bias=inp["dt_bias"], delta_softplus=False, order=order)
    assert rel_err(y, ref) <= TOL[dtype]


def test_ss2d_large_image_uses_workspace(ssm):
    """H W above the shared-memory accumulator limit: the fp32 accumulator lives
    in the caller's workspace."""
    H, W = 80, 81
    assert ssm.ss2d_scan_fwd_workspace_bytes(1, H, W, 16, 1) > 0
    inp = ss2d_inputs(1, H, W, 16, 1, "bf16", seed=8)
    y = gpu_ss2d(ssm, inp, H, W)
    assert rel_err(y, oracle_ss2d(inp, H, W)) <= 2e-2


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("order", ["cross", "snake"])
@pytest.mark.parametrize("d_in,offset", [(13, 0), (16, 4), (13, 4)])
def test_ss2d_workspace_odd_channels_or_4_byte_aligned(ssm, dtype, order, d_in, offset):
    """The workspace accumulator when channel pairs cannot be 8-byte accesses:
    odd d_in puts every other pair on an odd float, and a workspace that is
    4- but not 8-byte aligned (the entry point asks for 4) shifts all of them."""
    H, W = 80, 81
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    need = ssm.ss2d_scan_fwd_workspace_bytes(1, H, W, d_in, 1)
    assert need > 0
    raw = torch.empty(need + 16, dtype=torch.uint8, device="cuda")
    base = raw.data_ptr() % 8
    ws = raw[(offset - base) % 8:][:need]
    assert ws.data_ptr() % 8 == offset
    inp = ss2d_inputs(1, H, W, d_in, 1, dt, seed=d_in * 7 + offset, with_dt_bias=True)
    g = to_cuda(inp)
    y = ssm.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"],
                          dt_bias=g["dt_bias"], workspace=ws, order=order)
    ref = oracle.ss2d_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W,
                           D=inp["D"], dt_bias=inp["dt_bias"], order=order)
    assert rel_err(y, ref) <= TOL[dtype]


@pytest.mark.parametrize("order", ["cross", "snake"])
@pytest.mark.parametrize("H,W,smem", [(128, 49, True), (64, 98, False)])
def test_ss2d_shared_accumulator_limit(ssm, order, H, W, smem):
    """The shared accumulator holds H (W rounded up to odd) pixels of 8 fp32
    channels, at most 6272: 128 x 49 fills it exactly; 64 x 98 has as many
    pixels but pads to 64 x 99, so it takes the workspace."""
    need = ssm.ss2d_scan_fwd_workspace_bytes(1, H, W, 16, 1)
    assert (need == 0) == smem
    inp = ss2d_inputs(1, H, W, 16, 1, "bf16", seed=H + W, with_dt_bias=True)
    g = to_cuda(inp)
    y = ssm.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"],
                          dt_bias=g["dt_bias"], order=order)
    ref = oracle.ss2d_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W,
                           D=inp["D"], dt_bias=inp["dt_bias"], order=order)
    assert rel_err(y, ref) <= 2e-2


def test_ss2d_equals_composition_of_gpu_scans(ssm):
    """Fused SS2D == CrossScan, four 1-D scans, CrossMerge, all on the GPU."""
    b, H, W, d_in = 2, 12, 10, 16
    L = H * W
    inp = to_cuda(ss2d_inputs(b, H, W, d_in, 1, "fp32", seed=12, with_dt_bias=True))
    y = ssm.ss2d_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W, D=inp["D"],
                          dt_bias=inp["dt_bias"])
    xs = ssm.ss2d_cross_scan(inp["u"], H, W)
    ys = torch.empty(b, 4, L, d_in, device="cuda")
    for i in range(b):
        for k in range(4):
            sl = slice(k * d_in, (k + 1) * d_in)
            ys[i, k] = ssm.ssm_scan_fwd(xs[i, k][None].contiguous(), inp["delta"][i, k][None].contiguous(),
                                        inp["A"][sl].contiguous(), inp["B"][i, k][None].contiguous(),
                                        inp["C"][i, k][None].contiguous(), D=inp["D"][sl].contiguous(),
                                        dt_bias=inp["dt_bias"][sl].contiguous())[0]
    ref = ssm.ss2d_cross_merge(ys, H, W)
    assert rel_err(y, ref) <= 1e-5


def test_vmamba_ss2d_workload_sampled(ssm):
    w = WORKLOADS["vmamba-ss2d"]
    d = w.dims
    H, W, d_in = d["H"], d["W"], d["d_in"]
    inp = ss2d_inputs(d["b"], H, W, d_in, d["N"], w.dtype, w.seed)
    y = gpu_ss2d(ssm, inp, H, W)
    torch.cuda.synchronize()
    bsel = [0, d["b"] - 1]
    chans = [0, 7, 8, 95, 96, 183, 184, 191]
    rows = [k * d_in + c for k in range(4) for c in chans]
    ref_in = dict(u=inp["u"][bsel][:, :, chans].contiguous(),
                  delta=inp["delta"][bsel][:, :, :, chans].contiguous(),
                  A=inp["A"][rows], B=inp["B"][bsel], C=inp["C"][bsel], D=inp["D"][rows],
                  dt_bias=None)
    ref = oracle_ss2d(ref_in, H, W)
    got = y[bsel][:, :, chans]
    assert rel_err(got, ref) <= 2e-2


# ------------------------------------------------------------------ snake order
@pytest.mark.parametrize("H,W", [(5, 7), (6, 4), (1, 9), (8, 1), (2, 3)])
def test_snake_cross_scan_and_merge_bit_exact(ssm, H, W):
    u = torch.randn(2, H * W, 8).to(torch.bfloat16)
    xs = ssm.ss2d_cross_scan(u.cuda(), H, W, order="snake")
    np.testing.assert_array_equal(to64(xs), oracle.cross_scan(u, H, W, order="snake"))
    y = ssm.ss2d_cross_merge(xs, H, W, order="snake")
    assert torch.equal(y.cpu(), 4 * u)
    for k in range(4):                         # one direction at a time: exact inverse gather
        ys = torch.zeros(2, 4, H * W, 8)
        ys[:, k] = torch.randn(2, H * W, 8)
        ym = ssm.ss2d_cross_merge(ys.cuda(), H, W, order="snake")
        np.testing.assert_array_equal(to64(ym), oracle.cross_merge(ys, H, W, order="snake"))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,H,W,d_in", [(2, 5, 7, 8), (1, 1, 40, 16), (1, 37, 1, 8),
                                         (2, 16, 16, 24), (1, 56, 56, 16), (2, 9, 11, 12)])
def test_ss2d_snake_shapes(ssm, dtype, b, H, W, d_in):
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = ss2d_inputs(b, H, W, d_in, 1, dt, seed=H * 31 + W, with_dt_bias=True)
    g = to_cuda(inp)
    y = ssm.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"],
                          dt_bias=g["dt_bias"], order="snake")
    ref = oracle.ss2d_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W,
                           D=inp["D"], dt_bias=inp["dt_bias"], order="snake")
    assert rel_err(y, ref) <= TOL[dtype]


def test_ss2d_snake_large_image_workspace(ssm):
    H, W = 79, 83
    inp = ss2d_inputs(1, H, W, 8, 1, "bf16", seed=41)
    g = to_cuda(inp)
    y = ssm.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"],
                          order="snake")
    ref = oracle.ss2d_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W,
                           D=inp["D"], order="snake")
    assert rel_err(y, ref) <= 2e-2


def _permutation_probe(b, H, W, d_in, dtype, seed):
    """Inputs under which the fused SS2D result depends only on where each
    direction's step lands: dA underflows to exactly 0 (A = -exp(40)), B = C = 1,
    D = 0 and no softplus, so step l of direction k contributes exactly
    delta_k(l) u(p_k(l)) at pixel p_k(l).  delta is a power of two in {1, 2, 4, 8}
    drawn per (b, k, l, d) and u = +-2^m, m in {-2 .. 2}, per (b, p, d): every
    product and the four-term sum are exact in fp32, and the sum (an integer in
    4 .. 32 times 2^m) is exact in bf16 too.  A pixel that takes the wrong step
    of a direction, or a step that reads the wrong pixel of u, changes a sum."""
    g = torch.Generator().manual_seed(seed)
    L = H * W
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    delta = torch.pow(2.0, torch.randint(0, 4, (b, 4, L, d_in), generator=g).double())
    sign = torch.randint(0, 2, (b, L, d_in), generator=g).double() * 2 - 1
    u = sign * torch.pow(2.0, torch.randint(-2, 3, (b, L, d_in), generator=g).double())
    return dict(u=u.to(td), delta=delta.to(td), A=torch.full((4 * d_in, 1), -float(np.exp(40.0))),
                B=torch.ones(b, 4, L, 1, dtype=td), C=torch.ones(b, 4, L, 1, dtype=td),
                D=torch.zeros(4 * d_in), dt_bias=None)


@pytest.mark.parametrize("order", ["cross", "snake"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("b,H,W,d_in", [
    (2, 5, 7, 8), (2, 6, 8, 16), (1, 7, 6, 8), (1, 1, 9, 8), (1, 9, 1, 8), (2, 11, 13, 12),
    (1, 56, 56, 8), (1, 80, 81, 8),   # the last one keeps its accumulator in the workspace
])
def test_fused_ss2d_permutation_bit_exact(ssm, order, dtype, b, H, W, d_in):
    """The fused kernel's own index arithmetic (the scan orders generated while
    staging, the skewed accumulator rows, the un-skewing store) against the
    oracle, bit for bit ("关于代码SS2D中的d_state设置": the orders only arrange
    the sequence, so under the probe above the result is a sum of exact terms)."""
    inp = _permutation_probe(b, H, W, d_in, dtype, seed=H * 1000 + W * 10 + d_in)
    g = to_cuda(inp)
    y = ssm.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W, D=g["D"],
                          delta_softplus=False, order=order)
    ref = oracle.ss2d_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W, D=inp["D"],
                           delta_softplus=False, order=order)
    expect = torch.from_numpy(np.asarray(ref)).to(y.dtype)
    assert torch.equal(y.cpu(), expect)


@pytest.mark.parametrize("order", ["cross", "snake"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("b,H,W,d_in", [
    (1, 56, 56, 192),  # batch 1 of the VMamba shape: 24 tiles
    (2, 7, 9, 24), (1, 13, 11, 13), (1, 1, 37, 16), (1, 37, 1, 16), (3, 17, 5, 40),
    (1, 100, 100, 16),  # accumulator in the workspace
    (1, 80, 81, 13),    # ... with odd d_in (channel pairs as two 4-byte accesses)
    (80, 80, 81, 8),    # ... and a batch that fills the GPU (80 tiles)
])
def test_direction_split_is_bit_identical(ssm, order, dtype, b, H, W, d_in):
    """Small batches and large images with the fast workspace run one CTA per
    (tile, direction) and sum the four fp32 direction outputs in a second
    kernel; with the minimum workspace the same call runs the single kernel.
    Same operations in the same order: the outputs agree bit for bit (and
    with the oracle)."""
    fast = ssm.ss2d_scan_fwd_fast_workspace_bytes(b, H, W, d_in, 1)
    least = ssm.ss2d_scan_fwd_workspace_bytes(b, H, W, d_in, 1)
    assert fast == 4 * b * H * W * d_in * 4, "these shapes should take the direction split"
    inp = ss2d_inputs(b, H, W, d_in, 1, dtype, seed=H * 7 + W + d_in, with_dt_bias=True)
    g = to_cuda(inp)
    run = lambda ws: ssm.ss2d_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], H, W,
                                       D=g["D"], dt_bias=g["dt_bias"], order=order, workspace=ws)
    y_split = run(torch.empty(fast, dtype=torch.uint8, device="cuda"))
    y_one = run(torch.empty(least, dtype=torch.uint8, device="cuda"))
    assert torch.equal(y_split, y_one)
    ref = oracle.ss2d_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], H, W,
                           D=inp["D"], dt_bias=inp["dt_bias"], order=order)
    assert rel_err(y_split, ref) <= TOL[torch.bfloat16 if dtype == "bf16" else torch.float32]
