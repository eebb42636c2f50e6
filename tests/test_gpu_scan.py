"""GPU parity of ssm_scan_fwd against the fp64 oracle (through the C ABI).

Small shapes span several chunks and channel tiles with ragged tails; the
full-size workloads are checked on sampled channels, which the oracle
computes exactly (channels are independent)."""
import numpy as np
import pytest
import torch

import oracle
from _helpers import TOL, rel_err, to_cuda
from selective_state_space_25_b200.synthetic import WORKLOADS, scan_inputs

pytestmark = pytest.mark.gpu


def run_gpu(S, inp, **kw):
    g = to_cuda(inp)
    y = S.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                       dt_bias=g["dt_bias"], h0=g["h0"], **kw)
    return y, g


def run_oracle(inp, last=False, softplus=True):
    return oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                 z=inp["z"], dt_bias=inp["dt_bias"], h0=inp["h0"],
                                 delta_softplus=softplus, return_last_state=last)


def test_tiny_fp32_workload(ssm):
    w = WORKLOADS["tiny-fp32-scan"]
    d = w.dims
    inp = scan_inputs(d["b"], d["L"], d["d_in"], d["N"], w.dtype, w.seed)
    hl = torch.empty(d["b"], d["d_in"], d["N"], device="cuda")
    y, _ = run_gpu(ssm, inp, h_last=hl)
    y_ref, h_ref = run_oracle(inp, last=True)
    assert rel_err(y, y_ref) <= 1e-4
    assert rel_err(hl, h_ref) <= 1e-4


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,L,d_in,N", [
    (1, 1, 32, 16), (2, 63, 32, 16), (2, 64, 32, 16), (2, 65, 64, 16), (3, 130, 40, 16),
    (1, 200, 8, 16), (2, 77, 96, 8), (2, 50, 32, 32), (1, 40, 32, 64), (2, 33, 30, 16),
    (2, 45, 24, 4), (2, 45, 17, 2), (3, 90, 33, 1),
])
def test_shapes(ssm, dtype, b, L, d_in, N):
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = scan_inputs(b, L, d_in, N, dt, seed=100 + L + d_in + N, with_h0=True)
    hl = torch.empty(b, d_in, N, device="cuda")
    y, _ = run_gpu(ssm, inp, h_last=hl)
    y_ref, h_ref = run_oracle(inp, last=True)
    assert rel_err(y, y_ref) <= TOL[dtype]
    assert rel_err(hl, h_ref) <= TOL[dtype]


@pytest.mark.parametrize("with_z,with_D,with_bias,softplus", [
    (False, False, False, True), (True, False, True, False), (False, True, False, False),
])
def test_optional_terms(ssm, with_z, with_D, with_bias, softplus):
    inp = scan_inputs(2, 100, 64, 16, "fp32", seed=7, with_z=with_z, with_D=with_D,
                      with_dt_bias=with_bias)
    if not softplus:
        # without the softplus, delta = dt + dt_bias must stay positive
        inp["delta"] = inp["delta"].abs() * 0.1
        if with_bias:
            inp["dt_bias"] = inp["dt_bias"].abs() * 0.01
    y, _ = run_gpu(ssm, inp, delta_softplus=softplus)
    assert rel_err(y, run_oracle(inp, softplus=softplus)) <= 1e-4


def test_h_last_may_alias_h0(ssm):
    inp = scan_inputs(2, 70, 32, 16, "bf16", seed=3, with_h0=True)
    g = to_cuda(inp)
    h = g["h0"].clone()
    ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                      dt_bias=g["dt_bias"], h0=h, h_last=h)
    _, h_ref = run_oracle(inp, last=True)
    assert rel_err(h, h_ref) <= 2e-2


def test_resume_from_h_last_matches_one_pass(ssm):
    """Scanning [0, L1) then [L1, L) from the carried state equals one pass."""
    inp = scan_inputs(2, 150, 64, 16, "fp32", seed=5)
    g = to_cuda(inp)
    y_full = ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                               dt_bias=g["dt_bias"])
    L1 = 57
    h = torch.empty(2, 64, 16, device="cuda")
    sl1, sl2 = slice(0, L1), slice(L1, None)
    part = lambda t, s: t[:, s].contiguous()
    y1 = ssm.ssm_scan_fwd(part(g["u"], sl1), part(g["delta"], sl1), g["A"], part(g["B"], sl1),
                           part(g["C"], sl1), D=g["D"], z=part(g["z"], sl1), dt_bias=g["dt_bias"],
                           h_last=h)
    y2 = ssm.ssm_scan_fwd(part(g["u"], sl2), part(g["delta"], sl2), g["A"], part(g["B"], sl2),
                           part(g["C"], sl2), D=g["D"], z=part(g["z"], sl2), dt_bias=g["dt_bias"],
                           h0=h)
    assert rel_err(torch.cat([y1, y2], 1), y_full) <= 1e-5


def test_misaligned_pointers_take_the_generic_path(ssm):
    """A 2-byte offset breaks 16-byte alignment: the result must not change."""
    inp = scan_inputs(2, 90, 64, 16, "bf16", seed=9)
    g = to_cuda(inp)

    def shifted(t):
        buf = torch.empty(t.numel() + 8, dtype=t.dtype, device=t.device)
        v = buf[1:1 + t.numel()].view(t.shape)
        v.copy_(t)
        return v

    y_al = ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                             dt_bias=g["dt_bias"])
    y_mis = ssm.ssm_scan_fwd(shifted(g["u"]), shifted(g["delta"]), g["A"], shifted(g["B"]),
                              shifted(g["C"]), D=g["D"], z=shifted(g["z"]), dt_bias=g["dt_bias"])
    ref = run_oracle(inp)
    assert rel_err(y_al, ref) <= 2e-2 and rel_err(y_mis, ref) <= 2e-2


def test_empty_and_zero_length(ssm):
    inp = scan_inputs(2, 4, 32, 16, "fp32", seed=1, with_h0=True)
    g = to_cuda(inp)
    h = torch.full((2, 32, 16), 7.0, device="cuda")
    e = lambda t: t[:, :0].contiguous()
    y = ssm.ssm_scan_fwd(e(g["u"]), e(g["delta"]), g["A"], e(g["B"]), e(g["C"]), h0=g["h0"],
                          h_last=h)
    torch.cuda.synchronize()
    assert y.shape == (2, 0, 32)
    assert torch.equal(h, g["h0"])          # L = 0: the last state is the start state
    h.fill_(7.0)
    ssm.ssm_scan_fwd(e(g["u"]), e(g["delta"]), g["A"], e(g["B"]), e(g["C"]), h_last=h)
    torch.cuda.synchronize()
    assert torch.count_nonzero(h).item() == 0
    z = torch.empty(0, 5, 32, device="cuda")
    y0 = ssm.ssm_scan_fwd(z, z, g["A"], torch.empty(0, 5, 16, device="cuda"),
                           torch.empty(0, 5, 16, device="cuda"))
    assert y0.shape == (0, 5, 32)


def test_zero_input_gives_zero(ssm):
    inp = scan_inputs(2, 80, 32, 16, "bf16", seed=2)
    inp["u"] = torch.zeros_like(inp["u"])
    hl = torch.full((2, 32, 16), 1.0, device="cuda")
    y, _ = run_gpu(ssm, inp, h_last=hl)
    assert torch.count_nonzero(y).item() == 0 and torch.count_nonzero(hl).item() == 0


def _sampled_parity(S, name, n_ch, seed=0):
    w = WORKLOADS[name]
    d = w.dims
    inp = scan_inputs(d["b"], d["L"], d["d_in"], d["N"], w.dtype, w.seed)
    g = to_cuda(inp)
    hl = torch.empty(d["b"], d["d_in"], d["N"], device="cuda")
    y = S.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                       dt_bias=g["dt_bias"], h_last=hl)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed)
    # first and last channel of the tiles at both ends, plus random ones
    chans = sorted(set([0, 31, 32, d["d_in"] - 1] + rng.choice(d["d_in"], n_ch, False).tolist()))
    bsel = sorted(set([0, d["b"] - 1]))
    sub = lambda t: t[bsel][:, :, chans].contiguous()
    ref_in = dict(u=sub(inp["u"]), delta=sub(inp["delta"]), A=inp["A"][chans], B=inp["B"][bsel],
                  C=inp["C"][bsel], D=inp["D"][chans], z=sub(inp["z"]),
                  dt_bias=inp["dt_bias"][chans], h0=None)
    y_ref, h_ref = run_oracle(ref_in, last=True)
    y_got = y[bsel][:, :, chans]
    h_got = hl[bsel][:, chans]
    return rel_err(y_got, y_ref), rel_err(h_got, h_ref)


def test_mamba130m_workload_sampled(ssm):
    ey, eh = _sampled_parity(ssm, "mamba130m-scan", 28)
    assert ey <= 2e-2 and eh <= 2e-2, (ey, eh)


def test_mamba14b_long_workload_sampled(ssm):
    ey, eh = _sampled_parity(ssm, "mamba1.4b-long-scan", 12)
    assert ey <= 2e-2 and eh <= 2e-2, (ey, eh)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,L,d_in,N", [
    (1, 3000, 64, 16), (2, 777, 32, 8), (1, 1000, 32, 32), (1, 257, 32, 16), (3, 4100, 40, 16),
    (1, 16384, 8, 16),  # 128 blocks: four 32-block tiles of the carry scan
    (2, 10000, 16, 8),  # 63 blocks of 160 steps: a ragged second tile
])
def test_split_scan(ssm, dtype, b, L, d_in, N):
    """Few channels and a long sequence: the sequence is cut into blocks whose
    maps are summarised, composed from h0 (a warp-shuffle scan over the
    blocks, 32 at a time, each tile carrying into the next) and replayed in
    parallel.  The blocks' last one is ragged in every case but the first
    of the two long ones."""
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    need = ssm.ssm_scan_fwd_workspace_bytes(b, L, d_in, N)
    if d_in % 8 == 0:
        assert need > 0, "this shape should take the split scan"
    inp = scan_inputs(b, L, d_in, N, dt, seed=L + d_in + N, with_h0=True)
    hl = torch.empty(b, d_in, N, device="cuda")
    y, _ = run_gpu(ssm, inp, h_last=hl)
    y_ref, h_ref = run_oracle(inp, last=True)
    assert rel_err(y, y_ref) <= TOL[dtype]
    assert rel_err(hl, h_ref) <= TOL[dtype]


def test_split_scan_resume_and_zero_start(ssm):
    """The split scan from a carried state equals one scan over both parts,
    and without h0 its first block starts from zero."""
    inp = scan_inputs(1, 2048, 64, 16, "fp32", seed=21)
    g = to_cuda(inp)
    assert ssm.ssm_scan_fwd_workspace_bytes(1, 1024, 64, 16) > 0
    y_full = ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                               dt_bias=g["dt_bias"])
    h = torch.empty(1, 64, 16, device="cuda")
    part = lambda t, s: t[:, s].contiguous()
    s1, s2 = slice(0, 1024), slice(1024, None)
    y1 = ssm.ssm_scan_fwd(part(g["u"], s1), part(g["delta"], s1), g["A"], part(g["B"], s1),
                           part(g["C"], s1), D=g["D"], z=part(g["z"], s1), dt_bias=g["dt_bias"],
                           h_last=h)
    y2 = ssm.ssm_scan_fwd(part(g["u"], s2), part(g["delta"], s2), g["A"], part(g["B"], s2),
                           part(g["C"], s2), D=g["D"], z=part(g["z"], s2), dt_bias=g["dt_bias"],
                           h0=h)
    assert rel_err(torch.cat([y1, y2], 1), y_full) <= 1e-5
    assert rel_err(y_full, run_oracle(inp)) <= 1e-4


def test_split_scan_rejects_a_short_workspace(ssm):
    inp = scan_inputs(1, 3000, 64, 16, "bf16", seed=2)
    g = to_cuda(inp)
    need = ssm.ssm_scan_fwd_workspace_bytes(1, 3000, 64, 16)
    ws = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(Exception):
        ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], workspace=ws)
