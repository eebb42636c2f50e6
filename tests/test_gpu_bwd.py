"""GPU parity of ssm_scan_bwd (the reverse-time adjoint of the selective
scan) against the fp64 oracle's backward, through the C ABI.

Activation-dtype gradients (du, ddelta, dz) are held to the forward's
tolerances (1e-4 fp32, 2e-2 bf16: one rounding to bf16 at the store).  The
fp32 gradients (dA, dB, dC, dD, ddt_bias, dh0) come from fp32 arithmetic in
both modes; they are sums of up to b*L or d_in terms, so they are held to
1e-4 (fp32 inputs) / 2e-4 (bf16 inputs) in the same metric (fp32's 6e-8 unit
roundoff times the few hundred roundings of the longest accumulation chain,
with margin)."""
import numpy as np
import pytest
import torch

import oracle
from _helpers import TOL, rel_err, to64, to_cuda
from selective_state_space_25_b200.synthetic import WORKLOADS, scan_inputs

pytestmark = pytest.mark.gpu

ACT = ("du", "ddelta", "dz")
F32 = ("dA", "dB", "dC", "dD", "ddt_bias", "dh0")


def _tol(name, dtype):
    if name in ACT:
        return TOL[dtype]
    return 1e-4 if dtype == torch.float32 else 2e-4


def _dout(b, L, d_in, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(b, L, d_in, generator=g).to(dtype)


def _run(S, inp, dout, h0=None, dh_last=None, softplus=True):
    g = to_cuda(inp)
    return S.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout.cuda(), D=g["D"],
                          z=g["z"], dt_bias=g["dt_bias"], delta_softplus=softplus,
                          h0=None if h0 is None else h0.cuda(),
                          dh_last=None if dh_last is None else dh_last.cuda(), want_dh0=True)


def _ref(inp, dout, h0=None, dh_last=None, softplus=True):
    return oracle.selective_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dout,
                                     D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                     delta_softplus=softplus, h0=h0, dh_last=dh_last)


def _compare(got, ref, dtype, names=None):
    for k in names or ref:
        e = rel_err(got[k], ref[k])
        assert e <= _tol(k, dtype), (k, e)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,L,d_in,N", [
    (2, 64, 32, 16), (1, 97, 40, 16), (2, 33, 8, 4), (1, 50, 130, 1), (2, 17, 64, 2),
    (1, 70, 20, 8), (1, 45, 24, 32), (1, 31, 12, 64), (3, 1, 16, 16), (1, 300, 48, 16),
    (1, 50, 36, 16),
])
def test_bwd_shapes(ssm, dtype, b, L, d_in, N):
    """d_state 8, 16, 32 with 16-byte rows (d_in a multiple of 8 in bf16, of
    4 in fp32) take the forward kernel's states pass; the rest (d_in 20 or 36
    in bf16, other d_state) the backward kernel's own first pass."""
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = scan_inputs(b, L, d_in, N, dt, seed=b * 7 + L + d_in + N)
    dout = _dout(b, L, d_in, dtype, seed=L)
    g = torch.Generator().manual_seed(d_in)
    h0 = torch.randn(b, d_in, N, generator=g)
    dhl = torch.randn(b, d_in, N, generator=g)
    got = _run(ssm, inp, dout, h0, dhl)
    _compare(got, _ref(inp, dout, h0, dhl), dtype)


def test_bwd_no_softplus_no_gate_no_D(ssm):
    inp = scan_inputs(2, 77, 24, 16, "fp32", seed=3, with_z=False, with_D=False)
    inp["delta"] = inp["delta"].abs() * 0.2
    inp["dt_bias"] = None
    dout = _dout(2, 77, 24, torch.float32, seed=4)
    got = _run(ssm, inp, dout, softplus=False)
    ref = _ref(inp, dout, softplus=False)
    assert "dz" not in got
    _compare(got, ref, torch.float32)


def test_bwd_L0(ssm):
    """No steps: every summed gradient is zero and dh0 is dh_last."""
    b, d_in, N = 2, 16, 16
    A = -torch.rand(d_in, N, device="cuda") - 0.5
    e = torch.empty(b, 0, d_in, device="cuda")
    eB = torch.empty(b, 0, N, device="cuda")
    dhl = torch.randn(b, d_in, N, device="cuda")
    got = ssm.ssm_scan_bwd(e, e, A, eB, eB, e, D=torch.ones(d_in, device="cuda"),
                           dt_bias=torch.zeros(d_in, device="cuda"), dh_last=dhl, want_dh0=True)
    assert torch.equal(got["dh0"], dhl)
    assert not got["dA"].any() and not got["dD"].any() and not got["ddt_bias"].any()


def test_bwd_rejects_small_workspace(ssm):
    inp = to_cuda(scan_inputs(1, 40, 16, 16, "fp32", seed=5))
    dout = torch.randn(1, 40, 16, device="cuda")
    ws = torch.empty(ssm.ssm_scan_bwd_workspace_bytes(1, 40, 16, 16) - 4, dtype=torch.uint8,
                     device="cuda")
    with pytest.raises(ssm.SsmError, match="workspace"):
        ssm.ssm_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dout, workspace=ws)


def test_bwd_split_sequence_chains_through_dh(ssm):
    """Backward over [0, L) equals the backward of the second half (from the
    first half's last state) followed by the first half's backward with
    dh_last = the second half's dh0: the gradient of a resumed scan."""
    b, L, d_in, N, L1 = 2, 150, 32, 16, 61
    inp = to_cuda(scan_inputs(b, L, d_in, N, "fp32", seed=9))
    dout = torch.randn(b, L, d_in, device="cuda")
    full = ssm.ssm_scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dout, D=inp["D"],
                            z=inp["z"], dt_bias=inp["dt_bias"], want_dh0=True)
    part = lambda t, s: t[:, s].contiguous()
    first, second = slice(0, L1), slice(L1, L)
    h_mid = torch.empty(b, d_in, N, device="cuda")
    ssm.ssm_scan_fwd(part(inp["u"], first), part(inp["delta"], first), inp["A"],
                     part(inp["B"], first), part(inp["C"], first), D=inp["D"],
                     z=part(inp["z"], first), dt_bias=inp["dt_bias"], h_last=h_mid)
    g2 = ssm.ssm_scan_bwd(part(inp["u"], second), part(inp["delta"], second), inp["A"],
                          part(inp["B"], second), part(inp["C"], second), part(dout, second),
                          D=inp["D"], z=part(inp["z"], second), dt_bias=inp["dt_bias"],
                          h0=h_mid, want_dh0=True)
    g1 = ssm.ssm_scan_bwd(part(inp["u"], first), part(inp["delta"], first), inp["A"],
                          part(inp["B"], first), part(inp["C"], first), part(dout, first),
                          D=inp["D"], z=part(inp["z"], first), dt_bias=inp["dt_bias"],
                          dh_last=g2["dh0"], want_dh0=True)
    for k in ("du", "ddelta", "dz", "dB", "dC"):
        assert rel_err(torch.cat([g1[k], g2[k]], 1), full[k].cpu().double().numpy()) <= 1e-4, k
    for k in ("dA", "dD", "ddt_bias"):
        assert rel_err(g1[k] + g2[k], full[k].cpu().double().numpy()) <= 1e-4, k
    assert rel_err(g1["dh0"], full["dh0"].cpu().double().numpy()) <= 1e-4


def test_bwd_mamba130m_workload_sampled(ssm):
    """The Mamba-130M-shaped prefill (b=8, L=2048, d_in=1536, N=16, bf16) at
    full size: per-channel gradients on sampled channels of every batch, and
    the channel sums dB, dC on one whole batch."""
    w = WORKLOADS["mamba130m-scan"]
    d = w.dims
    b, L, d_in, N = d["b"], d["L"], d["d_in"], d["N"]
    inp = scan_inputs(b, L, d_in, N, w.dtype, w.seed)
    dout = _dout(b, L, d_in, torch.bfloat16, seed=11)
    got = _run(ssm, inp, dout)
    torch.cuda.synchronize()
    chans = [0, 1, 31, 32, 767, 1000, 1535]
    sl = lambda t: t[..., chans].contiguous()
    sub = dict(u=sl(inp["u"]), delta=sl(inp["delta"]), A=inp["A"][chans], B=inp["B"],
               C=inp["C"], D=inp["D"][chans], z=sl(inp["z"]), dt_bias=inp["dt_bias"][chans])
    ref = _ref(sub, sl(dout))
    for k in ("du", "ddelta", "dz"):
        assert rel_err(got[k][..., chans], ref[k]) <= TOL[torch.bfloat16], k
    for k in ("dA", "dD", "ddt_bias"):
        assert rel_err(got[k][chans], ref[k]) <= 2e-4, k
    one = lambda t: t[:1].contiguous()
    ref1 = _ref(dict(u=one(inp["u"]), delta=one(inp["delta"]), A=inp["A"], B=one(inp["B"]),
                     C=one(inp["C"]), D=inp["D"], z=one(inp["z"]), dt_bias=inp["dt_bias"]),
                one(dout))
    for k in ("dB", "dC"):
        assert rel_err(got[k][:1], ref1[k]) <= 2e-4, k


# ------------------------------------ forward-saved chunk states (training split)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,L,d_in,N,split", [
    (2, 100, 32, 16, False), (1, 33, 20, 4, False), (2, 48, 16, 1, False), (1, 70, 24, 8, False),
    (1, 16, 8, 64, False),
    (1, 1000, 32, 8, True),    # split scan: 7 blocks of 160 steps, the last ragged
    (2, 2100, 64, 16, True),   # 14 blocks, two batches
    (1, 1300, 48, 32, True),
])
def test_fwd_save_states_match_oracle_prefix_scans(ssm, dtype, b, L, d_in, N, split):
    """Saved state c is the state after the first 16 c steps: the oracle's
    h_last of the scan over that prefix (chunk 0 is h0).  Few channels over a
    long sequence take the split scan (the binding allocates its workspace):
    the scan pass of every block writes its chunks' states."""
    assert (ssm.ssm_scan_fwd_workspace_bytes(b, L, d_in, N) > 0) == split
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = scan_inputs(b, L, d_in, N, dt, seed=L + N, with_h0=True)
    g = to_cuda(inp)
    nbytes = ssm.ssm_scan_bwd_workspace_bytes(b, L, d_in, N)
    states = torch.empty(nbytes // 4, device="cuda")
    hl = torch.empty(b, d_in, N, device="cuda")
    y = ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                         dt_bias=g["dt_bias"], h0=g["h0"], h_last=hl, chunk_states=states)
    y_ref, h_ref = oracle.selective_scan(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                         D=inp["D"], z=inp["z"], dt_bias=inp["dt_bias"],
                                         h0=inp["h0"], return_last_state=True)
    assert rel_err(y, y_ref) <= TOL[dtype]
    assert rel_err(hl, h_ref) <= 1e-4
    nC = (L + 15) // 16
    got = states.view(b, nC, d_in, N)
    if split:  # the one-pass forward (no workspace) saves the same states within rounding
        one = torch.empty_like(states)
        y1 = ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                              dt_bias=g["dt_bias"], h0=g["h0"], chunk_states=one,
                              workspace=torch.empty(0, dtype=torch.uint8, device="cuda"))
        assert rel_err(states, to64(one)) <= 1e-4
        assert rel_err(y, to64(y1)) <= TOL[dtype]
    for c in range(0, nC, 1 if nC <= 40 else 5):
        if c == 0:
            ref = to64(inp["h0"])
        else:
            pre = lambda t: t[:, :16 * c].contiguous()
            _, ref = oracle.selective_scan(pre(inp["u"]), pre(inp["delta"]), inp["A"], pre(inp["B"]),
                                           pre(inp["C"]), dt_bias=inp["dt_bias"], h0=inp["h0"],
                                           return_last_state=True)
        assert rel_err(got[:, c], ref) <= 1e-4, c


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_bwd_saved_equals_self_contained(ssm, dtype):
    """The backward from the forward's saved states gives the gradients of
    the self-contained backward (the same states, the same arithmetic; only
    the order of the atomic channel sums may differ)."""
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    b, L, d_in, N = 2, 203, 48, 16
    inp = scan_inputs(b, L, d_in, N, dt, seed=17, with_h0=True)
    g = to_cuda(inp)
    dout = _dout(b, L, d_in, dtype, seed=18).cuda()
    dhl = torch.randn(b, d_in, N, device="cuda")
    states = torch.empty(ssm.ssm_scan_bwd_workspace_bytes(b, L, d_in, N) // 4, device="cuda")
    ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                     dt_bias=g["dt_bias"], h0=g["h0"], chunk_states=states)
    kw = dict(D=g["D"], z=g["z"], dt_bias=g["dt_bias"], dh_last=dhl, want_dh0=True)
    # the minimum workspace: the unsplit backward, the saved call's arithmetic
    least = torch.empty(ssm.ssm_scan_bwd_workspace_bytes(b, L, d_in, N), dtype=torch.uint8,
                        device="cuda")
    full = ssm.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout, h0=g["h0"],
                            workspace=least, **kw)
    # no workspace for the saved call: unsplit as well
    none = torch.empty(0, dtype=torch.uint8, device="cuda")
    saved = ssm.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout, states=states,
                             workspace=none, **kw)
    for k in full:
        assert rel_err(saved[k], to64(full[k])) <= 1e-5, k
    ref = _ref(inp, dout.cpu(), inp["h0"], dhl.cpu())
    _compare(saved, ref, dtype)


def test_fwd_save_rejects_small_buffer(ssm):
    inp = to_cuda(scan_inputs(1, 40, 16, 16, "fp32", seed=5))
    states = torch.empty(ssm.ssm_scan_bwd_workspace_bytes(1, 40, 16, 16) // 4 - 1, device="cuda")
    with pytest.raises(ssm.SsmError, match="chunk_states"):
        ssm.ssm_scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], chunk_states=states)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,L,d_in,N,with_z", [
    (1, 4096, 64, 16, True),   # 256 chunks in blocks; the forward's states pass split too
    (2, 1000, 32, 8, True),    # ragged last chunk and block
    (1, 777, 48, 32, False),   # no gate
    (1, 300, 64, 16, True),    # few blocks
])
def test_bwd_split(ssm, dtype, b, L, d_in, N, with_z):
    """Few channels: with the fast workspace ssm_scan_bwd cuts the chunks into
    blocks (the forward's split scan for the chunk-start states, each block's
    adjoint map composed from dh_last by the carry scan, every block's
    backward at once).  The gradients match the oracle and, within rounding,
    the unsplit backward the minimum workspace runs."""
    need = ssm.ssm_scan_bwd_workspace_bytes(b, L, d_in, N)
    fast = ssm.ssm_scan_bwd_fast_workspace_bytes(b, L, d_in, N)
    assert fast > need, "this shape should take the split backward"
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = scan_inputs(b, L, d_in, N, dt, seed=L + d_in + N, with_z=with_z)
    dout = _dout(b, L, d_in, dtype, seed=L + 1)
    g = torch.Generator().manual_seed(d_in + 3)
    h0 = torch.randn(b, d_in, N, generator=g)
    dhl = torch.randn(b, d_in, N, generator=g)
    c = to_cuda(inp)

    def run(nbytes):
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        return ssm.ssm_scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dout.cuda(),
                                D=c["D"], z=c["z"], dt_bias=c["dt_bias"], h0=h0.cuda(),
                                dh_last=dhl.cuda(), want_dh0=True, workspace=ws)

    split, one = run(fast), run(need)
    _compare(split, _ref(inp, dout, h0, dhl), dtype)
    # the chunk states and the adjoint reach each block by composed maps, so
    # the two paths round differently: they agree within the parity tolerances
    for k in one:
        assert rel_err(split[k], one[k]) <= _tol(k, dtype), k


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("b,L,d_in,N,with_z", [
    (1, 4096, 64, 16, True),
    (2, 1000, 32, 8, True),    # ragged last chunk and block
    (1, 777, 48, 32, False),
    (2, 203, 48, 16, True),    # three blocks
])
def test_bwd_saved_split(ssm, dtype, b, L, d_in, N, with_z):
    """Few channels, from the forward's saved chunk states: with
    ssm_scan_bwd_saved_workspace_bytes of workspace the backward runs in
    blocks (no states pass; the adjoint maps composed from dh_last), without
    it unsplit.  Both match the oracle, and each other within rounding."""
    aux = ssm.ssm_scan_bwd_saved_workspace_bytes(b, L, d_in, N)
    assert aux > 0, "this shape should take the split backward"
    dt = "bf16" if dtype == torch.bfloat16 else "fp32"
    inp = scan_inputs(b, L, d_in, N, dt, seed=3 * L + d_in, with_z=with_z, with_h0=True)
    dout = _dout(b, L, d_in, dtype, seed=L + 7)
    dhl = torch.randn(b, d_in, N, generator=torch.Generator().manual_seed(N + 5))
    c = to_cuda(inp)
    states = torch.empty(ssm.ssm_scan_bwd_workspace_bytes(b, L, d_in, N) // 4, device="cuda")
    ssm.ssm_scan_fwd(c["u"], c["delta"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                     dt_bias=c["dt_bias"], h0=c["h0"], chunk_states=states)
    kept = states.clone()

    def run(nbytes):
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        return ssm.ssm_scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dout.cuda(),
                                D=c["D"], z=c["z"], dt_bias=c["dt_bias"], states=states,
                                dh_last=dhl.cuda(), want_dh0=True, workspace=ws)

    split, one = run(aux), run(0)
    assert torch.equal(states, kept), "the saved states are read only"
    _compare(split, _ref(inp, dout, inp["h0"], dhl), dtype)
    for k in one:
        assert rel_err(split[k], one[k]) <= _tol(k, dtype), k
    # the binding's default allocates the split's workspace
    dflt = ssm.ssm_scan_bwd(c["u"], c["delta"], c["A"], c["B"], c["C"], dout.cuda(), D=c["D"],
                            z=c["z"], dt_bias=c["dt_bias"], states=states, dh_last=dhl.cuda(),
                            want_dh0=True)
    for k in ("du", "ddelta", "dh0"):
        assert torch.equal(dflt[k], split[k]), k
