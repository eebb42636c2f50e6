"""The library's calls can be captured in a CUDA graph and replayed: they
allocate nothing and never synchronise, so a serving or training loop can
run them from a graph.  Replays must equal eager calls bit for bit (same
kernels, same inputs)."""
import pytest
import torch

from _helpers import to_cuda
from selective_state_space_25_b200.synthetic import conv_inputs, scan_inputs, ss2d_inputs, step_inputs

pytestmark = pytest.mark.gpu


def test_decode_steps_in_a_graph(ssm):
    inp = to_cuda(step_inputs(4, 256, 16, "bf16", seed=3))
    c = to_cuda(conv_inputs(4, 256, 4, "bf16", seed=4))
    st_e, cs_e = inp["state"].clone(), c["conv_state"].clone()
    st_g, cs_g = inp["state"].clone(), c["conv_state"].clone()
    y_e = torch.empty_like(inp["x"])
    y_g = torch.empty_like(inp["x"])

    def step(st, cs, y):
        ssm.ssm_conv_state_update(cs, c["conv_weight"], st, inp["x"], inp["dt"], inp["A"], inp["B"],
                                  inp["C"], conv_bias=c["conv_bias"], D=inp["D"], z=inp["z"],
                                  dt_bias=inp["dt_bias"], y=y)

    step(st_e, cs_e, y_e)          # first call outside capture (sets kernel attributes)
    st_e.copy_(inp["state"]); cs_e.copy_(c["conv_state"])
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        for _ in range(5):         # five decode steps in one graph
            step(st_g, cs_g, y_g)
    st_g.copy_(inp["state"]); cs_g.copy_(c["conv_state"])
    torch.cuda.synchronize()
    for _ in range(2):             # two replays = ten steps
        graph.replay()
    for _ in range(10):
        step(st_e, cs_e, y_e)
    torch.cuda.synchronize()
    assert torch.equal(st_g, st_e) and torch.equal(cs_g, cs_e) and torch.equal(y_g, y_e)


def test_scan_fwd_bwd_and_ss2d_in_a_graph(ssm):
    b, L, d_in, N = 2, 100, 64, 16
    g = to_cuda(scan_inputs(b, L, d_in, N, "bf16", seed=5))
    dout = torch.randn(b, L, d_in, device="cuda").to(torch.bfloat16)
    states = torch.empty(ssm.ssm_scan_bwd_workspace_bytes(b, L, d_in, N) // 4, device="cuda")
    s2 = to_cuda(ss2d_inputs(2, 9, 7, 16, 1, "bf16", seed=6))
    y = torch.empty_like(g["u"])
    y2 = torch.empty_like(s2["u"])

    def work(out):
        ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                         dt_bias=g["dt_bias"], y=y, chunk_states=states)
        ssm.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout, D=g["D"], z=g["z"],
                         dt_bias=g["dt_bias"], states=states, out=out)
        ssm.ss2d_scan_fwd(s2["u"], s2["delta"], s2["A"], s2["B"], s2["C"], 9, 7, D=s2["D"], y=y2)

    eager = ssm.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout, D=g["D"], z=g["z"],
                             dt_bias=g["dt_bias"])
    work(eager)
    torch.cuda.synchronize()
    y_e, y2_e = y.clone(), y2.clone()
    ref = {k: v.clone() for k, v in eager.items()}
    out = {k: torch.empty_like(v) for k, v in eager.items()}
    work(out)                      # warm the captured variants' attributes
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        work(out)
    y.zero_(); y2.zero_()
    for v in out.values():
        v.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_e) and torch.equal(y2, y2_e)
    for k in ("du", "ddelta", "dz", "dA"):
        # dA sums over CTAs with atomics, so only its rounding order may differ
        if k == "dA":
            assert torch.allclose(out[k], ref[k], rtol=1e-5, atol=1e-6)
        else:
            assert torch.equal(out[k], ref[k]), k


def test_split_scan_in_a_graph(ssm):
    """The split scan (few channels, long sequence: summary, carry and scan
    passes, the last two launched to start while the pass before finishes)
    captured in a graph replays bit for bit."""
    b, L, d_in, N = 1, 4096, 64, 16
    need = ssm.ssm_scan_fwd_workspace_bytes(b, L, d_in, N)
    assert need > 0, "this shape should take the split scan"
    g = to_cuda(scan_inputs(b, L, d_in, N, "bf16", seed=9, with_h0=True))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    y = torch.empty_like(g["u"])
    hl = torch.empty(b, d_in, N, device="cuda")

    def work():
        ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                         dt_bias=g["dt_bias"], h0=g["h0"], h_last=hl, y=y, workspace=ws)

    work()
    torch.cuda.synchronize()
    y_e, hl_e = y.clone(), hl.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        work()
    y.zero_()
    hl.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(y, y_e) and torch.equal(hl, hl_e)


@pytest.mark.parametrize("saved", [False, True])
def test_split_backward_in_a_graph(ssm, saved):
    """The split backward (few channels: the chunk states from the forward's
    split scan or from the saved ones, the adjoint's block maps, the carry
    scan, every block at once) captured in a graph replays the eager call:
    the per-channel gradients bit for bit, the channel sums within rounding
    (they are taken with atomics)."""
    b, L, d_in, N = 1, 4096, 64, 16
    g = to_cuda(scan_inputs(b, L, d_in, N, "bf16", seed=10, with_h0=True))
    dout = torch.randn(b, L, d_in, device="cuda").to(torch.bfloat16)
    dhl = torch.randn(b, d_in, N, device="cuda")
    states = None
    if saved:
        states = torch.empty(ssm.ssm_scan_bwd_workspace_bytes(b, L, d_in, N) // 4, device="cuda")
        ssm.ssm_scan_fwd(g["u"], g["delta"], g["A"], g["B"], g["C"], D=g["D"], z=g["z"],
                         dt_bias=g["dt_bias"], h0=g["h0"], chunk_states=states)
        nbytes = ssm.ssm_scan_bwd_saved_workspace_bytes(b, L, d_in, N)
        assert nbytes > 0, "this shape should take the saved split"
    else:
        nbytes = ssm.ssm_scan_bwd_fast_workspace_bytes(b, L, d_in, N)
        assert nbytes > ssm.ssm_scan_bwd_workspace_bytes(b, L, d_in, N), "should split"
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    kw = dict(D=g["D"], z=g["z"], dt_bias=g["dt_bias"], dh_last=dhl, want_dh0=True,
              workspace=ws, h0=None if saved else g["h0"], states=states)
    ref = ssm.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout, **kw)
    out = {k: torch.empty_like(v) for k, v in ref.items()}

    def work():
        ssm.ssm_scan_bwd(g["u"], g["delta"], g["A"], g["B"], g["C"], dout, out=out, **kw)

    work()
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        work()
    for v in out.values():
        v.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for k in ("du", "ddelta", "dz", "dh0"):
        assert torch.equal(out[k], ref[k]), k
    for k in ("dA", "dB", "dC", "dD", "ddt_bias"):
        # a sum near zero takes the rounding of its terms: measured on the scale
        assert (out[k] - ref[k]).abs().max() <= 1e-5 * ref[k].abs().max(), k
