"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every function include/ssmscan.h declares, and rejects bad arguments with the
documented status before anything touches CUDA.  Pointers passed here are
fake (never dereferenced): every call below fails validation first, or is an
empty problem that returns before any CUDA call."""
import ctypes

import pytest

from selective_state_space_25_b200 import ssmscan as S

L = S.lib()
FAKE = 0x100000          # 16-byte aligned, never dereferenced
ODD = 0x100001           # misaligned for every element type


def test_exports_every_declared_function():
    names = S.header_functions()
    assert {"ssm_scan_fwd", "ss2d_scan_fwd", "ssm_state_update", "ss2d_cross_scan",
            "ss2d_cross_merge", "ssm_last_error", "ssm_check_device_errors",
            "ssm_scan_fwd_workspace_bytes", "ss2d_scan_fwd_workspace_bytes",
            "ssm_version"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"libssmscan.so does not export {n}"


def test_version_and_empty_error():
    assert S.version().count(".") == 2
    assert isinstance(S.last_error(), str)


def scan(**kw):
    a = dict(u=FAKE, delta=FAKE, A=FAKE, B=FAKE, C=FAKE, D=None, z=None, dt_bias=None, sp=1,
             h0=None, h_last=None, y=FAKE + 4096, b=2, L=8, d_in=16, N=16, dtype=S.SSM_BF16,
             ws=None, ws_bytes=0, stream=None)
    a.update(kw)
    return L.ssm_scan_fwd(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["dt_bias"],
                          a["sp"], a["h0"], a["h_last"], a["y"], a["b"], a["L"], a["d_in"], a["N"],
                          a["dtype"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(b=-1), S.SSM_ERR_INVALID_ARG),
    (dict(L=-3), S.SSM_ERR_INVALID_ARG),
    (dict(d_in=-1), S.SSM_ERR_INVALID_ARG),
    (dict(N=3), S.SSM_ERR_UNSUPPORTED),
    (dict(N=128), S.SSM_ERR_UNSUPPORTED),
    (dict(N=0), S.SSM_ERR_UNSUPPORTED),
    (dict(dtype=7), S.SSM_ERR_UNSUPPORTED),
    (dict(b=2 ** 40, L=2 ** 40), S.SSM_ERR_INVALID_ARG),
    (dict(u=None), S.SSM_ERR_INVALID_ARG),
    (dict(A=None), S.SSM_ERR_INVALID_ARG),
    (dict(y=None), S.SSM_ERR_INVALID_ARG),
    (dict(C=None), S.SSM_ERR_INVALID_ARG),
    (dict(u=ODD), S.SSM_ERR_INVALID_ARG),
    (dict(A=FAKE + 2), S.SSM_ERR_INVALID_ARG),
    (dict(h0=FAKE + 1), S.SSM_ERR_INVALID_ARG),
    (dict(y=FAKE), S.SSM_ERR_INVALID_ARG),            # y aliases u
    (dict(y=FAKE + 2), S.SSM_ERR_INVALID_ARG),        # y overlaps u, shifted by one element
    (dict(y=FAKE + 510), S.SSM_ERR_INVALID_ARG),      # y starts on u's last element
    (dict(y=FAKE + 512), S.SSM_ERR_INVALID_ARG),      # y overlaps A (d_in * N * 4 bytes at FAKE)
    (dict(y=FAKE + 4096, h_last=FAKE + 4096 + 256), S.SSM_ERR_INVALID_ARG),  # h_last overlaps y
    (dict(b=0), S.SSM_OK),                            # empty problem, no CUDA call
    (dict(d_in=0), S.SSM_OK),
])
def test_scan_validation(kw, status):
    assert scan(**kw) == status
    if status != S.SSM_OK:
        assert S.last_error() != ""


def test_workspace_query():
    # channels enough to fill the GPU: one pass, no workspace
    assert S.ssm_scan_fwd_workspace_bytes(8, 2048, 1536, 16) == 0
    assert S.ssm_scan_fwd_workspace_bytes(2, 16384, 4096, 16) == 0
    # few channels and a long sequence: the split scan keeps two fp32
    # (b, blocks, d_in, N) arrays (block decays and block states)
    ws = S.ssm_scan_fwd_workspace_bytes(1, 16384, 64, 16)
    assert ws > 0 and ws % (2 * 64 * 16 * 4) == 0
    # 48 CTAs of 32 channels on 148 SMs: 12 blocks (576 CTAs, two whole waves
    # of two per SM), not 13 (624, a third wave)
    assert S.ssm_scan_fwd_workspace_bytes(1, 16384, 1536, 16) == 2 * 12 * 1536 * 16 * 4
    assert S.ssm_scan_fwd_workspace_bytes(1, 200, 64, 16) == 0       # too short to split
    assert S.ssm_scan_fwd_workspace_bytes(1, 16384, 64, 64) == 0     # d_state 64: one pass
    assert S.ssm_scan_fwd_workspace_bytes(1, 16384, 60, 16) == 0     # d_in not a multiple of 8
    assert L.ssm_scan_fwd_workspace_bytes(-1, 1, 1, 16) == ctypes.c_size_t(-1).value
    assert S.ss2d_scan_fwd_workspace_bytes(32, 56, 56, 192, 1) == 0
    big = S.ss2d_scan_fwd_workspace_bytes(2, 100, 100, 16, 1)
    assert big == 2 * 100 * 100 * 16 * 4
    # the direction split's four fp32 slices for small batches; otherwise the
    # minimum
    assert S.ss2d_scan_fwd_fast_workspace_bytes(1, 56, 56, 192, 1) == 4 * 56 * 56 * 192 * 4
    assert S.ss2d_scan_fwd_fast_workspace_bytes(32, 56, 56, 192, 1) == 0
    assert S.ss2d_scan_fwd_fast_workspace_bytes(2, 100, 100, 16, 1) == 4 * big
    # large images take the split at any batch; small ones only at small batch
    assert S.ss2d_scan_fwd_fast_workspace_bytes(80, 100, 100, 16, 1) == \
        4 * S.ss2d_scan_fwd_workspace_bytes(80, 100, 100, 16, 1)
    assert S.ss2d_scan_fwd_fast_workspace_bytes(80, 56, 56, 16, 1) == 0
    assert L.ss2d_scan_fwd_fast_workspace_bytes(-1, 2, 2, 8, 1) == ctypes.c_size_t(-1).value


def ss2d(**kw):
    a = dict(u=FAKE, delta=FAKE, A=FAKE, B=FAKE, C=FAKE, D=None, dt_bias=None, sp=1,
             y=FAKE + 8192, b=2, H=4, W=5, d_in=8, N=1, dtype=S.SSM_BF16, ws=None, ws_bytes=0,
             stream=None)
    a.update(kw)
    return L.ss2d_scan_fwd(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["dt_bias"],
                           a["sp"], a["y"], a["b"], a["H"], a["W"], a["d_in"], a["N"], a["dtype"],
                           a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(H=-1), S.SSM_ERR_INVALID_ARG),
    (dict(N=16), S.SSM_ERR_UNSUPPORTED),
    (dict(dtype=5), S.SSM_ERR_UNSUPPORTED),
    (dict(delta=None), S.SSM_ERR_INVALID_ARG),
    (dict(y=FAKE), S.SSM_ERR_INVALID_ARG),
    (dict(y=FAKE + 2558), S.SSM_ERR_INVALID_ARG),     # y overlaps delta's last element
    (dict(B=ODD), S.SSM_ERR_INVALID_ARG),
    (dict(H=100, W=100), S.SSM_ERR_WORKSPACE),        # accumulator needs the workspace
    (dict(b=0), S.SSM_OK),
    (dict(W=0), S.SSM_OK),
])
def test_ss2d_validation(kw, status):
    assert ss2d(**kw) == status


BIG_WS = FAKE + (1 << 44)  # far from every input range, never dereferenced


@pytest.mark.parametrize("kw", [
    dict(b=1, H=2048, W=2048, d_in=8),     # H W = 2^22: per-image offsets are 32-bit
    dict(b=1, H=1024, W=1024, d_in=2048),  # H W d_in = 2^31
    dict(b=70000, H=4, W=5, d_in=8),       # grid.y limit
])
def test_ss2d_size_limits(kw):
    need = S.ss2d_scan_fwd_workspace_bytes(kw["b"], kw["H"], kw["W"], kw["d_in"], 1)
    assert need != ctypes.c_size_t(-1).value
    assert ss2d(ws=BIG_WS if need else None, ws_bytes=need, **kw) == S.SSM_ERR_UNSUPPORTED
    assert S.last_error() != ""


def test_ss2d_unknown_order():
    st = L.ss2d_scan_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, FAKE + 8192, 2, 4, 5, 8,
                            1, 7, S.SSM_BF16, None, 0, None)
    assert st == S.SSM_ERR_UNSUPPORTED and "order" in S.last_error()


def step(**kw):
    a = dict(state=FAKE + 65536, x=FAKE, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, D=None, z=None,
             dt_bias=None, sp=1, y=FAKE + 4096, b=2, d_in=16, N=16, dtype=S.SSM_BF16, stream=None)
    a.update(kw)
    return L.ssm_state_update(a["state"], a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["z"],
                              a["dt_bias"], a["sp"], a["y"], a["b"], a["d_in"], a["N"], a["dtype"],
                              a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(b=-2), S.SSM_ERR_INVALID_ARG),
    (dict(N=5), S.SSM_ERR_UNSUPPORTED),
    (dict(state=None), S.SSM_ERR_INVALID_ARG),
    (dict(state=FAKE + 2), S.SSM_ERR_INVALID_ARG),
    (dict(y=FAKE + 65536), S.SSM_ERR_INVALID_ARG),    # y aliases the state
    (dict(y=FAKE + 65536 + 2046), S.SSM_ERR_INVALID_ARG),  # y overlaps the state's last bytes
    (dict(state=FAKE + 32), S.SSM_ERR_INVALID_ARG),   # the state overlaps x
    (dict(x=ODD), S.SSM_ERR_INVALID_ARG),
    (dict(b=0), S.SSM_OK),
])
def test_step_validation(kw, status):
    assert step(**kw) == status


def test_cross_permutation_validation():
    assert L.ss2d_cross_scan(None, FAKE, 1, 2, 2, 4, S.SSM_BF16, None) == S.SSM_ERR_INVALID_ARG
    # xs (1 x 4 x 4 x 4 bf16, 128 bytes) must not overlap u (32 bytes)
    assert L.ss2d_cross_scan(FAKE, FAKE + 16, 1, 2, 2, 4, S.SSM_BF16, None) == S.SSM_ERR_INVALID_ARG
    assert L.ss2d_cross_merge(FAKE, FAKE + 96, 1, 2, 2, 4, S.SSM_BF16, None) == S.SSM_ERR_INVALID_ARG
    assert L.ss2d_cross_merge(FAKE, FAKE + 64, -1, 2, 2, 4, S.SSM_BF16, None) == S.SSM_ERR_INVALID_ARG
    assert L.ss2d_cross_scan(FAKE, FAKE + 64, 0, 2, 2, 4, S.SSM_BF16, None) == S.SSM_OK


def test_binding_rejects_wrong_tensors():
    import torch
    u = torch.zeros(1, 4, 8)
    with pytest.raises((ValueError, TypeError)):
        S.ssm_scan_fwd(u, u, torch.zeros(8, 16), torch.zeros(1, 4, 16), torch.zeros(1, 4, 15))


def bwd(saved=False, **kw):
    a = dict(u=FAKE, delta=FAKE, A=FAKE, B=FAKE, C=FAKE, D=None, z=None, dt_bias=None, sp=1,
             h0=None, dout=FAKE + 1024, dh_last=None, du=FAKE + 4096, ddelta=FAKE + 8192,
             dA=FAKE + 12288, dB=FAKE + 16384, dC=FAKE + 24576, dD=None, dz=None, ddt_bias=None,
             dh0=None, b=2, L=40, d_in=16, N=16, dtype=S.SSM_BF16, ws=FAKE + 65536,
             ws_bytes=1 << 20, stream=None)
    a.update(kw)
    if saved == "ex":
        return L.ssm_scan_bwd_saved_ex(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"],
                                       a["z"], a["dt_bias"], a["sp"], a["dout"], a["dh_last"],
                                       a["du"], a["ddelta"], a["dA"], a["dB"], a["dC"], a["dD"],
                                       a["dz"], a["ddt_bias"], a["dh0"], a["b"], a["L"],
                                       a["d_in"], a["N"], a["dtype"], a["ws"], a["ws_bytes"],
                                       a.get("aux"), a.get("aux_bytes", 0), a["stream"])
    if saved:
        return L.ssm_scan_bwd_saved(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"],
                                    a["dt_bias"], a["sp"], a["dout"], a["dh_last"], a["du"],
                                    a["ddelta"], a["dA"], a["dB"], a["dC"], a["dD"], a["dz"],
                                    a["ddt_bias"], a["dh0"], a["b"], a["L"], a["d_in"], a["N"],
                                    a["dtype"], a["ws"], a["ws_bytes"], a["stream"])
    return L.ssm_scan_bwd(a["u"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["dt_bias"],
                          a["sp"], a["h0"], a["dout"], a["dh_last"], a["du"], a["ddelta"], a["dA"],
                          a["dB"], a["dC"], a["dD"], a["dz"], a["ddt_bias"], a["dh0"], a["b"], a["L"],
                          a["d_in"], a["N"], a["dtype"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("saved", [False, True, "ex"])
@pytest.mark.parametrize("kw,status", [
    (dict(b=-1), S.SSM_ERR_INVALID_ARG),
    (dict(N=12), S.SSM_ERR_UNSUPPORTED),
    (dict(dtype=3), S.SSM_ERR_UNSUPPORTED),
    (dict(ws_bytes=16), S.SSM_ERR_WORKSPACE),
    (dict(ws=None), S.SSM_ERR_WORKSPACE),
    (dict(b=70000, L=1, d_in=8, ws_bytes=1 << 30), S.SSM_ERR_UNSUPPORTED),  # grid.y limit
    (dict(dA=None), S.SSM_ERR_INVALID_ARG),
    (dict(dout=None), S.SSM_ERR_INVALID_ARG),
    (dict(du=FAKE), S.SSM_ERR_INVALID_ARG),           # an output aliases an input
    (dict(dB=FAKE + 12288), S.SSM_ERR_INVALID_ARG),   # two outputs share a buffer
    (dict(dC=FAKE + 20480), S.SSM_ERR_INVALID_ARG),   # dC overlaps the end of dB
    (dict(ddelta=FAKE + 2048), S.SSM_ERR_INVALID_ARG),  # ddelta overlaps u and dout
    (dict(dout=ODD), S.SSM_ERR_INVALID_ARG),
    (dict(b=0), S.SSM_OK),
])
def test_bwd_validation(saved, kw, status):
    assert bwd(saved=saved, **kw) == status
    if status != S.SSM_OK:
        assert S.last_error() != ""


# b=1, L=16384, d_in=256, N=16 takes the saved split: outputs and the
# chunk states far apart, so that each case overlaps one argument only
SAVED_SPLIT = dict(b=1, L=16384, d_in=256, N=16, du=FAKE + (1 << 40), ddelta=FAKE + (2 << 40),
                   dout=FAKE + (3 << 40), dA=FAKE + (4 << 40), dB=FAKE + (5 << 40),
                   dC=FAKE + (6 << 40), ws=FAKE + (7 << 40), ws_bytes=1 << 30)


@pytest.mark.parametrize("aux,why", [
    (FAKE + (8 << 40) + 2, "not 4-byte aligned"),
    (FAKE + (2 << 40) + 4096, "ddelta and workspace overlap"),
    (FAKE + (1 << 20), "overlaps the input u"),
    (FAKE + (7 << 40) + 64, "overlaps the input chunk_states"),
])
def test_bwd_saved_ex_workspace_validation(aux, why):
    assert bwd(saved="ex", aux=aux, aux_bytes=1 << 22, **SAVED_SPLIT) == S.SSM_ERR_INVALID_ARG
    assert why in S.last_error()


def test_bwd_saved_workspace_query():
    # the saved split needs only the adjoint's block maps: the fast workspace
    # less the chunk states and the forward split's block buffers
    for shape in [(1, 16384, 256, 16), (1, 4096, 64, 16), (2, 1000, 32, 8), (1, 777, 48, 32)]:
        sv = S.ssm_scan_bwd_saved_workspace_bytes(*shape)
        assert sv > 0, shape
        assert sv == (S.ssm_scan_bwd_fast_workspace_bytes(*shape)
                      - S.ssm_scan_bwd_workspace_bytes(*shape)
                      - S.ssm_scan_fwd_workspace_bytes(*shape)), shape
        assert sv % (2 * shape[0] * shape[2] * shape[3] * 4) == 0, shape
    assert S.ssm_scan_bwd_saved_workspace_bytes(8, 2048, 1536, 16) == 0   # fills the GPU
    assert S.ssm_scan_bwd_saved_workspace_bytes(1, 16384, 256, 4) == 0    # d_state 4
    assert S.ssm_scan_bwd_saved_workspace_bytes(1, 40, 16, 16) == 0       # too few chunks
    assert L.ssm_scan_bwd_saved_workspace_bytes(-1, 1, 1, 16) == ctypes.c_size_t(-1).value


def test_bwd_workspace_query():
    assert S.ssm_scan_bwd_workspace_bytes(8, 2048, 1536, 16) == 8 * 128 * 1536 * 16 * 4
    # the split backward's block buffers follow the chunk states for few
    # channels; a shape that fills the GPU runs unsplit
    assert S.ssm_scan_bwd_fast_workspace_bytes(8, 2048, 1536, 16) == 8 * 128 * 1536 * 16 * 4
    need = S.ssm_scan_bwd_workspace_bytes(1, 16384, 256, 16)
    assert S.ssm_scan_bwd_fast_workspace_bytes(1, 16384, 256, 16) > need
    assert S.ssm_scan_bwd_fast_workspace_bytes(1, 16384, 256, 4) == \
        S.ssm_scan_bwd_workspace_bytes(1, 16384, 256, 4)      # d_state 4: no split
    assert L.ssm_scan_bwd_fast_workspace_bytes(-1, 1, 1, 16) == ctypes.c_size_t(-1).value
    assert S.ssm_scan_bwd_workspace_bytes(1, 17, 3, 4) == 1 * 2 * 3 * 4 * 4   # ceil(17 / 16) chunks
    assert L.ssm_scan_bwd_workspace_bytes(1, 1, 1, 3) == ctypes.c_size_t(-1).value


def test_fwd_save_validation():
    args = lambda cs, nbytes, b=2: (FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, None, None,
                                    FAKE + 4096, cs, nbytes, b, 40, 16, 16, S.SSM_BF16, None)
    need = S.ssm_scan_bwd_workspace_bytes(2, 40, 16, 16)
    assert L.ssm_scan_fwd_save(*args(FAKE + 65536, need - 16)) == S.SSM_ERR_WORKSPACE
    assert L.ssm_scan_fwd_save(*args(None, need)) == S.SSM_ERR_WORKSPACE
    assert L.ssm_scan_fwd_save(*args(FAKE + 65540, need)) == S.SSM_ERR_INVALID_ARG  # misaligned
    assert L.ssm_scan_fwd_save(*args(FAKE, need)) == S.SSM_ERR_INVALID_ARG         # aliases u
    assert L.ssm_scan_fwd_save(*args(FAKE + 6144, need)) == S.SSM_ERR_INVALID_ARG  # overlaps y
    assert L.ssm_scan_fwd_save(*args(None, 0, b=0)) == S.SSM_OK


@pytest.mark.parametrize("ws,why", [
    (FAKE + (8 << 40) + 2, "not 4-byte aligned"),
    (FAKE + 4096, "overlaps the input u"),
    (FAKE + (2 << 40) + 4096, "y and workspace overlap"),
    (FAKE + (3 << 40) + 64, "chunk_states and workspace overlap"),
])
def test_fwd_save_ex_workspace_validation(ws, why):
    # b=1, L=4096, d_in=64, N=16 takes the split scan when given its workspace
    b, Ls, d, N = 1, 4096, 64, 16
    nbytes = S.ssm_scan_fwd_workspace_bytes(b, Ls, d, N)
    assert nbytes > 0
    st = L.ssm_scan_fwd_save_ex(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1, None, None,
                                FAKE + (2 << 40), FAKE + (3 << 40),
                                S.ssm_scan_bwd_workspace_bytes(b, Ls, d, N), b, Ls, d, N,
                                S.SSM_BF16, ws, nbytes, None)
    assert st == S.SSM_ERR_INVALID_ARG
    assert why in S.last_error()


def test_split_scan_needs_its_workspace():
    need = S.ssm_scan_fwd_workspace_bytes(1, 4096, 64, 16)
    assert need > 0
    kw = dict(b=1, L=4096, d_in=64, N=16, y=FAKE + (1 << 22))
    assert scan(**kw) == S.SSM_ERR_WORKSPACE
    assert scan(ws=FAKE + (1 << 23), ws_bytes=need - 4, **kw) == S.SSM_ERR_WORKSPACE
    assert scan(ws=None, ws_bytes=need, **kw) == S.SSM_ERR_WORKSPACE
    assert scan(ws=FAKE + (1 << 23) + 4, ws_bytes=need, **kw) == S.SSM_ERR_INVALID_ARG  # misaligned
    assert scan(ws=FAKE, ws_bytes=need, **kw) == S.SSM_ERR_INVALID_ARG  # overlaps the inputs


def test_h_last_may_equal_h0_but_not_overlap_it():
    # L = 0 returns before any launch when h_last is h0 itself
    H0 = FAKE + 16384
    assert scan(L=0, h0=H0, h_last=H0) == S.SSM_OK
    assert scan(L=0, h0=H0, h_last=H0 + 4) == S.SSM_ERR_INVALID_ARG
    assert scan(L=0, h0=H0, h_last=H0 - 2044) == S.SSM_ERR_INVALID_ARG


def conv_step(**kw):
    a = dict(cs=FAKE + 32768, w=FAKE + 40960, cb=None, K=4, state=FAKE, x=FAKE + 4096,
             dt=FAKE + 5120, A=FAKE + 6144, B=FAKE + 8192, C=FAKE + 9216, D=None, z=None,
             dt_bias=None, sp=1, y=FAKE + 12288, b=2, d_in=16, N=16, dtype=S.SSM_BF16, stream=None)
    a.update(kw)
    return L.ssm_conv_state_update(a["cs"], a["w"], a["cb"], a["K"], a["state"], a["x"], a["dt"],
                                   a["A"], a["B"], a["C"], a["D"], a["z"], a["dt_bias"], a["sp"],
                                   a["y"], a["b"], a["d_in"], a["N"], a["dtype"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(K=0), S.SSM_ERR_UNSUPPORTED),
    (dict(K=9), S.SSM_ERR_UNSUPPORTED),
    (dict(cs=None), S.SSM_ERR_INVALID_ARG),
    (dict(w=None), S.SSM_ERR_INVALID_ARG),
    (dict(cs=FAKE + 4096), S.SSM_ERR_INVALID_ARG),    # conv_state aliases x
    (dict(cs=FAKE + 2000), S.SSM_ERR_INVALID_ARG),    # conv_state overlaps the ssm state
    (dict(w=FAKE + 2), S.SSM_ERR_INVALID_ARG),        # misaligned fp32 weight
    (dict(N=7), S.SSM_ERR_UNSUPPORTED),
    (dict(b=0), S.SSM_OK),
])
def test_conv_step_validation(kw, status):
    assert conv_step(**kw) == status


def test_debug_bounds_library_loads_and_exports_every_function():
    """libssmscan_debug.so (the kernels with every global index checked) has
    the release library's ABI and says which build it is; the release
    library's self-test is rejected before any CUDA call."""
    from selective_state_space_25_b200 import build as libbuild
    path = libbuild.build(debug_bounds=True)
    dbg = ctypes.CDLL(path)
    for n in S.header_functions():
        assert hasattr(dbg, n), f"libssmscan_debug.so does not export {n}"
    dbg.ssm_debug_bounds_enabled.restype = ctypes.c_int
    L.ssm_debug_bounds_enabled.restype = ctypes.c_int
    assert dbg.ssm_debug_bounds_enabled() == 1
    assert L.ssm_debug_bounds_enabled() == 0
    assert L.ssm_debug_bounds_self_test(None) == S.SSM_ERR_UNSUPPORTED
