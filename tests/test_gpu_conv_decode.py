"""GPU parity of the conv1d+SiLU and decode state-update entry points against
the fp64 oracle, on identical seeded inputs (called through the C ABI)."""
import math

import numpy as np
import pytest
import torch

import oracle
from parity_util import (TOL_STATE_F32, assert_output, cuda, f64, norm_max_abs)
from ssd_selective_scan_b200 import layer, synth

pytestmark = pytest.mark.gpu


def _conv_case(b, L, cd, k, dtype, bias, state, seed):
    g = torch.Generator().manual_seed(seed)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    xbc = torch.randn(b, L, cd, generator=g).to(td)
    w = torch.randn(cd, k, generator=g) * 0.5
    bs = torch.randn(cd, generator=g) * 0.3 if bias else None
    st = torch.randn(b, cd, k, generator=g).to(td) if state else None
    return xbc, w, bs, st


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("b,L,cd,k,bias,state", [
    (1, 256, 288, 4, False, False),      # the tiny fp32 layer's conv
    (2, 100, 64, 4, True, True),         # ragged token tile, cache in and out
    (3, 1, 40, 4, True, True),           # decode-step roll
    (2, 3, 16, 4, False, True),          # call shorter than the conv width
    (1, 37, 24, 3, True, True),
    (2, 70, 32, 2, True, False),
    # long sequences take 64-token tiles; a ragged last tile, cache in and out
    (2, 65600, 64, 4, True, True),
])
def test_conv1d_silu_matches_oracle(dtype, b, L, cd, k, bias, state):
    xbc, w, bs, st = _conv_case(b, L, cd, k, dtype, bias, state, seed=1000 + L + cd + k)
    u_ref, st_ref = oracle.conv1d_silu(f64(xbc), f64(w), None if bs is None else f64(bs),
                                       None if st is None else f64(st))
    st_dev = cuda(st)
    u = layer.conv1d_silu(cuda(xbc), cuda(w), cuda(bs), st_dev)
    torch.cuda.synchronize()
    assert_output(u, u_ref, dtype, "conv output")
    if state:
        # the new cache holds copies of inputs: bit-exact
        assert np.array_equal(f64(st_dev), st_ref), "conv cache"


def test_conv1d_silu_layer_shape_bf16():
    s = synth.CONFIGS[1].with_(b=2, L=300)
    inp = synth.layer_inputs(s, 7, conv_bias=True, conv_state=True)
    u_ref, st_ref = oracle.conv1d_silu(f64(inp["xBC"]), f64(inp["w"]), f64(inp["bias"]),
                                       f64(inp["conv_state"]))
    st = cuda(inp["conv_state"])
    u = layer.conv1d_silu(cuda(inp["xBC"]), cuda(inp["w"]), cuda(inp["bias"]), st)
    torch.cuda.synchronize()
    assert_output(u, u_ref, "bf16", "conv output")
    assert np.array_equal(f64(st), st_ref)


def _decode_ref(inp, s):
    cd = s.conv_dim
    u_ref, cs_ref = oracle.conv1d_silu(f64(inp["xBC"]).reshape(s.b, 1, cd), f64(inp["w"]), None,
                                       f64(inp["conv_state"]))
    return u_ref.reshape(s.b, cd), cs_ref


@pytest.mark.parametrize("b,H,P,N,G,dtype", [
    (256, 128, 64, 128, 8, "bf16"),     # the decode workload at full size
    (5, 8, 64, 128, 2, "bf16"),
    (3, 4, 64, 16, 1, "f32"),
    (4, 6, 24, 32, 3, "f32"),
    (2, 2, 8, 256, 1, "bf16"),
])
def test_state_update_matches_oracle(b, H, P, N, G, dtype):
    s = synth.LayerShape("decode", b, 1, H, P, N, G, 128, 4, dtype)
    inp = synth.decode_inputs(s, synth.config_seed(4) + b + N)
    u = inp["xBC"]                       # decode update alone: channels used as x | B | C directly
    x, B, C = synth.split_channels(u, s)
    y_ref, st_ref = oracle.state_update(
        f64(inp["state"]), f64(x).reshape(b, H, P), f64(B).reshape(b, G, N),
        f64(C).reshape(b, G, N), f64(inp["dt_raw"]), f64(inp["A"]), f64(inp["dt_bias"]),
        f64(inp["D"]))
    ud = cuda(u)
    xd, Bd, Cd = layer.split_channels(ud, H, P, G, N)
    state = cuda(inp["state"])
    y = layer.state_update(state, xd, Bd, Cd, cuda(inp["dt_raw"]), cuda(inp["A"]),
                           cuda(inp["dt_bias"]), cuda(inp["D"]))
    torch.cuda.synchronize()
    e_state = norm_max_abs(state, st_ref)
    assert e_state <= TOL_STATE_F32, f"decode state error {e_state:.3e}"
    assert_output(y, y_ref, dtype, "decode y")


def test_decode_step_full_layer_matches_oracle():
    """conv-cache roll + conv + SiLU, then the state update, at the decode
    workload's full size."""
    s = synth.CONFIGS[4]
    inp = synth.decode_inputs(s, synth.config_seed(4))
    u_ref, cs_ref = _decode_ref(inp, s)
    H, P, G, N, b = s.H, s.P, s.G, s.N, s.b
    x = u_ref[:, : H * P].reshape(b, H, P)
    B = u_ref[:, H * P: H * P + G * N].reshape(b, G, N)
    C = u_ref[:, H * P + G * N:].reshape(b, G, N)
    y_ref, st_ref = oracle.state_update(f64(inp["state"]), x, B, C, f64(inp["dt_raw"]),
                                        f64(inp["A"]), f64(inp["dt_bias"]), f64(inp["D"]))
    cs = cuda(inp["conv_state"])
    state = cuda(inp["state"])
    y = layer.decode_step(cuda(inp["xBC"]), cuda(inp["w"]), cs, state, cuda(inp["dt_raw"]),
                          cuda(inp["A"]), H, P, G, N, dt_bias=cuda(inp["dt_bias"]),
                          D=cuda(inp["D"]))
    torch.cuda.synchronize()
    assert np.array_equal(f64(cs), cs_ref), "conv cache roll"
    # the GPU state update consumes bf16-rounded conv outputs, the oracle fp64
    # ones, so the state is compared at the bf16 bound here; the exact-input
    # state comparison at 1e-5 is test_state_update_matches_oracle
    assert norm_max_abs(state, st_ref) <= 2e-2
    assert_output(y, y_ref, "bf16", "decode-step y")


@pytest.mark.parametrize("b,H,P,N,G,k,dtype,bias", [
    (256, 128, 64, 128, 8, 4, "bf16", False),   # the decode workload at full size
    (3, 8, 64, 128, 2, 4, "bf16", True),
    (5, 4, 64, 16, 1, 4, "f32", True),
    (4, 6, 24, 32, 3, 3, "f32", False),
    (2, 2, 8, 256, 1, 2, "bf16", True),
    (7, 12, 16, 64, 4, 4, "f32", True),
    (3, 4, 64, 128, 4, 4, "bf16", False),       # one head per group: every CTA is its group's last
])
@pytest.mark.parametrize("form", ["per_group", "per_head_ws"])
def test_decode_step_kernel_matches_oracle_and_two_calls(b, H, P, N, G, k, dtype, bias, form):
    """The one-kernel decode step, in both forms (one CTA per group; one per
    head with the workspace of arrival counters), against the oracle (conv
    from the raw token, then the recurrence step) and, bit for bit, against
    the two calls it fuses (conv1d_silu with L = 1, then state_update).  The
    workspace form must leave its counters at zero."""
    s = synth.LayerShape("decode", b, 1, H, P, N, G, 128, k, dtype)
    inp = synth.decode_inputs(s, 7700 + b + N + k)
    cd = s.conv_dim
    bs = torch.randn(cd, generator=torch.Generator().manual_seed(b + k)) * 0.3 if bias else None
    u_ref, cs_ref = oracle.conv1d_silu(f64(inp["xBC"]).reshape(b, 1, cd), f64(inp["w"]),
                                       None if bs is None else f64(bs), f64(inp["conv_state"]))
    u_ref = u_ref.reshape(b, cd)
    y_ref, st_ref = oracle.state_update(
        f64(inp["state"]), u_ref[:, : H * P].reshape(b, H, P), u_ref[:, H * P: H * P + G * N].reshape(b, G, N),
        u_ref[:, H * P + G * N:].reshape(b, G, N), f64(inp["dt_raw"]), f64(inp["A"]), f64(inp["dt_bias"]),
        f64(inp["D"]))
    args = dict(bias=cuda(bs), dt_bias=cuda(inp["dt_bias"]), D=cuda(inp["D"]))
    cs1, st1 = cuda(inp["conv_state"]), cuda(inp["state"])
    ws = layer.decode_step_workspace(b, G, "cuda") if form == "per_head_ws" else None
    y1 = layer.decode_step(cuda(inp["xBC"]), cuda(inp["w"]), cs1, st1, cuda(inp["dt_raw"]), cuda(inp["A"]),
                           H, P, G, N, workspace=ws, **args)
    # the two calls
    cs2, st2 = cuda(inp["conv_state"]), cuda(inp["state"])
    u = layer.conv1d_silu(cuda(inp["xBC"]).view(b, 1, cd), cuda(inp["w"]), cuda(bs), cs2).view(b, cd)
    xd, Bd, Cd = layer.split_channels(u, H, P, G, N)
    y2 = layer.state_update(st2, xd, Bd, Cd, cuda(inp["dt_raw"]), cuda(inp["A"]), args["dt_bias"], args["D"])
    torch.cuda.synchronize()
    assert np.array_equal(f64(cs1), cs_ref), "conv cache roll"
    assert torch.equal(cs1, cs2) and torch.equal(st1, st2) and torch.equal(y1, y2), "differs from the two calls"
    if ws is not None:
        assert int(ws.abs().sum()) == 0, "arrival counters not left at zero"
    # float32 conv outputs are within 1e-6 of the oracle's, so the state keeps
    # its 1e-5 bound; bf16-rounded ones move the state at the bf16 bound
    tol_state = TOL_STATE_F32 if dtype == "f32" else 2e-2
    e_state = norm_max_abs(st1, st_ref)
    assert e_state <= tol_state, f"decode state error {e_state:.3e}"
    assert_output(y1, y_ref, dtype, "decode-step y")


def test_decode_step_ws_successive_steps_equal_the_two_calls():
    """Three decode steps in a row through the workspace form (the arrival
    counters reset by each call are reused by the next) equal three steps of
    the two calls bit for bit: the group's shared B and C cache columns are
    rolled exactly once per step."""
    b, H, P, N, G, k = 6, 16, 64, 128, 2, 4
    s = synth.LayerShape("decode", b, 1, H, P, N, G, 128, k, "bf16")
    inp = synth.decode_inputs(s, 7811)
    cd = s.conv_dim
    ws = layer.decode_step_workspace(b, G, "cuda")
    cs1, st1 = cuda(inp["conv_state"]), cuda(inp["state"])
    cs2, st2 = cuda(inp["conv_state"]), cuda(inp["state"])
    g = torch.Generator().manual_seed(5)
    for step in range(3):
        xBC = (torch.randn(b, cd, generator=g) * 0.5).to(torch.bfloat16).cuda()
        dt_raw = (torch.rand(b, H, generator=g) * -3 - 1).to(torch.bfloat16).cuda()
        y1 = layer.decode_step(xBC, cuda(inp["w"]), cs1, st1, dt_raw, cuda(inp["A"]), H, P, G, N,
                               dt_bias=cuda(inp["dt_bias"]), D=cuda(inp["D"]), workspace=ws)
        u = layer.conv1d_silu(xBC.view(b, 1, cd), cuda(inp["w"]), None, cs2).view(b, cd)
        xd, Bd, Cd = layer.split_channels(u, H, P, G, N)
        y2 = layer.state_update(st2, xd, Bd, Cd, dt_raw, cuda(inp["A"]), cuda(inp["dt_bias"]), cuda(inp["D"]))
        torch.cuda.synchronize()
        assert torch.equal(cs1, cs2) and torch.equal(st1, st2) and torch.equal(y1, y2), f"step {step}"
    assert int(ws.abs().sum()) == 0

