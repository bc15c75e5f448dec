"""GPU parity of the scan's backward pass (ssd_chunk_scan_bwd) against the
fp64 oracle's gradients (oracle.selective_scan_bwd, pinned by finite
differences and by the chunked matrix form), on identical seeded inputs,
called through the C ABI.

Bounds: gradients are sums over tokens (and heads) with cancellation, held
like the forward's final states (parity_util.assert_state): float32 I/O to
1e-4 normalised max-abs and 1e-3 floored relative error; bf16 I/O (bf16
inputs, dy and gradient outputs) to the forward's bf16 bound, 2e-2
normalised max-abs.  One case runs the bench
layer's shape at 2048 tokens (16 chunks of the forward, 64 of the backward
kernel's 32-token chunks)."""
import pytest
import torch

import oracle
from parity_util import assert_state, cuda, f64
from ssd_selective_scan_b200 import layer, synth

pytestmark = pytest.mark.gpu


def _case(s, seed, init=True, dfinal=True, dt_bias=True):
    inp = synth.scan_inputs(s, seed, init_state=init, dt_bias=dt_bias)
    g = torch.Generator().manual_seed(seed + 1)
    dy = torch.randn(s.b, s.L, s.H, s.P, generator=g).to(s.torch_dtype)
    df = torch.randn(s.b, s.H, s.P, s.N, generator=g) if dfinal else None
    return inp, dy, df


def _run(s, inp, dy, df):
    ud = cuda(inp["u"])
    x, B, C = layer.split_channels(ud, s.H, s.P, s.G, s.N)
    return layer.chunk_scan_bwd(x, B, C, cuda(inp["dt_raw"]), cuda(inp["A"]), cuda(dy), cuda(inp["dt_bias"]),
                                cuda(inp["D"]), cuda(inp["init_state"]), cuda(df))


def _ref(s, inp, dy, df):
    x, B, C = synth.split_channels(inp["u"], s)
    return oracle.selective_scan_bwd(
        f64(x).reshape(s.b, s.L, s.H, s.P), f64(B).reshape(s.b, s.L, s.G, s.N),
        f64(C).reshape(s.b, s.L, s.G, s.N), f64(inp["dt_raw"]), f64(inp["A"]), f64(dy), f64(inp["dt_bias"]),
        f64(inp["D"]), None if inp["init_state"] is None else f64(inp["init_state"]),
        None if df is None else f64(df))


CASES = {
    "f32_small": (synth.CONFIGS[0].with_(b=2, L=70, H=4, P=8, N=32, G=2), {}),
    "f32_tiny_layer_n16": (synth.CONFIGS[0], dict(init=False)),
    "f32_ragged_one_token_chunk": (synth.CONFIGS[0].with_(b=1, L=33, H=2, P=16, N=64, G=1), {}),
    "bf16_layer_heads": (synth.CONFIGS[1].with_(b=2, L=300, H=8, G=2), {}),
    "bf16_no_state_grads": (synth.CONFIGS[1].with_(b=1, L=129, H=4, G=1), dict(init=False, dfinal=False,
                                                                                  dt_bias=False)),
    # the bench layer's heads and groups over a full 2048-token sequence
    "bf16_bench_layer_L2048": (synth.CONFIGS[1].with_(b=1, L=2048), dict(dt_bias=False)),
    "f32_L2048": (synth.CONFIGS[0].with_(b=1, L=2048, H=2, P=16, N=32, G=1), dict(dt_bias=False)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_scan_bwd_matches_oracle(name):
    s, kw = CASES[name]
    inp, dy, df = _case(s, 51000 + len(name), **kw)
    got = _run(s, inp, dy, df)
    ref = _ref(s, inp, dy, df)
    torch.cuda.synchronize()
    for k, r in ref.items():
        assert_state(got[k], r, s.dtype, f"{name}: {k}")


def test_scan_bwd_is_deterministic():
    s = synth.CONFIGS[1].with_(b=2, L=200, H=8, G=2)
    inp, dy, df = _case(s, 52000)
    a = _run(s, inp, dy, df)
    b = _run(s, inp, dy, df)
    torch.cuda.synchronize()
    for k in a:
        assert torch.equal(a[k], b[k]), f"{k} differs between two calls"


def test_scan_bwd_no_tokens():
    s = synth.CONFIGS[1].with_(b=2, L=0, H=8, G=2)
    x = torch.empty(2, 0, 8, 64, dtype=torch.bfloat16, device="cuda")
    Bv = torch.empty(2, 0, 2, 128, dtype=torch.bfloat16, device="cuda")
    dt = torch.empty(2, 0, 8, dtype=torch.bfloat16, device="cuda")
    df = torch.randn(2, 8, 64, 128, device="cuda")
    g = layer.chunk_scan_bwd(x, Bv, Bv, dt, -torch.ones(8, device="cuda"), x, dfinal=df)
    torch.cuda.synchronize()
    assert torch.equal(g["dinit"], df)
    for k in ("dA", "dD", "ddt_bias"):
        assert torch.count_nonzero(g[k]) == 0
