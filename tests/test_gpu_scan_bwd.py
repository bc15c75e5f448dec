"""GPU parity of the scan's backward pass (ssd_chunk_scan_bwd) against the
fp64 oracle's gradients (oracle.selective_scan_bwd, pinned by finite
differences and by the chunked matrix form), on identical seeded inputs,
called through the C ABI.

Bounds: gradients are sums over tokens (and heads) with cancellation, held
like the forward's final states (parity_util.assert_state): float32 I/O to
1e-4 normalised max-abs and 1e-3 floored relative error; bf16 I/O (bf16
inputs, dy and gradient outputs) to the forward's bf16 bound, 2e-2
normalised max-abs.

bf16 I/O with P = 64 and N = 128 runs the tensor-core backward
(scan_bwd_tc.cu: 128-token chunks, bf16 operands, the group's heads summed
in one CTA); other shapes, float32, and calls whose rows are not 16-byte
aligned run the CUDA-core kernel (scan_bwd.cu: 32-token chunks).  Cases
cover both, ragged last chunks, groups of 1 to 5 heads, strong and weak
decay, and the 3B layer (8 x 2048 tokens, 40 heads) element by element."""
import pytest
import torch

import oracle
from parity_util import assert_state, cuda, f64
from ssd_selective_scan_b200 import layer, synth

pytestmark = pytest.mark.gpu


def _case(s, seed, init=True, dfinal=True, dt_bias=True, **kw):
    inp = synth.scan_inputs(s, seed, init_state=init, dt_bias=dt_bias, **kw)
    g = torch.Generator().manual_seed(seed + 1)
    dy = torch.randn(s.b, s.L, s.H, s.P, generator=g).to(s.torch_dtype)
    df = torch.randn(s.b, s.H, s.P, s.N, generator=g) if dfinal else None
    return inp, dy, df


def _run(s, inp, dy, df, pad_rows=0):
    ud = cuda(inp["u"])
    if pad_rows:   # the same values in rows pad_rows elements longer
        wide = torch.zeros(s.b, s.L, ud.shape[2] + pad_rows, dtype=ud.dtype, device=ud.device)
        wide[:, :, :ud.shape[2]] = ud
        ud = wide[:, :, :ud.shape[2]]
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
    # tensor-core path: a group of 5 heads over 6 chunks, the last one ragged
    "bf16_tc_group5_ragged": (synth.CONFIGS[1].with_(b=2, L=700, H=10, G=2), {}),
    # one head per group
    "bf16_tc_heads_equal_groups": (synth.CONFIGS[1].with_(b=1, L=257, H=4, G=4), {}),
    # a single partial chunk per sequence
    "bf16_tc_one_short_chunk": (synth.CONFIGS[1].with_(b=3, L=5, H=2, G=1), {}),
    # long memory (weak decay) and strong decay
    "bf16_tc_weak_decay": (synth.CONFIGS[1].with_(b=1, L=1000, H=4, G=2), dict(a_range=(0.01, 2.0))),
    "bf16_tc_strong_decay": (synth.CONFIGS[1].with_(b=1, L=600, H=4, G=2), dict(a_range=(8.0, 64.0),
                                                                                dt_range=(-1.0, 1.0))),
    # the 8B layer's 16 heads per group (the longest head loop), two groups
    "bf16_tc_group16": (synth.CONFIGS[2].with_(b=1, L=300, H=32, G=2), {}),
    # one group of 16 heads over 47 chunks (the state passing walks a long chain)
    "bf16_tc_long_chain_g1": (synth.CONFIGS[1].with_(b=1, L=6000, H=16, G=1), dict(a_range=(0.01, 2.0))),
    # the general (CUDA-core) path in bf16: a state size the tensor-core path does not take
    "bf16_general_n64": (synth.CONFIGS[1].with_(b=2, L=300, H=4, G=2, N=64), {}),
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


def test_scan_bwd_general_path_unaligned_rows():
    """bf16 at P = 64, N = 128 with token rows one element longer than the
    channels (not 16-byte aligned): the CUDA-core kernel takes the call."""
    s = synth.CONFIGS[1].with_(b=2, L=300, H=8, G=2)
    inp, dy, df = _case(s, 51500)
    got = _run(s, inp, dy, df, pad_rows=1)
    ref = _ref(s, inp, dy, df)
    torch.cuda.synchronize()
    for k, r in ref.items():
        assert_state(got[k], r, s.dtype, f"unaligned rows: {k}")


def test_scan_bwd_full_3b_layer():
    """The FRANKENSTALLM-H 3B layer's full shape (8 x 2048 tokens, 40 heads,
    8 groups), every gradient element by element against the oracle."""
    s = synth.CONFIGS[1]
    inp, dy, df = _case(s, 51700, dt_bias=False)
    got = _run(s, inp, dy, df)
    ref = _ref(s, inp, dy, df)
    torch.cuda.synchronize()
    for k, r in ref.items():
        assert_state(got[k], r, s.dtype, f"3B layer: {k}")


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
