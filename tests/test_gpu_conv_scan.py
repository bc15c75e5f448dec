"""GPU parity of the one-call prefill layer (conv1d+SiLU, then the chunked
scan: ssd_conv_scan_fwd) against the fp64 oracle run from the raw xBC,
called through the C ABI.  Its y, final state and conv cache must also equal
the two separate calls (conv1d_silu, then chunk_scan_fwd on its output) bit
for bit."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import assert_output, assert_state, cuda, f64, norm_max_abs
from ssd_selective_scan_b200 import layer, synth

pytestmark = pytest.mark.gpu


def _oracle(inp, s):
    return oracle.layer_prefill(
        f64(inp["xBC"]), f64(inp["w"]), None if inp["bias"] is None else f64(inp["bias"]),
        None if inp["conv_state"] is None else f64(inp["conv_state"]), f64(inp["dt_raw"]),
        f64(inp["A"]), f64(inp["dt_bias"]), f64(inp["D"]),
        None if inp["init_state"] is None else f64(inp["init_state"]), s.H, s.P, s.G, s.N)


def _fused(inp, s, **kw):
    cs = cuda(inp["conv_state"])
    y, fs = layer.conv_scan_fwd(cuda(inp["xBC"]), cuda(inp["w"]), cuda(inp["dt_raw"]), cuda(inp["A"]),
                                s.H, s.P, s.G, s.N, bias=cuda(inp["bias"]), conv_state=cs,
                                dt_bias=cuda(inp["dt_bias"]), D=cuda(inp["D"]),
                                init_state=cuda(inp["init_state"]), Q=s.Q, **kw)
    return y, fs, cs


def _two_calls(inp, s):
    cs = cuda(inp["conv_state"])
    u = layer.conv1d_silu(cuda(inp["xBC"]), cuda(inp["w"]), cuda(inp["bias"]), cs)
    x, B, C = layer.split_channels(u, s.H, s.P, s.G, s.N)
    y, fs = layer.chunk_scan_fwd(x, B, C, cuda(inp["dt_raw"]), cuda(inp["A"]), cuda(inp["dt_bias"]),
                                 cuda(inp["D"]), cuda(inp["init_state"]), Q=s.Q)
    return y, fs, cs


def _check_oracle(got, ref, s, what):
    (y, fs, cs), (y_ref, fs_ref, cs_ref) = got, ref
    torch.cuda.synchronize()
    assert_output(y, y_ref, s.dtype, f"{what} y")
    assert_state(fs, fs_ref, s.dtype, f"{what} final state")
    if cs is not None:
        assert np.array_equal(f64(cs), cs_ref), f"{what}: conv cache differs (its columns are copies)"


BF16 = synth.CONFIGS[1]
CASES = {
    # the bench layer's shape, short: cache in and out, conv bias, initial state
    "h40_cache_bias_init": (BF16.with_(b=2, L=520), dict(conv_bias=True, conv_state=True, init_state=True)),
    # ragged last chunk, no cache, no bias
    "h40_ragged_tail": (BF16.with_(b=1, L=300), {}),
    # calls shorter than the conv width: the cache keeps old columns
    "short_L2_cache": (BF16.with_(b=3, L=2, H=8, G=2), dict(conv_state=True, conv_bias=True)),
    "short_L3_cache": (BF16.with_(b=2, L=3, H=8, G=2), dict(conv_state=True)),
    "L129_one_token_chunk": (BF16.with_(b=2, L=129, H=8, G=2), dict(conv_state=True)),
    # more chains than the persistent grid has CTAs: chains cut between CTAs
    "many_chains_handoff": (BF16.with_(b=4, L=520, H=40), dict(conv_state=True, init_state=True)),
    "h128_g8": (BF16.with_(b=2, L=300, H=128), dict(conv_state=True)),
    # one head per group, and two, on the tensor-core scan
    "tc_g_eq_h": (BF16.with_(b=2, L=300, H=8, G=8), dict(conv_state=True, init_state=True)),
    "tc_two_heads_per_group": (BF16.with_(b=2, L=300, H=8, G=4), dict(conv_state=True, conv_bias=True)),
    "g1_long_memory": (BF16.with_(b=1, L=640, H=6, G=1), dict(a_range=(0.01, 2.0), conv_state=True)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_conv_scan_matches_oracle_and_two_calls(name):
    s, kw = CASES[name]
    inp = synth.layer_inputs(s, 42000 + len(name), **kw)
    fused = _fused(inp, s)
    _check_oracle(fused, _oracle(inp, s), s, name)
    two = _two_calls(inp, s)
    torch.cuda.synchronize()
    for a, b, what in zip(fused, two, ("y", "final state", "conv cache")):
        if a is not None:
            assert torch.equal(a, b), f"{name}: fused {what} differs from the two-call path"


@pytest.mark.parametrize("name,s", [
    ("tiny_fp32", synth.CONFIGS[0]),                        # float32, general scan kernel
    ("bf16_k3", BF16.with_(b=2, L=300, H=8, G=2, k=3)),     # conv width 3
    ("bf16_n16", BF16.with_(b=1, L=200, H=4, N=16, G=1)),   # general scan kernel
    ("bf16_q64", BF16.with_(b=1, L=200, H=4, G=2, Q=64)),
])
def test_conv_scan_other_shapes(name, s):
    inp = synth.layer_inputs(s, 43000 + len(name), conv_bias=True, conv_state=True, init_state=True)
    _check_oracle(_fused(inp, s), _oracle(inp, s), s, name)


def test_conv_scan_full_size_matches_oracle():
    """The bench workload (8 x 2048 tokens, 40 heads), element by element."""
    s = synth.CONFIGS[1]
    inp = synth.layer_inputs(s, synth.config_seed(1), conv_state=True)
    fused = _fused(inp, s)
    _check_oracle(fused, _oracle(inp, s), s, s.name)
    two = _two_calls(inp, s)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(fused, two))


def test_conv_scan_chunked_prefill():
    """A prompt prefilled in two fused calls, the conv cache and the state
    handed from the first to the second, equals one call."""
    s = BF16.with_(b=2, L=450, H=8, G=2)
    inp = synth.layer_inputs(s, 4321, conv_state=True, conv_bias=True)
    y1, f1, c1 = _fused(inp, s)
    t = 203   # not a chunk boundary, nor a multiple of the conv width
    a = dict(inp, xBC=inp["xBC"][:, :t].contiguous(), dt_raw=inp["dt_raw"][:, :t].contiguous())
    ya, fa, ca = _fused(a, s.with_(L=t))
    b = dict(inp, xBC=inp["xBC"][:, t:].contiguous(), dt_raw=inp["dt_raw"][:, t:].contiguous(),
             conv_state=ca.cpu(), init_state=fa.cpu())
    yb, fb, cb = _fused(b, s.with_(L=s.L - t))
    torch.cuda.synchronize()
    assert torch.equal(cb, c1)
    assert norm_max_abs(torch.cat([ya, yb], 1), y1) <= 1e-2
    assert norm_max_abs(fb, f1) <= 1e-3
    _check_oracle((torch.cat([ya, yb], 1), fb, cb), _oracle(inp, s), s, "chunked prefill")


def test_conv_scan_empty_call():
    s = BF16.with_(b=2, L=0, H=8, G=2)
    init = torch.randn(2, 8, 64, 128, device="cuda")
    cs = torch.randn(2, s.conv_dim, 4, device="cuda").to(torch.bfloat16)
    cs0 = cs.clone()
    xbc = torch.empty(2, 0, s.conv_dim, dtype=torch.bfloat16, device="cuda")
    dt = torch.empty(2, 0, 8, dtype=torch.bfloat16, device="cuda")
    w = torch.randn(s.conv_dim, 4, device="cuda")
    y, fs = layer.conv_scan_fwd(xbc, w, dt, -torch.ones(8, device="cuda"), s.H, s.P, s.G, s.N,
                                conv_state=cs, init_state=init)
    torch.cuda.synchronize()
    assert y.numel() == 0 and torch.equal(fs, init) and torch.equal(cs, cs0)
